"""ctypes view of the C ABI in include/lact.h (liblact_b200.so).

Argument marshalling only: every step of the layer runs in the CUDA library.
The library is loaded from this package's directory; if it is missing the
import of any entry point raises -- there is no other implementation.
"""
import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblact_b200.so")

LACT_OK, LACT_EINVAL, LACT_ENOSPC, LACT_ECUDA, LACT_ETIMEOUT, LACT_ENODEV = 0, -1, -2, -3, -4, -5
LACT_ETOOBIG = -6
LACT_ECOMM = -7
REDUCE_SUM, REDUCE_MEAN = 0, 1
# int (*lact_allreduce_fn)(float* data, int64_t count, int op, void* stream, void* user)
ALLREDUCE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                ctypes.c_void_p, ctypes.c_void_p)
NOALLOC_SCRATCH_BYTES = 32 << 20  # LACT_NOALLOC_SCRATCH_BYTES
LACT_F32, LACT_BF16 = 0, 1
APPLY_THEN_UPDATE, UPDATE_THEN_APPLY = 0, 1
RULE_GD, RULE_MOMENTUM, RULE_MUON = 0, 1, 2


class LactProblem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int64), ("H", ctypes.c_int64), ("T", ctypes.c_int64),
        ("Tq", ctypes.c_int64), ("d", ctypes.c_int64), ("dh", ctypes.c_int64),
        ("chunk", ctypes.c_int64), ("order", ctypes.c_int32), ("rule", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("w_shared", ctypes.c_int32),
    ]


class LactFwdOpts(ctypes.Structure):
    """lact_fwd_opts: update_mask is a HOST byte array (one per chunk);
    out_scale, m1, m2, m3 are device pointers (0 = off); allreduce is the
    context-parallel hook (NULL = one rank)."""
    _fields_ = [
        ("update_mask", ctypes.c_void_p), ("out_scale", ctypes.c_void_p),
        ("m1", ctypes.c_void_p), ("m2", ctypes.c_void_p), ("m3", ctypes.c_void_p),
        ("allreduce", ALLREDUCE_FN), ("allreduce_user", ctypes.c_void_p),
    ]


class LactBwdMomentum(ctypes.Structure):
    """lact_bwd_momentum: dL/dM_final in (dm*_out, 0 = zero) and dL/dM_0 out
    (dm*), all device float32 pointers."""
    _fields_ = [("dm1_out", ctypes.c_void_p), ("dm2_out", ctypes.c_void_p), ("dm3_out", ctypes.c_void_p),
                ("dm1", ctypes.c_void_p), ("dm2", ctypes.c_void_p), ("dm3", ctypes.c_void_p)]


class LactSwaProblem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("T", ctypes.c_int64),
                ("d", ctypes.c_int64), ("window", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class LactError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})" if what else status_string(code))


_P = ctypes.POINTER(LactProblem)
_vp = ctypes.c_void_p
# name -> (restype, argtypes); the exported surface of include/lact.h
SIGNATURES = {
    "lact_ttt_workspace_bytes": (ctypes.c_size_t, [_P]),
    "lact_ttt_fwd": (ctypes.c_int, [_P] + [_vp] * 12 + [_vp, ctypes.c_size_t, _vp]),
    "lact_ttt_fwd_ex": (ctypes.c_int, [_P, ctypes.POINTER(LactFwdOpts)] + [_vp] * 12
                        + [_vp, ctypes.c_size_t, _vp]),
    "lact_ttt_fwd_noalloc": (ctypes.c_int, [_P] + [_vp] * 12 + [_vp]),
    "lact_ttt_bwd_workspace_bytes": (ctypes.c_size_t, [_P]),
    "lact_ttt_bwd": (ctypes.c_int, [_P, ctypes.POINTER(LactFwdOpts)] + [_vp] * 21
                     + [_vp, ctypes.c_size_t, _vp]),
    "lact_ttt_bwd_ex": (ctypes.c_int, [_P, ctypes.POINTER(LactFwdOpts), ctypes.POINTER(LactBwdMomentum)]
                        + [_vp] * 21 + [_vp, ctypes.c_size_t, _vp]),
    "lact_ttt_host_workspace_bytes": (ctypes.c_size_t, [_P]),
    "lact_ttt_fwd_host": (ctypes.c_int, [_P] + [_vp] * 12 + [_vp, ctypes.c_size_t, _vp]),
    "lact_swa_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(LactSwaProblem)]),
    "lact_swa_fwd": (ctypes.c_int, [ctypes.POINTER(LactSwaProblem)] + [_vp] * 8 + [_vp, ctypes.c_size_t, _vp]),
    "lact_ttt_status": (ctypes.c_int, [_vp]),
    "lact_device_check": (ctypes.c_int, []),
    "lact_ttt_launch_count": (ctypes.c_int64, [_P]),
    "lact_ttt_launch_count_ex": (ctypes.c_int64, [_P, ctypes.POINTER(LactFwdOpts)]),
    "lact_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_int64, _vp]),
    "lact_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "lact_profile_enable": (ctypes.c_int, [ctypes.c_int]),
    "lact_profile_read": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int64),
                                         ctypes.POINTER(ctypes.c_double), ctypes.c_int]),
    "lact_kernel_kinds": (ctypes.c_int, []),
    "lact_kernel_name": (ctypes.c_char_p, [ctypes.c_int]),
}

_lib = None


def lib():
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m chunk_test_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(code: int) -> str:
    return lib().lact_status_string(int(code)).decode()


def problem(B, H, T, Tq, d, dh, chunk, order, rule, dtype, w_shared) -> LactProblem:
    return LactProblem(int(B), int(H), int(T), int(Tq), int(d), int(dh), int(chunk),
                       int(order), int(rule), int(dtype), int(w_shared))


def workspace_bytes(p: LactProblem) -> int:
    return int(lib().lact_ttt_workspace_bytes(ctypes.byref(p)))


def bwd_workspace_bytes(p: LactProblem) -> int:
    return int(lib().lact_ttt_bwd_workspace_bytes(ctypes.byref(p)))


def host_workspace_bytes(p: LactProblem) -> int:
    return int(lib().lact_ttt_host_workspace_bytes(ctypes.byref(p)))


def launch_count(p: LactProblem) -> int:
    return int(lib().lact_ttt_launch_count(ctypes.byref(p)))


def profile_enable(on: bool) -> None:
    lib().lact_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """{kernel name: (launches, total device ms)} since the last read."""
    n = lib().lact_kernel_kinds()
    launches = (ctypes.c_int64 * n)()
    ms = (ctypes.c_double * n)()
    rc = lib().lact_profile_read(launches, ms, n)
    if rc != LACT_OK:
        raise LactError(rc, "lact_profile_read")
    return {lib().lact_kernel_name(i).decode(): (int(launches[i]), float(ms[i]))
            for i in range(n) if launches[i]}
