"""torch-facing wrapper of the LaCT TTT layer forward.

torch provides device memory and the stream; the CUDA library does all the
work.  Shapes follow include/lact.h:
  q [B,H,Tq,d], k, v [B,H,T,d] (fp32 or bf16), lr [B,H,T,3] fp32,
  beta [B,H,T] fp32 (momentum only), w1, w3 [Hw,dh,d], w2 [Hw,d,dh] fp32 with
  Hw = H (shared initial state) or B*H.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import LactError

_DT = {torch.float32: _abi.LACT_F32, torch.bfloat16: _abi.LACT_BF16}


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def make_problem(q, k, w1, chunk, order, rule) -> _abi.LactProblem:
    B, H, Tq, d = q.shape
    T = k.shape[2]
    dh = w1.shape[1]
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype}")
    if w1.shape[0] == B * H:
        w_shared = 0
    elif w1.shape[0] == H:
        w_shared = 1
    else:
        raise ValueError("w1/w2/w3 must hold H (shared) or B*H initial states")
    return _abi.problem(B, H, T, Tq, d, dh, chunk, order, rule, _DT[q.dtype], w_shared)


def _check(q, k, v, lr, beta, w1, w2, w3, device_kind):
    for name, t in (("q", q), ("k", k), ("v", v), ("lr", lr), ("w1", w1), ("w2", w2), ("w3", w3),
                    ("beta", beta)):
        if t is None:
            continue
        if t.device.type != device_kind:
            raise ValueError(f"{name} must be on {device_kind}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    for name, t in (("lr", lr), ("beta", beta), ("w1", w1), ("w2", w2), ("w3", w3)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q and k must be [B, H, T, d] tensors")
    B, H, _, d = q.shape
    T = k.shape[2]
    if tuple(k.shape) != (B, H, T, d) or tuple(v.shape) != (B, H, T, d):
        raise ValueError("k and v must be [B, H, T, d] with q's B, H and d")
    if tuple(lr.shape) != (B, H, T, 3):
        raise ValueError("lr must be [B, H, T, 3]")
    if beta is not None and tuple(beta.shape) != (B, H, T):
        raise ValueError("beta must be [B, H, T]")
    if w1.dim() != 3:
        raise ValueError("w1 must be [H or B*H, dh, d]")
    hw, dh = w1.shape[0], w1.shape[1]
    if tuple(w1.shape) != (hw, dh, d) or tuple(w3.shape) != (hw, dh, d) or tuple(w2.shape) != (hw, d, dh):
        raise ValueError("w1, w3 must be [Hw, dh, d] and w2 [Hw, d, dh] with one Hw")


def _check_outputs(q, w1, out, w_out, device_kind):
    """The caller-given outputs: `out` shaped like q in q's dtype, `w_out`
    three float32 tensors [B*H, dh, d], [B*H, d, dh], [B*H, dh, d]; all
    contiguous and on q's device.  The library checks only for null
    pointers, so a wrong size here would let the kernels write past the
    buffer."""
    B, H, _, d = q.shape
    dh = w1.shape[1]
    if (out.device != q.device or out.dtype != q.dtype or tuple(out.shape) != tuple(q.shape)
            or not out.is_contiguous()):
        raise ValueError("out must be a contiguous tensor shaped like q, in q's dtype, on q's device")
    if w_out is None or len(w_out) != 3:
        raise ValueError("w_out must hold three tensors")
    shapes = ((B * H, dh, d), (B * H, d, dh), (B * H, dh, d))
    for i, (t, shp) in enumerate(zip(w_out, shapes)):
        if (t.device.type != device_kind or t.device != q.device or t.dtype != torch.float32
                or tuple(t.shape) != shp or not t.is_contiguous()):
            raise ValueError(f"w_out[{i}] must be a contiguous float32 {list(shp)} tensor on q's device")


def _check_workspace(ws, device, need):
    if ws.device != device or ws.dtype != torch.uint8 or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 tensor on the device of the call")
    if ws.numel() < need:
        raise ValueError(f"workspace holds {ws.numel()} bytes; the call needs {need}")


def workspace_bytes(q, k, w1, chunk, order, rule) -> int:
    return _abi.workspace_bytes(make_problem(q, k, w1, chunk, order, rule))


def launch_count(q, k, w1, chunk, order, rule, update_mask=None) -> int:
    p = make_problem(q, k, w1, chunk, order, rule)
    if update_mask is None:
        return _abi.launch_count(p)
    opts, _keep = _options(p, update_mask, None, None, q)
    return int(_abi.lib().lact_ttt_launch_count_ex(ctypes.byref(p), ctypes.byref(opts)))


class _CudaBuf:
    """A device buffer of fp32 values seen through __cuda_array_interface__,
    so that torch can alias it without a copy."""

    def __init__(self, ptr: int, n: int):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<f4", "data": (ptr, False),
                                         "version": 2, "strides": None}


def _hook(py_fn, device, errors: list):
    """C hook (lact_allreduce_fn) around py_fn(buf, op, stream): buf is a
    float32 tensor aliasing the library's buffer, op the reduction (the
    library asks for REDUCE_SUM only), stream the torch stream of the call.  An exception is kept
    in `errors` and reported to the library as a failure."""

    def c_fn(ptr, count, op, stream_ptr, user):
        try:
            buf = torch.as_tensor(_CudaBuf(int(ptr), int(count)), device=device)
            st = torch.cuda.ExternalStream(int(stream_ptr or 0), device=device)
            py_fn(buf, int(op), st)
            return 0
        except BaseException as e:  # noqa: BLE001 - handed back to the caller
            errors.append(e)
            return 1

    return _abi.ALLREDUCE_FN(c_fn)


def torch_distributed_allreduce(group=None):
    """A context-parallel hook for ttt_fwd(allreduce=...): a sum all-reduce
    over the torch.distributed process group `group` (NCCL for CUDA tensors),
    enqueued on the layer's stream, so that the layer's later kernels see the
    sum.  The library asks only for sums (any mean it needs it forms on the
    device from summed sums and counts)."""
    import torch.distributed as dist

    def fn(buf, op, stream=None):
        if op != _abi.REDUCE_SUM:
            raise ValueError(f"unsupported reduction op {op}")
        ctx = torch.cuda.stream(stream) if (stream is not None and buf.is_cuda) else _nullctx()
        with ctx:
            dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)

    return fn


class _nullctx:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def _options(p, update_mask, out_scale, m_inout, q, allreduce=None, errors=None):
    """lact_fwd_opts for the given options (None when none is given) and the
    objects it points into (the host mask buffer, the C hook), which the
    caller keeps alive for the call."""
    if update_mask is None and out_scale is None and m_inout is None and allreduce is None:
        return None, None
    nch = -(-p.T // min(p.chunk, p.T))
    mask_buf = None
    if update_mask is not None:
        flags = [1 if int(x) else 0 for x in update_mask]
        if len(flags) != nch:
            raise ValueError(f"update_mask needs {nch} flags (one per chunk), got {len(flags)}")
        mask_buf = (ctypes.c_uint8 * nch)(*flags)
    if out_scale is not None:
        B, H, Tq, _ = q.shape
        if (out_scale.device != q.device or out_scale.dtype != torch.float32
                or not out_scale.is_contiguous() or tuple(out_scale.shape) != (B, H, Tq)):
            raise ValueError("out_scale must be a contiguous float32 [B, H, Tq] tensor on q's device")
    ms = (None, None, None)
    if m_inout is not None:
        ms = tuple(m_inout)
        for m in ms:
            if m.device != q.device or m.dtype != torch.float32 or not m.is_contiguous():
                raise ValueError("m_inout must be contiguous float32 tensors on q's device")
    hook = None if allreduce is None else _hook(allreduce, q.device, errors if errors is not None else [])
    o = _abi.LactFwdOpts(ctypes.addressof(mask_buf) if mask_buf is not None else None,
                         None if out_scale is None else out_scale.data_ptr(),
                         *(None if m is None else m.data_ptr() for m in ms))
    if hook is not None:
        o.allreduce = hook
    return o, (mask_buf, hook)


def ttt_fwd(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule, *, out=None, w_out=None,
            workspace=None, stream=None, update_mask=None, out_scale=None, m_inout=None,
            allreduce=None):
    """Runs the layer on the current CUDA device.  Returns (out, w1o, w2o, w3o).
    Optional `out`, `w_out` (a 3-tuple) and `workspace` (uint8 tensor) avoid
    allocations; `stream` defaults to torch's current stream.
    Options (lact_fwd_opts in include/lact.h): `update_mask`, one flag per
    chunk (0 = the chunk is applied but does not update the state);
    `out_scale`, a [B, H, Tq] float32 tensor of per-query output factors;
    `m_inout`, three float32 momentum tensors (shapes of the w_out) read as
    the initial momentum and overwritten with the final one;
    `allreduce`, a context-parallel hook fn(buf, op, stream) that reduces
    `buf` in place over the ranks (see torch_distributed_allreduce); each
    rank then passes its own equal share of every chunk's tokens, with
    `chunk` the local share's length."""
    _check(q, k, v, lr, beta, w1, w2, w3, "cuda")
    p = make_problem(q, k, w1, chunk, order, rule)
    errors = []
    opts, _keep = _options(p, update_mask, out_scale, m_inout, q, allreduce, errors)
    B, H, Tq, d = q.shape
    dh = w1.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if w_out is None:
        w_out = (torch.empty((B * H, dh, d), device=q.device, dtype=torch.float32),
                 torch.empty((B * H, d, dh), device=q.device, dtype=torch.float32),
                 torch.empty((B * H, dh, d), device=q.device, dtype=torch.float32))
    _check_outputs(q, w1, out, w_out, "cuda")
    need = _abi.workspace_bytes(p)
    if need == 0:
        raise LactError(_abi.LACT_EINVAL, "lact_ttt_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    _check_workspace(workspace, q.device, need)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = _abi.lib().lact_ttt_fwd_ex(
        ctypes.byref(p), None if opts is None else ctypes.byref(opts), _ptr(q), _ptr(k), _ptr(v),
        _ptr(lr), _ptr(beta), _ptr(w1), _ptr(w2), _ptr(w3), _ptr(out), _ptr(w_out[0]),
        _ptr(w_out[1]), _ptr(w_out[2]), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
        ctypes.c_void_p(stream.cuda_stream))
    if errors:
        raise errors[0]
    if rc != _abi.LACT_OK:
        raise LactError(rc, "lact_ttt_fwd_ex")
    return out, w_out[0], w_out[1], w_out[2]


def bwd_workspace_bytes(q, k, w1, chunk, order, rule) -> int:
    return _abi.bwd_workspace_bytes(make_problem(q, k, w1, chunk, order, rule))


def _check_momentum(name, ms, q, dh, d):
    B, H = q.shape[0], q.shape[1]
    shapes = ((B * H, dh, d), (B * H, d, dh), (B * H, dh, d))
    if len(ms) != 3:
        raise ValueError(f"{name} must be three tensors (m1, m2, m3)")
    for m, shp in zip(ms, shapes):
        if (m.device != q.device or m.dtype != torch.float32 or not m.is_contiguous()
                or tuple(m.shape) != shp):
            raise ValueError(f"{name} must be contiguous float32 tensors on q's device shaped {shapes}")


def ttt_bwd(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule, dout, *, dw_out=None,
            update_mask=None, out_scale=None, m_in=None, dm_out=None, momentum_grads=False,
            allreduce=None, workspace=None, stream=None):
    """The layer's backward on the current CUDA device (lact_ttt_bwd, or
    lact_ttt_bwd_ex for the momentum gradients): the gradients of a loss
    given dL/d out (`dout`, like q) and optionally dL/d w_out (`dw_out`,
    three tensors like the forward's w_out).  Returns a dict of float32
    tensors: dq, dk, dv, dlr, dbeta (momentum, else None), dw1, dw2, dw3
    (shaped like w1, w2, w3) and dout_scale (when out_scale is given, else
    None).  Momentum rule: `m_in` is the momentum the forward started from
    (the three tensors its m_inout held before the call), `dm_out` the
    gradient of the final momentum it wrote; with either given or
    `momentum_grads` set the dict also holds dm1, dm2, dm3, the gradients
    of m_in.  `allreduce`: the context-parallel hook of ttt_fwd; each rank
    passes its own tokens (and its own dout, dw_out and dm_out, the
    gradients of its share of the loss) and gets the gradients of its own
    tokens and, alike on every rank, of the shared initial state.  On bf16
    inputs some fp32 sums are accumulated with atomic adds, so repeated
    calls can differ in the last bits."""
    _check(q, k, v, lr, beta, w1, w2, w3, "cuda")
    if dout.shape != q.shape or dout.dtype != q.dtype or not dout.is_contiguous():
        raise ValueError("dout must be a contiguous tensor shaped like q, in q's dtype")
    dh, d = w1.shape[1], w1.shape[2]
    if m_in is not None:
        _check_momentum("m_in", m_in, q, dh, d)
    if dm_out is not None:
        _check_momentum("dm_out", dm_out, q, dh, d)
    want_dm = momentum_grads or m_in is not None or dm_out is not None
    p = make_problem(q, k, w1, chunk, order, rule)
    errors = []
    opts, _keep = _options(p, update_mask, out_scale, m_in, q, allreduce, errors)
    f32 = dict(device=q.device, dtype=torch.float32)
    res = {"dq": torch.empty(q.shape, **f32), "dk": torch.empty(k.shape, **f32),
           "dv": torch.empty(v.shape, **f32), "dlr": torch.empty(lr.shape, **f32),
           "dbeta": None if beta is None else torch.empty(beta.shape, **f32),
           "dw1": torch.empty(w1.shape, **f32), "dw2": torch.empty(w2.shape, **f32),
           "dw3": torch.empty(w3.shape, **f32),
           "dout_scale": None if out_scale is None else torch.empty(out_scale.shape, **f32)}
    need = _abi.bwd_workspace_bytes(p)
    if need == 0:
        raise LactError(_abi.LACT_EINVAL, "lact_ttt_bwd_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    dw = (None, None, None) if dw_out is None else tuple(dw_out)
    mg = None
    if want_dm:
        B, H = q.shape[0], q.shape[1]
        res["dm1"] = torch.empty((B * H, dh, d), **f32)
        res["dm2"] = torch.empty((B * H, d, dh), **f32)
        res["dm3"] = torch.empty((B * H, dh, d), **f32)
        dmo = (None, None, None) if dm_out is None else tuple(dm_out)
        mg = _abi.LactBwdMomentum(*(None if x is None else x.data_ptr()
                                    for x in dmo + (res["dm1"], res["dm2"], res["dm3"])))
    rc = _abi.lib().lact_ttt_bwd_ex(
        ctypes.byref(p), None if opts is None else ctypes.byref(opts), None if mg is None else ctypes.byref(mg),
        _ptr(q), _ptr(k), _ptr(v),
        _ptr(lr), _ptr(beta), _ptr(w1), _ptr(w2), _ptr(w3), _ptr(dout), *(_ptr(x) for x in dw),
        _ptr(res["dq"]), _ptr(res["dk"]), _ptr(res["dv"]), _ptr(res["dlr"]), _ptr(res["dbeta"]),
        _ptr(res["dw1"]), _ptr(res["dw2"]), _ptr(res["dw3"]), _ptr(res["dout_scale"]),
        _ptr(workspace), ctypes.c_size_t(workspace.numel()), ctypes.c_void_p(stream.cuda_stream))
    if errors:
        raise errors[0]
    if rc != _abi.LACT_OK:
        raise LactError(rc, "lact_ttt_bwd_ex")
    return res


def swa_problem(q, window) -> _abi.LactSwaProblem:
    B, H, T, d = q.shape
    return _abi.LactSwaProblem(int(B), int(H), int(T), int(d), int(window), _abi.LACT_BF16, 0)


def swa_workspace_bytes(q, window) -> int:
    return int(_abi.lib().lact_swa_workspace_bytes(ctypes.byref(swa_problem(q, window))))


def swa_fwd(q, k, v, q_scale, q_offset, k_scale, k_offset, window, *, out=None, workspace=None,
            stream=None):
    """Sliding-window attention of the LaCT block (lact_swa_fwd): q, k, v
    [B, H, T, d] bf16 CUDA tensors, scales and offsets [H, d] float32.
    Returns out [B, H, T, d] bf16."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.device.type != "cuda" or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    for name, t in (("q_scale", q_scale), ("q_offset", q_offset), ("k_scale", k_scale),
                    ("k_offset", k_offset)):
        if t.device != q.device or not t.is_contiguous() or t.dtype != torch.float32:
            raise ValueError(f"{name} must be a contiguous float32 tensor on q's device")
    p = swa_problem(q, window)
    need = int(_abi.lib().lact_swa_workspace_bytes(ctypes.byref(p)))
    if need == 0:
        raise LactError(_abi.LACT_EINVAL, "lact_swa_workspace_bytes")
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = _abi.lib().lact_swa_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_scale),
                                 _ptr(q_offset), _ptr(k_scale), _ptr(k_offset), _ptr(out),
                                 _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                 ctypes.c_void_p(stream.cuda_stream))
    if rc != _abi.LACT_OK:
        raise LactError(rc, "lact_swa_fwd")
    return out


def ttt_fwd_noalloc(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule, *, out, w_out,
                    stream=None):
    """The forward for callers that cannot allocate device memory: no
    workspace argument, the library's built-in scratch buffer is used (see
    lact_ttt_fwd_noalloc in include/lact.h for its size and sharing rules).
    `out` and `w_out` must be given (pre-allocated by the caller)."""
    _check(q, k, v, lr, beta, w1, w2, w3, "cuda")
    _check_outputs(q, w1, out, w_out, "cuda")
    p = make_problem(q, k, w1, chunk, order, rule)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    rc = _abi.lib().lact_ttt_fwd_noalloc(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lr), _ptr(beta), _ptr(w1), _ptr(w2),
        _ptr(w3), _ptr(out), _ptr(w_out[0]), _ptr(w_out[1]), _ptr(w_out[2]),
        ctypes.c_void_p(stream.cuda_stream))
    if rc != _abi.LACT_OK:
        raise LactError(rc, "lact_ttt_fwd_noalloc")
    return out, w_out[0], w_out[1], w_out[2]


def ttt_fwd_host(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule, *, out, w_out, workspace,
                 stream=None):
    """The same forward from HOST tensors (pinned for full-speed copies): the
    library copies in, runs, copies `out` and `w_out` back and returns when
    they are valid.  `workspace` is a device uint8 tensor of
    host_workspace_bytes() bytes."""
    _check(q, k, v, lr, beta, w1, w2, w3, "cpu")
    _check_outputs(q, w1, out, w_out, "cpu")
    p = make_problem(q, k, w1, chunk, order, rule)
    if workspace.device.type != "cuda":
        raise ValueError("workspace must be a CUDA tensor")
    _check_workspace(workspace, workspace.device, _abi.host_workspace_bytes(p))
    if stream is None:
        stream = torch.cuda.current_stream(workspace.device)
    rc = _abi.lib().lact_ttt_fwd_host(
        ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(lr), _ptr(beta), _ptr(w1), _ptr(w2),
        _ptr(w3), _ptr(out), _ptr(w_out[0]), _ptr(w_out[1]), _ptr(w_out[2]), _ptr(workspace),
        ctypes.c_size_t(workspace.numel()), ctypes.c_void_p(stream.cuda_stream))
    if rc != _abi.LACT_OK:
        raise LactError(rc, "lact_ttt_fwd_host")
    return out, w_out[0], w_out[1], w_out[2]


def host_workspace_bytes(q, k, w1, chunk, order, rule) -> int:
    return _abi.host_workspace_bytes(make_problem(q, k, w1, chunk, order, rule))


def status(stream=None) -> int:
    """Waits for the stream and returns (and clears) the device status word."""
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(_abi.lib().lact_ttt_status(ctypes.c_void_p(stream.cuda_stream)))


def device_check() -> int:
    return int(_abi.lib().lact_device_check())


def selftest_wait_timeout(budget_cycles: int, stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(_abi.lib().lact_selftest_wait_timeout(int(budget_cycles),
                                                    ctypes.c_void_p(stream.cuda_stream)))
