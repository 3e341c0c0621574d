"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, and its host logic (argument checks, workspace plan, launch
count) behaves.  No call here touches a GPU."""
import ctypes
import os
import re

import pytest

import chunk_test_b200 as ct
from chunk_test_b200 import _abi
from lact_inputs import WORKLOADS, BF16

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "lact.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lact_\w+)\s*\(", src)))


def test_library_builds_and_loads():
    from chunk_test_b200 import build
    build.build()
    assert os.path.exists(_abi.LIB_PATH)
    assert ct.lib() is not None


def test_every_declared_symbol_is_exported_and_bound():
    names = _declared()
    assert "lact_ttt_fwd" in names and "lact_ttt_workspace_bytes" in names
    handle = ctypes.CDLL(_abi.LIB_PATH)
    for n in names:
        assert hasattr(handle, n), n
    assert set(names) == set(_abi.SIGNATURES), "binding and header disagree"


def _prob(w, **kw):
    args = dict(B=w.B, H=w.H, T=w.T, Tq=w.Tq, d=w.d, dh=w.dh, chunk=w.chunk, order=w.order,
                rule=w.rule, dtype=1 if w.dtype == BF16 else 0, w_shared=1)
    args.update(kw)
    return _abi.problem(**args)


@pytest.mark.parametrize("idx", sorted(WORKLOADS))
def test_workspace_and_launch_count_for_each_workload(idx):
    w = WORKLOADS[idx]
    p = _prob(w)
    ws = _abi.workspace_bytes(p)
    assert ws > 0 and ws % 256 == 0
    assert _abi.host_workspace_bytes(p) > ws
    n = _abi.launch_count(p)
    per_chunk = None
    if w.dtype == BF16:  # fused apply for d <= 256, else forward + output GEMM
        fused_kg = w.rule != 2 and w.d == 64 and w.dh == 128   # key forward + gradient in one
        per_chunk = (20 if w.rule == 2 else 3) + (1 if w.d <= 256 else 2) - (1 if fused_kg else 0)
    if per_chunk is not None:
        fixed = 3 + (1 if w.rule == 1 else 0)
        assert n == fixed + per_chunk * w.n_chunks


@pytest.mark.parametrize("bad", [
    dict(B=0), dict(H=0), dict(T=0), dict(d=0), dict(dh=0), dict(chunk=0), dict(order=2),
    dict(rule=3), dict(dtype=7), dict(w_shared=2), dict(Tq=100),   # Tq != T with many chunks
    dict(d=96), dict(dh=100), dict(d=576, dh=1024),               # bf16 tile limits
])
def test_invalid_problems_are_rejected_by_the_host(bad):
    p = _prob(WORKLOADS[2], **bad)
    assert _abi.workspace_bytes(p) == 0
    assert _abi.launch_count(p) == 0
    nul = ctypes.c_void_p(0)
    rc = ct.lib().lact_ttt_fwd(ctypes.byref(p), *([nul] * 12), nul, ctypes.c_size_t(0), nul)
    assert rc == ct.LACT_EINVAL


def test_null_and_misaligned_pointers_are_rejected_without_a_gpu():
    p = _prob(WORKLOADS[1])
    fake = [ctypes.c_void_p((1 << 30) * (i + 1)) for i in range(12)]
    ws = ctypes.c_void_p(1 << 40)
    lib = ct.lib()
    args = list(fake)
    args[0] = ctypes.c_void_p(0)
    assert lib.lact_ttt_fwd(ctypes.byref(p), *args, ws, ctypes.c_size_t(1 << 40), None) == ct.LACT_EINVAL
    args = list(fake)
    args[2] = ctypes.c_void_p((3 << 30) + 8)                   # v not 16-byte aligned
    assert lib.lact_ttt_fwd(ctypes.byref(p), *args, ws, ctypes.c_size_t(1 << 40), None) == ct.LACT_EINVAL
    # workspace too small
    assert lib.lact_ttt_fwd(ctypes.byref(p), *fake, ws, ctypes.c_size_t(16), None) == ct.LACT_ENOSPC
    # w2_out overlapping w3_out
    args = list(fake)
    args[10] = ctypes.c_void_p(args[11].value)
    assert lib.lact_ttt_fwd(ctypes.byref(p), *args, ws, ctypes.c_size_t(1 << 40), None) == ct.LACT_EINVAL


def test_ragged_and_single_chunk_problems_are_accepted():
    base = WORKLOADS[1]
    assert _abi.workspace_bytes(_prob(base, T=1000, Tq=1000, chunk=384)) > 0
    assert _abi.workspace_bytes(_prob(base, T=1000, Tq=77, chunk=1000)) > 0
    assert _abi.workspace_bytes(_prob(base, T=1000, Tq=77, chunk=4096)) > 0
    assert _abi.workspace_bytes(_prob(base, d=5, dh=7, dtype=0)) > 0      # fp32: any size


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5):
        assert isinstance(ct.status_string(code), str) and ct.status_string(code)


def _opts(mask=None, scale=0, m=(0, 0, 0)):
    buf = None
    if mask is not None:
        buf = (ctypes.c_uint8 * len(mask))(*mask)
    o = _abi.LactFwdOpts(ctypes.addressof(buf) if buf is not None else None, scale or None,
                         *(x or None for x in m))
    return o, buf


@pytest.mark.parametrize("idx", [2, 3])
def test_masked_chunks_launch_no_update_kernels(idx):
    """lact_ttt_launch_count_ex: a chunk whose flag is 0 launches its apply
    only; the fixed launches (state set-up, prologue, beta means, write-back)
    stay."""
    w = WORKLOADS[idx]
    p = _prob(w)
    full = _abi.launch_count(p)
    o, keep = _opts(mask=[1] * w.n_chunks)
    assert ct.lib().lact_ttt_launch_count_ex(ctypes.byref(p), ctypes.byref(o)) == full
    mask = [1 if c % 3 == 0 else 0 for c in range(w.n_chunks)]
    o, keep = _opts(mask=mask)
    apply_per_chunk = 1 if w.d <= 256 else 2
    per_chunk = (full - (3 + (1 if w.rule == 1 else 0))) // w.n_chunks
    want = full - (per_chunk - apply_per_chunk) * mask.count(0)
    assert ct.lib().lact_ttt_launch_count_ex(ctypes.byref(p), ctypes.byref(o)) == want
    assert ct.lib().lact_ttt_launch_count_ex(ctypes.byref(p), None) == full


def test_bad_options_are_rejected_without_a_gpu():
    """Option checks of lact_ttt_fwd_ex run before anything is enqueued."""
    fake = [ctypes.c_void_p((1 << 30) * (i + 1)) for i in range(12)]
    ws = ctypes.c_void_p(1 << 40)
    lib = ct.lib()
    G = 1 << 30
    m_ok = (13 * G, 14 * G, 15 * G)

    def call(p, o):
        return lib.lact_ttt_fwd_ex(ctypes.byref(p), ctypes.byref(o), *fake, ws,
                                   ctypes.c_size_t(1 << 40), None)

    mom = _prob(WORKLOADS[1], rule=1)
    gd = _prob(WORKLOADS[1])
    o, _ = _opts(m=m_ok)
    assert call(gd, o) == ct.LACT_EINVAL                 # momentum buffers with GD
    o, _ = _opts(m=(13 * G, 0, 15 * G))
    assert call(mom, o) == ct.LACT_EINVAL                # only some of them
    o, _ = _opts(m=(13 * G + 8, 14 * G, 15 * G))
    assert call(mom, o) == ct.LACT_EINVAL                # not 16-byte aligned
    o, _ = _opts(m=(13 * G, 13 * G, 15 * G))
    assert call(mom, o) == ct.LACT_EINVAL                # m1 and m2 overlap
    o, _ = _opts(m=(13 * G, 11 * G, 15 * G))
    assert call(mom, o) == ct.LACT_EINVAL                # m2 on w2_out
    o, _ = _opts(m=(6 * G, 14 * G, 15 * G))
    assert call(mom, o) == ct.LACT_EINVAL                # m1 on the initial w1
    o, _ = _opts(scale=16 * G + 2)
    assert call(gd, o) == ct.LACT_EINVAL                 # scale not 4-byte aligned
    o, _ = _opts(scale=9 * G)
    assert call(gd, o) == ct.LACT_EINVAL                 # scale on out
    o, _ = _opts(scale=14 * G, m=m_ok)
    assert call(mom, o) == ct.LACT_EINVAL                # scale on m2


def test_backward_and_attention_arguments_are_checked_without_a_gpu():
    """lact_ttt_bwd and lact_swa_fwd reject bad problems, rules, options and
    pointers before anything is enqueued."""
    lib = ct.lib()
    G = 1 << 30
    ptrs = [ctypes.c_void_p(G * (i + 1)) for i in range(21)]
    ws = ctypes.c_void_p(1 << 40)
    big = ctypes.c_size_t(1 << 40)
    gd = _prob(WORKLOADS[1])
    assert _abi.bwd_workspace_bytes(gd) > 0
    # the Muon backward keeps every chunk's direction and the Newton-Schulz iterates
    assert _abi.bwd_workspace_bytes(_prob(WORKLOADS[1], rule=2)) > _abi.bwd_workspace_bytes(gd)
    call = lambda p, o, a: lib.lact_ttt_bwd(ctypes.byref(p), o, *a, ws, big, None)
    # momentum in/out (lact_ttt_bwd_ex): M_0 in opts, the gradients in a
    # lact_bwd_momentum; every buffer in a slot of its own
    mom = _prob(WORKLOADS[1], rule=1)
    m_in = _abi.LactFwdOpts(None, None, 30 * G, 31 * G, 32 * G)
    mg_ok = _abi.LactBwdMomentum(33 * G, 34 * G, 35 * G, 36 * G, 37 * G, 38 * G)
    call_ex = lambda p, o, mg, a: lib.lact_ttt_bwd_ex(ctypes.byref(p), o, mg, *a, ws, big, None)
    assert call_ex(gd, None, ctypes.byref(mg_ok), ptrs) == ct.LACT_EINVAL        # momentum grads with GD
    assert call(gd, ctypes.byref(m_in), ptrs) == ct.LACT_EINVAL                  # M_0 with GD
    some = _abi.LactFwdOpts(None, None, 30 * G, 0, 32 * G)
    assert call(mom, ctypes.byref(some), ptrs) == ct.LACT_EINVAL                 # only some of M_0
    for bad_mg in (_abi.LactBwdMomentum(33 * G, 34 * G, 35 * G, 36 * G, 0, 38 * G),   # a dM_0 missing
                   _abi.LactBwdMomentum(33 * G, 0, 35 * G, 36 * G, 37 * G, 38 * G),   # only some dM_final
                   _abi.LactBwdMomentum(33 * G, 34 * G, 35 * G, 36 * G + 8, 37 * G, 38 * G),  # misaligned
                   _abi.LactBwdMomentum(33 * G, 34 * G, 35 * G, 13 * G, 37 * G, 38 * G),  # dM_0 on dq
                   _abi.LactBwdMomentum(33 * G, 34 * G, 35 * G, 30 * G, 37 * G, 38 * G),  # dM_0 on M_0
                   _abi.LactBwdMomentum(33 * G, 34 * G, 35 * G, 36 * G, 36 * G, 38 * G)):  # dM_0s overlap
        assert call_ex(mom, ctypes.byref(m_in), ctypes.byref(bad_mg), ptrs) == ct.LACT_EINVAL
    bad = list(ptrs)
    bad[0] = ctypes.c_void_p(0)                                                # q missing
    assert call(gd, None, bad) == ct.LACT_EINVAL
    bad = list(ptrs)
    bad[12] = ctypes.c_void_p(ptrs[0].value)                                   # dq on q
    assert call(gd, None, bad) == ct.LACT_EINVAL
    bad = list(ptrs)
    bad[9] = ctypes.c_void_p(0)                                                # only some dw*_out
    assert call(gd, None, bad) == ct.LACT_EINVAL
    assert lib.lact_ttt_bwd(ctypes.byref(gd), None, *ptrs, ws, ctypes.c_size_t(16), None) == ct.LACT_ENOSPC

    sp = lambda **kw: _abi.LactSwaProblem(*[kw.get(n, v) for n, v in
                                            (("B", 1), ("H", 2), ("T", 1024), ("d", 128), ("window", 256),
                                             ("dtype", 1), ("reserved", 0))])
    assert lib.lact_swa_workspace_bytes(ctypes.byref(sp())) > 0
    for bad_p in (sp(T=1000), sp(window=100), sp(d=96), sp(dtype=0), sp(window=0), sp(d=576)):
        assert lib.lact_swa_workspace_bytes(ctypes.byref(bad_p)) == 0
        assert lib.lact_swa_fwd(ctypes.byref(bad_p), *ptrs[:8], ws, big, None) == ct.LACT_EINVAL
    p = sp()
    bad = list(ptrs[:8])
    bad[7] = ctypes.c_void_p(ptrs[1].value)                                    # out on k
    assert lib.lact_swa_fwd(ctypes.byref(p), *bad, ws, big, None) == ct.LACT_EINVAL
    assert lib.lact_swa_fwd(ctypes.byref(p), *ptrs[:8], ws, ctypes.c_size_t(16), None) == ct.LACT_ENOSPC


def test_attention_workspace_follows_the_documented_layout():
    """lact_swa_workspace_bytes (host arithmetic): for d up to 256 the scores
    stay on chip and the workspace is one bf16 copy of the transformed q;
    for larger d it also holds the fp32 scores, the bf16 probabilities
    (B*H*T*(window+128)*6 bytes) and the zero-padded k' and v copies."""
    lib = ct.lib()
    sp = lambda **kw: _abi.LactSwaProblem(*[kw.get(n, v) for n, v in
                                            (("B", 1), ("H", 2), ("T", 1024), ("d", 128), ("window", 256),
                                             ("dtype", 1), ("reserved", 0))])
    rup = lambda x: (x + 255) // 256 * 256
    for B, H, T, d, w in ((1, 2, 1024, 128, 256), (2, 6, 32768, 256, 2048), (1, 1, 384, 64, 1024)):
        got = lib.lact_swa_workspace_bytes(ctypes.byref(sp(B=B, H=H, T=T, d=d, window=w)))
        assert got == rup(B * H * T * d * 2), (B, H, T, d, w, got)
    B, H, T, d, w = 1, 1, 512, 512, 256
    got = lib.lact_swa_workspace_bytes(ctypes.byref(sp(B=B, H=H, T=T, d=d, window=w)))
    scores = B * H * T * (w + 128) * 6
    padded = 2 * (B * H * (w + T) + w) * d * 2
    assert got >= B * H * T * d * 2 + scores + padded
    assert got <= B * H * T * d * 2 + scores + padded + 4 * 256
