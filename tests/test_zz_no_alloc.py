"""GPU test of lact_ttt_fwd_noalloc, the entry point for callers that cannot
allocate device memory (code that may not call cudaMalloc on its hot path, or
a plugin whose host owns all device memory).  It must give the same results
as lact_ttt_fwd with a caller workspace, on two calls in a row (the built-in
scratch keeps the previous call's contents), and refuse a problem whose
scratch does not fit.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import chunk_test_b200 as ct
from chunk_test_b200 import _abi
from lact_inputs import (APPLY_THEN_UPDATE, BF16, F32, RULE_MOMENTUM, RULE_MUON, WORKLOADS,
                         Workload, make_inputs)

pytestmark = pytest.mark.gpu

TOL = {F32: 1e-4, BF16: 2e-2}
CASES = [
    Workload("noalloc-bf16-muon", 1, 2, 640, 640, 128, 256, 256, APPLY_THEN_UPDATE, RULE_MUON, BF16),
    Workload("noalloc-f32-momentum", 1, 2, 1000, 1000, 64, 128, 384, APPLY_THEN_UPDATE,
             RULE_MOMENTUM, F32),
]


def rel_l2(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_entry_point_on_two_calls(w):
    inp = make_inputs(w, seed=11)
    dev = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    args = (dev["q"], dev["k"], dev["v"], dev["lr"], dev["beta"], dev["w1"], dev["w2"], dev["w3"],
            w.chunk, w.order, w.rule)
    p = ct.make_problem(dev["q"], dev["k"], dev["w1"], w.chunk, w.order, w.rule)
    assert _abi.workspace_bytes(p) <= ct.NOALLOC_SCRATCH_BYTES
    want = ct.ttt_fwd(*args)
    assert ct.status() == ct.LACT_OK
    for _ in range(2):
        out = torch.empty_like(dev["q"])
        w_out = tuple(torch.empty_like(t) for t in want[1:])
        got = ct.ttt_fwd_noalloc(*args, out=out, w_out=w_out)
        assert ct.status() == ct.LACT_OK
        for g, r in zip(got, want):
            assert rel_l2(g, r) <= TOL[w.dtype]


def test_noalloc_rejects_a_problem_that_does_not_fit():
    w = WORKLOADS[2]
    p = _abi.problem(w.B, w.H, w.T, w.Tq, w.d, w.dh, w.chunk, w.order, w.rule, 1, 1)
    assert _abi.workspace_bytes(p) > ct.NOALLOC_SCRATCH_BYTES
    fake = [ctypes.c_void_p((1 << 30) * (i + 1)) for i in range(12)]
    rc = ct.lib().lact_ttt_fwd_noalloc(ctypes.byref(p), *fake, None)
    assert rc == ct.LACT_ETOOBIG
    assert "scratch" in ct.status_string(rc)
