"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerances: relative L2 error of `out` and of each final fast-weight matrix,
<= 1e-4 for fp32 runs and <= 2e-2 for bf16 runs.  Both sides read the same
(bf16-rounded where the workload is bf16) inputs.  Small cases span several
128-row tiles and end in ragged chunk tails; the full-size workloads run in
the launch configuration the benchmark times and are checked on sampled
(batch, head) pairs, each head being an independent problem.
"""
import numpy as np
import pytest
import torch

import chunk_test_b200 as ct
import oracle
from lact_inputs import (APPLY_THEN_UPDATE, BF16, F32, RULE_GD, RULE_MOMENTUM, RULE_MUON,
                         UPDATE_THEN_APPLY, WORKLOADS, Workload, make_inputs)

pytestmark = pytest.mark.gpu

TOL = {F32: 1e-4, BF16: 2e-2}


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def run_gpu(w: Workload, inp: dict, **kw):
    dev = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    res = ct.ttt_fwd(dev["q"], dev["k"], dev["v"], dev["lr"], dev["beta"], dev["w1"], dev["w2"],
                     dev["w3"], w.chunk, w.order, w.rule, **kw)
    assert ct.status() == ct.LACT_OK
    return [r.float().cpu() for r in res]


def run_oracle(w: Workload, inp: dict, heads=None):
    return oracle.ttt_layer(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"],
                            inp["w2"], inp["w3"], w.chunk, w.order, w.rule, heads=heads)


def check(w: Workload, got, want, heads):
    tol = TOL[w.dtype]
    errs = {}
    for b, h in heads:
        bh = b * w.H + h
        errs[(b, h, "out")] = rel_l2(got[0][b, h].numpy(), want[0][b, h])
        for j, name in enumerate(("w1", "w2", "w3")):
            errs[(b, h, name)] = rel_l2(got[1 + j][bh].numpy(), want[1 + j][bh])
    worst = max(errs.values())
    assert worst <= tol, f"{w.name}: worst rel-L2 {worst:.3e} > {tol:.0e}: {errs}"
    return worst


def all_heads(w):
    return [(b, h) for b in range(w.B) for h in range(w.H)]


SMALL = [
    # fp32 path (CUDA cores)
    WORKLOADS[1],
    Workload("f32-ragged-momentum", 1, 2, 1000, 1000, 48, 80, 384, APPLY_THEN_UPDATE, RULE_MOMENTUM, F32),
    Workload("f32-muon", 1, 2, 640, 640, 64, 128, 256, APPLY_THEN_UPDATE, RULE_MUON, F32),
    Workload("f32-set-queries", 1, 2, 900, 130, 64, 128, 900, UPDATE_THEN_APPLY, RULE_GD, F32),
    # bf16 path (tcgen05)
    Workload("bf16-gd-ragged", 1, 2, 640, 640, 64, 128, 256, APPLY_THEN_UPDATE, RULE_GD, BF16),
    Workload("bf16-mom-uta", 2, 2, 704, 704, 128, 256, 192, UPDATE_THEN_APPLY, RULE_MOMENTUM, BF16),
    Workload("bf16-muon", 1, 2, 512, 512, 128, 256, 256, APPLY_THEN_UPDATE, RULE_MUON, BF16),
    Workload("bf16-d256-ragged", 1, 2, 768, 768, 256, 512, 512, APPLY_THEN_UPDATE, RULE_GD, BF16),
    Workload("bf16-d384-momentum", 1, 1, 1024, 1024, 384, 768, 512, APPLY_THEN_UPDATE, RULE_MOMENTUM, BF16),
    Workload("bf16-d384-muon", 1, 1, 1024, 1024, 384, 768, 512, APPLY_THEN_UPDATE, RULE_MUON, BF16),
    Workload("bf16-set-queries", 1, 3, 1000, 300, 64, 128, 1000, UPDATE_THEN_APPLY, RULE_GD, BF16),
    Workload("bf16-set-apply-first", 1, 2, 1000, 300, 64, 128, 4096, APPLY_THEN_UPDATE, RULE_GD, BF16),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_parity(w):
    inp = make_inputs(w, seed=1)
    got = run_gpu(w, inp)
    want = run_oracle(w, inp)
    check(w, got, want, all_heads(w))


def test_per_batch_initial_state_and_in_place_update():
    w = Workload("bf16-per-batch", 2, 2, 512, 512, 64, 128, 256, APPLY_THEN_UPDATE, RULE_GD, BF16)
    inp = make_inputs(w, seed=2)
    for name in ("w1", "w2", "w3"):                     # [H,...] -> [B*H,...], distinct per batch
        base = inp[name]
        inp[name] = torch.cat([base, base.flip(-1)], dim=0).contiguous()
    want = run_oracle(w, inp)
    dev = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    w_in = (dev["w1"].clone(), dev["w2"].clone(), dev["w3"].clone())
    res = ct.ttt_fwd(dev["q"], dev["k"], dev["v"], dev["lr"], None, *w_in, w.chunk, w.order,
                     w.rule, w_out=w_in)                 # exact in-place aliasing
    assert ct.status() == ct.LACT_OK
    got = [r.float().cpu() for r in res]
    check(w, got, want, all_heads(w))


def test_fp32_and_bf16_paths_agree():
    w = Workload("x", 1, 2, 640, 640, 64, 128, 256, APPLY_THEN_UPDATE, RULE_MOMENTUM, BF16)
    inp = make_inputs(w, seed=3)
    a = run_gpu(w, inp)
    inp32 = dict(inp, q=inp["q"].float(), k=inp["k"].float(), v=inp["v"].float())
    b = run_gpu(w.scaled(dtype=F32), inp32)
    for x, y in zip(a, b):
        assert rel_l2(x.numpy(), y.numpy()) <= 2e-2


def test_deterministic_and_host_entry_matches():
    w = Workload("det", 1, 2, 640, 640, 128, 256, 256, APPLY_THEN_UPDATE, RULE_MUON, BF16)
    inp = make_inputs(w, seed=4)
    a = run_gpu(w, inp)
    b = run_gpu(w, inp)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    pin = {k: (None if v is None else v.pin_memory()) for k, v in inp.items()}
    out = torch.empty_like(inp["q"]).pin_memory()
    wo = tuple(torch.empty((w.B * w.H,) + tuple(inp[n].shape[1:]), dtype=torch.float32).pin_memory()
               for n in ("w1", "w2", "w3"))
    ws = torch.empty(ct.host_workspace_bytes(inp["q"], inp["k"], inp["w1"], w.chunk, w.order, w.rule),
                     dtype=torch.uint8, device="cuda")
    h = ct.ttt_fwd_host(pin["q"], pin["k"], pin["v"], pin["lr"], pin["beta"], pin["w1"], pin["w2"],
                        pin["w3"], w.chunk, w.order, w.rule, out=out, w_out=wo, workspace=ws)
    for x, y in zip(a, h):
        assert torch.equal(x, y.float())


def test_device_check_and_bounded_wait_timeout():
    assert ct.device_check() == ct.LACT_OK
    assert ct.status() == ct.LACT_OK
    assert ct.selftest_wait_timeout(200000) == ct.LACT_OK      # the launch itself succeeds
    assert ct.status() == ct.LACT_ETIMEOUT                     # the wait gave up and said so
    assert ct.status() == ct.LACT_OK                           # cleared
    w = SMALL[4]
    inp = make_inputs(w, seed=5)
    got = run_gpu(w, inp)                                      # context still usable
    check(w, got, run_oracle(w, inp), all_heads(w))


FULL = [2, 3, 4, 5]


@pytest.mark.parametrize("idx", FULL)
def test_full_size_sampled_heads(idx):
    w = WORKLOADS[idx]
    inp = make_inputs(w, seed=0)
    got = run_gpu(w, inp)
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    want = run_oracle(w, inp, heads=heads)
    worst = check(w, got, want, heads)
    print(f"{w.name}: worst rel-L2 over sampled heads {worst:.3e}")
