"""GPU parity on the layer's degenerate cases, and on every (batch, head) of
the full-size shapes cut to two chunks.

Each case runs the CUDA path through the C ABI and the fp64 oracle on the same
inputs, compared element by element (relative L2, <= 1e-4 fp32, <= 2e-2 bf16),
plus the exact property the pages fix for the case:
  - an all-zero q or k row: silu(0) = 0, so the normalised row stays zero
    ("LaCT架构核心思想解析" §1.2, the plain q / ||q||; an empty row has no
    direction): a zero query reads exactly zero, a zero key adds nothing;
  - an all-zero fast-weight row: its pre-update norm is zero, so the renorm
    returns it to zero ("大块测试时训练（LaCT）技术解析" §2.2.1 eq. 8);
  - lr = 0: the chunk gradient is zero, so no rule moves the weights (for
    Muon the Frobenius normalisation of a zero gradient gives a zero update);
  - beta = 0: the momentum rule is plain gradient descent.
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


def run_gpu(w: Workload, inp: dict):
    dev = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    res = ct.ttt_fwd(dev["q"], dev["k"], dev["v"], dev["lr"], dev["beta"], dev["w1"], dev["w2"],
                     dev["w3"], w.chunk, w.order, w.rule)
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


# Small shapes on every launch path: the fp32 CUDA-core path, the bf16 fused
# d = 64 key/gradient kernel, the bf16 d = 128 / 256 / 384 paths (side-stream
# apply, CTA-pair gradient, split-bf16 Muon), both orders, ragged chunk tails.
EDGE = [
    Workload("f32-gd", 1, 2, 640, 640, 64, 128, 256, APPLY_THEN_UPDATE, RULE_GD, F32),
    Workload("f32-muon", 1, 2, 640, 640, 64, 128, 256, APPLY_THEN_UPDATE, RULE_MUON, F32),
    Workload("bf16-d64-set", 1, 2, 900, 900, 64, 128, 900, UPDATE_THEN_APPLY, RULE_GD, BF16),
    Workload("bf16-d128-mom", 1, 2, 704, 704, 128, 256, 256, APPLY_THEN_UPDATE, RULE_MOMENTUM, BF16),
    Workload("bf16-d256-gd", 1, 2, 768, 768, 256, 512, 512, APPLY_THEN_UPDATE, RULE_GD, BF16),
    Workload("bf16-d384-muon", 1, 1, 1024, 1024, 384, 768, 512, APPLY_THEN_UPDATE, RULE_MUON, BF16),
]
ZERO_Q_ROWS = (0, 127, 128, 301)
ZERO_K_ROWS = (1, 129, 255, 256, 511)


def _zero_rows(inp, w):
    q, k = inp["q"].clone(), inp["k"].clone()
    for r in ZERO_Q_ROWS:
        if r < w.Tq:
            q[:, :, r, :] = 0
    for r in ZERO_K_ROWS:
        if r < w.T:
            k[:, :, r, :] = 0
    return dict(inp, q=q, k=k)


@pytest.mark.parametrize("w", EDGE, ids=lambda w: w.name)
def test_zero_query_and_key_rows(w):
    """All-zero q and k rows (the prologue's zero-norm branch) inside and at
    the edges of 128-row tiles."""
    inp = _zero_rows(make_inputs(w, seed=11), w)
    got = run_gpu(w, inp)
    check(w, got, run_oracle(w, inp), all_heads(w))
    for r in ZERO_Q_ROWS:
        if r < w.Tq:
            assert torch.count_nonzero(got[0][:, :, r, :]) == 0, f"query row {r} of zeros must read zero"


@pytest.mark.parametrize("w", EDGE, ids=lambda w: w.name)
def test_zero_fast_weight_rows_stay_zero(w):
    """Rows of W1, W3 (length d) and W2 (length dh) that start at zero have a
    zero pre-update norm, so every renorm puts them back to zero."""
    inp = make_inputs(w, seed=12)
    w1, w2, w3 = inp["w1"].clone(), inp["w2"].clone(), inp["w3"].clone()
    w1[:, 3, :] = 0
    w1[:, w.dh - 1, :] = 0
    w3[:, 64, :] = 0
    w2[:, 0, :] = 0
    w2[:, w.d - 1, :] = 0
    inp = dict(inp, w1=w1, w2=w2, w3=w3)
    got = run_gpu(w, inp)
    check(w, got, run_oracle(w, inp), all_heads(w))
    assert torch.count_nonzero(got[1][:, 3, :]) == 0 and torch.count_nonzero(got[1][:, w.dh - 1, :]) == 0
    assert torch.count_nonzero(got[3][:, 64, :]) == 0
    assert torch.count_nonzero(got[2][:, 0, :]) == 0 and torch.count_nonzero(got[2][:, w.d - 1, :]) == 0


@pytest.mark.parametrize("rule", [RULE_GD, RULE_MOMENTUM, RULE_MUON], ids=["gd", "momentum", "muon"])
@pytest.mark.parametrize("dtype", [F32, BF16])
@pytest.mark.parametrize("d,dh", [(64, 128), (256, 512)], ids=["d64", "d256"])
def test_zero_rates_leave_the_state_unchanged(rule, dtype, d, dh):
    """lr = 0: every chunk's gradient is zero and the weights never move, so
    every output is the net of the initial state and w_out = w_in."""
    if dtype == F32 and d == 256:
        pytest.skip("the fp32 path is exercised at d = 64")
    w = Workload("lr0", 1, 2, 768, 768, d, dh, 256, APPLY_THEN_UPDATE, rule, dtype)
    inp = make_inputs(w, seed=13)
    inp = dict(inp, lr=torch.zeros_like(inp["lr"]))
    got = run_gpu(w, inp)
    want = run_oracle(w, inp)
    check(w, got, want, all_heads(w))
    for j, name in enumerate(("w1", "w2", "w3")):
        w_in = inp[name].repeat(w.B, 1, 1) if inp[name].shape[0] == w.H else inp[name]
        assert rel_l2(got[1 + j].numpy(), w_in.numpy()) <= 1e-6, f"{name} moved with zero rates"


@pytest.mark.parametrize("d,dh,dtype", [(64, 128, F32), (64, 128, BF16), (256, 512, BF16)],
                         ids=["f32-d64", "bf16-d64", "bf16-d256"])
def test_momentum_with_zero_beta_is_gradient_descent(d, dh, dtype):
    """beta = 0: M_c = 0 * M_{c-1} + G_c = G_c, so the momentum rule takes the
    plain gradient step of every chunk."""
    w = Workload("beta0", 1, 2, 768, 768, d, dh, 256, APPLY_THEN_UPDATE, RULE_MOMENTUM, dtype)
    inp = make_inputs(w, seed=14)
    inp = dict(inp, beta=torch.zeros_like(inp["beta"]))
    mom = run_gpu(w, inp)
    gd = run_gpu(w.scaled(rule=RULE_GD), dict(inp, beta=None))
    for x, y in zip(mom, gd):
        assert rel_l2(x.numpy(), y.numpy()) <= 1e-6
    check(w, mom, run_oracle(w, inp), all_heads(w))


# The full-size shapes in their benchmark launch configuration, cut to two
# chunks, every (batch, head) checked (the full-length runs check sampled
# heads in test_parity_gpu.py).  The view-synthesis shape is one chunk: it
# runs at full length.
CUT = [(2, 2 * 2048), (3, 2 * 4096), (4, 2 * 4096), (5, None)]


@pytest.mark.parametrize("idx,T", CUT, ids=lambda x: str(x))
def test_full_shapes_every_head(idx, T):
    w = WORKLOADS[idx]
    if T is not None:
        w = w.scaled(name=f"{w.name}@T{T}", T=T, Tq=T)
    inp = make_inputs(w, seed=15)
    got = run_gpu(w, inp)
    want = run_oracle(w, inp)
    worst = check(w, got, want, all_heads(w))
    print(f"{w.name}: worst rel-L2 over all {w.B * w.H} heads {worst:.3e}")
