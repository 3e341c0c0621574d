"""GPU parity of the layer's options (lact_ttt_fwd_ex) against the fp64 oracle.

- update mask: only clean chunks update the fast weights, noisy chunks read
  them ("LaCT：以大分块更新人工智能的临时记忆" 「更新顺序必须遵守信息可见范围」,
  "LaCT架构核心思想解析" §3.2);
- per-query output scale ("LaCT架构核心思想解析" §2.1);
- momentum state in and out, so that a sequence split at chunk boundaries
  over several calls equals one call.

Same tolerances as the plain parity tests: relative L2 of `out`, of each
final fast-weight matrix and (momentum) of each final momentum matrix,
<= 1e-4 fp32, <= 2e-2 bf16.  Each case covers a different launch path: the
fused apply on the side stream with two shadow sets, update-then-apply, the
unfused apply of d > 256, the fused key + gradient of d = 64, the fp32 path.
"""
import numpy as np
import pytest
import torch

import chunk_test_b200 as ct
import oracle
from lact_inputs import (APPLY_THEN_UPDATE, BF16, F32, RULE_GD, RULE_MOMENTUM, RULE_MUON,
                         UPDATE_THEN_APPLY, WORKLOADS, Workload, make_inputs, make_out_scale,
                         video_update_mask)

pytestmark = pytest.mark.gpu

TOL = {F32: 1e-4, BF16: 2e-2}


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def _dev(inp):
    return {k: (None if v is None else v.cuda()) for k, v in inp.items()}


def run_gpu(w, inp, **kw):
    d = _dev(inp)
    res = ct.ttt_fwd(d["q"], d["k"], d["v"], d["lr"], d["beta"], d["w1"], d["w2"], d["w3"],
                     w.chunk, w.order, w.rule, **kw)
    assert ct.status() == ct.LACT_OK
    return [r.float().cpu() for r in res]


def run_oracle(w, inp, heads=None, **kw):
    return oracle.ttt_layer_ex(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"],
                               inp["w2"], inp["w3"], w.chunk, w.order, w.rule, heads=heads, **kw)


def check(w, got, want, heads, moms=None):
    """got: out, w1o, w2o, w3o [+ m1, m2, m3 in `moms`]; want: the oracle's
    seven arrays."""
    errs = {}
    for b, h in heads:
        bh = b * w.H + h
        errs[(b, h, "out")] = rel_l2(got[0][b, h].numpy(), want[0][b, h])
        for j, name in enumerate(("w1", "w2", "w3")):
            errs[(b, h, name)] = rel_l2(got[1 + j][bh].numpy(), want[1 + j][bh])
        if moms is not None:
            for j, name in enumerate(("m1", "m2", "m3")):
                errs[(b, h, name)] = rel_l2(moms[j][bh].numpy(), want[4 + j][bh])
    worst = max(errs.values())
    assert worst <= TOL[w.dtype], f"{w.name}: worst rel-L2 {worst:.3e}: {errs}"
    return worst


def heads_of(w):
    return [(b, h) for b in range(w.B) for h in range(w.H)]


MASKED = [
    Workload("bf16-d256-atu-mask", 1, 2, 2048, 2048, 256, 512, 256, APPLY_THEN_UPDATE, RULE_GD, BF16),
    Workload("bf16-d64-atu-mask", 1, 3, 1664, 1664, 64, 128, 256, APPLY_THEN_UPDATE, RULE_GD, BF16),
    Workload("bf16-d128-uta-mom-mask", 2, 2, 1344, 1344, 128, 256, 192, UPDATE_THEN_APPLY,
             RULE_MOMENTUM, BF16),
    Workload("bf16-d384-atu-mom-mask", 1, 1, 2560, 2560, 384, 768, 512, APPLY_THEN_UPDATE,
             RULE_MOMENTUM, BF16),
    Workload("bf16-d128-muon-mask", 1, 2, 1280, 1280, 128, 256, 256, APPLY_THEN_UPDATE, RULE_MUON,
             BF16),
    Workload("f32-atu-mom-mask", 1, 2, 1800, 1800, 48, 80, 256, APPLY_THEN_UPDATE, RULE_MOMENTUM,
             F32),
]


@pytest.mark.parametrize("w", MASKED, ids=lambda w: w.name)
@pytest.mark.parametrize("noisy", [1, 2])
def test_update_mask_parity(w, noisy):
    """Video chunk patterns [noisy x k, clean]: masked chunks are applied but
    do not update; the last chunk is a noisy one in some cases, a ragged one
    in others."""
    inp = make_inputs(w, seed=11)
    mask = video_update_mask(w.n_chunks, noisy)
    got = run_gpu(w, inp, update_mask=mask)
    want = run_oracle(w, inp, update_mask=mask)
    check(w, got, want, heads_of(w))


@pytest.mark.parametrize("w", [MASKED[0], MASKED[2], MASKED[5]], ids=lambda w: w.name)
@pytest.mark.parametrize("pattern", ["none", "first-only", "last-only"])
def test_degenerate_masks(w, pattern):
    """No chunk updates (every output is f_{W0}, the state comes back as it
    went in), only the first chunk updates, only the last one does."""
    inp = make_inputs(w, seed=12)
    n = w.n_chunks
    mask = {"none": [0] * n, "first-only": [1] + [0] * (n - 1),
            "last-only": [0] * (n - 1) + [1]}[pattern]
    got = run_gpu(w, inp, update_mask=mask)
    want = run_oracle(w, inp, update_mask=mask)
    check(w, got, want, heads_of(w))
    if pattern == "none":
        for j, name in enumerate(("w1", "w2", "w3")):
            init = inp[name].repeat(w.B, 1, 1)
            assert torch.equal(got[1 + j], init), name      # the masters pass through bit for bit


SCALED = [
    Workload("bf16-d256-atu-scale", 1, 2, 1536, 1536, 256, 512, 512, APPLY_THEN_UPDATE, RULE_GD, BF16),
    Workload("bf16-d64-uta-set-scale", 1, 3, 1000, 300, 64, 128, 1000, UPDATE_THEN_APPLY, RULE_GD,
             BF16),
    Workload("bf16-d384-atu-scale", 1, 1, 1024, 1024, 384, 768, 512, APPLY_THEN_UPDATE,
             RULE_MOMENTUM, BF16),
    Workload("f32-ragged-scale", 2, 2, 1000, 1000, 48, 80, 384, APPLY_THEN_UPDATE, RULE_GD, F32),
]


@pytest.mark.parametrize("w", SCALED, ids=lambda w: w.name)
def test_out_scale_parity(w):
    """Per-(batch, head, query) output factors, zeros and negatives among
    them, fused into each path's output epilogue."""
    inp = make_inputs(w, seed=13)
    s = make_out_scale(w, seed=13)
    s[0, 0, 5] = 0.0
    s[-1, -1, -1] = -3.0
    got = run_gpu(w, inp, out_scale=s.cuda())
    want = run_oracle(w, inp, out_scale=s)
    check(w, got, want, heads_of(w))
    assert torch.all(got[0][0, 0, 5] == 0)
    plain = run_gpu(w, inp)
    for x, y in zip(got[1:], plain[1:]):
        assert torch.equal(x, y)                          # the state does not see the scale


@pytest.mark.parametrize("w", [
    Workload("bf16-d128-mom-resume", 2, 2, 1536, 1536, 128, 256, 256, APPLY_THEN_UPDATE,
             RULE_MOMENTUM, BF16),
    Workload("bf16-d384-mom-resume", 1, 1, 2048, 2048, 384, 768, 512, APPLY_THEN_UPDATE,
             RULE_MOMENTUM, BF16),
    Workload("f32-mom-resume", 1, 2, 1536, 1536, 64, 128, 256, UPDATE_THEN_APPLY, RULE_MOMENTUM,
             F32),
], ids=lambda w: w.name)
def test_momentum_resume_in_two_calls(w):
    """Two calls over the halves with the first call's weights and momentum
    handed on (m_inout, in place) equal the oracle's single call; the final
    momentum matches the oracle's too.  A mask crosses the split."""
    inp = make_inputs(w, seed=14)
    mask = video_update_mask(w.n_chunks, 1)
    want = run_oracle(w, inp, update_mask=mask)
    half = (w.n_chunks // 2) * w.chunk
    first = {k: (None if v is None else (v[:, :, :half].contiguous() if k in
                 ("q", "k", "v", "lr", "beta") else v)) for k, v in inp.items()}
    second = {k: (None if v is None else (v[:, :, half:].contiguous() if k in
                  ("q", "k", "v", "lr", "beta") else v)) for k, v in inp.items()}
    BH = w.B * w.H
    m = (torch.zeros(BH, w.dh, w.d, device="cuda"), torch.zeros(BH, w.d, w.dh, device="cuda"),
         torch.zeros(BH, w.dh, w.d, device="cuda"))
    nc1 = half // w.chunk
    d1 = _dev(first)
    out1, a1, a2, a3 = ct.ttt_fwd(d1["q"], d1["k"], d1["v"], d1["lr"], d1["beta"], d1["w1"],
                                  d1["w2"], d1["w3"], w.chunk, w.order, w.rule,
                                  update_mask=mask[:nc1], m_inout=m)
    d2 = _dev(second)
    out2, b1, b2, b3 = ct.ttt_fwd(d2["q"], d2["k"], d2["v"], d2["lr"], d2["beta"], a1, a2, a3,
                                  w.chunk, w.order, w.rule, update_mask=mask[nc1:], m_inout=m)
    assert ct.status() == ct.LACT_OK
    got = [torch.cat([out1, out2], dim=2).float().cpu(), b1.cpu(), b2.cpu(), b3.cpu()]
    check(w, got, want, heads_of(w), moms=[x.cpu() for x in m])


def test_all_options_at_the_lm760m_shape():
    """The 760M language-model workload (B=2, H=6, T=32768, d=256, dh=512,
    chunk 2048) with a video-style mask and an output scale, in the launch
    configuration of the plain run; two sampled heads against the oracle."""
    w = WORKLOADS[2]
    inp = make_inputs(w, seed=0)
    mask = video_update_mask(w.n_chunks, 1)
    s = make_out_scale(w, seed=0)
    got = run_gpu(w, inp, update_mask=mask, out_scale=s.cuda())
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    want = run_oracle(w, inp, heads=heads, update_mask=mask, out_scale=s)
    worst = check(w, got, want, heads)
    print(f"{w.name} + mask + scale: worst rel-L2 over sampled heads {worst:.3e}")
