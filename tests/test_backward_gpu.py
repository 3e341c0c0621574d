"""GPU parity of the layer's backward (lact_ttt_bwd) against the fp64
autograd oracle (oracle/lact_oracle_bwd.py).

Every gradient (q, k, v, lr, beta, the initial weights, the output scale) is
compared by relative L2 over all heads: <= 1e-4 for fp32 workloads, <= 2e-2
for bf16 ones (the backward computes in fp32 in both; the oracle reads the
same bf16-rounded inputs).  Cases span the two orders, GD, momentum and Muon, a
ragged last chunk, masks, the output scale, given final-weight gradients,
shared and per-(b, h) initial weights and a single chunk with separate
queries; the full-size 760M LM shape is checked on sampled heads.
"""
import numpy as np
import pytest
import torch

import chunk_test_b200 as ct
from oracle import lact_oracle_bwd as ob
from lact_inputs import (APPLY_THEN_UPDATE, BF16, F32, RULE_GD, RULE_MOMENTUM, RULE_MUON,
                         UPDATE_THEN_APPLY,
                         WORKLOADS, Workload, make_inputs, make_momentum, make_out_scale,
                         make_output_grads, video_update_mask)

pytestmark = pytest.mark.gpu

TOL = {F32: 1e-4, BF16: 2e-2}
NAMES = ("dq", "dk", "dv", "dlr", "dbeta", "dw1", "dw2", "dw3", "dout_scale", "dm1", "dm2", "dm3")


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def run_both(w, seed, *, per_bh=False, mask=None, scaled=False, with_dw=False, heads=None, m_in=False,
             dm=False, mgrads=False):
    inp = make_inputs(w, seed=seed)
    if per_bh:
        for n in ("w1", "w2", "w3"):
            inp[n] = torch.cat([inp[n] * (1.0 + 0.1 * b) for b in range(w.B)], dim=0).contiguous()
    dout, dws = make_output_grads(w, seed=seed, with_weights=with_dw)
    scale = make_out_scale(w, seed=seed) if scaled else None
    m0 = make_momentum(w, seed=seed) if m_in else None
    dmf = make_momentum(w, seed=seed + 1) if dm else None
    dev = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    got = ct.ttt_bwd(dev["q"], dev["k"], dev["v"], dev["lr"], dev["beta"], dev["w1"], dev["w2"],
                     dev["w3"], w.chunk, w.order, w.rule, dout.cuda(),
                     dw_out=None if dws is None else tuple(x.cuda() for x in dws),
                     update_mask=mask, out_scale=None if scale is None else scale.cuda(),
                     m_in=None if m0 is None else tuple(x.cuda() for x in m0),
                     dm_out=None if dmf is None else tuple(x.cuda() for x in dmf), momentum_grads=mgrads)
    assert ct.status() == ct.LACT_OK
    want = ob.ttt_layer_bwd(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"],
                            inp["w2"], inp["w3"], w.chunk, w.order, w.rule, dout, dw=dws,
                            update_mask=mask, out_scale=scale, heads=heads, m_in=m0, dm=dmf)
    if mgrads and want.get("dm1") is None:   # the gradient of a zero M_0 (the oracle's zeros)
        want = ob.ttt_layer_bwd(inp["q"], inp["k"], inp["v"], inp["lr"], inp["beta"], inp["w1"],
                                inp["w2"], inp["w3"], w.chunk, w.order, w.rule, dout, dw=dws,
                                update_mask=mask, out_scale=scale, heads=heads,
                                m_in=tuple(torch.zeros_like(x) for x in make_momentum(w, seed=seed)))
    return got, want


def check(w, got, want, heads=None):
    errs = {}
    for n in NAMES:
        if want.get(n) is None:
            continue
        g, r = got[n].cpu().numpy(), want[n]
        if heads is not None and n not in ("dw1", "dw2", "dw3"):
            g = np.stack([g[b, h] for b, h in heads])
            r = np.stack([r[b, h] for b, h in heads])
        errs[n] = rel_l2(g, r)
    worst = max(errs.values())
    assert worst <= TOL[w.dtype], f"{w.name}: {errs}"
    return errs


CASES = [
    (Workload("bwd-f32-atu-ragged", 1, 2, 700, 700, 48, 80, 256, APPLY_THEN_UPDATE, RULE_GD, F32), {}),
    (Workload("bwd-f32-uta-mom", 1, 2, 768, 768, 64, 128, 256, UPDATE_THEN_APPLY, RULE_MOMENTUM, F32),
     dict(scaled=True, with_dw=True)),
    (Workload("bwd-f32-atu-mom-mask", 2, 1, 1024, 1024, 32, 64, 128, APPLY_THEN_UPDATE, RULE_MOMENTUM,
              F32), dict(mask=video_update_mask(8, 1), per_bh=True)),
    (Workload("bwd-bf16-d64-atu", 2, 2, 1024, 1024, 64, 128, 256, APPLY_THEN_UPDATE, RULE_GD, BF16), {}),
    (Workload("bwd-bf16-d128-uta-mom", 1, 2, 1024, 1024, 128, 256, 256, UPDATE_THEN_APPLY,
              RULE_MOMENTUM, BF16), dict(per_bh=True, with_dw=True, scaled=True)),
    (Workload("bwd-bf16-d64-set", 1, 2, 1500, 300, 64, 128, 1500, UPDATE_THEN_APPLY, RULE_GD, BF16),
     dict(with_dw=True)),
    (Workload("bwd-bf16-d256-atu-mom-mask", 1, 2, 1536, 1536, 256, 512, 256, APPLY_THEN_UPDATE,
              RULE_MOMENTUM, BF16), dict(mask=video_update_mask(6, 1), scaled=True, with_dw=True)),
    (Workload("bwd-bf16-d384-uta-ragged", 1, 1, 1100, 1100, 384, 768, 512, UPDATE_THEN_APPLY, RULE_GD,
              BF16), dict(mask=[1, 0, 1], per_bh=True)),
    # momentum handed in and out (M_0 in, dL/dM_final in, dL/dM_0 out)
    (Workload("bwd-f32-atu-mom-inout", 1, 2, 768, 768, 64, 128, 256, APPLY_THEN_UPDATE, RULE_MOMENTUM, F32),
     dict(m_in=True, dm=True, with_dw=True, mask=[1, 0, 1])),
    (Workload("bwd-bf16-d128-uta-mom-inout", 1, 2, 1024, 1024, 128, 256, 256, UPDATE_THEN_APPLY,
              RULE_MOMENTUM, BF16), dict(m_in=True, dm=True, per_bh=True)),
    (Workload("bwd-bf16-d256-atu-mom-grads", 1, 2, 1536, 1536, 256, 512, 512, APPLY_THEN_UPDATE,
              RULE_MOMENTUM, BF16), dict(mgrads=True, scaled=True)),
    # Muon: the vector-Jacobian product through five Newton-Schulz steps and
    # the Frobenius normalisation, in fp32 on both launch paths.
    (Workload("bwd-f32-atu-muon", 1, 2, 768, 768, 64, 128, 256, APPLY_THEN_UPDATE, RULE_MUON, F32),
     dict(scaled=True, with_dw=True)),
    (Workload("bwd-f32-uta-muon-mask", 2, 1, 700, 700, 32, 64, 128, UPDATE_THEN_APPLY, RULE_MUON, F32),
     dict(mask=[1, 1, 0, 1, 1, 1], per_bh=True)),
    (Workload("bwd-bf16-d128-atu-muon", 1, 2, 1024, 1024, 128, 256, 256, APPLY_THEN_UPDATE, RULE_MUON,
              BF16), dict(with_dw=True)),
    (Workload("bwd-bf16-d384-atu-muon", 1, 1, 1024, 1024, 384, 768, 512, APPLY_THEN_UPDATE, RULE_MUON,
              BF16), dict(scaled=True)),
]


@pytest.mark.parametrize("w,kw", CASES, ids=lambda x: x.name if hasattr(x, "name") else "")
def test_backward_parity(w, kw):
    got, want = run_both(w, seed=31, **kw)
    errs = check(w, got, want)
    print(w.name, {k: f"{v:.1e}" for k, v in errs.items()})


@pytest.mark.parametrize("idx", [2, 3, 4], ids=["lm760m-gd", "lm3b-momentum", "lm3b-muon"])
def test_backward_at_full_shapes_on_sampled_heads(idx):
    """The full LM workloads (760M: B=2, H=6, d=256, dh=512, chunk 2048, GD;
    3B: B=1, H=8, d=384, dh=768, chunk 4096, momentum and Muon; T=32768),
    two sampled heads against the autograd oracle on the gradients of the
    per-token inputs (dW0 sums over the batch, and over heads that share
    it, so it is left to the cases above)."""
    w = WORKLOADS[idx]
    heads = [(0, 0), (w.B - 1, w.H - 1)]
    got, want = run_both(w, seed=0, heads=heads)
    errs = {}
    for n in ("dq", "dk", "dv", "dlr") + (("dbeta",) if w.rule == RULE_MOMENTUM else ()):
        g = np.stack([got[n][b, h].cpu().numpy() for b, h in heads])
        r = np.stack([want[n][b, h] for b, h in heads])
        errs[n] = rel_l2(g, r)
    assert max(errs.values()) <= TOL[w.dtype], errs
    print(w.name, {k: f"{v:.1e}" for k, v in errs.items()})
