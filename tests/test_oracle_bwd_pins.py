"""Pins of the backward oracle (oracle/lact_oracle_bwd.py).

Its forward, restated in fp64 torch, must equal the numpy oracle; its
gradients (torch.autograd) must equal central finite differences of the
NUMPY oracle's forward, so a mistake in the restatement cannot hide in both.
"""
import numpy as np
import pytest

import oracle
from oracle import lact_oracle_bwd as ob
from oracle import APPLY_THEN_UPDATE, UPDATE_THEN_APPLY, RULE_GD, RULE_MOMENTUM, RULE_MUON

RNG = np.random.default_rng(99)


def _problem(B=1, H=2, T=12, Tq=None, d=4, dh=6, beta=True, w_per_bh=False, lr_scale=3.0):
    Tq = T if Tq is None else Tq
    Hw = B * H if w_per_bh else H
    return dict(
        q=RNG.standard_normal((B, H, Tq, d)), k=RNG.standard_normal((B, H, T, d)),
        v=RNG.standard_normal((B, H, T, d)),
        lr=np.log1p(np.exp(RNG.standard_normal((B, H, T, 3)) - 1.0)) * lr_scale,
        beta=(1 / (1 + np.exp(-(1 + RNG.standard_normal((B, H, T)))))) if beta else None,
        w1=RNG.standard_normal((Hw, dh, d)) / d ** 0.5, w2=RNG.standard_normal((Hw, d, dh)) / dh ** 0.5,
        w3=RNG.standard_normal((Hw, dh, d)) / d ** 0.5)


def _numpy_loss(p, chunk, order, rule, dout, dw, mask=None, scale=None, m_in=None, dm=None):
    out, w1o, w2o, w3o, m1o, m2o, m3o = oracle.ttt_layer_ex(
        p["q"], p["k"], p["v"], p["lr"], p["beta"], p["w1"], p["w2"], p["w3"], chunk, order, rule,
        update_mask=mask, out_scale=scale, m_in=m_in)
    loss = (out * dout).sum() + sum((a * b).sum() for a, b in zip((w1o, w2o, w3o), dw))
    if dm is not None:
        loss = loss + sum((a * b).sum() for a, b in zip((m1o, m2o, m3o), dm))
    return loss


CASES = [
    (APPLY_THEN_UPDATE, RULE_GD, None, False),
    (UPDATE_THEN_APPLY, RULE_GD, None, True),
    (APPLY_THEN_UPDATE, RULE_MOMENTUM, None, False),
    (UPDATE_THEN_APPLY, RULE_MOMENTUM, [1, 0, 1, 1], False),
    (APPLY_THEN_UPDATE, RULE_MOMENTUM, [0, 1, 1, 0], True),
    (APPLY_THEN_UPDATE, RULE_MUON, None, False),
    (UPDATE_THEN_APPLY, RULE_MUON, [1, 1, 0, 1], True),
]


@pytest.mark.parametrize("order,rule,mask,scaled", CASES)
def test_forward_restatement_equals_the_numpy_oracle(order, rule, mask, scaled):
    p = _problem(B=2, T=11)
    scale = RNG.standard_normal((2, 2, 11)) if scaled else None
    dout = RNG.standard_normal(p["q"].shape)
    g = ob.ttt_layer_bwd(**p, chunk=3, order=order, rule=rule, dout=dout, update_mask=mask,
                         out_scale=scale)
    want = oracle.ttt_layer_ex(p["q"], p["k"], p["v"], p["lr"], p["beta"], p["w1"], p["w2"], p["w3"],
                               3, order, rule, update_mask=mask, out_scale=scale)
    np.testing.assert_allclose(g["out"], want[0], rtol=1e-12, atol=1e-13)
    for a, b in zip((g["w1o"], g["w2o"], g["w3o"]), want[1:4]):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("order,rule,mask,scaled", CASES)
def test_gradients_match_central_differences(order, rule, mask, scaled):
    """<grad, delta> against (L(x + e delta) - L(x - e delta)) / 2e for a
    random direction in every input at once and in each input alone."""
    w_per_bh = scaled                          # cover both initial-state layouts
    p = _problem(B=2, T=11, w_per_bh=w_per_bh)
    scale = RNG.standard_normal((2, 2, 11)) if scaled else None
    dout = RNG.standard_normal(p["q"].shape)
    dw = (RNG.standard_normal((4, 6, 4)), RNG.standard_normal((4, 4, 6)), RNG.standard_normal((4, 6, 4)))
    g = ob.ttt_layer_bwd(**p, chunk=3, order=order, rule=rule, dout=dout, dw=dw, update_mask=mask,
                         out_scale=scale)
    names = ["q", "k", "v", "lr", "w1", "w2", "w3"] + (["beta"] if rule == RULE_MOMENTUM else [])
    eps = 1e-6

    def loss_at(delta, t):
        return _numpy_loss(dict(p, **{n: p[n] + t * delta[n] for n in names}), 3, order, rule, dout, dw,
                           mask, scale)

    for only in names + [None]:
        delta = {n: (RNG.standard_normal(p[n].shape) if (only is None or n == only) else 0 * p[n])
                 for n in names}
        if rule == RULE_MUON:
            # five Newton-Schulz quintic steps compose to a polynomial of very
            # high degree: the fourth-order stencil keeps the truncation error
            # below the tolerance (the second-order one misses by ~1e-6)
            fd = (-loss_at(delta, 2 * eps) + 8 * loss_at(delta, eps) - 8 * loss_at(delta, -eps)
                  + loss_at(delta, -2 * eps)) / (12 * eps)
        else:
            fd = (loss_at(delta, eps) - loss_at(delta, -eps)) / (2 * eps)
        an = sum((g["d" + n] * delta[n]).sum() for n in names)
        assert an == pytest.approx(fd, rel=1e-6, abs=1e-8), (only, an, fd)
    if scaled:
        ds = RNG.standard_normal(scale.shape)
        fd = (_numpy_loss(p, 3, order, rule, dout, dw, mask, scale + eps * ds)
              - _numpy_loss(p, 3, order, rule, dout, dw, mask, scale - eps * ds)) / (2 * eps)
        assert (g["dout_scale"] * ds).sum() == pytest.approx(fd, rel=1e-6, abs=1e-8)


def test_without_updates_only_the_apply_has_gradients():
    """All chunks masked: out = f_{W0}(q^), so k, v, lr and beta get zero
    gradients and dW0 is the apply's alone."""
    p = _problem(T=9)
    dout = RNG.standard_normal(p["q"].shape)
    g = ob.ttt_layer_bwd(**p, chunk=3, order=APPLY_THEN_UPDATE, rule=RULE_MOMENTUM, dout=dout,
                         update_mask=[0, 0, 0])
    for n in ("dk", "dv", "dlr", "dbeta"):
        assert np.all(g[n] == 0), n
    assert np.any(g["dq"] != 0) and np.any(g["dw2"] != 0)


def test_muon_with_zero_rates_has_no_path_through_the_update():
    """lr = 0: every chunk gradient is zero, the Frobenius normalisation maps
    it to zero (R7's eps) and no state moves, so out = f_{W0}(q^): the rates
    still get a gradient (the Newton-Schulz map's derivative at zero is
    1 / eps times the identity) while k and v get none through the apply."""
    p = _problem(T=9)
    p["lr"] = np.zeros_like(p["lr"])
    dout = RNG.standard_normal(p["q"].shape)
    g = ob.ttt_layer_bwd(**p, chunk=3, order=APPLY_THEN_UPDATE, rule=RULE_MUON, dout=dout)
    want = oracle.ttt_layer_ex(p["q"], p["k"], p["v"], p["lr"], p["beta"], p["w1"], p["w2"], p["w3"],
                               3, APPLY_THEN_UPDATE, RULE_MUON)
    np.testing.assert_allclose(g["out"], want[0], rtol=1e-12, atol=1e-13)
    for a, b in zip((g["w1o"], g["w2o"], g["w3o"]), (p["w1"], p["w2"], p["w3"])):
        np.testing.assert_allclose(a, np.concatenate([b]), rtol=1e-12, atol=1e-13)
    assert np.all(np.isfinite(g["dlr"])) and np.any(g["dlr"] != 0)


@pytest.mark.parametrize("order,mask", [(APPLY_THEN_UPDATE, None), (UPDATE_THEN_APPLY, [1, 0, 1, 1])])
def test_momentum_in_and_out_gradients_match_central_differences(order, mask):
    """R15: with an initial momentum M_0 handed in and a loss on the final
    momentum, the gradient of M_0 (and every other input) matches central
    differences of the numpy oracle's forward run from M_0."""
    p = _problem(B=2, T=11)
    dout = RNG.standard_normal(p["q"].shape)
    dw = (RNG.standard_normal((4, 6, 4)), RNG.standard_normal((4, 4, 6)), RNG.standard_normal((4, 6, 4)))
    m_in = (RNG.standard_normal((4, 6, 4)), RNG.standard_normal((4, 4, 6)), RNG.standard_normal((4, 6, 4)))
    dm = (RNG.standard_normal((4, 6, 4)), RNG.standard_normal((4, 4, 6)), RNG.standard_normal((4, 6, 4)))
    g = ob.ttt_layer_bwd(**p, chunk=3, order=order, rule=RULE_MOMENTUM, dout=dout, dw=dw, update_mask=mask,
                         m_in=m_in, dm=dm)
    want = oracle.ttt_layer_ex(p["q"], p["k"], p["v"], p["lr"], p["beta"], p["w1"], p["w2"], p["w3"], 3,
                               order, RULE_MOMENTUM, update_mask=mask, m_in=m_in)
    for a, b in zip((g["m1o"], g["m2o"], g["m3o"]), want[4:7]):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    names = ["q", "k", "v", "lr", "beta", "w1", "w2", "w3"]
    eps = 1e-6
    for only in ["m", "beta", None]:
        delta = {n: (RNG.standard_normal(p[n].shape) if only is None or n == only else 0 * p[n])
                 for n in names}
        dmv = tuple(RNG.standard_normal(m.shape) if only in ("m", None) else 0 * m for m in m_in)

        def loss_at(t):
            return _numpy_loss(dict(p, **{n: p[n] + t * delta[n] for n in names}), 3, order, RULE_MOMENTUM,
                               dout, dw, mask, None, tuple(m + t * e for m, e in zip(m_in, dmv)), dm)

        fd = (loss_at(eps) - loss_at(-eps)) / (2 * eps)
        an = sum((g["d" + n] * delta[n]).sum() for n in names)
        an += sum((g[f"dm{j + 1}"] * dmv[j]).sum() for j in range(3))
        assert an == pytest.approx(fd, rel=1e-6, abs=1e-8), (only, an, fd)


def test_momentum_gradient_passes_through_masked_chunks():
    """Every chunk masked: the momentum is handed through untouched, so the
    gradient of M_0 is the gradient given for the final momentum."""
    p = _problem(T=9)
    dout = RNG.standard_normal(p["q"].shape)
    m_in = (RNG.standard_normal((2, 6, 4)), RNG.standard_normal((2, 4, 6)), RNG.standard_normal((2, 6, 4)))
    dm = (RNG.standard_normal((2, 6, 4)), RNG.standard_normal((2, 4, 6)), RNG.standard_normal((2, 6, 4)))
    g = ob.ttt_layer_bwd(**p, chunk=3, order=APPLY_THEN_UPDATE, rule=RULE_MOMENTUM, dout=dout,
                         update_mask=[0, 0, 0], m_in=m_in, dm=dm)
    for j in range(3):
        np.testing.assert_array_equal(g[f"dm{j + 1}"], dm[j])
        np.testing.assert_array_equal(g[f"m{j + 1}o"], m_in[j])
