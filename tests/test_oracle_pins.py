"""Pins of the CPU fp64 oracle to things other than itself.

Each test checks the oracle against what the pages and the mathematics fix:
closed forms, library routines (torch autograd / nn.Linear / normalize,
numpy SVD), finite differences, invariants the pages state (apply-then-update
never lets a chunk see its own update; the renorm keeps row norms), a
per-token brute force, and the worked Newton-Schulz values stored under
tests/golden/.  Pages are cited by title and section as in oracle/__init__.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import (APPLY_THEN_UPDATE, UPDATE_THEN_APPLY, RULE_GD, RULE_MOMENTUM,
                    RULE_MUON)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def _rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def _weights(d, dh, H=None):
    lead = () if H is None else (H,)
    return (_rand(*lead, dh, d, scale=d ** -0.5), _rand(*lead, d, dh, scale=dh ** -0.5),
            _rand(*lead, dh, d, scale=d ** -0.5))


def _torch_swiglu(W1, W2, W3, X):
    """f_W built from library modules: nn.Linear stores weights as [out, in]
    and computes x W^T; F.silu is the library silu."""
    l1 = torch.nn.Linear(W1.shape[1], W1.shape[0], bias=False).double()
    l2 = torch.nn.Linear(W2.shape[1], W2.shape[0], bias=False).double()
    l3 = torch.nn.Linear(W3.shape[1], W3.shape[0], bias=False).double()
    with torch.no_grad():
        l1.weight.copy_(torch.as_tensor(W1))
        l2.weight.copy_(torch.as_tensor(W2))
        l3.weight.copy_(torch.as_tensor(W3))
        X = torch.as_tensor(X)
        return l2(torch.nn.functional.silu(l1(X)) * l3(X)).numpy()


def _layer(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule):
    return oracle.ttt_layer(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule)


def _problem(B=1, H=2, T=24, d=8, dh=12, Tq=None, beta=False, lr_scale=1.0):
    Tq = T if Tq is None else Tq
    q = _rand(B, H, Tq, d)
    k = _rand(B, H, T, d)
    v = _rand(B, H, T, d)
    lr = np.log1p(np.exp(_rand(B, H, T, 3) - 2.0)) * lr_scale
    bt = 1.0 / (1.0 + np.exp(-(2.0 + 0.5 * _rand(B, H, T)))) if beta else None
    w1, w2, w3 = _weights(d, dh, H)
    return q, k, v, lr, bt, w1, w2, w3


# ---------------------------------------------------------------- prologue
def test_prologue_closed_forms():
    """silu then L2 norm over the head dim ("LaCT架构核心思想解析" §1.2)."""
    d = 7
    x = np.zeros((5, d))
    x[0, 0] = 2.5                      # silu(0) = 0 elsewhere -> +e0
    x[1, 3] = -1.5                     # silu(-1.5) < 0 -> -e3
    x[2, :] = 0.7                      # constant row -> 1/sqrt(d) everywhere
    x[3, :] = -0.4                     # constant negative row -> -1/sqrt(d)
    y = oracle.qk_prologue(x)
    e = np.zeros(d); e[0] = 1.0
    np.testing.assert_allclose(y[0], e, atol=1e-15)
    e = np.zeros(d); e[3] = -1.0
    np.testing.assert_allclose(y[1], e, atol=1e-15)
    np.testing.assert_allclose(y[2], np.full(d, d ** -0.5), rtol=1e-14)
    np.testing.assert_allclose(y[3], np.full(d, -d ** -0.5), rtol=1e-14)
    np.testing.assert_array_equal(y[4], np.zeros(d))     # all-zero row stays 0


def test_prologue_matches_library_silu_direction():
    x = _rand(50, 16, scale=2.0)
    y = oracle.qk_prologue(x)
    s = torch.nn.functional.silu(torch.as_tensor(x)).numpy()
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(y * np.linalg.norm(s, axis=1, keepdims=True), s,
                               rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- fast net
def test_fast_net_is_a_swiglu_mlp():
    """SwiGLU memory of three matrices ("LaCT：以大分块更新…" 「局部注意力与
    非线性记忆相互补充」), checked against torch nn.Linear modules."""
    d, dh = 6, 10
    W1, W2, W3 = _weights(d, dh)
    X = _rand(9, d)
    np.testing.assert_allclose(oracle.fast_net(W1, W2, W3, X),
                               _torch_swiglu(W1, W2, W3, X), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- gradient
def _loss_j(W1, W2, W3, K, V, lr, j):
    """-sum_i lr[i, j] <f_W(k_i), v_i> with f_W from the oracle."""
    return -np.sum(lr[:, j] * np.sum(oracle.fast_net(W1, W2, W3, K) * V, axis=1))


def test_chunk_gradient_matches_autograd():
    """The chunk-summed, lr-weighted gradient of the negative inner-product
    loss equals torch.autograd's gradient of the same loss."""
    d, dh, n = 5, 9, 11
    W = [torch.tensor(w, requires_grad=True) for w in _weights(d, dh)]
    K = torch.as_tensor(oracle.qk_prologue(_rand(n, d)))
    V = torch.as_tensor(_rand(n, d))
    lr = torch.as_tensor(np.abs(_rand(n, 3)))
    G = oracle.chunk_gradient(*[w.detach().numpy() for w in W], K.numpy(), V.numpy(),
                              lr.numpy())
    f = torch.nn.functional
    for j, wj in enumerate(W):       # lr column j drives matrix j (W1, W2, W3)
        out = f.linear(f.silu(f.linear(K, W[0])) * f.linear(K, W[2]), W[1])
        loss = -(lr[:, j] * (out * V).sum(dim=1)).sum()
        (g,) = torch.autograd.grad(loss, wj)
        np.testing.assert_allclose(G[j], g.numpy(), rtol=1e-11, atol=1e-13)


def test_chunk_gradient_finite_differences():
    d, dh, n = 4, 6, 5
    W = list(_weights(d, dh))
    K = oracle.qk_prologue(_rand(n, d))
    V = _rand(n, d)
    lr = np.abs(_rand(n, 3))
    G = oracle.chunk_gradient(*W, K, V, lr)
    h = 1e-6
    for j in range(3):
        fd = np.zeros_like(W[j])
        for idx in np.ndindex(W[j].shape):
            Wp = [w.copy() for w in W]; Wm = [w.copy() for w in W]
            Wp[j][idx] += h; Wm[j][idx] -= h
            fd[idx] = (_loss_j(*Wp, K, V, lr, j) - _loss_j(*Wm, K, V, lr, j)) / (2 * h)
        np.testing.assert_allclose(G[j], fd, rtol=1e-6, atol=1e-9)


def test_gd_step_lowers_the_chunk_loss():
    """Sign pin: with a small rate the GD update (then renorm) lowers every
    L_j, i.e. moves f_W(k) toward v."""
    d, dh, n = 8, 16, 32
    W = _weights(d, dh)
    K = oracle.qk_prologue(_rand(n, d))
    V = _rand(n, d)
    lr = np.full((n, 3), 1e-3)
    G = oracle.chunk_gradient(*W, K, V, lr)
    W_new = tuple(oracle.renorm_rows(w - g, w) for w, g in zip(W, G))
    for j in range(3):
        Wj = list(W); Wj[j] = W_new[j]
        assert _loss_j(*Wj, K, V, lr, j) < _loss_j(*W, K, V, lr, j)


# ---------------------------------------------------------------- Muon
def _golden_ns():
    with open(os.path.join(GOLDEN, "ns5_worked_values.json")) as f:
        return json.load(f)


def test_ns_worked_values():
    g = _golden_ns()
    assert tuple(g["coeffs"]) == oracle.NS_COEFFS and g["steps"] == oracle.NS_STEPS
    X = oracle.newton_schulz5(np.diag([3.0, 4.0]))
    np.testing.assert_allclose(np.diag(X), [g["phi5"]["0.6"], g["phi5"]["0.8"]], rtol=1e-6)
    np.testing.assert_allclose(X - np.diag(np.diag(X)), 0.0, atol=1e-15)
    u, w = _rand(7), _rand(4)
    X = oracle.newton_schulz5(np.outer(u, w))
    np.testing.assert_allclose(X, g["phi5"]["1.0"] * np.outer(u / np.linalg.norm(u),
                                                              w / np.linalg.norm(w)),
                               rtol=1e-6, atol=1e-12)


@pytest.mark.parametrize("shape", [(6, 4), (4, 6), (5, 5), (12, 7)])
def test_ns_acts_on_singular_values(shape):
    """NS5(G) = U diag(phi5(s / ||G||_F)) V^T against numpy's SVD."""
    a, b, c = oracle.NS_COEFFS
    G = _rand(*shape)
    U, s, Vt = np.linalg.svd(G, full_matrices=False)
    x = s / (np.linalg.norm(G) + oracle.NS_EPS)
    for _ in range(oracle.NS_STEPS):
        x = a * x + b * x ** 3 + c * x ** 5
    np.testing.assert_allclose(oracle.newton_schulz5(G), (U * x) @ Vt, rtol=1e-9, atol=1e-12)


def test_ns_of_zero_is_zero():
    np.testing.assert_array_equal(oracle.newton_schulz5(np.zeros((3, 5))), 0.0)


# ---------------------------------------------------------------- renorm
def test_renorm_keeps_row_norms_and_direction():
    W = _rand(9, 5)
    Wn = W - _rand(9, 5)
    R = oracle.renorm_rows(Wn, W)
    np.testing.assert_allclose(np.linalg.norm(R, axis=1), np.linalg.norm(W, axis=1),
                               rtol=1e-13)
    ref = torch.nn.functional.normalize(torch.as_tensor(Wn), dim=1).numpy() \
        * np.linalg.norm(W, axis=1, keepdims=True)
    np.testing.assert_allclose(R, ref, rtol=1e-13)


def test_renorm_scalar_case_only_flips_sign():
    """With 1x1 matrices the renorm leaves |w| fixed: w <- |w| sign(w - u)."""
    for w, u in [(0.5, 0.2), (0.5, 0.9), (-0.3, -1.0), (-0.3, 0.4)]:
        r = oracle.renorm_rows(np.array([[w - u]]), np.array([[w]]))
        assert r[0, 0] == pytest.approx(abs(w) * np.sign(w - u), rel=1e-15)


def test_renorm_row_norm_equals_init_after_many_chunks():
    q, k, v, lr, beta, w1, w2, w3 = _problem(T=40, lr_scale=30.0)
    _, o1, o2, o3 = _layer(q, k, v, lr, beta, w1, w2, w3, 8, APPLY_THEN_UPDATE, RULE_GD)
    for wo, wi in ((o1, w1), (o2, w2), (o3, w3)):
        np.testing.assert_allclose(np.linalg.norm(wo, axis=2), np.linalg.norm(wi, axis=2),
                                   rtol=1e-12)


# ---------------------------------------------------------------- rules
@pytest.mark.parametrize("rule", [RULE_GD, RULE_MOMENTUM, RULE_MUON])
def test_zero_rate_leaves_weights_unchanged(rule):
    q, k, v, lr, beta, w1, w2, w3 = _problem(beta=True)
    lr[:] = 0.0
    out, o1, o2, o3 = _layer(q, k, v, lr, beta, w1, w2, w3, 8, APPLY_THEN_UPDATE, rule)
    np.testing.assert_allclose(o1, w1, rtol=1e-15)
    np.testing.assert_allclose(o2, w2, rtol=1e-15)
    np.testing.assert_allclose(o3, w3, rtol=1e-15)


def test_momentum_with_zero_beta_is_gd():
    q, k, v, lr, beta, w1, w2, w3 = _problem(beta=True, lr_scale=10.0)
    gd = _layer(q, k, v, lr, None, w1, w2, w3, 6, APPLY_THEN_UPDATE, RULE_GD)
    mo = _layer(q, k, v, lr, np.zeros_like(beta), w1, w2, w3, 6, APPLY_THEN_UPDATE,
                RULE_MOMENTUM)
    for a, b in zip(gd, mo):
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)


def test_momentum_accumulates_with_mean_beta():
    """Two chunks: M1 = G1, M2 = mean(beta_chunk2) M1 + G2 ("LaCT架构核心思想
    解析" §1.2), built here from the oracle's gradient on the right states."""
    d, dh, n = 6, 8, 5
    W = _weights(d, dh)
    k, v = _rand(2 * n, d), _rand(2 * n, d)
    lr = np.abs(_rand(2 * n, 3)) * 0.3
    beta = RNG.uniform(0.2, 0.9, 2 * n)
    kh = oracle.qk_prologue(k)
    G1 = oracle.chunk_gradient(*W, kh[:n], v[:n], lr[:n])
    W1s = tuple(oracle.renorm_rows(w - g, w) for w, g in zip(W, G1))
    G2 = oracle.chunk_gradient(*W1s, kh[n:], v[n:], lr[n:])
    M2 = tuple(beta[n:].mean() * g1 + g2 for g1, g2 in zip(G1, G2))
    W2s = tuple(oracle.renorm_rows(w - m, w) for w, m in zip(W1s, M2))
    q = _rand(2 * n, d)
    _, o1, o2, o3 = oracle.ttt_layer(q[None, None], k[None, None], v[None, None],
                                     lr[None, None], beta[None, None], W[0][None],
                                     W[1][None], W[2][None], n, APPLY_THEN_UPDATE,
                                     RULE_MOMENTUM)
    for got, want in zip((o1[0], o2[0], o3[0]), W2s):
        np.testing.assert_allclose(got, want, rtol=1e-12)


# ---------------------------------------------------------------- orders
def test_apply_then_update_single_chunk_reads_only_the_initial_weights():
    """Apply-then-update with chunk = T returns f_{W0}(q^) whatever k, v, lr
    are ("LaCT架构核心思想解析" §2.2: apply before update, no future leakage)."""
    q, k, v, lr, beta, w1, w2, w3 = _problem(T=20)
    out, *_ = _layer(q, k, v, lr, beta, w1, w2, w3, 20, APPLY_THEN_UPDATE, RULE_GD)
    for h in range(2):
        np.testing.assert_allclose(out[0, h], _torch_swiglu(w1[h], w2[h], w3[h],
                                                            oracle.qk_prologue(q[0, h])),
                                   rtol=1e-12, atol=1e-14)
    out2, *_ = _layer(q, _rand(*k.shape), _rand(*v.shape), lr * 5, beta, w1, w2, w3, 20,
                      APPLY_THEN_UPDATE, RULE_GD)
    np.testing.assert_array_equal(out, out2)


@pytest.mark.parametrize("rule", [RULE_GD, RULE_MOMENTUM, RULE_MUON])
def test_orders_make_the_same_updates(rule):
    """The update never reads q, so both orders end in the same weights."""
    q, k, v, lr, beta, w1, w2, w3 = _problem(beta=True, T=30)
    a = _layer(q, k, v, lr, beta, w1, w2, w3, 7, APPLY_THEN_UPDATE, rule)
    b = _layer(q, k, v, lr, beta, w1, w2, w3, 7, UPDATE_THEN_APPLY, rule)
    for x, y in zip(a[1:], b[1:]):
        np.testing.assert_array_equal(x, y)


def test_update_then_apply_reads_the_weights_after_its_chunk():
    """Order 1, chunk c: out_c = f_{W_c}(q^_c), with W_c the state after the
    first c+1 chunks, taken from a shorter run and checked through library
    modules; order 0 reads W_{c-1} instead."""
    q, k, v, lr, beta, w1, w2, w3 = _problem(T=24, H=1)
    ch = 8
    out1, *_ = _layer(q, k, v, lr, beta, w1, w2, w3, ch, UPDATE_THEN_APPLY, RULE_GD)
    out0, *_ = _layer(q, k, v, lr, beta, w1, w2, w3, ch, APPLY_THEN_UPDATE, RULE_GD)
    for c in range(3):
        rows = slice(c * ch, (c + 1) * ch)
        t = (c + 1) * ch
        _, a1, a2, a3 = _layer(q[:, :, :t], k[:, :, :t], v[:, :, :t], lr[:, :, :t], None,
                               w1, w2, w3, ch, APPLY_THEN_UPDATE, RULE_GD)
        want = _torch_swiglu(a1[0], a2[0], a3[0], oracle.qk_prologue(q[0, 0, rows]))
        np.testing.assert_allclose(out1[0, 0, rows], want, rtol=1e-11, atol=1e-13)
        if c + 1 < 3:
            np.testing.assert_allclose(out0[0, 0, (c + 1) * ch:(c + 2) * ch],
                                       _torch_swiglu(a1[0], a2[0], a3[0],
                                                     oracle.qk_prologue(
                                                         q[0, 0, (c + 1) * ch:(c + 2) * ch])),
                                       rtol=1e-11, atol=1e-13)


def test_single_chunk_separate_queries():
    """A posed image set: one chunk of keys, then separate target queries
    (update-then-apply, Tq != T)."""
    q, k, v, lr, beta, w1, w2, w3 = _problem(T=30, Tq=7, H=1)
    out, a1, a2, a3 = _layer(q, k, v, lr, beta, w1, w2, w3, 30, UPDATE_THEN_APPLY, RULE_GD)
    np.testing.assert_allclose(out[0, 0], _torch_swiglu(a1[0], a2[0], a3[0],
                                                        oracle.qk_prologue(q[0, 0])),
                               rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("rule", [RULE_GD, RULE_MUON])
def test_resume_in_two_calls(rule):
    """The final weights of one call over T equal two calls over the two
    halves with the first call's weights passed in; holds for a ragged last
    chunk too (T = 26, chunk 8 -> 8, 8, 8, 2)."""
    q, k, v, lr, beta, w1, w2, w3 = _problem(T=26, H=2)
    full = _layer(q, k, v, lr, beta, w1, w2, w3, 8, APPLY_THEN_UPDATE, rule)
    a = _layer(q[:, :, :16], k[:, :, :16], v[:, :, :16], lr[:, :, :16], None,
               w1, w2, w3, 8, APPLY_THEN_UPDATE, rule)
    b = _layer(q[:, :, 16:], k[:, :, 16:], v[:, :, 16:], lr[:, :, 16:], None,
               a[1], a[2], a[3], 8, APPLY_THEN_UPDATE, rule)
    np.testing.assert_allclose(full[0][:, :, :16], a[0], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(full[0][:, :, 16:], b[0], rtol=1e-13, atol=1e-15)
    for x, y in zip(full[1:], b[1:]):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- brute force
def test_chunk_of_one_token_matches_per_token_brute_force():
    """chunk = 1 equals a per-token loop written independently: torch autograd
    for each matrix's gradient, F.normalize for the renorm."""
    B, H, T, d, dh = 1, 1, 9, 5, 7
    q, k, v, lr, beta, w1, w2, w3 = _problem(B=B, H=H, T=T, d=d, dh=dh, lr_scale=20.0)
    out, o1, o2, o3 = _layer(q, k, v, lr, beta, w1, w2, w3, 1, APPLY_THEN_UPDATE, RULE_GD)
    f = torch.nn.functional
    W = [torch.tensor(w1[0]), torch.tensor(w2[0]), torch.tensor(w3[0])]
    norms = [w.norm(dim=1, keepdim=True) for w in W]
    qt = f.normalize(f.silu(torch.tensor(q[0, 0])), dim=1)
    kt = f.normalize(f.silu(torch.tensor(k[0, 0])), dim=1)
    vt, lt = torch.tensor(v[0, 0]), torch.tensor(lr[0, 0])
    outs = []
    for i in range(T):
        outs.append(f.linear(f.silu(f.linear(qt[i], W[0])) * f.linear(qt[i], W[2]), W[1]))
        Wr = [w.clone().requires_grad_(True) for w in W]
        fk = f.linear(f.silu(f.linear(kt[i], Wr[0])) * f.linear(kt[i], Wr[2]), Wr[1])
        new = []
        for j in range(3):
            (g,) = torch.autograd.grad(-lt[i, j] * torch.dot(fk, vt[i]), Wr[j],
                                       retain_graph=True)
            new.append(f.normalize(W[j] - g, dim=1) * norms[j])
        W = new
    np.testing.assert_allclose(out[0, 0], torch.stack(outs).numpy(), rtol=1e-11, atol=1e-13)
    for got, want in zip((o1[0], o2[0], o3[0]), W):
        np.testing.assert_allclose(got, want.numpy(), rtol=1e-11, atol=1e-13)


def test_shared_and_per_batch_initial_weights_agree():
    q, k, v, lr, beta, w1, w2, w3 = _problem(B=2, H=2, T=12)
    a = _layer(q, k, v, lr, beta, w1, w2, w3, 4, APPLY_THEN_UPDATE, RULE_GD)
    rep = lambda w: np.concatenate([w, w], axis=0)
    b = _layer(q, k, v, lr, beta, rep(w1), rep(w2), rep(w3), 4, APPLY_THEN_UPDATE, RULE_GD)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("order", [APPLY_THEN_UPDATE, UPDATE_THEN_APPLY])
def test_ragged_last_chunk_is_processed_as_a_short_chunk(order):
    """T = 10, chunk 4: chunks of 4, 4 and 2 tokens.  The result equals a run
    over the first 8 tokens followed by one exact 2-token chunk."""
    q, k, v, lr, beta, w1, w2, w3 = _problem(T=10, H=1, lr_scale=10.0)
    full = _layer(q, k, v, lr, beta, w1, w2, w3, 4, order, RULE_GD)
    a = _layer(q[:, :, :8], k[:, :, :8], v[:, :, :8], lr[:, :, :8], None,
               w1, w2, w3, 4, order, RULE_GD)
    b = _layer(q[:, :, 8:], k[:, :, 8:], v[:, :, 8:], lr[:, :, 8:], None,
               a[1], a[2], a[3], 2, order, RULE_GD)
    np.testing.assert_allclose(full[0][:, :, 8:], b[0], rtol=1e-13, atol=1e-15)
    assert np.all(np.abs(b[0]) > 0)
    for x, y in zip(full[1:], b[1:]):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-15)
    assert not np.allclose(full[1], a[1])


# ---------------------------------------------------------------- options
def _state_after(k, v, lr, beta, w1, w2, w3, ch, rule, n_tokens):
    """(W1, W2, W3) of every (b, h) after the first n_tokens keys, from a run
    without options (the initial weights when n_tokens is 0)."""
    if n_tokens == 0:
        return w1, w2, w3
    t = slice(0, n_tokens)
    q = k[:, :, t]                      # the queries do not touch the state
    _, a1, a2, a3 = _layer(q, k[:, :, t], v[:, :, t], lr[:, :, t],
                           None if beta is None else beta[:, :, t], w1, w2, w3, ch,
                           APPLY_THEN_UPDATE, rule)
    return a1, a2, a3


@pytest.mark.parametrize("rule", [RULE_GD, RULE_MOMENTUM, RULE_MUON])
@pytest.mark.parametrize("order", [APPLY_THEN_UPDATE, UPDATE_THEN_APPLY])
def test_masked_chunks_act_as_if_their_keys_were_absent(rule, order):
    """A chunk whose update flag is 0 is read but writes nothing ("LaCT：以大
    分块更新人工智能的临时记忆" 「更新顺序必须遵守信息可见范围」: video chunks
    with noise read the memory, only clean chunks update it; "LaCT架构核心思想
    解析" §3.2).  So the final weights and momentum equal a run over the
    unmasked chunks alone, and each chunk's output is f of the state that the
    unmasked chunks before it (order 0) or up to and including it (order 1)
    leave, checked through library modules."""
    ch, mask = 5, [1, 0, 0, 1, 0, 1]
    T = ch * len(mask)
    q, k, v, lr, beta, w1, w2, w3 = _problem(T=T, H=2, beta=True, lr_scale=5.0)
    res = oracle.ttt_layer_ex(q, k, v, lr, beta, w1, w2, w3, ch, order, rule, update_mask=mask)
    keep = np.concatenate([np.arange(c * ch, (c + 1) * ch) for c, m in enumerate(mask) if m])
    sub = lambda x: x[:, :, keep]
    red = oracle.ttt_layer_ex(sub(q), sub(k), sub(v), sub(lr), sub(beta), w1, w2, w3, ch, order,
                              rule)
    for x, y in zip(res[1:], red[1:]):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-15)
    for c in range(len(mask)):
        n_upd = sum(mask[:c]) + (mask[c] if order == UPDATE_THEN_APPLY else 0)
        W = _state_after(sub(k), sub(v), sub(lr), sub(beta), w1, w2, w3, ch, rule, n_upd * ch)
        rows = slice(c * ch, (c + 1) * ch)
        for h in range(2):
            want = _torch_swiglu(W[0][h], W[1][h], W[2][h], oracle.qk_prologue(q[0, h, rows]))
            np.testing.assert_allclose(res[0][0, h, rows], want, rtol=1e-11, atol=1e-13)
    assert not np.allclose(res[1], w1)


@pytest.mark.parametrize("order", [APPLY_THEN_UPDATE, UPDATE_THEN_APPLY])
def test_all_chunks_masked_reads_only_the_initial_state(order):
    """With every flag 0 nothing updates: out = f_{W0}(q^) for every query
    (library modules), the weights and the given momentum come back as they
    went in."""
    q, k, v, lr, beta, w1, w2, w3 = _problem(B=2, H=2, T=12, beta=True)
    m_in = tuple(_rand(4, *w.shape[1:]) for w in (w1, w2, w3))
    out, o1, o2, o3, m1, m2, m3 = oracle.ttt_layer_ex(
        q, k, v, lr, beta, w1, w2, w3, 4, order, RULE_MOMENTUM, update_mask=[0, 0, 0], m_in=m_in)
    for b in range(2):
        for h in range(2):
            np.testing.assert_allclose(out[b, h], _torch_swiglu(w1[h], w2[h], w3[h],
                                                                oracle.qk_prologue(q[b, h])),
                                       rtol=1e-12, atol=1e-14)
            np.testing.assert_array_equal(o1[b * 2 + h], w1[h])
            np.testing.assert_array_equal(o2[b * 2 + h], w2[h])
            np.testing.assert_array_equal(o3[b * 2 + h], w3[h])
    for got, want in zip((m1, m2, m3), m_in):
        np.testing.assert_array_equal(got, want)


def test_all_ones_mask_is_the_plain_layer():
    q, k, v, lr, beta, w1, w2, w3 = _problem(T=18, beta=True)
    a = _layer(q, k, v, lr, beta, w1, w2, w3, 6, APPLY_THEN_UPDATE, RULE_MOMENTUM)
    b = oracle.ttt_layer_ex(q, k, v, lr, beta, w1, w2, w3, 6, APPLY_THEN_UPDATE, RULE_MOMENTUM,
                            update_mask=[1, 1, 1])
    for x, y in zip(a, b[:4]):
        np.testing.assert_array_equal(x, y)


def test_momentum_resume_in_two_calls():
    """Momentum carried across calls ("LaCT架构核心思想解析" §1.2 momentum,
    resumed): one call over T equals two calls over the halves with the first
    call's weights AND momentum passed in.  Without the momentum the second
    half differs.  A masked chunk on each side of the split too."""
    q, k, v, lr, beta, w1, w2, w3 = _problem(B=2, H=2, T=24, beta=True, lr_scale=5.0)
    mask = [1, 0, 1, 1, 0, 1]
    full = oracle.ttt_layer_ex(q, k, v, lr, beta, w1, w2, w3, 4, APPLY_THEN_UPDATE,
                               RULE_MOMENTUM, update_mask=mask)
    h1, h2 = slice(0, 12), slice(12, 24)
    cut = lambda x, s: x[:, :, s]
    a = oracle.ttt_layer_ex(cut(q, h1), cut(k, h1), cut(v, h1), cut(lr, h1), cut(beta, h1),
                            w1, w2, w3, 4, APPLY_THEN_UPDATE, RULE_MOMENTUM, update_mask=mask[:3])
    b = oracle.ttt_layer_ex(cut(q, h2), cut(k, h2), cut(v, h2), cut(lr, h2), cut(beta, h2),
                            a[1], a[2], a[3], 4, APPLY_THEN_UPDATE, RULE_MOMENTUM,
                            update_mask=mask[3:], m_in=a[4:])
    np.testing.assert_allclose(full[0][:, :, h1], a[0], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(full[0][:, :, h2], b[0], rtol=1e-13, atol=1e-15)
    for x, y in zip(full[1:], b[1:]):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-15)
    c = oracle.ttt_layer_ex(cut(q, h2), cut(k, h2), cut(v, h2), cut(lr, h2), cut(beta, h2),
                            a[1], a[2], a[3], 4, APPLY_THEN_UPDATE, RULE_MOMENTUM,
                            update_mask=mask[3:])
    assert not np.allclose(c[1], b[1])


def test_given_momentum_is_the_first_decayed_term():
    """One chunk from M_0: U = mean(beta) M_0 + G ("LaCT架构核心思想解析"
    §1.2), built from the oracle's gradient; beta = 0 makes M_0 irrelevant."""
    d, dh, n = 6, 8, 5
    W = _weights(d, dh)
    M0 = tuple(_rand(*w.shape) * 0.05 for w in W)
    k, v, q = _rand(n, d), _rand(n, d), _rand(n, d)
    lr = np.abs(_rand(n, 3)) * 0.3
    beta = RNG.uniform(0.2, 0.9, n)
    G = oracle.chunk_gradient(*W, oracle.qk_prologue(k), v, lr)
    M1 = tuple(beta.mean() * m + g for m, g in zip(M0, G))
    want = tuple(oracle.renorm_rows(w - m, w) for w, m in zip(W, M1))
    one = lambda x: x[None, None]
    res = oracle.ttt_layer_ex(one(q), one(k), one(v), one(lr), one(beta), W[0][None], W[1][None],
                              W[2][None], n, APPLY_THEN_UPDATE, RULE_MOMENTUM,
                              m_in=tuple(m[None] for m in M0))
    for got, w in zip(res[1:4], want):
        np.testing.assert_allclose(got[0], w, rtol=1e-12)
    for got, m in zip(res[4:], M1):
        np.testing.assert_allclose(got[0], m, rtol=1e-12)
    zero = oracle.ttt_layer_ex(one(q), one(k), one(v), one(lr), one(0 * beta), W[0][None],
                               W[1][None], W[2][None], n, APPLY_THEN_UPDATE, RULE_MOMENTUM,
                               m_in=tuple(m[None] for m in M0))
    plain = _layer(one(q), one(k), one(v), one(lr), one(0 * beta), W[0][None], W[1][None],
                   W[2][None], n, APPLY_THEN_UPDATE, RULE_GD)
    for x, y in zip(zero[:4], plain):
        np.testing.assert_allclose(x, y, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("order", [APPLY_THEN_UPDATE, UPDATE_THEN_APPLY])
def test_output_scale_multiplies_each_query_row(order):
    """The per-head output scale ("LaCT架构核心思想解析" §2.1) multiplies the
    output row of its own (batch, head, query) and nothing else: a scale of 1
    changes no bit, other scales (negative and zero included) scale exactly
    that row, and the state is untouched."""
    B, H, T = 2, 3, 12
    q, k, v, lr, beta, w1, w2, w3 = _problem(B=B, H=H, T=T)
    base = _layer(q, k, v, lr, beta, w1, w2, w3, 4, order, RULE_GD)
    ones = oracle.ttt_layer_ex(q, k, v, lr, beta, w1, w2, w3, 4, order, RULE_GD,
                               out_scale=np.ones((B, H, T)))
    for x, y in zip(base, ones[:4]):
        np.testing.assert_array_equal(x, y)
    s = _rand(B, H, T)
    s[0, 1, 3] = 0.0
    s[1, 2, 5] = -2.0
    res = oracle.ttt_layer_ex(q, k, v, lr, beta, w1, w2, w3, 4, order, RULE_GD, out_scale=s)
    for b in range(B):
        for h in range(H):
            for t in range(T):
                np.testing.assert_allclose(res[0][b, h, t], s[b, h, t] * base[0][b, h, t],
                                           rtol=1e-15, atol=0)
    for x, y in zip(base[1:], res[1:4]):
        np.testing.assert_array_equal(x, y)
