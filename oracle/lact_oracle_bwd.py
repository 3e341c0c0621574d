"""CPU fp64 oracle of the LaCT TTT layer BACKWARD -- TEST INFRASTRUCTURE.

Imported only by tests/, __graft_entry__.smoke() and bench.py's CPU legs.

The backward of a function has a plain definition: the vector-Jacobian
product of the forward.  This module restates the forward chunk loop of
`lact_oracle.ttt_head_state` in plain fp64 torch operations (same steps, same
order: [P1 §1.2, §2.2], [P2 §2.1, §2.2.1], [P3] 「局部注意力与非线性记忆相互
补充」, 「更新顺序必须遵守信息可见范围」) and takes the gradients with
torch.autograd, a library routine, as one step.  The pins check this forward
against the numpy oracle and the gradients against central finite
differences.

Covered: the GD, momentum and Muon rules (the Muon backward runs through
the Frobenius normalisation and the five Newton-Schulz steps), both orders,
the per-chunk update mask, the output scale, shared or per-(b, h) initial
weights.
"""
from __future__ import annotations

import numpy as np
import torch

APPLY_THEN_UPDATE, UPDATE_THEN_APPLY = 0, 1
RULE_GD, RULE_MOMENTUM, RULE_MUON = 0, 1, 2

# Newton-Schulz quintic of the Muon rule (R7): coefficients, steps, eps.
NS_COEFFS = (3.4445, -4.7750, 2.0315)
NS_STEPS = 5
NS_EPS = 1e-7


def _t(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64)
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def _silu(z):
    return z * torch.sigmoid(z)


def _prologue(x):
    """silu, then the row's L2 norm over the head dim [P1 §1.2]."""
    s = _silu(x)
    return s / s.norm(dim=-1, keepdim=True)


def _fast_net(W1, W2, W3, X):
    """f_W(x) = W2 (silu(W1 x) * (W3 x)) for the rows of X."""
    return (_silu(X @ W1.T) * (X @ W3.T)) @ W2.T


def _chunk_grads(W1, W2, W3, K, V, lr):
    """Per-token-rate chunk gradient of -sum lr[i, j] <f_W(k_i), v_i> with
    respect to W_j, written out as the oracle does (R1, R3), so that its own
    derivative (the second-order terms of the backward) comes from autograd."""
    Z1 = K @ W1.T
    Z3 = K @ W3.T
    S1 = _silu(Z1)
    sg = torch.sigmoid(Z1)
    Sp = sg * (1.0 + Z1 * (1.0 - sg))          # silu'(z1)
    U = V @ W2
    G1 = -((lr[:, 0:1] * (U * Z3 * Sp)).T @ K)
    G2 = -((lr[:, 1:2] * V).T @ (S1 * Z3))
    G3 = -((lr[:, 2:3] * (U * S1)).T @ K)
    return G1, G2, G3


def _newton_schulz5(G):
    """Muon's orthogonalised update of a gradient matrix [P2 §2.2.1]
    eqs. 9-10: X = G / (||G||_F + eps), then five times
    X <- a X + (b A + c A A) X with A = X X^T, X oriented so that A is the
    smaller Gram matrix (the same result in exact arithmetic either way)."""
    a, b, c = NS_COEFFS
    X = G / (G.norm() + NS_EPS)
    transposed = X.shape[0] > X.shape[1]
    if transposed:
        X = X.T
    for _ in range(NS_STEPS):
        A = X @ X.T
        X = a * X + (b * A + c * (A @ A)) @ X
    return X.T if transposed else X


def _renorm(W_new, W_old):
    """Each row of W_new scaled to the norm its row had before (R4, R5)."""
    return W_new * (W_old.norm(dim=1, keepdim=True) / W_new.norm(dim=1, keepdim=True))


def head_forward(q, k, v, lr, beta, W1, W2, W3, chunk, order, rule, update_mask=None,
                 out_scale=None, M0=None):
    """The layer for one (batch, head) in torch fp64: returns out [Tq, d],
    the final (W1, W2, W3) and the final momentum (zeros for GD).  M0: the
    momentum before the first chunk (R15), zeros if None."""
    T, Tq = k.shape[0], q.shape[0]
    starts = list(range(0, T, chunk))
    qh, kh = _prologue(q), _prologue(k)
    W = (W1, W2, W3)
    M = tuple(torch.zeros_like(w) for w in W) if M0 is None else tuple(M0)
    outs = []
    for ci, c0 in enumerate(starts):
        c1 = min(c0 + chunk, T)
        rows = slice(0, Tq) if len(starts) == 1 else slice(c0, c1)
        upd = update_mask is None or bool(update_mask[ci])
        if order == APPLY_THEN_UPDATE:
            outs.append(_fast_net(*W, qh[rows]))
        if upd:
            G = _chunk_grads(*W, kh[c0:c1], v[c0:c1], lr[c0:c1])
            if rule == RULE_MOMENTUM:
                bbar = beta[c0:c1].mean()
                M = tuple(bbar * m + g for m, g in zip(M, G))
                U = M
            elif rule == RULE_GD:
                U = G
            elif rule == RULE_MUON:
                U = tuple(_newton_schulz5(g) for g in G)
            else:
                raise ValueError(f"unknown rule {rule}")
            W = tuple(_renorm(w - u, w) for w, u in zip(W, U))
        if order == UPDATE_THEN_APPLY:
            outs.append(_fast_net(*W, qh[rows]))
    out = torch.cat(outs, dim=0)
    if out_scale is not None:
        out = out_scale[:, None] * out
    return out, W, M


def ttt_layer_bwd(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule, dout, dw=None,
                  update_mask=None, out_scale=None, heads=None, m_in=None, dm=None):
    """Gradients of sum(out * dout) + sum_j <w_j_out, dw_j> over the layer's
    inputs, on the ABI layout (q [B,H,Tq,d]; k, v [B,H,T,d]; lr [B,H,T,3];
    beta [B,H,T] or None; w1, w3 [Hw,dh,d], w2 [Hw,d,dh] with Hw = H or B*H;
    dout like out; dw = (dw1, dw2, dw3) like w_out, or None).

    Returns a dict with dq, dk, dv, dlr, dbeta (or None), dw1, dw2, dw3 (the
    shape of the initial weights: summed over the batch when they are
    shared), dout_scale (or None) and, for the forward check, out and the
    final weights (w1o, w2o, w3o).  heads: optional (b, h) pairs; the others
    are left as NaN (the initial-weight gradients then sum only those).

    Momentum in/out (R15, momentum rule): m_in = (m1, m2, m3), each [B*H]
    in the layout of w*_out, the momentum before the first chunk (zeros if
    None); dm = the gradients of the final momentum, added to the loss as
    sum_j <m_j_out, dm_j>.  With either given, the dict also holds dm1,
    dm2, dm3 (the gradients of m_in) and the final momentum (m1o, m2o,
    m3o)."""
    q, k, v, lr, beta = _t(q), _t(k), _t(v), _t(lr), _t(beta)
    w1, w2, w3, dout = _t(w1), _t(w2), _t(w3), _t(dout)
    dw = None if dw is None else tuple(_t(x) for x in dw)
    out_scale = _t(out_scale)
    with_m = m_in is not None or dm is not None
    if with_m and rule != RULE_MOMENTUM:
        raise ValueError("momentum in/out needs the momentum rule")
    m_in = None if m_in is None else tuple(_t(x) for x in m_in)
    dm = None if dm is None else tuple(_t(x) for x in dm)
    B, H, Tq, d = q.shape
    T = k.shape[2]
    dh = w1.shape[1]
    per_bh = w1.shape[0] == B * H
    nan = float("nan")
    res = {
        "dq": torch.full_like(q, nan), "dk": torch.full_like(k, nan), "dv": torch.full_like(v, nan),
        "dlr": torch.full_like(lr, nan), "dbeta": None if beta is None else torch.full_like(beta, nan),
        "dw1": torch.zeros_like(w1), "dw2": torch.zeros_like(w2), "dw3": torch.zeros_like(w3),
        "dout_scale": None if out_scale is None else torch.full_like(out_scale, nan),
        "out": torch.full_like(q, nan), "w1o": torch.full((B * H, dh, d), nan, dtype=torch.float64),
        "w2o": torch.full((B * H, d, dh), nan, dtype=torch.float64),
        "w3o": torch.full((B * H, dh, d), nan, dtype=torch.float64),
    }
    if with_m:
        for j, shp in ((1, (dh, d)), (2, (d, dh)), (3, (dh, d))):
            res[f"dm{j}"] = torch.full((B * H,) + shp, nan, dtype=torch.float64)
            res[f"m{j}o"] = torch.full((B * H,) + shp, nan, dtype=torch.float64)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    mask = None if update_mask is None else [int(x) for x in update_mask]
    for b, h in todo:
        wi = b * H + h if per_bh else h
        leaves = [q[b, h].clone(), k[b, h].clone(), v[b, h].clone(), lr[b, h].clone(),
                  None if beta is None else beta[b, h].clone(),
                  w1[wi].clone(), w2[wi].clone(), w3[wi].clone(),
                  None if out_scale is None else out_scale[b, h].clone()]
        bh = b * H + h
        M0 = None
        if with_m:
            M0 = [torch.zeros_like(x) if m_in is None else m_in[j][bh].clone()
                  for j, x in enumerate((w1[wi], w2[wi], w3[wi]))]
            leaves += M0
        for x in leaves:
            if x is not None:
                x.requires_grad_(True)
        qq, kk, vv, ll, bb, W1, W2, W3, ss = leaves[:9]
        out, W, M = head_forward(qq, kk, vv, ll, bb, W1, W2, W3, chunk, order, rule, mask, ss, M0)
        loss = (out * dout[b, h]).sum()
        if dw is not None:
            loss = loss + sum((wf * g[bh]).sum() for wf, g in zip(W, dw))
        if dm is not None:
            loss = loss + sum((mf * g[bh]).sum() for mf, g in zip(M, dm))
        want = [x for x in leaves if x is not None]
        grads = torch.autograd.grad(loss, want, allow_unused=True)
        it = iter(grads)
        g = {}
        for name, x in zip(("dq", "dk", "dv", "dlr", "dbeta", "dw1", "dw2", "dw3", "dout_scale",
                            "dm1", "dm2", "dm3"), leaves):
            if x is not None:
                gx = next(it)
                g[name] = torch.zeros_like(x) if gx is None else gx
        res["dq"][b, h], res["dk"][b, h], res["dv"][b, h] = g["dq"], g["dk"], g["dv"]
        res["dlr"][b, h] = g["dlr"]
        if beta is not None:
            res["dbeta"][b, h] = g["dbeta"]
        if out_scale is not None:
            res["dout_scale"][b, h] = g["dout_scale"]
        res["dw1"][wi] += g["dw1"]
        res["dw2"][wi] += g["dw2"]
        res["dw3"][wi] += g["dw3"]
        res["out"][b, h] = out.detach()
        res["w1o"][bh], res["w2o"][bh], res["w3o"][bh] = (x.detach() for x in W)
        if with_m:
            for j in range(3):
                res[f"dm{j + 1}"][bh] = g[f"dm{j + 1}"]
                res[f"m{j + 1}o"][bh] = M[j].detach()
    return {k_: (None if v_ is None else v_.numpy()) for k_, v_ in res.items()}
