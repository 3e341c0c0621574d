"""CPU fp64 oracle of the LaCT fast-weight TTT layer -- TEST INFRASTRUCTURE.

Imported only by tests/, __graft_entry__.smoke() and bench.py's CPU legs.
Page citations ([P1], [P2], [P3]) and the readings R1..R10 are defined in
this package's __init__ docstring.
"""
from __future__ import annotations

import numpy as np

APPLY_THEN_UPDATE, UPDATE_THEN_APPLY = 0, 1
RULE_GD, RULE_MOMENTUM, RULE_MUON = 0, 1, 2

# Newton-Schulz quintic coefficients and step count of the Muon rule (R7).
NS_COEFFS = (3.4445, -4.7750, 2.0315)
NS_STEPS = 5
NS_EPS = 1e-7


def sigmoid(z):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    """silu(z) = z * sigmoid(z)  [P1 §1.2]."""
    return z * sigmoid(z)


def silu_prime(z):
    """d/dz silu(z) = s + z s (1 - s), s = sigmoid(z)."""
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


def qk_prologue(x):
    """q, k <- silu(q), silu(k); then q, k <- q/||q||, k/||k|| over the head
    dim (last axis) [P1 §1.2].  An all-zero row stays zero (R8)."""
    s = silu(np.asarray(x, dtype=np.float64))
    n = np.sqrt((s * s).sum(axis=-1, keepdims=True))
    safe = np.where(n > 0.0, n, 1.0)
    return np.where(n > 0.0, s / safe, 0.0)


def fast_net(W1, W2, W3, X):
    """The SwiGLU fast-weight net f_W(x) = W2 (silu(W1 x) * (W3 x)) applied to
    every row x of X [n, d] (the "apply" of [P2 §2.1], eq. 2; three-matrix
    SwiGLU memory of [P3] 「局部注意力与非线性记忆相互补充」).
    W1, W3: [dh, d]; W2: [d, dh].  Returns [n, d]."""
    Z1 = X @ W1.T                      # row i: W1 x_i
    Z3 = X @ W3.T                      # row i: W3 x_i
    Hid = silu(Z1) * Z3                # row i: silu(W1 x_i) * (W3 x_i)
    return Hid @ W2.T                  # row i: W2 h_i


def chunk_gradient(W1, W2, W3, K, V, lr):
    """Gradient of the chunk loss with per-token rates (R1, R3):
         G_j = d/dW_j [ - sum_i lr[i, j] * <f_W(k_i), v_i> ],  j = 1, 2, 3
    summed over the whole chunk ([P2 §2.1] eqs. 4-5; loss and per-token
    rates from [P3] 「局部注意力与非线性记忆相互补充」).

    Per token, with z1 = W1 k, z3 = W3 k, h = silu(z1) * z3 and
    u = W2^T v (= d<W2 h, v>/dh):
        d<f,v>/dW2 = v h^T
        d<f,v>/dW1 = (u * z3 * silu'(z1)) k^T
        d<f,v>/dW3 = (u * silu(z1)) k^T
    The sums over tokens of these outer products are written as products of
    the stacked rows.  Returns (G1 [dh,d], G2 [d,dh], G3 [dh,d])."""
    Z1 = K @ W1.T
    Z3 = K @ W3.T
    S1 = silu(Z1)
    Hid = S1 * Z3
    U = V @ W2                         # row i: u_i = W2^T v_i
    D1 = U * Z3 * silu_prime(Z1)       # d<f,v>/dz1 per token
    D3 = U * S1                        # d<f,v>/dz3 per token
    G1 = -((lr[:, 0:1] * D1).T @ K)
    G2 = -((lr[:, 1:2] * V).T @ Hid)
    G3 = -((lr[:, 2:3] * D3).T @ K)
    return G1, G2, G3


def newton_schulz5(G):
    """Muon's orthogonalisation of a gradient matrix ([P2 §2.2.1] eqs. 9-10,
    [P3] "Newton-Schulz"; coefficients, step count and eps per R7):
        X <- G / (||G||_F + eps)
        5 times:  A = X X^T;  B = b A + c A A;  X <- a X + B X
    run with X oriented so that X X^T is the smaller Gram matrix."""
    a, b, c = NS_COEFFS
    X = G / (np.sqrt((G * G).sum()) + NS_EPS)
    transposed = X.shape[0] > X.shape[1]
    if transposed:
        X = X.T
    for _ in range(NS_STEPS):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
    return X.T if transposed else X


def renorm_rows(W_new, W_old):
    """Row-wise L2 renormalisation after an update ([P2 §2.2.1] eq. 8,
    [P1 §1.2] "W <- L2_norm(W - M)", [P3]): every row of W_new is scaled to
    the L2 norm its row had before the update (R4, R5).  A row that the
    update zeroed stays zero."""
    old = np.sqrt((W_old * W_old).sum(axis=1, keepdims=True))
    new = np.sqrt((W_new * W_new).sum(axis=1, keepdims=True))
    safe = np.where(new > 0.0, new, 1.0)
    return np.where(new > 0.0, W_new * (old / safe), 0.0)


def rule_step(rule, G, M, beta_chunk):
    """Turn the chunk gradients G = (G1, G2, G3) into updates U (R2, R6, R7).
    GD: U = G.  Momentum [P1 §1.2]: M <- mean(beta_chunk) M + G, U = M.
    Muon [P2 §2.2.1]: U = NS5(G).  Returns (U, new M)."""
    if rule == RULE_GD:
        return G, M
    if rule == RULE_MOMENTUM:
        bbar = float(np.mean(beta_chunk))
        M = tuple(bbar * m + g for m, g in zip(M, G))
        return M, M
    if rule == RULE_MUON:
        return tuple(newton_schulz5(g) for g in G), M
    raise ValueError(f"unknown rule {rule}")


def ttt_head_state(q, k, v, lr, beta, W1, W2, W3, chunk, order, rule,
                   update_mask=None, out_scale=None, M0=None):
    """The layer for one (batch, head): q [Tq, d], k, v [T, d], lr [T, 3],
    beta [T] (momentum only), W1, W3 [dh, d], W2 [d, dh].

    Chunk loop, in the order of [P3] 「更新顺序必须遵守信息可见范围」 and
    [P1 §2.2]:
      order 0 (apply-then-update, causal): o_c = f_{W_{c-1}}(q_c), then
              W_c = renorm(W_{c-1} - U(grad of chunk c on W_{c-1}));
      order 1 (update-then-apply, sets):  W_c first, then o_c = f_{W_c}(q_c).
    Options (R13-R15):
      update_mask  one flag per chunk; a chunk whose flag is 0 is applied in
                   its place in the order but skips the whole update
                   (gradient, rule, momentum, renorm), so W_c = W_{c-1}
                   (noisy video chunks read the memory, clean ones write
                   it: [P3] 「更新顺序…」, [P1 §3.2]).
      out_scale    [Tq] per-query factor s_t: o_t = s_t * f_W(q_t)
                   ([P1 §2.1] per-head output scale).
      M0           initial momentum (M1, M2, M3) instead of zeros.
    Returns out [Tq, d], the final (W1, W2, W3) and the final momentum."""
    T, Tq = k.shape[0], q.shape[0]
    starts = list(range(0, T, chunk))
    if len(starts) > 1 and Tq != T:
        raise ValueError("Tq != T needs a single chunk (R10)")
    if update_mask is not None and len(update_mask) != len(starts):
        raise ValueError("update_mask needs one flag per chunk")
    qh = qk_prologue(q)
    kh = qk_prologue(k)
    W = (np.array(W1, dtype=np.float64), np.array(W2, dtype=np.float64),
         np.array(W3, dtype=np.float64))
    if M0 is None:
        M = tuple(np.zeros_like(w) for w in W)
    else:
        M = tuple(np.array(m, dtype=np.float64) for m in M0)
    out = np.zeros_like(qh)
    for ci, c0 in enumerate(starts):
        c1 = min(c0 + chunk, T)                       # R9: ragged last chunk
        rows = slice(0, Tq) if len(starts) == 1 else slice(c0, c1)
        updates = update_mask is None or bool(update_mask[ci])
        if order == APPLY_THEN_UPDATE:
            out[rows] = fast_net(*W, qh[rows])
        if updates:
            G = chunk_gradient(*W, kh[c0:c1], v[c0:c1], lr[c0:c1])
            U, M = rule_step(rule, G, M, None if beta is None else beta[c0:c1])
            W = tuple(renorm_rows(w - u, w) for w, u in zip(W, U))
        if order == UPDATE_THEN_APPLY:
            out[rows] = fast_net(*W, qh[rows])
    if out_scale is not None:
        out = np.asarray(out_scale, dtype=np.float64)[:, None] * out
    return out, W, M


def ttt_head(q, k, v, lr, beta, W1, W2, W3, chunk, order, rule):
    """ttt_head_state without options; returns out [Tq, d] and the final
    (W1, W2, W3)."""
    out, W, _ = ttt_head_state(q, k, v, lr, beta, W1, W2, W3, chunk, order, rule)
    return out, W


def _f64(t):
    if t is None:
        return None
    if hasattr(t, "detach"):                          # a torch tensor
        t = t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def ttt_layer_ex(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule, heads=None,
                 update_mask=None, out_scale=None, m_in=None):
    """The whole layer on the ABI layout: q [B,H,Tq,d], k, v [B,H,T,d],
    lr [B,H,T,3], beta [B,H,T] or None, w1, w3 [Hw,dh,d], w2 [Hw,d,dh] with
    Hw = H (initial state shared across the batch) or B*H.  Inputs may be
    torch tensors or arrays; each head's slice is upcast to fp64.

    heads: optional list of (b, h) pairs to compute (the heads are
    independent); the others are left as NaN.
    update_mask: one flag per chunk, shared by every (b, h) (R13).
    out_scale: [B,H,Tq] per-query output factors (R14).
    m_in: (m1 [B*H,dh,d], m2 [B*H,d,dh], m3 [B*H,dh,d]) initial momentum (R15).
    Returns out [B,H,Tq,d], w1o [B*H,dh,d], w2o [B*H,d,dh], w3o [B*H,dh,d],
    m1o, m2o, m3o (the final momentum, zeros unless the rule is momentum)."""
    B, H, Tq, d = q.shape
    dh = w1.shape[1]
    if w1.shape[0] not in (H, B * H):
        raise ValueError("fast-weight init must have H or B*H leading entries")
    out = np.full((B, H, Tq, d), np.nan)
    w1o = np.full((B * H, dh, d), np.nan)
    w2o = np.full((B * H, d, dh), np.nan)
    w3o = np.full((B * H, dh, d), np.nan)
    m1o, m2o, m3o = np.full_like(w1o, np.nan), np.full_like(w2o, np.nan), np.full_like(w3o, np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    mask = None if update_mask is None else [int(x) for x in update_mask]
    for b, h in todo:
        wi = b * H + h if w1.shape[0] == B * H else h
        bh = b * H + h
        M0 = None if m_in is None else tuple(_f64(m[bh]) for m in m_in)
        o, W, M = ttt_head_state(
            _f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(lr[b, h]),
            None if beta is None else _f64(beta[b, h]),
            _f64(w1[wi]), _f64(w2[wi]), _f64(w3[wi]), chunk, order, rule,
            update_mask=mask, out_scale=None if out_scale is None else _f64(out_scale[b, h]),
            M0=M0)
        out[b, h] = o
        w1o[bh], w2o[bh], w3o[bh] = W
        m1o[bh], m2o[bh], m3o[bh] = M
    return out, w1o, w2o, w3o, m1o, m2o, m3o


def ttt_layer(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule, heads=None):
    """ttt_layer_ex without options.  Returns out [B,H,Tq,d], w1o [B*H,dh,d],
    w2o [B*H,d,dh], w3o [B*H,dh,d]."""
    return ttt_layer_ex(q, k, v, lr, beta, w1, w2, w3, chunk, order, rule, heads=heads)[:4]


def blas_threads() -> int:
    """Threads numpy's BLAS uses for the oracle's matrix products."""
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 1) for p in threadpool_info()
             if p.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # pragma: no cover - threadpoolctl missing
        return 1
