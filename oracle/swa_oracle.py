"""CPU fp64 oracle of LaCT's sliding-window attention -- TEST INFRASTRUCTURE.

Imported only by tests/, __graft_entry__.smoke() and bench.py's CPU legs.

The other half of the LaCT block ("LaCT架构核心思想解析" §1.1): local window
attention in which every token sees only a window of preceding tokens, with
per-channel learnable scales and offsets applied to the queries and keys
before the dot products.  Readings (also in the design notes):
  A1 the window is causal and holds the w most recent tokens, the token
     itself included: keys j with t - w < j <= t;
  A2 the scales and offsets are per head and channel, [H, d]:
     q' = q * q_scale + q_offset, k' = k * k_scale + k_offset;
  A3 softmax of q' . k' / sqrt(d) over the window (plain scaled dot-product
     attention), then the weighted sum of the values v (not transformed).
"""
from __future__ import annotations

import numpy as np


def _f64(t):
    if hasattr(t, "detach"):
        t = t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def swa_head(q, k, v, qs, qo, ks, ko, window, rows=None):
    """One (batch, head): q, k, v [T, d]; qs, qo, ks, ko [d].  Returns [T, d]
    (only the query rows in `rows` when given; the others are NaN)."""
    T, d = q.shape
    qp = q * qs + qo
    kp = k * ks + ko
    out = np.full_like(v, np.nan) if rows is not None else np.zeros_like(v)
    for t in (range(T) if rows is None else rows):
        j0 = max(0, t - window + 1)
        s = kp[j0:t + 1] @ qp[t] / np.sqrt(d)
        p = np.exp(s - s.max())
        out[t] = (p / p.sum()) @ v[j0:t + 1]
    return out


def swa_layer(q, k, v, q_scale, q_offset, k_scale, k_offset, window, heads=None, rows=None):
    """q, k, v [B, H, T, d]; scales and offsets [H, d].  Returns [B, H, T, d]
    (heads not in `heads` and query rows not in `rows`, when given, are NaN)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    qs, qo, ks, ko = (_f64(x) for x in (q_scale, q_offset, k_scale, k_offset))
    B, H, T, d = q.shape
    out = np.full((B, H, T, d), np.nan)
    for b, h in (heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]):
        out[b, h] = swa_head(q[b, h], k[b, h], v[b, h], qs[h], qo[h], ks[h], ko[h], window, rows)
    return out
