"""Pins of the sliding-window attention oracle (oracle/swa_oracle.py) to the
library attention and to closed forms ("LaCT架构核心思想解析" §1.1)."""
import numpy as np
import pytest
import torch

from oracle import swa_oracle as so

RNG = np.random.default_rng(3)


def _inputs(B=1, H=2, T=40, d=8):
    q, k, v = (RNG.standard_normal((B, H, T, d)) for _ in range(3))
    qs, ks = 1 + 0.3 * RNG.standard_normal((H, d)), 1 + 0.3 * RNG.standard_normal((H, d))
    qo, ko = 0.2 * RNG.standard_normal((H, d)), 0.2 * RNG.standard_normal((H, d))
    return q, k, v, qs, qo, ks, ko


def _torch_sdpa(q, k, v, qs, qo, ks, ko, window):
    """torch's scaled dot-product attention in fp64 with an explicit band mask."""
    T = q.shape[2]
    t = torch.arange(T)
    mask = (t[None, :] <= t[:, None]) & (t[None, :] > t[:, None] - window)
    Q = torch.tensor(q) * torch.tensor(qs)[None, :, None, :] + torch.tensor(qo)[None, :, None, :]
    K = torch.tensor(k) * torch.tensor(ks)[None, :, None, :] + torch.tensor(ko)[None, :, None, :]
    return torch.nn.functional.scaled_dot_product_attention(Q, K, torch.tensor(v), attn_mask=mask).numpy()


@pytest.mark.parametrize("window", [1, 3, 16, 40, 100])
def test_matches_library_attention_with_a_band_mask(window):
    q, k, v, qs, qo, ks, ko = _inputs(B=2)
    got = so.swa_layer(q, k, v, qs, qo, ks, ko, window)
    np.testing.assert_allclose(got, _torch_sdpa(q, k, v, qs, qo, ks, ko, window), rtol=1e-11, atol=1e-12)


def test_window_one_returns_the_values():
    q, k, v, qs, qo, ks, ko = _inputs()
    np.testing.assert_allclose(so.swa_layer(q, k, v, qs, qo, ks, ko, 1), v, rtol=0, atol=1e-15)


def test_a_key_offset_cancels_in_the_softmax():
    """Adding the same vector to every key shifts each query's scores by one
    constant, which the softmax removes: the key offset does not change the
    output (a property of the method, not of the implementation)."""
    q, k, v, qs, qo, ks, ko = _inputs()
    a = so.swa_layer(q, k, v, qs, qo, ks, ko, 7)
    b = so.swa_layer(q, k, v, qs, qo, ks, 5 * RNG.standard_normal(ko.shape), 7)
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)
    c = so.swa_layer(q, k, v, qs, qo + 1.0, ks, ko, 7)
    assert not np.allclose(a, c)
