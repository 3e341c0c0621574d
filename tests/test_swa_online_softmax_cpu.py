"""The window attention's online softmax with a lazily raised reference max
is the plain softmax up to rounding (a property of the algorithm that the
fused kernel runs; its GPU parity is tested in test_swa_gpu.py).

The model below walks one query row's keys in blocks of 128, as the kernel
does: a block's unnormalised probabilities are 2^(s log2(e)/sqrt(d) - ref)
with the row's reference max `ref`, which is raised (and the running output
and sum rescaled) only when a block's max exceeds it by more than 8 in log2
units.  With exact arithmetic this equals softmax(s/sqrt(d)) v; with the
probabilities rounded to bf16, as the kernel stores them, it stays within
bf16 rounding of it."""
import numpy as np
import pytest

LOG2E = 1.4426950408889634


def bf16_round(x):
    """Round float32 values to bfloat16 (nearest, ties to even), as float32."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def lazy_online_row(s, v, scale, round_p, stats=None):
    """One query row: scores s [n] (already masked to its window), values v [n, d].
    `stats`, if given, receives the number of rescales under "rescales"."""
    c2 = scale * LOG2E
    ref = -np.inf
    acc = np.zeros(v.shape[1], dtype=np.float64)
    total = 0.0
    for b0 in range(0, len(s), 128):
        sb, vb = s[b0:b0 + 128], v[b0:b0 + 128]
        bm = sb.max()
        if ref == -np.inf:
            ref = bm
        elif (bm - ref) * c2 > 8.0:
            a = 2.0 ** ((ref - bm) * c2)
            acc *= a
            total *= a
            ref = bm
            if stats is not None:
                stats["rescales"] = stats.get("rescales", 0) + 1
        p = 2.0 ** (sb * c2 - ref * c2)
        assert p.max() <= 2.0 ** 8 + 1e-9
        if round_p:
            p = bf16_round(p).astype(np.float64)
        acc += p @ vb
        total += p.sum()
    return acc / total


def exact_row(s, v, scale):
    z = s * scale
    e = np.exp(z - z.max())
    return (e / e.sum()) @ v


@pytest.mark.parametrize("spread", [1.0, 6.0, 25.0])
def test_lazy_reference_max_is_the_plain_softmax(spread):
    rng = np.random.default_rng(7)
    d, n = 64, 2176            # 17 blocks: a 2048-key window and the diagonal block
    scale = 1.0 / np.sqrt(d)
    # scores that drift upwards across the window, so later blocks raise the max
    s = rng.standard_normal(n) * spread + np.linspace(0.0, 3.0 * spread, n)
    v = rng.standard_normal((n, d))
    want = exact_row(s, v, scale)
    got = lazy_online_row(s, v, scale, round_p=False)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    got16 = lazy_online_row(s, v, scale, round_p=True)
    err = np.linalg.norm(got16 - want) / np.linalg.norm(want)
    assert err <= 4e-3, err


def test_a_rescale_happens_and_a_small_rise_does_not():
    """Scores rising by less than 8 / (log2(e) / sqrt(d)) keep the first
    block's reference; a larger rise moves it."""
    d = 64
    c2 = LOG2E / np.sqrt(d)
    small = np.concatenate([np.zeros(128), np.full(128, 7.9 / c2)])
    large = np.concatenate([np.zeros(128), np.full(128, 8.1 / c2)])
    v = np.random.default_rng(3).standard_normal((256, 4))
    for s, rescales in ((small, 0), (large, 1)):
        stats = {}
        got = lazy_online_row(s, v, 1.0 / np.sqrt(d), round_p=False, stats=stats)
        assert stats.get("rescales", 0) == rescales
        np.testing.assert_allclose(got, exact_row(s, v, 1.0 / np.sqrt(d)), rtol=1e-12)
