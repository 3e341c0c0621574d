"""GPU parity of the sliding-window attention (lact_swa_fwd) against the fp64
oracle (oracle/swa_oracle.py): relative L2 <= 2e-2 (bf16 inputs and output,
bf16 probabilities).  Cases span head dims 64..256, windows shorter than,
equal to and longer than the sequence, several 128-query blocks and the
blocks at the start whose window reaches before the first token; the full
760M LM shape (window 2048) is checked on sampled heads and query rows."""
import numpy as np
import pytest
import torch

import chunk_test_b200 as ct
from lact_inputs import make_swa_inputs
from oracle import swa_oracle as so

pytestmark = pytest.mark.gpu


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-300))


def run(inp):
    dev = {k: v.cuda() for k, v in inp.items()}
    out = ct.swa_fwd(dev["q"], dev["k"], dev["v"], dev["q_scale"], dev["q_offset"], dev["k_scale"],
                     dev["k_offset"], WINDOW[0])
    assert ct.status() == ct.LACT_OK
    return out.float().cpu().numpy()


WINDOW = [0]


@pytest.mark.parametrize("B,H,T,d,window", [
    (1, 2, 512, 64, 128), (1, 2, 1024, 128, 256), (2, 1, 768, 256, 512), (1, 1, 384, 64, 1024),
    (1, 2, 640, 192, 128), (1, 1, 512, 512, 256),
])
def test_swa_parity(B, H, T, d, window):
    inp = make_swa_inputs(B, H, T, d, seed=B * 7 + T)
    WINDOW[0] = window
    got = run(inp)
    want = so.swa_layer(inp["q"], inp["k"], inp["v"], inp["q_scale"], inp["q_offset"], inp["k_scale"],
                        inp["k_offset"], window)
    err = rel_l2(got, want)
    assert err <= 2e-2, err
    print(f"swa B{B} H{H} T{T} d{d} w{window}: rel-L2 {err:.2e}")


def test_swa_window_one_block_is_causal_attention():
    """A window of the whole sequence is causal attention: compare with
    torch's own causal scaled-dot-product attention on the GPU in fp32 on the
    same (scaled, offset) inputs."""
    inp = make_swa_inputs(1, 2, 512, 128, seed=5)
    WINDOW[0] = 512
    got = run(inp)
    qp = inp["q"].float() * inp["q_scale"][None, :, None] + inp["q_offset"][None, :, None]
    kp = inp["k"].float() * inp["k_scale"][None, :, None] + inp["k_offset"][None, :, None]
    ref = torch.nn.functional.scaled_dot_product_attention(qp.cuda(), kp.cuda(), inp["v"].float().cuda(),
                                                           is_causal=True).cpu().numpy()
    assert rel_l2(got, ref) <= 2e-2


def test_swa_at_the_lm760m_shape_on_sampled_rows():
    B, H, T, d, window = 2, 6, 32768, 256, 2048
    inp = make_swa_inputs(B, H, T, d, seed=0)
    WINDOW[0] = window
    got = run(inp)
    rows = [0, 1, 127, 128, 2047, 2048, 2049, 16383, 32767]
    heads = [(0, 0), (1, 5)]
    want = so.swa_layer(inp["q"], inp["k"], inp["v"], inp["q_scale"], inp["q_offset"], inp["k_scale"],
                        inp["k_offset"], window, heads=heads, rows=rows)
    g = np.stack([got[b, h, rows] for b, h in heads])
    r = np.stack([want[b, h, rows] for b, h in heads])
    err = rel_l2(g, r)
    assert err <= 2e-2, err
    print(f"swa lm760m sampled: rel-L2 {err:.2e}")


@pytest.mark.parametrize("d", [128, 512])
def test_swa_with_wide_scales_and_offsets(d):
    """Offsets of order one and scales far from one.  The fused path (d up to
    256) drops the key offset, a constant per query in the scores, and folds
    the key scale into the queries; the materialised path (d 512) applies
    both to the keys.  The oracle applies them as defined."""
    inp = make_swa_inputs(1, 2, 768, d, seed=11)
    g = torch.Generator().manual_seed(12)
    shape = inp["q_scale"].shape
    inp["q_scale"] = 1.0 + 0.5 * torch.randn(shape, generator=g)
    inp["q_offset"] = torch.randn(shape, generator=g)
    inp["k_scale"] = 1.0 + 0.5 * torch.randn(shape, generator=g)
    inp["k_offset"] = 2.0 * torch.randn(shape, generator=g)
    WINDOW[0] = 256
    got = run(inp)
    want = so.swa_layer(inp["q"], inp["k"], inp["v"], inp["q_scale"], inp["q_offset"], inp["k_scale"],
                        inp["k_offset"], 256)
    err = rel_l2(got, want)
    assert err <= 2e-2, err
    print(f"swa wide scales d{d}: rel-L2 {err:.2e}")
