"""Seeded synthetic inputs for the LaCT fast-weight TTT layer.

This module is shared by the oracle side (tests, the CPU baseline) and the CUDA
side (tests, bench).  It holds NONE of the layer's arithmetic: it only draws
random tensors with the shapes and distributions of the workloads described in
"Test-Time Training Done Right" (LaCT) -- the 760M / 3B language-model
configurations of its throughput table and the 48-view novel-view-synthesis
prefill of its Table 2 -- and casts them to the storage dtype.

Recipe (one torch CPU generator, seeded, drawn in this order, all fp32):
  q [B,H,Tq,d] ~ N(0,1), k [B,H,T,d] ~ N(0,1), v [B,H,T,d] ~ N(0,1),
  lr [B,H,T,3] = softplus(N(-5,1))          (per-token rates for W1, W2, W3),
  beta [B,H,T] = sigmoid(N(2,0.5))          (only drawn for the momentum rule),
  w1 [H,dh,d] ~ N(0,1/d), w2 [H,d,dh] ~ N(0,1/dh), w3 [H,dh,d] ~ N(0,1/d)
then q, k, v are cast to bf16 for the bf16 workloads.  The fast-weight
initialisation is one per head, shared by every batch element (a learned
initial state is a per-head parameter of the model).

Option inputs (their own generator, so the layer inputs above do not move):
  out_scale [B,H,Tq] = z * sigmoid(z), z ~ N(0,1): the per-head, per-token
      output factor, drawn as the silu of a unit-variance linear map of x
      (the multi-head fusion of "LaCT架构核心思想解析" §2.1);
  update mask: the chunk pattern of an autoregressive video sequence whose
      noisy chunks precede each clean one, [noisy x k, clean] repeated
      ("LaCT架构核心思想解析" §3.2: one noisy copy per clean chunk, or two in
      the teacher-forcing sequence);
  momentum (m1, m2, m3) in the final weights' layouts ~ N(0, 0.01/row length),
      a momentum handed in from an earlier call, or a final momentum's gradient.
"""
from __future__ import annotations

import dataclasses

import torch

F32, BF16 = "f32", "bf16"
APPLY_THEN_UPDATE, UPDATE_THEN_APPLY = 0, 1
RULE_GD, RULE_MOMENTUM, RULE_MUON = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int          # key/value tokens
    Tq: int         # query tokens (== T unless a single chunk covers T)
    d: int          # head dim
    dh: int         # fast-net hidden dim
    chunk: int
    order: int
    rule: int
    dtype: str

    @property
    def n_chunks(self) -> int:
        return -(-self.T // self.chunk)

    @property
    def tokens(self) -> int:
        """Tokens one forward processes: keys plus the separate queries of a
        single-chunk set input, or just the sequence for a causal input."""
        return self.B * (self.T if self.Tq == self.T else self.T + self.Tq)

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads.  1 is the tiny fp32 case; 2-4 are the 760M/3B language
# model shapes at 32K context; 5 is 48 views x 4096 patch tokens, one chunk.
WORKLOADS = {
    1: Workload("tiny-fp32-causal-gd", 1, 2, 2048, 2048, 64, 128, 512,
                APPLY_THEN_UPDATE, RULE_GD, F32),
    2: Workload("lm760m-32k-bf16-causal-gd", 2, 6, 32768, 32768, 256, 512, 2048,
                APPLY_THEN_UPDATE, RULE_GD, BF16),
    3: Workload("lm3b-32k-bf16-causal-momentum", 1, 8, 32768, 32768, 384, 768, 4096,
                APPLY_THEN_UPDATE, RULE_MOMENTUM, BF16),
    4: Workload("lm3b-32k-bf16-causal-muon", 1, 8, 32768, 32768, 384, 768, 4096,
                APPLY_THEN_UPDATE, RULE_MUON, BF16),
    5: Workload("nvs-48x4096-bf16-bidir-gd", 1, 12, 196608, 4096, 64, 128, 196608,
                UPDATE_THEN_APPLY, RULE_GD, BF16),
}


def make_inputs(w: Workload, seed: int = 0) -> dict:
    """Draw the inputs of workload `w` on the CPU.  Returns torch tensors:
    q,k,v in the workload dtype; lr, beta (or None), w1, w2, w3 in fp32."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((w.B, w.H, w.Tq, w.d), generator=g, dtype=torch.float32)
    k = torch.randn((w.B, w.H, w.T, w.d), generator=g, dtype=torch.float32)
    v = torch.randn((w.B, w.H, w.T, w.d), generator=g, dtype=torch.float32)
    lr = torch.nn.functional.softplus(
        torch.randn((w.B, w.H, w.T, 3), generator=g, dtype=torch.float32) - 5.0)
    beta = None
    if w.rule == RULE_MOMENTUM:
        beta = torch.sigmoid(
            2.0 + 0.5 * torch.randn((w.B, w.H, w.T), generator=g, dtype=torch.float32))
    w1 = torch.randn((w.H, w.dh, w.d), generator=g, dtype=torch.float32) / w.d ** 0.5
    w2 = torch.randn((w.H, w.d, w.dh), generator=g, dtype=torch.float32) / w.dh ** 0.5
    w3 = torch.randn((w.H, w.dh, w.d), generator=g, dtype=torch.float32) / w.d ** 0.5
    if w.dtype == BF16:
        q, k, v = q.bfloat16(), k.bfloat16(), v.bfloat16()
    return dict(q=q, k=k, v=v, lr=lr, beta=beta, w1=w1, w2=w2, w3=w3)


def head_slice(inp: dict, b: int, h: int) -> dict:
    """Inputs of one (batch, head) pair with B = H = 1 kept as leading dims."""
    out = {}
    for name in ("q", "k", "v", "lr", "beta"):
        t = inp[name]
        out[name] = None if t is None else t[b:b + 1, h:h + 1]
    for name in ("w1", "w2", "w3"):
        out[name] = inp[name][h:h + 1]
    return out


def make_out_scale(w: Workload, seed: int = 0) -> torch.Tensor:
    """out_scale [B,H,Tq] fp32 = silu of N(0,1) draws."""
    g = torch.Generator(device="cpu")
    g.manual_seed(10_000 + seed)
    z = torch.randn((w.B, w.H, w.Tq), generator=g, dtype=torch.float32)
    return z * torch.sigmoid(z)


def video_update_mask(n_chunks: int, noisy_per_clean: int = 1) -> list:
    """One flag per chunk: 0 for the noisy chunks, 1 for the clean chunk
    that follows them, in groups of noisy_per_clean + 1 chunks."""
    period = noisy_per_clean + 1
    return [1 if c % period == period - 1 else 0 for c in range(n_chunks)]


def make_output_grads(w: Workload, seed: int = 0, with_weights: bool = False):
    """Seeded gradients of a loss with respect to the layer's outputs, for
    the backward: dout [B,H,Tq,d] ~ N(0,1) in the workload dtype and, when
    asked, (dw1, dw2, dw3) ~ N(0,1) fp32 in the layouts of the final weights
    [B*H, dh, d], [B*H, d, dh], [B*H, dh, d]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(20_000 + seed)
    dout = torch.randn((w.B, w.H, w.Tq, w.d), generator=g, dtype=torch.float32)
    if w.dtype == BF16:
        dout = dout.bfloat16()
    dws = None
    if with_weights:
        BH = w.B * w.H
        dws = (torch.randn((BH, w.dh, w.d), generator=g), torch.randn((BH, w.d, w.dh), generator=g),
               torch.randn((BH, w.dh, w.d), generator=g))
    return dout, dws


def make_momentum(w: Workload, seed: int = 0):
    """A seeded momentum state (m1, m2, m3) fp32 in the layouts of the final
    weights [B*H, dh, d], [B*H, d, dh], [B*H, dh, d]: N(0,1) scaled by
    0.1/sqrt(row length), rows a tenth of the initial weights' norm (a
    momentum that leaves the renormalised rows well away from zero); used as
    a momentum handed in and as the gradient of a final momentum."""
    g = torch.Generator(device="cpu")
    g.manual_seed(40_000 + seed)
    BH = w.B * w.H
    return (0.1 * torch.randn((BH, w.dh, w.d), generator=g) / w.d ** 0.5,
            0.1 * torch.randn((BH, w.d, w.dh), generator=g) / w.dh ** 0.5,
            0.1 * torch.randn((BH, w.dh, w.d), generator=g) / w.d ** 0.5)


def make_swa_inputs(B: int, H: int, T: int, d: int, seed: int = 0) -> dict:
    """Seeded inputs of the sliding-window attention: q, k, v [B,H,T,d] ~ N(0,1)
    in bf16, and per head and channel q/k scales 1 + 0.1 N(0,1) and offsets
    0.1 N(0,1) [H,d] in fp32 (learnable parameters near their identity
    initialisation)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(30_000 + seed)
    q, k, v = (torch.randn((B, H, T, d), generator=g).bfloat16() for _ in range(3))
    qs = 1.0 + 0.1 * torch.randn((H, d), generator=g)
    qo = 0.1 * torch.randn((H, d), generator=g)
    ks = 1.0 + 0.1 * torch.randn((H, d), generator=g)
    ko = 0.1 * torch.randn((H, d), generator=g)
    return dict(q=q, k=k, v=v, q_scale=qs, q_offset=qo, k_scale=ks, k_offset=ko)
