"""CPU fp64 oracle of the LaCT chunked fast-weight TTT layer (forward).

TEST INFRASTRUCTURE.  Only `tests/`, `__graft_entry__.smoke()` and the
`cpu_baseline` / reference legs of `bench.py` may import or call this
package.  It shares no code with the CUDA path (`chunk_test_b200`), and the
CUDA path never imports it.  It is plain, slow and written to be checked by
eye against the pages; numpy's fp64 matmul is the only library step it uses
(a matrix product *is* the sum over tokens of per-token outer products the
method defines).

Sources, cited by page title and section:
  [P1]  "LaCT架构核心思想解析" (gsyq.cn) -- §1.2 (q/k silu + L2 norm, momentum
        with a per-token beta, W <- L2_norm(W - M)), §2.1 (per-token softplus
        learning rates, one per fast-weight matrix), §2.2 (apply, then update,
        per chunk for causal inputs).
  [P2]  "大块测试时训练（LaCT）技术解析" (dpshk.com) -- §2.1 (update = sum of
        the gradient over the whole chunk, eqs. 4-5; apply = run the updated
        net on the queries, eq. 2), §2.2.1 (L2 weight normalisation, eq. 8;
        Muon = orthogonalised gradient, eqs. 9-10).
  [P3]  "LaCT：以大分块更新人工智能的临时记忆" (iplexlaw.co.kr) -- section
        「局部注意力与非线性记忆相互补充」 (SwiGLU memory of three matrices;
        loss = negative inner product of the net's output on the key with the
        value; per-token learning rates weight the chunk-summed gradient; GD,
        momentum and Muon rules, Muon via Newton-Schulz; L2 normalisation of
        the fast weights after each update) and section
        「更新顺序必须遵守信息可见范围」 (causal inputs apply the memory of the
        previous chunks first, then update; posed image sets update first,
        then read).

Readings where the pages are silent or garbled (each also listed in the
design notes):
  R1  the chunk gradient is a SUM over the chunk's tokens, not a mean [P2 §2.1].
  R2  W <- W - U with U derived from the gradient of L = -sum eta <f(k), v>.
  R3  lr column 0 -> W1, 1 -> W2, 2 -> W3 [P1 §2.1 gives only "(nh 3)"].
  R4  "row-wise" renorm runs over each matrix's input dimension: the dh rows
      of W1/W3 (length d) and the d rows of W2 (length dh), in the
      f_W(x) = W2 (silu(W1 x) * (W3 x)) convention, W1,W3 [dh,d], W2 [d,dh].
  R5  each row is scaled back to its norm from before the update.
  R6  momentum: M <- mean_{i in chunk}(beta_i) * M + G, M_0 = 0, U = M; one
      beta per token shared by the three matrices; M itself is not renormed.
  R7  Muon: U = NS5(G / (||G||_F + 1e-7)) with (a,b,c) = (3.4445, -4.7750,
      2.0315), the iteration run on the smaller Gram matrix; no momentum.
  R8  q/k L2 norm has no epsilon; an all-zero row stays zero.
  R9  a final chunk shorter than `chunk` is processed as it is.
  R10 with a single chunk the queries may have their own length Tq (the target
      views of a posed image set); with several chunks Tq must equal T.
  R13 the update mask has one flag per chunk, shared by every (batch, head)
      (the clean/noisy pattern is a property of the sequence).  A chunk whose
      flag is 0 is still applied in its place in the order, but skips the
      whole update -- gradient, rule, momentum and renorm -- so the state
      passes through unchanged (video: only clean-frame chunks update the
      memory, noisy chunks read what the earlier chunks wrote; [P3]
      「更新顺序必须遵守信息可见范围」, [P1 §3.2]).
  R14 the per-head output scale [P1 §2.1] is given as its values s (after
      the silu of the page's linear map), one per (batch, head, query
      token); the output row is s_t * f_W(q_t).
  R15 resuming a sequence across calls: the momentum may start from a given
      M_0 (zeros otherwise) and the final M is returned, so two calls split
      at a chunk boundary equal one call.
"""
from .lact_oracle import (  # noqa: F401
    APPLY_THEN_UPDATE, UPDATE_THEN_APPLY, RULE_GD, RULE_MOMENTUM, RULE_MUON,
    NS_COEFFS, NS_STEPS, NS_EPS,
    sigmoid, silu, silu_prime, qk_prologue, fast_net, chunk_gradient,
    newton_schulz5, renorm_rows, rule_step, ttt_head, ttt_head_state, ttt_layer, ttt_layer_ex,
    blas_threads,
)
from . import lact_oracle_bwd  # noqa: F401,E402
