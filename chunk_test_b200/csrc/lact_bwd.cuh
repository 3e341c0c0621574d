// lact_bwd.cuh -- host side of the layer's backward (lact_ttt_bwd), included
// by lact_api.cu after the forward's planning and launch helpers.
//
// The backward is the vector-Jacobian product of the forward:
//   1. the prologue and the updates of the forward are recomputed (the
//      outputs are not needed), keeping every state W^c, the momentum before
//      each update and the row norms |W'_r| before each renorm;
//   2. a reverse chunk loop carries A = dL/dW^c (and Bm = dL/dM^c): the
//      apply's backward at the state it read, then the renorm and rule
//      backward (k_renorm_bwd), then the gradient step's backward: the keys'
//      forward is recomputed at W^{c-1}, the second-order factors come from
//      k_hvp_elem, and the weight, key, value and rate gradients are their
//      contractions;
//   3. the prologue's backward gives dq and dk; the initial weights'
//      gradient is summed over the batch when the batch shares it.
// Muon: the recompute keeps each chunk's update direction S (its negated
// gradient, all three planes as [dh, d]); the reverse loop takes the renorm
// backward's gradient with respect to the update, re-runs the five
// Newton-Schulz steps on S keeping their iterates, and walks their
// vector-Jacobian product back to S (ns_keep, ns_vjp), in fp32 on the CUDA
// cores.  bf16 Muon problems take the fp32 path whole, on fp32 copies of
// their inputs: the iteration's Jacobian magnifies operand rounding (rounding
// only the chunk gradient to bf16 moves the exact backward by a few percent),
// so bf16 operands would not hold the bf16 tolerance.  The rule kernel applies the orthogonalised
// direction as GD applies S, so the renorm backward's GD output is the
// gradient with respect to that direction in GD's sign, and the (linear) VJP
// carries it to the gradient with respect to the chunk's gradient.
// Context parallelism (the all-reduce hook): every rank holds the same
// states, so dL/dW^c is the sum over the ranks of their own contributions
// (the apply's backward on their queries, the chunk gradient's
// second-order terms on their keys, their dL/dw_out) plus the part carried
// through the renorm backward, which every rank computes alike from the
// summed gradient.  The own contributions accumulate in Aloc, are summed
// over the ranks before each renorm backward (which reads and clears them)
// and once after the loop; the recompute sums each chunk's gradient and the
// beta sums and counts as the forward does.
// fp32 problems run every contraction as a batched k_simt_gemm over the B*H
// heads in fp32.  bf16 problems run them on the tensor cores (GemmOp, bf16
// operands through TMA, fp32 accumulation); the elementwise kernels write
// their results as bf16 operands, and the states, the gradients being
// accumulated (dL/dW, dk^, dq^, dv) and all reductions stay fp32.
#pragma once

#include "bwd_kernels.cuh"
#include "bwd_key_op.cuh"

namespace lact {

struct BwdInputs {
  const void *q, *k, *v;
  const float *lr, *beta, *w1, *w2, *w3;
  const void* dout;
  const float *dw1f, *dw2f, *dw3f;       // gradients of the final weights, or null
  const uint8_t* mask;
  const float* scale;
  float *dq, *dk, *dv, *dlr, *dbeta, *dw1, *dw2, *dw3, *dscale;
  const float* m0[3];    // momentum: M_0 (the layouts of w*_out), or null (zeros)
  const float* dmf[3];   // momentum: dL/dM_final, or null (zero)
  float* dm0[3];         // momentum: out dL/dM_0, or null
  lact_allreduce_fn allreduce;   // context parallelism: the ranks' sum, or null
  void* allreduce_user;
};

struct BwdBufs {
  float *q32, *k32, *v32, *do32, *dos32, *qh, *kh;
  float *hist, *mh, *Mm, *mnorm, *bbar;
  float *Z, *Pz, *E, *P;
  float *A, *Ap, *Gam, *Bm;
  float* Aloc;   // context parallelism: this rank's own contributions to dL/dW
  float *dqh, *dkh, *ofull, *part;
  // bf16 problems (tensor-core contractions): bf16 operands
  __nv_bfloat16 *qh16, *kh16, *dos16, *hist16, *op16, *Gam16;
  __nv_bfloat16 *Bk, *Bv;   // stacked operands of the merged contractions
  // Muon: per-chunk directions [nch][3BH][dh][d]; Newton-Schulz iterates
  // X0..X5 (planes), Gram matrices A0..A4 and polynomials B0..B4
  // ([3BH][d][d] each), two [d][d] temporaries, two VJP planes, the update in
  // the weights' layout, the norms' partial sums
  float *Phist, *nsX, *nsA, *nsB, *nsT, *nsY, *dir, *nspart;
  int64_t zr;   // rows per head of the per-chunk [rows][dh] planes
};

static int64_t rule_rows(const Dims& D) { return 2 * D.BH * D.dh + D.BH * D.d; }

// bf16 problems run their contractions on the tensor cores, except under
// Muon (fp32 on the CUDA cores, see above).
static bool bwd_on_tc(const Dims& D) { return D.dtype == LACT_BF16 && D.rule != LACT_RULE_MUON; }

static void plan_bwd(const Dims& D, Bump& bp, BwdBufs& b) {
  std::memset(&b, 0, sizeof(b));
  const int64_t planes = 3 * D.BH * D.dh * D.d;
  const int64_t nq = D.BH * D.Tq * D.d, nk = D.BH * D.T * D.d;
  const bool bf = bwd_on_tc(D);
  const bool mom = D.rule == LACT_RULE_MOMENTUM;
  b.zr = std::max<int64_t>(D.chunk, D.nch == 1 ? D.Tq : D.chunk);
  const int64_t zpl = D.BH * b.zr * D.dh;
  if (bf) {
    b.do32 = bp.take<float>(nq);         // dout, for the scale's gradient
    b.qh16 = bp.take<__nv_bfloat16>(nq);
    b.kh16 = bp.take<__nv_bfloat16>(nk);
    b.dos16 = bp.take<__nv_bfloat16>(nq);
    b.hist16 = bp.take<__nv_bfloat16>((D.nch + 1) * planes);
    b.op16 = bp.take<__nv_bfloat16>(6 * zpl);
    b.Gam16 = bp.take<__nv_bfloat16>(planes);
    b.Bk = bp.take<__nv_bfloat16>(4 * D.BH * D.dh * D.d);
    b.Bv = bp.take<__nv_bfloat16>(2 * D.BH * D.dh * D.d);
  } else {
    if (D.dtype == LACT_BF16) {   // fp32 copies of the inputs
      b.q32 = bp.take<float>(nq);
      b.k32 = bp.take<float>(nk);
      b.v32 = bp.take<float>(nk);
      b.do32 = bp.take<float>(nq);
    }
    b.dos32 = bp.take<float>(nq);
    b.qh = bp.take<float>(nq);
    b.kh = bp.take<float>(nk);
    b.E = bp.take<float>(3 * zpl);
    b.Gam = bp.take<float>(planes);
  }
  b.hist = bp.take<float>((D.nch + 1) * planes);
  if (mom) {
    b.mh = bp.take<float>(D.nch * planes);
    b.Mm = bp.take<float>(planes);
    b.bbar = bp.take<float>(2 * D.BH * D.nch);   // means, then (context parallel) token counts
    b.Bm = bp.take<float>(planes);
    b.part = bp.take<float>(rule_rows(D));
  }
  b.mnorm = bp.take<float>(D.nch * rule_rows(D));
  if (D.rule == LACT_RULE_MUON) {
    const int64_t grams = 3 * D.BH * D.d * D.d;
    b.Phist = bp.take<float>(D.nch * planes);
    b.nsX = bp.take<float>(6 * planes);
    b.nsA = bp.take<float>(5 * grams);
    b.nsB = bp.take<float>(5 * grams);
    b.nsT = bp.take<float>(2 * grams);
    b.nsY = bp.take<float>(2 * planes);
    b.dir = bp.take<float>(planes);
    b.nspart = bp.take<float>(3 * D.BH * kNsBlocks);
  }
  if (!bf) {
    b.Z = bp.take<float>(3 * zpl);
    b.Pz = bp.take<float>(3 * zpl);
  }
  b.P = bp.take<float>(planes);
  b.A = bp.take<float>(planes);
  b.Aloc = bp.take<float>(planes);
  b.Ap = bp.take<float>(planes);
  b.dqh = bp.take<float>(nq);
  b.dkh = bp.take<float>(nk);
  b.ofull = bp.take<float>(nq);
}

static size_t bwd_workspace_bytes(const Dims& D) {
  Bump bp{0, 0};
  BwdBufs b;
  plan_bwd(D, bp, b);
  return static_cast<size_t>(rup(static_cast<int64_t>(bp.off), 256));
}

static unsigned grid_for(int64_t n, int per_thread = 1) {
  return static_cast<unsigned>(std::min<int64_t>(std::max<int64_t>(cdiv(n, 256LL * per_thread), 1), 148 * 32));
}

// ------------------------------------------------------------------ Muon
// C[item] = alpha * A(item) B(item)^T + beta * cin over the 3 BH matrices,
// fp32 on the CUDA cores (k_simt_gemm indexing).
static void ns_gemm(const Dims& D, Launcher& L, cudaStream_t st, const float* A, int64_t a_item, int64_t a_m,
                    int64_t a_k, const float* B, int64_t b_item, int64_t b_n, int64_t b_k, int M, int N, int K,
                    float alpha, float beta, const float* cin, float* out, int64_t out_item, int64_t ld) {
  L(K_SIMT_GEMM, [&] {
    SimtGemmParams s = simt_params();
    s.A = A; s.a_item = a_item; s.a_m = a_m; s.a_k = a_k;
    s.B = B; s.b_item = b_item; s.b_n = b_n; s.b_k = b_k;
    s.M = M; s.N = N; s.K = K; s.alpha = alpha; s.beta = beta; s.cin = cin;
    s.outf = out; s.item_stride = out_item; s.ld = ld;
    return simt(s, static_cast<int>(3 * D.BH), st);
  });
}

// W2's planes between the weights' layout [d, dh] and the Newton-Schulz
// layout [dh, d] (the other two planes are copied): dst = src with plane
// group 1 transposed; `to_ns` picks the direction.
static void ns_relayout(const Dims& D, Launcher& L, cudaStream_t st, const float* src, float* dst, bool to_ns) {
  const int64_t plane = D.dh * D.d, jst = D.BH * plane;
  if (!L.dry && L.err == LACT_OK) {
    if (cudaMemcpyAsync(dst, src, static_cast<size_t>(jst) * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(dst + 2 * jst, src + 2 * jst, static_cast<size_t>(jst) * 4, cudaMemcpyDeviceToDevice,
                        st) != cudaSuccess)
      L.err = LACT_ECUDA;
  }
  const int rows = static_cast<int>(to_ns ? D.d : D.dh), cols = static_cast<int>(to_ns ? D.dh : D.d);
  L(K_BWD_ELEM, [&] {
    (void)launch_pdl(k_transpose_planes, dim3(cdiv(cols, 32), cdiv(rows, 32), D.BH), dim3(32, 8), 0, st,
                     src + jst, dst + jst, rows, cols);
    return cudaGetLastError();
  });
}

// The Newton-Schulz steps on S ([3BH][dh][d]), keeping X0..X5, A0..A4 and
// B0..B4 and the norms' partial sums:
//   X0 = S / (||S||_F + eps);  A = X^T X;  B = b A + c A A;  X <- a X + X B
// (the forward's arithmetic, "大块测试时训练（LaCT）技术解析" §2.2.1).
static void ns_keep(const Dims& D, const BwdBufs& b, const float* S, cudaStream_t st, Launcher& L) {
  const int d = static_cast<int>(D.d), dh = static_cast<int>(D.dh), n3 = static_cast<int>(3 * D.BH);
  const int64_t plane = D.dh * D.d, planes = 3 * D.BH * plane, dd = D.d * D.d, grams = n3 * dd;
  L(K_NS_SUMSQ, [&] {
    (void)launch_pdl(k_ns_sumsq, dim3(kNsBlocks, n3), 256, 0, st, S, 1, planes, plane, b.nsX, b.nspart);
    return cudaGetLastError();
  });
  L(K_NS_SCALE, [&] {
    (void)launch_pdl(k_ns_scale, dim3(kNsBlocks, n3), 256, 0, st, b.nsX, static_cast<__nv_bfloat16*>(nullptr),
                     static_cast<__nv_bfloat16*>(nullptr), plane, static_cast<const float*>(b.nspart), kNsBlocks,
                     kNsEps);
    return cudaGetLastError();
  });
  for (int k = 0; k < kNsSteps; ++k) {
    const float* X = b.nsX + k * planes;
    float* A = b.nsA + k * grams;
    float* B = b.nsB + k * grams;
    ns_gemm(D, L, st, X, plane, 1, d, X, plane, 1, d, d, d, dh, 1.0f, 0.0f, nullptr, A, dd, d);        // X^T X
    ns_gemm(D, L, st, A, dd, d, 1, A, dd, 1, d, d, d, d, kNsC, kNsB, A, B, dd, d);                       // c A A + b A
    ns_gemm(D, L, st, X, plane, d, 1, B, dd, 1, d, dh, d, d, 1.0f, kNsA, X, b.nsX + (k + 1) * planes, plane,
            d);                                                                                          // X B + a X
  }
}

// dL/dS = VJP of S -> X5 at the iterates ns_keep kept, applied to Y
// (= dL/dX5, [3BH][dh][d], b.nsY; overwritten), written to `out`.  One step
// back, with Y = dL/dX' for X' = a X + X B, B = b A + c A A, A = X^T X:
//   dB = X^T Y,  dA = b dB + c (dB A + A dB),  dL/dX = a Y + Y B + X (dA + dA^T)
// (A and B are symmetric).  Then the normalisation's VJP (k_ns_norm_vjp).
static void ns_vjp(const Dims& D, const BwdBufs& b, const float* S, float* out, cudaStream_t st, Launcher& L) {
  const int d = static_cast<int>(D.d), dh = static_cast<int>(D.dh), n3 = static_cast<int>(3 * D.BH);
  const int64_t plane = D.dh * D.d, planes = 3 * D.BH * plane, dd = D.d * D.d, grams = n3 * dd;
  float* Y = b.nsY;
  float* Yn = b.nsY + planes;
  float* dB = b.nsT;
  float* T = b.nsT + grams;
  for (int k = kNsSteps - 1; k >= 0; --k) {
    const float* X = b.nsX + k * planes;
    const float* A = b.nsA + k * grams;
    const float* B = b.nsB + k * grams;
    ns_gemm(D, L, st, X, plane, 1, d, Y, plane, 1, d, d, d, dh, 1.0f, 0.0f, nullptr, dB, dd, d);       // X^T Y
    ns_gemm(D, L, st, dB, dd, d, 1, A, dd, 1, d, d, d, d, kNsC, kNsB, dB, T, dd, d);                    // c dB A + b dB
    ns_gemm(D, L, st, A, dd, d, 1, dB, dd, 1, d, d, d, d, kNsC, 1.0f, T, T, dd, d);                     // + c A dB
    L(K_BWD_ELEM, [&] {
      (void)launch_pdl(k_sym_add, grid_for(grams, 1), 256, 0, st, T, d, static_cast<int64_t>(n3));
      return cudaGetLastError();
    });
    ns_gemm(D, L, st, Y, plane, d, 1, B, dd, 1, d, dh, d, d, 1.0f, kNsA, Y, Yn, plane, d);              // Y B + a Y
    ns_gemm(D, L, st, X, plane, d, 1, T, dd, 1, d, dh, d, d, 1.0f, 1.0f, Yn, Yn, plane, d);             // + X (dA + dA^T)
    std::swap(Y, Yn);
  }
  L(K_BWD_ELEM, [&] {
    (void)launch_pdl(k_ns_norm_vjp, static_cast<unsigned>(n3), 1024, 0, st, S, static_cast<const float*>(Y),
                     static_cast<const float*>(b.nspart), kNsBlocks, kNsEps, plane, out);
    return cudaGetLastError();
  });
}

// Forward recompute, Muon: the chunk's direction S (= b.P, [dh, d] planes)
// kept for the reverse loop, and its orthogonalised update in the weights'
// layout (b.dir) for the rule kernel.
static void muon_forward_step(const Dims& D, const BwdBufs& b, int64_t c, cudaStream_t st, Launcher& L) {
  const int64_t planes = 3 * D.BH * D.dh * D.d;
  float* S = b.Phist + c * planes;
  if (!L.dry && L.err == LACT_OK &&
      cudaMemcpyAsync(S, b.P, static_cast<size_t>(planes) * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    L.err = LACT_ECUDA;
  ns_keep(D, b, S, st, L);
  ns_relayout(D, L, st, b.nsX + kNsSteps * planes, b.dir, false);
}

// Reverse loop, Muon: b.Gam holds the gradient with respect to the update
// (the renorm backward's GD output, weights' layout); replaced by the
// gradient with respect to the chunk's negated gradient S.
static void muon_backward_step(const Dims& D, const BwdBufs& b, int64_t c, cudaStream_t st, Launcher& L) {
  const int64_t planes = 3 * D.BH * D.dh * D.d;
  const float* S = b.Phist + c * planes;
  ns_relayout(D, L, st, b.Gam, b.nsY, true);
  ns_keep(D, b, S, st, L);
  ns_vjp(D, b, S, b.dir, st, L);
  ns_relayout(D, L, st, b.dir, b.Gam, false);
}

// fp32 problems: every contraction on the CUDA cores in fp32.
static void run_bwd_f32(const Dims& D, const BwdBufs& b, const BwdInputs& in, cudaStream_t st, Launcher& L) {
  L.st = st;
  const bool mom = D.rule == LACT_RULE_MOMENTUM;
  const bool muon = D.rule == LACT_RULE_MUON;
  const int BH = static_cast<int>(D.BH), d = static_cast<int>(D.d), dh = static_cast<int>(D.dh);
  const int64_t plane = D.dh * D.d, planes = 3 * D.BH * plane, jst = D.BH * plane;
  const int64_t nq = D.BH * D.Tq * D.d, nk = D.BH * D.T * D.d;
  const int64_t zr = b.zr, zpl = D.BH * zr * D.dh, rows_all = rule_rows(D);
  auto memop = [&](cudaError_t e) {
    if (!L.dry && L.err == LACT_OK && e != cudaSuccess) L.err = LACT_ECUDA;
  };
  auto zero = [&](void* p, int64_t bytes) {
    if (!L.dry && p) memop(cudaMemsetAsync(p, 0, static_cast<size_t>(bytes), st));
  };
  auto copy = [&](void* dst, const void* src, int64_t bytes) {
    if (!L.dry) memop(cudaMemcpyAsync(dst, src, static_cast<size_t>(bytes), cudaMemcpyDeviceToDevice, st));
  };
  const bool cp = in.allreduce != nullptr;
  auto reduce = [&](float* data, int64_t count) {   // in place over the ranks, op SUM
    if (!cp || L.dry || L.err != LACT_OK) return;
    if (in.allreduce(data, count, LACT_REDUCE_SUM, static_cast<void*>(st), in.allreduce_user) != 0)
      L.err = LACT_ECOMM;
  };
  // one batched fp32 GEMM over the heads (see k_simt_gemm for the indexing)
  auto gemm = [&](const float* A, int64_t a_item, int64_t a_m, int64_t a_k, const float* B, int64_t b_item,
                  int64_t b_n, int64_t b_k, int M, int N, int K, float* out, int64_t out_item, int64_t ld,
                  bool accumulate) {
    L(K_SIMT_GEMM, [&] {
      SimtGemmParams s = simt_params();
      s.A = A; s.a_item = a_item; s.a_m = a_m; s.a_k = a_k;
      s.B = B; s.b_item = b_item; s.b_n = b_n; s.b_k = b_k;
      s.M = M; s.N = N; s.K = K;
      s.outf = out; s.item_stride = out_item; s.ld = ld;
      if (accumulate) { s.beta = 1.0f; s.cin = out; }
      return simt(s, BH, st);
    });
  };

  // ---- fp32 inputs (copies of bf16 ones), the scaled output gradient, zeroed accumulators
  const float* q32 = static_cast<const float*>(in.q);
  const float* k32 = static_cast<const float*>(in.k);
  const float* v32 = static_cast<const float*>(in.v);
  const float* do32 = static_cast<const float*>(in.dout);
  if (D.dtype == LACT_BF16) {
    const void* src[4] = {in.q, in.k, in.v, in.dout};
    float* dst[4] = {b.q32, b.k32, b.v32, b.do32};
    const int64_t n[4] = {nq, nk, nk, nq};
    for (int i = 0; i < 4; ++i)
      L(K_BWD_ELEM, [&] {
        (void)launch_pdl(k_bf16_to_f32, grid_for(n[i], 4), 256, 0, st, static_cast<const __nv_bfloat16*>(src[i]),
                         dst[i], n[i]);
        return cudaGetLastError();
      });
    q32 = b.q32; k32 = b.k32; v32 = b.v32; do32 = b.do32;
  }
  const float* dos = do32;
  if (in.scale) {
    L(K_BWD_ELEM, [&] {
      (void)launch_pdl(k_scale_rows, grid_for(nq, 4), 256, 0, st, do32, in.scale, b.dos32, D.BH * D.Tq, d);
      return cudaGetLastError();
    });
    dos = b.dos32;
  }
  zero(in.dlr, D.BH * D.T * 3 * 4);
  if (mom) zero(in.dbeta, D.BH * D.T * 4);
  zero(in.dv, nk * 4);
  zero(b.dqh, nq * 4);
  zero(b.dkh, nk * 4);
  if (mom) {   // dL/dM after the last chunk
    for (int j = 0; j < 3; ++j) {
      if (in.dmf[j]) copy(b.Bm + j * jst, in.dmf[j], jst * 4);
      else zero(b.Bm + j * jst, jst * 4);
    }
  }
  if (mom && in.dmf[0]) reduce(b.Bm, planes);   // the ranks' gradients of the final momentum
  const float* dwf[3] = {in.dw1f, in.dw2f, in.dw3f};
  float* dw_init = cp ? b.Aloc : b.A;   // dL/dw_out is this rank's own
  if (cp) zero(b.A, planes * 4);
  for (int j = 0; j < 3; ++j) {
    if (dwf[j]) copy(dw_init + j * jst, dwf[j], jst * 4);
    else zero(dw_init + j * jst, jst * 4);
  }

  // ---- forward recompute: q^, k^ (fp32), initial state, beta means
  L(K_PROLOGUE, [&] {
    const int64_t rows = D.BH * D.Tq + D.BH * D.T;
    constexpr int ROWS = 4;
    const unsigned blocks = static_cast<unsigned>(cdiv(cdiv(rows, ROWS) * 32, 256));
    if (D.d % 4 == 0)
      (void)launch_pdl(k_qk_prologue<float, 4, 32, 4, ROWS>, blocks, 256, 0, st, q32, b.qh, D.BH * D.Tq, k32,
                       b.kh, D.BH * D.T, d, static_cast<float*>(nullptr));
    else
      (void)launch_pdl(k_qk_prologue<float, 1, 32, 16, ROWS>, blocks, 256, 0, st, q32, b.qh, D.BH * D.Tq, k32,
                       b.kh, D.BH * D.T, d, static_cast<float*>(nullptr));
    return cudaGetLastError();
  });
  L(K_INIT, [&] {
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(cdiv(planes, 1024), 148 * 16));
    (void)launch_pdl(k_init_state, blocks, 256, 0, st, in.w1, in.w2, in.w3, static_cast<int>(D.H), D.w_shared,
                     BH, d, dh, b.hist, static_cast<__nv_bfloat16*>(nullptr),
                     static_cast<__nv_bfloat16*>(nullptr), mom ? b.Mm : nullptr,
                     in.m0[0], in.m0[1], in.m0[2]);
    return cudaGetLastError();
  });
  if (mom) {   // per-chunk beta means (context parallel: sums and counts over the ranks)
    const int64_t w = D.BH * D.nch;
    L(K_BETA_MEAN, [&] {
      (void)launch_pdl(k_beta_mean, static_cast<unsigned>(cdiv(w * 32, 256)), 256, 0, st, in.beta, BH, D.T,
                       D.chunk, static_cast<int>(D.nch), b.bbar, cp ? 1 : 0);
      return cudaGetLastError();
    });
    if (cp) {
      reduce(b.bbar, 2 * w);
      L(K_BETA_MEAN, [&] {
        (void)launch_pdl(k_beta_div, static_cast<unsigned>(cdiv(w, 256)), 256, 0, st, b.bbar, w);
        return cudaGetLastError();
      });
    }
  }
  // the keys' forward at state W: Z = (k^ W1^T, v W2, k^ W3^T), rows of chunk c
  auto key_forward = [&](const float* W, int64_t c0, int nc, float* Zout) {
    for (int j = 0; j < 3; ++j)
      gemm((j == 1 ? v32 : b.kh) + c0 * d, D.T * D.d, d, 1, W + j * jst, plane, j == 1 ? 1 : d,
           j == 1 ? dh : 1, nc, dh, d, Zout + j * zpl, zr * D.dh, dh, false);
  };
  for (int64_t c = 0; c < D.nch; ++c) {
    const int64_t c0 = c * D.chunk;
    const int nc = static_cast<int>(std::min(c0 + D.chunk, D.T) - c0);
    float* Wc = b.hist + c * planes;
    float* Wn = b.hist + (c + 1) * planes;
    copy(Wn, Wc, planes * 4);
    if (in.mask && in.mask[c] == 0) continue;
    if (mom) copy(b.mh + c * planes, b.Mm, planes * 4);
    key_forward(Wc, c0, nc, b.Z);
    L(K_FWD_ELEM_F32, [&] {
      (void)launch_pdl(k_fwd_elem_f32, static_cast<unsigned>(cdiv(zpl, 256)), 256, 0, st, b.Z, BH, zr, dh, nc,
                       1, in.lr, D.T, c0, b.E);
      return cudaGetLastError();
    });
    L(K_SIMT_GEMM, [&] {   // -G = E^T [k^, v, k^], W2's plane stored transposed
      SimtGemmParams s = simt_params();
      s.A = b.E; s.a_item = zr * D.dh; s.a_m = 1; s.a_k = dh;
      s.B = b.kh + c0 * d; s.B2 = v32 + c0 * d; s.b_item = D.T * D.d; s.b_n = 1; s.b_k = d;
      s.zb_mod = BH; s.alt_b = 1;
      s.M = dh; s.N = d; s.K = nc;
      s.outf = b.P; s.item_stride = plane; s.ld = d;
      if (!muon) { s.tr_group = 1; s.tr_mod = BH; s.ld_t = dh; }   // Muon keeps [dh, d] planes
      return simt(s, 3 * BH, st);
    });
    reduce(b.P, planes);   // the whole chunk's gradient
    if (muon) muon_forward_step(D, b, c, st, L);
    L(K_RULE, [&] {
      RuleParams r;
      std::memset(&r, 0, sizeof(r));
      r.Wm = Wn; r.S = muon ? b.dir : b.P; r.splits = 1; r.split_stride = planes;
      r.Mm = mom ? b.Mm : nullptr; r.beta_bar = b.bbar; r.nch = static_cast<int>(D.nch);
      r.chunk_idx = static_cast<int>(c); r.rule = D.rule; r.BH = BH; r.dh = dh; r.d = d;
      r.nrm_out = b.mnorm + c * rows_all;
      (void)launch_pdl(k_rule_renorm, static_cast<unsigned>(cdiv(rows_all * 32, 256)), 256, 0, st, r);
      return cudaGetLastError();
    });
  }

  // ---- reverse chunk loop
  float* A = b.A;
  float* Ap = b.Ap;
  auto apply_bwd = [&](const float* W, int64_t qr0, int nq_c) {
    // Zq = (q^ W1^T, dO W2, q^ W3^T) -> (dz1, hq, dz3)
    for (int j = 0; j < 3; j += 2)
      gemm(b.qh + qr0 * d, D.Tq * D.d, d, 1, W + j * jst, plane, d, 1, nq_c, dh, d, b.Z + j * zpl, zr * D.dh, dh,
           false);
    gemm(dos + qr0 * d, D.Tq * D.d, d, 1, W + jst, plane, 1, dh, nq_c, dh, d, b.Z + zpl, zr * D.dh, dh, false);
    L(K_BWD_ELEM, [&] {
      (void)launch_pdl(k_apply_bwd_elem, grid_for(zpl, 4), 256, 0, st, b.Z, zpl);
      return cudaGetLastError();
    });
    // dW1 += dz1^T q^, dW3 += dz3^T q^, dW2 += dO^T hq (this rank's own part)
    float* Aq = cp ? b.Aloc : A;
    for (int j = 0; j < 3; j += 2)
      gemm(b.Z + j * zpl, zr * D.dh, 1, dh, b.qh + qr0 * d, D.Tq * D.d, 1, d, dh, d, nq_c, Aq + j * jst, plane, d,
           true);
    gemm(dos + qr0 * d, D.Tq * D.d, 1, d, b.Z + zpl, zr * D.dh, 1, dh, d, dh, nq_c, Aq + jst, plane, dh, true);
    // dq^ += dz1 W1 + dz3 W3
    for (int j = 0; j < 3; j += 2)
      gemm(b.Z + j * zpl, zr * D.dh, dh, 1, W + j * jst, plane, 1, d, nq_c, d, dh, b.dqh + qr0 * d, D.Tq * D.d, d,
           true);
    if (in.scale)   // the unscaled output, for the scale's gradient
      gemm(b.Z + zpl, zr * D.dh, dh, 1, W + jst, plane, dh, 1, nq_c, d, dh, b.ofull + qr0 * d, D.Tq * D.d, d,
           false);
  };
  for (int64_t c = D.nch - 1; c >= 0; --c) {
    const int64_t c0 = c * D.chunk;
    const int nc = static_cast<int>(std::min(c0 + D.chunk, D.T) - c0);
    const int64_t qr0 = D.nch == 1 ? 0 : c0;
    const int nq_c = static_cast<int>(D.nch == 1 ? D.Tq : nc);
    const float* Wp = b.hist + c * planes;
    const float* Wc = b.hist + (c + 1) * planes;
    const bool upd = !in.mask || in.mask[c] != 0;
    if (D.order == LACT_UPDATE_THEN_APPLY) apply_bwd(Wc, qr0, nq_c);
    if (upd) {
      reduce(b.Aloc, planes);   // the ranks' own contributions to dL/dW^c
      L(K_BWD_ELEM, [&] {
        RenormBwdParams r;
        std::memset(&r, 0, sizeof(r));
        r.A = A; r.A2 = cp ? b.Aloc : nullptr; r.Wc = Wc; r.Wp = Wp; r.mnorm = b.mnorm + c * rows_all; r.Gam = b.Gam; r.Ap = Ap;
        r.rule = muon ? LACT_RULE_GD : D.rule; r.Bm = b.Bm; r.Mprev = mom ? b.mh + c * planes : nullptr;
        r.beta_bar = b.bbar; r.nch = static_cast<int>(D.nch); r.chunk_idx = static_cast<int>(c); r.part = b.part;
        r.BH = BH; r.dh = dh; r.d = d;
        (void)launch_pdl(k_renorm_bwd, static_cast<unsigned>(cdiv(rows_all * 32, 256)), 256, 0, st, r);
        return cudaGetLastError();
      });
      if (muon) muon_backward_step(D, b, c, st, L);   // through the Newton-Schulz steps
      if (mom)
        L(K_BWD_ELEM, [&] {
          (void)launch_pdl(k_head_dbeta, static_cast<unsigned>(BH), 256, 0, st, b.part, BH, dh, d, D.T, c0, nc,
                           cp ? static_cast<const float*>(b.bbar + D.BH * D.nch + c) : nullptr, D.nch, in.dbeta);
          return cudaGetLastError();
        });
      // the keys' forward at W^{c-1}, and (p, q, r) = (k^ Gam1^T, v Gam2, k^ Gam3^T)
      key_forward(Wp, c0, nc, b.Z);
      key_forward(b.Gam, c0, nc, b.Pz);
      L(K_BWD_ELEM, [&] {
        (void)launch_pdl(k_hvp_elem, static_cast<unsigned>(cdiv(D.BH * nc * 32, 256)), 256, 0, st, b.Z, b.Pz, BH,
                         zr, dh, nc, in.lr, D.T, c0, in.dlr);
        return cudaGetLastError();
      });
      // dW1 += dz1^T k^, dW3 += dz3^T k^, dW2 += v^T du (this rank's own part)
      float* Ak = cp ? b.Aloc : Ap;
      for (int j = 0; j < 3; j += 2)
        gemm(b.Z + j * zpl, zr * D.dh, 1, dh, b.kh + c0 * d, D.T * D.d, 1, d, dh, d, nc, Ak + j * jst, plane, d,
             true);
      gemm(v32 + c0 * d, D.T * D.d, 1, d, b.Z + zpl, zr * D.dh, 1, dh, d, dh, nc, Ak + jst, plane, dh, true);
      // dk^ += dz1 W1 + dz3 W3 + dp Gam1 + dr Gam3
      for (int j = 0; j < 3; j += 2) {
        gemm(b.Z + j * zpl, zr * D.dh, dh, 1, Wp + j * jst, plane, 1, d, nc, d, dh, b.dkh + c0 * d, D.T * D.d, d,
             true);
        gemm(b.Pz + j * zpl, zr * D.dh, dh, 1, b.Gam + j * jst, plane, 1, d, nc, d, dh, b.dkh + c0 * d, D.T * D.d,
             d, true);
      }
      // dv += du W2^T + dq Gam2^T
      gemm(b.Z + zpl, zr * D.dh, dh, 1, Wp + jst, plane, dh, 1, nc, d, dh, in.dv + c0 * d, D.T * D.d, d, true);
      gemm(b.Pz + zpl, zr * D.dh, dh, 1, b.Gam + jst, plane, dh, 1, nc, d, dh, in.dv + c0 * d, D.T * D.d, d, true);
      std::swap(A, Ap);
    }
    if (D.order == LACT_APPLY_THEN_UPDATE) apply_bwd(Wp, qr0, nq_c);
  }

  // ---- prologue backward, the scale's gradient, the initial weights' gradient
  L(K_BWD_ELEM, [&] {
    (void)launch_pdl(k_prologue_bwd, static_cast<unsigned>(cdiv(D.BH * D.Tq * 32, 256)), 256, 0, st, q32, b.dqh,
                     in.dq, D.BH * D.Tq, d);
    return cudaGetLastError();
  });
  L(K_BWD_ELEM, [&] {
    (void)launch_pdl(k_prologue_bwd, static_cast<unsigned>(cdiv(D.BH * D.T * 32, 256)), 256, 0, st, k32, b.dkh,
                     in.dk, D.BH * D.T, d);
    return cudaGetLastError();
  });
  if (in.scale)
    L(K_BWD_ELEM, [&] {
      (void)launch_pdl(k_rowdot, static_cast<unsigned>(cdiv(D.BH * D.Tq * 32, 256)), 256, 0, st, do32, b.ofull,
                       in.dscale, D.BH * D.Tq, d);
      return cudaGetLastError();
    });
  if (cp) {   // the own contributions left after chunk 0, summed over the ranks
    reduce(b.Aloc, planes);
    L(K_BWD_ELEM, [&] {
      (void)launch_pdl(k_add_planes, grid_for(planes, 4), 256, 0, st, A, static_cast<const float*>(b.Aloc), planes);
      return cudaGetLastError();
    });
  }
  L(K_BWD_ELEM, [&] {
    (void)launch_pdl(k_sum_batch, grid_for(planes, 4), 256, 0, st, static_cast<const float*>(A),
                     static_cast<int>(D.B), static_cast<int>(D.H), plane, D.w_shared, in.dw1, in.dw2, in.dw3);
    return cudaGetLastError();
  });
  if (mom)   // after chunk 0, B holds dL/dM_0
    for (int j = 0; j < 3; ++j)
      if (in.dm0[j]) copy(in.dm0[j], b.Bm + j * jst, jst * 4);
}

// One bf16 operand: a dense [batch][rows][inner] tensor.
struct Opnd {
  const void* p;
  int64_t inner, rows, batch;
};

static int pick_bn(int64_t n) {
  if (n <= 256) return static_cast<int>(n);
  if (n % 256 == 0) return 256;
  if (n % 192 == 0) return 192;
  if (n % 128 == 0) return 128;
  return 64;
}

// bf16 problems: the contractions on the tensor cores.
static void run_bwd_tc(const Dims& D, const BwdBufs& b, const BwdInputs& in, cudaStream_t st, Launcher& L) {
  L.st = st;
  const bool mom = D.rule == LACT_RULE_MOMENTUM;
  const int BH = static_cast<int>(D.BH), d = static_cast<int>(D.d), dh = static_cast<int>(D.dh);
  const int64_t plane = D.dh * D.d, planes = 3 * D.BH * plane, jst = D.BH * plane;
  const int64_t nq = D.BH * D.Tq * D.d, nk = D.BH * D.T * D.d;
  const int64_t zr = b.zr, zpl = D.BH * zr * D.dh, rows_all = rule_rows(D);
  using B16 = __nv_bfloat16;
  auto memop = [&](cudaError_t e) {
    if (!L.dry && L.err == LACT_OK && e != cudaSuccess) L.err = LACT_ECUDA;
  };
  auto zero = [&](void* p, int64_t bytes) {
    if (!L.dry && p) memop(cudaMemsetAsync(p, 0, static_cast<size_t>(bytes), st));
  };
  auto copy = [&](void* dst, const void* src, int64_t bytes) {
    if (!L.dry) memop(cudaMemcpyAsync(dst, src, static_cast<size_t>(bytes), cudaMemcpyDeviceToDevice, st));
  };
  const bool cp = in.allreduce != nullptr;
  auto reduce = [&](float* data, int64_t count) {   // in place over the ranks, op SUM
    if (!cp || L.dry || L.err != LACT_OK) return;
    if (in.allreduce(data, count, LACT_REDUCE_SUM, static_cast<void*>(st), in.allreduce_user) != 0)
      L.err = LACT_ECOMM;
  };
  // out[item] (+)= A(item) B(item)^T with A [M x K], B [N x K] per head, both
  // bf16 through TMA: K-major A read from row a_m0, MN-major operands from K
  // coordinate a_k0 / b_k0; rows of out past M are not written.
  auto tcg = [&](auto a_mn, auto b_mn, Opnd a, int a_m0, int a_k0, Opnd bo, int b_k0, int M, int N, int K,
                 float* out, int64_t out_item, int64_t ld, bool acc) {
    constexpr bool AMN = decltype(a_mn)::value, BMN = decltype(b_mn)::value;
    L(K_BWD_GEMM, [&] {
      GemmParams g = gemm_params();
      // An accumulating contraction splits K into up to 4 parts of at least 4
      // K blocks (each split adds its part into out with atomics) when that
      // fills the last wave of tiles better; the others halve the N tile while
      // they have too few tiles to fill the SMs.
      int bn = pick_bn(N);
      const int kbt = static_cast<int>(cdiv(K, 64));
      const int64_t tiles = static_cast<int64_t>(N / bn) * cdiv(M, 128) * BH;
      int splits = 1;
      if (acc) {
        const int64_t sms = sm_count();
        auto fill = [&](int64_t t) { return static_cast<double>(t) / static_cast<double>(cdiv(t, sms) * sms); };
        double best = fill(tiles);
        for (int sp = 2; sp <= 4 && kbt / sp >= 4; ++sp)
          if (fill(tiles * sp) > best + 0.05) {
            best = fill(tiles * sp);
            splits = sp;
          }
      }
      if (splits > 1) {
        splits = static_cast<int>(cdiv(kbt, cdiv(kbt, splits)));   // no empty split
      } else {
        while (bn >= 128 && (bn / 2) % 64 == 0 && N % (bn / 2) == 0 &&
               static_cast<int64_t>(N / bn) * cdiv(M, 128) * BH < 100)
          bn /= 2;
      }
      if (!map3d(&g.tmA, a.p, a.inner, a.rows, a.batch, 64, AMN ? 64 : 128) ||
          !map3d(&g.tmB, bo.p, bo.inner, bo.rows, bo.batch, 64, BMN ? 64 : bn))
        return cudaErrorInvalidValue;
      g.items = BH; g.kb_total = kbt; g.kb_count = static_cast<int>(cdiv(kbt, splits));
      g.a_m0 = a_m0; g.a_k0 = a_k0; g.b_k0 = b_k0;
      g.zb_mod = BH; g.m_valid = M;
      g.outf = out; g.item_stride = out_item; g.ld = ld;
      if (splits > 1) {
        g.red = 1;
      } else if (acc) {
        g.beta = 1.0f;
        g.cin = out;
      }
      return launch_gemm<AMN, BMN>(bn, dim3(N / bn, cdiv(M, 128), splits * BH), g, st);
    });
  };
  const std::false_type KM;   // K-major operand
  const std::true_type MN;    // MN-major operand
  const Opnd qh{b.qh16, D.d, D.Tq, D.BH}, kh{b.kh16, D.d, D.T, D.BH}, vv{in.v, D.d, D.T, D.BH};
  auto Wop = [&](const B16* W, int j) {   // plane j of a state: W1, W3 [dh][d]; W2 [d][dh]
    return j == 1 ? Opnd{W + jst, D.dh, D.d, D.BH} : Opnd{W + j * jst, D.d, D.dh, D.BH};
  };

  // ---- dout in fp32 (the scale's gradient), bf16 q^, k^
  if (in.scale)
    L(K_BWD_ELEM, [&] {
      (void)launch_pdl(k_bf16_to_f32, grid_for(nq, 4), 256, 0, st, static_cast<const B16*>(in.dout), b.do32, nq);
      return cudaGetLastError();
    });
  const B16* dos16 = static_cast<const B16*>(in.dout);
  if (in.scale) {
    L(K_BWD_ELEM, [&] {
      (void)launch_pdl(k_scale_rows_bf16, grid_for(nq, 4), 256, 0, st, static_cast<const B16*>(in.dout),
                       in.scale, b.dos16, D.BH * D.Tq, d);
      return cudaGetLastError();
    });
    dos16 = b.dos16;
  }
  const Opnd dos{dos16, D.d, D.Tq, D.BH};
  zero(in.dlr, D.BH * D.T * 3 * 4);
  if (mom) zero(in.dbeta, D.BH * D.T * 4);
  zero(in.dv, nk * 4);
  zero(b.dqh, nq * 4);
  zero(b.dkh, nk * 4);
  if (mom) {   // dL/dM after the last chunk
    for (int j = 0; j < 3; ++j) {
      if (in.dmf[j]) copy(b.Bm + j * jst, in.dmf[j], jst * 4);
      else zero(b.Bm + j * jst, jst * 4);
    }
  }
  if (mom && in.dmf[0]) reduce(b.Bm, planes);   // the ranks' gradients of the final momentum
  const float* dwf[3] = {in.dw1f, in.dw2f, in.dw3f};
  float* dw_init = cp ? b.Aloc : b.A;   // dL/dw_out is this rank's own
  if (cp) zero(b.A, planes * 4);
  for (int j = 0; j < 3; ++j) {
    if (dwf[j]) copy(dw_init + j * jst, dwf[j], jst * 4);
    else zero(dw_init + j * jst, jst * 4);
  }
  L(K_PROLOGUE, [&] {
    constexpr int ROWS = 4;
    const int64_t rows = D.BH * D.Tq + D.BH * D.T;
    const int nv = d / 8;
    auto launch = [&](auto kern, int S) {
      (void)launch_pdl(kern, static_cast<unsigned>(cdiv(cdiv(rows, ROWS) * S, 256)), 256, 0, st,
                       static_cast<const B16*>(in.q), b.qh16, D.BH * D.Tq, static_cast<const B16*>(in.k), b.kh16,
                       D.BH * D.T, d, static_cast<B16*>(nullptr));
    };
    if (nv <= 8) launch(k_qk_prologue_bf16<8, 1, ROWS, false>, 8);
    else if (nv <= 16) launch(k_qk_prologue_bf16<16, 1, ROWS, false>, 16);
    else if (nv <= 32) launch(k_qk_prologue_bf16<32, 1, ROWS, false>, 32);
    else launch(k_qk_prologue_bf16<32, 2, ROWS, false>, 32);
    return cudaGetLastError();
  });
  L(K_INIT, [&] {
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(cdiv(planes, 1024), 148 * 16));
    (void)launch_pdl(k_init_state, blocks, 256, 0, st, in.w1, in.w2, in.w3, static_cast<int>(D.H), D.w_shared,
                     BH, d, dh, b.hist, b.hist16, static_cast<B16*>(nullptr), mom ? b.Mm : nullptr,
                     in.m0[0], in.m0[1], in.m0[2]);
    return cudaGetLastError();
  });
  if (mom) {   // per-chunk beta means (context parallel: sums and counts over the ranks)
    const int64_t w = D.BH * D.nch;
    L(K_BETA_MEAN, [&] {
      (void)launch_pdl(k_beta_mean, static_cast<unsigned>(cdiv(w * 32, 256)), 256, 0, st, in.beta, BH, D.T,
                       D.chunk, static_cast<int>(D.nch), b.bbar, cp ? 1 : 0);
      return cudaGetLastError();
    });
    if (cp) {
      reduce(b.bbar, 2 * w);
      L(K_BETA_MEAN, [&] {
        (void)launch_pdl(k_beta_div, static_cast<unsigned>(cdiv(w, 256)), 256, 0, st, b.bbar, w);
        return cudaGetLastError();
      });
    }
  }
  // The forward's fused key kernel at a state W (bf16): z1 = X W1^T, z3 = X W3^T,
  // g = Y W2 for rows x_row0 .. x_row0 + n of X and Y ([BH][rows][d]), and the
  // factor planes E [3][BH][zr][dh] = (lr1 g z3 silu'(z1), lr2 silu(z1) z3,
  // lr3 g silu(z1)); lr null means unit rates.
  auto fwd_key = [&](int kind, const B16* W, const Opnd& X, const void* Y, int x_row0, int n, const float* lr,
                     B16* E) {
    L(kind, [&] {
      FwdParams f;
      std::memset(&f, 0, sizeof(f));
      if (!map3d(&f.tmX, X.p, D.d, X.rows, D.BH, 64, 128) || !map3d(&f.tmV, Y, D.d, X.rows, D.BH, 64, 128) ||
          !map3d(&f.tmW, W, D.d, D.dh, 3 * D.BH, 64, 64) || !map3d(&f.tmW2, W + jst, D.dh, D.d, D.BH, 64, 64) ||
          !map3d(&f.tmE, E, D.dh, zr, 3 * D.BH, 64, 32))
        return cudaErrorInvalidValue;
      f.bh_count = BH; f.n_slices = dh / 64; f.n_row_tiles = static_cast<int>(cdiv(n, 128));
      f.x_row0 = x_row0; f.rows_valid = n; f.kb_count = d / 64; f.dh = dh; f.T = static_cast<int>(X.rows);
      f.e = E; f.buf_rows = zr; f.lr = lr;
      return launch_umma<FwdOp<true>>(static_cast<int64_t>(f.n_slices) * f.n_row_tiles * BH, f, st);
    });
  };

  // ---- forward recompute: the states, momenta and pre-renorm row norms
  for (int64_t c = 0; c < D.nch; ++c) {
    const int64_t c0 = c * D.chunk;
    const int nc = static_cast<int>(std::min(c0 + D.chunk, D.T) - c0);
    copy(b.hist + (c + 1) * planes, b.hist + c * planes, planes * 4);
    copy(b.hist16 + (c + 1) * planes, b.hist16 + c * planes, planes * 2);
    if (in.mask && in.mask[c] == 0) continue;
    if (mom) copy(b.mh + c * planes, b.Mm, planes * 4);
    fwd_key(K_FWD_KEY, b.hist16 + c * planes, kh, in.v, static_cast<int>(c0), nc, in.lr, b.op16);
    L(K_BWD_GEMM, [&] {   // -G = E^T [k^, v, k^] over the chunk, W2's plane stored transposed
      GemmParams g = gemm_params();
      if (!map3d(&g.tmA, b.op16, dh, zr, 3 * BH, 64, 64) || !map3d(&g.tmB, b.kh16, d, D.T, BH, 64, 64) ||
          !map3d(&g.tmB2, in.v, d, D.T, BH, 64, 64))
        return cudaErrorInvalidValue;
      const int bn = pick_bn(D.d);
      g.items = 3 * BH; g.kb_count = g.kb_total = static_cast<int>(cdiv(nc, 64));
      g.a_k0 = 0; g.b_k0 = static_cast<int>(c0);
      g.zb_mod = BH; g.alt_group = 1; g.m_valid = dh;
      g.outf = b.P; g.item_stride = plane; g.ld = d;
      g.tr_group = 1; g.tr_mod = BH; g.ld_t = dh;
      return launch_gemm<true, true>(bn, dim3(d / bn, cdiv(dh, 128), 3 * BH), g, st);
    });
    reduce(b.P, planes);   // the whole chunk's gradient
    L(K_RULE, [&] {
      RuleParams r;
      std::memset(&r, 0, sizeof(r));
      r.Wm = b.hist + (c + 1) * planes; r.Ws = b.hist16 + (c + 1) * planes; r.S = b.P; r.splits = 1;
      r.split_stride = planes; r.Mm = mom ? b.Mm : nullptr; r.beta_bar = b.bbar;
      r.nch = static_cast<int>(D.nch); r.chunk_idx = static_cast<int>(c); r.rule = D.rule;
      r.BH = BH; r.dh = dh; r.d = d; r.nrm_out = b.mnorm + c * rows_all;
      (void)launch_pdl(k_rule_renorm, static_cast<unsigned>(cdiv(rows_all * 32, 256)), 256, 0, st, r);
      return cudaGetLastError();
    });
  }

  // ---- reverse chunk loop, on merged contractions:
  //   [z1|z3|p|r] = k^ [W1; W3; Gam1; Gam3]^T,  [u|q] = v [W2 | Gam2]
  //   dk^ += [dz1|dz3|dp|dr] [W1; W3; Gam1; Gam3],  dv += [du|dq] [W2 | Gam2]^T
  //   apply: [zq1|zq3] = q^ [W1; W3]^T,  dq^ += [dz1|dz3] [W1; W3]
  float* A = b.A;
  float* Ap = b.Ap;
  const int64_t pb = plane * 2;   // bytes of one bf16 plane
  auto copy2d = [&](void* dst, int64_t dpitch, const void* src, int64_t spitch, int64_t width, int64_t height) {
    if (!L.dry)
      memop(cudaMemcpy2DAsync(dst, static_cast<size_t>(dpitch), src, static_cast<size_t>(spitch),
                              static_cast<size_t>(width), static_cast<size_t>(height), cudaMemcpyDeviceToDevice,
                              st));
  };
  // stack per head: dst [BH][n_slots * dh][d] from [dh][d] planes
  auto stack_rows = [&](B16* dst, int n_slots, int slot, const B16* src_plane) {
    copy2d(dst + slot * plane, n_slots * pb, src_plane, pb, pb, D.BH);
  };
  const int64_t dh4 = 4 * D.dh, dh2 = 2 * D.dh;
  B16* Phik = b.op16;                 // [BH][zr][4 dh]
  B16* Phiv = b.op16 + 4 * zpl;       // [BH][zr][2 dh]
  const Opnd Zk_op{Phik, dh4, zr, D.BH}, Zv_op{Phiv, dh2, zr, D.BH};
  auto apply_bwd = [&](const B16* W, int64_t qr0, int nq_c) {
    const int r0 = static_cast<int>(qr0);
    // [z1|z3] = q^ [W1; W3]^T and g = dO W2 with the factors dz1 = g z3 silu'(z1),
    // hq = silu(z1) z3 and dz3 = g silu(z1): the fused key kernel with unit
    // rates and dO in place of v, planes Ea = (dz1, hq, dz3)
    B16* Ea = b.op16;
    fwd_key(K_BWD_APPLY, W, qh, dos.p, r0, nq_c, nullptr, Ea);
    const Opnd E1{Ea, D.dh, zr, D.BH}, Eh{Ea + zpl, D.dh, zr, D.BH}, E3{Ea + 2 * zpl, D.dh, zr, D.BH};
    // dW1 += dz1^T q^, dW3 += dz3^T q^, dW2 += dO^T hq (this rank's own part)
    float* Aq = cp ? b.Aloc : A;
    tcg(MN, MN, E1, 0, 0, qh, r0, dh, d, nq_c, Aq, plane, d, true);
    tcg(MN, MN, E3, 0, 0, qh, r0, dh, d, nq_c, Aq + 2 * jst, plane, d, true);
    tcg(MN, MN, dos, 0, r0, Eh, 0, d, dh, nq_c, Aq + jst, plane, dh, true);
    // dq^ += dz1 W1 + dz3 W3
    tcg(KM, MN, E1, 0, 0, Wop(W, 0), 0, nq_c, d, dh, b.dqh + qr0 * d, D.Tq * D.d, d, true);
    tcg(KM, MN, E3, 0, 0, Wop(W, 2), 0, nq_c, d, dh, b.dqh + qr0 * d, D.Tq * D.d, d, true);
    if (in.scale)   // the unscaled output hq W2^T, for the scale's gradient
      tcg(KM, KM, Eh, 0, 0, Wop(W, 1), 0, nq_c, d, dh, b.ofull + qr0 * d, D.Tq * D.d, d, false);
  };
  for (int64_t c = D.nch - 1; c >= 0; --c) {
    const int64_t c0 = c * D.chunk;
    const int nc = static_cast<int>(std::min(c0 + D.chunk, D.T) - c0);
    const int64_t qr0 = D.nch == 1 ? 0 : c0;
    const int nq_c = static_cast<int>(D.nch == 1 ? D.Tq : nc);
    const B16* Wp16 = b.hist16 + c * planes;
    const B16* Wc16 = b.hist16 + (c + 1) * planes;
    const bool upd = !in.mask || in.mask[c] != 0;
    if (D.order == LACT_UPDATE_THEN_APPLY) apply_bwd(Wc16, qr0, nq_c);
    if (upd) {
      reduce(b.Aloc, planes);   // the ranks' own contributions to dL/dW^c
      L(K_BWD_ELEM, [&] {
        RenormBwdParams r;
        std::memset(&r, 0, sizeof(r));
        r.A = A; r.A2 = cp ? b.Aloc : nullptr; r.Wc = b.hist + (c + 1) * planes; r.Wp = b.hist + c * planes; r.mnorm = b.mnorm + c * rows_all;
        r.Gam16 = b.Gam16; r.Ap = Ap; r.rule = D.rule; r.Bm = b.Bm;
        r.Mprev = mom ? b.mh + c * planes : nullptr; r.beta_bar = b.bbar; r.nch = static_cast<int>(D.nch);
        r.chunk_idx = static_cast<int>(c); r.part = b.part; r.BH = BH; r.dh = dh; r.d = d;
        (void)launch_pdl(k_renorm_bwd, static_cast<unsigned>(cdiv(rows_all * 32, 256)), 256, 0, st, r);
        return cudaGetLastError();
      });
      if (mom)
        L(K_BWD_ELEM, [&] {
          (void)launch_pdl(k_head_dbeta, static_cast<unsigned>(BH), 256, 0, st, b.part, BH, dh, d, D.T, c0, nc,
                           cp ? static_cast<const float*>(b.bbar + D.BH * D.nch + c) : nullptr, D.nch, in.dbeta);
          return cudaGetLastError();
        });
      // stacked operands: Bk = [W1; W3; Gam1; Gam3] [BH][4 dh][d], Bv = [W2 | Gam2] [BH][d][2 dh]
      stack_rows(b.Bk, 4, 0, Wp16);
      stack_rows(b.Bk, 4, 1, Wp16 + 2 * jst);
      stack_rows(b.Bk, 4, 2, b.Gam16);
      stack_rows(b.Bk, 4, 3, b.Gam16 + 2 * jst);
      copy2d(b.Bv, dh2 * 2, Wp16 + jst, D.dh * 2, D.dh * 2, D.BH * D.d);
      copy2d(b.Bv + D.dh, dh2 * 2, b.Gam16 + jst, D.dh * 2, D.dh * 2, D.BH * D.d);
      const Opnd Bk_op{b.Bk, D.d, dh4, D.BH};
      const int k0 = static_cast<int>(c0);
      // [z1|z3|p|r] = k^ Bk^T, [u|q] = v Bv and their second-order factors, one kernel
      L(K_BWD_KEY, [&] {
        BwdKeyParams f;
        std::memset(&f, 0, sizeof(f));
        if (!map3d(&f.tmX, kh.p, D.d, D.T, D.BH, 64, 128) || !map3d(&f.tmV, in.v, D.d, D.T, D.BH, 64, 128) ||
            !map3d(&f.tmBk, b.Bk, D.d, dh4, D.BH, 64, 64) || !map3d(&f.tmBv, b.Bv, dh2, D.d, D.BH, 64, 64) ||
            !map3d_plain(&f.tmPk, Phik, dh4, zr, D.BH, 16, 32) || !map3d_plain(&f.tmPv, Phiv, dh2, zr, D.BH, 16, 32))
          return cudaErrorInvalidValue;
        f.bh_count = BH; f.n_slices = dh / 64; f.n_row_tiles = static_cast<int>(cdiv(zr, 128));
        f.kb_count = d / 64; f.x_row0 = k0; f.rows_valid = nc; f.dh = dh;
        f.T = D.T; f.lr = in.lr; f.dlr = in.dlr;
        return launch_umma<BwdKeyOp>(static_cast<int64_t>(f.n_slices) * f.n_row_tiles * BH, f, st);
      });
      // dW1 += dz1^T k^, dW3 += dz3^T k^, dW2 += v^T du (this rank's own part)
      float* Ak = cp ? b.Aloc : Ap;
      tcg(MN, MN, Zk_op, 0, 0, kh, k0, dh, d, nc, Ak, plane, d, true);
      tcg(MN, MN, Zk_op, dh, 0, kh, k0, dh, d, nc, Ak + 2 * jst, plane, d, true);
      tcg(MN, MN, vv, 0, k0, Zv_op, 0, d, dh, nc, Ak + jst, plane, dh, true);
      // dk^ += [dz1|dz3|dp|dr] [W1; W3; Gam1; Gam3],  dv += [du|dq] [W2 | Gam2]^T
      tcg(KM, MN, Zk_op, 0, 0, Bk_op, 0, nc, d, 4 * dh, b.dkh + c0 * d, D.T * D.d, d, true);
      tcg(KM, KM, Zv_op, 0, 0, Opnd{b.Bv, dh2, D.d, D.BH}, 0, nc, d, 2 * dh, in.dv + c0 * d, D.T * D.d, d, true);
      std::swap(A, Ap);
    }
    if (D.order == LACT_APPLY_THEN_UPDATE) apply_bwd(Wp16, qr0, nq_c);
  }

  // ---- prologue backward, the scale's gradient, the initial weights' gradient
  L(K_BWD_ELEM, [&] {
    (void)launch_pdl(k_prologue_bwd_bf16, grid_for(D.BH * D.Tq * 32, 1), 256, 0, st, static_cast<const B16*>(in.q),
                     static_cast<const float*>(b.dqh), in.dq, D.BH * D.Tq, d);
    return cudaGetLastError();
  });
  L(K_BWD_ELEM, [&] {
    (void)launch_pdl(k_prologue_bwd_bf16, grid_for(D.BH * D.T * 32, 1), 256, 0, st, static_cast<const B16*>(in.k),
                     static_cast<const float*>(b.dkh), in.dk, D.BH * D.T, d);
    return cudaGetLastError();
  });
  if (in.scale)
    L(K_BWD_ELEM, [&] {
      (void)launch_pdl(k_rowdot, static_cast<unsigned>(cdiv(D.BH * D.Tq * 32, 256)), 256, 0, st,
                       static_cast<const float*>(b.do32), static_cast<const float*>(b.ofull), in.dscale,
                       D.BH * D.Tq, d);
      return cudaGetLastError();
    });
  if (cp) {   // the own contributions left after chunk 0, summed over the ranks
    reduce(b.Aloc, planes);
    L(K_BWD_ELEM, [&] {
      (void)launch_pdl(k_add_planes, grid_for(planes, 4), 256, 0, st, A, static_cast<const float*>(b.Aloc), planes);
      return cudaGetLastError();
    });
  }
  L(K_BWD_ELEM, [&] {
    (void)launch_pdl(k_sum_batch, grid_for(planes, 4), 256, 0, st, static_cast<const float*>(A),
                     static_cast<int>(D.B), static_cast<int>(D.H), plane, D.w_shared, in.dw1, in.dw2, in.dw3);
    return cudaGetLastError();
  });
  if (mom)   // after chunk 0, B holds dL/dM_0
    for (int j = 0; j < 3; ++j)
      if (in.dm0[j]) copy(in.dm0[j], b.Bm + j * jst, jst * 4);
}

static void run_bwd(const Dims& D, const BwdBufs& b, const BwdInputs& in, cudaStream_t st, Launcher& L) {
  if (bwd_on_tc(D)) run_bwd_tc(D, b, in, st, L);
  else run_bwd_f32(D, b, in, st, L);
}

}  // namespace lact
