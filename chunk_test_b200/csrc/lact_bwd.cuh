// lact_bwd.cuh -- host side of the layer's backward (lact_ttt_bwd), included
// by lact_api.cu after the forward's planning and launch helpers.
//
// The backward is the vector-Jacobian product of the forward, in fp32:
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
// Every contraction is a batched k_simt_gemm over the B*H heads.
#pragma once

#include "bwd_kernels.cuh"

namespace lact {

struct BwdInputs {
  const void *q, *k, *v;
  const float *lr, *beta, *w1, *w2, *w3;
  const void* dout;
  const float *dw1f, *dw2f, *dw3f;       // gradients of the final weights, or null
  const uint8_t* mask;
  const float* scale;
  float *dq, *dk, *dv, *dlr, *dbeta, *dw1, *dw2, *dw3, *dscale;
};

struct BwdBufs {
  float *q32, *k32, *v32, *do32, *dos32, *qh, *kh;
  float *hist, *mh, *Mm, *mnorm, *bbar;
  float *Z, *Pz, *E, *P;
  float *A, *Ap, *Gam, *Bm;
  float *dqh, *dkh, *ofull, *part;
  int64_t zr;   // rows per head of the per-chunk [rows][dh] planes
};

static int64_t rule_rows(const Dims& D) { return 2 * D.BH * D.dh + D.BH * D.d; }

static void plan_bwd(const Dims& D, Bump& bp, BwdBufs& b) {
  std::memset(&b, 0, sizeof(b));
  const int64_t planes = 3 * D.BH * D.dh * D.d;
  const int64_t nq = D.BH * D.Tq * D.d, nk = D.BH * D.T * D.d;
  const bool bf = D.dtype == LACT_BF16;
  const bool mom = D.rule == LACT_RULE_MOMENTUM;
  b.zr = std::max<int64_t>(D.chunk, D.nch == 1 ? D.Tq : D.chunk);
  if (bf) {
    b.q32 = bp.take<float>(nq);
    b.k32 = bp.take<float>(nk);
    b.v32 = bp.take<float>(nk);
    b.do32 = bp.take<float>(nq);
  }
  b.dos32 = bp.take<float>(nq);
  b.qh = bp.take<float>(nq);
  b.kh = bp.take<float>(nk);
  b.hist = bp.take<float>((D.nch + 1) * planes);
  if (mom) {
    b.mh = bp.take<float>(D.nch * planes);
    b.Mm = bp.take<float>(planes);
    b.bbar = bp.take<float>(D.BH * D.nch);
    b.Bm = bp.take<float>(planes);
    b.part = bp.take<float>(rule_rows(D));
  }
  b.mnorm = bp.take<float>(D.nch * rule_rows(D));
  const int64_t zpl = D.BH * b.zr * D.dh;
  b.Z = bp.take<float>(3 * zpl);
  b.Pz = bp.take<float>(3 * zpl);
  b.E = bp.take<float>(3 * zpl);
  b.P = bp.take<float>(planes);
  b.A = bp.take<float>(planes);
  b.Ap = bp.take<float>(planes);
  b.Gam = bp.take<float>(planes);
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

static void run_bwd(const Dims& D, const BwdBufs& b, const BwdInputs& in, cudaStream_t st, Launcher& L) {
  L.st = st;
  const bool bf = D.dtype == LACT_BF16, mom = D.rule == LACT_RULE_MOMENTUM;
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

  // ---- fp32 inputs, the scaled output gradient, zeroed accumulators
  const float* q32 = bf ? b.q32 : static_cast<const float*>(in.q);
  const float* k32 = bf ? b.k32 : static_cast<const float*>(in.k);
  const float* v32 = bf ? b.v32 : static_cast<const float*>(in.v);
  const float* do32 = bf ? b.do32 : static_cast<const float*>(in.dout);
  if (bf) {
    const void* src[4] = {in.q, in.k, in.v, in.dout};
    float* dst[4] = {b.q32, b.k32, b.v32, b.do32};
    const int64_t n[4] = {nq, nk, nk, nq};
    for (int i = 0; i < 4; ++i)
      L(K_BWD_ELEM, [&] {
        (void)launch_pdl(k_bf16_to_f32, grid_for(n[i], 4), 256, 0, st,
                         static_cast<const __nv_bfloat16*>(src[i]), dst[i], n[i]);
        return cudaGetLastError();
      });
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
  if (mom) zero(b.Bm, planes * 4);
  const float* dwf[3] = {in.dw1f, in.dw2f, in.dw3f};
  for (int j = 0; j < 3; ++j) {
    if (dwf[j]) copy(b.A + j * jst, dwf[j], jst * 4);
    else zero(b.A + j * jst, jst * 4);
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
                     static_cast<const float*>(nullptr), static_cast<const float*>(nullptr),
                     static_cast<const float*>(nullptr));
    return cudaGetLastError();
  });
  if (mom) {
    L(K_BETA_MEAN, [&] {
      const int64_t w = D.BH * D.nch;
      (void)launch_pdl(k_beta_mean, static_cast<unsigned>(cdiv(w * 32, 256)), 256, 0, st, in.beta, BH, D.T,
                       D.chunk, static_cast<int>(D.nch), b.bbar);
      return cudaGetLastError();
    });
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
      s.tr_group = 1; s.tr_mod = BH; s.ld_t = dh;
      return simt(s, 3 * BH, st);
    });
    L(K_RULE, [&] {
      RuleParams r;
      std::memset(&r, 0, sizeof(r));
      r.Wm = Wn; r.S = b.P; r.splits = 1; r.split_stride = planes;
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
    // dW1 += dz1^T q^, dW3 += dz3^T q^, dW2 += dO^T hq
    for (int j = 0; j < 3; j += 2)
      gemm(b.Z + j * zpl, zr * D.dh, 1, dh, b.qh + qr0 * d, D.Tq * D.d, 1, d, dh, d, nq_c, A + j * jst, plane, d,
           true);
    gemm(dos + qr0 * d, D.Tq * D.d, 1, d, b.Z + zpl, zr * D.dh, 1, dh, d, dh, nq_c, A + jst, plane, dh, true);
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
      L(K_BWD_ELEM, [&] {
        RenormBwdParams r;
        std::memset(&r, 0, sizeof(r));
        r.A = A; r.Wc = Wc; r.Wp = Wp; r.mnorm = b.mnorm + c * rows_all; r.Gam = b.Gam; r.Ap = Ap;
        r.rule = D.rule; r.Bm = b.Bm; r.Mprev = mom ? b.mh + c * planes : nullptr; r.beta_bar = b.bbar;
        r.nch = static_cast<int>(D.nch); r.chunk_idx = static_cast<int>(c); r.part = b.part;
        r.BH = BH; r.dh = dh; r.d = d;
        (void)launch_pdl(k_renorm_bwd, static_cast<unsigned>(cdiv(rows_all * 32, 256)), 256, 0, st, r);
        return cudaGetLastError();
      });
      if (mom)
        L(K_BWD_ELEM, [&] {
          (void)launch_pdl(k_head_dbeta, static_cast<unsigned>(BH), 256, 0, st, b.part, BH, dh, d, D.T, c0, nc,
                           in.dbeta);
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
      // dW1 += dz1^T k^, dW3 += dz3^T k^, dW2 += v^T du
      for (int j = 0; j < 3; j += 2)
        gemm(b.Z + j * zpl, zr * D.dh, 1, dh, b.kh + c0 * d, D.T * D.d, 1, d, dh, d, nc, Ap + j * jst, plane, d,
             true);
      gemm(v32 + c0 * d, D.T * D.d, 1, d, b.Z + zpl, zr * D.dh, 1, dh, d, dh, nc, Ap + jst, plane, dh, true);
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
  L(K_BWD_ELEM, [&] {
    (void)launch_pdl(k_sum_batch, grid_for(planes, 4), 256, 0, st, static_cast<const float*>(A),
                     static_cast<int>(D.B), static_cast<int>(D.H), plane, D.w_shared, in.dw1, in.dw2, in.dw3);
    return cudaGetLastError();
  });
}

}  // namespace lact
