// lact_swa.cuh -- host side of the sliding-window attention (lact_swa_fwd),
// included by lact_api.cu after the forward's launch helpers.
//
// Per block of 128 queries (item z = bh * nb + m):
//   1. k_swa_prologue: q', k' (scale and offset per head and channel) and v
//      into Qp and the zero-padded window buffers Kp, Vp;
//   2. S = Qp_z Kp_window^T on the tensor cores (GemmOp, K-major operands;
//      the window of block m is the strided view of Kp starting at padded
//      row m*128, so B's batch for item z is bh * nbp + m);
//   3. k_swa_softmax: the sliding causal mask, 1/sqrt(d) and the softmax,
//      P in bf16;
//   4. out_z = P_z Vp_window on the tensor cores (V MN-major), bf16 out.
// For head dims up to 256 the path is two launches: k_swa_prologue_q writes
// Qt = q' * k_scale (the key offset only adds a per-query constant to the
// scores, which the softmax removes), and k_swa_flash reads Qt with the
// caller's k and v as they are, the scores staying on chip (online
// softmax).  Larger head dims take the path above, whose scores make a round
// trip through HBM (fp32 S, bf16 P).
#pragma once

#include "swa_flash.cuh"
#include "swa_kernels.cuh"

namespace lact {

struct SwaDims {
  int64_t B, H, BH, T, d, window, nb, nbp, Lw, tail;
};

static int swa_validate(const lact_swa_problem* p, SwaDims& S) {
  if (!p) return LACT_EINVAL;
  if (p->B < 1 || p->H < 1 || p->T < 1 || p->d < 1 || p->window < 1) return LACT_EINVAL;
  if (p->dtype != LACT_BF16) return LACT_EINVAL;
  if (p->d % 64 != 0 || p->d > 512 || p->T % 128 != 0 || p->window % 128 != 0) return LACT_EINVAL;
  if (p->B * p->H > 4096 || p->T > (int64_t(1) << 24) || p->window > 16384) return LACT_EINVAL;
  S.B = p->B; S.H = p->H; S.BH = p->B * p->H; S.T = p->T; S.d = p->d; S.window = p->window;
  S.nb = S.T / 128;
  S.nbp = (S.window + S.T) / 128;
  S.Lw = S.window + 128;
  S.tail = S.window;   // rows after the last head, so the last views stay inside the buffer
  if (S.BH * S.nb > (int64_t(1) << 24)) return LACT_EINVAL;
  return LACT_OK;
}

struct SwaBufs {
  __nv_bfloat16 *Qp, *Kp, *Vp, *P;
  float* S;
};

static bool swa_fused(const SwaDims& S) { return S.d <= 256; }

static void swa_plan(const SwaDims& S, Bump& bp, SwaBufs& b) {
  b.Qp = bp.take<__nv_bfloat16>(S.BH * S.T * S.d);
  b.Kp = b.Vp = b.P = nullptr;
  b.S = nullptr;
  if (swa_fused(S)) return;
  const int64_t pad_rows = S.BH * (S.window + S.T) + S.tail;
  b.Kp = bp.take<__nv_bfloat16>(pad_rows * S.d);
  b.Vp = bp.take<__nv_bfloat16>(pad_rows * S.d);
  b.S = bp.take<float>(S.BH * S.T * S.Lw);
  b.P = bp.take<__nv_bfloat16>(S.BH * S.T * S.Lw);
}

template <int D>
static cudaError_t launch_swa_flash(const SwaDims& S, const SwaBufs& b, const void* k, const void* v, void* out,
                                    cudaStream_t st) {
  constexpr int smem = SwaCfg<D>::kSmem;
  static_assert(smem <= kMaxSmemPerBlock, "dynamic shared memory above the per-CTA limit");
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !attr_set[dev]) {
    e = cudaFuncSetAttribute(k_swa_flash<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  SwaFlashParams f;
  std::memset(&f, 0, sizeof(f));
  if (!map3d(&f.tmQ, b.Qp, S.d, S.T, S.BH, 64, 128) || !map3d(&f.tmK, k, S.d, S.T, S.BH, 64, 128) ||
      !map3d(&f.tmV, v, S.d, S.T, S.BH, 64, 64))
    return cudaErrorInvalidValue;
  f.bh_count = static_cast<int>(S.BH); f.nb = static_cast<int>(S.nb); f.window = static_cast<int>(S.window);
  f.scale = 1.0f / sqrtf(static_cast<float>(S.d));
  f.out = static_cast<__nv_bfloat16*>(out); f.T = S.T;
  const int64_t ntiles = S.BH * S.nb;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ntiles, sm_count()));
  (void)launch_pdl(k_swa_flash<D>, grid, kSwaThreads, smem, st, f);
  return cudaGetLastError();
}

static size_t swa_workspace_bytes(const SwaDims& S) {
  Bump bp{0, 0};
  SwaBufs b;
  swa_plan(S, bp, b);
  return static_cast<size_t>(rup(static_cast<int64_t>(bp.off), 256));
}

// 3-D bf16 map whose batch dimension has its own stride (elements), so that
// consecutive batches may overlap: the query blocks' key and value windows.
static bool map3d_strided(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint64_t batch,
                          uint64_t batch_stride, uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner * 2, batch_stride * 2};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int pick_bn_swa(int64_t n) {
  if (n <= 256) return static_cast<int>(n);
  if (n % 256 == 0) return 256;
  if (n % 128 == 0) return 128;
  return 64;
}

static void swa_run(const SwaDims& S, const SwaBufs& b, const void* q, const void* k, const void* v,
                    const float* qs, const float* qo, const float* ks, const float* ko, void* out,
                    cudaStream_t st, Launcher& L) {
  L.st = st;
  const int64_t items = S.BH * S.nb;
  if (swa_fused(S)) {
    L(K_SWA, [&] {
      const int64_t n = S.BH * S.T * (S.d / 8);
      const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(cdiv(n, 256), 148 * 32));
      (void)launch_pdl(k_swa_prologue_q, blocks, 256, 0, st, static_cast<const __nv_bfloat16*>(q), qs, qo, ks,
                       static_cast<int>(S.H), S.T, static_cast<int>(S.d), n, b.Qp);
      return cudaGetLastError();
    });
    L(K_SWA_FLASH, [&] {
      switch (S.d) {
        case 64: return launch_swa_flash<64>(S, b, k, v, out, st);
        case 128: return launch_swa_flash<128>(S, b, k, v, out, st);
        case 192: return launch_swa_flash<192>(S, b, k, v, out, st);
        default: return launch_swa_flash<256>(S, b, k, v, out, st);
      }
    });
    return;
  }
  L(K_SWA, [&] {
    const int64_t n = (S.BH * S.T + S.BH * S.window + S.tail) * (S.d / 8);
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(cdiv(n, 256), 148 * 32));
    (void)launch_pdl(k_swa_prologue, blocks, 256, 0, st, static_cast<const __nv_bfloat16*>(q),
                     static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), qs, qo, ks, ko,
                     static_cast<int>(S.H), static_cast<int>(S.BH), S.T, static_cast<int>(S.d), S.window, S.tail,
                     b.Qp, b.Kp, b.Vp);
    return cudaGetLastError();
  });
  L(K_SWA_GEMM, [&] {   // S_z = Qp_z Kp_window(z)^T, fp32
    GemmParams g = gemm_params();
    const int bn = pick_bn_swa(S.Lw);
    if (!map3d(&g.tmA, b.Qp, S.d, 128, items, 64, 128) ||
        !map3d_strided(&g.tmB, b.Kp, S.d, S.Lw, S.BH * S.nbp, 128 * S.d, 64, bn))
      return cudaErrorInvalidValue;
    g.items = static_cast<int>(items); g.kb_count = g.kb_total = static_cast<int>(S.d / 64);
    g.zb_div = static_cast<int>(S.nb); g.zb_mul = static_cast<int>(S.nbp); g.m_valid = 128;
    g.outf = b.S; g.item_stride = 128 * S.Lw; g.ld = S.Lw;
    return launch_gemm<false, false>(bn, dim3(static_cast<unsigned>(S.Lw / bn), 1, static_cast<unsigned>(items)),
                                     g, st);
  });
  L(K_SWA, [&] {
    const int64_t rows = S.BH * S.T;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(cdiv(rows * 32, 256), 148 * 64));
    const float scale = 1.0f / sqrtf(static_cast<float>(S.d));
    const float* Sf = b.S;
    const int nb = static_cast<int>(S.nb);
    // rows of up to 33 x 128 scores are held in registers (read once)
    switch (S.Lw / 128) {
#define LACT_SWA_REG(NV) \
      case NV: (void)launch_pdl(k_swa_softmax_reg<NV>, blocks, 256, 0, st, Sf, rows, nb, S.window, scale, b.P); break;
      LACT_SWA_REG(2) LACT_SWA_REG(3) LACT_SWA_REG(5) LACT_SWA_REG(9) LACT_SWA_REG(17) LACT_SWA_REG(33)
#undef LACT_SWA_REG
      default:
        (void)launch_pdl(k_swa_softmax, blocks, 256, 0, st, Sf, rows, nb, static_cast<int>(S.Lw), S.window, scale,
                         b.P);
    }
    return cudaGetLastError();
  });
  L(K_SWA_GEMM, [&] {   // out_z = P_z Vp_window(z), bf16
    GemmParams g = gemm_params();
    const int bn = pick_bn_swa(S.d);
    if (!map3d(&g.tmA, b.P, S.Lw, 128, items, 64, 128) ||
        !map3d_strided(&g.tmB, b.Vp, S.d, S.Lw, S.BH * S.nbp, 128 * S.d, 64, 64))
      return cudaErrorInvalidValue;
    g.items = static_cast<int>(items); g.kb_count = g.kb_total = static_cast<int>(S.Lw / 64);
    g.zb_div = static_cast<int>(S.nb); g.zb_mul = static_cast<int>(S.nbp); g.m_valid = 128;
    g.outb = static_cast<__nv_bfloat16*>(out); g.item_stride = 128 * S.d; g.ld = S.d;
    return launch_gemm<false, true>(bn, dim3(static_cast<unsigned>(S.d / bn), 1, static_cast<unsigned>(items)),
                                    g, st);
  });
}

}  // namespace lact
