// lact_api.cu -- C ABI of the LaCT fast-weight TTT layer forward (see
// include/lact.h): argument checks, the workspace plan, TMA tensor maps and
// the per-chunk launch sequence on the caller's stream.
//
// Per chunk c (tokens [c0, c0 + nc)), in the order the problem asks for
// ("LaCT：以大分块更新…" 「更新顺序必须遵守信息可见范围」):
//   apply  : FwdOp<query>  Hq = silu(q^ W1^T) * (q^ W3^T)
//            GemmOp        out_c = Hq W2^T
//   update : FwdOp<key>    E1, Eh, E3 (per-token gradient factors, lr-scaled)
//            GemmOp        -G_j = E_j^T X_j   (X = k^, v, k^), split over tokens
//            [Muon]        X0 = -G/||G||, 5 x (A = X^T X; B = bA + cA^2;
//                          X = aX + XB) on the d-side Gram matrix
//            k_rule_renorm W <- renorm(W - U)
// The fp32 path runs the same sequence with CUDA-core kernels.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/lact.h"
#include "elem_kernels.cuh"
#include "simt_kernels.cuh"
#include "sm100.cuh"
#include "umma_kernels.cuh"
#include "apply_kernel.cuh"
#include "key_grad_kernel.cuh"
#include "pair_kernels.cuh"

namespace lact {

static inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
static inline int64_t rup(int64_t a, int64_t b) { return cdiv(a, b) * b; }

constexpr float kNsA = 3.4445f, kNsB = -4.7750f, kNsC = 2.0315f;
constexpr int kNsSteps = 5;
constexpr float kNsEps = 1e-7f;
constexpr int kNsBlocks = 64;  // partial-sum blocks per matrix for ||G||_F

struct Dims {
  int64_t B, H, BH, T, Tq, d, dh, chunk, nch;
  int order, rule, dtype, w_shared;
  int64_t key_rows;  // rows per head of the per-chunk key buffers (E / Z)
  int64_t q_rows;    // rows per head of the per-chunk query buffer (Hq)
  int splits;        // token splits of the gradient contraction (bf16)
  int bn;            // N tile over d (bf16 GEMMs)
  bool split;        // split-bf16 update path (bf16 + Muon)
  bool fused_kg;     // fused key forward + gradient (bf16, d = 64, dh = 128, not split)
  bool dbuf;         // two bf16 shadow sets (bf16, apply-then-update): chunk c reads set c % 2
  int kg_splits;     // its token splits per head
};

// Planning constant for the fused key + gradient kernel: work items are
// (head, token split) with about one item per SM of a B200.
constexpr int kPlanSMs = 148;

static int choose_bn(int64_t d) {
  if (d <= 256) return static_cast<int>(d);
  if (d % 256 == 0) return 256;
  if (d % 192 == 0) return 192;
  if (d % 128 == 0) return 128;
  return 64;
}

static int validate(const lact_problem* p, Dims& D) {
  if (!p) return LACT_EINVAL;
  if (p->B < 1 || p->H < 1 || p->T < 1 || p->Tq < 1 || p->d < 1 || p->dh < 1 || p->chunk < 1)
    return LACT_EINVAL;
  if (p->order != LACT_APPLY_THEN_UPDATE && p->order != LACT_UPDATE_THEN_APPLY) return LACT_EINVAL;
  if (p->rule < LACT_RULE_GD || p->rule > LACT_RULE_MUON) return LACT_EINVAL;
  if (p->dtype != LACT_F32 && p->dtype != LACT_BF16) return LACT_EINVAL;
  if (p->w_shared != 0 && p->w_shared != 1) return LACT_EINVAL;
  D.B = p->B; D.H = p->H; D.BH = p->B * p->H; D.T = p->T; D.Tq = p->Tq; D.d = p->d; D.dh = p->dh;
  D.chunk = p->chunk < p->T ? p->chunk : p->T;
  D.nch = cdiv(p->T, D.chunk);
  D.order = p->order; D.rule = p->rule; D.dtype = p->dtype; D.w_shared = p->w_shared;
  if (D.nch > 1 && D.Tq != D.T) return LACT_EINVAL;
  if (D.d > 512 || D.dh > 4096) return LACT_EINVAL;
  if (D.BH > 4096 || D.T > (int64_t(1) << 30) || D.Tq > (int64_t(1) << 30)) return LACT_EINVAL;
  if (D.dtype == LACT_BF16 && (D.d % 64 != 0 || D.dh % 64 != 0)) return LACT_EINVAL;
  D.key_rows = rup(D.chunk, 128);
  D.q_rows = rup(D.nch == 1 ? D.Tq : D.chunk, 128);
  if (D.key_rows / 128 > 65535 || D.q_rows / 128 > 65535) return LACT_EINVAL;
  D.bn = choose_bn(D.d);
  D.split = D.dtype == LACT_BF16 && D.rule == LACT_RULE_MUON;
  D.fused_kg = D.dtype == LACT_BF16 && !D.split && D.d == 64 && D.dh == 128;
  D.dbuf = D.dtype == LACT_BF16 && D.order == LACT_APPLY_THEN_UPDATE && D.nch > 1;
  D.kg_splits = 1;
  // Token splits of the gradient contraction: fill ~2 waves of 148 SMs when
  // the output tiles alone do not.
  const int64_t tiles = (D.d / D.bn) * cdiv(D.dh, 128) * 3 * D.BH;
  int64_t s = tiles >= 120 ? 1 : cdiv(296, tiles);
  const int64_t kbt = cdiv(D.chunk, 64);
  if (s > kbt) s = kbt;
  if (s * 3 * D.BH > 65535) s = 65535 / (3 * D.BH);
  D.splits = static_cast<int>(s < 1 ? 1 : s);
  if (D.fused_kg) {
    // (head, token split) items, about one per SM; no split left empty.
    const int64_t tiles = cdiv(D.chunk, 128);
    int64_t ks = std::max<int64_t>(1, kPlanSMs / D.BH);
    if (ks > tiles) ks = tiles;
    const int64_t tps = cdiv(tiles, ks);
    ks = cdiv(tiles, tps);
    D.kg_splits = static_cast<int>(ks);
    D.splits = std::max(D.splits, D.kg_splits);
  }
  if (3 * D.BH * D.splits > 65535) return LACT_EINVAL;
  return LACT_OK;
}

struct Bufs {
  void* qh; void* kh; __nv_bfloat16* kh_lo;
  float* Wm; __nv_bfloat16* Ws; __nv_bfloat16* Ws_lo; float* P; float* Mm; float* bbar;
  void* E; void* E_lo; void* Hq; float* Z;
  float* Yf[2]; __nv_bfloat16* Yb[2]; __nv_bfloat16* Yb_lo[2];
  float* Af; __nv_bfloat16* Ab; __nv_bfloat16* Ab_lo; float* Bf; __nv_bfloat16* Bb;
  __nv_bfloat16* Bb_lo; float* part;
};

struct Bump {
  uintptr_t base, off;
  template <class T> T* take(int64_t count) {
    off = static_cast<uintptr_t>(rup(static_cast<int64_t>(off), 256));
    T* r = reinterpret_cast<T*>(base + off);
    off += static_cast<uintptr_t>(count) * sizeof(T);
    return r;
  }
};

static void plan(const Dims& D, Bump& bp, Bufs& b) {
  std::memset(&b, 0, sizeof(b));
  const bool bf = D.dtype == LACT_BF16;
  const int64_t esz = bf ? 2 : 4;
  const int64_t plane = D.dh * D.d, planes = 3 * D.BH * plane;
  b.qh = bp.take<uint8_t>(D.BH * D.Tq * D.d * esz);
  b.kh = bp.take<uint8_t>(D.BH * D.T * D.d * esz);
  if (D.split) b.kh_lo = bp.take<__nv_bfloat16>(D.BH * D.T * D.d);
  b.Wm = bp.take<float>(planes);
  if (bf) b.Ws = bp.take<__nv_bfloat16>((D.dbuf ? 2 : 1) * planes);
  if (D.split) b.Ws_lo = bp.take<__nv_bfloat16>((D.dbuf ? 2 : 1) * planes);
  b.P = bp.take<float>((bf ? D.splits : 1) * planes);
  if (D.rule == LACT_RULE_MOMENTUM) {
    b.Mm = bp.take<float>(planes);
    b.bbar = bp.take<float>(2 * D.BH * D.nch);   // sums, then token counts (context parallelism)
  }
  if (!D.fused_kg) b.E = bp.take<uint8_t>(3 * D.BH * D.key_rows * D.dh * esz);
  if (D.split) b.E_lo = bp.take<uint8_t>(3 * D.BH * D.key_rows * D.dh * esz);
  if (!bf || D.d > 256) b.Hq = bp.take<uint8_t>(D.BH * D.q_rows * D.dh * esz);  // unfused apply only
  if (!bf) b.Z = bp.take<float>(3 * D.BH * (D.key_rows > D.q_rows ? D.key_rows : D.q_rows) * D.dh);
  if (D.rule == LACT_RULE_MUON) {
    for (int i = 0; i < 2; ++i) {
      b.Yf[i] = bp.take<float>(planes);
      if (bf) b.Yb[i] = bp.take<__nv_bfloat16>(planes);
      if (D.split) b.Yb_lo[i] = bp.take<__nv_bfloat16>(planes);
    }
    b.Af = bp.take<float>(3 * D.BH * D.d * D.d);
    if (bf) {
      b.Ab = bp.take<__nv_bfloat16>(3 * D.BH * D.d * D.d);
      b.Bb = bp.take<__nv_bfloat16>(3 * D.BH * D.d * D.d);
      if (D.split) {
        b.Ab_lo = bp.take<__nv_bfloat16>(3 * D.BH * D.d * D.d);
        b.Bb_lo = bp.take<__nv_bfloat16>(3 * D.BH * D.d * D.d);
      }
    } else {
      b.Bf = bp.take<float>(3 * D.BH * D.d * D.d);
    }
    b.part = bp.take<float>(3 * D.BH * kNsBlocks);
  }
}

static size_t workspace_bytes(const Dims& D) {
  Bump bp{0, 0};
  Bufs b;
  plan(D, bp, b);
  return static_cast<size_t>(rup(static_cast<int64_t>(bp.off), 256));
}

// ------------------------------------------------------------------ TMA maps
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 3-D bf16 map over [batch][rows][inner] (dense), 128-byte swizzle,
// out-of-bounds elements read as zero.
static bool map3d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint64_t batch,
                  uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same map without swizzle: boxes are dense row-major in shared memory
// (used for bulk stores of narrow staging tiles).
static bool map3d_plain(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint64_t batch,
                        uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 map over [batch][rows][inner] (dense), 32 x 32 boxes with
// 128-byte swizzle (the fp32 staging tiles of bulk-store epilogues).
static bool map3d_f32(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint64_t batch) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner * 4, inner * rows * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launches
// Opt-in dynamic shared memory per CTA on sm_100 (227 KB).
constexpr int kMaxSmemPerBlock = 232448;
// Every kernel is launched with programmatic stream serialization: the
// next kernel of the stream may start while this one drains, does its local
// setup (barrier init, TMEM allocation, tensor-map prefetch), and waits in
// griddep_wait() for this one to finish before touching global memory.
template <class... KArgs, class... Args>
static cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// SMs of the current device (the persistent kernels launch one CTA per SM).
static int sm_count() {
  static int sms[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    sms[dev] = n;
  }
  return sms[dev];
}

template <class Op>
static cudaError_t launch_umma(int64_t ntiles, const typename Op::Params& p, cudaStream_t st) {
  constexpr int smem = umma_smem_bytes<Op>();
  static_assert(smem <= kMaxSmemPerBlock, "dynamic shared memory above the per-CTA limit");
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !attr_set[dev]) {
    e = cudaFuncSetAttribute(umma_kernel<Op>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  if (ntiles <= 0 || ntiles > (int64_t(1) << 31) - 1) return cudaErrorInvalidValue;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ntiles, sm_count()));
  (void)launch_pdl(umma_kernel<Op>, grid, umma_threads<Op>(), smem, st, p);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_apply(int64_t ntiles, const ApplyParams& p, cudaStream_t st) {
  constexpr int smem = ApplyCfg<D>::kSmem;
  static_assert(smem <= kMaxSmemPerBlock, "dynamic shared memory above the per-CTA limit");
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !attr_set[dev]) {
    e = cudaFuncSetAttribute(k_apply<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  if (ntiles <= 0 || ntiles > (int64_t(1) << 31) - 1) return cudaErrorInvalidValue;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ntiles, sm_count()));
  (void)launch_pdl(k_apply<D>, grid, kApplyThreads, smem, st, p);
  return cudaGetLastError();
}

static cudaError_t launch_key_grad(int64_t items, const KeyGradParams& p, cudaStream_t st) {
  constexpr int smem = KGCfg::kSmem;
  static_assert(smem <= kMaxSmemPerBlock, "dynamic shared memory above the per-CTA limit");
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !attr_set[dev]) {
    e = cudaFuncSetAttribute(k_key_grad64, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  if (items <= 0 || items > (int64_t(1) << 31) - 1) return cudaErrorInvalidValue;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(items, sm_count()));
  (void)launch_pdl(k_key_grad64, grid, kKGThreads, smem, st, p);
  return cudaGetLastError();
}

// CTA-pair kernels: one 2-CTA cluster per pair tile, up to one CTA per SM.
template <class Op>
static cudaError_t launch_pair(int64_t ntiles, const typename Op::Params& p, cudaStream_t st) {
  constexpr int smem = umma_pair_smem_bytes<Op>();
  static_assert(smem <= kMaxSmemPerBlock, "dynamic shared memory above the per-CTA limit");
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !attr_set[dev]) {
    e = cudaFuncSetAttribute(umma_pair_kernel<Op>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // Pairs that fit at once (a cluster's two CTAs share a GPC, so an SM can
  // be left without a partner).
  static int max_pairs[64] = {};
  if (dev < 64 && !max_pairs[dev]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sm_count() / 2));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, umma_pair_kernel<Op>, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = sm_count() / 2;
    }
    max_pairs[dev] = std::min(n, sm_count() / 2);
  }
  const int cap = dev < 64 ? max_pairs[dev] : sm_count() / 2;
  if (ntiles <= 0 || ntiles > (int64_t(1) << 30)) return cudaErrorInvalidValue;
  const unsigned pairs = static_cast<unsigned>(std::min<int64_t>(ntiles, cap));
  (void)launch_pdl(umma_pair_kernel<Op>, 2 * pairs, kThreads, smem, st, p);
  return cudaGetLastError();
}

// Pair GEMM: grid.y counts 256-row tiles.
template <bool A_MN, bool B_MN>
static cudaError_t launch_gemm_pair(int bn, dim3 grid, GemmParams p, cudaStream_t st) {
  p.nt_n = static_cast<int>(grid.x);
  p.nt_m = static_cast<int>(grid.y);
  const int64_t ntiles = int64_t(grid.x) * grid.y * grid.z;
  p.n_tiles = static_cast<int>(ntiles);
  switch (bn) {
    case 128: return launch_pair<GemmPairOp<A_MN, B_MN, 128>>(ntiles, p, st);
    case 256: return launch_pair<GemmPairOp<A_MN, B_MN, 256>>(ntiles, p, st);
    default: return cudaErrorInvalidValue;
  }
}

// grid = (tiles along N, tiles along M, splits * items), as a tile list.
template <bool A_MN, bool B_MN, bool SPLIT = false>
static cudaError_t launch_gemm(int bn, dim3 grid, GemmParams p, cudaStream_t st) {
  p.nt_n = static_cast<int>(grid.x);
  p.nt_m = static_cast<int>(grid.y);
  const int64_t ntiles = int64_t(grid.x) * grid.y * grid.z;
  p.n_tiles = static_cast<int>(ntiles);
  switch (bn) {
    case 64: return launch_umma<GemmOp<A_MN, B_MN, 64, SPLIT>>(ntiles, p, st);
    case 128: return launch_umma<GemmOp<A_MN, B_MN, 128, SPLIT>>(ntiles, p, st);
    case 192: return launch_umma<GemmOp<A_MN, B_MN, 192, SPLIT>>(ntiles, p, st);
    case 256: return launch_umma<GemmOp<A_MN, B_MN, 256, SPLIT>>(ntiles, p, st);
    default: return cudaErrorInvalidValue;
  }
}

template <bool A_MN, bool B_MN>
static cudaError_t launch_gemm_any(bool split, int bn, dim3 grid, const GemmParams& p, cudaStream_t st) {
  return split ? launch_gemm<A_MN, B_MN, true>(bn, grid, p, st) : launch_gemm<A_MN, B_MN, false>(bn, grid, p, st);
}

// Kernel kinds, for the launch profiler (lact_profile_*).
enum Kind {
  K_INIT, K_PROLOGUE, K_BETA_MEAN, K_FWD_QUERY, K_APPLY_OUT, K_FWD_KEY, K_GRAD, K_NS_SUMSQ,
  K_NS_SCALE, K_NS_GRAM, K_NS_POLY, K_NS_UPDATE, K_RULE, K_FINALIZE, K_SIMT_GEMM, K_FWD_ELEM_F32,
  K_APPLY_FUSED, K_KEY_GRAD, K_BWD_ELEM, K_BWD_GEMM, K_SWA, K_SWA_GEMM, K_SWA_FLASH, K_BWD_KEY, K_BWD_APPLY, K_COUNT
};
static const char* const kKindNames[K_COUNT] = {
    "init_state", "qk_prologue", "beta_mean", "fwd_query_umma", "apply_out_umma", "fwd_key_umma",
    "grad_umma", "ns_sumsq", "ns_scale", "ns_gram_umma", "ns_poly_umma", "ns_update_umma",
    "rule_renorm", "finalize_state", "simt_gemm_f32", "fwd_elem_f32", "apply_fused_umma",
    "key_grad_umma", "bwd_elem", "bwd_gemm_umma", "swa_elem", "swa_gemm_umma", "swa_flash_umma",
    "bwd_key_umma", "bwd_apply_umma"};

// Optional per-launch CUDA-event pairs on the launching stream.
struct ProfRec { int kind; cudaEvent_t a, b; };
static std::mutex g_prof_mu;
static bool g_prof_on = false;
static std::vector<ProfRec> g_prof;
static std::vector<cudaEvent_t> g_event_pool;

static cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

struct Launcher {
  bool dry;
  cudaStream_t st = nullptr;
  int64_t count = 0;
  int err = LACT_OK;
  template <class F> void operator()(int kind, F&& f) {
    ++count;
    if (dry || err != LACT_OK) return;
    cudaEvent_t a = nullptr, b = nullptr;
    std::unique_lock<std::mutex> lk(g_prof_mu, std::defer_lock);
    if (g_prof_on) {
      lk.lock();
      a = take_event();
      b = take_event();
      if (a && b) cudaEventRecord(a, st);
    }
    if (f() != cudaSuccess) err = LACT_ECUDA;
    if (a && b) {
      cudaEventRecord(b, st);
      g_prof.push_back({kind, a, b});
    }
  }
};

// Per host thread and device: a library-owned side stream and three events,
// used to run a chunk's apply concurrently with its key forward + gradient
// (both read only the previous state) in apply-then-update order.  Each
// thread has its own, so calls made at the same time from several threads
// never record over each other's events.  They live until the process exits.
struct SideRes {
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join[2] = {nullptr, nullptr};
};
static thread_local SideRes tl_side[64];

static const SideRes* side_resources() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideRes& r = tl_side[dev];
  if (!r.side) {
    if (cudaStreamCreateWithFlags(&r.side, cudaStreamNonBlocking) != cudaSuccess) return r.side = nullptr, nullptr;
    if (cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&r.join[0], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&r.join[1], cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
  }
  return &r;
}

struct Inputs {
  const void *q, *k, *v;
  const float *lr, *beta, *w1, *w2, *w3;
  void* out;
  float *w1o, *w2o, *w3o;
  // options (null = off)
  const uint8_t* mask;     // host, one byte per chunk: 0 = the chunk does not update
  const float* scale;      // [BH, Tq] output factors
  float *m1, *m2, *m3;     // momentum in/out
  lact_allreduce_fn allreduce;   // context-parallel reduction hook
  void* allreduce_user;
};

template <typename T, int VEC, int S, int MAXV>
static cudaError_t prologue_as(const Dims& D, const Bufs& b, const Inputs& in, cudaStream_t st) {
  constexpr int ROWS = 4;  // rows per thread group, loads issued together
  const int64_t rows = D.BH * D.Tq + D.BH * D.T;
  const unsigned blocks = static_cast<unsigned>(cdiv(cdiv(rows, ROWS) * S, 256));
  (void)launch_pdl(k_qk_prologue<T, VEC, S, MAXV, ROWS>, blocks, 256, 0, st, 
      static_cast<const T*>(in.q), static_cast<T*>(b.qh), D.BH * D.Tq, static_cast<const T*>(in.k),
      static_cast<T*>(b.kh), D.BH * D.T, static_cast<int>(D.d), reinterpret_cast<T*>(b.kh_lo));
  return cudaGetLastError();
}

template <int S, int MAXV>
static cudaError_t prologue_bf16(const Dims& D, const Bufs& b, const Inputs& in, cudaStream_t st) {
  constexpr int ROWS = 4;  // rows per lane group, loads issued together
  const int64_t rows = D.BH * D.Tq + D.BH * D.T;
  const unsigned blocks = static_cast<unsigned>(cdiv(cdiv(rows, ROWS) * S, 256));
  using B16 = __nv_bfloat16;
  auto kern = b.kh_lo ? k_qk_prologue_bf16<S, MAXV, ROWS, true> : k_qk_prologue_bf16<S, MAXV, ROWS, false>;
  (void)launch_pdl(kern, blocks, 256, 0, st, static_cast<const B16*>(in.q), static_cast<B16*>(b.qh),
                   D.BH * D.Tq, static_cast<const B16*>(in.k), static_cast<B16*>(b.kh), D.BH * D.T,
                   static_cast<int>(D.d), b.kh_lo);
  return cudaGetLastError();
}

// Rows of d elements: 16-byte vectors, S = the power of two >= vectors per
// row (at most a warp), MAXV vectors per thread.
static cudaError_t launch_prologue(const Dims& D, const Bufs& b, const Inputs& in, cudaStream_t st) {
  if (D.dtype == LACT_BF16) {
    const int nv = static_cast<int>(D.d / 8);  // d is a multiple of 64
    if (nv <= 8) return prologue_bf16<8, 1>(D, b, in, st);
    if (nv <= 16) return prologue_bf16<16, 1>(D, b, in, st);
    if (nv <= 32) return prologue_bf16<32, 1>(D, b, in, st);
    return prologue_bf16<32, 2>(D, b, in, st);
  }
  if (D.d % 4 == 0) return prologue_as<float, 4, 32, 4>(D, b, in, st);
  return prologue_as<float, 1, 32, 16>(D, b, in, st);
}

static GemmParams gemm_params() {
  GemmParams g;
  std::memset(&g, 0, sizeof(g));
  g.alt_group = -1;
  g.tr_group = -1;
  g.tr_mod = 1;
  g.alpha = 1.0f;
  return g;
}

static SimtGemmParams simt_params() {
  SimtGemmParams s;
  std::memset(&s, 0, sizeof(s));
  s.alt_a = -1;
  s.alt_b = -1;
  s.za_mod = 1 << 30;
  s.zb_mod = 1 << 30;
  s.tr_group = -1;
  s.tr_mod = 1;
  s.alpha = 1.0f;
  return s;
}

static cudaError_t simt(const SimtGemmParams& p, int items, cudaStream_t st) {
  (void)launch_pdl(k_simt_gemm, dim3(cdiv(p.N, 64), cdiv(p.M, 64), items), 256, 0, st, p);
  return cudaGetLastError();
}

static void run(const Dims& D, const Bufs& b, const Inputs& in, cudaStream_t main_st, Launcher& L,
                const SideRes* side) {
  cudaStream_t st = main_st;  // the stream the next launch goes to
  L.st = st;
  const bool bf = D.dtype == LACT_BF16;
  const int BH = static_cast<int>(D.BH), d = static_cast<int>(D.d), dh = static_cast<int>(D.dh);
  const int64_t plane = D.dh * D.d, planes = 3 * D.BH * plane;
  const unsigned state_blocks = static_cast<unsigned>(std::min<int64_t>(cdiv(planes, 1024), 148 * 16));
  // Context parallelism: reduce a buffer over the ranks, in place, ordered on
  // the main stream (the hook enqueues the collective there).
  auto reduce = [&](float* data, int64_t count, int op) {
    if (!in.allreduce || L.dry || L.err != LACT_OK) return;
    if (in.allreduce(data, count, op, static_cast<void*>(main_st), in.allreduce_user) != 0) L.err = LACT_ECOMM;
  };

  // Fast-weight masters (+ bf16 shadows), momentum = the caller's or 0.
  L(K_INIT, [&] {
    (void)launch_pdl(k_init_state, state_blocks, 256, 0, st, in.w1, in.w2, in.w3, static_cast<int>(D.H),
                     D.w_shared, BH, d, dh, b.Wm, b.Ws, b.Ws_lo, b.Mm, static_cast<const float*>(in.m1),
                     static_cast<const float*>(in.m2), static_cast<const float*>(in.m3));
    return cudaGetLastError();
  });
  // q^, k^ = silu + L2 norm rows.
  L(K_PROLOGUE, [&] { return launch_prologue(D, b, in, st); });
  if (D.rule == LACT_RULE_MOMENTUM) {
    // With context parallelism: per-chunk sums and token counts, added over
    // the ranks, then divided on the device.
    const int sums = in.allreduce ? 1 : 0;
    const int64_t w = D.BH * D.nch;
    L(K_BETA_MEAN, [&] {
      (void)launch_pdl(k_beta_mean, static_cast<unsigned>(cdiv(w * 32, 256)), 256, 0, st, in.beta, BH, D.T, D.chunk,
                       static_cast<int>(D.nch), b.bbar, sums);
      return cudaGetLastError();
    });
    if (sums) {
      reduce(b.bbar, 2 * w, LACT_REDUCE_SUM);
      L(K_BETA_MEAN, [&] {
        (void)launch_pdl(k_beta_div, static_cast<unsigned>(cdiv(w, 256)), 256, 0, st, b.bbar, w);
        return cudaGetLastError();
      });
    }
  }

  bool join_before_rule = false, side_used = false;
  // Updates done so far.  With two bf16 shadow sets the state after `ver`
  // updates is in set ver % 2; a chunk that does not update leaves it there.
  int64_t ver = 0;
  // Per shadow set: an apply that reads it was launched on the side stream
  // and the set's join event was recorded after it.
  bool set_joined[2] = {false, false};
  int last_join = 0;
  for (int64_t c = 0; c < D.nch; ++c) {
    const int64_t c0 = c * D.chunk;
    const int nc = static_cast<int>((c0 + D.chunk < D.T ? c0 + D.chunk : D.T) - c0);
    const int64_t qr0 = D.nch == 1 ? 0 : c0;
    const int nq = static_cast<int>(D.nch == 1 ? D.Tq : nc);
    const bool upd = !in.mask || in.mask[c] != 0;
    // bf16 shadows of the current state (read by this chunk's kernels) and
    // of the next one (written by its rule): with two sets, chunk c's apply
    // may still run while chunk c's rule writes the other set.
    const int64_t cur = D.dbuf ? (ver & 1) : 0, nxt = D.dbuf ? 1 - cur : 0;
    __nv_bfloat16* const Wsc = b.Ws ? b.Ws + cur * planes : nullptr;
    __nv_bfloat16* const Wsc_lo = b.Ws_lo ? b.Ws_lo + cur * planes : nullptr;
    __nv_bfloat16* const Wsn = b.Ws ? b.Ws + nxt * planes : nullptr;
    __nv_bfloat16* const Wsn_lo = b.Ws_lo ? b.Ws_lo + nxt * planes : nullptr;

    auto apply = [&] {
      if (bf && d <= 256) {
        L(K_APPLY_FUSED, [&] {
          ApplyParams a;
          std::memset(&a, 0, sizeof(a));
          if (!map3d(&a.tmQ, b.qh, d, D.Tq, BH, 64, 128) || !map3d(&a.tmW, Wsc, d, dh, 3 * BH, 64, 64) ||
              !map3d(&a.tmW2, Wsc + D.BH * plane, dh, d, BH, 64, d))
            return cudaErrorInvalidValue;
          a.bh_count = BH; a.dh = dh; a.n_row_tiles = static_cast<int>(cdiv(nq, 128));
          a.q_row0 = static_cast<int>(qr0); a.rows_valid = nq;
          a.out = static_cast<__nv_bfloat16*>(in.out); a.Tq = D.Tq; a.scale = in.scale;
          const int64_t tiles = int64_t(a.n_row_tiles) * BH;
          switch (d) {
            case 64: return launch_apply<64>(tiles, a, st);
            case 128: return launch_apply<128>(tiles, a, st);
            case 192: return launch_apply<192>(tiles, a, st);
            default: return launch_apply<256>(tiles, a, st);
          }
        });
      } else if (bf) {
        L(K_FWD_QUERY, [&] {
          FwdParams f;
          std::memset(&f, 0, sizeof(f));
          if (!map3d(&f.tmX, b.qh, d, D.Tq, BH, 64, 128) || !map3d(&f.tmW, Wsc, d, dh, 3 * BH, 64, 64))
            return cudaErrorInvalidValue;
          f.bh_count = BH; f.x_row0 = static_cast<int>(qr0); f.rows_valid = nq; f.kb_count = d / 64;
          f.dh = dh; f.T = static_cast<int>(D.T); f.hq = static_cast<__nv_bfloat16*>(b.Hq);
          f.buf_rows = D.q_rows; f.lr = in.lr;
          const bool wide = dh % 128 == 0;                    // 128-wide hidden slices
          f.n_slices = dh / (wide ? 128 : 64); f.n_row_tiles = static_cast<int>(cdiv(nq, 128));
          if (wide && !map3d(&f.tmW, Wsc, d, dh, 3 * BH, 64, 128)) return cudaErrorInvalidValue;
          const int64_t tiles = int64_t(f.n_slices) * f.n_row_tiles * BH;
          return wide ? launch_umma<FwdOp<false, false, 128>>(tiles, f, st)
                      : launch_umma<FwdOp<false>>(tiles, f, st);
        });
        L(K_APPLY_OUT, [&] {
          GemmParams g = gemm_params();
          if (!map3d(&g.tmA, b.Hq, dh, D.q_rows, BH, 64, 128) ||
              !map3d(&g.tmB, Wsc + D.BH * plane, dh, d, BH, 64, D.bn))
            return cudaErrorInvalidValue;
          g.items = BH; g.kb_count = dh / 64; g.kb_total = g.kb_count;
          g.zb_mod = BH; g.zb_add = 0; g.m_valid = nq;
          g.outb = static_cast<__nv_bfloat16*>(in.out) + qr0 * d;
          g.item_stride = D.Tq * D.d; g.ld = d;
          g.row_scale = in.scale ? in.scale + qr0 : nullptr; g.rs_item = D.Tq;
          return launch_gemm<false, false>(D.bn, dim3(d / D.bn, cdiv(nq, 128), BH), g, st);
        });
      } else {
        float* Z = b.Z;
        const int64_t zpl = D.BH * D.q_rows * D.dh;
        for (int j = 0; j < 3; j += 2) {
          L(K_SIMT_GEMM, [&] {
            SimtGemmParams s = simt_params();
            s.A = static_cast<const float*>(b.qh) + qr0 * d; s.a_item = D.Tq * D.d; s.a_m = d; s.a_k = 1;
            s.B = b.Wm + j * D.BH * plane; s.b_item = plane; s.b_n = d; s.b_k = 1;
            s.M = nq; s.N = dh; s.K = d;
            s.outf = Z + j * zpl; s.item_stride = D.q_rows * D.dh; s.ld = dh;
            return simt(s, BH, st);
          });
        }
        L(K_FWD_ELEM_F32, [&] {
          const int64_t n = zpl;
          (void)launch_pdl(k_fwd_elem_f32, static_cast<unsigned>(cdiv(n, 256)), 256, 0, st, 
              Z, BH, D.q_rows, dh, nq, 0, nullptr, D.T, 0, static_cast<float*>(b.Hq));
          return cudaGetLastError();
        });
        L(K_SIMT_GEMM, [&] {
          SimtGemmParams s = simt_params();
          s.A = static_cast<const float*>(b.Hq); s.a_item = D.q_rows * D.dh; s.a_m = dh; s.a_k = 1;
          s.B = b.Wm + D.BH * plane; s.b_item = plane; s.b_n = dh; s.b_k = 1;   // W2[i][r]
          s.M = nq; s.N = d; s.K = dh;
          s.outf = static_cast<float*>(in.out) + qr0 * d; s.item_stride = D.Tq * D.d; s.ld = d;
          s.row_scale = in.scale ? in.scale + qr0 : nullptr; s.rs_item = D.Tq;
          return simt(s, BH, st);
        });
      }
    };

    auto update = [&] {
      int splits = 1;
      if (bf && D.fused_kg) {
        const int tiles = static_cast<int>(cdiv(nc, 128));
        int ks = std::min(D.kg_splits, tiles);
        const int tps = static_cast<int>(cdiv(tiles, ks));
        ks = static_cast<int>(cdiv(tiles, tps));
        splits = ks;
        L(K_KEY_GRAD, [&] {
          KeyGradParams k;
          std::memset(&k, 0, sizeof(k));
          if (!map3d(&k.tmK, b.kh, d, D.T, BH, 64, 128) || !map3d(&k.tmV, in.v, d, D.T, BH, 64, 128) ||
              !map3d(&k.tmW, Wsc, d, dh, 3 * BH, 64, 64) ||
              !map3d(&k.tmW2, Wsc + D.BH * plane, dh, d, BH, 64, 64))
            return cudaErrorInvalidValue;
          k.bh_count = BH; k.splits = ks; k.n_tiles = tiles; k.x_row0 = static_cast<int>(c0);
          k.rows_valid = nc; k.T = static_cast<int>(D.T); k.lr = in.lr; k.P = b.P;
          return launch_key_grad(int64_t(BH) * ks, k, st);
        });
      } else if (bf) {
        L(K_FWD_KEY, [&] {
          FwdParams f;
          std::memset(&f, 0, sizeof(f));
          if (!map3d(&f.tmX, b.kh, d, D.T, BH, 64, 128) || !map3d(&f.tmV, in.v, d, D.T, BH, 64, 128) ||
              !map3d(&f.tmW, Wsc, d, dh, 3 * BH, 64, 64))
            return cudaErrorInvalidValue;
          if (!map3d(&f.tmW2, Wsc + D.BH * plane, dh, d, BH, 64, 64)) return cudaErrorInvalidValue;
          if (D.split && (!map3d(&f.tmXlo, b.kh_lo, d, D.T, BH, 64, 128) ||
                          !map3d(&f.tmWlo, Wsc_lo, d, dh, 3 * BH, 64, 64) ||
                          !map3d(&f.tmW2lo, Wsc_lo + D.BH * plane, dh, d, BH, 64, 64)))
            return cudaErrorInvalidValue;
          f.bh_count = BH; f.x_row0 = static_cast<int>(c0); f.rows_valid = nc; f.kb_count = d / 64;
          f.dh = dh; f.T = static_cast<int>(D.T); f.e = static_cast<__nv_bfloat16*>(b.E);
          f.e_lo = static_cast<__nv_bfloat16*>(b.E_lo);
          f.buf_rows = D.key_rows; f.lr = in.lr;
          // 128-wide hidden slices (Z MMAs of N = 256) unless split mode needs the smem.
          // 64-wide hidden slices: double-buffered TMEM and TMA-stored E measured
          // faster than 128-wide ones (N = 256 MMAs, single-buffered), and than
          // 256-token x 128-unit tiles on CTA pairs (half the weight bytes per
          // CTA, but one accumulator buffer: 53.8 against 43.2 us per chunk at
          // d 256, dh 512, 12 heads).
          const bool wide = false;
          if (!D.split && !map3d(&f.tmE, b.E, dh, D.key_rows, 3 * BH, 64, 32)) return cudaErrorInvalidValue;
          f.n_slices = dh / (wide ? 128 : 64); f.n_row_tiles = static_cast<int>(cdiv(nc, 128));
          if (wide && !map3d(&f.tmW, Wsc, d, dh, 3 * BH, 64, 128)) return cudaErrorInvalidValue;
          const int64_t tiles = int64_t(f.n_slices) * f.n_row_tiles * BH;
          if (D.split) return launch_umma<FwdOp<true, true>>(tiles, f, st);
          return wide ? launch_umma<FwdOp<true, false, 128>>(tiles, f, st) : launch_umma<FwdOp<true>>(tiles, f, st);
        });
      }
      if (bf && !D.fused_kg) {
        const int kbt = static_cast<int>(cdiv(nc, 64));
        const int kbp = static_cast<int>(cdiv(kbt, D.splits));
        splits = static_cast<int>(cdiv(kbt, kbp));
        L(K_GRAD, [&] {
          GemmParams g = gemm_params();
          if (!map3d(&g.tmA, b.E, dh, D.key_rows, 3 * BH, 64, 64) || !map3d(&g.tmB, b.kh, d, D.T, BH, 64, 64) ||
              !map3d(&g.tmB2, in.v, d, D.T, BH, 64, 64))
            return cudaErrorInvalidValue;
          if (D.split && (!map3d(&g.tmAlo, b.E_lo, dh, D.key_rows, 3 * BH, 64, 64) ||
                          !map3d(&g.tmBlo, b.kh_lo, d, D.T, BH, 64, 64)))
            return cudaErrorInvalidValue;
          g.items = 3 * BH; g.kb_count = kbp; g.kb_total = kbt;
          g.a_k0 = 0; g.b_k0 = static_cast<int>(c0);
          g.zb_mod = BH; g.zb_add = 0; g.alt_group = 1; g.m_valid = dh;
          g.outf = b.P; g.item_stride = plane; g.ld = d;
          if (D.rule != LACT_RULE_MUON) {  // W2's gradient straight into its [d, dh] layout
            g.tr_group = 1; g.tr_mod = BH; g.ld_t = dh;
          }
          if (!D.split && (D.bn == 128 || D.bn == 256)) {  // 256-row pair tiles over dh
            // the partial planes leave through bulk tensor stores: W1's and
            // W3's as [dh, d], W2's transposed into [d, dh]
            const uint64_t nplanes = static_cast<uint64_t>(splits) * 3 * BH;
            if (g.tr_group == 1) {
              if (!map3d_f32(&g.tmOut, b.P, d, dh, nplanes) || !map3d_f32(&g.tmOutT, b.P, dh, d, nplanes))
                return cudaErrorInvalidValue;
              g.out_tma = 1;
            }
            return launch_gemm_pair<true, true>(D.bn, dim3(d / D.bn, cdiv(dh, 256), splits * 3 * BH), g, st);
          }
          return launch_gemm_any<true, true>(D.split, D.bn, dim3(d / D.bn, cdiv(dh, 128), splits * 3 * BH), g, st);
        });
      } else if (!bf) {
        const int64_t zpl = D.BH * D.key_rows * D.dh;
        for (int j = 0; j < 3; ++j) {
          L(K_SIMT_GEMM, [&] {
            SimtGemmParams s = simt_params();
            s.A = (j == 1 ? static_cast<const float*>(in.v) : static_cast<const float*>(b.kh)) + c0 * d;
            s.a_item = D.T * D.d; s.a_m = d; s.a_k = 1;
            s.B = b.Wm + j * D.BH * plane; s.b_item = plane;
            s.b_n = j == 1 ? 1 : d; s.b_k = j == 1 ? dh : 1;   // W2[a][r] for DH = V W2
            s.M = nc; s.N = dh; s.K = d;
            s.outf = b.Z + j * zpl; s.item_stride = D.key_rows * D.dh; s.ld = dh;
            return simt(s, BH, st);
          });
        }
        L(K_FWD_ELEM_F32, [&] {
          (void)launch_pdl(k_fwd_elem_f32, static_cast<unsigned>(cdiv(zpl, 256)), 256, 0, st, 
              b.Z, BH, D.key_rows, dh, nc, 1, in.lr, D.T, c0, static_cast<float*>(b.E));
          return cudaGetLastError();
        });
        L(K_SIMT_GEMM, [&] {
          SimtGemmParams s = simt_params();
          s.A = static_cast<const float*>(b.E); s.a_item = D.key_rows * D.dh; s.a_m = 1; s.a_k = dh;
          s.B = static_cast<const float*>(b.kh) + c0 * d; s.B2 = static_cast<const float*>(in.v) + c0 * d;
          s.b_item = D.T * D.d; s.b_n = 1; s.b_k = d; s.zb_mod = BH; s.alt_b = 1;
          s.M = dh; s.N = d; s.K = nc;
          s.outf = b.P; s.item_stride = plane; s.ld = d;
          if (D.rule != LACT_RULE_MUON) {
            s.tr_group = 1; s.tr_mod = BH; s.ld_t = dh;
          }
          return simt(s, 3 * BH, st);
        });
      }

      // the chunk's gradient is the sum of every rank's partial planes
      reduce(b.P, static_cast<int64_t>(splits) * planes, LACT_REDUCE_SUM);
      const float* dir = b.P;
      int dir_splits = splits;
      if (D.rule == LACT_RULE_MUON) {
        L(K_NS_SUMSQ, [&] {
          (void)launch_pdl(k_ns_sumsq, dim3(kNsBlocks, 3 * BH), 256, 0, st, b.P, splits, planes, plane, b.Yf[0], b.part);
          return cudaGetLastError();
        });
        L(K_NS_SCALE, [&] {
          (void)launch_pdl(k_ns_scale, dim3(kNsBlocks, 3 * BH), 256, 0, st, b.Yf[0], b.Yb[0], b.Yb_lo[0], plane, b.part,
                                                              kNsBlocks, kNsEps);
          return cudaGetLastError();
        });
        for (int it = 0; it < kNsSteps; ++it) {
          const int cur = it & 1, nxt = cur ^ 1;
          if (bf) {
            L(K_NS_GRAM, [&] {  // A = X^T X  (d x d, K = dh)
              GemmParams g = gemm_params();
              if (!map3d(&g.tmA, b.Yb[cur], d, dh, 3 * BH, 64, 64)) return cudaErrorInvalidValue;
              g.tmB = g.tmA;
              if (D.split) {
                if (!map3d(&g.tmAlo, b.Yb_lo[cur], d, dh, 3 * BH, 64, 64)) return cudaErrorInvalidValue;
                g.tmBlo = g.tmAlo;
              }
              g.items = 3 * BH; g.kb_count = g.kb_total = static_cast<int>(cdiv(dh, 64));
              g.zb_mod = 3 * BH; g.m_valid = d;
              g.outf = b.Af; g.outb = b.Ab; g.outb_lo = b.Ab_lo; g.item_stride = D.d * D.d; g.ld = d;
              return launch_gemm_any<true, true>(D.split, D.bn, dim3(d / D.bn, cdiv(d, 128), 3 * BH), g, st);
            });
            L(K_NS_POLY, [&] {  // B = b A + c A A
              GemmParams g = gemm_params();
              if (!map3d(&g.tmA, b.Ab, d, d, 3 * BH, 64, 128) || !map3d(&g.tmB, b.Ab, d, d, 3 * BH, 64, D.bn))
                return cudaErrorInvalidValue;
              if (D.split && (!map3d(&g.tmAlo, b.Ab_lo, d, d, 3 * BH, 64, 128) ||
                              !map3d(&g.tmBlo, b.Ab_lo, d, d, 3 * BH, 64, D.bn)))
                return cudaErrorInvalidValue;
              g.items = 3 * BH; g.kb_count = g.kb_total = d / 64;
              g.zb_mod = 3 * BH; g.m_valid = d;
              g.alpha = kNsC; g.beta = kNsB; g.cin = b.Af;
              g.outb = b.Bb; g.outb_lo = b.Bb_lo; g.item_stride = D.d * D.d; g.ld = d;
              return launch_gemm_any<false, false>(D.split, D.bn, dim3(d / D.bn, cdiv(d, 128), 3 * BH), g, st);
            });
            L(K_NS_UPDATE, [&] {  // X <- a X + X B
              GemmParams g = gemm_params();
              if (!map3d(&g.tmA, b.Yb[cur], d, dh, 3 * BH, 64, 128) ||
                  !map3d(&g.tmB, b.Bb, d, d, 3 * BH, 64, D.bn))
                return cudaErrorInvalidValue;
              if (D.split && (!map3d(&g.tmAlo, b.Yb_lo[cur], d, dh, 3 * BH, 64, 128) ||
                              !map3d(&g.tmBlo, b.Bb_lo, d, d, 3 * BH, 64, D.bn)))
                return cudaErrorInvalidValue;
              g.items = 3 * BH; g.kb_count = g.kb_total = d / 64;
              g.zb_mod = 3 * BH; g.m_valid = dh;
              g.alpha = 1.0f; g.beta = kNsA; g.cin = b.Yf[cur];
              g.outf = b.Yf[nxt]; g.outb = b.Yb[nxt]; g.outb_lo = b.Yb_lo[nxt]; g.item_stride = plane; g.ld = d;
              if (it == kNsSteps - 1) {  // W2's update back in its [d, dh] layout
                g.tr_group = 1; g.tr_mod = BH; g.ld_t = dh;
              }
              return launch_gemm_any<false, false>(D.split, D.bn, dim3(d / D.bn, cdiv(dh, 128), 3 * BH), g, st);
            });
          } else {
            L(K_SIMT_GEMM, [&] {
              SimtGemmParams s = simt_params();
              s.A = b.Yf[cur]; s.a_item = plane; s.a_m = 1; s.a_k = d;
              s.B = b.Yf[cur]; s.b_item = plane; s.b_n = 1; s.b_k = d;
              s.M = d; s.N = d; s.K = dh;
              s.outf = b.Af; s.item_stride = D.d * D.d; s.ld = d;
              return simt(s, 3 * BH, st);
            });
            L(K_SIMT_GEMM, [&] {
              SimtGemmParams s = simt_params();
              s.A = b.Af; s.a_item = D.d * D.d; s.a_m = d; s.a_k = 1;
              s.B = b.Af; s.b_item = D.d * D.d; s.b_n = 1; s.b_k = d;
              s.M = d; s.N = d; s.K = d;
              s.alpha = kNsC; s.beta = kNsB; s.cin = b.Af;
              s.outf = b.Bf; s.item_stride = D.d * D.d; s.ld = d;
              return simt(s, 3 * BH, st);
            });
            L(K_SIMT_GEMM, [&] {
              SimtGemmParams s = simt_params();
              s.A = b.Yf[cur]; s.a_item = plane; s.a_m = d; s.a_k = 1;
              s.B = b.Bf; s.b_item = D.d * D.d; s.b_n = 1; s.b_k = d;
              s.M = dh; s.N = d; s.K = d;
              s.alpha = 1.0f; s.beta = kNsA; s.cin = b.Yf[cur];
              s.outf = b.Yf[nxt]; s.item_stride = plane; s.ld = d;
              if (it == kNsSteps - 1) {
                s.tr_group = 1; s.tr_mod = BH; s.ld_t = dh;
              }
              return simt(s, 3 * BH, st);
            });
          }
        }
        dir = b.Yf[kNsSteps & 1];
        dir_splits = 1;
      }
      if (join_before_rule) {
        // the rule rewrites the shadow set that the applies of the previous
        // state (two sets) or of this chunk (one set) read
        if (set_joined[nxt] && L.err == LACT_OK &&
            cudaStreamWaitEvent(main_st, side->join[nxt], 0) != cudaSuccess)
          L.err = LACT_ECUDA;
        join_before_rule = false;
      }
      L(K_RULE, [&] {
        RuleParams r;
        std::memset(&r, 0, sizeof(r));
        r.Wm = b.Wm; r.Ws = Wsn; r.Ws_lo = Wsn_lo; r.S = dir; r.splits = dir_splits; r.split_stride = planes;
        r.Mm = b.Mm; r.beta_bar = b.bbar; r.nch = static_cast<int>(D.nch); r.chunk_idx = static_cast<int>(c);
        r.rule = D.rule; r.BH = BH; r.dh = dh; r.d = d;
        const int64_t rows = 2 * D.BH * D.dh + D.BH * D.d;
        const unsigned grid = static_cast<unsigned>(cdiv(rows * 32, 256));
        const int64_t longest = std::max(D.d, D.dh);
        if (D.d % 4 != 0 || D.dh % 4 != 0 || longest > 128 * 8)
          (void)launch_pdl(k_rule_renorm, grid, 256, 0, st, r);
        else if (longest <= 128 * 2)
          (void)launch_pdl(k_rule_renorm_v4<2, 1>, grid, 256, 0, st, r);
        else if (longest <= 128 * 4)
          (void)launch_pdl(k_rule_renorm_v4<4, 1>, grid, 256, 0, st, r);
        else
          (void)launch_pdl(k_rule_renorm_v4<8, 1>, grid, 256, 0, st, r);
        return cudaGetLastError();
      });
    };

    if (D.order == LACT_APPLY_THEN_UPDATE && side && bf && !L.dry) {
      side_used = true;
      // apply on the side stream, concurrently with the key forward and the
      // gradient; joined before the rule rewrites the state.
      if (L.err == LACT_OK && (cudaEventRecord(side->fork, main_st) != cudaSuccess ||
                               cudaStreamWaitEvent(side->side, side->fork, 0) != cudaSuccess))
        L.err = LACT_ECUDA;
      st = side->side;
      L.st = st;
      apply();
      if (L.err == LACT_OK && cudaEventRecord(side->join[cur], side->side) != cudaSuccess) L.err = LACT_ECUDA;
      set_joined[cur] = true;
      last_join = static_cast<int>(cur);
      st = main_st;
      L.st = st;
      if (upd) {
        join_before_rule = true;
        update();
      }
    } else if (D.order == LACT_APPLY_THEN_UPDATE) {
      apply();
      if (upd) update();
    } else {
      if (upd) update();
      apply();
    }
    if (upd) ++ver;
  }

  // The last chunks' applies are done before the call's work ends, also when
  // a launch failed after an apply was forked: the side stream may still read
  // or write the caller's buffers, which the caller may free once the call
  // returns.  The first error code is kept.
  if (side_used) {
    const bool joined_ok = cudaEventRecord(side->join[last_join], side->side) == cudaSuccess &&
                           cudaStreamWaitEvent(main_st, side->join[last_join], 0) == cudaSuccess;
    if (!joined_ok && L.err == LACT_OK) L.err = LACT_ECUDA;
  }
  L(K_FINALIZE, [&] {
    (void)launch_pdl(k_finalize_state, state_blocks, 256, 0, st, b.Wm, BH, d, dh, in.w1o, in.w2o, in.w3o,
                     static_cast<const float*>(b.Mm), in.m1, in.m2, in.m3);
    return cudaGetLastError();
  });
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

static int check_pointers(const Dims& D, const Inputs& in) {
  const void* need[] = {in.q, in.k, in.v, in.lr, in.w1, in.w2, in.w3, in.out, in.w1o, in.w2o, in.w3o};
  for (const void* p : need)
    if (!p || !aligned16(p)) return LACT_EINVAL;
  if (D.rule == LACT_RULE_MOMENTUM && (!in.beta || !aligned16(in.beta))) return LACT_EINVAL;
  const size_t wn = static_cast<size_t>((D.w_shared ? D.H : D.BH) * D.d * D.dh) * 4;
  const size_t won = static_cast<size_t>(D.BH * D.d * D.dh) * 4;
  const float* ins[3] = {in.w1, in.w2, in.w3};
  const float* outs[3] = {in.w1o, in.w2o, in.w3o};
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) {
      if (!overlaps(outs[i], won, ins[j], wn)) continue;
      // Exact in-place aliasing of the matching matrix is allowed for
      // per-(b,h) initial states; any other overlap is rejected.
      if (!(i == j && outs[i] == ins[j] && wn == won)) return LACT_EINVAL;
    }
  for (int i = 0; i < 3; ++i)
    for (int j = i + 1; j < 3; ++j)
      if (overlaps(outs[i], won, outs[j], won)) return LACT_EINVAL;
  const size_t on = static_cast<size_t>(D.BH * D.Tq * D.d) * (D.dtype == LACT_BF16 ? 2 : 4);
  for (int i = 0; i < 3; ++i)
    if (overlaps(in.out, on, outs[i], won)) return LACT_EINVAL;
  return LACT_OK;
}

// Options of lact_ttt_fwd_ex: momentum buffers all or none, momentum rule
// only, aligned, and no overlap of an option buffer with a buffer the call
// writes (or, for the in-place momentum, with the initial weights).
static int check_options(const Dims& D, const Inputs& in) {
  const size_t won = static_cast<size_t>(D.BH * D.d * D.dh) * 4;
  const size_t wn = static_cast<size_t>((D.w_shared ? D.H : D.BH) * D.d * D.dh) * 4;
  const size_t on = static_cast<size_t>(D.BH * D.Tq * D.d) * (D.dtype == LACT_BF16 ? 2 : 4);
  const void* wouts[4] = {in.out, in.w1o, in.w2o, in.w3o};
  const size_t wout_n[4] = {on, won, won, won};
  const bool any_m = in.m1 || in.m2 || in.m3;
  const float* ms[3] = {in.m1, in.m2, in.m3};
  if (any_m) {
    if (!in.m1 || !in.m2 || !in.m3 || D.rule != LACT_RULE_MOMENTUM) return LACT_EINVAL;
    const float* wins[3] = {in.w1, in.w2, in.w3};
    for (int i = 0; i < 3; ++i) {
      if (!aligned16(ms[i])) return LACT_EINVAL;
      for (int j = i + 1; j < 3; ++j)
        if (overlaps(ms[i], won, ms[j], won)) return LACT_EINVAL;
      for (int j = 0; j < 4; ++j)
        if (overlaps(ms[i], won, wouts[j], wout_n[j])) return LACT_EINVAL;
      for (int j = 0; j < 3; ++j)
        if (overlaps(ms[i], won, wins[j], wn)) return LACT_EINVAL;
    }
  }
  if (in.scale) {
    if ((reinterpret_cast<uintptr_t>(in.scale) & 3u) != 0) return LACT_EINVAL;
    const size_t sn = static_cast<size_t>(D.BH * D.Tq) * 4;
    for (int j = 0; j < 4; ++j)
      if (overlaps(in.scale, sn, wouts[j], wout_n[j])) return LACT_EINVAL;
    for (int i = 0; any_m && i < 3; ++i)
      if (overlaps(in.scale, sn, ms[i], won)) return LACT_EINVAL;
  }
  return LACT_OK;
}

static void set_options(Inputs& in, const lact_fwd_opts* o) {
  in.mask = o ? o->update_mask : nullptr;
  in.scale = o ? o->out_scale : nullptr;
  in.m1 = o ? o->m1 : nullptr;
  in.m2 = o ? o->m2 : nullptr;
  in.m3 = o ? o->m3 : nullptr;
  in.allreduce = o ? o->allreduce : nullptr;
  in.allreduce_user = o ? o->allreduce_user : nullptr;
}

static int input_bytes(const Dims& D, size_t sz[8]) {
  const size_t e = D.dtype == LACT_BF16 ? 2 : 4;
  const size_t hw = static_cast<size_t>(D.w_shared ? D.H : D.BH);
  sz[0] = static_cast<size_t>(D.BH * D.Tq * D.d) * e;
  sz[1] = static_cast<size_t>(D.BH * D.T * D.d) * e;
  sz[2] = sz[1];
  sz[3] = static_cast<size_t>(D.BH * D.T * 3) * 4;
  sz[4] = D.rule == LACT_RULE_MOMENTUM ? static_cast<size_t>(D.BH * D.T) * 4 : 0;
  sz[5] = hw * D.dh * D.d * 4;
  sz[6] = sz[5];
  sz[7] = sz[5];
  return 0;
}

// Scratch of lact_ttt_fwd_noalloc: a file-scope device buffer, so callers
// that may not allocate still get a workspace.  Host code must not use the
// symbol itself as a device address; the address is looked up for the
// current device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[LACT_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.  Looked up on
// every call (a lookup allocates nothing): after a device reset the module
// is loaded again and the buffer may sit at another address, so a cached
// address could go stale.
static int noalloc_scratch(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return LACT_ECUDA;
  *out = ptr;
  return LACT_OK;
}

// One thread waits on a barrier that expects one arrival nobody makes.
// The budget is the kernel's own argument, so calls running at the same
// time keep their normal budget.
__global__ void k_selftest_wait(long long budget) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait_for(&bar, 0, budget);
  }
}

}  // namespace lact

#include "lact_bwd.cuh"
#include "lact_swa.cuh"

using namespace lact;

extern "C" {

size_t lact_ttt_workspace_bytes(const lact_problem* p) {
  Dims D;
  if (validate(p, D) != LACT_OK) return 0;
  return workspace_bytes(D);
}

int64_t lact_ttt_launch_count_ex(const lact_problem* p, const lact_fwd_opts* opts) {
  Dims D;
  if (validate(p, D) != LACT_OK) return 0;
  Bump bp{0, 0};
  Bufs b;
  plan(D, bp, b);
  Inputs in;
  std::memset(&in, 0, sizeof(in));
  // the options that change the launches: the update mask, and the
  // context-parallel hook (the momentum rule's beta means then take a
  // second kernel)
  in.mask = opts ? opts->update_mask : nullptr;
  in.allreduce = opts ? opts->allreduce : nullptr;
  Launcher L{true, nullptr};
  run(D, b, in, nullptr, L, nullptr);
  return L.count;
}

int64_t lact_ttt_launch_count(const lact_problem* p) { return lact_ttt_launch_count_ex(p, nullptr); }

static int ttt_fwd_impl(const lact_problem* p, const lact_fwd_opts* opts, const void* q,
                        const void* k, const void* v, const float* lr, const float* beta,
                        const float* w1, const float* w2, const float* w3, void* out,
                        float* w1_out, float* w2_out, float* w3_out, void* workspace,
                        size_t workspace_bytes_, void* stream, bool allow_side) {
  Dims D;
  int rc = validate(p, D);
  if (rc != LACT_OK) return rc;
  Inputs in;
  std::memset(&in, 0, sizeof(in));
  in.q = q; in.k = k; in.v = v; in.lr = lr; in.beta = beta; in.w1 = w1; in.w2 = w2; in.w3 = w3;
  in.out = out; in.w1o = w1_out; in.w2o = w2_out; in.w3o = w3_out;
  set_options(in, opts);
  rc = check_pointers(D, in);
  if (rc != LACT_OK) return rc;
  rc = check_options(D, in);
  if (rc != LACT_OK) return rc;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LACT_EINVAL;
  if (workspace_bytes_ < workspace_bytes(D)) return LACT_ENOSPC;
  if (D.dtype == LACT_BF16 && !encode_fn()) return LACT_ECUDA;
  Bump bp{reinterpret_cast<uintptr_t>(workspace), 0};
  Bufs b;
  plan(D, bp, b);
  Launcher L{false, static_cast<cudaStream_t>(stream)};
  bool profiling;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    profiling = g_prof_on;
  }
  // While the launch profiler is on, every launch goes to the caller's
  // stream, one after another, so each event pair times one kernel alone.
  const SideRes* side = (allow_side && !profiling) ? side_resources() : nullptr;
  run(D, b, in, static_cast<cudaStream_t>(stream), L, side);
  return L.err;
}

int lact_ttt_fwd(const lact_problem* p, const void* q, const void* k, const void* v, const float* lr,
                 const float* beta, const float* w1, const float* w2, const float* w3, void* out,
                 float* w1_out, float* w2_out, float* w3_out, void* workspace, size_t workspace_bytes_,
                 void* stream) {
  return ttt_fwd_impl(p, nullptr, q, k, v, lr, beta, w1, w2, w3, out, w1_out, w2_out, w3_out, workspace,
                      workspace_bytes_, stream, true);
}

int lact_ttt_fwd_ex(const lact_problem* p, const lact_fwd_opts* opts, const void* q, const void* k,
                    const void* v, const float* lr, const float* beta, const float* w1,
                    const float* w2, const float* w3, void* out, float* w1_out, float* w2_out,
                    float* w3_out, void* workspace, size_t workspace_bytes_, void* stream) {
  return ttt_fwd_impl(p, opts, q, k, v, lr, beta, w1, w2, w3, out, w1_out, w2_out, w3_out, workspace,
                      workspace_bytes_, stream, true);
}

int lact_ttt_fwd_noalloc(const lact_problem* p, const void* q, const void* k, const void* v,
                         const float* lr, const float* beta, const float* w1, const float* w2,
                         const float* w3, void* out, float* w1_out, float* w2_out, float* w3_out,
                         void* stream) {
  Dims D;
  int rc = validate(p, D);
  if (rc != LACT_OK) return rc;
  if (workspace_bytes(D) > LACT_NOALLOC_SCRATCH_BYTES) return LACT_ETOOBIG;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != LACT_OK) return rc;
  return ttt_fwd_impl(p, nullptr, q, k, v, lr, beta, w1, w2, w3, out, w1_out, w2_out, w3_out, scratch,
                      LACT_NOALLOC_SCRATCH_BYTES, stream, false);
}

size_t lact_ttt_host_workspace_bytes(const lact_problem* p) {
  Dims D;
  if (validate(p, D) != LACT_OK) return 0;
  size_t sz[8];
  input_bytes(D, sz);
  size_t total = workspace_bytes(D);
  for (size_t s : sz) total += (s + 255) / 256 * 256;
  const size_t e = D.dtype == LACT_BF16 ? 2 : 4;
  total += (static_cast<size_t>(D.BH * D.Tq * D.d) * e + 255) / 256 * 256;
  total += 3 * ((static_cast<size_t>(D.BH * D.d * D.dh) * 4 + 255) / 256 * 256);
  return total;
}

int lact_ttt_fwd_host(const lact_problem* p, const void* q, const void* k, const void* v,
                      const float* lr, const float* beta, const float* w1, const float* w2,
                      const float* w3, void* out, float* w1_out, float* w2_out, float* w3_out,
                      void* workspace, size_t workspace_bytes_, void* stream) {
  Dims D;
  int rc = validate(p, D);
  if (rc != LACT_OK) return rc;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LACT_EINVAL;
  if (workspace_bytes_ < lact_ttt_host_workspace_bytes(p)) return LACT_ENOSPC;
  const void* hin[8] = {q, k, v, lr, beta, w1, w2, w3};
  size_t sz[8];
  input_bytes(D, sz);
  for (int i = 0; i < 8; ++i)
    if (sz[i] && !hin[i]) return LACT_EINVAL;
  if (!out || !w1_out || !w2_out || !w3_out) return LACT_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Bump bp{reinterpret_cast<uintptr_t>(workspace), static_cast<uintptr_t>(workspace_bytes(D))};
  void* dev[8];
  for (int i = 0; i < 8; ++i) dev[i] = sz[i] ? bp.take<uint8_t>(static_cast<int64_t>(sz[i])) : nullptr;
  const size_t e = D.dtype == LACT_BF16 ? 2 : 4;
  const size_t osz = static_cast<size_t>(D.BH * D.Tq * D.d) * e;
  const size_t wsz = static_cast<size_t>(D.BH * D.d * D.dh) * 4;
  void* dout = bp.take<uint8_t>(static_cast<int64_t>(osz));
  float* dw[3];
  for (int i = 0; i < 3; ++i) dw[i] = bp.take<float>(D.BH * D.d * D.dh);
  for (int i = 0; i < 8; ++i)
    if (sz[i] && cudaMemcpyAsync(dev[i], hin[i], sz[i], cudaMemcpyHostToDevice, st) != cudaSuccess)
      return LACT_ECUDA;
  rc = lact_ttt_fwd(p, dev[0], dev[1], dev[2], static_cast<const float*>(dev[3]),
                    static_cast<const float*>(dev[4]), static_cast<const float*>(dev[5]),
                    static_cast<const float*>(dev[6]), static_cast<const float*>(dev[7]), dout, dw[0],
                    dw[1], dw[2], workspace, workspace_bytes(D), stream);
  if (rc != LACT_OK) return rc;
  if (cudaMemcpyAsync(out, dout, osz, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(w1_out, dw[0], wsz, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(w2_out, dw[1], wsz, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(w3_out, dw[2], wsz, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return LACT_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LACT_ECUDA;
  return LACT_OK;
}

size_t lact_ttt_bwd_workspace_bytes(const lact_problem* p) {
  Dims D;
  if (validate(p, D) != LACT_OK) return 0;
  return bwd_workspace_bytes(D);
}

int lact_ttt_bwd(const lact_problem* p, const lact_fwd_opts* opts, const void* q, const void* k,
                 const void* v, const float* lr, const float* beta, const float* w1, const float* w2,
                 const float* w3, const void* dout, const float* dw1_out, const float* dw2_out,
                 const float* dw3_out, float* dq, float* dk, float* dv, float* dlr, float* dbeta,
                 float* dw1, float* dw2, float* dw3, float* dout_scale, void* workspace,
                 size_t workspace_bytes_, void* stream) {
  return lact_ttt_bwd_ex(p, opts, nullptr, q, k, v, lr, beta, w1, w2, w3, dout, dw1_out, dw2_out, dw3_out, dq,
                         dk, dv, dlr, dbeta, dw1, dw2, dw3, dout_scale, workspace, workspace_bytes_, stream);
}

int lact_ttt_bwd_ex(const lact_problem* p, const lact_fwd_opts* opts, const lact_bwd_momentum* mg,
                    const void* q, const void* k, const void* v, const float* lr, const float* beta,
                    const float* w1, const float* w2, const float* w3, const void* dout, const float* dw1_out,
                    const float* dw2_out, const float* dw3_out, float* dq, float* dk, float* dv, float* dlr,
                    float* dbeta, float* dw1, float* dw2, float* dw3, float* dout_scale, void* workspace,
                    size_t workspace_bytes_, void* stream) {
  Dims D;
  int rc = validate(p, D);
  if (rc != LACT_OK) return rc;
  const float* scale = opts ? opts->out_scale : nullptr;
  const bool mom = D.rule == LACT_RULE_MOMENTUM;
  const float* m0[3] = {opts ? opts->m1 : nullptr, opts ? opts->m2 : nullptr, opts ? opts->m3 : nullptr};
  const float* dmf[3] = {mg ? mg->dm1_out : nullptr, mg ? mg->dm2_out : nullptr, mg ? mg->dm3_out : nullptr};
  float* dm0[3] = {mg ? mg->dm1 : nullptr, mg ? mg->dm2 : nullptr, mg ? mg->dm3 : nullptr};
  const bool any_m0 = m0[0] || m0[1] || m0[2], any_dmf = dmf[0] || dmf[1] || dmf[2];
  if ((any_m0 || mg) && !mom) return LACT_EINVAL;
  if (any_m0 && !(m0[0] && m0[1] && m0[2])) return LACT_EINVAL;
  if (any_dmf && !(dmf[0] && dmf[1] && dmf[2])) return LACT_EINVAL;
  if (mg && !(dm0[0] && dm0[1] && dm0[2])) return LACT_EINVAL;
  const size_t e = D.dtype == LACT_BF16 ? 2 : 4;
  const size_t nq = static_cast<size_t>(D.BH * D.Tq * D.d), nk = static_cast<size_t>(D.BH * D.T * D.d);
  const size_t hw = static_cast<size_t>(D.w_shared ? D.H : D.BH) * D.d * D.dh * 4;
  const size_t wo = static_cast<size_t>(D.BH * D.d * D.dh) * 4;
  struct Buf { const void* p; size_t n; bool need; };
  const Buf ins[] = {{q, nq * e, true}, {k, nk * e, true}, {v, nk * e, true},
                     {lr, static_cast<size_t>(D.BH * D.T) * 12, true}, {beta, static_cast<size_t>(D.BH * D.T) * 4, mom},
                     {w1, hw, true}, {w2, hw, true}, {w3, hw, true}, {dout, nq * e, true},
                     {dw1_out, wo, false}, {dw2_out, wo, false}, {dw3_out, wo, false},
                     {scale, static_cast<size_t>(D.BH * D.Tq) * 4, false},
                     {m0[0], wo, false}, {m0[1], wo, false}, {m0[2], wo, false},
                     {dmf[0], wo, false}, {dmf[1], wo, false}, {dmf[2], wo, false}};
  const bool with_dm = mg != nullptr;
  const Buf outs[] = {{dq, nq * 4, true}, {dk, nk * 4, true}, {dv, nk * 4, true},
                      {dlr, static_cast<size_t>(D.BH * D.T) * 12, true},
                      {dbeta, static_cast<size_t>(D.BH * D.T) * 4, mom}, {dw1, hw, true}, {dw2, hw, true},
                      {dw3, hw, true}, {dout_scale, static_cast<size_t>(D.BH * D.Tq) * 4, scale != nullptr},
                      {dm0[0], wo, with_dm}, {dm0[1], wo, with_dm}, {dm0[2], wo, with_dm}};
  for (const Buf& b : ins)
    if ((b.need && !b.p) || (b.p && !aligned16(b.p) && b.p != scale)) return LACT_EINVAL;
  for (const Buf& b : outs)
    if (b.need && (!b.p || (b.p != dout_scale && !aligned16(b.p)))) return LACT_EINVAL;
  if (scale && (reinterpret_cast<uintptr_t>(scale) & 3u)) return LACT_EINVAL;
  if (dout_scale && (reinterpret_cast<uintptr_t>(dout_scale) & 3u)) return LACT_EINVAL;
  if ((dw1_out || dw2_out || dw3_out) && !(dw1_out && dw2_out && dw3_out)) return LACT_EINVAL;
  for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
    if (!outs[i].need) continue;
    for (const Buf& b : ins)
      if (b.p && overlaps(outs[i].p, outs[i].n, b.p, b.n)) return LACT_EINVAL;
    for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
      if (outs[j].need && overlaps(outs[i].p, outs[i].n, outs[j].p, outs[j].n)) return LACT_EINVAL;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LACT_EINVAL;
  if (workspace_bytes_ < bwd_workspace_bytes(D)) return LACT_ENOSPC;
  Bump bp{reinterpret_cast<uintptr_t>(workspace), 0};
  BwdBufs b;
  plan_bwd(D, bp, b);
  BwdInputs in{q, k, v, lr, beta, w1, w2, w3, dout, dw1_out, dw2_out, dw3_out,
               opts ? opts->update_mask : nullptr, scale, dq, dk, dv, dlr, dbeta, dw1, dw2, dw3, dout_scale,
               {m0[0], m0[1], m0[2]}, {dmf[0], dmf[1], dmf[2]}, {dm0[0], dm0[1], dm0[2]},
               opts ? opts->allreduce : nullptr, opts ? opts->allreduce_user : nullptr};
  Launcher L{false, static_cast<cudaStream_t>(stream)};
  run_bwd(D, b, in, static_cast<cudaStream_t>(stream), L);
  return L.err;
}

size_t lact_swa_workspace_bytes(const lact_swa_problem* p) {
  SwaDims S;
  if (swa_validate(p, S) != LACT_OK) return 0;
  return swa_workspace_bytes(S);
}

int lact_swa_fwd(const lact_swa_problem* p, const void* q, const void* k, const void* v, const float* q_scale,
                 const float* q_offset, const float* k_scale, const float* k_offset, void* out, void* workspace,
                 size_t workspace_bytes_, void* stream) {
  SwaDims S;
  int rc = swa_validate(p, S);
  if (rc != LACT_OK) return rc;
  const void* need[] = {q, k, v, q_scale, q_offset, k_scale, k_offset, out};
  for (const void* x : need)
    if (!x || !aligned16(x)) return LACT_EINVAL;
  const size_t n = static_cast<size_t>(S.BH * S.T * S.d) * 2;
  const void* ins[] = {q, k, v};
  for (const void* x : ins)
    if (overlaps(out, n, x, n)) return LACT_EINVAL;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return LACT_EINVAL;
  if (workspace_bytes_ < swa_workspace_bytes(S)) return LACT_ENOSPC;
  if (!encode_fn()) return LACT_ECUDA;
  Bump bp{reinterpret_cast<uintptr_t>(workspace), 0};
  SwaBufs b;
  swa_plan(S, bp, b);
  Launcher L{false, static_cast<cudaStream_t>(stream)};
  swa_run(S, b, q, k, v, q_scale, q_offset, k_scale, k_offset, out, static_cast<cudaStream_t>(stream), L);
  return L.err;
}

int lact_ttt_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return LACT_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return LACT_ECUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return LACT_ECUDA;
    return LACT_ETIMEOUT;
  }
  return LACT_OK;
}

int lact_device_check(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LACT_ECUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return LACT_ECUDA;
  return (prop.major == 10 && prop.minor == 0) ? LACT_OK : LACT_ENODEV;
}

int lact_selftest_wait_timeout(int64_t budget_cycles, void* stream) {
  if (budget_cycles < 1 || budget_cycles > (int64_t(1) << 31)) return LACT_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  k_selftest_wait<<<1, 32, 0, st>>>(static_cast<long long>(budget_cycles));
  const cudaError_t e = cudaGetLastError();
  if (cudaStreamSynchronize(st) != cudaSuccess) return LACT_ECUDA;
  return e == cudaSuccess ? LACT_OK : LACT_ECUDA;
}

int lact_kernel_kinds(void) { return K_COUNT; }

const char* lact_kernel_name(int kind) {
  return (kind >= 0 && kind < K_COUNT) ? kKindNames[kind] : "unknown";
}

int lact_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return LACT_OK;
}

int lact_profile_read(int64_t* launches, double* ms, int nkinds) {
  if (!launches || !ms || nkinds < K_COUNT) return LACT_EINVAL;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (int i = 0; i < nkinds; ++i) {
    launches[i] = 0;
    ms[i] = 0.0;
  }
  int rc = LACT_OK;
  for (const ProfRec& r : g_prof) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      rc = LACT_ECUDA;
    launches[r.kind] += 1;
    ms[r.kind] += t;
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof.clear();
  return rc;
}

const char* lact_status_string(int code) {
  switch (code) {
    case LACT_OK: return "ok";
    case LACT_EINVAL: return "invalid argument";
    case LACT_ENOSPC: return "workspace too small";
    case LACT_ECUDA: return "CUDA error";
    case LACT_ETIMEOUT: return "a bounded device wait gave up";
    case LACT_ENODEV: return "not an sm_100 device";
    case LACT_ETOOBIG:
      return "problem needs more scratch than lact_ttt_fwd_noalloc's built-in buffer "
             "(LACT_NOALLOC_SCRATCH_BYTES) holds; use lact_ttt_fwd with a caller workspace";
    case LACT_ECOMM: return "the context-parallel all-reduce hook returned an error";
    default: return "unknown status";
  }
}

}  // extern "C"
