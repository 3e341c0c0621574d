// umma_kernels.cuh -- tcgen05 (sm_100a) tensor-core kernels of the bf16 path.
//
// Every kernel here is a persistent, warp-specialized tile loop (one CTA per
// SM, 192 threads) over output tiles of 128 rows:
//   warp 0      TMA producer (one elected lane): a STAGES-deep smem ring that
//               runs on across tiles
//   warp 1      TMEM allocator + MMA issuer (one elected lane), accumulating
//               tile i into TMEM buffer (i & 1)
//   warp 6      (Ops with kIssuers = 2) a second MMA issuer for an
//               independent part of the tile's MMAs: an MMA issue holds its
//               thread until the tensor core takes it, so the barrier waits
//               and commits of one issuer idle the tensor core unless another
//               issuer has MMAs to give it
//   warps 2..5  epilogue: tcgen05.ld of one 32-lane TMEM quarter each, fused
//               elementwise math, stores to global memory; the buffer is
//               handed back to the MMA warp when read, so tile i's epilogue
//               overlaps tile i+1's loads and MMAs
// Operands are bf16 in 128-byte-swizzled smem tiles fed by TMA, accumulators
// fp32 in TMEM.  K is consumed in blocks of 64 (one 128-byte swizzle row).
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace lact {

constexpr int kBM = 128;  // rows of every output tile (one TMEM lane per row)
constexpr int kBK = 64;   // K elements per stage (128 bytes of bf16)
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int kIssuer2Warp = 6;

// Block size of a kernel whose Op has kIssuers MMA issuers.
// Epilogue warp groups of an Op: 1 unless the Op sets kEpiGroups.  Each
// group has 4 warps (one TMEM lane quarter each) and takes its share of the
// tile's columns; the extra groups' warps follow the issuers.
template <class Op, class = void>
struct EpiGroups {
  static constexpr int value = 1;
};
template <class Op>
struct EpiGroups<Op, std::void_t<decltype(Op::kEpiGroups)>> {
  static constexpr int value = Op::kEpiGroups;
};

template <class Op>
constexpr int umma_threads() {
  return (Op::kIssuers == 2 ? kThreads + 32 : kThreads) + (EpiGroups<Op>::value - 1) * 32 * kEpiWarps;
}

template <int N>
struct TmemCols {
  static constexpr int value = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : N <= 256 ? 256 : 512;
};

// The shared pipeline: Op supplies kStages, kStageBytes, kExtraBytes (shared
// memory for the epilogue, after the ring), kAccCols (TMEM column stride of
// one accumulator buffer), kAccBufs (1 or 2 buffers), kIssuers (1 or 2),
// Tile, num_tiles(), map_tile(), num_kb(), stage_bytes(), prefetch(),
// load(), mma(p, t, stage, tmem, kb, issuer), epilogue(), epilogue_done().
template <class Op>
__global__ void __launch_bounds__(umma_threads<Op>(), 1)
    umma_kernel(const __grid_constant__ typename Op::Params p) {
  griddep_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int S = Op::kStages;
  constexpr int NB = Op::kAccBufs;
  constexpr int EG = EpiGroups<Op>::value;
  constexpr int kExtraEpi0 = Op::kIssuers == 2 ? kIssuer2Warp + 1 : 2 + kEpiWarps;   // first warp of group 1
  constexpr uint32_t kCols = TmemCols<NB * Op::kAccCols>::value;
  static_assert(NB * Op::kAccCols <= 512, "accumulator buffers must fit in TMEM");
  uint8_t* extra = smem + S * Op::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(extra + Op::kExtraBytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;   // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  // Once a bounded wait anywhere has given up, later CTAs do no work (the
  // results are already invalid and flagged); decided once per CTA.
  __shared__ int abort_cta;
  if (threadIdx.x == 0) abort_cta = *reinterpret_cast<volatile int*>(&g_status);
  __syncthreads();
  if (abort_cta) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = Op::num_tiles(p);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Op::kIssuers);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], Op::kIssuers);
      mbar_init(&acc_empty[b], kEpiWarps * EG);
    }
    fence_barrier_init();
    Op::prefetch(p);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync_converged();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // after the local setup, before any global access

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
        const typename Op::Tile t = Op::map_tile(p, tile);
        const int nkb = Op::num_kb(p, t);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          if (it >= S && !mbar_wait(&empty[s], ((it / S) - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], Op::stage_bytes(p, t));
          Op::load(p, t, kb, smem + s * Op::kStageBytes, &full[s]);
        }
      }
    }
  } else if (warp == 1 || (Op::kIssuers == 2 && warp == kIssuer2Warp)) {
    if (lane == 0) {
      const int issuer = warp == 1 ? 0 : 1;
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++local) {
        const typename Op::Tile t = Op::map_tile(p, tile);
        const int nkb = Op::num_kb(p, t);
        const int buf = local % NB, use = local / NB;
        if (use > 0 && !mbar_wait(&acc_empty[buf], (use - 1) & 1)) break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * Op::kAccCols;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(&full[s], (it / S) & 1)) { ok = false; break; }
          Op::mma(p, t, smem_u32(smem + s * Op::kStageBytes), acc, kb, issuer);
          umma_commit(&empty[s]);
        }
        umma_commit(&acc_full[buf]);
      }
    }
  } else if (warp < 2 + kEpiWarps || (EG > 1 && warp >= kExtraEpi0)) {
    const int group = warp < 2 + kEpiWarps ? 0 : 1 + (warp - kExtraEpi0) / kEpiWarps;
    int local = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++local) {
      const typename Op::Tile t = Op::map_tile(p, tile);
      const int buf = local % NB, use = local / NB;
      if (!mbar_wait(&acc_full[buf], use & 1)) break;
      tc_fence_after();
      if constexpr (EG > 1)
        Op::epilogue(p, t, tmem + buf * Op::kAccCols, warp & 3, lane, extra, group);
      else
        Op::epilogue(p, t, tmem + buf * Op::kAccCols, warp & 3, lane, extra);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
    Op::epilogue_done(lane);
  }
  tc_fence_before();
  cta_sync_converged();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// Issue the 4 UMMAs (K = 16 each) of one 64-wide K block.
// a_mn / b_mn: operand is MN-major (64-element MN blocks `*_lbo` bytes apart,
// 16 K rows = 2048 bytes per step) or K-major (32 bytes per step).
template <bool A_MN, bool B_MN>
__device__ __forceinline__ void mma_kblock(uint32_t d_tmem, uint32_t a_base, uint32_t a_lbo,
                                           uint32_t b_base, uint32_t b_lbo, uint32_t idesc,
                                           bool first) {
#pragma unroll
  for (int k = 0; k < kBK / 16; ++k) {
    const uint32_t ao = A_MN ? k * 2048u : k * 32u;
    const uint32_t bo = B_MN ? k * 2048u : k * 32u;
    const uint64_t ad = smem_desc_sw128(a_base + ao, A_MN ? a_lbo : 16u, 1024u);
    const uint64_t bd = smem_desc_sw128(b_base + bo, B_MN ? b_lbo : 16u, 1024u);
    umma_bf16(d_tmem, ad, bd, idesc, (first && k == 0) ? 0u : 1u);
  }
}

// Split-bf16 ("3-product") mode.  An fp32 value x is carried as
// x_hi = bf16(x) and x_lo = bf16(x - x_hi); a product is accumulated as
// x_hi*y_hi + x_hi*y_lo + x_lo*y_hi (fp32 accumulate), which keeps about 16
// mantissa bits.  Used for the update path of the Muon rule, whose O(1)
// orthogonalised updates carry operand rounding from chunk to chunk.  An
// operand that is an exact bf16 input (v) has no lo part and takes 2 products.
__device__ __forceinline__ uint32_t pack_lo_bf16x2(float a, float b, uint32_t hi) {
  const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&hi);
  return pack_bf16x2(a - __low2float(h), b - __high2float(h));
}

// ---------------------------------------------------------------------------
// Fast-net forward on one chunk, one (128-token x 64-hidden-unit) tile.
//   Z1 = X W1^T, Z3 = X W3^T   (X = q^ or k^ rows, K = d)      -> TMEM [0,128)
//   KMODE also: DH = V W2[:, slice] (W2 [d, dh], an MN-major tile) -> TMEM [128,192)
// Epilogue, per token t and hidden unit r (s1 = sigmoid(z1)):
//   query tile: Hq = silu(z1) z3                                  (bf16)
//   key tile:   E1 = lr1 dh z3 s1 (1 + z1 (1 - s1))               (d<f,v>/dz1)
//               Eh = lr2 silu(z1) z3                              (h, for G2)
//               E3 = lr3 dh silu(z1)                              (d<f,v>/dz3)
// so that the negated chunk gradients are  -G1 = E1^T k^,  -G3 = E3^T k^,
// -G2^T = Eh^T v  ("大块测试时训练（LaCT）技术解析" §2.1 eqs. 4-5; loss and
// per-token rates of "LaCT：以大分块更新…" 「局部注意力与非线性记忆相互补充」).
// Rows past the chunk's end are written as zeros (key tiles) or skipped.
// SPLIT (key tiles only): k^ and the weight shadows come as hi/lo pairs, the
// E factors are written as hi/lo pairs.
// ---------------------------------------------------------------------------
struct FwdParams {
  CUtensorMap tmX;   // q^ or k^ [BH, rows, d] bf16, box {64, 128, 1}
  CUtensorMap tmXlo; // k^ lo part (split)
  CUtensorMap tmV;   // v [BH, T, d] bf16, box {64, 128, 1}          (key tiles)
  CUtensorMap tmW;   // bf16 shadows as [3*BH, dh, d] (W1, -, W3 planes), box {64, 64, 1}
  CUtensorMap tmWlo; // shadow lo parts (split)
  CUtensorMap tmW2;  // W2 shadow plane [BH, d, dh], box {64 (dh), 64 (d), 1}
  CUtensorMap tmW2lo;
  CUtensorMap tmE;   // E as [3*BH, buf_rows, dh], box {64, 32, 1}: the epilogue's TMA stores
  int bh_count;      // B*H
  int n_slices;      // dh / 64 hidden slices
  int n_row_tiles;   // 128-token tiles of the chunk
  int x_row0;        // first token of the chunk in tmX / tmV
  int rows_valid;    // tokens in this chunk
  int kb_count;      // d / 64
  int dh;
  int T;             // rows of lr per head
  __nv_bfloat16* hq; // query tiles: Hq [BH, buf_rows, dh]
  __nv_bfloat16* e;  // key tiles:   E [3][BH][buf_rows][dh]  (E1, Eh, E3)
  __nv_bfloat16* e_lo;  // split: lo parts, same layout
  int64_t buf_rows;
  const float* lr;   // [BH, T, 3]; null: unit rates on the chunk's rows (the apply's backward:
                     // E1 = dz1, Eh = hq, E3 = dz3 for the output gradient in place of v)
};

// Key-tile gradient factors of 64 hidden units for one epilogue warp's 32
// rows (row0 + 32 quarter + lane of the chunk), per token t and unit r with
// s1 = sigmoid(z1):  E1 = lr1 u z3 s1 (1 + z1 (1 - s1)),  Eh = lr2 silu(z1) z3,
// E3 = lr3 u silu(z1)  (unit rates when p.lr is null), in bf16 through the
// warp's three swizzled 32 x 64 staging tiles in `extra` and bulk tensor
// stores at columns col0 .. col0 + 63.  tz1, tz3, tu: the warp's TMEM
// addresses of the 64 columns of z1, z3 and u.
__device__ __forceinline__ void key_factors_tma(const FwdParams& p, int bh, int row0, int col0, uint32_t tz1,
                                                uint32_t tz3, uint32_t tu, int quarter, int lane, uint8_t* extra) {
  const int grow = row0 + quarter * 32 + lane;
  const bool valid = grow < p.rows_valid;
  float eta0 = 0.f, eta1 = 0.f, eta2 = 0.f;
  if (valid) {
    if (p.lr) {
      const float* l = p.lr + (static_cast<int64_t>(bh) * p.T + p.x_row0 + grow) * 3;
      eta0 = l[0];
      eta1 = l[1];
      eta2 = l[2];
    } else {
      eta0 = eta1 = eta2 = 1.0f;
    }
  }
  const uint32_t stg = smem_u32(extra) + quarter * 3 * 4096 + lane * 128;
  if (lane == 0) bulk_wait_read_all();  // the previous tile's stores have read the staging
  __syncwarp();
#pragma unroll 1
  for (int j = 0; j < 64; j += 16) {
    float z1[16], z3[16], u[16];
    __syncwarp();
    tmem_ld16(tz1 + j, z1);
    tmem_ld16(tz3 + j, z3);
    tmem_ld16(tu + j, u);
    tmem_ld_wait();
    uint32_t w[3][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float e1[2], eh[2], e3[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float a = z1[2 * i + c], b = z3[2 * i + c], g = u[2 * i + c];
        const float s = sigmoid_fast(a);
        const float sa = a * s;
        const float ds = fmaf(sa, 1.0f - s, s);
        e1[c] = (eta0 * g) * (b * ds);
        eh[c] = eta1 * (sa * b);
        e3[c] = (eta2 * g) * sa;
      }
      w[0][i] = pack_bf16x2(e1[0], e1[1]);
      w[1][i] = pack_bf16x2(eh[0], eh[1]);
      w[2][i] = pack_bf16x2(e3[0], e3[1]);
    }
    // row `lane` of each staging tile; 16-byte chunk c at c ^ (lane % 8)
    const uint32_t c0 = ((j / 8) ^ (lane & 7)) << 4, c1 = ((j / 8 + 1) ^ (lane & 7)) << 4;
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      st_shared_v4(stg + m * 4096 + c0, w[m][0], w[m][1], w[m][2], w[m][3]);
      st_shared_v4(stg + m * 4096 + c1, w[m][4], w[m][5], w[m][6], w[m][7]);
    }
  }
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    const uint8_t* src = extra + quarter * 3 * 4096;
    const int row = row0 + quarter * 32;
#pragma unroll
    for (int m = 0; m < 3; ++m)
      tma_store_3d(&p.tmE, src + m * 4096, col0, row, m * p.bh_count + bh);
    bulk_commit_group();
  }
}


template <bool KMODE, bool SPLIT = false, int NSL = 64>
struct FwdOp {
  static_assert(KMODE || !SPLIT, "split mode is for key tiles");
  static_assert(NSL == 64 || NSL == 128, "hidden slice width");
  using Params = FwdParams;
  static constexpr int kXBytes = kBM * kBK * 2;           // 16 KB
  static constexpr int kWBytes = NSL * kBK * 2;           // one NSL-row weight slice of a K block
  // stage layout: X [X_lo] [V] W1 W3 [W1_lo W3_lo] [W2 [W2_lo]]
  static constexpr int kOffXlo = kXBytes;
  static constexpr int kOffV = kXBytes * (SPLIT ? 2 : 1);
  static constexpr int kOffW = kOffV + (KMODE ? kXBytes : 0);
  static constexpr int kOffWlo = kOffW + 2 * kWBytes;
  static constexpr int kOffW2 = kOffW + (SPLIT ? 4 : 2) * kWBytes;
  static constexpr int kStageBytes = kOffW2 + (KMODE ? (SPLIT ? 2 : 1) * kWBytes : 0);
  static constexpr int kStages = (196608 / kStageBytes) < 6 ? (196608 / kStageBytes) : 6;
  // Plain key tiles stage E in shared memory (per epilogue warp: 3 swizzled
  // 32-row x 64-column tiles) and write it with TMA bulk stores.
  static constexpr bool kTmaStore = KMODE && !SPLIT && NSL == 64;
  static constexpr int kExtraBytes = kTmaStore ? 4 * 3 * 4096 : 0;
  // TMEM per tile: Z1 | Z3 (2 * NSL) [| DH (NSL)]
  static constexpr int kAccCols = KMODE ? (NSL == 64 ? 256 : 384) : 2 * NSL;
  static constexpr int kAccBufs = (2 * kAccCols <= 512) ? 2 : 1;
  // Key tiles: issuer 0 the Z MMAs, issuer 1 the DH MMAs (independent
  // accumulators and A operands).
  static constexpr int kIssuers = KMODE ? 2 : 1;
  struct Tile { int slice, row0, bh; };

  // Tile order: hidden slice fastest, so CTAs running together share the
  // same token tile of q^ / k^ / v in L2.
  __device__ static int num_tiles(const Params& p) { return p.n_slices * p.n_row_tiles * p.bh_count; }
  __device__ static Tile map_tile(const Params& p, int idx) {
    const int sl = idx % p.n_slices;
    const int rt = (idx / p.n_slices) % p.n_row_tiles;
    const int bh = idx / (p.n_slices * p.n_row_tiles);
    return Tile{sl, rt * kBM, bh};
  }
  __device__ static int num_kb(const Params& p, const Tile&) { return p.kb_count; }
  __device__ static uint32_t stage_bytes(const Params&, const Tile&) { return kStageBytes; }
  __device__ static void prefetch(const Params& p) {
    tma_prefetch_map(&p.tmX);
    tma_prefetch_map(&p.tmW);
    if (KMODE) tma_prefetch_map(&p.tmV);
    if (KMODE) tma_prefetch_map(&p.tmW2);
    if (SPLIT) {
      tma_prefetch_map(&p.tmXlo);
      tma_prefetch_map(&p.tmWlo);
      tma_prefetch_map(&p.tmW2lo);
    }
  }
  __device__ static void load(const Params& p, const Tile& t, int kb, uint8_t* st, uint64_t* bar) {
    const int k = kb * kBK, row = p.x_row0 + t.row0, hs = t.slice * NSL;
    const int z1 = t.bh, z3 = 2 * p.bh_count + t.bh;
    tma_load_3d(st, &p.tmX, bar, k, row, t.bh);
    tma_load_3d(st + kOffW, &p.tmW, bar, k, hs, z1);                 // W1 rows of the slice
    tma_load_3d(st + kOffW + kWBytes, &p.tmW, bar, k, hs, z3);       // W3 rows of the slice
    if (SPLIT) {
      tma_load_3d(st + kOffXlo, &p.tmXlo, bar, k, row, t.bh);
      tma_load_3d(st + kOffWlo, &p.tmWlo, bar, k, hs, z1);
      tma_load_3d(st + kOffWlo + kWBytes, &p.tmWlo, bar, k, hs, z3);
    }
    if (KMODE) {
      tma_load_3d(st + kOffV, &p.tmV, bar, k, row, t.bh);
#pragma unroll
      for (int b = 0; b < NSL / 64; ++b) {                           // W2[k.., hs..]: MN blocks of 64
        tma_load_3d(st + kOffW2 + b * 8192, &p.tmW2, bar, hs + 64 * b, k, t.bh);
        if (SPLIT) tma_load_3d(st + kOffW2 + kWBytes + b * 8192, &p.tmW2lo, bar, hs + 64 * b, k, t.bh);
      }
    }
  }
  __device__ static void mma(const Params&, const Tile&, uint32_t st, uint32_t tmem, int kb, int issuer) {
    const bool f = kb == 0;
    if (issuer == 0) {
      constexpr uint32_t id0 = idesc_bf16(kBM, 2 * NSL, false, false);
      mma_kblock<false, false>(tmem, st, 0, st + kOffW, 0, id0, f);
      if (SPLIT) {
        mma_kblock<false, false>(tmem, st, 0, st + kOffWlo, 0, id0, false);
        mma_kblock<false, false>(tmem, st + kOffXlo, 0, st + kOffW, 0, id0, false);
      }
    }
    if (KMODE && issuer == 1) {
      constexpr uint32_t id1 = idesc_bf16(kBM, NSL, false, true);
      mma_kblock<false, true>(tmem + 2 * NSL, st + kOffV, 0, st + kOffW2, 8192u, id1, f);
      if (SPLIT) mma_kblock<false, true>(tmem + 2 * NSL, st + kOffV, 0, st + kOffW2 + kWBytes, 8192u, id1, false);
    }
  }
  __device__ static void epilogue_done(int lane) {
    if (kTmaStore && lane == 0) bulk_wait_all();
  }
  __device__ static void epilogue(const Params& p, const Tile& t, uint32_t tmem, int quarter,
                                  int lane, uint8_t* extra) {
    const int r = quarter * 32 + lane;
    const int grow = t.row0 + r;
    const bool valid = grow < p.rows_valid;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int64_t col0 = static_cast<int64_t>(t.slice) * NSL;
    if constexpr (kTmaStore) {
      key_factors_tma(p, t.bh, t.row0, static_cast<int>(col0), tq, tq + 64, tq + 128, quarter, lane, extra);
      return;
    }
    if (!KMODE) {
      __nv_bfloat16* dst = p.hq + (static_cast<int64_t>(t.bh) * p.buf_rows + grow) * p.dh + col0;
#pragma unroll 1
      for (int j = 0; j < NSL; j += 16) {
        float z1[16], z3[16];
        __syncwarp();
        tmem_ld16(tq + j, z1);
        tmem_ld16(tq + NSL + j, z3);
        tmem_ld_wait();
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float h0 = z1[2 * i] * sigmoid_fast(z1[2 * i]) * z3[2 * i];
          const float h1 = z1[2 * i + 1] * sigmoid_fast(z1[2 * i + 1]) * z3[2 * i + 1];
          w[i] = pack_bf16x2(h0, h1);
        }
        if (valid) {
          st_global_v4(dst + j, w[0], w[1], w[2], w[3]);
          st_global_v4(dst + j + 8, w[4], w[5], w[6], w[7]);
        }
      }
    } else {
      float eta0 = 0.f, eta1 = 0.f, eta2 = 0.f;
      if (valid) {
        if (p.lr) {
          const float* l = p.lr + (static_cast<int64_t>(t.bh) * p.T + p.x_row0 + grow) * 3;
          eta0 = l[0];
          eta1 = l[1];
          eta2 = l[2];
        } else {
          eta0 = eta1 = eta2 = 1.0f;
        }
      }
      const int64_t plane = static_cast<int64_t>(p.bh_count) * p.buf_rows * p.dh;
      const int64_t off = (static_cast<int64_t>(t.bh) * p.buf_rows + grow) * p.dh + col0;
#pragma unroll 1
      for (int j = 0; j < NSL; j += 16) {
        float z1[16], z3[16], u[16];
        __syncwarp();
        tmem_ld16(tq + j, z1);
        tmem_ld16(tq + NSL + j, z3);
        tmem_ld16(tq + 2 * NSL + j, u);
        tmem_ld_wait();
        float e[3][16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a = z1[i], b = z3[i], g = u[i];
          const float s = SPLIT ? sigmoidf_(a) : sigmoid_fast(a);
          const float sa = a * s;
          e[0][i] = eta0 * g * b * (s * (1.0f + a * (1.0f - s)));
          e[1][i] = eta1 * sa * b;
          e[2][i] = eta2 * g * sa;
        }
#pragma unroll
        for (int m = 0; m < 3; ++m) {
          uint32_t hw[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) hw[i] = pack_bf16x2(e[m][2 * i], e[m][2 * i + 1]);
          __nv_bfloat16* d = p.e + m * plane + off + j;
          st_global_v4(d, hw[0], hw[1], hw[2], hw[3]);
          st_global_v4(d + 8, hw[4], hw[5], hw[6], hw[7]);
          if (SPLIT) {
            uint32_t lw[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) lw[i] = pack_lo_bf16x2(e[m][2 * i], e[m][2 * i + 1], hw[i]);
            __nv_bfloat16* dl = p.e_lo + m * plane + off + j;
            st_global_v4(dl, lw[0], lw[1], lw[2], lw[3]);
            st_global_v4(dl + 8, lw[4], lw[5], lw[6], lw[7]);
          }
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Generic batched GEMM with a fused affine epilogue:
//   C[m][n] = alpha * sum_k A(m,k) B(n,k) + beta * Cin[m][n]
// stored as fp32 (outf) and/or bf16 (outb [+ outb_lo in split mode]) at
//   base + item * item_stride + m * ld + n,  rows m < m_valid.
// A is K-major (rows of A in memory) or MN-major (A^T rows in memory), same
// for B.  Batch index z = split * items + item; split s covers K blocks
// [s*kb_count, (s+1)*kb_count) and writes output item (s*items + item).
// B's batch coordinate is (item % zb_mod) + zb_add, read from tmB2 instead of
// tmB when item / zb_mod == alt_group (tmB2 is an exact bf16 input in split
// mode: no lo part).  Items with item / tr_mod == tr_group store their fp32
// output transposed, at n * ld_t + m (coalesced: lanes hold consecutive m).
// Used for: the apply output (Hq W2), the chunk gradients (E^T X), and the
// three Newton-Schulz products.
// ---------------------------------------------------------------------------
struct GemmParams {
  CUtensorMap tmA, tmB, tmB2;
  CUtensorMap tmAlo, tmBlo;  // split mode
  int nt_n, nt_m;            // tiles along N and M; the z extent is splits * items
  int n_tiles;               // nt_n * nt_m * splits * items
  int items;
  int kb_count;           // K blocks per split
  int kb_total;           // K blocks in all (the last split may hold fewer)
  int a_k0, b_k0;
  int zb_mod, zb_add, alt_group;
  int m_valid;
  float alpha, beta;
  const float* cin;
  float* outf;
  __nv_bfloat16* outb;
  __nv_bfloat16* outb_lo;  // split mode
  int64_t item_stride, ld;
  int tr_group, tr_mod;
  int64_t ld_t;
  const float* row_scale;  // or null: row m of output item z scaled by row_scale[z * rs_item + m]
  int64_t rs_item;
  int a_m0;                // first M coordinate of A's map that tile row 0 reads (MN-major A:
                           // a multiple of 8, the map's inner coordinate)
  int zb_div, zb_mul;      // if zb_div > 0: B's batch = (item / zb_div) * zb_mul + item % zb_div
  int red;                 // fp32 output added into outf with atomics (no cin): the K splits of
                           // an item all add into output item `item`
  // Store-only fp32 output through bulk tensor stores (CTA-pair kernel; alpha
  // 1, no cin, row scale, bf16 output or atomics): tmOut views outf as
  // [items][rows][ld] fp32, tmOutT (items stored transposed) as
  // [items][ld_t rows][m], both with 32 x 32 boxes and 128-byte swizzle.
  int out_tma;
  CUtensorMap tmOut, tmOutT;
};

template <bool A_MN, bool B_MN, int BN, bool SPLIT = false>
struct GemmOp {
  using Params = GemmParams;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  // stage layout: A [A_lo] B [B_lo]
  static constexpr int kOffB = kABytes * (SPLIT ? 2 : 1);
  static constexpr int kStageBytes = kOffB + kBBytes * (SPLIT ? 2 : 1);
  static constexpr int kStages = (196608 / kStageBytes) < 6 ? (196608 / kStageBytes) : 6;
  static constexpr int kAccCols = TmemCols<BN>::value;
  static constexpr int kAccBufs = 2;
  // Per epilogue warp: a 32-row x 16-column fp32 staging tile with a row
  // pitch of 17 floats (a thread's row writes are conflict-free).  When the
  // tile reads an fp32 input cin, cin and the fp32 output pass through it as
  // 64-byte row segments, 8 rows per warp access, instead of one row (one
  // cache line) per thread: the row-per-thread loads stalled those epilogues
  // (Newton-Schulz update 69 -> 52.5 us).  Store-only epilogues keep the
  // direct row stores, which measured faster there (chunk gradient 30.1 us
  // direct, 33.8 us staged).
  static constexpr int kStgPitch = 17;
  static constexpr int kExtraBytes = kEpiWarps * 32 * kStgPitch * 4;
  static constexpr int kIssuers = 1;
  struct Tile { int m0, n0, item, out_item, split, zb; bool alt; };

  __device__ static int num_tiles(const Params& p) { return p.n_tiles; }
  __device__ static Tile map_tile(const Params& p, int idx) {
    Tile t;
    const int z = idx / (p.nt_n * p.nt_m);
    t.n0 = (idx % p.nt_n) * BN;
    t.m0 = ((idx / p.nt_n) % p.nt_m) * kBM;
    t.item = z % p.items;
    t.split = z / p.items;
    t.out_item = p.red ? t.item : z;
    t.zb = p.zb_div > 0 ? (t.item / p.zb_div) * p.zb_mul + t.item % p.zb_div : (t.item % p.zb_mod) + p.zb_add;
    t.alt = p.alt_group >= 0 && (t.item / p.zb_mod) == p.alt_group;
    return t;
  }
  __device__ static int num_kb(const Params& p, const Tile& t) {
    const int left = p.kb_total - t.split * p.kb_count;
    return left < p.kb_count ? left : p.kb_count;
  }
  __device__ static uint32_t stage_bytes(const Params&, const Tile& t) {
    return kABytes * (SPLIT ? 2 : 1) + kBBytes * ((SPLIT && !t.alt) ? 2 : 1);
  }
  __device__ static void prefetch(const Params& p) {
    tma_prefetch_map(&p.tmA);
    tma_prefetch_map(&p.tmB);
    if (p.alt_group >= 0) tma_prefetch_map(&p.tmB2);
    if (SPLIT) {
      tma_prefetch_map(&p.tmAlo);
      tma_prefetch_map(&p.tmBlo);
    }
  }
  __device__ static void load_a(const CUtensorMap* m, uint8_t* dst, uint64_t* bar, int m0, int ak, int z) {
    if (A_MN) {
      tma_load_3d(dst, m, bar, m0, ak, z);
      tma_load_3d(dst + 8192, m, bar, m0 + 64, ak, z);
    } else {
      tma_load_3d(dst, m, bar, ak, m0, z);
    }
  }
  __device__ static void load_b(const CUtensorMap* m, uint8_t* dst, uint64_t* bar, int n0, int bk, int z) {
    if (B_MN) {
#pragma unroll
      for (int b = 0; b < BN / 64; ++b) tma_load_3d(dst + b * 8192, m, bar, n0 + b * 64, bk, z);
    } else {
      tma_load_3d(dst, m, bar, bk, n0, z);
    }
  }
  __device__ static void load(const Params& p, const Tile& t, int kb, uint8_t* st, uint64_t* bar) {
    const int kk = (t.split * p.kb_count + kb) * kBK;
    const int ak = p.a_k0 + kk, bk = p.b_k0 + kk;
    const int am = t.m0 + p.a_m0;
    load_a(&p.tmA, st, bar, am, ak, t.item);
    load_b(t.alt ? &p.tmB2 : &p.tmB, st + kOffB, bar, t.n0, bk, t.zb);
    if (SPLIT) {
      load_a(&p.tmAlo, st + kABytes, bar, am, ak, t.item);
      if (!t.alt) load_b(&p.tmBlo, st + kOffB + kBBytes, bar, t.n0, bk, t.zb);
    }
  }
  __device__ static void mma(const Params&, const Tile& t, uint32_t st, uint32_t tmem, int kb, int) {
    constexpr uint32_t id = idesc_bf16(kBM, BN, A_MN, B_MN);
    mma_kblock<A_MN, B_MN>(tmem, st, 8192u, st + kOffB, 8192u, id, kb == 0);
    if (SPLIT) {
      if (!t.alt) mma_kblock<A_MN, B_MN>(tmem, st, 8192u, st + kOffB + kBBytes, 8192u, id, false);
      mma_kblock<A_MN, B_MN>(tmem, st + kABytes, 8192u, st + kOffB, 8192u, id, false);
    }
  }
  __device__ static void epilogue_done(int) {}
  __device__ static void epilogue(const Params& p, const Tile& t, uint32_t tmem, int quarter,
                                  int lane, uint8_t* extra) {
    const int r = quarter * 32 + lane;
    const int grow = t.m0 + r;
    const bool valid = grow < p.m_valid;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int64_t base = static_cast<int64_t>(t.out_item) * p.item_stride + t.n0;
    const int64_t off = base + static_cast<int64_t>(grow) * p.ld;
    const bool tr = p.tr_group >= 0 && (t.item / p.tr_mod) == p.tr_group;
    const float rs = (p.row_scale && valid) ? __ldg(p.row_scale + t.out_item * p.rs_item + grow) : 1.0f;
    float* stg = reinterpret_cast<float*>(extra) + quarter * 32 * kStgPitch;
    // In the coalesced passes this lane moves rows 8 k + lane / 4 (k < 4) of
    // the warp's 32, columns 4 (lane % 4) .. + 3 of the 16.
    const int wrow0 = t.m0 + quarter * 32, cr = lane >> 2, cc = (lane & 3) * 4;
    const bool has_c = p.cin != nullptr;
    // cin of the next 16 columns is loaded while this step's are used, so
    // the epilogue does not wait on one global load latency per step
    float4 cn[4];
    auto load_c = [&](int j) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rr = wrow0 + 8 * k + cr;
        cn[k] = rr < p.m_valid ? *reinterpret_cast<const float4*>(p.cin + base + static_cast<int64_t>(rr) * p.ld + j + cc)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    if (has_c) load_c(0);
#pragma unroll 1
    for (int j = 0; j < BN; j += 16) {
      float v[16], c[16];
      if (has_c) {
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float* sp = stg + (8 * k + cr) * kStgPitch + cc;
          sp[0] = cn[k].x;
          sp[1] = cn[k].y;
          sp[2] = cn[k].z;
          sp[3] = cn[k].w;
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 16; ++i) c[i] = stg[lane * kStgPitch + i];
        if (j + 16 < BN) load_c(j + 16);
      }
      __syncwarp();
      tmem_ld16(tq + j, v);
      tmem_ld_wait();
      if (has_c) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = p.alpha * v[i] + p.beta * c[i];
      } else if (p.alpha != 1.0f) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] *= p.alpha;
      }
      if (p.row_scale) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] *= rs;
      }
      if (p.outf && tr) {
        if (valid) {
          float* o = p.outf + static_cast<int64_t>(t.out_item) * p.item_stride +
                     static_cast<int64_t>(t.n0 + j) * p.ld_t + grow;
          if (p.red) {
#pragma unroll
            for (int i = 0; i < 16; ++i) atomicAdd(o + i * p.ld_t, v[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i * p.ld_t] = v[i];
          }
        }
      } else if (p.outf && !has_c) {
        if (valid) {
          float* o = p.outf + off + j;
          if (p.red) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              atomicAdd(reinterpret_cast<float4*>(o) + i, make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]));
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              st_global_v4(o + 4 * i, __float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]),
                           __float_as_uint(v[4 * i + 2]), __float_as_uint(v[4 * i + 3]));
          }
        }
      } else if (p.outf) {
        __syncwarp();   // every lane has read its cin row from the staging tile
#pragma unroll
        for (int i = 0; i < 16; ++i) stg[lane * kStgPitch + i] = v[i];
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int rr = wrow0 + 8 * k + cr;
          if (rr >= p.m_valid) continue;
          const float* sp = stg + (8 * k + cr) * kStgPitch + cc;
          float* o = p.outf + base + static_cast<int64_t>(rr) * p.ld + j + cc;
          if (p.red)
            atomicAdd(reinterpret_cast<float4*>(o), make_float4(sp[0], sp[1], sp[2], sp[3]));
          else
            st_global_v4(o, __float_as_uint(sp[0]), __float_as_uint(sp[1]), __float_as_uint(sp[2]),
                         __float_as_uint(sp[3]));
        }
      }
      if (valid) {
        if (p.outb) {
          uint32_t hw[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) hw[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
          __nv_bfloat16* o = p.outb + off + j;
          st_global_v4(o, hw[0], hw[1], hw[2], hw[3]);
          st_global_v4(o + 8, hw[4], hw[5], hw[6], hw[7]);
          if (SPLIT) {
            uint32_t lw[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) lw[i] = pack_lo_bf16x2(v[2 * i], v[2 * i + 1], hw[i]);
            __nv_bfloat16* ol = p.outb_lo + off + j;
            st_global_v4(ol, lw[0], lw[1], lw[2], lw[3]);
            st_global_v4(ol + 8, lw[4], lw[5], lw[6], lw[7]);
          }
        }
      }
    }
  }
};

template <class Op>
constexpr int umma_smem_bytes() {
  return Op::kStages * Op::kStageBytes + Op::kExtraBytes + (2 * Op::kStages + 4) * 8 + 16 + 1024;
}

}  // namespace lact
