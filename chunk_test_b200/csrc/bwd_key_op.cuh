// bwd_key_op.cuh -- the key side of the layer's backward for one chunk as a
// single persistent tensor-core kernel (the directional derivative of the
// chunk gradient, "大块测试时训练（LaCT）技术解析" §2.1 eqs. 4-5 with the
// per-token rates of "LaCT：以大分块更新…").  Per (128-token x 64-hidden-unit)
// tile, with Bk = [W1; W3; Gam1; Gam3] and Bv = [W2 | Gam2] the stacked
// state and gradient-direction operands of the chunk:
//   [z1 | z3 | p | r] = k^ Bk[slice rows]^T     (issuer 0, TMEM columns [0, 256))
//   [u | q]           = v  Bv[:, slice cols]    (issuer 1, TMEM columns [256, 384))
// and, in the epilogue (two groups of 4 warps, 32 hidden units each), the
// second-order factors of hvp_factors, one token row per thread, written as
// the bf16 operands of the contractions that follow:
//   Phik = [dz1 | dz3 | dp | dr]   [BH][rows][4 dh]
//   Phiv = [du | dq]               [BH][rows][2 dh]
// Each warp stages its 32 rows x 16 columns of every factor plane in shared
// memory and writes them with bulk tensor stores, so the rows (4 dh apart in
// Phik) go out as whole 32-byte sectors instead of one line per thread.  The
// per-token lr gradients (sums over the hidden units) are added into dlr
// with one fp32 atomic per row, column and warp group; dlr starts at zero.
// Rows past the chunk's end get zero factors (their rates are taken as zero)
// and no lr gradient; rows past the buffer are clipped by the stores.  Replaces two stacked contractions with fp32 outputs and
// an elementwise pass over them.
#pragma once

#include "bwd_kernels.cuh"
#include "umma_kernels.cuh"

namespace lact {

struct BwdKeyParams {
  CUtensorMap tmX;    // k^ bf16 [BH][T][d], box {64, 128}
  CUtensorMap tmV;    // v  bf16 [BH][T][d], box {64, 128}
  CUtensorMap tmBk;   // Bk bf16 [BH][4 dh][d], box {64, 64}
  CUtensorMap tmBv;   // Bv bf16 [BH][d][2 dh], box {64, 64}
  CUtensorMap tmPk;   // Phik bf16 [BH][rows][4 dh], box {16, 32}, no swizzle (stores)
  CUtensorMap tmPv;   // Phiv bf16 [BH][rows][2 dh], box {16, 32}, no swizzle (stores)
  int bh_count, n_slices, n_row_tiles, kb_count;
  int x_row0;         // first token of the chunk
  int rows_valid;     // tokens in the chunk
  int dh;
  int64_t T;
  const float* lr;    // [BH][T][3]
  float* dlr;         // [BH][T][3], accumulated
};

struct BwdKeyOp {
  using Params = BwdKeyParams;
  static constexpr int kXBytes = kBM * kBK * 2;          // 16 KB: 128 rows x 64 K
  static constexpr int kSBytes = 64 * kBK * 2;           // 8 KB: one 64-wide operand slice
  static constexpr int kOffV = kXBytes;
  static constexpr int kOffBk = 2 * kXBytes;              // 4 slices of 64 rows, K-major (N = 256)
  static constexpr int kOffBv = kOffBk + 4 * kSBytes;     // 2 MN blocks of 64 columns (N = 128)
  static constexpr int kStageBytes = kOffBv + 2 * kSBytes;   // 80 KB
  static constexpr int kStages = 2;
  static constexpr int kStgPlane = 32 * 16 * 2;         // 32 rows x 16 bf16, dense
  static constexpr int kStgWarp = 6 * kStgPlane;          // the 6 factor planes of one warp
  static constexpr int kExtraBytes = 2 * kEpiWarps * kStgWarp;   // 48 KB
  static constexpr int kAccCols = 384;
  static constexpr int kAccBufs = 1;
  static constexpr int kIssuers = 2;
  static constexpr int kEpiGroups = 2;   // group g: hidden units 32 g .. 32 g + 31 of the slice
  struct Tile { int slice, row0, bh; };

  // Hidden slice fastest: CTAs running together share the token tile in L2.
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
    tma_prefetch_map(&p.tmV);
    tma_prefetch_map(&p.tmBk);
    tma_prefetch_map(&p.tmBv);
  }
  __device__ static void load(const Params& p, const Tile& t, int kb, uint8_t* st, uint64_t* bar) {
    const int k = kb * kBK, row = p.x_row0 + t.row0, hs = t.slice * 64;
    tma_load_3d(st, &p.tmX, bar, k, row, t.bh);
    tma_load_3d(st + kOffV, &p.tmV, bar, k, row, t.bh);
#pragma unroll
    for (int g = 0; g < 4; ++g) tma_load_3d(st + kOffBk + g * kSBytes, &p.tmBk, bar, k, g * p.dh + hs, t.bh);
    tma_load_3d(st + kOffBv, &p.tmBv, bar, hs, k, t.bh);
    tma_load_3d(st + kOffBv + kSBytes, &p.tmBv, bar, p.dh + hs, k, t.bh);
  }
  __device__ static void mma(const Params&, const Tile&, uint32_t st, uint32_t tmem, int kb, int issuer) {
    const bool f = kb == 0;
    if (issuer == 0) {
      constexpr uint32_t id0 = idesc_bf16(kBM, 256, false, false);
      mma_kblock<false, false>(tmem, st, 0, st + kOffBk, 0, id0, f);
    } else {
      constexpr uint32_t id1 = idesc_bf16(kBM, 128, false, true);
      mma_kblock<false, true>(tmem + 256, st + kOffV, 0, st + kOffBv, 8192u, id1, f);
    }
  }
  __device__ static void epilogue_done(int lane) {
    if (lane == 0) bulk_wait_all();
  }
  __device__ static void epilogue(const Params& p, const Tile& t, uint32_t tmem, int quarter, int lane,
                                  uint8_t* extra, int group) {
    const int r = quarter * 32 + lane;
    const int grow = t.row0 + r;
    const bool valid = grow < p.rows_valid;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int dh = p.dh;
    const int64_t lrow = static_cast<int64_t>(t.bh) * p.T + p.x_row0 + grow;
    float e1 = 0.f, e2 = 0.f, e3 = 0.f;
    if (valid) {
      e1 = p.lr[lrow * 3];
      e2 = p.lr[lrow * 3 + 1];
      e3 = p.lr[lrow * 3 + 2];
    }
    uint8_t* stg = extra + (group * kEpiWarps + quarter) * kStgWarp;
    const uint32_t srow = smem_u32(stg) + lane * 32;   // this thread's row in each staged plane
    const int y = t.row0 + quarter * 32;
    float g1 = 0.f, g2 = 0.f, g3 = 0.f;
#pragma unroll 1
    for (int j = 32 * group; j < 32 * group + 32; j += 16) {
      float z1[16], z3[16], pp[16], rr[16], u[16], qq[16];
      __syncwarp();
      tmem_ld16(tq + j, z1);
      tmem_ld16(tq + 64 + j, z3);
      tmem_ld16(tq + 128 + j, pp);
      tmem_ld16(tq + 192 + j, rr);
      tmem_ld16(tq + 256 + j, u);
      tmem_ld16(tq + 320 + j, qq);
      tmem_ld_wait();
      // the previous chunk's bulk stores have read the staging tiles
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {   // columns j + 8 hf .. j + 8 hf + 7, stored as soon as computed
        uint32_t w[6][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int c = 8 * hf + 2 * i;
          const HvpOut a = hvp_factors<true>(z1[c], u[c], z3[c], pp[c], qq[c], rr[c], e1, e2, e3);
          const HvpOut b =
              hvp_factors<true>(z1[c + 1], u[c + 1], z3[c + 1], pp[c + 1], qq[c + 1], rr[c + 1], e1, e2, e3);
          w[0][i] = pack_bf16x2(a.fz1, b.fz1);
          w[1][i] = pack_bf16x2(a.fz3, b.fz3);
          w[2][i] = pack_bf16x2(a.fp, b.fp);
          w[3][i] = pack_bf16x2(a.fr, b.fr);
          w[4][i] = pack_bf16x2(a.fu, b.fu);
          w[5][i] = pack_bf16x2(a.fq, b.fq);
          g1 += a.g1 + b.g1;
          g2 += a.g2 + b.g2;
          g3 += a.g3 + b.g3;
        }
#pragma unroll
        for (int m = 0; m < 6; ++m) st_shared_v4(srow + m * kStgPlane + 16 * hf, w[m][0], w[m][1], w[m][2], w[m][3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int x = t.slice * 64 + j;
#pragma unroll
        for (int m = 0; m < 4; ++m) tma_store_3d(&p.tmPk, stg + m * kStgPlane, m * dh + x, y, t.bh);
#pragma unroll
        for (int m = 0; m < 2; ++m) tma_store_3d(&p.tmPv, stg + (4 + m) * kStgPlane, m * dh + x, y, t.bh);
        bulk_commit_group();
      }
    }
    if (valid) {
      atomicAdd(p.dlr + lrow * 3, g1);
      atomicAdd(p.dlr + lrow * 3 + 1, g2);
      atomicAdd(p.dlr + lrow * 3 + 2, g3);
    }
  }
};

}  // namespace lact
