// apply_kernel.cuh -- the fused apply of one chunk on the tensor cores:
//   out = (silu(Q^ W1^T) * (Q^ W3^T)) W2^T      ("大块测试时训练（LaCT）技术解析"
//   §2.1, eq. 2; SwiGLU memory of "LaCT：以大分块更新…" 「局部注意力与非线性
//   记忆相互补充」)
// for one 128-query tile per step of a persistent tile loop.  The q^ tile
// stays in shared memory; the hidden dimension is walked in slices of 64:
//   Z_s = Q^ [W1_s; W3_s]^T          tcgen05, fp32 in TMEM (2 buffers)
//   H_s = silu(Z1_s) * Z3_s          epilogue warps, bf16 into shared memory
//   O  += H_s W2[:, s]^T             tcgen05, fp32 in TMEM
// so the gated hidden activations never leave the SM.
//
// Two warps issue the MMAs: warp 1 the Z MMAs and warp 6 the O MMAs, each
// from one lane.  An MMA issue holds its thread until the tensor core takes
// it, so every barrier wait or commit between two MMAs of one issuer leaves
// the tensor core idle for tens of cycles; with the Z and O streams on
// separate warps, one issuer's waits overlap the other's MMAs (and the
// tensor core computes Z_{s+1} while the epilogue warps gate slice s).
//
// Warps: 0 TMA producer, 1 TMEM allocator + Z issuer, 2..5 epilogue,
// 6 O issuer.
// Head dims D = 64, 128, 192 or 256 (TMEM: D columns of O + 2 x 128 of Z).
#pragma once

#include "umma_kernels.cuh"

namespace lact {

struct ApplyParams {
  CUtensorMap tmQ;    // q^ [BH, Tq, d] bf16, box {64, 128, 1}
  CUtensorMap tmW;    // shadows as [3*BH, dh, d] (planes 0 and 2 used), box {64, 64, 1}
  CUtensorMap tmW2;   // W2 shadow plane [BH, d, dh], box {64, d, 1}
  int bh_count, dh;
  int n_row_tiles;    // 128-query tiles of this chunk
  int q_row0;         // first query row of the chunk
  int rows_valid;     // queries in this chunk
  __nv_bfloat16* out; // [BH, Tq, d]
  int64_t Tq;
  const float* scale; // [BH, Tq] per-query output factor, or null
};

constexpr int kApplyThreads = 224;   // 7 warps
constexpr int kApplyOWarp = 6;

template <int D>
struct ApplyCfg {
  static_assert(D % 64 == 0 && D >= 64 && D <= 256, "apply kernel head dim");
  static constexpr int kKb = D / 64;              // K blocks of d
  static constexpr int kQBytes = kKb * 16384;     // resident q^ tile
  static constexpr int kABytes = 16384;           // W1_s + W3_s rows of one K block
  static constexpr int kAStages = 3;
  static constexpr int kBBytes = D * 128;         // W2[:, s] (D rows x 64 hidden)
  static constexpr int kBStages = 2;
  static constexpr int kHBytes = 16384;           // H_s (128 rows x 64 hidden)
  static constexpr int kOffA = kQBytes;
  static constexpr int kOffB = kOffA + kAStages * kABytes;
  static constexpr int kOffH = kOffB + kBStages * kBBytes;
  static constexpr int kOffBar = kOffH + 2 * kHBytes;
  static constexpr int kBars = 2 + 2 * kAStages + 2 * kBStages + 2 + 2 + 2 + 2 + 2;
  static constexpr int kSmem = kOffBar + kBars * 8 + 16 + 1024;
  static constexpr uint32_t kColO = 0, kColZ = 256;
};

template <int D>
__global__ void __launch_bounds__(kApplyThreads, 1) k_apply(const __grid_constant__ ApplyParams p) {
  griddep_launch();
  using C = ApplyCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* qfull = bar;
  uint64_t* qempty = bar + 1;
  uint64_t* afull = bar + 2;
  uint64_t* aempty = afull + C::kAStages;
  uint64_t* bfull = aempty + C::kAStages;
  uint64_t* bempty = bfull + C::kBStages;
  uint64_t* zfull = bempty + C::kBStages;
  uint64_t* zempty = zfull + 2;
  uint64_t* hfull = zempty + 2;
  uint64_t* hempty = hfull + 2;
  uint64_t* ofull = hempty + 2;
  uint64_t* oempty = ofull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + C::kBars);

  __shared__ int abort_cta;
  if (threadIdx.x == 0) abort_cta = *reinterpret_cast<volatile int*>(&g_status);
  __syncthreads();
  if (abort_cta) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.n_row_tiles * p.bh_count;
  const int S = p.dh / 64;

  if (warp == 0 && lane == 0) {
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int i = 0; i < C::kAStages; ++i) { mbar_init(&afull[i], 1); mbar_init(&aempty[i], 1); }
    for (int i = 0; i < C::kBStages; ++i) { mbar_init(&bfull[i], 1); mbar_init(&bempty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&zfull[i], 1);
      mbar_init(&zempty[i], kEpiWarps);
      mbar_init(&hfull[i], kEpiWarps);
      mbar_init(&hempty[i], 1);
    }
    mbar_init(ofull, 1);
    mbar_init(oempty, kEpiWarps);
    fence_barrier_init();
    tma_prefetch_map(&p.tmQ);
    tma_prefetch_map(&p.tmW);
    tma_prefetch_map(&p.tmW2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync_converged();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // after the local setup, before any global access

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int ia = 0, ib = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tc) {
        const int rt = tile % p.n_row_tiles, bh = tile / p.n_row_tiles;
        const int row = p.q_row0 + rt * kBM;
        if (tc > 0 && !mbar_wait(qempty, (tc - 1) & 1)) break;
        mbar_arrive_expect_tx(qfull, C::kQBytes);
        for (int kb = 0; kb < C::kKb; ++kb) tma_load_3d(smem + kb * 16384, &p.tmQ, qfull, kb * 64, row, bh);
        for (int s = 0; ok && s < S; ++s) {
          for (int kb = 0; kb < C::kKb; ++kb, ++ia) {
            const int st = ia % C::kAStages;
            if (ia >= C::kAStages && !mbar_wait(&aempty[st], ((ia / C::kAStages) - 1) & 1)) { ok = false; break; }
            uint8_t* dst = smem + C::kOffA + st * C::kABytes;
            mbar_arrive_expect_tx(&afull[st], C::kABytes);
            tma_load_3d(dst, &p.tmW, &afull[st], kb * 64, s * 64, bh);                       // W1_s
            tma_load_3d(dst + 8192, &p.tmW, &afull[st], kb * 64, s * 64, 2 * p.bh_count + bh);  // W3_s
          }
          if (!ok) break;
          const int st = ib % C::kBStages;
          if (ib >= C::kBStages && !mbar_wait(&bempty[st], ((ib / C::kBStages) - 1) & 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&bfull[st], C::kBBytes);
          tma_load_3d(smem + C::kOffB + st * C::kBBytes, &p.tmW2, &bfull[st], s * 64, 0, bh);   // W2[:, s]
          ++ib;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ Z issuer
    if (lane == 0) {
      constexpr uint32_t idz = idesc_bf16(kBM, 128, false, false);
      const uint32_t sbase = smem_u32(smem);
      int ia = 0, tc = 0, zc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tc) {
        if (!mbar_wait(qfull, tc & 1)) break;
        for (int s = 0; ok && s < S; ++s) {  // Z_s = Q^ [W1; W3]_s^T
          const int zb = zc & 1;
          if (zc >= 2 && !mbar_wait(&zempty[zb], ((zc >> 1) - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t zd = tmem + C::kColZ + zb * 128;
          for (int kb = 0; kb < C::kKb; ++kb, ++ia) {
            const int st = ia % C::kAStages;
            if (!mbar_wait(&afull[st], (ia / C::kAStages) & 1)) { ok = false; break; }
            mma_kblock<false, false>(zd, sbase + kb * 16384, 0, sbase + C::kOffA + st * C::kABytes, 0,
                                     idz, kb == 0);
            umma_commit(&aempty[st]);
          }
          if (!ok) break;
          umma_commit(&zfull[zb]);
          ++zc;
        }
        if (ok) umma_commit(qempty);  // every read of this tile's q^ issued
      }
    }
  } else if (warp == kApplyOWarp) {
    // ------------------------------------------------------------ O issuer
    if (lane == 0) {
      constexpr uint32_t ido = idesc_bf16(kBM, D, false, false);
      const uint32_t sbase = smem_u32(smem);
      int ib = 0, tc = 0, hc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tc) {
        for (int s = 0; ok && s < S; ++s) {  // O += H_s W2[:, s]^T
          const int hb = hc & 1, st = ib % C::kBStages;
          if (s == 0 && tc > 0 && !mbar_wait(oempty, (tc - 1) & 1)) { ok = false; break; }
          if (!mbar_wait(&hfull[hb], (hc >> 1) & 1)) { ok = false; break; }
          if (!mbar_wait(&bfull[st], (ib / C::kBStages) & 1)) { ok = false; break; }
          tc_fence_after();
          mma_kblock<false, false>(tmem + C::kColO, sbase + C::kOffH + hb * C::kHBytes, 0,
                                   sbase + C::kOffB + st * C::kBBytes, 0, ido, s == 0);
          umma_commit(&bempty[st]);
          umma_commit(&hempty[hb]);
          ++ib;
          ++hc;
        }
        if (ok) umma_commit(ofull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t hrow = smem_u32(smem + C::kOffH) + r * 128;
    int zc = 0, hc = 0, tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tc) {
      const int rt = tile % p.n_row_tiles, bh = tile / p.n_row_tiles;
      for (int s = 0; s < S; ++s, ++zc, ++hc) {
        const int zb = zc & 1, hb = hc & 1;
        if (!mbar_wait(&zfull[zb], (zc >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        uint32_t hw[32];
#pragma unroll
        for (int j = 0; j < 64; j += 16) {
          float z1[16], z3[16];
          __syncwarp();
          tmem_ld16(tq + C::kColZ + zb * 128 + j, z1);
          tmem_ld16(tq + C::kColZ + zb * 128 + 64 + j, z3);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float a0 = z1[2 * i], a1 = z1[2 * i + 1];
            hw[j / 2 + i] = pack_bf16x2(a0 * sigmoid_fast(a0) * z3[2 * i], a1 * sigmoid_fast(a1) * z3[2 * i + 1]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&zempty[zb]);
        if (hc >= 2 && !mbar_wait(&hempty[hb], ((hc >> 1) - 1) & 1)) { ok = false; break; }
        // Row r of a K-major, 128-byte-swizzled tile: 16-byte chunk c sits at
        // chunk position c ^ (r % 8).
        const uint32_t base = hrow + hb * C::kHBytes;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(base + ((c ^ (r & 7)) << 4), hw[4 * c], hw[4 * c + 1], hw[4 * c + 2], hw[4 * c + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&hfull[hb]);
      }
      if (!ok) break;
      if (!mbar_wait(ofull, tc & 1)) break;
      tc_fence_after();
      const int grow = rt * kBM + r;
      const bool valid = grow < p.rows_valid;
      const int64_t orow = static_cast<int64_t>(bh) * p.Tq + p.q_row0 + grow;
      __nv_bfloat16* dst = p.out + orow * D;
      const float s = (p.scale && valid) ? __ldg(p.scale + orow) : 1.0f;
#pragma unroll 1
      for (int j = 0; j < D; j += 16) {
        float v[16];
        __syncwarp();
        tmem_ld16(tq + C::kColO + j, v);
        tmem_ld_wait();
        if (valid) {
          if (p.scale) {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= s;
          }
          st_global_v4(dst + j, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                       pack_bf16x2(v[6], v[7]));
          st_global_v4(dst + j + 8, pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                       pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(oempty);
    }
  }
  tc_fence_before();
  cta_sync_converged();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace lact
