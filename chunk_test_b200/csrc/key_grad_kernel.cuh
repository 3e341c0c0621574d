// key_grad_kernel.cuh -- fused key forward + chunk gradient for small heads
// (d = 64, dh = 128), the shape of a posed-image-set chunk of ~200K tokens:
// per 128-token tile
//   DH   = V W2                        (N = 128, all hidden units)
//   Z_h  = K^ [W1_h; W3_h]^T           (N = 128, hidden half h = 0, 1)
//   E1 = lr1 DH z3 silu'(z1), Eh = lr2 silu(z1) z3, E3 = lr3 DH silu(z1)
//        (epilogue warps, bf16, into swizzled shared-memory operands)
//   -G1 += E1^T K^, -G3 += E3^T K^, -G2^T += Eh^T V   (M = 128 hidden, N = 64)
// ("大块测试时训练（LaCT）技术解析" §2.1 eqs. 4-5; loss and per-token rates of
// "LaCT：以大分块更新…" 「局部注意力与非线性记忆相互补充」).
// The three gradients accumulate in TMEM over the CTA's whole token range,
// so the per-token factors never leave the SM; each work item (head, token
// split) writes one fp32 partial gradient set, summed later in fixed order.
// The k^ / v tiles serve twice: as the K-major A operand of the forward and,
// viewed MN-major (d contiguous), as the B operand of the gradients.
//
// Warps: 0 TMA producer, 1 TMEM allocator and forward MMA issuer, 2..17
// epilogue (four warps per 32-lane TMEM quarter, each taking 16 of every 64
// columns), 18 gradient MMA issuer.  Each issuer runs an MMA group as soon
// as the epilogue's mbarrier arrivals free its inputs: warp 1 Z_1 once Z_0
// is read (zempty) and the next tile's DH and Z_0 once Z_1 and DH are read
// (zempty); warp 18 the gradients once E is written (efull), an item's
// first once the previous item's accumulators are read (gempty).  An MMA
// issue holds its thread until the tensor core takes it, and one thread
// keeps the tensor core fed only part of the time with these small MMAs
// (measured: about 90 cycles per N = 64 gradient MMA), so the two streams
// come from two warps, which overlap each other's gaps; issued from an
// epilogue thread (about 3.6K of a tile's 7K cycles) the waits held back
// the whole epilogue group at its next barrier.
#pragma once

#include "apply_kernel.cuh"

namespace lact {

struct KeyGradParams {
  CUtensorMap tmK;    // k^ [BH, T, 64] bf16, box {64, 128, 1}
  CUtensorMap tmV;    // v  [BH, T, 64] bf16, box {64, 128, 1}
  CUtensorMap tmW;    // shadows as [3*BH, 128, 64] (planes 0 and 2), box {64, 64, 1}
  CUtensorMap tmW2;   // W2 shadow plane [BH, 64, 128], box {64, 64, 1}
  int bh_count;
  int splits;         // token splits per head (work items = bh_count * splits)
  int n_tiles;        // 128-token tiles of the chunk
  int x_row0;         // first token of the chunk
  int rows_valid;     // tokens in the chunk
  int T;
  const float* lr;    // [BH, T, 3]
  float* P;           // partial gradients [splits][3][BH][plane], W2's in [d, dh]
};

constexpr int kKGThreads = 608;   // 19 warps
constexpr int kKGGradWarp = 18;
constexpr int kKGEpiWarps = 16;

struct KGCfg {
  static constexpr int kOffW13 = 0;          // [W1 rows 0-63 | W3 rows 0-63 | W1 64-127 | W3 64-127]
  static constexpr int kOffW2 = 32768;       // [W2 hidden 0-63 | 64-127] MN blocks of 64 d rows
  static constexpr int kOffRing = 49152;     // 2 slots x (k^ 16 KB, v 16 KB)
  static constexpr int kSlot = 32768;
  static constexpr int kOffE = kOffRing + 2 * kSlot;  // E1, Eh, E3: 2 MN blocks of 16 KB each
  static constexpr int kEBytes = 32768;
  static constexpr int kOffBar = kOffE + 3 * kEBytes;
  static constexpr int kBars = 2 + 4 + 2 + 1 + 2 + 2;
  static constexpr int kSmem = kOffBar + kBars * 8 + 16 + 1024;
  // TMEM columns
  static constexpr uint32_t kColG = 0;       // G1 [0,64), G3 [64,128), G2^T [128,192)
  static constexpr uint32_t kColZ = 192;     // Z_h: z1 [0,64), z3 [64,128)
  static constexpr uint32_t kColD = 320;     // DH [0,128)
};

__global__ void __launch_bounds__(kKGThreads, 1) k_key_grad64(const __grid_constant__ KeyGradParams p) {
  griddep_launch();
  using C = KGCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* wfull = bar;
  uint64_t* wempty = bar + 1;
  uint64_t* tfull = bar + 2;        // [2]
  uint64_t* tempty = bar + 4;       // [2]
  uint64_t* zfull = bar + 6;
  uint64_t* zempty = bar + 7;
  uint64_t* efull = bar + 9;
  uint64_t* eempty = bar + 10;
  uint64_t* gfull = bar + 11;
  uint64_t* gempty = bar + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + C::kBars);

  __shared__ int abort_cta;
  if (threadIdx.x == 0) abort_cta = *reinterpret_cast<volatile int*>(&g_status);
  __syncthreads();
  if (abort_cta) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int items = p.bh_count * p.splits;
  const int tps = (p.n_tiles + p.splits - 1) / p.splits;   // tiles per split

  if (warp == 0 && lane == 0) {
    mbar_init(wfull, 1);
    mbar_init(wempty, 1);
    // a ring slot is free once both issuers' MMAs that read it are done
    for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], 2); }
    mbar_init(zfull, 1);
    mbar_init(zempty, kKGEpiWarps);
    mbar_init(efull, kKGEpiWarps);
    mbar_init(eempty, 1);
    mbar_init(gfull, 1);
    mbar_init(gempty, kKGEpiWarps);
    fence_barrier_init();
    tma_prefetch_map(&p.tmK);
    tma_prefetch_map(&p.tmV);
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

  // item -> (head, split); its tiles [t0, t1)
  auto item_range = [&](int item, int& bh, int& s, int& t0, int& t1) {
    bh = item / p.splits;
    s = item % p.splits;
    t0 = s * tps;
    t1 = t0 + tps < p.n_tiles ? t0 + tps : p.n_tiles;
  };

  constexpr uint32_t idf = idesc_bf16(kBM, 128, false, false);   // Z_h
  constexpr uint32_t idd = idesc_bf16(kBM, 128, false, true);    // DH (W2 MN-major)
  constexpr uint32_t idg = idesc_bf16(kBM, 64, true, true);      // gradients
  const uint32_t sb = smem_u32(smem);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0, ic = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
        int bh, s, t0, t1;
        item_range(item, bh, s, t0, t1);
        if (t0 >= t1) continue;
        if (ic > 0 && !mbar_wait(wempty, (ic - 1) & 1)) break;
        ++ic;
        mbar_arrive_expect_tx(wfull, 49152);
        tma_load_3d(smem + C::kOffW13, &p.tmW, wfull, 0, 0, bh);                          // W1 0-63
        tma_load_3d(smem + C::kOffW13 + 8192, &p.tmW, wfull, 0, 0, 2 * p.bh_count + bh);  // W3 0-63
        tma_load_3d(smem + C::kOffW13 + 16384, &p.tmW, wfull, 0, 64, bh);                 // W1 64-127
        tma_load_3d(smem + C::kOffW13 + 24576, &p.tmW, wfull, 0, 64, 2 * p.bh_count + bh);
        tma_load_3d(smem + C::kOffW2, &p.tmW2, wfull, 0, 0, bh);                          // W2[:, 0-63]
        tma_load_3d(smem + C::kOffW2 + 8192, &p.tmW2, wfull, 64, 0, bh);                  // W2[:, 64-127]
        for (int t = t0; t < t1; ++t, ++it) {
          const int slot = it & 1;
          if (it >= 2 && !mbar_wait(&tempty[slot], ((it >> 1) - 1) & 1)) { ok = false; break; }
          uint8_t* dst = smem + C::kOffRing + slot * C::kSlot;
          const int row = p.x_row0 + t * kBM;
          mbar_arrive_expect_tx(&tfull[slot], C::kSlot);
          tma_load_3d(dst, &p.tmK, &tfull[slot], 0, row, bh);
          tma_load_3d(dst + 16384, &p.tmV, &tfull[slot], 0, row, bh);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, ic = 0, zr = 0;
      bool ok = true;
      // DH and Z_0 of the tile in ring slot `slot` (after its k^ / v landed)
      auto first_half = [&](int it_) -> bool {
        const int slot = it_ & 1;
        if (!mbar_wait(&tfull[slot], (it_ >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t kx = sb + C::kOffRing + slot * C::kSlot, vx = kx + 16384;
        mma_kblock<false, true>(tmem + C::kColD, vx, 0, sb + C::kOffW2, 8192u, idd, true);
        mma_kblock<false, false>(tmem + C::kColZ, kx, 0, sb + C::kOffW13, 0, idf, true);
        umma_commit(zfull);
        return true;
      };
      for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
        int bh, s, t0, t1;
        item_range(item, bh, s, t0, t1);
        if (t0 >= t1) continue;
        // the weights of this item; the Z / DH buffers free (the previous
        // tile's last reads, zempty phase zr - 1)
        ok = mbar_wait(wfull, ic & 1) && (zr == 0 || mbar_wait(zempty, (zr - 1) & 1)) && first_half(it);
        for (int t = t0; ok && t < t1; ++t, ++it) {
          const int slot = it & 1;
          const uint32_t kx = sb + C::kOffRing + slot * C::kSlot;
          // Z_1 once Z_0 is read
          if (!mbar_wait(zempty, zr & 1)) { ok = false; break; }
          ++zr;
          tc_fence_after();
          mma_kblock<false, false>(tmem + C::kColZ, kx, 0, sb + C::kOffW13 + 16384, 0, idf, true);
          umma_commit(zfull);
          umma_commit(&tempty[slot]);          // this issuer's reads of the slot are issued
          if (t == t1 - 1) umma_commit(wempty);  // and of the item's weights
          // the next tile's DH and Z_0 once Z_1 and DH are read
          if (t + 1 < t1) {
            if (!mbar_wait(zempty, zr & 1)) { ok = false; break; }
            ++zr;
            if (!first_half(it + 1)) { ok = false; break; }
          }
        }
        // the last tile's second Z read frees the buffers for the next item
        // (its zempty phase is waited at the next item's start)
        if (ok) ++zr;
        ++ic;
      }
    }
  } else if (warp == kKGGradWarp) {
    // ------------------------------------------------------------ gradient MMA issuer
    if (lane == 0) {
      int it = 0, ic = 0, g = 0;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
        int bh, s, t0, t1;
        item_range(item, bh, s, t0, t1);
        if (t0 >= t1) continue;
        for (int t = t0; ok && t < t1; ++t, ++it, ++g) {
          const int slot = it & 1;
          const uint32_t kx = sb + C::kOffRing + slot * C::kSlot, vx = kx + 16384;
          const bool first = t == t0;
          // E written; the slot's k^ / v landed (its phase is already
          // complete: the epilogue read this tile's Z); for an item's first
          // tile, the previous item's accumulators read
          if (!mbar_wait(efull, g & 1) || !mbar_wait(&tfull[slot], (it >> 1) & 1) ||
              (first && ic > 0 && !mbar_wait(gempty, (ic - 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {   // two 64-token halves of the tile
            const uint32_t ko = kk * 8192;   // 64 token rows x 128 B
            mma_kblock<true, true>(tmem + C::kColG, sb + C::kOffE + ko, 16384u, kx + ko, 8192u, idg,
                                   first && kk == 0);
            mma_kblock<true, true>(tmem + C::kColG + 64, sb + C::kOffE + 2 * C::kEBytes + ko, 16384u,
                                   kx + ko, 8192u, idg, first && kk == 0);
            mma_kblock<true, true>(tmem + C::kColG + 128, sb + C::kOffE + C::kEBytes + ko, 16384u,
                                   vx + ko, 8192u, idg, first && kk == 0);
          }
          umma_commit(eempty);
          umma_commit(&tempty[slot]);
          if (t == t1 - 1) umma_commit(gfull);
        }
        ++ic;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;                 // 0..15
    const int quarter = warp & 3;
    const int cg = ew >> 2;                  // which 16 of every 64 columns
    const int r = quarter * 32 + lane;       // token row (TMEM lane) of the tile
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const int64_t plane = 128 * 64;
    const uint32_t erow = sb + C::kOffE + r * 128;
    const uint32_t sw0 = ((2 * cg) ^ (r & 7)) << 4, sw1 = ((2 * cg + 1) ^ (r & 7)) << 4;
    int ic = 0, zc = 0, g = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < items; item += gridDim.x) {
      int bh, s, t0, t1;
      item_range(item, bh, s, t0, t1);
      if (t0 >= t1) continue;
      for (int t = t0; ok && t < t1; ++t, ++g) {
        const int grow = t * kBM + r;
        float eta0 = 0.f, eta1 = 0.f, eta2 = 0.f;
        if (grow < p.rows_valid) {
          const float* l = p.lr + (static_cast<int64_t>(bh) * p.T + p.x_row0 + grow) * 3;
          eta0 = l[0];
          eta1 = l[1];
          eta2 = l[2];
        }
        for (int h = 0; h < 2; ++h, ++zc) {
          if (!mbar_wait(zfull, zc & 1)) { ok = false; break; }
          tc_fence_after();
          float z1[16], z3[16], u[16];
          const int c = cg * 16;
          __syncwarp();
          tmem_ld16(tq + C::kColZ + c, z1);
          tmem_ld16(tq + C::kColZ + 64 + c, z3);
          tmem_ld16(tq + C::kColD + h * 64 + c, u);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(zempty);   // Z_h (and, for h = 1, DH) read
          uint32_t e1w[8], ehw[8], e3w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float v1[2], vh[2], v3[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const float a = z1[2 * i + q], bz = z3[2 * i + q], gd = u[2 * i + q];
              const float sg = sigmoid_fast(a);
              const float sa = a * sg;
              const float ds = fmaf(sa, 1.0f - sg, sg);       // silu'(a) = s + a s (1 - s)
              v1[q] = (eta0 * gd) * (bz * ds);
              vh[q] = eta1 * (sa * bz);
              v3[q] = (eta2 * gd) * sa;
            }
            e1w[i] = pack_bf16x2(v1[0], v1[1]);
            ehw[i] = pack_bf16x2(vh[0], vh[1]);
            e3w[i] = pack_bf16x2(v3[0], v3[1]);
          }
          if (h == 0 && g > 0 && !mbar_wait(eempty, (g - 1) & 1)) { ok = false; break; }
          // Row r of MN block h of each factor; 16-byte chunk c sits at c ^ (r % 8).
          const uint32_t rb = erow + h * 16384;
          st_shared_v4(rb + sw0, e1w[0], e1w[1], e1w[2], e1w[3]);
          st_shared_v4(rb + sw1, e1w[4], e1w[5], e1w[6], e1w[7]);
          st_shared_v4(rb + C::kEBytes + sw0, ehw[0], ehw[1], ehw[2], ehw[3]);
          st_shared_v4(rb + C::kEBytes + sw1, ehw[4], ehw[5], ehw[6], ehw[7]);
          st_shared_v4(rb + 2 * C::kEBytes + sw0, e3w[0], e3w[1], e3w[2], e3w[3]);
          st_shared_v4(rb + 2 * C::kEBytes + sw1, e3w[4], e3w[5], e3w[6], e3w[7]);
        }
        if (!ok) break;
        fence_async_smem();   // the gradient MMAs read E through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(efull);
      }
      if (!ok) break;
      // this item's partial gradients: TMEM lane = hidden unit
      if (!mbar_wait(gfull, ic & 1)) break;
      tc_fence_after();
      const int hr = r;  // hidden row of the gradient tile
      float* base = p.P + static_cast<int64_t>(s) * 3 * p.bh_count * plane;
#pragma unroll 1
      for (int cc = 0; cc < 48; cc += 16) {
        const int col = cg * 48 + cc;          // of the 192 gradient columns
        float v[16];
        __syncwarp();
        tmem_ld16(tq + C::kColG + col, v);
        tmem_ld_wait();
        const int j = col / 64, c0 = col % 64;   // 0: W1, 1: W3, 2: W2^T
        if (j < 2) {
          float* o = base + (static_cast<int64_t>(j == 0 ? 0 : 2) * p.bh_count + bh) * plane + hr * 64 + c0;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            st_global_v4(o + 4 * i, __float_as_uint(v[4 * i]), __float_as_uint(v[4 * i + 1]),
                         __float_as_uint(v[4 * i + 2]), __float_as_uint(v[4 * i + 3]));
        } else {  // W2's gradient stored in W2's [d, dh] layout
          float* o = base + (static_cast<int64_t>(p.bh_count) + bh) * plane + hr;
#pragma unroll
          for (int i = 0; i < 16; ++i) o[(c0 + i) * 128] = v[i];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(gempty);   // the accumulators may be overwritten by the next item
      ++ic;
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
