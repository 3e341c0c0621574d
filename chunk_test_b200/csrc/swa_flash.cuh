// swa_flash.cuh -- fused sliding-window attention for head dims up to 256:
// the scores and probabilities of a block of 128 queries stay on chip (TMEM
// and shared memory) while it walks the key blocks of its window, with an
// online softmax ("LaCT架构核心思想解析" §1.1).  Inputs: Qt [BH][T][d]
// from k_swa_prologue_q (q' times the key scale) and the caller's k and v
// [BH][T][d] as given; the scores Qt . k differ from q' . k' by a constant
// per query, which the softmax removes.
//
// Persistent CTAs over tiles (head, 128-query block m); per tile the key
// blocks j0..m, j0 = max(0, m - w/128), each of 128 keys.  Warps:
//   0     TMA producer of the queries (once per tile) and of each key
//         block's K tile (K-major operand of S).
//   7     TMA producer of the V tiles (MN-major operand of P V), in two
//         halves of 64 keys with their own barriers, so the next block's
//         first half loads while the second half of P V runs.  Keys and
//         values have separate producers: a K load never waits for P V.
//   1     S issuer: S_j = Q K_j^T into one of two TMEM buffers (128 cols).
//   2..5  softmax, one query row per thread: masked row max of S_j, the
//         online rescale of the output row in TMEM when the max grows,
//         P_j = exp(s - max) in bf16 into a swizzled K-major smem tile, and
//         the row sum; after the last block, out = O / sum in bf16.  The
//         softmax is the plain one up to rounding: the reference max of a
//         row only lags the true running max by at most 8 in log2 units.
//   6     P V issuer: O += P_j V_j (TMEM, D columns).
// Every wait is bounded (mbar_wait); a wait that gives up records the
// timeout in the device status word and the CTA stops.
#pragma once

#include "umma_kernels.cuh"

namespace lact {

struct SwaFlashParams {
  CUtensorMap tmQ;   // Qt [BH][T][d], box {64, 128}
  CUtensorMap tmK;   // k  [BH][T][d], box {64, 128}
  CUtensorMap tmV;   // v  [BH][T][d], box {64, 64}
  int bh_count, nb;  // heads, 128-query blocks per head
  int window;        // w (a multiple of 128)
  float scale;       // 1 / sqrt(d)
  __nv_bfloat16* out;
  int64_t T;
};

constexpr int kSwaThreads = 256;
constexpr int kSwaPvWarp = 6;
constexpr int kSwaVWarp = 7;

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])));
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x by the ex2.approx instruction (-inf gives 0)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
struct SwaCfg {
  static_assert(D % 64 == 0 && D >= 64 && D <= 256, "flash window attention head dim");
  static constexpr int kKb = D / 64;
  static constexpr int kQBytes = kKb * 16384;       // 128 rows x D
  static constexpr int kKBytes = kKb * 16384;       // 128 keys x D (K-major)
  static constexpr int kVBytes = 2 * kKb * 8192;    // 128 keys x D (MN-major, 64-key x 64-d boxes)
  static constexpr int kPBytes = 2 * 16384;         // 128 rows x 128 keys
  static constexpr int kBudget = 229376 - kQBytes - kPBytes;
  static constexpr int kStagesRaw = kBudget / (kKBytes + kVBytes);
  static constexpr int kStages = kStagesRaw < 1 ? 1 : (kStagesRaw > 3 ? 3 : kStagesRaw);
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKBytes;
  static constexpr int kOffP = kOffV + kStages * kVBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  // qfull qempty | kfull kempty (x stages) | vfull vempty (x 2 halves x stages) | sfull[2] sempty[2] |
  // pfull pempty | ofull oempty
  static constexpr int kBars = 2 + 2 * kStages + 4 * kStages + 4 + 2 + 2;
  static constexpr int kSmem = kOffBar + kBars * 8 + 16 + 1024;
  static constexpr uint32_t kColO = 0, kColS = 256;
};

template <int D>
__global__ void __launch_bounds__(kSwaThreads, 1) k_swa_flash(const __grid_constant__ SwaFlashParams p) {
  griddep_launch();
  using C = SwaCfg<D>;
  constexpr int KS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* qfull = bar;
  uint64_t* qempty = bar + 1;
  uint64_t* kfull = bar + 2;
  uint64_t* kempty = kfull + KS;
  uint64_t* vfull = kempty + KS;     // [stage * 2 + half]
  uint64_t* vempty = vfull + 2 * KS;
  uint64_t* sfull = vempty + 2 * KS;
  uint64_t* sempty = sfull + 2;
  uint64_t* pfull = sempty + 2;
  uint64_t* pempty = pfull + 1;
  uint64_t* ofull = pempty + 1;
  uint64_t* oempty = ofull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + C::kBars);

  __shared__ int abort_cta;
  if (threadIdx.x == 0) abort_cta = *reinterpret_cast<volatile int*>(&g_status);
  __syncthreads();
  if (abort_cta) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.nb * p.bh_count;
  const int wb = p.window / 128;   // key blocks strictly before the query block

  if (warp == 0 && lane == 0) {
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(&kfull[i], 1);
      mbar_init(&kempty[i], 1);
    }
    for (int i = 0; i < 2 * KS; ++i) {
      mbar_init(&vfull[i], 1);
      mbar_init(&vempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&sempty[i], kEpiWarps);
    }
    mbar_init(pfull, kEpiWarps);
    mbar_init(pempty, 1);
    mbar_init(ofull, 1);
    mbar_init(oempty, kEpiWarps);
    fence_barrier_init();
    tma_prefetch_map(&p.tmQ);
    tma_prefetch_map(&p.tmK);
    tma_prefetch_map(&p.tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync_converged();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int ik = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tc) {
        const int m = tile % p.nb, bh = tile / p.nb;
        if (tc > 0 && !mbar_wait(qempty, (tc - 1) & 1)) break;
        mbar_arrive_expect_tx(qfull, C::kQBytes);
        for (int kb = 0; kb < C::kKb; ++kb) tma_load_3d(smem + kb * 16384, &p.tmQ, qfull, kb * 64, m * 128, bh);
        const int j0 = m - wb > 0 ? m - wb : 0;
        for (int j = j0; j <= m; ++j, ++ik) {
          const int st = ik % KS;
          const int prow = j * 128;   // first key of block j
          if (ik >= KS && !mbar_wait(&kempty[st], ((ik / KS) - 1) & 1)) { ok = false; break; }
          uint8_t* kd = smem + C::kOffK + st * C::kKBytes;
          mbar_arrive_expect_tx(&kfull[st], C::kKBytes);
          for (int kb = 0; kb < C::kKb; ++kb) tma_load_3d(kd + kb * 16384, &p.tmK, &kfull[st], kb * 64, prow, bh);
        }
      }
    }
  } else if (warp == kSwaVWarp) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) {
      int ik = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
        const int m = tile % p.nb, bh = tile / p.nb;
        const int j0 = m - wb > 0 ? m - wb : 0;
        for (int j = j0; ok && j <= m; ++j, ++ik) {
          const int st = ik % KS;
          uint8_t* vd = smem + C::kOffV + st * C::kVBytes;
          for (int h = 0; h < 2; ++h) {
            uint64_t* full = &vfull[2 * st + h];
            if (ik >= KS && !mbar_wait(&vempty[2 * st + h], ((ik / KS) - 1) & 1)) { ok = false; break; }
            mbar_arrive_expect_tx(full, C::kVBytes / 2);
            for (int nb = 0; nb < C::kKb; ++nb)
              tma_load_3d(vd + (h * C::kKb + nb) * 8192, &p.tmV, full, nb * 64, j * 128 + h * 64, bh);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S issuer
    if (lane == 0) {
      constexpr uint32_t ids = idesc_bf16(kBM, 128, false, false);
      const uint32_t sbase = smem_u32(smem);
      int ik = 0, sc = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tc) {
        const int m = tile % p.nb;
        const int j0 = m - wb > 0 ? m - wb : 0;
        if (!mbar_wait(qfull, tc & 1)) break;
        for (int j = j0; ok && j <= m; ++j, ++ik, ++sc) {
          const int st = ik % KS, sb = sc & 1;
          if (sc >= 2 && !mbar_wait(&sempty[sb], ((sc >> 1) - 1) & 1)) { ok = false; break; }
          if (!mbar_wait(&kfull[st], (ik / KS) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sd = tmem + C::kColS + sb * 128;
          for (int kb = 0; kb < C::kKb; ++kb)
            mma_kblock<false, false>(sd, sbase + kb * 16384, 0, sbase + C::kOffK + st * C::kKBytes + kb * 16384, 0,
                                     ids, kb == 0);
          umma_commit(&kempty[st]);
          umma_commit(&sfull[sb]);
        }
        if (ok) umma_commit(qempty);
      }
    }
  } else if (warp == kSwaPvWarp) {
    // ------------------------------------------------------------ P V issuer
    if (lane == 0) {
      constexpr uint32_t ido = idesc_bf16(kBM, D, false, true);
      const uint32_t sbase = smem_u32(smem);
      int ik = 0, pc = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tc) {
        const int m = tile % p.nb;
        const int j0 = m - wb > 0 ? m - wb : 0;
        for (int j = j0; j <= m; ++j, ++ik, ++pc) {
          const int st = ik % KS;
          if (j == j0 && tc > 0 && !mbar_wait(oempty, (tc - 1) & 1)) { ok = false; break; }
          if (!mbar_wait(pfull, pc & 1)) { ok = false; break; }
          const uint32_t vb = sbase + C::kOffV + st * C::kVBytes;
          for (int kk = 0; kk < 2 && ok; ++kk) {   // keys 64 kk .. 64 kk + 63
            if (!mbar_wait(&vfull[2 * st + kk], (ik / KS) & 1)) { ok = false; break; }
            tc_fence_after();
            mma_kblock<false, true>(tmem + C::kColO, sbase + C::kOffP + kk * 16384, 0, vb + kk * C::kKb * 8192,
                                    8192, ido, j == j0 && kk == 0);
            umma_commit(&vempty[2 * st + kk]);
          }
          if (!ok) break;
          umma_commit(pempty);
        }
        if (ok) umma_commit(ofull);
      }
    }
  } else if (warp >= 2 && warp < 2 + kEpiWarps) {
    // ------------------------------------------------------------ softmax
    // One query row per thread.  The row of S_j is loaded into registers in
    // one go, so the S buffer is released before the exponentials.  Scores
    // stay in raw units; exp(x) is computed as 2^(x log2 e) with the ex2
    // instruction, the scale folded into one FMA per score.  The reference
    // max mx of a row is raised only when a block's max exceeds it by more
    // than 8 in log2 units, so the output row is rescaled rarely and the
    // unnormalised probabilities stay below 2^8.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t prow_s = smem_u32(smem + C::kOffP) + r * 128;
    const float c2 = p.scale * 1.4426950408889634f;   // log2 e / sqrt(d)
    int sc = 0, pc = 0, tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tc) {
      const int m = tile % p.nb, bh = tile / p.nb;
      const int j0 = m - wb > 0 ? m - wb : 0;
      float mx = -INFINITY, sum = 0.f;
      for (int j = j0; j <= m; ++j, ++sc, ++pc) {
        const int sb = sc & 1;
        // waits are made warp-uniform: the TMEM loads and stores below are
        // warp-collective, so every lane must take the same path
        if (!__all_sync(0xffffffffu, mbar_wait(&sfull[sb], (sc >> 1) & 1))) { ok = false; break; }
        tc_fence_after();
        const uint32_t ts = tq + C::kColS + sb * 128;
        float sv[128];
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 16) tmem_ld16(ts + c0, sv + c0);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
        // only the diagonal block and the block at the window's start are cut
        if (j == m || j == m - wb) {
          const int hi = j == m ? r : 127;
          const int lo = j == m - wb ? r + 1 : 0;
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i < lo || i > hi) sv[i] = -INFINITY;
        }
        float b8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) b8[i] = sv[i];
#pragma unroll
        for (int i = 8; i < 128; ++i) b8[i & 7] = fmaxf(b8[i & 7], sv[i]);
        const float bm = fmaxf(fmaxf(fmaxf(b8[0], b8[1]), fmaxf(b8[2], b8[3])),
                               fmaxf(fmaxf(b8[4], b8[5]), fmaxf(b8[6], b8[7])));
        float a = 1.0f;
        bool grow = false;
        if (mx == -INFINITY) {
          mx = bm;   // no earlier key of this row: its output row and sum are zero
        } else if ((bm - mx) * c2 > 8.0f) {
          grow = true;
          a = ex2_approx((mx - bm) * c2);
          mx = bm;
        }
        const float off = mx == -INFINITY ? 0.f : -mx * c2;
        uint32_t hw[64];
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float e0 = ex2_approx(fmaf(sv[2 * i], c2, off));
          const float e1 = ex2_approx(fmaf(sv[2 * i + 1], c2, off));
          ps[i & 3] += e0 + e1;
          hw[i] = pack_bf16x2(e0, e1);
        }
        // the previous block's P V has finished with O and with the P tile
        if (pc > 0 && !__all_sync(0xffffffffu, mbar_wait(pempty, (pc - 1) & 1))) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {   // the whole warp runs it; factor 1 in other rows
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            __syncwarp();
            tmem_ld16(tq + C::kColO + c0, o);
            tmem_ld16(tq + C::kColO + c0 + 16, o + 16);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= a;
            tmem_st16(tq + C::kColO + c0, o);
            tmem_st16(tq + C::kColO + c0 + 16, o + 16);
          }
          tmem_st_wait();
        }
        sum = sum * a + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
        // row r of the K-major 128-byte-swizzled P tile: 64 keys per 16 KB
        // block, 16-byte chunk g holds keys 8g..8g+7
#pragma unroll
        for (int g = 0; g < 16; ++g)
          st_shared_v4(prow_s + (g >> 3) * 16384 + (((g & 7) ^ (r & 7)) << 4), hw[4 * g], hw[4 * g + 1],
                       hw[4 * g + 2], hw[4 * g + 3]);
        tc_fence_before();
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(pfull);
      }
      if (!ok) break;
      // O is complete: out = O / sum
      if (!__all_sync(0xffffffffu, mbar_wait(ofull, tc & 1))) break;
      tc_fence_after();
      const float inv = sum > 0.f ? 1.0f / sum : 0.f;
      __nv_bfloat16* dst = p.out + (static_cast<int64_t>(bh) * p.T + static_cast<int64_t>(m) * 128 + r) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        __syncwarp();
        tmem_ld16(tq + C::kColO + c0, o);
        tmem_ld16(tq + C::kColO + c0 + 16, o + 16);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < 4; ++g)
          st_global_v4(dst + c0 + 8 * g, pack_bf16x2(o[8 * g] * inv, o[8 * g + 1] * inv),
                       pack_bf16x2(o[8 * g + 2] * inv, o[8 * g + 3] * inv),
                       pack_bf16x2(o[8 * g + 4] * inv, o[8 * g + 5] * inv),
                       pack_bf16x2(o[8 * g + 6] * inv, o[8 * g + 7] * inv));
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
