// pair_kernels.cuh -- CTA-pair (cta_group::2) tcgen05 GEMM tiles.
//
// Two CTAs of a 2-CTA cluster (on two SMs) share one 256-row output tile:
// each CTA stages its own 128 rows of A and half of B's N columns, and the
// even CTA issues M = 256 MMAs that read A and B from both CTAs' shared
// memory and accumulate each CTA's 128 rows in its own TMEM.  Per SM this
// halves the B operand's TMA traffic and its shared-memory reads relative
// to a 128-row tile of the same N, which is what limits the one-CTA kernels
// (their TMA writes and operand reads share one SM's shared memory).
//
// Pipeline (persistent, one pair per two SMs):
//   warp 0  both CTAs: TMA producer.  The even CTA posts the stage's byte
//           count (both halves) on its `full` barrier, and both CTAs' tile
//           loads (their cta_group::2 form) count their bytes there.
//   warp 1  TMEM allocation (cta_group::2, both CTAs); the even CTA's lane 0
//           issues the MMAs; each commit arrives on the same barrier in
//           both CTAs (stage releases, accumulator completion).
//   warps 2..5  both CTAs: epilogue of their own 128 rows; they release an
//           accumulator buffer by arriving on the even CTA's barrier.
// All waits are bounded (mbar_wait); no thread leaves before the closing
// cluster barrier, so a timed-out wait ends the pair together.
#pragma once

#include "umma_kernels.cuh"

namespace lact {

// ------------------------------------------------------------------ cluster
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared::cluster address of `saddr` (a shared::cta address) in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Cluster-wide barrier of every thread (warp-divergent callers allowed).
__device__ __forceinline__ void cluster_sync_all() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Arrive on an mbarrier of any CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Tile load into this CTA's shared memory, its bytes counted on an mbarrier
// of either CTA of the pair.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// ------------------------------------------------------------------ tcgen05, pair
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (+)= A * B over the pair: M = 256 (128 rows per CTA), B's N split in halves.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this offset in both CTAs of the pair when
// every pair MMA issued so far by this thread is done.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 4 pair UMMAs (K = 16 each) of one 64-wide K block; same layouts as mma_kblock.
template <bool A_MN, bool B_MN>
__device__ __forceinline__ void mma_kblock_pair(uint32_t d_tmem, uint32_t a_base, uint32_t a_lbo, uint32_t b_base,
                                                uint32_t b_lbo, uint32_t idesc, bool first) {
#pragma unroll
  for (int k = 0; k < kBK / 16; ++k) {
    const uint32_t ao = A_MN ? k * 2048u : k * 32u;
    const uint32_t bo = B_MN ? k * 2048u : k * 32u;
    const uint64_t ad = smem_desc_sw128(a_base + ao, A_MN ? a_lbo : 16u, 1024u);
    const uint64_t bd = smem_desc_sw128(b_base + bo, B_MN ? b_lbo : 16u, 1024u);
    umma_bf16_pair(d_tmem, ad, bd, idesc, (first && k == 0) ? 0u : 1u);
  }
}

// The pair pipeline.  Op supplies kStages, kStageBytes (per CTA; both CTAs
// load the same number of bytes), kExtraBytes (shared memory for the
// epilogue, after the ring), kAccCols, kAccBufs, Tile, num_tiles() (pair
// tiles), map_tile(p, idx, rank), num_kb(), prefetch(),
// load(p, t, kb, stage, bar_cluster_addr), mma(p, t, stage, tmem, kb)
// (even CTA), epilogue(p, t, tmem, quarter, lane, extra) and
// epilogue_done(lane).
template <class Op>
__global__ void __launch_bounds__(kThreads, 1) __cluster_dims__(2, 1, 1)
    umma_pair_kernel(const __grid_constant__ typename Op::Params p) {
  griddep_launch();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int S = Op::kStages;
  constexpr int NB = Op::kAccBufs;
  constexpr uint32_t kCols = TmemCols<NB * Op::kAccCols>::value;
  static_assert(NB * Op::kAccCols <= 512, "accumulator buffers must fit in TMEM");
  uint8_t* extra = smem + S * Op::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(extra + Op::kExtraBytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;      // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2], used in the even CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int ntiles = Op::num_tiles(p);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);
    }
    fence_barrier_init();
    Op::prefetch(p);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // after the local setup, before any global access

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < ntiles; tile += npairs) {
        const typename Op::Tile t = Op::map_tile(p, tile, rank);
        const int nkb = Op::num_kb(p, t);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          if (it >= S && !mbar_wait(&empty[s], ((it / S) - 1) & 1)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[s], 2u * Op::kStageBytes);
          Op::load(p, t, kb, smem + s * Op::kStageBytes, mapa_rank(smem_u32(&full[s]), 0));
        }
      }
      // Every stage release (including the last S, committed by the even
      // CTA's MMAs) has landed before this CTA may leave.
      for (int i = it > S ? it - S : 0; ok && i < it; ++i)
        if (!mbar_wait(&empty[i % S], (i / S) & 1)) ok = false;
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < ntiles; tile += npairs, ++local) {
        const typename Op::Tile t = Op::map_tile(p, tile, rank);
        const int nkb = Op::num_kb(p, t);
        const int buf = local % NB, use = local / NB;
        if (use > 0 && !mbar_wait(&acc_empty[buf], (use - 1) & 1)) break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * Op::kAccCols;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(&full[s], (it / S) & 1)) { ok = false; break; }
          tc_fence_after();
          Op::mma(p, t, smem_u32(smem + s * Op::kStageBytes), acc, kb);
          umma_commit_pair(&empty[s]);
        }
        umma_commit_pair(&acc_full[buf]);
      }
    }
  } else {
    const uint32_t acc_empty_leader = mapa_rank(smem_u32(&acc_empty[0]), 0);
    int local = 0;
    for (int tile = pair; tile < ntiles; tile += npairs, ++local) {
      const typename Op::Tile t = Op::map_tile(p, tile, rank);
      const int buf = local % NB, use = local / NB;
      if (!mbar_wait(&acc_full[buf], use & 1)) break;
      tc_fence_after();
      Op::epilogue(p, t, tmem + buf * Op::kAccCols, warp & 3, lane, extra);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader + buf * 8u);
    }
    Op::epilogue_done(lane);
  }
  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still use its memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, kCols);
  }
}

// ---------------------------------------------------------------------------
// GemmOp on CTA pairs: 256-row tiles, B's BN columns split between the CTAs.
// Same parameters and epilogue as GemmOp (no split-bf16 mode).
// ---------------------------------------------------------------------------
template <bool A_MN, bool B_MN, int BN>
struct GemmPairOp {
  using Base = GemmOp<A_MN, B_MN, BN, false>;
  using Params = GemmParams;
  static_assert(BN % 128 == 0, "each CTA holds BN / 2 columns of B, a multiple of 64");
  static constexpr int kHalfN = BN / 2;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = kHalfN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (196608 / kStageBytes) < 8 ? (196608 / kStageBytes) : 8;
  static constexpr int kAccCols = TmemCols<BN>::value;
  static constexpr int kAccBufs = 2;
  // The epilogue's staging: per epilogue warp two 32 x 32 fp32 tiles (the
  // bulk-store path) or the generic path's tile, whichever is larger.
  static constexpr int kStgBytes = 2 * 32 * 32 * 4;
  static constexpr int kExtraBytes =
      kEpiWarps * kStgBytes > Base::kExtraBytes ? kEpiWarps * kStgBytes : Base::kExtraBytes;
  using Tile = typename Base::Tile;   // m0 is this CTA's first row

  __device__ static int num_tiles(const Params& p) { return p.n_tiles; }
  // Pair tiles: nt_m counts 256-row tiles.
  __device__ static Tile map_tile(const Params& p, int idx, uint32_t rank) {
    Tile t = Base::map_tile(p, idx);
    t.m0 = 2 * t.m0 + static_cast<int>(rank) * kBM;
    return t;
  }
  __device__ static int num_kb(const Params& p, const Tile& t) { return Base::num_kb(p, t); }
  __device__ static void prefetch(const Params& p) {
    tma_prefetch_map(&p.tmA);
    tma_prefetch_map(&p.tmB);
    if (p.alt_group >= 0) tma_prefetch_map(&p.tmB2);
  }
  __device__ static void load(const Params& p, const Tile& t, int kb, uint8_t* st, uint32_t bar) {
    const int kk = (t.split * p.kb_count + kb) * kBK;
    const int ak = p.a_k0 + kk, bk = p.b_k0 + kk;
    const int half = (t.m0 / kBM) & 1;  // this CTA's rank in the pair
    const int n0 = t.n0 + half * kHalfN;
    if (A_MN) {
      tma_load_3d_pair(st, &p.tmA, bar, t.m0, ak, t.item);
      tma_load_3d_pair(st + 8192, &p.tmA, bar, t.m0 + 64, ak, t.item);
    } else {
      tma_load_3d_pair(st, &p.tmA, bar, ak, t.m0, t.item);
    }
    const CUtensorMap* mb = t.alt ? &p.tmB2 : &p.tmB;
    if (B_MN) {
#pragma unroll
      for (int b = 0; b < kHalfN / 64; ++b) tma_load_3d_pair(st + kABytes + b * 8192, mb, bar, n0 + b * 64, bk, t.zb);
    } else {
      tma_load_3d_pair(st + kABytes, mb, bar, bk, n0, t.zb);
    }
  }
  __device__ static void mma(const Params&, const Tile&, uint32_t st, uint32_t tmem, int kb) {
    constexpr uint32_t id = idesc_bf16(2 * kBM, BN, A_MN, B_MN);
    mma_kblock_pair<A_MN, B_MN>(tmem, st, 8192u, st + kABytes, 8192u, id, kb == 0);
  }
  __device__ static void epilogue(const Params& p, const Tile& t, uint32_t tmem, int quarter, int lane,
                                  uint8_t* extra) {
    if (!p.out_tma) {
      Base::epilogue(p, t, tmem, quarter, lane, extra);
      return;
    }
    // The warp's 32 rows leave in 32-column pieces: TMEM -> registers ->
    // a swizzled 4 KB staging tile -> one bulk tensor store, two tiles in
    // flight per warp.  Row-per-thread global stores (one cache line per
    // thread per instruction) took about 6 us per 128 x 256 fp32 tile.
    const uint32_t tq = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool tr = p.tr_group >= 0 && (t.item / p.tr_mod) == p.tr_group;
    uint8_t* stg = extra + quarter * kStgBytes;
    const uint32_t sb = smem_u32(stg);
    const int row0 = t.m0 + quarter * 32;
#pragma unroll 1
    for (int j = 0; j < BN; j += 32) {
      const int slot = (j >> 5) & 1;
      float v[32];
      __syncwarp();
      tmem_ld16(tq + j, v);
      tmem_ld16(tq + j + 16, v + 16);
      tmem_ld_wait();
      if (lane == 0) bulk_wait_read_le1();  // the store that last used this slot has read it
      __syncwarp();
      const uint32_t tb = sb + slot * 4096;
      if (!tr) {
        // row `lane` (an output row), 16-byte chunk c at c ^ (lane % 8)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(tb + lane * 128 + ((c ^ (lane & 7)) << 4), __float_as_uint(v[4 * c]),
                       __float_as_uint(v[4 * c + 1]), __float_as_uint(v[4 * c + 2]), __float_as_uint(v[4 * c + 3]));
      } else {
        // transposed: staging row i holds output column n0 + j + i, element
        // `lane` of it this thread's row; 16-byte chunk lane / 4 at (lane / 4) ^ (i % 8)
#pragma unroll
        for (int i = 0; i < 32; ++i)
          st_shared_f32(tb + i * 128 + (((lane >> 2) ^ (i & 7)) << 4) + (lane & 3) * 4, v[i]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (!tr)
          tma_store_3d(&p.tmOut, stg + slot * 4096, t.n0 + j, row0, t.out_item);
        else
          tma_store_3d(&p.tmOutT, stg + slot * 4096, row0, t.n0 + j, t.out_item);
        bulk_commit_group();
      }
    }
  }
  __device__ static void epilogue_done(int lane) {
    if (lane == 0) bulk_wait_all();
  }
};

template <class Op>
constexpr int umma_pair_smem_bytes() {
  return Op::kStages * Op::kStageBytes + Op::kExtraBytes + (2 * Op::kStages + 4) * 8 + 16 + 1024;
}

}  // namespace lact
