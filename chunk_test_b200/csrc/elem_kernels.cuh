// elem_kernels.cuh -- memory-bound kernels of the LaCT layer, shared by the
// bf16 and fp32 paths: the q/k prologue, fast-weight state set-up and
// write-back, per-chunk mean of beta, the update rule with the row-wise
// renorm, and the Frobenius normalisation that starts Newton-Schulz.
//
// Internal fast-weight layout ("hidden-major"): three fp32 masters per
// (b, h), each [dh, d]:  plane 0 = W1, plane 1 = W2^T, plane 2 = W3, stored
// as Wm[j][bh][dh][d].  Renorm rows of W1/W3 are rows of their planes; rows
// of W2 are COLUMNS of plane 1.
#pragma once

#include "sm100.cuh"

namespace lact {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// q, k <- silu(q)/||silu(q)||, silu(k)/||silu(k)|| over the head dim
// ("LaCT架构核心思想解析" §1.2).  One warp per row; rows of q first, then k.
// An all-zero row stays zero.
// ---------------------------------------------------------------------------
constexpr int kMaxRowPerLane = 16;  // d <= 512

// With kh_lo (bf16 only) the keys are also written as the lo part of a
// split-bf16 pair (kh_lo = bf16(k^ - kh)).
template <typename T>
__global__ void __launch_bounds__(256) k_qk_prologue(const T* __restrict__ q, T* __restrict__ qh,
                                                     int64_t q_rows, const T* __restrict__ k,
                                                     T* __restrict__ kh, int64_t k_rows, int d,
                                                     T* __restrict__ kh_lo) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= q_rows + k_rows) return;
  const T* src = row < q_rows ? q + row * d : k + (row - q_rows) * d;
  T* dst = row < q_rows ? qh + row * d : kh + (row - q_rows) * d;
  float s[kMaxRowPerLane];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxRowPerLane; ++i) {
    const int c = lane + 32 * i;
    float x = 0.f;
    if (c < d) x = to_f(src[c]);
    const float y = x / (1.0f + __expf(-x));
    s[i] = y;
    ss += y * y;
  }
  ss = warp_sum(ss);
  const float inv = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
  T* dst_lo = (kh_lo && row >= q_rows) ? kh_lo + (row - q_rows) * d : nullptr;
#pragma unroll
  for (int i = 0; i < kMaxRowPerLane; ++i) {
    const int c = lane + 32 * i;
    if (c < d) {
      const float y = s[i] * inv;
      const T hi = from_f<T>(y);
      dst[c] = hi;
      if (dst_lo) dst_lo[c] = from_f<T>(y - to_f(hi));
    }
  }
}

// bf16 shadow of an fp32 value, and its split-bf16 lo part when asked for.
__device__ __forceinline__ void store_shadow(__nv_bfloat16* hi, __nv_bfloat16* lo, int64_t o, float x) {
  if (!hi) return;
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  hi[o] = h;
  if (lo) lo[o] = __float2bfloat16_rn(x - __bfloat162float(h));
}

// ---------------------------------------------------------------------------
// State set-up: Wm[j][bh] from the caller's initial weights (plane 1 is the
// transpose of W2), optional bf16 shadow, momentum zeroed.  32x32 tiles of
// the [dh, d] planes; grid (ceil(d/32), ceil(dh/32), 3*BH), block (32, 8).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_init_state(const float* __restrict__ w1,
                                                    const float* __restrict__ w2,
                                                    const float* __restrict__ w3, int H,
                                                    int w_shared, int BH, int d, int dh,
                                                    float* __restrict__ Wm,
                                                    __nv_bfloat16* __restrict__ Ws,
                                                    __nv_bfloat16* __restrict__ Ws_lo,
                                                    float* __restrict__ Mm) {
  __shared__ float tile[32][33];
  const int j = blockIdx.z / BH, bh = blockIdx.z % BH;
  const int src_h = w_shared ? bh % H : bh;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int64_t plane = static_cast<int64_t>(dh) * d;
  if (j == 1) {
    // W2 [d, dh]: read rows c (= output column) coalesced along dh.
    const float* s = w2 + static_cast<int64_t>(src_h) * plane;
    for (int i = ty; i < 32; i += 8) {
      const int c = c0 + i, r = r0 + tx;
      tile[i][tx] = (c < d && r < dh) ? s[static_cast<int64_t>(c) * dh + r] : 0.f;
    }
    __syncthreads();
    for (int i = ty; i < 32; i += 8) {
      const int r = r0 + i, c = c0 + tx;
      if (r < dh && c < d) {
        const int64_t o = (static_cast<int64_t>(j) * BH + bh) * plane + static_cast<int64_t>(r) * d + c;
        const float x = tile[tx][i];
        Wm[o] = x;
        store_shadow(Ws, Ws_lo, o, x);
        if (Mm) Mm[o] = 0.f;
      }
    }
  } else {
    const float* s = (j == 0 ? w1 : w3) + static_cast<int64_t>(src_h) * plane;
    for (int i = ty; i < 32; i += 8) {
      const int r = r0 + i, c = c0 + tx;
      if (r < dh && c < d) {
        const int64_t o = (static_cast<int64_t>(j) * BH + bh) * plane + static_cast<int64_t>(r) * d + c;
        const float x = s[static_cast<int64_t>(r) * d + c];
        Wm[o] = x;
        store_shadow(Ws, Ws_lo, o, x);
        if (Mm) Mm[o] = 0.f;
      }
    }
  }
}

// Write-back: w1_out, w3_out from planes 0, 2; w2_out = plane 1 transposed.
__global__ void __launch_bounds__(256) k_finalize_state(const float* __restrict__ Wm, int BH, int d,
                                                        int dh, float* __restrict__ w1o,
                                                        float* __restrict__ w2o,
                                                        float* __restrict__ w3o) {
  __shared__ float tile[32][33];
  const int j = blockIdx.z / BH, bh = blockIdx.z % BH;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int64_t plane = static_cast<int64_t>(dh) * d;
  const float* s = Wm + (static_cast<int64_t>(j) * BH + bh) * plane;
  if (j == 1) {
    for (int i = ty; i < 32; i += 8) {
      const int r = r0 + i, c = c0 + tx;
      tile[i][tx] = (r < dh && c < d) ? s[static_cast<int64_t>(r) * d + c] : 0.f;
    }
    __syncthreads();
    float* o = w2o + static_cast<int64_t>(bh) * plane;
    for (int i = ty; i < 32; i += 8) {
      const int c = c0 + i, r = r0 + tx;
      if (c < d && r < dh) o[static_cast<int64_t>(c) * dh + r] = tile[tx][i];
    }
  } else {
    float* o = (j == 0 ? w1o : w3o) + static_cast<int64_t>(bh) * plane;
    for (int i = ty; i < 32; i += 8) {
      const int r = r0 + i, c = c0 + tx;
      if (r < dh && c < d) o[static_cast<int64_t>(r) * d + c] = s[static_cast<int64_t>(r) * d + c];
    }
  }
}

// beta_bar[bh][c] = mean of beta over chunk c's tokens (one warp per entry).
__global__ void __launch_bounds__(256) k_beta_mean(const float* __restrict__ beta, int BH, int64_t T,
                                                   int64_t chunk, int nch,
                                                   float* __restrict__ beta_bar) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<int64_t>(BH) * nch) return;
  const int bh = static_cast<int>(w / nch), c = static_cast<int>(w % nch);
  const int64_t t0 = c * chunk, t1 = (t0 + chunk < T) ? t0 + chunk : T;
  const float* b = beta + static_cast<int64_t>(bh) * T;
  float s = 0.f;
  for (int64_t t = t0 + lane; t < t1; t += 32) s += b[t];
  s = warp_sum(s);
  if (lane == 0) beta_bar[w] = s / static_cast<float>(t1 - t0);
}

// ---------------------------------------------------------------------------
// Update rule + row-wise renorm ("大块测试时训练（LaCT）技术解析" §2.2.1 eq. 8;
// "LaCT架构核心思想解析" §1.2).  The source S holds the NEGATED update
// direction: the negated chunk gradient summed over `splits` partial planes
// (GD, momentum) or the Newton-Schulz output of the negated gradient (Muon;
// the quintic is odd, so NS(-G) = -NS(G)).  With U' = -U:
//   GD / Muon:  U' = S
//   momentum:   M' <- beta_bar M' + S,  U' = M'       (M' = -M)
//   W' = W + U', then each renorm row of W' scaled to its norm before.
// Blocks [0, row_blocks): rows of planes 0 and 2 (one warp per row, length d).
// Blocks [row_blocks, ...): plane 1 in groups of 32 columns (length dh each).
// ---------------------------------------------------------------------------
struct RuleParams {
  float* Wm;
  __nv_bfloat16* Ws;      // bf16 shadow or null
  __nv_bfloat16* Ws_lo;   // split-bf16 lo part of the shadow or null
  const float* S;         // [splits][3][BH][dh][d]
  int splits;
  int64_t split_stride;   // elements between partial planes
  float* Mm;              // momentum (rule 1) or null
  const float* beta_bar;  // [BH][nch]
  int nch, chunk_idx;
  int rule;
  int BH, dh, d;
  int row_blocks;
};

__device__ __forceinline__ float rule_dir(const RuleParams& p, int64_t o, float bb) {
  float s = 0.f;
  for (int i = 0; i < p.splits; ++i) s += p.S[i * p.split_stride + o];
  if (p.rule == 1) {
    s = bb * p.Mm[o] + s;
    p.Mm[o] = s;
  }
  return s;
}

__global__ void __launch_bounds__(256) k_rule_renorm(const RuleParams p) {
  const int64_t plane = static_cast<int64_t>(p.dh) * p.d;
  if (static_cast<int>(blockIdx.x) < p.row_blocks) {
    const int64_t row = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t rows_per_plane = static_cast<int64_t>(p.BH) * p.dh;
    if (row >= 2 * rows_per_plane) return;
    const int j = row < rows_per_plane ? 0 : 2;
    const int64_t rr = row % rows_per_plane;  // bh * dh + r
    const int bh = static_cast<int>(rr / p.dh);
    const float bb = p.rule == 1 ? p.beta_bar[bh * p.nch + p.chunk_idx] : 0.f;
    const int64_t base = static_cast<int64_t>(j) * p.BH * plane + rr * p.d;
    float on = 0.f, nn = 0.f;
    for (int c = lane; c < p.d; c += 32) {
      const float w = p.Wm[base + c];
      const float wn = w + rule_dir(p, base + c, bb);
      p.Wm[base + c] = wn;
      on += w * w;
      nn += wn * wn;
    }
    on = warp_sum(on);
    nn = warp_sum(nn);
    const float sc = nn > 0.f ? sqrtf(on) / sqrtf(nn) : 0.f;
    __syncwarp();
    for (int c = lane; c < p.d; c += 32) {
      const float w = p.Wm[base + c] * sc;
      p.Wm[base + c] = w;
      store_shadow(p.Ws, p.Ws_lo, base + c, w);
    }
  } else {
    __shared__ float red_o[8][32], red_n[8][32], scale[32];
    const int cb = blockIdx.x - p.row_blocks;
    const int groups = (p.d + 31) / 32;
    const int bh = cb / groups, c = (cb % groups) * 32 + (threadIdx.x & 31);
    const int wrp = threadIdx.x >> 5;
    const bool cv = c < p.d;
    const float bb = p.rule == 1 ? p.beta_bar[bh * p.nch + p.chunk_idx] : 0.f;
    const int64_t base = (static_cast<int64_t>(1) * p.BH + bh) * plane;
    float on = 0.f, nn = 0.f;
    if (cv) {
      for (int r = wrp; r < p.dh; r += 8) {
        const int64_t o = base + static_cast<int64_t>(r) * p.d + c;
        const float w = p.Wm[o];
        const float wn = w + rule_dir(p, o, bb);
        p.Wm[o] = wn;
        on += w * w;
        nn += wn * wn;
      }
    }
    red_o[wrp][threadIdx.x & 31] = on;
    red_n[wrp][threadIdx.x & 31] = nn;
    __syncthreads();
    if (wrp == 0) {
      float so = 0.f, sn = 0.f;
      for (int i = 0; i < 8; ++i) {
        so += red_o[i][threadIdx.x];
        sn += red_n[i][threadIdx.x];
      }
      scale[threadIdx.x] = sn > 0.f ? sqrtf(so) / sqrtf(sn) : 0.f;
    }
    __syncthreads();
    if (cv) {
      const float sc = scale[threadIdx.x & 31];
      for (int r = wrp; r < p.dh; r += 8) {
        const int64_t o = base + static_cast<int64_t>(r) * p.d + c;
        const float w = p.Wm[o] * sc;
        p.Wm[o] = w;
        store_shadow(p.Ws, p.Ws_lo, o, w);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Newton-Schulz start ("大块测试时训练（LaCT）技术解析" §2.2.1, eqs. 9-10):
// X0 = S / (||S||_F + 1e-7) per matrix, S = sum of the partial gradient
// planes.  Pass 1 writes S into Y and a fixed-order partial sum of squares
// per block; pass 2 sums the partials of its matrix in a fixed order and
// scales Y in place (plus the bf16 copy).  Deterministic.
// grid (nblk, items) with items = 3*BH, 256 threads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float block_sum_256(float v, float* red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 8; ++i) s += red[i];
    red[8] = s;
  }
  __syncthreads();
  s = red[8];
  __syncthreads();
  return s;
}

__global__ void __launch_bounds__(256) k_ns_sumsq(const float* __restrict__ S, int splits,
                                                  int64_t split_stride, int64_t plane,
                                                  float* __restrict__ Y, float* __restrict__ part) {
  __shared__ float red[9];
  const int item = blockIdx.y;
  const int64_t per = (plane + gridDim.x - 1) / gridDim.x;
  const int64_t e0 = blockIdx.x * per, e1 = (e0 + per < plane) ? e0 + per : plane;
  const int64_t base = static_cast<int64_t>(item) * plane;
  float ss = 0.f;
  for (int64_t e = e0 + threadIdx.x; e < e1; e += 256) {
    float s = 0.f;
    for (int i = 0; i < splits; ++i) s += S[i * split_stride + base + e];
    Y[base + e] = s;
    ss += s * s;
  }
  ss = block_sum_256(ss, red);
  if (threadIdx.x == 0) part[static_cast<int64_t>(item) * gridDim.x + blockIdx.x] = ss;
}

__global__ void __launch_bounds__(256) k_ns_scale(float* __restrict__ Y,
                                                  __nv_bfloat16* __restrict__ Yb,
                                                  __nv_bfloat16* __restrict__ Yb_lo, int64_t plane,
                                                  const float* __restrict__ part, int nblk,
                                                  float eps) {
  __shared__ float sc;
  const int item = blockIdx.y;
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < nblk; ++i) s += part[static_cast<int64_t>(item) * nblk + i];
    sc = 1.0f / (sqrtf(s) + eps);
  }
  __syncthreads();
  const int64_t per = (plane + gridDim.x - 1) / gridDim.x;
  const int64_t e0 = blockIdx.x * per, e1 = (e0 + per < plane) ? e0 + per : plane;
  const int64_t base = static_cast<int64_t>(item) * plane;
  for (int64_t e = e0 + threadIdx.x; e < e1; e += 256) {
    const float y = Y[base + e] * sc;
    Y[base + e] = y;
    store_shadow(Yb, Yb_lo, base + e, y);
  }
}

}  // namespace lact
