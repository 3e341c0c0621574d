// elem_kernels.cuh -- memory-bound kernels of the LaCT layer, shared by the
// bf16 and fp32 paths: the q/k prologue, fast-weight state set-up and
// write-back, per-chunk mean of beta, the update rule with the row-wise
// renorm, and the Frobenius normalisation that starts Newton-Schulz.
//
// Internal fast-weight layout: three fp32 masters per (b, h) in their
// natural layouts, Wm[j][bh]: plane 0 = W1 [dh, d], plane 1 = W2 [d, dh],
// plane 2 = W3 [dh, d] (dh*d elements each).  Every renorm row (rows of W1
// and W3 of length d, rows of W2 of length dh) is a contiguous row.
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
// ("LaCT架构核心思想解析" §1.2).  Rows of q first, then k.  S threads share a
// row (S a power of two <= 32, so a row's reduction stays inside its warp);
// each thread moves 16-byte vectors of VEC elements.  An all-zero row stays
// zero.  With kh_lo (bf16 only) the keys are also written as the lo part of
// a split-bf16 pair (kh_lo = bf16(k^ - kh)).
// ---------------------------------------------------------------------------
template <typename T, int VEC> struct Vec;
template <> struct Vec<__nv_bfloat16, 8> {
  uint4 u;
  __device__ float get(int i) const {
    const __nv_bfloat162 h = reinterpret_cast<const __nv_bfloat162*>(&u)[i >> 1];
    return (i & 1) ? __high2float(h) : __low2float(h);
  }
  __device__ void set(int i, float x) {
    __nv_bfloat16* b = reinterpret_cast<__nv_bfloat16*>(&u);
    b[i] = __float2bfloat16_rn(x);
  }
};
template <> struct Vec<float, 4> {
  float4 u;
  __device__ float get(int i) const { return reinterpret_cast<const float*>(&u)[i]; }
  __device__ void set(int i, float x) { reinterpret_cast<float*>(&u)[i] = x; }
};
template <> struct Vec<float, 1> {
  float u;
  __device__ float get(int) const { return u; }
  __device__ void set(int, float x) { u = x; }
};

template <typename T, int VEC, int S, int MAXV, int ROWS>
__global__ void __launch_bounds__(256) k_qk_prologue(const T* __restrict__ q, T* __restrict__ qh,
                                                     int64_t q_rows, const T* __restrict__ k,
                                                     T* __restrict__ kh, int64_t k_rows, int d,
                                                     T* __restrict__ kh_lo) {
  griddep_launch();
  griddep_wait();
  // Each group of S threads handles ROWS rows, all loads issued before any
  // reduction, so every thread keeps ROWS * MAXV 16-byte loads in flight.
  using V = Vec<T, VEC>;
  using U = decltype(V::u);
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t group = gtid / S;
  const int sl = static_cast<int>(gtid % S);
  const int64_t total = q_rows + k_rows;
  const int nv = d / VEC;
  V in[ROWS][MAXV];
#pragma unroll
  for (int rr = 0; rr < ROWS; ++rr) {
    const int64_t row = group * ROWS + rr;
    const T* src = row < q_rows ? q + row * d : k + (row - q_rows) * d;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = sl + i * S;
      if (row < total && v < nv) in[rr][i].u = reinterpret_cast<const U*>(src)[v];
    }
  }
#pragma unroll
  for (int rr = 0; rr < ROWS; ++rr) {
    const int64_t row = group * ROWS + rr;
    const bool active = row < total;
    float y[MAXV][VEC];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = sl + i * S;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        float t = 0.f;
        if (active && v < nv) {
          const float a = in[rr][i].get(e);
          // Split-bf16 keys (kh_lo) need the accurate sigmoid; plain bf16
          // rounding hides the one-op approximation.
          t = (kh_lo || VEC != 8) ? __fdividef(a, 1.0f + __expf(-a)) : a * sigmoid_fast(a);
        }
        y[i][e] = t;
        ss += t * t;
      }
    }
#pragma unroll
    for (int o = S / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (!active) continue;
    const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
    const bool is_q = row < q_rows;
    T* dst = is_q ? qh + row * d : kh + (row - q_rows) * d;
    T* dst_lo = (kh_lo && !is_q) ? kh_lo + (row - q_rows) * d : nullptr;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = sl + i * S;
      if (v < nv) {
        V hi, lo;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float val = y[i][e] * inv;
          hi.set(e, val);
          lo.set(e, val - hi.get(e));
        }
        reinterpret_cast<U*>(dst)[v] = hi.u;
        if (dst_lo) reinterpret_cast<U*>(dst_lo)[v] = lo.u;
      }
    }
  }
}

// bf16 prologue.  Rows of d bf16 values, 8 per 16-byte vector: S lanes per
// row (the power of two >= d / 8, at most 32), MAXV vectors per lane, ROWS
// rows per lane group with every load issued before any arithmetic.  The bf16
// pairs are widened with two integer ops, and silu(a) = h + h * tanh(h) with
// h = a / 2 (the logistic written through tanh) costs one hardware tanh and
// two FP ops per element.  SPLIT also writes the lo part x - bf16(x) of each
// key value (split-bf16 operands) and then uses the exact-form logistic for
// every row, since the lo part would carry the tanh approximation's error.
template <int S, int MAXV, int ROWS, bool SPLIT>
__global__ void __launch_bounds__(256) k_qk_prologue_bf16(const __nv_bfloat16* __restrict__ q,
                                                          __nv_bfloat16* __restrict__ qh,
                                                          int64_t q_rows,
                                                          const __nv_bfloat16* __restrict__ k,
                                                          __nv_bfloat16* __restrict__ kh,
                                                          int64_t k_rows, int d,
                                                          __nv_bfloat16* __restrict__ kh_lo) {
  griddep_launch();
  griddep_wait();
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t group = gtid / S;
  const int sl = static_cast<int>(gtid % S);
  const int64_t total = q_rows + k_rows;
  const int nv = d >> 3;
  uint4 in[ROWS][MAXV];
#pragma unroll
  for (int rr = 0; rr < ROWS; ++rr) {
    const int64_t row = group * ROWS + rr;
    const __nv_bfloat16* src = row < q_rows ? q + row * d : k + (row - q_rows) * d;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = sl + i * S;
      in[rr][i] = (row < total && v < nv) ? reinterpret_cast<const uint4*>(src)[v]
                                          : make_uint4(0u, 0u, 0u, 0u);   // silu(0) = 0
    }
  }
#pragma unroll
  for (int rr = 0; rr < ROWS; ++rr) {
    const int64_t row = group * ROWS + rr;
    float y[MAXV][8];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const uint32_t w[4] = {in[rr][i].x, in[rr][i].y, in[rr][i].z, in[rr][i].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float a = __uint_as_float((e & 1) ? (w[e >> 1] & 0xffff0000u) : (w[e >> 1] << 16));
        float t;
        if (SPLIT) {
          t = __fdividef(a, 1.0f + __expf(-a));
        } else {
          const float h = 0.5f * a;
          t = fmaf(h, tanh_approx(h), h);
        }
        y[i][e] = t;
        ss = fmaf(t, t, ss);
      }
    }
#pragma unroll
    for (int o = S / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (row >= total) continue;
    const float inv = ss > 0.f ? rsqrtf(ss) : 0.f;
    const bool is_q = row < q_rows;
    __nv_bfloat16* dst = is_q ? qh + row * d : kh + (row - q_rows) * d;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = sl + i * S;
      if (v >= nv) continue;
      uint32_t hw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) hw[e] = pack_bf16x2(y[i][2 * e] * inv, y[i][2 * e + 1] * inv);
      reinterpret_cast<uint4*>(dst)[v] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      if (SPLIT && !is_q) {
        uint32_t lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = y[i][2 * e] * inv, x1 = y[i][2 * e + 1] * inv;
          lw[e] = pack_bf16x2(x0 - __uint_as_float(hw[e] << 16), x1 - __uint_as_float(hw[e] & 0xffff0000u));
        }
        reinterpret_cast<uint4*>(kh_lo + (row - q_rows) * d)[v] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
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
// State set-up: Wm[j][bh] = the caller's initial weights (state h of the H
// shared ones, or state bh), plus the bf16 shadow (and its split lo part);
// momentum = the caller's m1/m2/m3 ([BH] states each) or zero, held negated
// like the rule's M' = -M (an exact sign flip).  Grid-stride over
// 3 * BH * dh * d elements.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_init_state(const float* __restrict__ w1,
                                                    const float* __restrict__ w2,
                                                    const float* __restrict__ w3, int H,
                                                    int w_shared, int BH, int d, int dh,
                                                    float* __restrict__ Wm,
                                                    __nv_bfloat16* __restrict__ Ws,
                                                    __nv_bfloat16* __restrict__ Ws_lo,
                                                    float* __restrict__ Mm,
                                                    const float* __restrict__ m1,
                                                    const float* __restrict__ m2,
                                                    const float* __restrict__ m3) {
  griddep_launch();
  griddep_wait();
  const int64_t plane = static_cast<int64_t>(dh) * d;
  const int64_t total = 3 * BH * plane;
  const int64_t per = BH * plane;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  if (plane % 4 == 0) {  // 16-byte steps
    for (int64_t o = 4 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x); o < total;
         o += 4 * stride) {
      const int64_t jb = o / plane, e = o % plane;
      const int j = static_cast<int>(jb / BH), bh = static_cast<int>(jb % BH);
      const int src_h = w_shared ? bh % H : bh;
      const float* src = j == 0 ? w1 : (j == 1 ? w2 : w3);
      const float4 x = *reinterpret_cast<const float4*>(src + static_cast<int64_t>(src_h) * plane + e);
      *reinterpret_cast<float4*>(Wm + o) = x;
      if (Ws) {
        store_shadow(Ws, Ws_lo, o, x.x);
        store_shadow(Ws, Ws_lo, o + 1, x.y);
        store_shadow(Ws, Ws_lo, o + 2, x.z);
        store_shadow(Ws, Ws_lo, o + 3, x.w);
      }
      if (Mm) {
        const float* m = j == 0 ? m1 : (j == 1 ? m2 : m3);
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (m) {
          x = *reinterpret_cast<const float4*>(m + (o - j * per));
          x = make_float4(-x.x, -x.y, -x.z, -x.w);
        }
        *reinterpret_cast<float4*>(Mm + o) = x;
      }
    }
    return;
  }
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < total; o += stride) {
    const int64_t jb = o / plane, e = o % plane;
    const int j = static_cast<int>(jb / BH), bh = static_cast<int>(jb % BH);
    const int src_h = w_shared ? bh % H : bh;
    const float* src = j == 0 ? w1 : (j == 1 ? w2 : w3);
    const float x = src[static_cast<int64_t>(src_h) * plane + e];
    Wm[o] = x;
    store_shadow(Ws, Ws_lo, o, x);
    if (Mm) {
      const float* m = j == 0 ? m1 : (j == 1 ? m2 : m3);
      Mm[o] = m ? -m[o - j * per] : 0.f;
    }
  }
}

// Write-back of the final state into w1_out, w2_out, w3_out, and of the
// final momentum M = -M' into m1o, m2o, m3o when they are given.
__global__ void __launch_bounds__(256) k_finalize_state(const float* __restrict__ Wm, int BH, int d,
                                                        int dh, float* __restrict__ w1o,
                                                        float* __restrict__ w2o,
                                                        float* __restrict__ w3o,
                                                        const float* __restrict__ Mm,
                                                        float* __restrict__ m1o,
                                                        float* __restrict__ m2o,
                                                        float* __restrict__ m3o) {
  griddep_launch();
  griddep_wait();
  const int64_t plane = static_cast<int64_t>(dh) * d;
  const int64_t per = BH * plane;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const bool mom = Mm && m1o;
  if (per % 4 == 0) {
    for (int64_t o = 4 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x); o < 3 * per;
         o += 4 * stride) {
      const int j = static_cast<int>(o / per);
      float* dst = j == 0 ? w1o : (j == 1 ? w2o : w3o);
      *reinterpret_cast<float4*>(dst + (o - j * per)) = *reinterpret_cast<const float4*>(Wm + o);
      if (mom) {
        float* mdst = j == 0 ? m1o : (j == 1 ? m2o : m3o);
        const float4 x = *reinterpret_cast<const float4*>(Mm + o);
        *reinterpret_cast<float4*>(mdst + (o - j * per)) = make_float4(-x.x, -x.y, -x.z, -x.w);
      }
    }
    return;
  }
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; o < 3 * per; o += stride) {
    const int j = static_cast<int>(o / per);
    float* dst = j == 0 ? w1o : (j == 1 ? w2o : w3o);
    dst[o - j * per] = Wm[o];
    if (mom) (j == 0 ? m1o : (j == 1 ? m2o : m3o))[o - j * per] = -Mm[o];
  }
}

// beta_bar[bh][c] = mean of beta over chunk c's tokens (one warp per entry).
// With `sums` set the kernel writes the sum instead, and the token count at
// beta_bar[BH * nch + w]: context-parallel ranks each hold a share of every
// chunk, so their sums and counts are added over the ranks first and
// k_beta_div forms the mean.
__global__ void __launch_bounds__(256) k_beta_mean(const float* __restrict__ beta, int BH, int64_t T,
                                                   int64_t chunk, int nch,
                                                   float* __restrict__ beta_bar, int sums) {
  griddep_launch();
  griddep_wait();
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<int64_t>(BH) * nch) return;
  const int bh = static_cast<int>(w / nch), c = static_cast<int>(w % nch);
  const int64_t t0 = c * chunk, t1 = (t0 + chunk < T) ? t0 + chunk : T;
  const float* b = beta + static_cast<int64_t>(bh) * T;
  float s = 0.f;
  for (int64_t t = t0 + lane; t < t1; t += 32) s += b[t];
  s = warp_sum(s);
  if (lane != 0) return;
  if (sums) {
    beta_bar[w] = s;
    beta_bar[static_cast<int64_t>(BH) * nch + w] = static_cast<float>(t1 - t0);
  } else {
    beta_bar[w] = s / static_cast<float>(t1 - t0);
  }
}

// beta_bar[i] /= beta_bar[n + i]: the mean of beta over a chunk whose sum and
// token count were added over the context-parallel ranks.
__global__ void __launch_bounds__(256) k_beta_div(float* __restrict__ beta_bar, int64_t n) {
  griddep_launch();
  griddep_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) beta_bar[i] = beta_bar[i] / beta_bar[n + i];
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
// One warp per row: BH*dh rows of W1 (length d), BH*d rows of W2 (length
// dh), BH*dh rows of W3 (length d), in plane order.
// ---------------------------------------------------------------------------
struct RuleParams {
  float* Wm;
  __nv_bfloat16* Ws;      // bf16 shadow or null
  __nv_bfloat16* Ws_lo;   // split-bf16 lo part of the shadow or null
  const float* S;         // [splits][3][BH][plane]
  int splits;
  int64_t split_stride;   // elements between partial planes
  float* Mm;              // momentum (rule 1) or null
  const float* beta_bar;  // [BH][nch]
  int nch, chunk_idx;
  int rule;
  int BH, dh, d;
  float* nrm_out;         // or null: per row, the norm of W - U before the renorm
};

struct RuleRow {
  int j, bh, len;
  int64_t base;
};

__device__ __forceinline__ bool rule_row(const RuleParams& p, int64_t row, RuleRow& r) {
  const int64_t r13 = static_cast<int64_t>(p.BH) * p.dh, r2 = static_cast<int64_t>(p.BH) * p.d;
  if (row >= 2 * r13 + r2) return false;
  const int64_t plane = static_cast<int64_t>(p.dh) * p.d;
  int64_t rr;
  if (row < r13) { r.j = 0; rr = row; }
  else if (row < r13 + r2) { r.j = 1; rr = row - r13; }
  else { r.j = 2; rr = row - r13 - r2; }
  r.len = r.j == 1 ? p.dh : p.d;
  r.bh = static_cast<int>(rr / (r.j == 1 ? p.d : p.dh));
  r.base = static_cast<int64_t>(r.j) * p.BH * plane + rr * r.len;
  return true;
}

// Generic form (any row length): two passes over the row in global memory.
__global__ void __launch_bounds__(256) k_rule_renorm(const RuleParams p) {
  griddep_launch();
  griddep_wait();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  RuleRow r;
  if (!rule_row(p, row, r)) return;
  const float bb = p.rule == 1 ? p.beta_bar[r.bh * p.nch + p.chunk_idx] : 0.f;
  float on = 0.f, nn = 0.f;
  for (int c = lane; c < r.len; c += 32) {
    const int64_t o = r.base + c;
    float s = 0.f;
    for (int i = 0; i < p.splits; ++i) s += p.S[i * p.split_stride + o];
    if (p.rule == 1) {
      s = bb * p.Mm[o] + s;
      p.Mm[o] = s;
    }
    const float w = p.Wm[o];
    const float wn = w + s;
    p.Wm[o] = wn;
    on += w * w;
    nn += wn * wn;
  }
  on = warp_sum(on);
  nn = warp_sum(nn);
  const float sc = nn > 0.f ? sqrtf(on) / sqrtf(nn) : 0.f;
  if (p.nrm_out && lane == 0) p.nrm_out[row] = sqrtf(nn);
  for (int c = lane; c < r.len; c += 32) {
    const int64_t o = r.base + c;
    const float w = p.Wm[o] * sc;
    p.Wm[o] = w;
    store_shadow(p.Ws, p.Ws_lo, o, w);
  }
}

// Rows whose length is a multiple of 4 and at most 128 * MAXV: one pass,
// 16-byte accesses, the updated rows kept in registers until they are
// scaled.  Each warp takes ROWS consecutive rows.  Every load of a row (all
// gradient splits, the momentum buffer, the master weights) is issued before
// the first arithmetic or store, so the row costs one memory latency rather
// than one per 16-byte chunk.
template <int MAXV, int ROWS>
__global__ void __launch_bounds__(256) k_rule_renorm_v4(const RuleParams p) {
  griddep_launch();
  griddep_wait();
  const int64_t row0 = ((static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5) * ROWS;
  const int lane = threadIdx.x & 31;
  RuleRow r[ROWS];
  bool have[ROWS];
  float4 wn[ROWS][MAXV];
  float on[ROWS], nn[ROWS];
  const float* __restrict__ S = p.S;
  const float* __restrict__ W = p.Wm;
  const bool mom = p.rule == 1;
#pragma unroll
  for (int k = 0; k < ROWS; ++k) {
    have[k] = rule_row(p, row0 + k, r[k]);
    on[k] = 0.f;
    nn[k] = 0.f;
    if (!have[k]) continue;
    const int nv = r[k].len >> 2;
    float4 g[MAXV], w[MAXV], m[MAXV];
    // loads
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = lane + 32 * i;
      g[i] = w[i] = m[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (v < nv) {
        const int64_t o = r[k].base + 4 * v;
        g[i] = __ldcs(reinterpret_cast<const float4*>(S + o));
        w[i] = *reinterpret_cast<const float4*>(W + o);
        if (mom) m[i] = *reinterpret_cast<const float4*>(p.Mm + o);
      }
    }
    for (int t = 1; t < p.splits; ++t) {
#pragma unroll
      for (int i = 0; i < MAXV; ++i) {
        const int v = lane + 32 * i;
        if (v < nv) {
          const float4 x = __ldcs(reinterpret_cast<const float4*>(S + t * p.split_stride + r[k].base + 4 * v));
          g[i].x += x.x; g[i].y += x.y; g[i].z += x.z; g[i].w += x.w;
        }
      }
    }
    // update (momentum: S <- beta_bar S + G) and the new row
    const float bb = mom ? p.beta_bar[r[k].bh * p.nch + p.chunk_idx] : 0.f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = lane + 32 * i;
      if (v < nv) {
        float4 s4 = g[i];
        if (mom) {
          s4.x += bb * m[i].x; s4.y += bb * m[i].y; s4.z += bb * m[i].z; s4.w += bb * m[i].w;
          *reinterpret_cast<float4*>(p.Mm + r[k].base + 4 * v) = s4;
        }
        on[k] += w[i].x * w[i].x + w[i].y * w[i].y + w[i].z * w[i].z + w[i].w * w[i].w;
        wn[k][i] = make_float4(w[i].x + s4.x, w[i].y + s4.y, w[i].z + s4.z, w[i].w + s4.w);
        nn[k] += wn[k][i].x * wn[k][i].x + wn[k][i].y * wn[k][i].y + wn[k][i].z * wn[k][i].z +
                 wn[k][i].w * wn[k][i].w;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < ROWS; ++k) {
    on[k] = warp_sum(on[k]);
    nn[k] = warp_sum(nn[k]);
  }
#pragma unroll
  for (int k = 0; k < ROWS; ++k) {
    if (!have[k]) continue;
    const float sc = nn[k] > 0.f ? sqrtf(on[k]) / sqrtf(nn[k]) : 0.f;
    const int nv = r[k].len >> 2;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = lane + 32 * i;
      if (v < nv) {
        const int64_t o = r[k].base + 4 * v;
        const float4 w = make_float4(wn[k][i].x * sc, wn[k][i].y * sc, wn[k][i].z * sc, wn[k][i].w * sc);
        *reinterpret_cast<float4*>(p.Wm + o) = w;
        if (p.Ws) {
          uint2 hi;
          hi.x = pack_bf16x2(w.x, w.y);
          hi.y = pack_bf16x2(w.z, w.w);
          *reinterpret_cast<uint2*>(p.Ws + o) = hi;
          if (p.Ws_lo) {
            const __nv_bfloat162 h0 = *reinterpret_cast<const __nv_bfloat162*>(&hi.x);
            const __nv_bfloat162 h1 = *reinterpret_cast<const __nv_bfloat162*>(&hi.y);
            uint2 lo;
            lo.x = pack_bf16x2(w.x - __low2float(h0), w.y - __high2float(h0));
            lo.y = pack_bf16x2(w.z - __low2float(h1), w.w - __high2float(h1));
            *reinterpret_cast<uint2*>(p.Ws_lo + o) = lo;
          }
        }
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
  griddep_launch();
  griddep_wait();
  __shared__ float red[9];
  const int item = blockIdx.y;
  const int64_t base = static_cast<int64_t>(item) * plane;
  float ss = 0.f;
  if ((plane & 3) == 0 && (split_stride & 3) == 0) {
    // 16-byte steps, four vectors in flight per thread
    const int64_t nv = plane >> 2, sv = split_stride >> 2;
    const int64_t per = (nv + gridDim.x - 1) / gridDim.x;
    const int64_t v0 = blockIdx.x * per, v1 = (v0 + per < nv) ? v0 + per : nv;
    const float4* Sv = reinterpret_cast<const float4*>(S + base);
    float4* Yv = reinterpret_cast<float4*>(Y + base);
    for (int64_t v = v0 + threadIdx.x; v < v1; v += 4 * 256) {
      float4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t vv = v + u * 256;
        x[u] = vv < v1 ? Sv[vv] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      for (int i = 1; i < splits; ++i) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t vv = v + u * 256;
          if (vv < v1) {
            const float4 y = Sv[i * sv + vv];
            x[u].x += y.x; x[u].y += y.y; x[u].z += y.z; x[u].w += y.w;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t vv = v + u * 256;
        if (vv < v1) {
          Yv[vv] = x[u];
          ss += x[u].x * x[u].x + x[u].y * x[u].y + x[u].z * x[u].z + x[u].w * x[u].w;
        }
      }
    }
  } else {
    const int64_t per = (plane + gridDim.x - 1) / gridDim.x;
    const int64_t e0 = blockIdx.x * per, e1 = (e0 + per < plane) ? e0 + per : plane;
    for (int64_t e = e0 + threadIdx.x; e < e1; e += 256) {
      float s = 0.f;
      for (int i = 0; i < splits; ++i) s += S[i * split_stride + base + e];
      Y[base + e] = s;
      ss += s * s;
    }
  }
  ss = block_sum_256(ss, red);
  if (threadIdx.x == 0) part[static_cast<int64_t>(item) * gridDim.x + blockIdx.x] = ss;
}

__global__ void __launch_bounds__(256) k_ns_scale(float* __restrict__ Y,
                                                  __nv_bfloat16* __restrict__ Yb,
                                                  __nv_bfloat16* __restrict__ Yb_lo, int64_t plane,
                                                  const float* __restrict__ part, int nblk,
                                                  float eps) {
  griddep_launch();
  griddep_wait();
  __shared__ float sc;
  const int item = blockIdx.y;
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int i = 0; i < nblk; ++i) s += part[static_cast<int64_t>(item) * nblk + i];
    sc = 1.0f / (sqrtf(s) + eps);
  }
  __syncthreads();
  const float c = sc;
  const int64_t base = static_cast<int64_t>(item) * plane;
  if ((plane & 3) == 0) {
    // 16-byte steps, four vectors in flight per thread; the bf16 copies as 8-byte stores
    const int64_t nv = plane >> 2;
    const int64_t per = (nv + gridDim.x - 1) / gridDim.x;
    const int64_t v0 = blockIdx.x * per, v1 = (v0 + per < nv) ? v0 + per : nv;
    float4* Yv = reinterpret_cast<float4*>(Y + base);
    for (int64_t v = v0 + threadIdx.x; v < v1; v += 4 * 256) {
      float4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t vv = v + u * 256;
        x[u] = vv < v1 ? Yv[vv] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t vv = v + u * 256;
        if (vv >= v1) continue;
        const float4 y = make_float4(x[u].x * c, x[u].y * c, x[u].z * c, x[u].w * c);
        Yv[vv] = y;
        if (Yb) {
          uint2 hi;
          hi.x = pack_bf16x2(y.x, y.y);
          hi.y = pack_bf16x2(y.z, y.w);
          *reinterpret_cast<uint2*>(Yb + base + 4 * vv) = hi;
          if (Yb_lo) {
            const __nv_bfloat162 h0 = *reinterpret_cast<const __nv_bfloat162*>(&hi.x);
            const __nv_bfloat162 h1 = *reinterpret_cast<const __nv_bfloat162*>(&hi.y);
            uint2 lo;
            lo.x = pack_bf16x2(y.x - __low2float(h0), y.y - __high2float(h0));
            lo.y = pack_bf16x2(y.z - __low2float(h1), y.w - __high2float(h1));
            *reinterpret_cast<uint2*>(Yb_lo + base + 4 * vv) = lo;
          }
        }
      }
    }
  } else {
    const int64_t per = (plane + gridDim.x - 1) / gridDim.x;
    const int64_t e0 = blockIdx.x * per, e1 = (e0 + per < plane) ? e0 + per : plane;
    for (int64_t e = e0 + threadIdx.x; e < e1; e += 256) {
      const float y = Y[base + e] * c;
      Y[base + e] = y;
      store_shadow(Yb, Yb_lo, base + e, y);
    }
  }
}

}  // namespace lact
