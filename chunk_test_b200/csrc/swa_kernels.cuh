// swa_kernels.cuh -- sliding-window attention of the LaCT block
// ("LaCT架构核心思想解析" §1.1): q' = q * q_scale + q_offset and
// k' = k * k_scale + k_offset per head and channel, then for every token t
// softmax(q'_t . k'_j / sqrt(d)) over the w most recent tokens j
// (t - w < j <= t) weights the values v_j.
//
// Layout of the per-query-block windows: keys and values are copied into
// per-head buffers with w zero rows in front, Kp/Vp [BH][w + T][d], so the
// keys a block of 128 queries starting at token m*128 can see lie in the
// padded rows [m*128, m*128 + w + 128).  Those windows are overlapping
// strided views of Kp/Vp, read by the tensor-core GEMMs.
#pragma once

#include "elem_kernels.cuh"

namespace lact {

// q' -> Qp [BH][T][d]; k' -> Kp rows w.., v -> Vp rows w..; the w padding
// rows of each head and `tail` rows after the last head are zeroed.
// Grid-stride over 16-byte vectors (8 bf16; d is a multiple of 64).
__global__ void __launch_bounds__(256) k_swa_prologue(const __nv_bfloat16* __restrict__ q,
                                                      const __nv_bfloat16* __restrict__ k,
                                                      const __nv_bfloat16* __restrict__ v,
                                                      const float* __restrict__ qs,
                                                      const float* __restrict__ qo,
                                                      const float* __restrict__ ks,
                                                      const float* __restrict__ ko, int H, int BH,
                                                      int64_t T, int d, int64_t window, int64_t tail,
                                                      __nv_bfloat16* __restrict__ Qp,
                                                      __nv_bfloat16* __restrict__ Kp,
                                                      __nv_bfloat16* __restrict__ Vp) {
  griddep_launch();
  griddep_wait();
  const int nv = d >> 3;
  const int64_t Tp = window + T;
  const int64_t n_main = static_cast<int64_t>(BH) * T * nv;
  const int64_t n_pad = (static_cast<int64_t>(BH) * window + tail) * nv;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_main + n_pad; i += stride) {
    if (i >= n_main) {                      // zero padding rows
      const int64_t j = i - n_main;
      const int64_t row = j / nv, c = (j % nv) * 8;
      int64_t dst;
      if (row < static_cast<int64_t>(BH) * window) dst = (row / window) * Tp + row % window;
      else dst = static_cast<int64_t>(BH) * Tp + (row - static_cast<int64_t>(BH) * window);
      *reinterpret_cast<uint4*>(Kp + dst * d + c) = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(Vp + dst * d + c) = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const int64_t row = i / nv;             // bh * T + t
    const int c = static_cast<int>(i % nv) * 8;
    const int64_t bh = row / T, t = row % T;
    const int h = static_cast<int>(bh % H);
    const uint4 qv = *reinterpret_cast<const uint4*>(q + row * d + c);
    const uint4 kv = *reinterpret_cast<const uint4*>(k + row * d + c);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w}, kw[4] = {kv.x, kv.y, kv.z, kv.w};
    uint32_t qo_w[4], ko_w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int ch = c + 2 * e;
      const float q0 = __uint_as_float(qw[e] << 16), q1 = __uint_as_float(qw[e] & 0xffff0000u);
      const float k0 = __uint_as_float(kw[e] << 16), k1 = __uint_as_float(kw[e] & 0xffff0000u);
      const float* s1 = qs + h * d + ch;
      const float* o1 = qo + h * d + ch;
      const float* s2 = ks + h * d + ch;
      const float* o2 = ko + h * d + ch;
      qo_w[e] = pack_bf16x2(fmaf(q0, s1[0], o1[0]), fmaf(q1, s1[1], o1[1]));
      ko_w[e] = pack_bf16x2(fmaf(k0, s2[0], o2[0]), fmaf(k1, s2[1], o2[1]));
    }
    const int64_t prow = bh * Tp + window + t;
    *reinterpret_cast<uint4*>(Qp + row * d + c) = make_uint4(qo_w[0], qo_w[1], qo_w[2], qo_w[3]);
    *reinterpret_cast<uint4*>(Kp + prow * d + c) = make_uint4(ko_w[0], ko_w[1], ko_w[2], ko_w[3]);
    *reinterpret_cast<uint4*>(Vp + prow * d + c) = *reinterpret_cast<const uint4*>(v + row * d + c);
  }
}

// Query prologue of the fused path: Qt = (q * q_scale + q_offset) * k_scale
// per head and channel, so that Qt . k = q' . k' - q' . k_offset.  The last
// term is the same for every key of a query and the softmax removes it, so
// the keys and values are read as given.  Grid-stride over 16-byte vectors.
__global__ void __launch_bounds__(256) k_swa_prologue_q(const __nv_bfloat16* __restrict__ q,
                                                        const float* __restrict__ qs,
                                                        const float* __restrict__ qo,
                                                        const float* __restrict__ ks, int H, int64_t T,
                                                        int d, int64_t n, __nv_bfloat16* __restrict__ Qt) {
  griddep_launch();
  griddep_wait();
  const int nv = d >> 3;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t row = i / nv;             // bh * T + t
    const int c = static_cast<int>(i % nv) * 8;
    const int h = static_cast<int>((row / T) % H);
    const uint4 qv = *reinterpret_cast<const uint4*>(q + row * d + c);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
    const float4* s4 = reinterpret_cast<const float4*>(qs + h * d + c);
    const float4* o4 = reinterpret_cast<const float4*>(qo + h * d + c);
    const float4* k4 = reinterpret_cast<const float4*>(ks + h * d + c);
    const float4 sa = s4[0], sb = s4[1], oa = o4[0], ob = o4[1], ka = k4[0], kb = k4[1];
    const float sc[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    const float of[8] = {oa.x, oa.y, oa.z, oa.w, ob.x, ob.y, ob.z, ob.w};
    const float kc[8] = {ka.x, ka.y, ka.z, ka.w, kb.x, kb.y, kb.z, kb.w};
    uint32_t ow[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float q0 = __uint_as_float(qw[e] << 16), q1 = __uint_as_float(qw[e] & 0xffff0000u);
      ow[e] = pack_bf16x2(fmaf(q0, sc[2 * e], of[2 * e]) * kc[2 * e],
                          fmaf(q1, sc[2 * e + 1], of[2 * e + 1]) * kc[2 * e + 1]);
    }
    *reinterpret_cast<uint4*>(Qt + row * d + c) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
}

// Masked softmax of the window scores, one warp per query row.  S and P are
// [BH * nb][128][Lw] (Lw = w + 128, a multiple of 128): row r of block z
// (query t = m*128 + r, m = z % nb) sees padded window rows p with
// r + 1 <= p <= r + w (the keys t - w < j <= t) and p >= w - m*128 (j >= 0).
// Two passes over S: the running max and sum, then P = exp(s - max) / sum in
// bf16 (zeros outside the window).  scale = 1 / sqrt(d).
__global__ void __launch_bounds__(256) k_swa_softmax(const float* __restrict__ S, int64_t rows, int nb,
                                                     int Lw, int64_t window, float scale,
                                                     __nv_bfloat16* __restrict__ P) {
  griddep_launch();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; w < rows;
       w += nwarps) {
    const int64_t z = w >> 7;
    const int r = static_cast<int>(w & 127);
    const int64_t m = z % nb;
    const int64_t lo0 = window - m * 128;
    const int64_t lo = lo0 > r + 1 ? lo0 : r + 1, hi = r + window;
    const float* s = S + w * Lw;
    __nv_bfloat16* p = P + w * Lw;
    float mx = -INFINITY, sum = 0.f;
    for (int c = 4 * lane; c < Lw; c += 128) {
      const float4 x = *reinterpret_cast<const float4*>(s + c);
      const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (c + e < lo || c + e > hi) continue;
        const float y = xs[e] * scale;
        if (y > mx) {
          sum = sum * __expf(mx - y) + 1.0f;
          mx = y;
        } else {
          sum += __expf(y - mx);
        }
      }
    }
    // combine the lanes' (max, sum) pairs
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float om = __shfl_xor_sync(0xffffffffu, mx, o);
      const float os = __shfl_xor_sync(0xffffffffu, sum, o);
      const float nm = fmaxf(mx, om);
      sum = (mx == -INFINITY ? 0.f : sum * __expf(mx - nm)) + (om == -INFINITY ? 0.f : os * __expf(om - nm));
      mx = nm;
    }
    const float inv = 1.0f / sum;
    for (int c = 4 * lane; c < Lw; c += 128) {
      const float4 x = *reinterpret_cast<const float4*>(s + c);
      const float xs[4] = {x.x, x.y, x.z, x.w};
      float y[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        y[e] = (c + e < lo || c + e > hi) ? 0.f : __expf(xs[e] * scale - mx) * inv;
      *reinterpret_cast<uint2*>(p + c) = make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
    }
  }
}

// The same softmax with the row held in registers: NV float4 per lane
// (Lw = 128 * NV), so the scores are read once.
template <int NV>
__global__ void __launch_bounds__(256) k_swa_softmax_reg(const float* __restrict__ S, int64_t rows, int nb,
                                                         int64_t window, float scale,
                                                         __nv_bfloat16* __restrict__ P) {
  griddep_launch();
  griddep_wait();
  constexpr int Lw = 128 * NV;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; w < rows;
       w += nwarps) {
    const int64_t z = w >> 7;
    const int r = static_cast<int>(w & 127);
    const int64_t m = z % nb;
    const int64_t lo0 = window - m * 128;
    const int64_t lo = lo0 > r + 1 ? lo0 : r + 1, hi = r + window;
    const float* s = S + w * Lw;
    float4 x[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) x[i] = *reinterpret_cast<const float4*>(s + 4 * lane + 128 * i);
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = 4 * lane + 128 * i;
      const float xs[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (c + e >= lo && c + e <= hi) mx = fmaxf(mx, xs[e] * scale);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = 4 * lane + 128 * i;
      float* xs = reinterpret_cast<float*>(&x[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float y = (c + e >= lo && c + e <= hi) ? __expf(xs[e] * scale - mx) : 0.f;
        xs[e] = y;
        sum += y;
      }
    }
    sum = warp_sum(sum);
    const float inv = 1.0f / sum;
    __nv_bfloat16* p = P + w * Lw;
#pragma unroll
    for (int i = 0; i < NV; ++i)
      *reinterpret_cast<uint2*>(p + 4 * lane + 128 * i) =
          make_uint2(pack_bf16x2(x[i].x * inv, x[i].y * inv), pack_bf16x2(x[i].z * inv, x[i].w * inv));
  }
}

}  // namespace lact
