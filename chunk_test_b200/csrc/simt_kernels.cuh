// simt_kernels.cuh -- the fp32 path (CUDA-core FFMA).  fp32 tensor-core
// formats (tf32) round operands to 10 mantissa bits, too coarse for a 1e-4
// relative match, so this path keeps every operand in fp32.
#pragma once

#include "elem_kernels.cuh"

namespace lact {

// Batched strided GEMM: C[item][m][n] = alpha * sum_k A(m,k) B(n,k) + beta * Cin,
//   A(m,k) = Abase[(item % za_mod) * a_item + m * a_m + k * a_k]
//   B(n,k) = Bbase[((item % zb_mod) + zb_add) * b_item + n * b_n + k * b_k]
// where Abase is A2 when item / za_mod == alt_a (else A), Bbase likewise.
// Output at item * item_stride + m * ld + n for m < M, n < N.
struct SimtGemmParams {
  const float* A;
  const float* A2;
  int64_t a_item, a_m, a_k;
  int za_mod, alt_a;
  const float* B;
  const float* B2;
  int64_t b_item, b_n, b_k;
  int zb_mod, zb_add, alt_b;
  int M, N, K;
  float alpha, beta;
  const float* cin;
  float* outf;
  int64_t item_stride, ld;
  int tr_group, tr_mod;   // items with item / tr_mod == tr_group store C^T
  int64_t ld_t;           //   at n * ld_t + m
  const float* row_scale; // or null: row m of item z scaled by row_scale[z * rs_item + m]
  int64_t rs_item;
};

__global__ void __launch_bounds__(256) k_simt_gemm(const SimtGemmParams p) {
  griddep_launch();
  griddep_wait();
  __shared__ float As[16][68], Bs[16][68];
  const int item = blockIdx.z;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const float* A = (p.alt_a >= 0 && item / p.za_mod == p.alt_a) ? p.A2 : p.A;
  A += static_cast<int64_t>(item % p.za_mod) * p.a_item;
  const float* B = (p.alt_b >= 0 && item / p.zb_mod == p.alt_b) ? p.B2 : p.B;
  B += static_cast<int64_t>((item % p.zb_mod) + p.zb_add) * p.b_item;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < p.K; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      // Walk the tile along whichever of (row, k) is contiguous in memory.
      int kk, mm;
      if (p.a_k == 1) { kk = i & 15; mm = i >> 4; } else { kk = i >> 6; mm = i & 63; }
      const int m = m0 + mm, k = k0 + kk;
      As[kk][mm] = (m < p.M && k < p.K) ? A[m * p.a_m + k * p.a_k] : 0.f;
      int kb, nn;
      if (p.b_k == 1) { kb = i & 15; nn = i >> 4; } else { kb = i >> 6; nn = i & 63; }
      const int n = n0 + nn, kq = k0 + kb;
      Bs[kb][nn] = (n < p.N && kq < p.K) ? B[n * p.b_n + kq * p.b_k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= p.N) continue;
      const int64_t o = static_cast<int64_t>(item) * p.item_stride + static_cast<int64_t>(m) * p.ld + n;
      float v = p.alpha * acc[i][j];
      if (p.cin) v += p.beta * p.cin[o];
      if (p.row_scale) v *= p.row_scale[static_cast<int64_t>(item) * p.rs_item + m];
      if (p.tr_group >= 0 && item / p.tr_mod == p.tr_group)
        p.outf[static_cast<int64_t>(item) * p.item_stride + static_cast<int64_t>(n) * p.ld_t + m] = v;
      else
        p.outf[o] = v;
    }
  }
}

// Fast-net elementwise step on fp32 pre-activations Z [3][BH][rows][dh]
// (plane 0: X W1^T, plane 1: V W2, plane 2: X W3^T).
//   query chunk: Hq = silu(z1) z3
//   key chunk:   E1 = lr1 u z3 silu'(z1), Eh = lr2 silu(z1) z3, E3 = lr3 u silu(z1)
// (same algebra as the tensor-core epilogue; rows >= rows_valid -> 0).
__global__ void __launch_bounds__(256) k_fwd_elem_f32(const float* __restrict__ Z, int BH,
                                                      int64_t rows, int dh, int rows_valid,
                                                      int kmode, const float* __restrict__ lr,
                                                      int64_t T, int64_t row0,
                                                      float* __restrict__ out) {
  griddep_launch();
  griddep_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t plane = static_cast<int64_t>(BH) * rows * dh;
  if (i >= plane) return;
  const int64_t r = (i / dh) % rows;
  const int64_t bh = i / (rows * dh);
  const float z1 = Z[i], z3 = Z[2 * plane + i];
  const float s = 1.0f / (1.0f + __expf(-z1));
  const float sa = z1 * s;
  if (!kmode) {
    out[i] = sa * z3;
    return;
  }
  float e1 = 0.f, eh = 0.f, e3 = 0.f;
  if (r < rows_valid) {
    const float u = Z[plane + i];
    const float* l = lr + (bh * T + row0 + r) * 3;
    e1 = l[0] * u * z3 * (s * (1.0f + z1 * (1.0f - s)));
    eh = l[1] * sa * z3;
    e3 = l[2] * u * sa;
  }
  out[i] = e1;
  out[plane + i] = eh;
  out[2 * plane + i] = e3;
}

}  // namespace lact
