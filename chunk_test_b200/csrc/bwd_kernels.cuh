// bwd_kernels.cuh -- elementwise and row kernels of the layer's backward
// (fp32).  The contractions run on k_simt_gemm.
//
// Per (batch, head) and chunk c, with state W = W^{c-1} before the update,
// W' = W - U the updated matrices before the renorm and W^c = renorm(W'):
//   renorm:   W^c_r = n_r W'_r / m_r, n_r = |W^{c-1}_r|, m_r = |W'_r|
//   gradient: G = d/dW [-sum_i lr_i,j <f_W(k_i), v_i>]  ("大块测试时训练（LaCT）
//             技术解析" §2.1 eqs. 4-5; "LaCT：以大分块更新人工智能的临时记忆"
//             「局部注意力与非线性记忆相互补充」)
// The reverse loop carries A = dL/dW^c (and, momentum, Bm = dL/dM^c) and
// takes, for the gradient step, the directional derivative of phi = <G, Gam>
// with Gam = dL/dG.  Per token, with z1 = W1 k, z3 = W3 k, u = W2^T v,
// s = silu(z1), s' = silu'(z1), s'' = silu''(z1), p = Gam1 k, r = Gam3 k,
// q = Gam2^T v:
//   phi = -sum_i [lr1 <u z3 s', p> + lr2 <q, s z3> + lr3 <u s, r>]
// and its partials below are what k_hvp_elem writes.
#pragma once

#include "elem_kernels.cuh"

namespace lact {

__global__ void __launch_bounds__(256) k_bf16_to_f32(const __nv_bfloat16* __restrict__ x,
                                                     float* __restrict__ y, int64_t n) {
  griddep_launch();
  griddep_wait();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    y[i] = __bfloat162float(x[i]);
}

// y[r][:] = s[r] * x[r][:]  (rows of d values)
__global__ void __launch_bounds__(256) k_scale_rows(const float* __restrict__ x,
                                                    const float* __restrict__ s,
                                                    float* __restrict__ y, int64_t rows, int d) {
  griddep_launch();
  griddep_wait();
  const int64_t n = rows * d;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    y[i] = s[i / d] * x[i];
}

// out[r] = <a[r], b[r]> over d values; one warp per row.
__global__ void __launch_bounds__(256) k_rowdot(const float* __restrict__ a, const float* __restrict__ b,
                                                float* __restrict__ out, int64_t rows, int d) {
  griddep_launch();
  griddep_wait();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
  for (int c = lane; c < d; c += 32) acc += a[row * d + c] * b[row * d + c];
  acc = warp_sum(acc);
  if (lane == 0) out[row] = acc;
}

struct RenormBwdParams {
  const float* A;       // dL/dW^c            [3][BH][plane]
  float* A2;            // or null: a second part of dL/dW^c (the ranks' summed
                        // own contributions), added to A and then cleared
  const float* Wc;      // W^c (after renorm)
  const float* Wp;      // W^{c-1}
  const float* mnorm;   // |W'_r| per row (rule row order)
  float* Gam;           // out: dL/dG (fp32), or null
  __nv_bfloat16* Gam16; // out: dL/dG (bf16), or null
  float* Ap;            // out: dL/dW^{c-1}, the renorm and direct parts
  int rule;             // 0 GD, 1 momentum
  float* Bm;            // momentum: dL/dM^c in, dL/dM^{c-1} out
  const float* Mprev;   // momentum: M'^{c-1} = -M^{c-1} (the rule kernel's sign)
  const float* beta_bar;
  int nch, chunk_idx;
  float* part;          // momentum: per row <E, M^{c-1}>
  int BH, dh, d;
};

// Renorm and rule backward, one warp per row (the rows of the rule kernel).
//   u = W^c_r / n_r (= W'_r / m_r),  dot = <u, A_r>
//   D   = dL/dW'_r = (n_r / m_r) (A_r - u dot)
//   Ap  = D + dot W^{c-1}_r / n_r        (the norm n_r depends on W^{c-1})
//   GD:       Gam = -D
//   momentum: E = Bm - D, Gam = E, Bm <- beta_bar E, part_r = <E, M^{c-1}_r>
__global__ void __launch_bounds__(256) k_renorm_bwd(const RenormBwdParams p) {
  griddep_launch();
  griddep_wait();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  RuleParams rp;
  rp.BH = p.BH; rp.dh = p.dh; rp.d = p.d;
  RuleRow r;
  if (!rule_row(rp, row, r)) return;
  float nn = 0.f, wa = 0.f;
  for (int c = lane; c < r.len; c += 32) {
    const int64_t o = r.base + c;
    nn += p.Wp[o] * p.Wp[o];
    wa += p.Wc[o] * (p.A2 ? p.A[o] + p.A2[o] : p.A[o]);
  }
  nn = warp_sum(nn);
  wa = warp_sum(wa);
  const float n = sqrtf(nn), m = p.mnorm[row];
  const bool live = n > 0.f && m > 0.f;
  const float inv_n = live ? 1.0f / n : 0.f;
  const float dot = wa * inv_n;
  const float g = live ? n / m : 0.f;
  const float bb = p.rule == 1 ? p.beta_bar[r.bh * p.nch + p.chunk_idx] : 0.f;
  float pe = 0.f;
  for (int c = lane; c < r.len; c += 32) {
    const int64_t o = r.base + c;
    const float u = p.Wc[o] * inv_n;
    float a = p.A[o];
    if (p.A2) {
      a += p.A2[o];
      p.A2[o] = 0.f;
    }
    const float D = g * (a - u * dot);
    p.Ap[o] = D + dot * p.Wp[o] * inv_n;
    float gam;
    if (p.rule == 1) {
      const float E = p.Bm[o] - D;
      gam = E;
      pe -= E * p.Mprev[o];   // <E, M^{c-1}>, Mprev holding -M^{c-1}
      p.Bm[o] = bb * E;
    } else {
      gam = -D;
    }
    if (p.Gam) p.Gam[o] = gam;
    if (p.Gam16) p.Gam16[o] = __float2bfloat16_rn(gam);
  }
  if (p.rule == 1) {
    pe = warp_sum(pe);
    if (lane == 0) p.part[row] = pe;
  }
}

// Momentum: dL/dbeta_bar_c = sum over the head's rows of <E, M^{c-1}>, spread
// over the chunk's tokens (beta_bar is their mean): n local tokens, of
// count[bh] in the whole chunk (the ranks' summed counts under context
// parallelism; n when count is null).  One block per head.
__global__ void __launch_bounds__(256) k_head_dbeta(const float* __restrict__ part, int BH, int dh,
                                                    int d, int64_t T, int64_t c0, int n,
                                                    const float* __restrict__ count, int64_t count_stride,
                                                    float* __restrict__ dbeta) {
  griddep_launch();
  griddep_wait();
  __shared__ float red[256];
  const int bh = blockIdx.x;
  const int64_t r13 = static_cast<int64_t>(BH) * dh, r2 = static_cast<int64_t>(BH) * d;
  float acc = 0.f;
  for (int i = threadIdx.x; i < 2 * dh + d; i += 256) {
    int64_t row;
    if (i < dh) row = static_cast<int64_t>(bh) * dh + i;                        // W1
    else if (i < dh + d) row = r13 + static_cast<int64_t>(bh) * d + (i - dh);   // W2
    else row = r13 + r2 + static_cast<int64_t>(bh) * dh + (i - dh - d);         // W3
    acc += part[row];
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  const float per = red[0] / (count ? count[bh * count_stride] : static_cast<float>(n));
  for (int t = threadIdx.x; t < n; t += 256) dbeta[static_cast<int64_t>(bh) * T + c0 + t] = per;
}

__device__ __forceinline__ float sigm(float z) { return 1.0f / (1.0f + expf(-z)); }

// The second-order factors of one element: the partials of phi with respect
// to (z1, u, z3, p, q, r), and the element's terms of dphi/dlr.
struct HvpOut { float fz1, fu, fz3, fp, fq, fr, g1, g2, g3; };
// FAST: the sigmoid on the fast exponential and division (relative error
// about 1e-6, far below the bf16 rounding of the factors on the tensor-core
// path); otherwise the accurate expf and IEEE division of the fp32 path.
template <bool FAST = false>
__device__ __forceinline__ HvpOut hvp_factors(float z1, float u, float z3, float pp, float qq, float rr,
                                              float e1, float e2, float e3) {
  const float sg = FAST ? sigmoidf_(z1) : 1.0f / (1.0f + expf(-z1));
  const float s = z1 * sg;
  const float sp = sg * (1.0f + z1 * (1.0f - sg));
  const float spp = sg * (1.0f - sg) * (2.0f + z1 * (1.0f - 2.0f * sg));
  const float a1 = u * z3 * sp, a3 = u * s, h = s * z3;
  HvpOut o;
  o.fz1 = -(e1 * u * z3 * spp * pp + e3 * u * sp * rr + e2 * qq * z3 * sp);
  o.fu = -(e1 * z3 * sp * pp + e3 * s * rr);
  o.fz3 = -(e1 * u * sp * pp + e2 * qq * s);
  o.fp = -e1 * a1;
  o.fq = -e2 * h;
  o.fr = -e3 * a3;
  o.g1 = -a1 * pp;
  o.g2 = -qq * h;
  o.g3 = -a3 * rr;
  return o;
}

// Second-order factors of the gradient step, one warp per (head, token row).
// In: Z = (z1, u, z3), Pz = (p, q, r) as [3][BH][rows][dh] planes.  Out, in
// place: Z = (dphi/dz1, dphi/du, dphi/dz3), Pz = (dphi/dp, dphi/dq,
// dphi/dr); dlr[bh][row0 + i] = (dphi/dlr1, dphi/dlr2, dphi/dlr3).
__global__ void __launch_bounds__(256) k_hvp_elem(float* __restrict__ Z, float* __restrict__ Pz, int BH,
                                                  int64_t rows, int dh, int n,
                                                  const float* __restrict__ lr, int64_t T,
                                                  int64_t row0, float* __restrict__ dlr) {
  griddep_launch();
  griddep_wait();
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<int64_t>(BH) * n) return;
  const int64_t bh = w / n, i = w % n;
  const int64_t plane = static_cast<int64_t>(BH) * rows * dh;
  const int64_t base = (bh * rows + i) * dh;
  const float* l = lr + (bh * T + row0 + i) * 3;
  const float e1 = l[0], e2 = l[1], e3 = l[2];
  float g1 = 0.f, g2 = 0.f, g3 = 0.f;
  for (int c = lane; c < dh; c += 32) {
    const int64_t o = base + c;
    const HvpOut f = hvp_factors(Z[o], Z[plane + o], Z[2 * plane + o], Pz[o], Pz[plane + o],
                                 Pz[2 * plane + o], e1, e2, e3);
    Z[o] = f.fz1;
    Z[plane + o] = f.fu;
    Z[2 * plane + o] = f.fz3;
    Pz[o] = f.fp;
    Pz[plane + o] = f.fq;
    Pz[2 * plane + o] = f.fr;
    g1 += f.g1;
    g2 += f.g2;
    g3 += f.g3;
  }
  g1 = warp_sum(g1);
  g2 = warp_sum(g2);
  g3 = warp_sum(g3);
  if (lane == 0) {
    float* o = dlr + (bh * T + row0 + i) * 3;
    o[0] = g1;
    o[1] = g2;
    o[2] = g3;
  }
}

// bf16 copy of y = s[r] * x[r][:] (the scaled output gradient).
__global__ void __launch_bounds__(256) k_scale_rows_bf16(const __nv_bfloat16* __restrict__ x,
                                                         const float* __restrict__ s,
                                                         __nv_bfloat16* __restrict__ y, int64_t rows, int d) {
  griddep_launch();
  griddep_wait();
  const int64_t n = rows * d;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    y[i] = __float2bfloat16_rn(s[i / d] * __bfloat162float(x[i]));
}

// Apply backward, elementwise over [3][BH][rows][dh] planes:
// in (z1, g, z3) with g = dO W2 (dO already scaled), out (dz1, hq, dz3):
// dz1 = g z3 silu'(z1), dz3 = g silu(z1), hq = silu(z1) z3.
__global__ void __launch_bounds__(256) k_apply_bwd_elem(float* __restrict__ Zq, int64_t plane) {
  griddep_launch();
  griddep_wait();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < plane; i += stride) {
    const float z1 = Zq[i], g = Zq[plane + i], z3 = Zq[2 * plane + i];
    const float sg = sigm(z1);
    const float s = z1 * sg;
    Zq[i] = g * z3 * sg * (1.0f + z1 * (1.0f - sg));
    Zq[plane + i] = s * z3;
    Zq[2 * plane + i] = g * s;
  }
}

// Prologue backward, one warp per row: x^ = s / |s|, s = silu(x).
// dx = silu'(x) (dx^ - x^ <x^, dx^>) / |s|; a zero row gets zero.
__global__ void __launch_bounds__(256) k_prologue_bwd(const float* __restrict__ x,
                                                      const float* __restrict__ dxh,
                                                      float* __restrict__ dx, int64_t rows, int d) {
  griddep_launch();
  griddep_wait();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* xr = x + row * d;
  const float* gr = dxh + row * d;
  float ss = 0.f, sg = 0.f;
  for (int c = lane; c < d; c += 32) {
    const float s = xr[c] * sigm(xr[c]);
    ss += s * s;
    sg += s * gr[c];
  }
  ss = warp_sum(ss);
  sg = warp_sum(sg);
  const float n = sqrtf(ss);
  const float inv = n > 0.f ? 1.0f / n : 0.f;
  const float dot = sg * inv;   // <x^, dx^>
  for (int c = lane; c < d; c += 32) {
    const float z = xr[c], sgz = sigm(z);
    const float xh = z * sgz * inv;
    dx[row * d + c] = (gr[c] - xh * dot) * inv * sgz * (1.0f + z * (1.0f - sgz));
  }
}

// The same for bf16 inputs x, one warp per row with the row in registers:
// 8 elements per lane and step, two steps at most (d a multiple of 64, at
// most 512).  Grid-stride over the rows.
__global__ void __launch_bounds__(256) k_prologue_bwd_bf16(const __nv_bfloat16* __restrict__ x,
                                                           const float* __restrict__ dxh,
                                                           float* __restrict__ dx, int64_t rows, int d) {
  griddep_launch();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int nc = d >> 3;   // 8-element chunks per row
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; row < rows;
       row += nwarps) {
    float xv[2][8], gv[2][8];
    float ss = 0.f, sg = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = lane + 32 * i;
      if (c >= nc) continue;
      const uint4 raw = *reinterpret_cast<const uint4*>(x + row * d + 8 * c);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      const float4 g0 = *reinterpret_cast<const float4*>(dxh + row * d + 8 * c);
      const float4 g1 = *reinterpret_cast<const float4*>(dxh + row * d + 8 * c + 4);
      const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        xv[i][2 * e] = __uint_as_float(w[e] << 16);
        xv[i][2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        gv[i][e] = gg[e];
        const float s = xv[i][e] * sigm(xv[i][e]);
        ss += s * s;
        sg += s * gg[e];
      }
    }
    ss = warp_sum(ss);
    sg = warp_sum(sg);
    const float n = sqrtf(ss);
    const float inv = n > 0.f ? 1.0f / n : 0.f;
    const float dot = sg * inv;   // <x^, dx^>
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = lane + 32 * i;
      if (c >= nc) continue;
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float z = xv[i][e], sgz = sigm(z);
        o[e] = (gv[i][e] - z * sgz * inv * dot) * inv * sgz * (1.0f + z * (1.0f - sgz));
      }
      float4* out = reinterpret_cast<float4*>(dx + row * d + 8 * c);
      out[0] = make_float4(o[0], o[1], o[2], o[3]);
      out[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
  }
}

// Gradient of the initial weights: A [3][BH][plane] summed over the batch
// for an initial state shared by it (w_shared), else copied.
__global__ void __launch_bounds__(256) k_sum_batch(const float* __restrict__ A, int B, int H,
                                                   int64_t plane, int w_shared,
                                                   float* __restrict__ d1, float* __restrict__ d2,
                                                   float* __restrict__ d3) {
  griddep_launch();
  griddep_wait();
  const int Hw = w_shared ? H : B * H;
  const int64_t per = static_cast<int64_t>(Hw) * plane;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < 3 * per; i += stride) {
    const int j = static_cast<int>(i / per);
    const int64_t e = i % per;
    const int64_t hw = e / plane, off = e % plane;
    const float* src = A + static_cast<int64_t>(j) * B * H * plane;
    float acc;
    if (w_shared) {
      acc = 0.f;
      for (int b = 0; b < B; ++b) acc += src[(static_cast<int64_t>(b) * H + hw) * plane + off];
    } else {
      acc = src[hw * plane + off];
    }
    (j == 0 ? d1 : (j == 1 ? d2 : d3))[e] = acc;
  }
}

// A += B over n floats (16-byte steps when n is a multiple of 4).
__global__ void __launch_bounds__(256) k_add_planes(float* __restrict__ A, const float* __restrict__ B, int64_t n) {
  griddep_launch();
  griddep_wait();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n % 4 == 0) {
    for (int64_t i = t0; i < n / 4; i += stride) {
      float4 a = reinterpret_cast<float4*>(A)[i];
      const float4 b = reinterpret_cast<const float4*>(B)[i];
      a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
      reinterpret_cast<float4*>(A)[i] = a;
    }
  } else {
    for (int64_t i = t0; i < n; i += stride) A[i] += B[i];
  }
}

// ---------------------------------------------------------------------------
// Muon rule backward: the vector-Jacobian product of
//   U = NS5(S / (||S||_F + eps))     ("大块测试时训练（LaCT）技术解析" §2.2.1,
//                                     eqs. 9-10; five steps of
//   X <- a X + X (b A + c A A),  A = X^T X)
// runs as fp32 batched GEMMs (k_simt_gemm) over the kept iterates; these
// kernels are its elementwise and layout steps.
// ---------------------------------------------------------------------------

// out[p][c][r] = in[p][r][c] for `nplanes` planes of rows x cols (32 x 32
// tiles through shared memory).  grid (cdiv(cols, 32), cdiv(rows, 32),
// nplanes), block (32, 8).
__global__ void __launch_bounds__(256) k_transpose_planes(const float* __restrict__ in, float* __restrict__ out,
                                                          int rows, int cols) {
  griddep_launch();
  griddep_wait();
  __shared__ float tile[32][33];
  const int64_t base = static_cast<int64_t>(blockIdx.z) * rows * cols;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[base + static_cast<int64_t>(r) * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[base + static_cast<int64_t>(c) * rows + r] = tile[threadIdx.x][i];
  }
}

// M <- M + M^T for `items` n x n matrices, in place: one thread per pair
// (i <= j).
__global__ void __launch_bounds__(256) k_sym_add(float* __restrict__ M, int n, int64_t items) {
  griddep_launch();
  griddep_wait();
  const int64_t per = static_cast<int64_t>(n) * n;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < items * per; t += stride) {
    const int64_t item = t / per, e = t % per;
    const int i = static_cast<int>(e / n), j = static_cast<int>(e % n);
    if (i > j) continue;
    float* m = M + item * per;
    const float s = m[static_cast<int64_t>(i) * n + j] + m[static_cast<int64_t>(j) * n + i];
    m[static_cast<int64_t>(i) * n + j] = s;
    m[static_cast<int64_t>(j) * n + i] = s;
  }
}

// The normalisation's VJP, one block per matrix: with n = ||S||_F (from the
// forward's fixed-order partial sums of squares, `part`) and Y0 = dL/dX0,
//   dL/dS = Y0 / (n + eps) - <Y0, S> / (n (n + eps)^2) S     (n > 0)
//   dL/dS = Y0 / eps                                         (S = 0)
__global__ void __launch_bounds__(1024) k_ns_norm_vjp(const float* __restrict__ S, const float* __restrict__ Y0,
                                                     const float* __restrict__ part, int nblk, float eps,
                                                     int64_t plane, float* __restrict__ out) {
  griddep_launch();
  griddep_wait();
  __shared__ float red[32];
  __shared__ float coef[2];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * plane;
  float dot = 0.f;
  for (int64_t e = threadIdx.x; e < plane; e += blockDim.x) dot = fmaf(Y0[base + e], S[base + e], dot);
  dot = warp_sum(dot);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dot;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) {
      float ss = 0.f;
      for (int i = 0; i < nblk; ++i) ss += part[static_cast<int64_t>(blockIdx.x) * nblk + i];
      const float nrm = sqrtf(ss), den = nrm + eps;
      coef[0] = 1.0f / den;
      coef[1] = nrm > 0.f ? v / (nrm * den * den) : 0.f;
    }
  }
  __syncthreads();
  const float c0 = coef[0], c1 = coef[1];
  for (int64_t e = threadIdx.x; e < plane; e += blockDim.x) out[base + e] = c0 * Y0[base + e] - c1 * S[base + e];
}

}  // namespace lact
