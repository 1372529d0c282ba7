// AWQ scale search (dingiv.github.io "量化" page, section AWQ): the salient
// input channels are those with large mean activation magnitude s_X; the
// weights of channel k are multiplied by s_k = s_X[k]^alpha before 4-bit
// quantization and the activations divided by s_k (an equivalent
// transform), with alpha chosen on a 20-point grid over [0, 1] by the
// layer's output error.
//
// The output error of one alpha is evaluated through the calibration
// Hessian H = 2 X X^T, which the GPTQ path already builds with its tcgen05
// SYRK: with dW = W - Q(W diag(s)) diag(s)^-1,
//     ||W X - W^ X||_F^2 = 1/2 sum_r dW_r H dW_r^T.
// The d_row x d_col x d_col contraction dW H runs on the 5th-generation
// tensor cores through the split-TF32 kernel of the trailing update
// (three TF32 products of hi/lo splits, near-fp32 accuracy), then one pass
// takes the elementwise product with dW.  Per alpha:
//   scales_kernel   s = s_X^alpha (fp64 pow, rounded to fp32; 1 where s_X = 0)
//   delta_kernel    per (row, group): min-max parameters of W diag(s), codes,
//                   dW = W - s_g (q - z) / s, written as its TF32 hi/lo split
//   (memset)        T = 0
//   trailing kernel T -= dW H
//   dot_kernel      per-block fp64 partials of sum dW * T
//   finalize        loss = -1/2 sum of partials (fixed order)
// then argmin_kernel picks the first smallest loss and writes s*, and
// pack_kernel writes the 4-bit codes, scales and zero points of W diag(s*).
// The min-max quantizer is the GPTQ path's (quant::make_params), with the
// same fp32 operations, so alpha = 0 gives round-to-nearest exactly.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "quantize.cuh"

namespace gptq {
namespace awq {

constexpr int THREADS = 256;
constexpr int COLS_PER_BLOCK = 2 * THREADS;  // channel-scale kernel: one bf16 pair per thread
constexpr int DOT_BLOCKS = 1184;             // 8 per SM

// ------------------------------------------------------------ channel scale
// sum_t |x[t][k]| in fp64 over a chunk of tokens, added into sum[k].  The
// inputs are bf16, so every partial sum is exact in fp64 whatever the order
// (8 significant bits per term), and the result does not depend on the
// atomic order.
__global__ void absum_kernel(const __nv_bfloat16* __restrict__ X, int n, int d, long long ldx,
                             int tok_per_block, double* __restrict__ sum) {
  const int c2 = blockIdx.x * THREADS + threadIdx.x;  // column pair
  if (2 * c2 >= d) return;
  const int t0 = blockIdx.y * tok_per_block, t1 = min(n, t0 + tok_per_block);
  double a = 0.0, b = 0.0;
  const __nv_bfloat162* p =
      reinterpret_cast<const __nv_bfloat162*>(X + static_cast<size_t>(t0) * ldx) + c2;
  const size_t step = static_cast<size_t>(ldx / 2);
  for (int t = t0; t < t1; ++t, p += step) {
    const float2 v = __bfloat1622float2(*p);
    a += fabs(static_cast<double>(v.x));
    b += fabs(static_cast<double>(v.y));
  }
  atomicAdd(sum + 2 * c2, a);
  atomicAdd(sum + 2 * c2 + 1, b);
}

__global__ void mean_kernel(double* __restrict__ sx, int d, int n) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < d) sx[k] = sx[k] / static_cast<double>(n);
}

// --------------------------------------------------------- H, symmetric split
// The SYRK writes the upper triangle; the contraction reads whole rows of H.
__global__ void sym_split_kernel(const float* __restrict__ H, int d, float* __restrict__ hi,
                                 float* __restrict__ lo) {
  const size_t n = static_cast<size_t>(d) * d;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / d), c = static_cast<int>(i % d);
    const float v = r <= c ? H[i] : H[static_cast<size_t>(c) * d + r];
    const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    hi[i] = h;
    lo[i] = v - h;
  }
}

__device__ __forceinline__ float scale_of(double sx, double alpha) {
  return sx > 0.0 ? static_cast<float>(pow(sx, alpha)) : 1.0f;
}

__global__ void scales_kernel(const double* __restrict__ sx, int d, double alpha,
                              float* __restrict__ s) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < d) s[k] = scale_of(sx[k], alpha);
}

// ------------------------------------------------- per (row, group) quantize
// One warp per (row, group); lane l holds 8 consecutive columns at a time
// (two float4 of W and of s).  Min and max of W diag(s) over the group, the
// quantizer's scale and zero point, then per column the code
// q = clip(rint(w s / s_g) + z, 0, 15).
struct Group {
  int r, c0, c1, gi;
};

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void group_params(const float* __restrict__ W,
                                             const float* __restrict__ s, int d_col,
                                             const Group& gr, int lane, float& sg, float& z) {
  const float* wr = W + static_cast<size_t>(gr.r) * d_col;
  float mn = 0.0f, mx = 0.0f;  // the quantizer widens the range to contain 0 anyway
  for (int c = gr.c0 + 8 * lane; c < gr.c1; c += 256) {
    float w[8], sc[8];
    load8(wr + c, w);
    load8(s + c, sc);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v = w[i] * sc[i];
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  quant::make_params(mn, mx, 4, 0, sg, z);
}

__device__ __forceinline__ float code_of(float v, float sg, float z) {
  return fminf(fmaxf(rintf(v / sg) + z, 0.0f), 15.0f);
}

__device__ __forceinline__ Group group_at(int u, int n_groups, int gw) {
  Group g;
  g.r = u / n_groups;
  g.gi = u - g.r * n_groups;
  g.c0 = g.gi * gw;
  g.c1 = g.c0 + gw;
  return g;
}

// dW = W - s_g (q - z) / s for one alpha, written as its TF32 hi/lo split.
__global__ void __launch_bounds__(THREADS)
delta_kernel(const float* __restrict__ W, const float* __restrict__ s, int d_row, int d_col,
             int gw, float* __restrict__ ehi, float* __restrict__ elo) {
  const int lane = threadIdx.x & 31;
  const int n_groups = d_col / gw;
  const int units = d_row * n_groups;
  for (int u = blockIdx.x * (THREADS / 32) + (threadIdx.x >> 5); u < units;
       u += gridDim.x * (THREADS / 32)) {
    const Group gr = group_at(u, n_groups, gw);
    float sg, z;
    group_params(W, s, d_col, gr, lane, sg, z);
    const size_t row = static_cast<size_t>(gr.r) * d_col;
    for (int c = gr.c0 + 8 * lane; c < gr.c1; c += 256) {
      float w[8], sc[8], h[8], l[8];
      load8(W + row + c, w);
      load8(s + c, sc);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float q = code_of(w[i] * sc[i], sg, z);
        const float dw = w[i] - sg * (q - z) / sc[i];
        h[i] = __uint_as_float(__float_as_uint(dw) & 0xFFFFE000u);
        l[i] = dw - h[i];
      }
      *reinterpret_cast<float4*>(ehi + row + c) = make_float4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<float4*>(ehi + row + c + 4) = make_float4(h[4], h[5], h[6], h[7]);
      *reinterpret_cast<float4*>(elo + row + c) = make_float4(l[0], l[1], l[2], l[3]);
      *reinterpret_cast<float4*>(elo + row + c + 4) = make_float4(l[4], l[5], l[6], l[7]);
    }
  }
}

// --------------------------------------------------------------- the loss
// Per-block fp64 partials of sum (ehi + elo) * T over n elements (n % 4 == 0).
__global__ void __launch_bounds__(THREADS)
dot_kernel(const float* __restrict__ ehi, const float* __restrict__ elo,
           const float* __restrict__ T, size_t n4, double* __restrict__ partials) {
  __shared__ double red[THREADS / 32];
  double acc = 0.0;
  for (size_t i = blockIdx.x * static_cast<size_t>(THREADS) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * THREADS) {
    const float4 a = reinterpret_cast<const float4*>(ehi)[i];
    const float4 b = reinterpret_cast<const float4*>(elo)[i];
    const float4 t = reinterpret_cast<const float4*>(T)[i];
    acc += static_cast<double>(a.x + b.x) * t.x + static_cast<double>(a.y + b.y) * t.y +
           static_cast<double>(a.z + b.z) * t.z + static_cast<double>(a.w + b.w) * t.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < THREADS / 32; ++w) t += red[w];
    partials[blockIdx.x] = t;
  }
}

// loss = -1/2 sum of the partials (T = -dW H), summed in a fixed order.
__global__ void finalize_kernel(const double* __restrict__ partials, int n,
                                double* __restrict__ loss) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += partials[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += red[w];
    *loss = -0.5 * t;
  }
}

// The first smallest loss (ties go to the smaller alpha); s* for every column.
__global__ void argmin_kernel(const double* __restrict__ losses, int n_grid,
                              const double* __restrict__ sx, int d, int32_t* __restrict__ best,
                              float* __restrict__ s_out) {
  __shared__ int b;
  if (threadIdx.x == 0) {
    int k = 0;
    for (int a = 1; a < n_grid; ++a)
      if (losses[a] < losses[k]) k = a;
    b = k;
    *best = k;
  }
  __syncthreads();
  const double alpha = static_cast<double>(b) / static_cast<double>(n_grid - 1);
  for (int k = threadIdx.x; k < d; k += blockDim.x) s_out[k] = scale_of(sx[k], alpha);
}

// 4-bit codes of W diag(s*), packed 8 per word (code k of a row at bits
// 4 (k % 8) of word k / 8), with the group's scale and zero point.
__global__ void __launch_bounds__(THREADS)
pack_kernel(const float* __restrict__ W, const float* __restrict__ s, int d_row, int d_col,
            int gw, uint32_t* __restrict__ qweight, float* __restrict__ scales,
            uint8_t* __restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int n_groups = d_col / gw;
  const int units = d_row * n_groups;
  for (int u = blockIdx.x * (THREADS / 32) + (threadIdx.x >> 5); u < units;
       u += gridDim.x * (THREADS / 32)) {
    const Group gr = group_at(u, n_groups, gw);
    float sg, z;
    group_params(W, s, d_col, gr, lane, sg, z);
    const size_t row = static_cast<size_t>(gr.r) * d_col;
    for (int c = gr.c0 + 8 * lane; c < gr.c1; c += 256) {
      float w[8], sc[8];
      load8(W + row + c, w);
      load8(s + c, sc);
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        word |= static_cast<uint32_t>(code_of(w[i] * sc[i], sg, z)) << (4 * i);
      qweight[(row + c) / 8] = word;
    }
    if (lane == 0) {
      scales[static_cast<size_t>(gr.r) * n_groups + gr.gi] = sg;
      zeros[static_cast<size_t>(gr.r) * n_groups + gr.gi] = static_cast<uint8_t>(z);
    }
  }
}

}  // namespace awq
}  // namespace gptq
