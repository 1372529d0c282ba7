// GPTQ column sweep on the GPU (dingiv.github.io "量化" page, section GPTQ):
// fixed left-to-right order, every update through G (the upper Cholesky
// factor of H^-1), blocks of B columns with immediate in-block updates and
// one lazy batched update of the columns to the right after each block.
//
// Per block j0:
//   block_quant_kernel   the B columns of every row: parameters at a group
//                        start, code, dequantize, e = (w - w^)/G_qq, subtract
//                        e * G[q, k] from the later columns of the block,
//                        keep e in E; then bit-pack the block's codes.
//                        A row's B values live in registers of 4 threads
//                        (interleaved in 4-column chunks); G's diagonal
//                        block sits in shared memory and is read as
//                        broadcast float4s; e crosses the 4 threads by shuffle.
//   trailing_update_kernel  W[:, j0+B:] -= E * G[j0:j0+B, j0+B:]  (fp32 FFMA,
//                        128x128 register-tiled).
//
// Quantizer (dingiv.github.io page, section 量化基础; youleyou.com page,
// sections 二 and 四): asymmetric q = clip(rint(w/s) + z, 0, 2^b-1) with
// s = (max(0,max) - min(0,min)) / (2^b-1), z = rint(-min(0,min)/s);
// symmetric s = max|w| / (2^(b-1)-1), z = 2^(b-1); w^ = s (q - z).  The
// integer decisions are taken in fp32 with IEEE division and
// round-half-to-even.
#pragma once

#include "common.cuh"

namespace gptq {
namespace quant {

__device__ __forceinline__ void make_params(float mn, float mx, int bits, int sym, float& s,
                                            float& z) {
  if (sym) {
    float amax = fmaxf(fabsf(mn), fabsf(mx));
    if (amax == 0.0f) amax = 1.0f;
    s = amax / static_cast<float>((1 << (bits - 1)) - 1);
    z = static_cast<float>(1 << (bits - 1));
  } else {
    mn = fminf(mn, 0.0f);
    mx = fmaxf(mx, 0.0f);
    if (mn == 0.0f && mx == 0.0f) { mn = -1.0f; mx = 1.0f; }
    s = (mx - mn) / static_cast<float>((1 << bits) - 1);
    z = rintf(-mn / s);
  }
}

// Copy W into the working buffer (dead columns zeroed) and, for one scale per
// output channel, compute each row's parameters from that copy.  One warp per row.
__global__ void prepare_rows_kernel(const float* __restrict__ W, float* __restrict__ Wk,
                                    const uint8_t* __restrict__ dead, int d_row, int d_col,
                                    int bits, int sym, int per_channel,
                                    float* __restrict__ scales, uint8_t* __restrict__ zeros) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= d_row) return;
  const float4* src = reinterpret_cast<const float4*>(W + static_cast<size_t>(r) * d_col);
  float4* dst = reinterpret_cast<float4*>(Wk + static_cast<size_t>(r) * d_col);
  float mn = 0.0f, mx = 0.0f;
  for (int c4 = lane; c4 < d_col / 4; c4 += 32) {
    float4 v = src[c4];
    if (dead) {
      const uchar4 dm = reinterpret_cast<const uchar4*>(dead)[c4];
      if (dm.x) v.x = 0.0f;
      if (dm.y) v.y = 0.0f;
      if (dm.z) v.z = 0.0f;
      if (dm.w) v.w = 0.0f;
    }
    dst[c4] = v;
    mn = fminf(mn, fminf(fminf(v.x, v.y), fminf(v.z, v.w)));
    mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
  }
  if (!per_channel) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    float s, z;
    make_params(mn, mx, bits, sym, s, z);
    scales[r] = s;
    zeros[r] = static_cast<uint8_t>(z);
  }
}

constexpr int QROWS = 32;            // rows per CTA
constexpr int QTHREADS = QROWS * 4;  // 4 threads per row

template <int B>
constexpr int block_quant_smem() {
  return B * B * 4 + B * 4 + QROWS * B;
}

// Mode flags for the group handling at the block start (GS == 0 variants):
//   pc_mode 1: parameters per output channel, precomputed;
//   pc_mode 0: group_size is a multiple of B: a group starts here when
//              j0 % group == 0 (parameters over columns [j0, j0+group) of the
//              current W, the part beyond this block read from memory),
//              otherwise the group's parameters were written by an earlier block.
template <int B, int GS>
__global__ void __launch_bounds__(QTHREADS)
block_quant_kernel(const float* __restrict__ Wk, int d_row, int d_col, int j0, int ncols,
                   const float* __restrict__ G, float* __restrict__ E,
                   uint32_t* __restrict__ qweight, float* __restrict__ scales,
                   uint8_t* __restrict__ zeros, int bits, int sym, int group, int n_groups,
                   int pc_mode) {
  static_assert(B % 16 == 0 && (GS == 0 || (GS % 16 == 0 && B % GS == 0)), "shape");
  constexpr int V = B / 4;       // values per thread
  constexpr int NCH = B / 16;    // 16-column chunks; thread t owns columns 16c+4t..16c+4t+3
  extern __shared__ __align__(16) uint8_t qsm[];
  float* gs = reinterpret_cast<float*>(qsm);  // B x B block of G
  float* inv_diag = gs + B * B;
  uint8_t* cstage = reinterpret_cast<uint8_t*>(inv_diag + B);  // QROWS x B codes

  const int tid = threadIdx.x;
  const int rloc = tid >> 2, t = tid & 3;
  const int lane = tid & 31;
  const int qbase = lane & ~3;
  const int r = blockIdx.x * QROWS + rloc;
  const bool rv = r < d_row;

  for (int idx = tid; idx < B * B / 4; idx += QTHREADS) {
    const int q = (idx * 4) / B, k = (idx * 4) % B;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (q < ncols && k < ncols)
      v = *reinterpret_cast<const float4*>(G + static_cast<size_t>(j0 + q) * d_col + j0 + k);
    reinterpret_cast<float4*>(gs)[idx] = v;
  }
  for (int q = tid; q < B; q += QTHREADS)
    inv_diag[q] = (q < ncols) ? 1.0f / G[static_cast<size_t>(j0 + q) * d_col + j0 + q] : 0.0f;

  float w[V], ev[V];
  const float* wrow = Wk + static_cast<size_t>(rv ? r : 0) * d_col + j0;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const int col = 16 * c + 4 * t;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rv && col < ncols) v = *reinterpret_cast<const float4*>(wrow + col);
    w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
    ev[4 * c] = ev[4 * c + 1] = ev[4 * c + 2] = ev[4 * c + 3] = 0.0f;
  }

  const float maxq = static_cast<float>((1 << bits) - 1);
  float s = 1.0f, z = 0.0f;
  if (GS == 0) {
    const int g = pc_mode ? 0 : j0 / group;
    if (!pc_mode && (j0 % group) == 0) {
      float mn = w[0], mx = w[0];
#pragma unroll
      for (int i = 1; i < V; ++i) { mn = fminf(mn, w[i]); mx = fmaxf(mx, w[i]); }
      const float* rest = Wk + static_cast<size_t>(rv ? r : 0) * d_col;
      for (int c = j0 + B + t; c < j0 + group; c += 4) {
        const float v = rest[c];
        mn = fminf(mn, v); mx = fmaxf(mx, v);
      }
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      make_params(mn, mx, bits, sym, s, z);
      if (rv && t == 0) {
        scales[static_cast<size_t>(r) * n_groups + g] = s;
        zeros[static_cast<size_t>(r) * n_groups + g] = static_cast<uint8_t>(z);
      }
    } else if (rv) {
      s = scales[static_cast<size_t>(r) * n_groups + g];
      z = static_cast<float>(zeros[static_cast<size_t>(r) * n_groups + g]);
    }
  }
  __syncthreads();

#pragma unroll
  for (int q = 0; q < B; ++q) {
    if (q < ncols) {
    if (GS != 0 && (q % (GS > 0 ? GS : 1)) == 0) {
      float mn = 3.4e38f, mx = -3.4e38f;
#pragma unroll
      for (int c = q / 16; c < (q + (GS > 0 ? GS : 16)) / 16; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) { mn = fminf(mn, w[4 * c + e]); mx = fmaxf(mx, w[4 * c + e]); }
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      make_params(mn, mx, bits, sym, s, z);
      if (rv && t == 0) {
        const int g = (j0 + q) / (GS > 0 ? GS : 1);
        scales[static_cast<size_t>(r) * n_groups + g] = s;
        zeros[static_cast<size_t>(r) * n_groups + g] = static_cast<uint8_t>(z);
      }
    }
    const int tq = (q >> 2) & 3;        // owner thread of column q
    const int slot = (q >> 4) * 4 + (q & 3);
    float e = 0.0f;
    if (t == tq) {
      const float x = w[slot];
      float qf = rintf(x / s) + z;
      qf = fminf(fmaxf(qf, 0.0f), maxq);
      const float xh = s * (qf - z);
      e = (x - xh) * inv_diag[q];
      ev[slot] = e;
      cstage[rloc * B + q] = static_cast<uint8_t>(qf);
    }
    e = __shfl_sync(0xffffffffu, e, qbase | tq);
    const float* grow = gs + q * B;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      if (16 * c + 15 <= q) continue;  // chunk entirely at or left of q
      const float4 g4 = *reinterpret_cast<const float4*>(grow + 16 * c + 4 * t);
      const int kb = 16 * c + 4 * t;
      if (16 * c > q) {
        w[4 * c] -= e * g4.x; w[4 * c + 1] -= e * g4.y;
        w[4 * c + 2] -= e * g4.z; w[4 * c + 3] -= e * g4.w;
      } else {
        if (kb > q) w[4 * c] -= e * g4.x;
        if (kb + 1 > q) w[4 * c + 1] -= e * g4.y;
        if (kb + 2 > q) w[4 * c + 2] -= e * g4.z;
        if (kb + 3 > q) w[4 * c + 3] -= e * g4.w;
      }
    }
    }
  }

  // E for the trailing update
  if (rv) {
    float* erow = E + static_cast<size_t>(r) * B;
#pragma unroll
    for (int c = 0; c < NCH; ++c)
      *reinterpret_cast<float4*>(erow + 16 * c + 4 * t) =
          make_float4(ev[4 * c], ev[4 * c + 1], ev[4 * c + 2], ev[4 * c + 3]);
  }
  __syncwarp();
  // bit-pack this block's codes: little-endian stream, code k at bits [b k, b k + b)
  if (rv) {
    const int nw = ncols * bits / 32;
    const size_t row_words = static_cast<size_t>(d_col) * bits / 32;
    uint32_t* qrow = qweight + static_cast<size_t>(r) * row_words + (static_cast<size_t>(j0) * bits) / 32;
    const uint8_t* cs = cstage + rloc * B;
    for (int wi = t; wi < nw; wi += 4) {
      const int bit0 = 32 * wi;
      const int kf = bit0 / bits, kl = (bit0 + 31) / bits;
      uint32_t val = 0;
      for (int k = kf; k <= kl; ++k) {
        const int sh = k * bits - bit0;
        const uint32_t c = cs[k];
        val |= (sh >= 0) ? (c << sh) : (c >> (-sh));
      }
      qrow[wi] = val;
    }
  }
}

// W[:, n0:] -= E * G[j0:j0+K, n0:]  -- C (ldc = d_col) -= A (ld K) * B (ld d_col).
constexpr int UT = 128, UK = 16, UTHREADS = 256;

__global__ void __launch_bounds__(UTHREADS, 1)
trailing_update_kernel(float* __restrict__ C, const float* __restrict__ A,
                       const float* __restrict__ Bm, int M, int N, int K, int ldc, int ldb) {
  __shared__ __align__(16) float As[2][UK][UT];
  __shared__ __align__(16) float Bs[2][UK][UT];
  const int m0 = blockIdx.x * UT, n0 = blockIdx.y * UT;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  float4 ra[2], rb[2];
  auto load = [&](int k0) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int idx = tid + e * UTHREADS;  // 512 float4 per operand slice
      const int am = idx >> 2, ak = (idx & 3) * 4;  // A: 128 rows x 16 k
      ra[e] = (m0 + am < M) ? *reinterpret_cast<const float4*>(A + static_cast<size_t>(m0 + am) * K + k0 + ak)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      const int bk = idx >> 5, bn = (idx & 31) * 4;  // B: 16 k x 128 cols
      rb[e] = (n0 + bn < N) ? *reinterpret_cast<const float4*>(Bm + static_cast<size_t>(k0 + bk) * ldb + n0 + bn)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int idx = tid + e * UTHREADS;
      const int am = idx >> 2, ak = (idx & 3) * 4;
      As[buf][ak][am] = ra[e].x; As[buf][ak + 1][am] = ra[e].y;
      As[buf][ak + 2][am] = ra[e].z; As[buf][ak + 3][am] = ra[e].w;
      const int bk = idx >> 5, bn = (idx & 31) * 4;
      *reinterpret_cast<float4*>(&Bs[buf][bk][bn]) = rb[e];
    }
  };

  load(0);
  store(0);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < K; k0 += UK) {
    const bool more = k0 + UK < K;
    if (more) load(k0 + UK);
#pragma unroll
    for (int k = 0; k < UK; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][k][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (more) {
      store(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (gm >= M) continue;
    float* crow = C + static_cast<size_t>(gm) * ldc + n0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cn = h * 64 + tx * 4;
      if (n0 + cn >= N) continue;  // N % 32 == 0, so a float4 is all in or all out
      float4 c = *reinterpret_cast<float4*>(crow + cn);
      c.x -= acc[i][4 * h]; c.y -= acc[i][4 * h + 1];
      c.z -= acc[i][4 * h + 2]; c.w -= acc[i][4 * h + 3];
      *reinterpret_cast<float4*>(crow + cn) = c;
    }
  }
}

// ---------------------------------------------------------- dequant / loss
__device__ __forceinline__ float dequant_at(const uint32_t* __restrict__ qrow,
                                            const float* __restrict__ srow,
                                            const uint8_t* __restrict__ zrow, int k, int bits,
                                            int group) {
  const int bit = k * bits;
  const int wi = bit >> 5, off = bit & 31;
  uint64_t v = qrow[wi];
  if (off + bits > 32) v |= static_cast<uint64_t>(qrow[wi + 1]) << 32;
  const uint32_t q = static_cast<uint32_t>(v >> off) & ((1u << bits) - 1u);
  const int g = group ? k / group : 0;
  return srow[g] * (static_cast<float>(q) - static_cast<float>(zrow[g]));
}

__global__ void dequant_kernel(const uint32_t* __restrict__ qweight,
                               const float* __restrict__ scales, const uint8_t* __restrict__ zeros,
                               int d_row, int d_col, int bits, int group, int n_groups,
                               float* __restrict__ W_hat) {
  const size_t total = static_cast<size_t>(d_row) * d_col;
  const size_t row_words = static_cast<size_t>(d_col) * bits / 32;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / d_col), k = static_cast<int>(i % d_col);
    W_hat[i] = dequant_at(qweight + r * row_words, scales + static_cast<size_t>(r) * n_groups,
                          zeros + static_cast<size_t>(r) * n_groups, k, bits, group);
  }
}

// Partial sums of 1/2 sum_r dW_r H dW_r^T over 128 x 128 output tiles of
// T = dW * H (H symmetric, read from its upper triangle); fp64 accumulation.
__global__ void __launch_bounds__(256)
loss_tiles_kernel(const uint32_t* __restrict__ qweight, const float* __restrict__ scales,
                  const uint8_t* __restrict__ zeros, const float* __restrict__ W,
                  const float* __restrict__ H, int d_row, int d_col, int bits, int group,
                  int n_groups, double* __restrict__ partials) {
  __shared__ float As[16][128];
  __shared__ float Bs[16][128];
  __shared__ double red[8];
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * 128;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const size_t row_words = static_cast<size_t>(d_col) * bits / 32;
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;

  for (int k0 = 0; k0 < d_col; k0 += 16) {
    for (int idx = tid; idx < 2048; idx += 256) {
      const int m = idx >> 4, k = idx & 15;
      const int gm = m0 + m, gk = k0 + k;
      float v = 0.0f;
      if (gm < d_row && gk < d_col)
        v = W[static_cast<size_t>(gm) * d_col + gk] -
            dequant_at(qweight + gm * row_words, scales + static_cast<size_t>(gm) * n_groups,
                       zeros + static_cast<size_t>(gm) * n_groups, gk, bits, group);
      As[k][m] = v;
      const int kk = idx >> 7, n = idx & 127;
      const int gk2 = k0 + kk, gn = n0 + n;
      float h = 0.0f;
      if (gk2 < d_col && gn < d_col)
        h = (gk2 <= gn) ? H[static_cast<size_t>(gk2) * d_col + gn] : H[static_cast<size_t>(gn) * d_col + gk2];
      Bs[kk][n] = h;
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
      double a[8], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[k][ty * 4 + i]; a[4 + i] = As[k][64 + ty * 4 + i];
        b[i] = Bs[k][tx * 4 + i]; b[4 + i] = Bs[k][64 + tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  double part = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (gm >= d_row) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (gn >= d_col) continue;
      const float dw = W[static_cast<size_t>(gm) * d_col + gn] -
                       dequant_at(qweight + gm * row_words, scales + static_cast<size_t>(gm) * n_groups,
                                  zeros + static_cast<size_t>(gm) * n_groups, gn, bits, group);
      part += acc[i][j] * static_cast<double>(dw);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((tid & 31) == 0) red[tid >> 5] = part;
  __syncthreads();
  if (tid == 0) {
    double s = 0.0;
    for (int i = 0; i < 8; ++i) s += red[i];
    partials[blockIdx.y * gridDim.x + blockIdx.x] = 0.5 * s;
  }
}

__global__ void sum_partials_kernel(const double* __restrict__ partials, int n,
                                    double* __restrict__ out) {
  __shared__ double red[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += partials[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += red[i];
    *out = t;
  }
}

}  // namespace quant
}  // namespace gptq
