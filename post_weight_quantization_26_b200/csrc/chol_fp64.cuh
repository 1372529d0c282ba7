// fp64 pipeline from the accumulated Hessian to G, the upper triangular U
// with U^T U = (H + lambda I)^-1  (dingiv.github.io "量化" page, section
// GPTQ: the updates go through the Cholesky factor of H^-1, chosen there for
// numerical stability of a near-singular H).
//
// Route: with J the order-reversing permutation, factor A = J H' J = L L^T
// (so H' = V V^T with V = J L J upper triangular), invert X = L^-1, and
// G = J X J = V^-1.  That is one Cholesky (d^3/3 flops) and one triangular
// inverse (d^3/3) instead of factor + invert + multiply + factor.
//
// Blocked right-looking Cholesky over NB = 128 column panels:
//   leaf   one CTA factors the 128x128 diagonal block in shared memory and
//          builds its inverse in the same column sweep;
//   panel  L21 = A21 * X11^T  (grouped DGEMM, in place);
//   update A22 -= L21 * L21^T on the lower tiles only (grouped DGEMM).
// Triangular inverse by recursive halving, bottom-up by tree height, every
// node of a height in one grouped launch:
//   T  = L21 * X11  (kept transposed in the free upper triangle),
//   X21 = -X22 * T.
// All arithmetic is fp64 FMA; the matrix lives in one d x d fp64 buffer.
#pragma once

#include "common.cuh"

namespace gptq {
namespace chol {

constexpr int NB = 128;  // panel / leaf width

// -------------------------------------------------------------- damping
// One CTA: mean of diag(H), dead channels, NaN/Inf check.
//   stats[0] = lambda (fp64), istat[0] = nonfinite flag.
__global__ void __launch_bounds__(1024)
diag_stats_kernel(const float* __restrict__ H, int d, double damp_rel,
                  uint8_t* __restrict__ dead, double* __restrict__ stats,
                  int* __restrict__ istat) {
  __shared__ double red[32];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  double s = 0.0;
  int nonfinite = 0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const float h = H[static_cast<size_t>(i) * d + i];
    if (!isfinite(h)) nonfinite = 1;
    dead[i] = (h == 0.0f) ? 1 : 0;
    s += static_cast<double>(h);
  }
  if (nonfinite) atomicOr(&bad, 1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) {
      stats[0] = damp_rel * (s / d);
      istat[0] = bad;
    }
  }
}

// A[i][j] = H'[d-1-i][d-1-j] for i >= j (lower triangle of the reversed,
// damped matrix), read from H's upper triangle.  Strict upper untouched.
__global__ void reverse_damp_fill_kernel(const float* __restrict__ H, int d,
                                         const double* __restrict__ stats,
                                         double* __restrict__ A) {
  const int i = blockIdx.y;
  const double lam = stats[0];
  const float* hrow = H + static_cast<size_t>(d - 1 - i) * d;
  double* arow = A + static_cast<size_t>(i) * d;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j <= i; j += gridDim.x * blockDim.x) {
    double v = static_cast<double>(hrow[d - 1 - j]);
    if (j == i) v = (v == 0.0) ? 1.0 : v + lam;
    arow[j] = v;
  }
}

// ------------------------------------------------------------------ leaf
// Factor the n x n (n <= 128) diagonal block at (k0,k0) of A in place
// (lower triangle gets L, strict upper gets 0) and write X = L^-1 (lower,
// zero above) to Xout (n x n, leading dimension NB).  The inverse is built
// in the same sweep: starting from M = I, column step j scales row j of M
// by 1/l_jj and subtracts l_ij * (row j) from every row i > j, so that after
// the last step M = L^-1.  M's strict lower part is kept transposed in the
// strict upper half of the shared array.
// A non-positive or non-finite pivot records the original-order column
// index d-1-(k0+j) in *bad_pivot (first failure only) and the sweep goes on.
constexpr int LEAF_THREADS = 512;
constexpr int LEAF_LD = NB + 1;  // padded row: column reads hit distinct banks
constexpr int LEAF_SMEM = (NB * LEAF_LD + 2 * NB) * 8;

__global__ void __launch_bounds__(LEAF_THREADS)
leaf_potrf_inv_kernel(double* __restrict__ A, int d, int k0, int n,
                      double* __restrict__ Xout, long long* __restrict__ bad_pivot) {
  extern __shared__ double sm[];
  double* S = sm;                 // n x LEAF_LD
  double* dinv = sm + NB * LEAF_LD;  // 1 / l_jj
  double* ldiag = dinv + NB;         // l_jj (S[j][j] keeps the pivot during the sweep)
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, nwarps = LEAF_THREADS / 32;
  double* Ablk = A + static_cast<size_t>(k0) * d + k0;

  for (int idx = tid; idx < n * n; idx += LEAF_THREADS) {
    const int i = idx / n, k = idx - i * n;
    S[i * LEAF_LD + k] = (k <= i) ? Ablk[static_cast<size_t>(i) * d + k] : 0.0;
  }
  __syncthreads();

  for (int j = 0; j < n; ++j) {
    const double piv = S[j * LEAF_LD + j];
    if (tid == 0 && !(piv > 0.0 && isfinite(piv))) {
      atomicCAS(reinterpret_cast<unsigned long long*>(bad_pivot),
                static_cast<unsigned long long>(-1ll),
                static_cast<unsigned long long>(d - 1 - (k0 + j)));
    }
    const double ljj = sqrt(piv);
    const double r = 1.0 / ljj;
    // scale column j below the diagonal (l_ij) and row j of M (stored at
    // S[c][j], c < j).  S[j][j] is left alone: other warps may still read it.
    for (int i = tid; i < n; i += LEAF_THREADS)
      if (i != j) S[i * LEAF_LD + j] *= r;
    if (tid == 0) { ldiag[j] = ljj; dinv[j] = r; }
    __syncthreads();
    // rows i > j: Cholesky trailing update (k in (j, i]) and inverse rows (c in [0, j])
    for (int i = j + 1 + warp; i < n; i += nwarps) {
      const double lij = S[i * LEAF_LD + j];
      for (int k = j + 1 + lane; k <= i; k += 32)
        S[i * LEAF_LD + k] -= lij * S[k * LEAF_LD + j];
      for (int c = lane; c < j; c += 32)
        S[c * LEAF_LD + i] -= lij * S[c * LEAF_LD + j];
      if (lane == 0) S[j * LEAF_LD + i] = -lij * r;
    }
    __syncthreads();
  }

  for (int idx = tid; idx < n * n; idx += LEAF_THREADS) {
    const int i = idx / n, k = idx - i * n;
    Ablk[static_cast<size_t>(i) * d + k] = (k < i) ? S[i * LEAF_LD + k] : (k == i ? ldiag[i] : 0.0);
    double x = 0.0;
    if (k < i) x = S[k * LEAF_LD + i];
    else if (k == i) x = dinv[i];
    Xout[i * NB + k] = x;
  }
}

// Copy the leaf inverses into the diagonal blocks of A (zero above).
__global__ void place_diag_inverses_kernel(double* __restrict__ A, int d,
                                           const double* __restrict__ Xd) {
  const int b = blockIdx.x;
  const int k0 = b * NB;
  const int n = min(NB, d - k0);
  const double* X = Xd + static_cast<size_t>(b) * NB * NB;
  for (int idx = threadIdx.x; idx < n * n; idx += blockDim.x) {
    const int i = idx / n, k = idx - i * n;
    A[static_cast<size_t>(k0 + i) * d + k0 + k] = X[i * NB + k];
  }
}

// G[i][j] = X[d-1-i][d-1-j] (fp32) for i <= j, 0 below the diagonal.
__global__ void write_g_kernel(const double* __restrict__ X, int d, float* __restrict__ G) {
  const int i = blockIdx.y;
  const double* xrow = X + static_cast<size_t>(d - 1 - i) * d;
  float* grow = G + static_cast<size_t>(i) * d;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < d; j += gridDim.x * blockDim.x)
    grow[j] = (j >= i) ? static_cast<float>(xrow[d - 1 - j]) : 0.0f;
}

// ------------------------------------------------------------ grouped DGEMM
// C = alpha * op(A) op(B) + beta * C for up to MAXP problems per launch.
//   op(A)(m,k) = a_trans ? A[k*lda + m] : A[m*lda + k]
//   op(B)(k,n) = b_trans ? B[n*ldb + k] : B[k*ldb + n]
//   kmode 0: full K; 1: op(A) lower triangular in (m,k) -> k < tile_m_end;
//         2: op(A) upper (k >= m) -> k >= tile_m_begin.
//   lower_only: only output tiles with tile_n <= tile_m.
// 128 x 128 tile per CTA, 256 threads, 8 x 8 fp64 accumulators per thread,
// 16-deep K slices double-buffered through shared memory.
constexpr int TM = 128, TN = 128, TK = 16;
constexpr int GEMM_THREADS = 256;
constexpr int MAXP = 64;
constexpr int GEMM_SMEM = 2 * TK * (TM + TN) * 8;  // 64 KB, dynamic

struct GemmProblem {
  const double* A;
  const double* B;
  double* C;
  long long lda, ldb, ldc;
  int M, N, K;
  int a_trans, b_trans, kmode, lower_only;
  double alpha, beta;
};

struct GemmBatch {
  int count;
  int tile_start[MAXP + 1];
  GemmProblem p[MAXP];
};

__global__ void __launch_bounds__(GEMM_THREADS, 1)
dgemm_grouped_kernel(const __grid_constant__ GemmBatch batch) {
  extern __shared__ __align__(16) double gsm[];
  double (*As)[TK][TM] = reinterpret_cast<double (*)[TK][TM]>(gsm);
  double (*Bs)[TK][TN] = reinterpret_cast<double (*)[TK][TN]>(gsm + 2 * TK * TM);

  // find the problem and tile of this CTA
  const int bid = blockIdx.x;
  int pi = 0;
  while (pi + 1 < batch.count && batch.tile_start[pi + 1] <= bid) ++pi;
  const GemmProblem& q = batch.p[pi];
  int t = bid - batch.tile_start[pi];
  int tm_i, tn_i;
  if (q.lower_only) {  // row-major enumeration of the lower (incl. diagonal) tiles
    int r = 0;
    while ((r + 1) * (r + 2) / 2 <= t) ++r;
    tm_i = r;
    tn_i = t - r * (r + 1) / 2;
  } else {
    const int tn = (q.N + TN - 1) / TN;
    tm_i = t / tn;
    tn_i = t - tm_i * tn;
  }
  const int m0 = tm_i * TM, n0 = tn_i * TN;
  int kb = 0, ke = q.K;
  if (q.kmode == 1) ke = min(q.K, m0 + TM);
  if (q.kmode == 2) kb = (m0 / TK) * TK;

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;

  // global -> register staging: each thread loads 8 elements of A and 8 of B per slice
  double ra[8], rb[8];
  auto load_slice = [&](int k0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int idx = tid + e * GEMM_THREADS;  // 0..2047 over a 128 x 16 tile
      // A: element (m, k) of the slice
      int m, k;
      if (q.a_trans) { k = idx >> 7; m = idx & 127; } else { m = idx >> 4; k = idx & 15; }
      const int gm = m0 + m, gk = k0 + k;
      ra[e] = (gm < q.M && gk < ke)
                  ? (q.a_trans ? q.A[static_cast<size_t>(gk) * q.lda + gm]
                               : q.A[static_cast<size_t>(gm) * q.lda + gk])
                  : 0.0;
      int n, kk;
      if (q.b_trans) { n = idx >> 4; kk = idx & 15; } else { kk = idx >> 7; n = idx & 127; }
      const int gn = n0 + n, gk2 = k0 + kk;
      rb[e] = (gn < q.N && gk2 < ke)
                  ? (q.b_trans ? q.B[static_cast<size_t>(gn) * q.ldb + gk2]
                               : q.B[static_cast<size_t>(gk2) * q.ldb + gn])
                  : 0.0;
    }
  };
  auto store_slice = [&](int buf) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int idx = tid + e * GEMM_THREADS;
      int m, k;
      if (q.a_trans) { k = idx >> 7; m = idx & 127; } else { m = idx >> 4; k = idx & 15; }
      As[buf][k][m] = ra[e];
      int n, kk;
      if (q.b_trans) { n = idx >> 4; kk = idx & 15; } else { kk = idx >> 7; n = idx & 127; }
      Bs[buf][kk][n] = rb[e];
    }
  };

  if (kb < ke) {
    load_slice(kb);
    store_slice(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = kb; k0 < ke; k0 += TK) {
      const bool more = k0 + TK < ke;
      if (more) load_slice(k0 + TK);
#pragma unroll
      for (int k = 0; k < TK; ++k) {
        double a[8], b[8];
        const double2* ap = reinterpret_cast<const double2*>(&As[buf][k][0]);
        const double2* bp = reinterpret_cast<const double2*>(&Bs[buf][k][0]);
        double2 a0 = ap[ty * 2], a1 = ap[ty * 2 + 1], a2 = ap[32 + ty * 2], a3 = ap[32 + ty * 2 + 1];
        double2 b0 = bp[tx * 2], b1 = bp[tx * 2 + 1], b2 = bp[32 + tx * 2], b3 = bp[32 + tx * 2 + 1];
        a[0] = a0.x; a[1] = a0.y; a[2] = a1.x; a[3] = a1.y;
        a[4] = a2.x; a[5] = a2.y; a[6] = a3.x; a[7] = a3.y;
        b[0] = b0.x; b[1] = b0.y; b[2] = b1.x; b[3] = b1.y;
        b[4] = b2.x; b[5] = b2.y; b[6] = b3.x; b[7] = b3.y;
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
      }
      if (more) {
        store_slice(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }

  // epilogue: rows {ty*4..ty*4+3, 64+ty*4..}, columns {tx*4..tx*4+3, 64+tx*4..}
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (gm >= q.M) continue;
    double* crow = q.C + static_cast<size_t>(gm) * q.ldc;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (gn >= q.N) continue;
      const double v = q.alpha * acc[i][j];
      crow[gn] = (q.beta == 0.0) ? v : fma(q.beta, crow[gn], v);
    }
  }
}

}  // namespace chol
}  // namespace gptq
