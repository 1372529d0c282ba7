// fp64 pipeline from the accumulated Hessian to G, the upper triangular U
// with U^T U = (H + lambda I)^-1  (dingiv.github.io "量化" page, section
// GPTQ: all updates go through the Cholesky factor of H^-1, chosen there for
// numerical stability of a near-singular H).
//
// Route: with J the order-reversing permutation, factor A = J H' J = L L^T
// and form M = L^-1; then H' = V V^T with V = J L J upper triangular and
// G = V^-1 = J M J.  One Cholesky (d^3/3 flops) and one triangular inverse
// (d^3/3), no explicit H'^-1.
//
// Blocked right-looking sweep over NB = 128 column blocks k, with M built
// in the same sweep (block forward substitution on the identity) and kept
// transposed (Mt = M^T, upper block triangle):
//   leaf(k)  one CTA factors the diagonal block A_kk = L_kk L_kk^T and forms
//            X_kk = L_kk^-1 in registers (column sweep, 4x4 tiles/thread);
//   P_k      L_ik = A_ik X_kk^T (rows below), Mt[:k, k] <- Mt[:k, k] X_kk^T;
//   U_k      A_ij -= L_ik L_jk^T on the lower tiles (i, j > k) and
//            Mt[:k+1, i] -= Mt[:k+1, k] L_ik^T for the rows i > k; the CTA
//            that computes the next diagonal tile then runs leaf(k+1), so the
//            serial leaf hides behind the rest of the update.
// Every product is an "NT" GEMM (both operands row-major along K) on the
// fp64 MMA path (mma.sync m8n8k4 f64), staged by cp.async through a 3-deep
// ring of padded shared-memory tiles.
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


// ------------------------------------------------------------- cp.async
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }


// ------------------------------------------------------------------ leaf
// Factor the n x n (n <= NB, n % 8 == 0) diagonal block at A (leading dim
// lda) and write X = L^-1: row-major to Xout (NB x NB, zero above the
// diagonal) and transposed to Mt (leading dim ldm; zero below the diagonal
// there).  One CTA of 32 warps; the lower triangle is cut into 4x4 tiles
// held in registers: warp w owns tile row w and lane l the tile in column l
// (lanes right of the diagonal idle), which keeps the per-step code small
// enough to stay in the instruction cache.  The sweep takes 4 columns per
// step J:
//   1. the step's 4x4 diagonal tile was handed over by its owner and
//      factored once into X4 = chol(D)^-1;
//   2. lane J's tiles below the diagonal form L = A X4^T (and then hold M,
//      starting from 0); row J's tiles left of it rescale M_J <- X4 M_J; all
//      of these go to Vt (V transposed, 4 x NB);
//   3. every tile below the step does t -= V_i V_x^T: the row operand is one
//      broadcast per warp, the column operand a contiguous per-lane read.
//      The owner of the next diagonal tile updates and factors it first.
// Each position holds A's value until its columns are eliminated and M's
// value afterwards, so one sweep yields M = L^-1.  A non-positive or
// non-finite pivot records the original-order column d-1-(gcol0+j) in
// *bad_pivot (first failure only) and the sweep goes on.
constexpr int LEAF_THREADS = 1024;  // 32 warps: one tile row each
constexpr int LSLOTS = 1;
constexpr int TS = NB + 2;   // staging row stride (doubles)

// In place on a 4x4 tile (row-major, lower part read): Cholesky D = L4 L4^T,
// then L4 -> X4 = L4^-1 (lower, upper part zeroed).  Row i of X is formed
// left to right, so each l_ij is read before it is overwritten.
__device__ __forceinline__ void chol_inv4_inplace(double (&a)[16], int col0, int d,
                                                  long long* bad_pivot) {
  double iv[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    double p = a[5 * c];
#pragma unroll
    for (int k = 0; k < c; ++k) p = fma(-a[4 * c + k], a[4 * c + k], p);
    if (!(p > 0.0 && isfinite(p)))
      atomicCAS(reinterpret_cast<unsigned long long*>(bad_pivot),
                static_cast<unsigned long long>(-1ll),
                static_cast<unsigned long long>(d - 1 - (col0 + c)));
    iv[c] = rsqrt(p);
    a[5 * c] = p * iv[c];
#pragma unroll
    for (int i = c + 1; i < 4; ++i) {
      double t = a[4 * i + c];
#pragma unroll
      for (int k = 0; k < c; ++k) t = fma(-a[4 * i + k], a[4 * c + k], t);
      a[4 * i + c] = t * iv[c];
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < i; ++j) {
      double t = 0.0;  // sum_{k=j}^{i-1} l_ik x_kj  (x_jj = iv[j], rows k < i already X)
#pragma unroll
      for (int k = j; k < i; ++k) t = fma(a[4 * i + k], (k == j) ? iv[j] : a[4 * k + j], t);
      a[4 * i + j] = -iv[i] * t;
    }
#pragma unroll
    for (int j = i + 1; j < 4; ++j) a[4 * i + j] = 0.0;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) a[5 * i] = iv[i];
}

__device__ __forceinline__ void dmma_8x8x4(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

__device__ __forceinline__ int leaf_tile_row(int warp, int /*s*/) { return warp; }

__device__ void leaf_factor_invert(const double* __restrict__ A, long long lda, int n,
                                   double* __restrict__ Xout, double* __restrict__ Mt,
                                   long long ldm, long long* __restrict__ bad_pivot, int gcol0,
                                   int d, double* __restrict__ sm) {
  double* Vt = sm;             // 4 x NB
  double* Xs = Vt + 4 * NB;    // X4 of the current step
  double* Dg = Xs + 16;        // the next diagonal tile, handed to its factorization
  double* T = Dg + 16;         // NB x TS staging of the whole block
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  {  // the block's rows into shared memory, 16-byte chunks in flight at once
    const int cpr = n / 2;
    for (int c = tid; c < n * cpr; c += LEAF_THREADS) {
      const int i = c / cpr, x = (c - i * cpr) * 2;
      cp_async16(smem_u32(T + i * TS + x), A + static_cast<long long>(i) * lda + x, 16);
    }
    cp_async_commit();
    cp_async_wait<0>();
  }
  __syncthreads();
  const int nt = n / 4;  // tile rows/columns in use
  double r[LSLOTS][16];
#pragma unroll
  for (int s = 0; s < LSLOTS; ++s) {
    const int bi = leaf_tile_row(warp, s);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int i = 4 * bi + (e >> 2), x = 4 * lane + (e & 3);
      r[s][e] = (bi < nt && x <= i) ? T[i * TS + x] : 0.0;
    }
  }
  // the 4x4 diagonal tile at (j, j) went to Dg; factor it once into Xs
  auto factor_diag = [&](int j) {
    double t[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) t[e] = Dg[e];
    chol_inv4_inplace(t, gcol0 + 4 * j, d, bad_pivot);
#pragma unroll
    for (int e = 0; e < 16; ++e) Xs[e] = t[e];
  };
  if (warp == 0 && lane == 0) {  // step 0's diagonal tile is final already
#pragma unroll
    for (int e = 0; e < 16; ++e) Dg[e] = r[0][e];
    factor_diag(0);
  }
  double* Cs = T + NB * TS;   // raw column-block values of the step, NB x 4
  for (int J = 0; J < nt; ++J) {
    __syncthreads();  // X4 of step J is in Xs; the last update's reads of Vt are done
    const double* X4 = Xs;  // read through shared memory (a broadcast) to save registers
    // (warp-uniform branches; lane J's tile travels by shuffle)
    constexpr unsigned FULL = 0xffffffffu;
#pragma unroll
    for (int s = 0; s < LSLOTS; ++s) {
      const int bi = leaf_tile_row(warp, s);
      if (bi >= nt) continue;
      if (bi > J) {  // stage lane J's raw values (column block J); M starts at 0 there
        double mine = 0.0;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const double v = __shfl_sync(FULL, r[s][e], J);
          if (lane == e) mine = v;
        }
        if (lane < 16) Cs[(4 * bi + (lane >> 2)) * 4 + (lane & 3)] = mine;
        const bool z = lane == J;
#pragma unroll
        for (int e = 0; e < 16; ++e) r[s][e] = z ? 0.0 : r[s][e];
      } else if (bi == J) {  // the diagonal tile becomes X4; row block J: M_J <- X4 M_J
        double m[16];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            double t = 0.0;
#pragma unroll
            for (int bb = 0; bb <= a; ++bb) t = fma(X4[4 * a + bb], r[s][4 * bb + c], t);
            m[4 * a + c] = t;
          }
        const bool diag = lane == J, left = lane < J;
#pragma unroll
        for (int e = 0; e < 16; ++e) r[s][e] = diag ? X4[e] : (left ? m[e] : r[s][e]);
        if (lane <= J) {
#pragma unroll
          for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < 4; ++c) Vt[a * NB + 4 * lane + c] = r[s][4 * a + c];
        }
      }
    }
    __syncthreads();  // the step's column block is staged
    // L = A X4^T for every row below the step: two outputs per thread
    for (int o = tid; o < 2 * n; o += LEAF_THREADS) {
      const int i = o >> 1, c0 = 2 * (o & 1);
      if (i <= 4 * J + 3) continue;
      const double2 ra = *reinterpret_cast<const double2*>(Cs + i * 4);
      const double2 rb = *reinterpret_cast<const double2*>(Cs + i * 4 + 2);
      auto lrow = [&](int c, double x0, double x1, double x2, double x3) {
        double t = ra.x * x0;
        t = fma(ra.y, x1, t);
        t = fma(rb.x, x2, t);
        t = fma(rb.y, x3, t);
        Vt[c * NB + i] = t;
      };
      if (c0 == 0) {
        lrow(0, X4[0], X4[1], X4[2], X4[3]);
        lrow(1, X4[4], X4[5], X4[6], X4[7]);
      } else {
        lrow(2, X4[8], X4[9], X4[10], X4[11]);
        lrow(3, X4[12], X4[13], X4[14], X4[15]);
      }
    }
    __syncthreads();  // Vt is complete
    // t -= V_i V_x^T for every tile row below the step.  The owner of the
    // next diagonal tile hands it over (Dg) and factors it after its rows.
    const int Jn = J + 1;
    bool owner = false;
#pragma unroll
    for (int s = 0; s < LSLOTS; ++s) {
      const int bi = leaf_tile_row(warp, s);
      if (bi >= nt || bi <= J) continue;
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const double2* pv = reinterpret_cast<const double2*>(Vt + bb * NB + 4 * bi);
        const double2* px = reinterpret_cast<const double2*>(Vt + bb * NB + 4 * lane);
        const double2 v0 = pv[0], v1 = pv[1], x0 = px[0], x1 = px[1];
        const double vi[4] = {v0.x, v0.y, v1.x, v1.y};
        const double vx[4] = {x0.x, x0.y, x1.x, x1.y};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) r[s][4 * a + c] = fma(-vi[a], vx[c], r[s][4 * a + c]);
      }
      if (bi == Jn && lane == Jn) {
        owner = true;
#pragma unroll
        for (int e = 0; e < 16; ++e) Dg[e] = r[s][e];
      }
    }
    if (owner) factor_diag(Jn);
  }
  __syncthreads();  // everyone is done with T's input values
#pragma unroll
  for (int s = 0; s < LSLOTS; ++s) {
    const int bi = leaf_tile_row(warp, s);
    if (bi >= nt || lane > bi) continue;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int i = 4 * bi + (e >> 2), x = 4 * lane + (e & 3);
      if (x <= i) T[i * TS + x] = r[s][e];
    }
  }
  __syncthreads();
  // coalesced writes: X row-major (zero above), M^T into the diagonal block
  for (int idx = tid; idx < NB * NB / 2; idx += LEAF_THREADS) {
    const int i = (2 * idx) / NB, x = 2 * idx - i * NB;
    const double v0 = (x <= i && i < n) ? T[i * TS + x] : 0.0;
    const double v1 = (x + 1 <= i && i < n) ? T[i * TS + x + 1] : 0.0;
    reinterpret_cast<double2*>(Xout)[idx] = make_double2(v0, v1);
  }
  for (int idx = tid; idx < n * n; idx += LEAF_THREADS) {
    const int row = idx / n, col = idx - row * n;  // Mt[row][col] = M[col][row]
    Mt[static_cast<long long>(row) * ldm + col] = (row <= col) ? T[col * TS + row] : 0.0;
  }
}

// One CTA factors the diagonal block at (off, off) of A: X -> Xout, M^T -> Mt.
__global__ void __launch_bounds__(LEAF_THREADS, 1)
leaf_kernel(double* __restrict__ A, double* __restrict__ Mt, double* __restrict__ Xout, int d,
            int off, int n, long long* __restrict__ bad_pivot) {
  extern __shared__ __align__(16) double lsm[];
  const long long o = off;
  leaf_factor_invert(A + o * d + o, d, n, Xout, Mt + o * d + o, d, bad_pivot, off, d, lsm);
}

// ------------------------------------------------------------ NT DGEMM
// C[m][n] = alpha * sum_k A[m][k] B[n][k] + beta * C[m][n]  for up to MAXP
// problems per launch.  TM x 128 tile per CTA, 8 warps in a WGM x (8/WGM)
// grid, each warp an (MI*8) x (NI*8) block of m8n8k4 fp64 MMAs.  A and B
// slices of 16 along K are copied by cp.async (16-byte chunks, zero fill
// outside the matrix) into [row][k] tiles padded to 20 doubles per row, so
// both the copies and the fragment reads are free of bank conflicts.
constexpr int TN = 128, TK = 16, LDS = TK + 4, GSTAGES = 3;
constexpr int GEMM_THREADS = 256;
constexpr int MAXP = 64;

struct GemmProblem {
  const double* A;
  const double* B;
  double* C;
  long long lda, ldb, ldc;
  int M, N, K;
  int lower_only;  // square problem: only tiles with tile_n <= tile_m
  double alpha, beta;
};

struct GemmBatch {
  int count;
  int tile_start[MAXP + 1];
  GemmProblem p[MAXP];
};

template <int TM>
constexpr int gemm_smem() {
  return GSTAGES * (TM + TN) * LDS * 8;
}
constexpr int LEAF_SMEM = (4 * NB + 32 + NB * TS + NB * 4) * 8;



template <int TM, int WGM>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
dgemm_nt_kernel(const __grid_constant__ GemmBatch batch) {
  constexpr int WGN = 8 / WGM;
  constexpr int WM = TM / WGM, WN = TN / WGN;
  constexpr int MI = WM / 8, NI = WN / 8;
  extern __shared__ __align__(16) double gsm[];
  double* As = gsm;                              // GSTAGES x TM x LDS
  double* Bs = gsm + GSTAGES * TM * LDS;         // GSTAGES x TN x LDS

  const int bid = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp / WGN, wn = warp % WGN;
  const int total = batch.tile_start[batch.count];
  // Static persistent schedule: CTA c takes tiles c, c + grid, ...
  int t = bid;
  const int step = static_cast<int>(gridDim.x);

  struct Tile { const GemmProblem* q; int m0, n0, ns; };
  auto decode = [&](int tt) {
    Tile T;
    int pi = 0;
    while (pi + 1 < batch.count && batch.tile_start[pi + 1] <= tt) ++pi;
    const GemmProblem& q = batch.p[pi];
    const int lt = tt - batch.tile_start[pi];
    int tm_i, tn_i;
    if (q.lower_only) {
      int rr = static_cast<int>((sqrt(8.0 * lt + 1.0) - 1.0) * 0.5);
      while ((rr + 1) * (rr + 2) / 2 <= lt) ++rr;
      while (rr * (rr + 1) / 2 > lt) --rr;
      tm_i = rr;
      tn_i = lt - rr * (rr + 1) / 2;
    } else {
      const int tn = (q.N + TN - 1) / TN;
      tm_i = lt / tn;
      tn_i = lt - tm_i * tn;
    }
    T.q = &q; T.m0 = tm_i * TM; T.n0 = tn_i * TN; T.ns = (q.K + TK - 1) / TK;
    return T;
  };
  auto issue = [&](const Tile& T, int slice, int stage) {
    const GemmProblem& q = *T.q;
    const int k0 = slice * TK;
    const uint32_t sa = smem_u32(As + stage * TM * LDS);
    const uint32_t sb = smem_u32(Bs + stage * TN * LDS);
    for (int c = tid; c < (TM + TN) * (TK / 2); c += GEMM_THREADS) {
      const bool isA = c < TM * (TK / 2);
      const int cc = isA ? c : c - TM * (TK / 2);
      const int row = cc >> 3, kc = (cc & 7) * 2;
      const int grow = (isA ? T.m0 : T.n0) + row;
      const int lim = isA ? q.M : q.N;
      const double* base = isA ? q.A : q.B;
      const long long ld = isA ? q.lda : q.ldb;
      const bool ok = grow < lim && k0 + kc < q.K;
      const double* src = ok ? base + static_cast<long long>(grow) * ld + k0 + kc : base;
      const uint32_t dst = (isA ? sa : sb) + (row * LDS + kc) * 8;
      cp_async16(dst, src, ok ? 16 : 0);
    }
  };
  auto prologue = [&](const Tile& T, int g0) {
#pragma unroll
    for (int st = 0; st < GSTAGES - 1; ++st) {
      if (st < T.ns) issue(T, st, (g0 + st) % GSTAGES);
      cp_async_commit();
    }
    const GemmProblem& q = *T.q;
    if (q.beta != 0.0) {  // pull this tile of C into L2 for the epilogue
      for (int c = tid; c < TM * 8; c += GEMM_THREADS) {
        const int row = c >> 3, col = T.n0 + (c & 7) * 16;
        if (T.m0 + row < q.M && col < q.N)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(q.C + static_cast<long long>(T.m0 + row) * q.ldc + col));
      }
    }
  };

  int g = 0;  // running slice count: stage of a slice = its running index mod GSTAGES
  Tile cur;
  if (t < total) { cur = decode(t); prologue(cur, g); }
  while (t < total) {
    const GemmProblem& q = *cur.q;
    double acc[MI][NI][2];
#pragma unroll
    for (int i = 0; i < MI; ++i)
#pragma unroll
      for (int j = 0; j < NI; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    for (int sl = 0; sl < cur.ns; ++sl) {
      cp_async_wait<GSTAGES - 2>();
      __syncthreads();
      if (sl + GSTAGES - 1 < cur.ns) issue(cur, sl + GSTAGES - 1, (g + sl + GSTAGES - 1) % GSTAGES);
      cp_async_commit();
      const int stg = (g + sl) % GSTAGES;
      const double* a_s = As + stg * TM * LDS + (wm * WM + (lane >> 2)) * LDS + (lane & 3);
      const double* b_s = Bs + stg * TN * LDS + (wn * WN + (lane >> 2)) * LDS + (lane & 3);
#pragma unroll
      for (int kk = 0; kk < TK / 4; ++kk) {
        double af[MI], bf[NI];
#pragma unroll
        for (int i = 0; i < MI; ++i) af[i] = a_s[i * 8 * LDS + kk * 4];
#pragma unroll
        for (int j = 0; j < NI; ++j) bf[j] = b_s[j * 8 * LDS + kk * 4];
#pragma unroll
        for (int i = 0; i < MI; ++i)
#pragma unroll
          for (int j = 0; j < NI; ++j) dmma_8x8x4(acc[i][j][0], acc[i][j][1], af[i], bf[j]);
      }
    }
    g += cur.ns;
    // start the next tile's copies before this tile's epilogue
    const int next = t + step;
    __syncthreads();  // all warps are done reading the stages
    Tile nxt;
    if (next < total) { nxt = decode(next); prologue(nxt, g); }

    // epilogue: lane holds C[8i + lane/4][8j + 2(lane%4) + {0,1}] of its warp
    // block; C is read two row groups at a time so the loads overlap.
#pragma unroll
    for (int i0 = 0; i0 < MI; i0 += 2) {
      double2 old[2][NI];
#pragma unroll
      for (int ii = 0; ii < 2; ++ii)
#pragma unroll
        for (int j = 0; j < NI; ++j) {
          old[ii][j] = make_double2(0.0, 0.0);
          const int gm = cur.m0 + wm * WM + 8 * (i0 + ii) + (lane >> 2);
          const int gn = cur.n0 + wn * WN + 8 * j + 2 * (lane & 3);
          if (q.beta != 0.0 && i0 + ii < MI && gm < q.M && gn < q.N) {
            const double* cp = q.C + static_cast<long long>(gm) * q.ldc + gn;
            old[ii][j] = (gn + 1 < q.N) ? *reinterpret_cast<const double2*>(cp)
                                        : make_double2(*cp, 0.0);
          }
        }
#pragma unroll
      for (int ii = 0; ii < 2; ++ii) {
        if (i0 + ii >= MI) continue;
        const int gm = cur.m0 + wm * WM + 8 * (i0 + ii) + (lane >> 2);
        if (gm >= q.M) continue;
        double* crow = q.C + static_cast<long long>(gm) * q.ldc;
#pragma unroll
        for (int j = 0; j < NI; ++j) {
          const int gn = cur.n0 + wn * WN + 8 * j + 2 * (lane & 3);
          if (gn >= q.N) continue;
          const double c0 = fma(q.beta, old[ii][j].x, q.alpha * acc[i0 + ii][j][0]);
          const double c1 = fma(q.beta, old[ii][j].y, q.alpha * acc[i0 + ii][j][1]);
          if (gn + 1 < q.N) *reinterpret_cast<double2*>(crow + gn) = make_double2(c0, c1);
          else crow[gn] = c0;
        }
      }
    }
    t = next;
    cur = nxt;
  }
  cp_async_wait<0>();
}

// G[i][j] = M[d-1-i][d-1-j] = Mt[d-1-j][d-1-i] (fp32) for i <= j, 0 below.
// 32 x 32 tiles transposed through shared memory.
__global__ void write_g_kernel(const double* __restrict__ Mt, int d, float* __restrict__ G) {
  __shared__ double tile[32][33];
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  // rows of Mt: d-1-j for j in [j0, j0+32); columns: d-1-i for i in [i0, i0+32)
  for (int yy = ty; yy < 32; yy += 8) {
    const int j = j0 + yy, i = i0 + tx;
    double v = 0.0;
    if (j < d && i < d && i <= j) v = Mt[static_cast<long long>(d - 1 - j) * d + (d - 1 - i)];
    tile[yy][tx] = v;
  }
  __syncthreads();
  for (int yy = ty; yy < 32; yy += 8) {
    const int i = i0 + yy, j = j0 + tx;
    if (i < d && j < d) G[static_cast<long long>(i) * d + j] = static_cast<float>(tile[tx][yy]);
  }
}

}  // namespace chol
}  // namespace gptq
