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
//            X_kk = L_kk^-1, in 16-column panels held in shared memory;
//   P_k      L_ik = A_ik X_kk^T (rows below), Mt[:k, k] <- Mt[:k, k] X_kk^T;
//   D_k      the next diagonal block, A_{k+1,k+1} -= L_{k+1,k} L_{k+1,k}^T,
//            then leaf(k+1), both on a second stream;
//   U_k      A_ij -= L_ik L_jk^T on the other lower tiles (i, j > k) and
//            Mt[:k+1, i] -= Mt[:k+1, k] L_ik^T for the rows i > k, on all
//            SMs but two, so that D_k and the serial leaf run beside it.
// The trailing updates are lazy over windows of m panels (window_panels):
// inside a window U_k and D_k apply panel k only to the window's remaining
// columns; the window's last panel applies all m panels (K = 128 m) to
// everything right of the window.  Same sums, regrouped, so most of the
// 2/3 d^3 flops run with an m times longer K per output tile and 1/m of the
// trailing matrix's read-modify-write traffic.
// Every product is an "NT" GEMM (both operands row-major along K) on the
// fp64 MMA path (mma.sync m8n8k4 f64), staged by cp.async through a 3-deep
// ring of padded shared-memory tiles.
#pragma once

#include "common.cuh"

namespace gptq {
namespace chol {

constexpr int NB = 128;  // panel / leaf width

// Panels per lazy-update window (see gptq_prepare_hinv): the window's last
// panel applies all of them to the trailing matrix at once (K = 128 m).
#ifndef GPTQ_WINDOW_PANELS
#define GPTQ_WINDOW_PANELS 8
#endif
inline int window_panels(int d) { return d >= 8192 ? GPTQ_WINDOW_PANELS : 1; }

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
  const double lam = stats[0];
  // rows grid-strided: gridDim.y is capped at 65535 and d may be 65536
  for (int i = blockIdx.y; i < d; i += gridDim.y) {
    const float* hrow = H + static_cast<size_t>(d - 1 - i) * d;
    double* arow = A + static_cast<size_t>(i) * d;
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j <= i; j += gridDim.x * blockDim.x) {
      double v = static_cast<double>(hrow[d - 1 - j]);
      if (j == i) v = (v == 0.0) ? 1.0 : v + lam;
      arow[j] = v;
    }
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
// d) and form X = L^-1.  Output: X row-major to Xout (NB x NB, zero above
// the diagonal, identity past n) and X^T into the block of Mt (leading dim
// d; zero below the diagonal there).
//
// One CTA of 8 warps keeps the whole block in shared memory S (identity past
// n, zero above the diagonal).  With the block cut into 16 x 16 blocks
// (i, j), the sweep takes the 16-column panels p = 0..7:
//   (i)   one warp factors the diagonal block A_pp = L_pp L_pp^T in
//         registers (lane = row; pivots and L entries travel by shuffle)
//         and inverts it, X_pp = L_pp^-1 (lane = column), into Xd[p];
//   (ii)  L_ip = A_ip X_pp^T for the blocks below the diagonal block, and
//         X_pj = X_pp R_pj for the blocks left of it (one warp per block);
//   (iii) A_ik -= L_ip L_kp^T for p < k <= i, and R_ij -= L_ip X_pj for
//         i > p, j <= p.  R_ij starts at 0 and collects -sum_{k<p} L_ik X_kj,
//         so X_ij = X_ii R_ij once panel i is reached (block forward
//         substitution on the identity).
// R_ij, and then X_ij, live transposed in S's strict upper blocks (block
// (j, i)), which is the layout of X^T that Mt wants.  Steps (ii) and (iii)
// run on the fp64 MMA (m8n8k4), one 16 x 16 block per warp job.  In (iii)
// warp 0 updates the next diagonal block first and factors it while the
// other warps finish the rest, so the serial part overlaps the updates.
// Two barriers per panel.  A non-positive or non-finite pivot records the
// original-order column d-1-(gcol0+j) in *bad_pivot (first failure only)
// and the sweep goes on.
constexpr int LEAF_THREADS = 256;
constexpr int LS = NB + 4;       // S row stride (doubles): fragment loads in two wavefronts
constexpr int XDS = 20;          // Xd row stride (doubles)
constexpr int LEAF_SMEM = (NB * LS + 8 * 16 * XDS) * 8;

__device__ __forceinline__ void dmma_8x8x4(double& c0, double& c1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(c0), "+d"(c1)
               : "d"(a), "d"(b));
}

// 16 x 16 x 16 block product on one warp, acc += A B, with A(r, q) and
// B(q, c) given by accessors.  acc[rt][ct][e] is the m8n8 fragment element
// (8 rt + lane/4, 8 ct + 2 (lane%4) + e).
template <class FA, class FB>
__device__ __forceinline__ void blk16_mma(double (&acc)[2][2][2], FA fa, FB fb, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int k4 = 0; k4 < 4; ++k4) {
    const double a0 = fa(g, 4 * k4 + t), a1 = fa(8 + g, 4 * k4 + t);
    const double b0 = fb(4 * k4 + t, g), b1 = fb(4 * k4 + t, 8 + g);
    dmma_8x8x4(acc[0][0][0], acc[0][0][1], a0, b0);
    dmma_8x8x4(acc[0][1][0], acc[0][1][1], a0, b1);
    dmma_8x8x4(acc[1][0][0], acc[1][0][1], a1, b0);
    dmma_8x8x4(acc[1][1][0], acc[1][1][1], a1, b1);
  }
}

// (i) on one warp: factor the diagonal block p of S, A_pp = L_pp L_pp^T, and
// write X_pp = L_pp^-1 row-major (stride XDS, zero above the diagonal) to
// Xd[p].  Lane c holds column c of the block in registers (lanes 16..31
// shadow lanes 0..15), unscaled during the sweep.  At pivot j every lane
// receives the pivot and column j by shuffle (issued together) and scales
// what it receives by 1/sqrt(pivot); lane c > j then updates its column,
// a_ic -= l_ij l_cj.  The serial chain per pivot is one shuffle, rsqrt, one
// multiply and one FMA.  After the sweep each lane scales its own column
// once.  Branch-free; a bad pivot is reported once, after the sweep.
__device__ __noinline__ void leaf_diag_factor(const double* __restrict__ S,
                                              double* __restrict__ Xd, int p, int n,
                                              int gcol0, int d, long long* bad_pivot,
                                              int lane) {
  constexpr unsigned FULL = 0xffffffffu;
  const int c0 = 16 * p, c = lane & 15;
  const double* D = S + c0 * LS + c0;
  double col[16], rme = 0.0;
#pragma unroll
  for (int i = 0; i < 16; ++i) col[i] = (i >= c) ? D[i * LS + c] : 0.0;
  unsigned badmask = 0u;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    double aij[16];
    const double piv = __shfl_sync(FULL, col[j], j);
#pragma unroll
    for (int i = j + 1; i < 16; ++i) aij[i] = __shfl_sync(FULL, col[i], j);
    badmask |= (piv > 0.0 && isfinite(piv)) ? 0u : (1u << j);
    const double r = rsqrt(piv);
    rme = (c == j) ? r : rme;
    // l_cj becomes known at i == c; rows above c see l_cj = 0 and stay put
    double lcj = 0.0;
#pragma unroll
    for (int i = j + 1; i < 16; ++i) {
      const double lij = aij[i] * r;
      lcj = (c == i) ? lij : lcj;
      col[i] = fma(-lij, lcj, col[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) col[i] = (i >= c) ? col[i] * rme : 0.0;  // L's column c
  // column c of X = L^-1: x_kc = -(sum_{m<k} l_km x_mc) / l_kk, right-looking
  double x[16], acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.0;
#pragma unroll
  for (int m = 0; m < 16; ++m) {
    // row entries l_km (k > m) from lane m, fetched before x_m is needed
    double lkm[16];
#pragma unroll
    for (int k = m + 1; k < 16; ++k) lkm[k] = __shfl_sync(FULL, col[k], m);
    const double rm = __shfl_sync(FULL, rme, m);
    x[m] = (m == c) ? rm : ((m > c) ? -acc[m] * rm : 0.0);
#pragma unroll
    for (int k = m + 1; k < 16; ++k) acc[k] = fma(lkm[k], x[m], acc[k]);
  }
  if (lane < 16) {
    double* xo = Xd + p * 16 * XDS;
#pragma unroll
    for (int k = 0; k < 16; ++k) xo[k * XDS + c] = x[k];
  }
  if (lane == 0 && badmask) {
    const int j = __ffs(badmask) - 1;
    if (c0 + j < n)
      atomicCAS(reinterpret_cast<unsigned long long*>(bad_pivot),
                static_cast<unsigned long long>(-1ll),
                static_cast<unsigned long long>(d - 1 - (gcol0 + c0 + j)));
  }
}

__global__ void __launch_bounds__(LEAF_THREADS, 1)
leaf_kernel(const double* __restrict__ A, double* __restrict__ Mt, double* __restrict__ Xout,
            int d, int off, int n, long long* __restrict__ bad_pivot) {
  extern __shared__ __align__(16) double lsm[];
  double* S = lsm;
  double* Xd = lsm + NB * LS;
  const double* Ab = A + static_cast<long long>(off) * d + off;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;

  {  // rows r < n up to the end of their diagonal 16-block, in 16-byte chunks
    for (int r = warp; r < n; r += LEAF_THREADS / 32) {
      const int cend = min(n, 16 * (r / 16 + 1));
      for (int c = 2 * lane; c < cend; c += 64)
        cp_async16(smem_u32(S + r * LS + c), Ab + static_cast<long long>(r) * d + c, 16);
    }
    cp_async_commit();
    // meanwhile zero the strictly-upper 16-blocks (R starts at 0 there) and
    // make rows past n identity rows; 16-column segments, 8 per row
    for (int sg = tid; sg < NB * 8; sg += LEAF_THREADS) {
      const int r = sg >> 3, b = sg & 7;
      if (r >= n || b > (r >> 4)) {
        double2* z = reinterpret_cast<double2*>(S + r * LS + 16 * b);
#pragma unroll
        for (int i = 0; i < 8; ++i) z[i] = make_double2(0.0, 0.0);
        if (r >= n && b == (r >> 4)) S[r * LS + r] = 1.0;
      }
    }
    cp_async_wait<0>();
  }
  __syncthreads();
  if (warp == 0) leaf_diag_factor(S, Xd, 0, n, off, d, bad_pivot, lane);

  // fragment element (r, c) of a 16 x 16 block, r = 8 rt + g, c = 8 ct + 2 t4 + e
  auto frag_rc = [=](int rt, int ct, int e, int& r, int& c) {
    r = 8 * rt + g;
    c = 8 * ct + 2 * t4 + e;
  };
  for (int p = 0; p < 8; ++p) {
    __syncthreads();  // X_pp is in Xd[p]; the previous panel's updates are done
    const double* Xp = Xd + p * 16 * XDS;
    if (warp < 7) {  // (ii): 7 - p blocks below, p blocks to the left
      double acc[2][2][2] = {};
      if (warp < 7 - p) {  // L_ip = A_ip X_pp^T, in place
        double* blk = S + 16 * (p + 1 + warp) * LS + 16 * p;
        blk16_mma(acc, [=](int r, int q) { return blk[r * LS + q]; },
                  [=](int q, int c) { return Xp[c * XDS + q]; }, lane);
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
          for (int ct = 0; ct < 2; ++ct)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              int r, c;
              frag_rc(rt, ct, e, r, c);
              blk[r * LS + c] = acc[rt][ct][e];
            }
      } else {  // X_pj = X_pp R_pj; R_pj^T sits at block (j, p)
        double* bt = S + 16 * (warp - (7 - p)) * LS + 16 * p;   // R_pj(q, c) = bt[c * LS + q]
        blk16_mma(acc, [=](int r, int q) { return Xp[r * XDS + q]; },
                  [=](int q, int c) { return bt[c * LS + q]; }, lane);
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
          for (int ct = 0; ct < 2; ++ct)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              int r, c;
              frag_rc(rt, ct, e, r, c);
              bt[c * LS + r] = acc[rt][ct][e];
            }
        // X_pj is final: its rows of Xout (row-major X), two columns per store
        const int j = warp - (7 - p);
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
          for (int ct = 0; ct < 2; ++ct) {
            int r, c;
            frag_rc(rt, ct, 0, r, c);
            *reinterpret_cast<double2*>(Xout + (16 * p + r) * NB + 16 * j + c) =
                make_double2(acc[rt][ct][0], acc[rt][ct][1]);
          }
      }
    }
    __syncthreads();  // L_ip and X_pj are complete
    if (p == 7) break;
    // (iii): A_ik -= L_ip L_kp^T (p < k <= i) and R_ij -= L_ip X_pj (i > p, j <= p)
    auto job_a = [&](int i, int k) {
      double* C = S + 16 * i * LS + 16 * k;
      const double* Li = S + 16 * i * LS + 16 * p;
      const double* Lk = S + 16 * k * LS + 16 * p;
      double acc[2][2][2];
#pragma unroll
      for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int ct = 0; ct < 2; ++ct)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            int r, c;
            frag_rc(rt, ct, e, r, c);
            acc[rt][ct][e] = C[r * LS + c];
          }
      blk16_mma(acc, [=](int r, int q) { return Li[r * LS + q]; },
                [=](int q, int c) { return -Lk[c * LS + q]; }, lane);
#pragma unroll
      for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int ct = 0; ct < 2; ++ct)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            int r, c;
            frag_rc(rt, ct, e, r, c);
            C[r * LS + c] = acc[rt][ct][e];
          }
    };
    auto job_r = [&](int i, int j) {
      double* RT = S + 16 * j * LS + 16 * i;        // R_ij(r, c) = RT[c * LS + r]
      const double* Li = S + 16 * i * LS + 16 * p;
      const double* XT = S + 16 * j * LS + 16 * p;  // X_pj(q, c) = XT[c * LS + q], j < p
      double acc[2][2][2];
#pragma unroll
      for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int ct = 0; ct < 2; ++ct)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            int r, c;
            frag_rc(rt, ct, e, r, c);
            acc[rt][ct][e] = RT[c * LS + r];
          }
      if (j < p)
        blk16_mma(acc, [=](int r, int q) { return Li[r * LS + q]; },
                  [=](int q, int c) { return -XT[c * LS + q]; }, lane);
      else
        blk16_mma(acc, [=](int r, int q) { return Li[r * LS + q]; },
                  [=](int q, int c) { return -Xp[q * XDS + c]; }, lane);
#pragma unroll
      for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int ct = 0; ct < 2; ++ct)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            int r, c;
            frag_rc(rt, ct, e, r, c);
            RT[c * LS + r] = acc[rt][ct][e];
          }
    };
    if (warp == 0) {  // the next diagonal block first, then its factorization
      job_a(p + 1, p + 1);
      __syncwarp();
      leaf_diag_factor(S, Xd, p + 1, n, off, d, bad_pivot, lane);
    } else {
      const int na = (7 - p) * (8 - p) / 2, nr = (7 - p) * (p + 1);
      for (int jb = warp - 1; jb < na - 1 + nr; jb += 7) {
        if (jb < na - 1) {
          int a = jb + 1, k = p + 1;  // pairs (i, k), k = p+1..7, i = k..7; pair 0 is warp 0's
          while (a >= 8 - k) { a -= 8 - k; ++k; }
          job_a(k + a, k);
        } else {
          const int r = jb - (na - 1);
          job_r(p + 1 + r / (p + 1), r % (p + 1));
        }
      }
    }
  }
  __syncthreads();
  // Xout: the diagonal blocks from Xd and zeros above them (the blocks
  // below were written as they were formed); consecutive lanes take
  // consecutive 16-byte pieces of a row
  double2* Xo2 = reinterpret_cast<double2*>(Xout);
  for (int i2 = tid; i2 < NB * NB / 2; i2 += LEAF_THREADS) {
    const int r = i2 >> 6, c = (i2 & 63) * 2;
    const int br = r >> 4, bc = c >> 4;
    if (bc > br)
      Xo2[i2] = make_double2(0.0, 0.0);
    else if (bc == br)
      Xo2[i2] = *reinterpret_cast<const double2*>(Xd + br * 16 * XDS + (r & 15) * XDS + (c & 15));
  }
  // X^T into the n x n block of Mt: S's strict upper blocks hold it; the
  // diagonal blocks are X_pp^T; zero below the diagonal
  double* Mb = Mt + static_cast<long long>(off) * d + off;
  for (int r = warp; r < n; r += LEAF_THREADS / 32) {
    const int br = r >> 4;
    for (int c = 2 * lane; c < n; c += 64) {
      double v0, v1;
      const int bc = c >> 4;
      if (bc > br) {
        const double2 v = *reinterpret_cast<const double2*>(S + r * LS + c);
        v0 = v.x;
        v1 = v.y;
      } else if (bc == br) {
        const double* xd = Xd + br * 16 * XDS;
        const int a = r & 15, b0 = c & 15;
        v0 = (b0 >= a) ? xd[b0 * XDS + a] : 0.0;
        v1 = (b0 + 1 >= a) ? xd[(b0 + 1) * XDS + a] : 0.0;
      } else {
        v0 = v1 = 0.0;
      }
      *reinterpret_cast<double2*>(Mb + static_cast<long long>(r) * d + c) = make_double2(v0, v1);
    }
  }
}

// ------------------------------------------------------------ NT DGEMM
// C[m][n] = alpha * sum_k A[m][k] B[n][k] + beta * C[m][n]  for up to MAXP
// problems per launch.  A CTA holds NG independent warp groups; each group
// runs its own persistent loop over TM x TNG tiles with NW warps in a
// WGM x (NW/WGM) grid (each warp an (MI*8) x (NI*8) block of m8n8k4 fp64
// MMAs), its own STG-deep ring of shared-memory stages and its own named
// barrier, so one group's epilogue and slice barriers overlap the other
// group's MMAs.  A and B slices of TKG along K are copied by cp.async
// (16-byte chunks, zero fill outside the matrix) into [row][k] tiles padded
// to TKG + 4 doubles per row, so both the copies and the fragment reads are
// free of bank conflicts.
#ifndef GPTQ_DGEMM_TK
#define GPTQ_DGEMM_TK 32
#endif
constexpr int TN = 128, TK = GPTQ_DGEMM_TK, LDS = TK + 4, GSTAGES = 3;
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

template <int TM, int TNG = TN, int NG = 1, int TKG = TK, int STG = GSTAGES>
constexpr int gemm_smem() {
  return NG * STG * (TM + TNG) * (TKG + 4) * 8;
}

// Tiles of a lower_only (square) problem: those whose first column is on
// or left of the tile row's last row, tile_n * TNG <= (tile_m + 1) TM - 1.
// (The kernel decodes this order for TM == TNG and TM == 2 TNG, the shapes
// that lower_only problems are launched with.)
template <int TM, int TNG>
inline int lower_tiles(int M, int N) {
  const int tm = (M + TM - 1) / TM, tn = (N + TNG - 1) / TNG;
  int n = 0;
  for (int r = 0; r < tm; ++r) {
    const int c = ((r + 1) * TM - 1) / TNG + 1;
    n += c < tn ? c : tn;
  }
  return n;
}

// NW warps per group (NW * 32 threads) in a WGM x (NW / WGM) grid.
template <int TM, int WGM, int NW = 8, int TNG = TN, int NG = 1, int TKG = TK,
          int STG = GSTAGES>
__global__ void __launch_bounds__(NG * NW * 32, 1)
dgemm_nt_kernel(const __grid_constant__ GemmBatch batch) {
  constexpr int NTHREADS = NW * 32;  // threads per group
  constexpr int LDS = TKG + 4;       // padded stage row (doubles)
  constexpr int WGN = NW / WGM;
  constexpr int WM = TM / WGM, WN = TNG / WGN;
  constexpr int MI = WM / 8, NI = WN / 8;
  extern __shared__ __align__(16) double gsm[];
  const int grp = NG > 1 ? static_cast<int>(threadIdx.x) / NTHREADS : 0;
  double* As = gsm + grp * STG * (TM + TNG) * LDS;   // STG x TM x LDS
  double* Bs = As + STG * TM * LDS;                   // STG x TNG x LDS
  auto group_sync = [&]() {
    if (NG == 1) __syncthreads();
    else named_bar(1 + grp, NTHREADS);
  };

  const int tid = static_cast<int>(threadIdx.x) - grp * NTHREADS, lane = tid & 31, warp = tid >> 5;
  const int wm = warp / WGN, wn = warp % WGN;
  const int total = batch.tile_start[batch.count];
  // Static persistent schedule: group g of CTA c takes tiles c NG + g, then
  // every NG * grid-th tile after it
  int t = static_cast<int>(blockIdx.x) * NG + grp;
  const int step = static_cast<int>(gridDim.x) * NG;

  // A tile's problem lives in registers (the batch is only read here, once
  // per tile: fields read through a pointer into the parameter block would
  // be reloaded from memory at every use).
  struct Tile {
    const double* A;
    const double* B;
    double* C;
    long long lda, ldb, ldc;
    int M, N, K, m0, n0, ns;
    double alpha, beta;
  };
  auto decode = [&](int tt) {
    int pi = 0;
    while (pi + 1 < batch.count && batch.tile_start[pi + 1] <= tt) ++pi;
    const GemmProblem& q = batch.p[pi];
    const int lt = tt - batch.tile_start[pi];
    int tm_i, tn_i;
    if (q.lower_only && TM == TNG) {  // row r holds r + 1 tiles
      int rr = static_cast<int>((sqrt(8.0 * lt + 1.0) - 1.0) * 0.5);
      while ((rr + 1) * (rr + 2) / 2 <= lt) ++rr;
      while (rr * (rr + 1) / 2 > lt) --rr;
      tm_i = rr;
      tn_i = lt - rr * (rr + 1) / 2;
    } else if (q.lower_only && TM == 2 * TNG) {  // row r holds 2r + 2 tiles (the last may hold fewer)
      int rr = static_cast<int>((sqrt(4.0 * lt + 1.0) - 1.0) * 0.5);
      while ((rr + 1) * (rr + 2) <= lt) ++rr;
      while (rr * (rr + 1) > lt) --rr;
      tm_i = rr;
      tn_i = lt - rr * (rr + 1);
    } else {
      const int tn = (q.N + TNG - 1) / TNG;
      tm_i = lt / tn;
      tn_i = lt - tm_i * tn;
    }
    Tile T;
    T.A = q.A; T.B = q.B; T.C = q.C;
    T.lda = q.lda; T.ldb = q.ldb; T.ldc = q.ldc;
    T.M = q.M; T.N = q.N; T.K = q.K;
    T.alpha = q.alpha; T.beta = q.beta;
    T.m0 = tm_i * TM; T.n0 = tn_i * TNG; T.ns = (q.K + TKG - 1) / TKG;
    return T;
  };
  // Each thread copies APT 16-byte pieces of A and CPT - APT of B per slice,
  // all in the same k column, RSTEP rows apart.
  constexpr int CPT = (TM + TNG) * (TKG / 2) / NTHREADS;
  constexpr int APT = TM * (TKG / 2) / NTHREADS;
  constexpr int RSTEP = NTHREADS / (TKG / 2);
  static_assert(CPT * NTHREADS == (TM + TNG) * (TKG / 2) && APT * NTHREADS == TM * (TKG / 2),
                "the copies must split evenly over the threads");
  const int crow0 = tid / (TKG / 2), ckc = (tid % (TKG / 2)) * 2;
  auto issue = [&](const Tile& T, int slice, int stage) {
    const int k = slice * TKG + ckc;
    const bool kin = k < T.K;
    const uint32_t sa = smem_u32(As + stage * TM * LDS) + (crow0 * LDS + ckc) * 8;
    const uint32_t sb = smem_u32(Bs + stage * TNG * LDS) + (crow0 * LDS + ckc) * 8;
#pragma unroll
    for (int i = 0; i < APT; ++i) {
      const int grow = T.m0 + crow0 + i * RSTEP;
      const bool ok = kin && grow < T.M;
      const double* src = ok ? T.A + static_cast<long long>(grow) * T.lda + k : T.A;
      cp_async16(sa + i * RSTEP * LDS * 8, src, ok ? 16 : 0);
    }
#pragma unroll
    for (int i = 0; i < CPT - APT; ++i) {
      const int grow = T.n0 + crow0 + i * RSTEP;
      const bool ok = kin && grow < T.N;
      const double* src = ok ? T.B + static_cast<long long>(grow) * T.ldb + k : T.B;
      cp_async16(sb + i * RSTEP * LDS * 8, src, ok ? 16 : 0);
    }
  };
  auto prologue = [&](const Tile& T, int g0) {
#pragma unroll
    for (int st = 0; st < STG - 1; ++st) {
      if (st < T.ns) issue(T, st, (g0 + st) % STG);
      cp_async_commit();
    }
    if (T.beta != 0.0) {  // pull this tile of C into L2 for the epilogue
      constexpr int CH = TNG / 16;  // 128-byte pieces per tile row
      for (int c = tid; c < TM * CH; c += NTHREADS) {
        const int row = c / CH, col = T.n0 + (c % CH) * 16;
        if (T.m0 + row < T.M && col < T.N)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(T.C + static_cast<long long>(T.m0 + row) * T.ldc + col));
      }
    }
  };

  int g = 0;  // running slice count: stage of a slice = its running index mod STG
  Tile cur;
  if (t < total) { cur = decode(t); prologue(cur, g); }
  while (t < total) {
    const Tile& q = cur;
    double acc[MI][NI][2];
#pragma unroll
    for (int i = 0; i < MI; ++i)
#pragma unroll
      for (int j = 0; j < NI; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    for (int sl = 0; sl < cur.ns; ++sl) {
      cp_async_wait<STG - 2>();
      group_sync();
      if (sl + STG - 1 < cur.ns) issue(cur, sl + STG - 1, (g + sl + STG - 1) % STG);
      cp_async_commit();
      const int stg = (g + sl) % STG;
      const double* a_s = As + stg * TM * LDS + (wm * WM + (lane >> 2)) * LDS + (lane & 3);
      const double* b_s = Bs + stg * TNG * LDS + (wn * WN + (lane >> 2)) * LDS + (lane & 3);
      // fragments double-buffered: step kk+1's loads are in flight while
      // step kk's MMAs issue
      double af[2][MI], bf[2][NI];
#pragma unroll
      for (int i = 0; i < MI; ++i) af[0][i] = a_s[i * 8 * LDS];
#pragma unroll
      for (int j = 0; j < NI; ++j) bf[0][j] = b_s[j * 8 * LDS];
#pragma unroll
      for (int kk = 0; kk < TKG / 4; ++kk) {
        const int cb = kk & 1;
        if (kk + 1 < TKG / 4) {
#pragma unroll
          for (int i = 0; i < MI; ++i) af[cb ^ 1][i] = a_s[i * 8 * LDS + (kk + 1) * 4];
#pragma unroll
          for (int j = 0; j < NI; ++j) bf[cb ^ 1][j] = b_s[j * 8 * LDS + (kk + 1) * 4];
        }
#pragma unroll
        for (int i = 0; i < MI; ++i)
#pragma unroll
          for (int j = 0; j < NI; ++j) dmma_8x8x4(acc[i][j][0], acc[i][j][1], af[cb][i], bf[cb][j]);
      }
    }
    g += cur.ns;
    // one group: start the next tile's copies before this tile's epilogue;
    // several: after it (the other group's MMAs cover the epilogue, and the
    // next tile's fields are not held in registers across it)
    const int next = t + step;
    group_sync();  // the group's warps are done reading the stages
    Tile nxt;
    if (NG == 1 && next < total) { nxt = decode(next); prologue(nxt, g); }

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
    if (NG > 1 && next < total) { nxt = decode(next); prologue(nxt, g); }
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

// F (fp32, the sweep's order) from the blocks the factor route leaves in
// Mt.  With V = J L J the upper factor of H' = V V^T and G = V^-1:
//   inside a diagonal 128-block b:  F_bb = G_bb = (V_bb)^-1 = J X_kk J,
//     read like G above (Mt's diagonal blocks hold X_kk^T);
//   right of it (i < j, blocks a < b):  F_ab = V_ab G_bb, which is
//     J (L_{>k,k} X_kk) J, left by the factorization in Mt's lower part:
//     F[i][j] = Mt[d-1-i][d-1-j];
//   below the diagonal: 0.
// A 32 x 32 tile never straddles a 128-block boundary.
__global__ void write_f_kernel(const double* __restrict__ Mt, int d, float* __restrict__ F) {
  __shared__ double tile[32][33];
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  if (i0 / NB == j0 / NB) {  // diagonal block: as write_g_kernel
    for (int yy = ty; yy < 32; yy += 8) {
      const int j = j0 + yy, i = i0 + tx;
      double v = 0.0;
      if (j < d && i < d && i <= j) v = Mt[static_cast<long long>(d - 1 - j) * d + (d - 1 - i)];
      tile[yy][tx] = v;
    }
    __syncthreads();
    for (int yy = ty; yy < 32; yy += 8) {
      const int i = i0 + yy, j = j0 + tx;
      if (i < d && j < d) F[static_cast<long long>(i) * d + j] = static_cast<float>(tile[tx][yy]);
    }
    return;
  }
  for (int yy = ty; yy < 32; yy += 8) {
    const int i = i0 + yy, j = j0 + tx;
    if (i >= d || j >= d) continue;
    const float v = (i0 < j0) ? static_cast<float>(Mt[static_cast<long long>(d - 1 - i) * d + (d - 1 - j)])
                              : 0.0f;
    F[static_cast<long long>(i) * d + j] = v;
  }
}

}  // namespace chol
}  // namespace gptq
