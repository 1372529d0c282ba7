// GPTQ column sweep on the GPU (dingiv.github.io "量化" page, section GPTQ):
// fixed left-to-right order, every update through G (the upper Cholesky
// factor of H^-1), blocks of B columns with immediate in-block updates and
// one lazy batched update of the columns to the right after each block.
//
// Per block j0 (block_step_kernel, one CTA per 32 rows):
//   (a) apply the previous block's errors to this block, W -= E_prev G
//       (m16n8k8 tf32 MMAs on the split operands); at the first block of a
//       lazy-update window, the errors of the whole previous window;
//   (b) the B columns of every row: parameters at a group start, code,
//       dequantize, e = (w - w^)/G_qq, subtract e * G[q, k] from the later
//       columns of the block, keep e in E.  One warp sweeps, one thread per
//       row, 16 columns at a time in registers, so the dependent chain from
//       one column to the next crosses no other thread; three warps apply
//       each finished 16 columns' errors to the rest of the block.  G's
//       diagonal block sits in shared memory and is read as broadcast
//       float4s;
//   (c) write E as a TF32 split for the trailing update and bit-pack the
//       block's codes.
// The columns right of block j0 + B are updated by trailing_tf32x3_kernel
// (trailing_tf32.cuh).

// Quantizer (dingiv.github.io page, section 量化基础; youleyou.com page,
// sections 二 and 四): asymmetric q = clip(rint(w/s) + z, 0, 2^b-1) with
// s = (max(0,max) - min(0,min)) / (2^b-1), z = rint(-min(0,min)/s);
// symmetric s = max|w| / (2^(b-1)-1), z = 2^(b-1); w^ = s (q - z).  The
// codes are decided in fp32 with IEEE division and round-half-to-even; the
// zero point is rint((2^b-1)(-min)/(max-min)) as one fp64 division of exact
// operands, which is -min/s with s unrounded.
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
    const int maxq = (1 << bits) - 1;
    s = (mx - mn) / static_cast<float>(maxq);
    // z = rint(-mn / s) with s taken exactly: one fp64 division of exact
    // operands, so an exact tie (a symmetric range gives 7.5 at 4 bits) is
    // rounded half to even rather than decided by the rounding of s.
    z = static_cast<float>(rint(static_cast<double>(maxq) * static_cast<double>(-mn) /
                                (static_cast<double>(mx) - static_cast<double>(mn))));
  }
}

// Copy W into the working buffer (dead columns zeroed) and, for one scale per
// output channel, compute each row's parameters from that copy.  One warp per
// row.  A NaN or Inf outside the dead columns sets the device status word to
// GPTQ_ERR_NONFINITE.
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
  bool finite = true;
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
    finite = finite && isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
    mn = fminf(mn, fminf(fminf(v.x, v.y), fminf(v.z, v.w)));
    mx = fmaxf(mx, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
  }
  if (!__all_sync(0xffffffffu, finite) && lane == 0) report_nonfinite();
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

// ------------------------------------------------------------- block step
// One block of B columns for a slab of QROWS rows (4 warps; the staging and
// the write-out run 4 threads per row, the sweep one thread per row):
//   (a) if a previous block exists, apply its errors to this block only:
//       W[rows, blk] -= E_prev[rows] * G[prev blk, blk]  (the columns
//       further right get them from the trailing-update kernel);
//   (b) quantize the block column by column in 16-column sub-blocks: the
//       sweeping thread codes w_q, takes e = (w_q - w^_q) / G_qq and updates
//       the sub-block's later columns in its registers; one rank-16 update
//       per sub-block (by the helper warps) carries its errors to the rest
//       of the block (same sums as column-at-a-time, grouped);
//   (c) bit-pack the block's codes and write E: as it is (for the next
//       block's step) and as a TF32 split (for the trailing update).
// Group parameters are taken from the current weights when a group's first
// column is reached (always a sub-block start, as groups are multiples of 32).
constexpr int QROWS = 32;            // rows per CTA
constexpr int QTHREADS = QROWS * 4;  // 4 threads per row

// Blocks per lazy-update window of the sweep (see gptq_quantize_layer): the
// trailing update after each block touches only the window's remaining
// columns, and the window's last block updates everything to the right of
// the next block with all m blocks at once (K = m B).  Wide layers only: it
// cuts the trailing read-modify-write traffic on W by m, which is what
// bounds the sweep there.
#ifndef GPTQ_SWEEP_WINDOW
#define GPTQ_SWEEP_WINDOW 4
#endif
inline int sweep_window_blocks(int64_t d_col) { return d_col >= 8192 ? GPTQ_SWEEP_WINDOW : 1; }

template <int B>
struct StepSmem {
  static constexpr int LDG = B + 4;  // padded rows (floats)
  static constexpr int G_OFF = 0;
  static constexpr int W_OFF = G_OFF + B * LDG * 4;
  static constexpr int E_OFF = W_OFF + QROWS * LDG * 4;
  static constexpr int INV_OFF = E_OFF + QROWS * LDG * 4;
  static constexpr int C_OFF = INV_OFF + B * 4;
  static constexpr int LDC = B + 4;  // code row stride (bytes): the 8 rows of a warp on 8 banks
  static constexpr int BYTES = C_OFF + QROWS * LDC;
};

template <int B>
constexpr int block_step_smem() { return StepSmem<B>::BYTES; }

// x = hi + lo with hi a TF32 value (low 13 mantissa bits cleared); both
// returned as the bit patterns the tf32 MMA reads.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = __float_as_uint(x) & 0xFFFFE000u;
  lo = __float_as_uint(x - __uint_as_float(hi));
}

// D += A B, m16n8k8, A row-major tf32 (a0: row g col t, a1: row g+8 col t,
// a2: row g col t+4, a3: row g+8 col t+4; g = lane/4, t = lane%4), B
// column-major (b0: row t col g, b1: row t+4 col g), fp32 accumulators
// (d0, d1: row g cols 2t, 2t+1; d2, d3: row g+8).
__device__ __forceinline__ void mma_tf32_m16n8k8(float (&d)[4], const uint32_t (&a)[4],
                                                 uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int B>
__device__ __forceinline__ void stage_rows(float* dst, const float* src, long long ld, int r0,
                                           int d_row, int ncols, int tid) {
  // QROWS x ncols floats -> dst (row stride LDG); rows beyond d_row are zero
  constexpr int LDG = StepSmem<B>::LDG;
  const int cpr = ncols / 4;
  for (int c = tid; c < QROWS * cpr; c += QTHREADS) {
    const int rr = c / cpr, k = (c - rr * cpr) * 4;
    const bool ok = r0 + rr < d_row;
    const float* sp = ok ? src + static_cast<long long>(r0 + rr) * ld + k : src;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst + rr * LDG + k)),
                 "l"(sp), "r"(ok ? 16 : 0)
                 : "memory");
  }
}

template <int B>
__device__ __forceinline__ void stage_gblock(float* dst, const float* G, int d_col, int r0,
                                             int c0, int nrows, int ncols, int tid) {
  constexpr int LDG = StepSmem<B>::LDG;
  const int cpr = ncols / 4;
  for (int c = tid; c < nrows * cpr; c += QTHREADS) {
    const int rr = c / cpr, k = (c - rr * cpr) * 4;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, 16;" ::"r"(smem_u32(dst + rr * LDG + k)),
                 "l"(G + static_cast<long long>(r0 + rr) * d_col + c0 + k)
                 : "memory");
  }
}

// FACTOR: G is the matrix F of gptq_prepare_factor (G's diagonal blocks,
// V_ab G_bb right of them) and the errors written for the later blocks are
// w^ - w_orig (Wo, the caller's weights, dead columns read as 0) instead of
// e; inside the block the sweep is unchanged.
template <int B, bool FACTOR = false>
__global__ void __launch_bounds__(QTHREADS)
block_step_kernel(const float* __restrict__ Wk, int d_row, int d_col, int j0, int ncols,
                  const float* __restrict__ G, const float* __restrict__ Eprev, int jp0,
                  int nprev, int lde, float* __restrict__ Ecur, float* __restrict__ Ecur_hi,
                  float* __restrict__ Ecur_lo,
                  uint32_t* __restrict__ qweight, float* __restrict__ scales,
                  uint8_t* __restrict__ zeros, int bits, int sym, int group, int n_groups,
                  int pc_mode, const float* __restrict__ Wo,
                  const uint8_t* __restrict__ dead) {
  using L = StepSmem<B>;
  constexpr int LDG = L::LDG;
  extern __shared__ __align__(16) uint8_t qsm[];
  float* Gs = reinterpret_cast<float*>(qsm + L::G_OFF);
  float* Ws = reinterpret_cast<float*>(qsm + L::W_OFF);
  float* Es = reinterpret_cast<float*>(qsm + L::E_OFF);
  float* invd = reinterpret_cast<float*>(qsm + L::INV_OFF);
  uint8_t* codes = qsm + L::C_OFF;

  const int tid = threadIdx.x;
  const int rloc = tid >> 2, t = tid & 3;
  const int lane = tid & 31;
  const int r0 = blockIdx.x * QROWS;
  const int r = r0 + rloc;
  const bool rv = r < d_row;

  // E_prev (nprev columns, row stride lde) and the G rows [jp0, jp0 + nprev)
  // are taken in chunks of B columns
  auto stage_chunk = [&](int kc) {
    stage_rows<B>(Es, Eprev + kc, lde, r0, d_row, B, tid);
    stage_gblock<B>(Gs, G, d_col, jp0 + kc, j0, B, ncols, tid);
  };
  stage_rows<B>(Ws, Wk + j0, d_col, r0, d_row, ncols, tid);
  if (nprev > 0) stage_chunk(0);
  else stage_gblock<B>(Gs, G, d_col, j0, j0, ncols, ncols, tid);
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  float* erow = Es + rloc * LDG;
  if (nprev > 0) {
    // (a) W[rows, blk] -= E_prev[rows] * G[prev cols, blk] on the MMA path:
    // m16n8k8 tf32, three products of the split operands (hi hi + hi lo +
    // lo hi; hi = the low 13 mantissa bits cleared), fp32 accumulate, the
    // same arithmetic as the trailing update.  The previous columns are the
    // previous block, or at a window's first block all the blocks of the
    // previous window, B at a time.  Warp w takes the output columns
    // [w B/4, (w+1) B/4) of both 16-row halves of the slab; ncols is a
    // multiple of 32, so a warp's columns are all inside or all past it.
    constexpr int NTW = B / 32;  // 8-column tiles per warp
    const int warp = tid >> 5, g = lane >> 2, t4 = lane & 3;
    const int cw = warp * (B / 4);
    float acc[2][NTW][4];
    if (cw < ncols) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
          const float* w0 = Ws + (16 * mt + g) * LDG + cw + 8 * nt + 2 * t4;
          acc[mt][nt][0] = w0[0];
          acc[mt][nt][1] = w0[1];
          acc[mt][nt][2] = w0[8 * LDG];
          acc[mt][nt][3] = w0[8 * LDG + 1];
        }
    }
    // each chunk of B columns is summed from zero and then added into the
    // block with round-to-nearest fp32 adds: the MMA's own accumulation does
    // not round to nearest, and its error grows with the MMAs it chains
    float part[2][NTW][4];
    for (int kc = 0; kc < nprev; kc += B) {
      if (kc > 0) {
        stage_chunk(kc);
        asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) part[mt][nt][e] = 0.0f;
      if (cw < ncols) {
#pragma unroll 2
        for (int k0 = 0; k0 < B; k0 += 8) {
          uint32_t ah[2][4], al[2][4];
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            const float* e0 = Es + (16 * mt + g) * LDG + k0 + t4;
            const float v[4] = {-e0[0], -e0[8 * LDG], -e0[4], -e0[8 * LDG + 4]};
#pragma unroll
            for (int q = 0; q < 4; ++q) split_tf32(v[q], ah[mt][q], al[mt][q]);
          }
#pragma unroll
          for (int nt = 0; nt < NTW; ++nt) {
            const float* g0 = Gs + (k0 + t4) * LDG + cw + 8 * nt + g;
            uint32_t bh0, bl0, bh1, bl1;
            split_tf32(g0[0], bh0, bl0);
            split_tf32(g0[4 * LDG], bh1, bl1);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
              mma_tf32_m16n8k8(part[mt][nt], ah[mt], bh0, bh1);
              mma_tf32_m16n8k8(part[mt][nt], ah[mt], bl0, bl1);
              mma_tf32_m16n8k8(part[mt][nt], al[mt], bh0, bh1);
            }
          }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[mt][nt][e] += part[mt][nt][e];
      }
      __syncthreads();  // every thread is done with this chunk's E and G rows
    }
    if (cw < ncols) {
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NTW; ++nt) {
          float* w0 = Ws + (16 * mt + g) * LDG + cw + 8 * nt + 2 * t4;
          w0[0] = acc[mt][nt][0];
          w0[1] = acc[mt][nt][1];
          w0[8 * LDG] = acc[mt][nt][2];
          w0[8 * LDG + 1] = acc[mt][nt][3];
        }
    }
    stage_gblock<B>(Gs, G, d_col, j0, j0, ncols, ncols, tid);
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
  }
  for (int q = tid; q < ncols; q += QTHREADS) invd[q] = 1.0f / Gs[q * LDG + q];
  __syncthreads();

  // (b) 16-column sub-blocks.  Warp 0 sweeps: lane l holds row r0 + l, takes
  // a sub-block's 16 values into registers and runs its dependent column
  // steps with no exchange between threads.  Warps 1..3 apply each finished
  // sub-block's 16 errors to the block's later columns (a rank-16 update,
  // lane l again on row r0 + l, 4-column chunks split over the 3 warps).
  // Two named barriers hand the work over: 1 = "the errors of sub-block sb
  // are in E", 2 = "the columns of sub-block sb + 1 carry every earlier
  // error".  The helpers update the next sub-block's columns first and
  // release the sweeper before the rest, except where a group starts at the
  // next sub-block: its parameters read the whole group, so they release it
  // after all their updates.
  const float maxq = static_cast<float>((1 << bits) - 1);
  const int warp_id = tid >> 5;
  const int nsb = ncols / 16;
  float* hw = Ws + lane * LDG;  // this thread's row in (b)
  float* he = Es + lane * LDG;
  if (warp_id == 0) {
    const int rs = r0 + lane;
    const bool rvs = rs < d_row;
    float s = 1.0f, z = 0.0f;
    if (pc_mode) {
      if (rvs) { s = scales[rs]; z = static_cast<float>(zeros[rs]); }
    } else if (group > B && (j0 % group) != 0) {  // the group began in an earlier block
      const int g = j0 / group;
      if (rvs) { s = scales[static_cast<size_t>(rs) * n_groups + g];
                 z = static_cast<float>(zeros[static_cast<size_t>(rs) * n_groups + g]); }
    }
    uint32_t* crow = reinterpret_cast<uint32_t*>(codes + lane * L::LDC);
    for (int sb = 0; sb < nsb; ++sb) {
      const int q0 = 16 * sb;
      if (sb > 0) named_bar(2, QTHREADS);
      if (!pc_mode && ((j0 + q0) % group) == 0) {  // a group starts here
        // four independent min/max chains, 16 columns per step (a group
        // and the block are multiples of 16 columns)
        const int gend = min(q0 + group, ncols);
        float mn[4] = {3.4e38f, 3.4e38f, 3.4e38f, 3.4e38f};
        float mx[4] = {-3.4e38f, -3.4e38f, -3.4e38f, -3.4e38f};
        auto scan16 = [&](const float* p) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 v = *reinterpret_cast<const float4*>(p + 4 * i);
            mn[i] = fminf(mn[i], fminf(fminf(v.x, v.y), fminf(v.z, v.w)));
            mx[i] = fmaxf(mx[i], fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
          }
        };
        for (int c = q0; c < gend; c += 16) scan16(hw + c);
        if (group > B && rvs) {  // the rest of the group lies right of this block
          const float* rest = Wk + static_cast<size_t>(rs) * d_col;
          for (int c = j0 + B; c < j0 + group; c += 16) scan16(rest + c);
        }
        make_params(fminf(fminf(mn[0], mn[1]), fminf(mn[2], mn[3])),
                    fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), bits, sym, s, z);
        if (rvs) {
          const int g = (j0 + q0) / group;
          scales[static_cast<size_t>(rs) * n_groups + g] = s;
          zeros[static_cast<size_t>(rs) * n_groups + g] = static_cast<uint8_t>(z);
        }
      }
      float w[16], iv[16], ev[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = *reinterpret_cast<const float4*>(hw + q0 + 4 * i);
        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        const float4 d = *reinterpret_cast<const float4*>(invd + q0 + 4 * i);
        iv[4 * i] = d.x; iv[4 * i + 1] = d.y; iv[4 * i + 2] = d.z; iv[4 * i + 3] = d.w;
      }
      uint32_t cw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float x = w[u];
        float qf = rintf(x / s) + z;
        qf = fminf(fmaxf(qf, 0.0f), maxq);
        const float xh = s * (qf - z);
        const float e = (x - xh) * iv[u];
        ev[u] = e;
        if (FACTOR) w[u] = xh;  // w[u] is not read again
        cw[u >> 2] |= static_cast<uint32_t>(qf) << (8 * (u & 3));
        // the later columns of the sub-block: w -= e G[q, later]
        const float* grow = Gs + (q0 + u) * LDG + q0;
#pragma unroll
        for (int i = (u + 1) >> 2; i < 4; ++i) {
          const float4 g4 = *reinterpret_cast<const float4*>(grow + 4 * i);
          const float gv[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (4 * i + k > u) w[4 * i + k] = fmaf(-e, gv[k], w[4 * i + k]);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        *reinterpret_cast<float4*>(he + q0 + 4 * i) =
            make_float4(ev[4 * i], ev[4 * i + 1], ev[4 * i + 2], ev[4 * i + 3]);
        crow[q0 / 4 + i] = cw[i];
        // the sub-block's own columns of W are no longer read: keep w^ there
        if (FACTOR)
          *reinterpret_cast<float4*>(hw + q0 + 4 * i) =
              make_float4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
      if (sb + 1 < nsb) named_bar_arrive(1, QTHREADS);
    }
  } else {
    const int h = warp_id - 1;  // 0..2
    for (int sb = 0; sb + 1 < nsb; ++sb) {
      const int q0 = 16 * sb;
      named_bar(1, QTHREADS);
      float ev[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 v = *reinterpret_cast<const float4*>(he + q0 + 4 * i);
        ev[4 * i] = v.x; ev[4 * i + 1] = v.y; ev[4 * i + 2] = v.z; ev[4 * i + 3] = v.w;
      }
      // W[row, c..c+3] -= sum_u e_u G[q0 + u, c..c+3], u in order
      auto update = [&](int c) {
        float4 acc = *reinterpret_cast<const float4*>(hw + c);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float4 g4 = *reinterpret_cast<const float4*>(Gs + (q0 + u) * LDG + c);
          acc.x = fmaf(-ev[u], g4.x, acc.x); acc.y = fmaf(-ev[u], g4.y, acc.y);
          acc.z = fmaf(-ev[u], g4.z, acc.z); acc.w = fmaf(-ev[u], g4.w, acc.w);
        }
        *reinterpret_cast<float4*>(hw + c) = acc;
      };
      // two chunks with their FMA chains interleaved
      auto update2 = [&](int c, int c2) {
        float4 a = *reinterpret_cast<const float4*>(hw + c);
        float4 b = *reinterpret_cast<const float4*>(hw + c2);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float4 g4 = *reinterpret_cast<const float4*>(Gs + (q0 + u) * LDG + c);
          const float4 g5 = *reinterpret_cast<const float4*>(Gs + (q0 + u) * LDG + c2);
          a.x = fmaf(-ev[u], g4.x, a.x); a.y = fmaf(-ev[u], g4.y, a.y);
          a.z = fmaf(-ev[u], g4.z, a.z); a.w = fmaf(-ev[u], g4.w, a.w);
          b.x = fmaf(-ev[u], g5.x, b.x); b.y = fmaf(-ev[u], g5.y, b.y);
          b.z = fmaf(-ev[u], g5.z, b.z); b.w = fmaf(-ev[u], g5.w, b.w);
        }
        *reinterpret_cast<float4*>(hw + c) = a;
        *reinterpret_cast<float4*>(hw + c2) = b;
      };
      const bool group_next = !pc_mode && ((j0 + q0 + 16) % group) == 0;
      if (h == 0) update2(q0 + 16, q0 + 28);
      else update(q0 + 16 + 4 * h);
      if (!group_next) named_bar_arrive(2, QTHREADS);
      for (int c = q0 + 32 + 4 * h; c < ncols; c += 12) update(c);
      if (group_next) named_bar_arrive(2, QTHREADS);
    }
  }
  __syncthreads();
  // (c) E for the trailing update as a TF32 split (hi = low 13 mantissa bits
  // cleared, lo = E - hi), and the packed codes
  if (rv) {
    float* ef = Ecur + static_cast<size_t>(r) * lde;
    float* eh = Ecur_hi + static_cast<size_t>(r) * lde;
    float* el = Ecur_lo + static_cast<size_t>(r) * lde;
    const float* xrow = Ws + rloc * LDG;
    const float* worow = FACTOR ? Wo + static_cast<size_t>(r) * d_col + j0 : nullptr;
    for (int c = 4 * t; c < B; c += 16) {
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < ncols) {
        if (FACTOR) {
          const float4 xh = *reinterpret_cast<const float4*>(xrow + c);
          float4 wo = *reinterpret_cast<const float4*>(worow + c);
          if (dead) {
            const uchar4 dm = *reinterpret_cast<const uchar4*>(dead + j0 + c);
            if (dm.x) wo.x = 0.0f;
            if (dm.y) wo.y = 0.0f;
            if (dm.z) wo.z = 0.0f;
            if (dm.w) wo.w = 0.0f;
          }
          v = make_float4(xh.x - wo.x, xh.y - wo.y, xh.z - wo.z, xh.w - wo.w);
        } else {
          v = *reinterpret_cast<const float4*>(erow + c);
        }
      }
      *reinterpret_cast<float4*>(ef + c) = v;
      const float4 h = make_float4(__uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u),
                                   __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u),
                                   __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u),
                                   __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u));
      *reinterpret_cast<float4*>(eh + c) = h;
      *reinterpret_cast<float4*>(el + c) = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
    }
    const int nw = ncols * bits / 32;
    const size_t row_words = static_cast<size_t>(d_col) * bits / 32;
    uint32_t* qrow = qweight + static_cast<size_t>(r) * row_words + (static_cast<size_t>(j0) * bits) / 32;
    const uint8_t* cs = codes + rloc * L::LDC;
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
