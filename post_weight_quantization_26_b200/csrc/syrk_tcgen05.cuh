// Hessian accumulation H += scale * X^T X on the 5th-generation tensor cores.
//
// dingiv.github.io "量化" page, section GPTQ: H = 2 X X^T over the
// calibration tokens.  X arrives token-major (n rows of d bf16 values), so
// with K = tokens both MMA operands are "MN-major": A(m,k) = X[k][i0+m] and
// B(n,k) = X[k][j0+n] come from the same tensor.  Only tiles that touch the
// upper triangle (i <= j) are computed, 128 x 256 per tile, in an order that
// keeps the units in flight on a compact block of tiles (decode_tile), and
// tokens are split into S chunks so that tiles x chunks fill the 148 SMs
// evenly; the chunk partials meet in H through TMA bulk reduce-adds (fp32 add
// in L2).
//
// Accuracy: the tensor cores' fp32 accumulation is not round-to-nearest, and
// over a long chain of MMAs its error grows with the chain (about 1.5e-4
// relative after 2300 MMAs, measured against an fp64 sum).  So a TMEM
// accumulator only ever sums CHAIN_TOKENS tokens from zero; each finished
// chain is folded into fp32 registers of the epilogue with ordinary
// round-to-nearest adds, and the chunk's sum leaves through a TMA reduce-add.
// With one chunk (nsplit = 1) every element of H receives exactly one add
// per launch, so H does not depend on the order in which units finish.
//
// Warp roles (320 threads, one CTA per SM, persistent over work units):
//   warp 0      TMA producer: 64-token stages, A = 2 boxes of 64 features,
//               B = 4 boxes, 128-byte swizzle, STAGES-deep ring.
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators)
//               and issues tcgen05.mma (one thread), K = 16 per instruction.
//   warps 2..9  epilogue: warp w reads TMEM lane quarter (w % 4) and column
//               half (w - 2) / 4, keeps that 32 x 128 slice of the chunk sum
//               in registers (128 per thread).  At the end of the unit it
//               scales the slice, zeroes what lies below the diagonal, and
//               stages it in 128 x 32 pieces (128-byte swizzle) that one
//               thread per half adds into H with a TMA reduce-add.
// The two TMEM accumulators alternate between chains, so the fold of one
// chain overlaps the MMAs of the next.  Every mbarrier wait is bounded.
#pragma once

#include "common.cuh"

namespace gptq {
namespace syrk {

constexpr int BM = 128;     // rows of H per tile (features i)
constexpr int BN = 256;     // columns of H per tile (features j)
constexpr int BK = 64;      // tokens per pipeline stage
constexpr int STAGES = 4;
constexpr int BOX = 64;     // TMA box: 64 features (128 B) x 64 tokens
constexpr int BOX_BYTES = BOX * BK * 2;               // 8 KB
constexpr int A_BYTES = BM * BK * 2;                  // 16 KB
constexpr int B_BYTES = BN * BK * 2;                  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;        // 48 KB
constexpr int NUM_THREADS = 320;
constexpr int EPI_WARPS = 8;
constexpr int CHAIN_KB = 16;                          // k-stages per TMEM chain
constexpr int CHAIN_TOKENS = CHAIN_KB * BK;           // 1024 tokens
constexpr int OUT_COLS = 32;                          // staged piece: 128 x 32 fp32
constexpr int OUT_BYTES = BM * OUT_COLS * 4;          // 16 KB, one per column half
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_BYTES =
    STAGES * STAGE_BYTES + 2 * OUT_BYTES + 1024 /*align*/ + 256 /*barriers*/;

// Instruction descriptor, kind::f16: fp32 accumulate (bits 4-5 = 1), A and B
// bf16 (bits 7-9 = 1, 10-12 = 1), both MN-major (bits 15, 16), N>>3 at
// bits 17-22, M>>4 at bits 24-28.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                           (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

struct Params {
  float* H;
  int d;
  int n;
  float scale;
  int nti;        // row tiles: ceil(d / BM)
  int ntj;        // column tiles: ceil(d / BN)
  int ntiles;     // tiles touching the upper triangle
  int split_tokens;  // tokens per chunk (multiple of BK)
  int nsplit;
  int units;      // ntiles * nsplit
  uint64_t wait_ns;  // limit of every bounded wait (ns)
  int stall;      // fault injection: the producer issues nothing, so the
                  // MMA thread's first wait runs out (0 in normal use)
};

// Tile order.  The tiles (ti, tj) touching the upper triangle are those with
// tj >= ti / 2 (BN = 2 BM).  They are taken in groups of GROUP_COLS column
// tiles; within a group, row tile by row tile, the group's column tiles left
// to right.  The ~148 units in flight then cover about 18 row tiles x 8
// column tiles, so they read about a fifth of X's features per token window
// (d = 22016), and concurrent units reuse each window from L2: ~10 passes
// over X per launch instead of ~34 for plain row-major order.
constexpr int GROUP_COLS = 8;

__device__ __forceinline__ void decode_tile(int t, int nti, int ntj, int& ti, int& tj) {
  for (int a = 0; a < ntj; a += GROUP_COLS) {
    const int b = min(ntj, a + GROUP_COLS), w = b - a;
    const int rows = min(nti, 2 * b);   // rows with a tile in [a, b)
    const int full = min(rows, 2 * a);  // rows whose w tiles are all above the diagonal
    if (t < full * w) {
      ti = t / w;
      tj = a + t % w;
      return;
    }
    t -= full * w;
    for (int r = full; r < rows; ++r) {  // diagonal rows: tiles r/2 .. b-1
      const int c = b - (r >> 1);
      if (t < c) {
        ti = r;
        tj = (r >> 1) + t;
        return;
      }
      t -= c;
    }
  }
  ti = tj = 0;  // not reached for t < ntiles
}

__device__ __forceinline__ void decode_unit(const Params& p, int u, int& ti, int& tj,
                                            int& k0, int& nk) {
  const int s = u / p.ntiles;
  decode_tile(u - s * p.ntiles, p.nti, p.ntj, ti, tj);
  k0 = s * p.split_tokens;
  const int k1 = min(p.n, k0 + p.split_tokens);
  nk = (k1 - k0 + BK - 1) / BK;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
syrk_bf16_tcgen05_kernel(const __grid_constant__ CUtensorMap tmap_x,
                         const __grid_constant__ CUtensorMap tmap_h, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned ring of stages (128B-swizzle atoms are 1024 B).
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t ring = (raw + 1023u) & ~1023u;
  uint8_t* ring_ptr = smem_raw + (ring - raw);
  const uint32_t outbuf0 = ring + STAGES * STAGE_BYTES;  // 2 x 16 KB, 1024-aligned
  float* out_ptr = reinterpret_cast<float*>(ring_ptr + STAGES * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring_ptr + STAGES * STAGE_BYTES + 2 * OUT_BYTES);
  // bars[0..S) full, [S..2S) empty, [2S..2S+2) tmem_full, [2S+2..2S+4) tmem_empty
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8u * STAGES;
  const uint32_t tfull0 = full0 + 16u * STAGES;
  const uint32_t tempty0 = tfull0 + 16u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8u * a, 1);
      mbar_init(tempty0 + 8u * a, EPI_WARPS);  // one arrive per epilogue warp
    }
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_h);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !p.stall) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        int ti, tj, k0, nk;
        decode_unit(p, u, ti, tj, k0, nk);
        for (int kt = 0; kt < nk; ++kt) {
          if (!mbar_wait_bounded(empty0 + 8u * stage, phase ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
          const uint32_t fb = full0 + 8u * stage;
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          const uint32_t sa = ring + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          const int tok = k0 + kt * BK;
#pragma unroll
          for (int c = 0; c < BM / BOX; ++c) tma_load_2d(sa + c * BOX_BYTES, &tmap_x, fb, ti * BM + c * BOX, tok);
#pragma unroll
          for (int c = 0; c < BN / BOX; ++c) tma_load_2d(sb + c * BOX_BYTES, &tmap_x, fb, tj * BN + c * BOX, tok);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t gc = 0;  // chains issued by this CTA
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        int ti, tj, k0, nk;
        decode_unit(p, u, ti, tj, k0, nk);
        uint32_t d_tmem = tmem_base;
        for (int kt = 0; kt < nk; ++kt) {
          const int kc = kt % CHAIN_KB;
          if (kc == 0) {  // a new chain starts in the other accumulator
            const uint32_t acc = gc & 1u;
            if (!mbar_wait_bounded(tempty0 + 8u * acc, ((gc >> 1) & 1u) ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            d_tmem = tmem_base + acc * BN;
          }
          if (!mbar_wait_bounded(full0 + 8u * stage, phase, abort_flag, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = ring + stage * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // 16 tokens = two 8-row core groups of 128 B each = 2048 B.
            const uint64_t ad = smem_desc_sw128(sa + kk * 2048, BOX_BYTES, 1024);
            const uint64_t bd = smem_desc_sw128(sb + kk * 2048, BOX_BYTES, 1024);
            mma_f16_ss(d_tmem, ad, bd, IDESC, (kc | kk) != 0);
          }
          mma_commit(empty0 + 8u * stage);  // frees the stage when these MMAs finish
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          if (kc == CHAIN_KB - 1 || kt == nk - 1) {
            mma_commit(tfull0 + 8u * (gc & 1u));  // chain ready for the fold
            ++gc;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;          // TMEM lanes [32*quarter, +32)
    const int half = (warp - 2) >> 2;      // columns [128*half, +128) of the tile
    // The eight epilogue warps meet at named barriers, so their control flow
    // stays uniform even after a wait gives up: a warp that timed out keeps
    // looping (skipping the work) instead of leaving the others waiting.
    uint32_t gc = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
      int ti, tj, k0, nk;
      decode_unit(p, u, ti, tj, k0, nk);
      float acc_r[BN / 2];
#pragma unroll
      for (int j = 0; j < BN / 2; ++j) acc_r[j] = 0.f;
      const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
      const int nchains = (nk + CHAIN_KB - 1) / CHAIN_KB;
      for (int ch = 0; ch < nchains; ++ch, ++gc) {
        const uint32_t acc = gc & 1u;
        if (ok && !mbar_wait_bounded(tfull0 + 8u * acc, (gc >> 1) & 1u, abort_flag, p.wait_ns)) ok = false;
        if (!ok) continue;
        tc_fence_after();
        const uint32_t t0 = tmem_base + lane_off + acc * BN + half * (BN / 2);
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(t0 + c * 16, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) acc_r[16 * c + j] += __uint_as_float(r[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty0 + 8u * acc);
      }
      // scale, mask to the upper triangle, stage, and reduce-add into H
      const int rl = quarter * 32 + lane;           // row within the tile
      const int row = ti * BM + rl;
      const bool issuer = lane == 0 && quarter == 2;  // warps 2 and 6
      float* orow = out_ptr + half * (OUT_BYTES / 4) + rl * OUT_COLS;
#pragma unroll
      for (int c = 0; c < BN / 2 / OUT_COLS; ++c) {
        const int x0 = tj * BN + half * (BN / 2) + c * OUT_COLS;  // first column of the piece
        // pieces past the matrix or wholly below the diagonal add nothing
        const bool live = ok && x0 < p.d && x0 + OUT_COLS - 1 >= ti * BM;
        if (issuer) bulk_wait_read0();   // this half's previous piece has left the buffer
        named_bar(1, 32 * EPI_WARPS);
        if (live) {
#pragma unroll
          for (int q = 0; q < OUT_COLS / 4; ++q) {
            const int j = x0 + 4 * q;
            float4 v;
            v.x = (j >= row) ? acc_r[c * OUT_COLS + 4 * q] * p.scale : 0.f;
            v.y = (j + 1 >= row) ? acc_r[c * OUT_COLS + 4 * q + 1] * p.scale : 0.f;
            v.z = (j + 2 >= row) ? acc_r[c * OUT_COLS + 4 * q + 2] * p.scale : 0.f;
            v.w = (j + 3 >= row) ? acc_r[c * OUT_COLS + 4 * q + 3] * p.scale : 0.f;
            // 128-byte swizzle: 16-byte chunk q of row r sits at chunk q ^ (r & 7)
            *reinterpret_cast<float4*>(orow + 4 * (q ^ (rl & 7))) = v;
          }
          fence_proxy_async_smem();
        }
        named_bar(1, 32 * EPI_WARPS);
        if (issuer && live) {
          tma_reduce_add_2d(&tmap_h, outbuf0 + half * OUT_BYTES, x0, ti * BM);
          bulk_commit();
        }
      }
    }
    if (lane == 0 && quarter == 2) bulk_wait0();  // the reduce-adds have landed in H
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace syrk
}  // namespace gptq
