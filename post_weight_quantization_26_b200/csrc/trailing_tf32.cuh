// Lazy batched update of the columns right of a block on the 5th-generation
// tensor cores (dingiv.github.io "量化" page, section GPTQ: after a block of B
// columns is quantized, all columns to its right are updated at once by one
// matrix product):
//     W[:, n0:n0+N] -= E[:, ek0:ek0+K] * G[j0:j0+K, n0:n0+N]
// E (d_row x K) and G are fp32; the product runs as three TF32 MMAs per
// K-step on the split operands x = x_hi + x_lo (x_hi = x with the low 13
// mantissa bits cleared, x_lo = x - x_hi, exact):
//     E G ~ E_hi G_hi + E_hi G_lo + E_lo G_hi
// which keeps close to fp32 accuracy (the dropped E_lo G_lo term is ~2^-20
// of the product).
//
// Persistent kernel, 192 threads, tiles of 128 (rows of W) x 256 (columns):
//   warp 0      TMA producer: per 16-wide K slice, E_hi/E_lo boxes (K-major,
//               64-byte swizzle) and G_hi/G_lo boxes (MN-major, 128-byte
//               swizzle with 32-byte atoms, the one MN-major form tf32
//               operands take; G is addressed as 32-column chunks x rows x
//               chunks, so each split's 256 columns come in one copy),
//               two-deep ring: four copies per K slice;
//   warp 1      allocates 512 TMEM columns (two fp32 128x256 accumulators,
//               used by alternate tiles so that one tile's epilogue overlaps
//               the next tile's MMAs) and issues tcgen05.mma kind::tf32 from
//               one thread;
//   warps 2..5  epilogue, each on its own 32 rows (its TMEM lane quarter):
//               tcgen05.ld 32 columns at a time, negate, write a 32x32 piece
//               to its own 4 KB of shared memory (128-byte swizzle), and add
//               it into W with its own TMA reduce-add (the L2 does the read-
//               modify-write); no barrier between the four warps.  A long K
//               is summed in chains of `chain` K-steps, each added into W on
//               its own, in order.
// Shared memory is kept near 112 KB so a block-step CTA fits on the same SM
// (the two kernels run concurrently on different streams).  Every mbarrier
// wait is bounded.
#pragma once

#include "common.cuh"

namespace gptq {
namespace trail {

constexpr int BM = 128, BN = 256, BK = 16;
constexpr int STAGES = 2;
constexpr int A_BYTES = BM * BK * 4;              // 8 KB (one split)
constexpr int B_BOX = 32;                          // 32 fp32 = 128 B inner box
constexpr int B_BOX_BYTES = B_BOX * BK * 4;        // 2 KB
constexpr int B_BYTES = BN * BK * 4;               // 16 KB (one split)
constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;  // 48 KB
constexpr int OUT_COLS = 32;
constexpr int OUT_ROWS = 32;                       // rows of one epilogue warp's W box
constexpr int OUT_BYTES = BM * OUT_COLS * 4;       // 16 KB: 4 warps x 4 KB
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + OUT_BYTES + 1024 + 256;

// kind::tf32 instruction descriptor: fp32 accumulate, A and B tf32 (format
// 2), A K-major, B MN-major (bit 16), N>>3 at bits 17-22, M>>4 at 24-28.
constexpr uint32_t IDESC = (1u << 4) | (2u << 7) | (2u << 10) | (1u << 16) |
                           (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

struct Params {
  int M;        // rows of W
  int N;        // columns to update (from n0)
  int K;        // block width (E and G read as zero past it)
  int n0;       // first column to update (also the column coordinate into G)
  int j0;       // first row of G's block
  int ek0;      // first column of E's block in the E buffer
  int chain;    // K-steps (of BK) summed per TMEM chain; 0: the whole K in one
  int tiles_m, tiles_n, tiles;
  uint64_t wait_ns;  // limit of every bounded wait (ns)
  int stall;    // fault injection: the producer issues nothing, so the MMA
                // thread's first wait runs out (0 in normal use)
};

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(layout) << 61;
  return d;
}

__device__ __forceinline__ void tmem_alloc1(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
trailing_tf32x3_kernel(const __grid_constant__ CUtensorMap tm_ehi,
                       const __grid_constant__ CUtensorMap tm_elo,
                       const __grid_constant__ CUtensorMap tm_ghi,
                       const __grid_constant__ CUtensorMap tm_glo,
                       const __grid_constant__ CUtensorMap tm_w, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t ring = base;                                 // STAGES x 48 KB
  const uint32_t outbuf = base + STAGES * STAGE_BYTES;        // 16 KB, 1024-aligned
  float* out_ptr = reinterpret_cast<float*>(base_ptr + STAGES * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base_ptr + STAGES * STAGE_BYTES + OUT_BYTES);
  // bars: [0,S) full, [S,2S) empty, [2S,2S+2) tmem_full, [2S+2,2S+4) tmem_empty
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8u * STAGES;
  const uint32_t tfull0 = full0 + 16u * STAGES, tempty0 = tfull0 + 16u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8u * a, 1);
      mbar_init(tempty0 + 8u * a, 4);  // one arrive per epilogue warp
    }
    *abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tm_ehi); tma_prefetch_desc(&tm_elo);
    tma_prefetch_desc(&tm_ghi); tma_prefetch_desc(&tm_glo); tma_prefetch_desc(&tm_w);
  }
  if (warp == 1) {
    tmem_alloc1(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nk = (p.K + BK - 1) / BK;  // E is zero past K
  // K-steps per TMEM chain: each chain is summed from zero and added into W
  // on its own (round-to-nearest in L2), since the MMA's accumulation does
  // not round to nearest and its error grows with the MMAs it chains
  const int chain = p.chain > 0 ? p.chain : nk;

  if (warp == 0) {
    if (lane == 0 && !p.stall) {  // -------------------------------- producer
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.tiles && ok; u += gridDim.x) {
        const int tm = u % p.tiles_m, tn = u / p.tiles_m;
        for (int ks = 0; ks < nk; ++ks) {
          if (!mbar_wait_bounded(empty0 + 8u * stage, phase ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
          const uint32_t fb = full0 + 8u * stage;
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          const uint32_t s0 = ring + stage * STAGE_BYTES;
          tma_load_2d(s0, &tm_ehi, fb, p.ek0 + ks * BK, tm * BM);
          tma_load_2d(s0 + A_BYTES, &tm_elo, fb, p.ek0 + ks * BK, tm * BM);
          // G: all BN / 32 column chunks of the K slice in one copy per split
          const int gz = (p.n0 + tn * BN) / B_BOX, gy = p.j0 + ks * BK;
          tma_load_3d(s0 + 2 * A_BYTES, &tm_ghi, fb, 0, gy, gz);
          tma_load_3d(s0 + 2 * A_BYTES + B_BYTES, &tm_glo, fb, 0, gy, gz);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {  // ----------------------------------------------- MMA
      uint32_t stage = 0, phase = 0;
      int lu = 0;  // chains issued by this CTA
      bool ok = true;
      for (int u = blockIdx.x; u < p.tiles && ok; u += gridDim.x) {
       for (int c0 = 0; c0 < nk && ok; c0 += chain, ++lu) {
        const uint32_t acc = lu & 1;
        if (!mbar_wait_bounded(tempty0 + 8u * acc, ((lu >> 1) & 1) ^ 1u, abort_flag, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int ks = c0; ks < min(nk, c0 + chain); ++ks) {
          if (!mbar_wait_bounded(full0 + 8u * stage, phase, abort_flag, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t s0 = ring + stage * STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 8; ++kk) {
            // A: K-major, 64-byte swizzle: 8-row groups 512 B apart; K step = 32 B.
            const uint64_t ahi = smem_desc(s0 + kk * 32, 16, 512, 4);
            const uint64_t alo = smem_desc(s0 + A_BYTES + kk * 32, 16, 512, 4);
            // B: MN-major tf32 takes only the 128-byte swizzle with 32-byte
            // atoms (4 K-rows of 128 B per atom): 32-column chunks one box
            // (2 KB) apart, 4-row K groups 512 B apart; this K step's 8 rows
            // are the kk-th 1 KB slice.
            const uint64_t bhi = smem_desc(s0 + 2 * A_BYTES + kk * 1024, B_BOX_BYTES, 512, 1);
            const uint64_t blo = smem_desc(s0 + 2 * A_BYTES + B_BYTES + kk * 1024, B_BOX_BYTES, 512, 1);
            mma_tf32_ss(d_tmem, ahi, bhi, IDESC, ((ks - c0) | kk) != 0);
            mma_tf32_ss(d_tmem, ahi, blo, IDESC, 1);
            mma_tf32_ss(d_tmem, alo, bhi, IDESC, 1);
          }
          mma_commit(empty0 + 8u * stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit(tfull0 + 8u * acc);
       }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp q (= warp & 3) owns TMEM lanes [32q, 32q + 32), rows 32q.. of the
    // tile.  It stages its own 32 x 32 piece in its own 4 KB of the output
    // buffer and adds it into W with its own TMA reduce-add, so the four
    // warps never wait for one another.  The next piece's TMEM load is in
    // flight while the warp waits for its previous reduce to read the buffer.
    const int quarter = warp & 3;
    float* obuf = out_ptr + quarter * OUT_ROWS * OUT_COLS;
    const uint32_t obuf_s = outbuf + quarter * OUT_ROWS * OUT_COLS * 4;
    bool ok = true;
    int lu = 0;
    for (int u = blockIdx.x; u < p.tiles; u += gridDim.x) {
     const int tm = u % p.tiles_m, tn = u / p.tiles_m;
     const int row0 = tm * BM + quarter * OUT_ROWS;  // this warp's first row of W
     for (int c0 = 0; c0 < nk; c0 += chain, ++lu) {
      const uint32_t acc = lu & 1;
      if (ok && !mbar_wait_bounded(tfull0 + 8u * acc, (lu >> 1) & 1, abort_flag, p.wait_ns)) ok = false;
      tc_fence_after();
      // a tile's chains land in W in order: this warp's previous adds first
      if (lane == 0 && c0 > 0) bulk_wait0();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
      for (int c = 0; c < BN / OUT_COLS; ++c) {
        if (tn * BN + c * OUT_COLS >= p.N) break;  // past the columns to update
        uint32_t r[32];
        if (ok) {
          tmem_ld_32x32b_x32(t_row + c * OUT_COLS, r);
        }
        if (lane == 0) bulk_wait_read0();  // the previous reduce has read the buffer
        __syncwarp();
        if (ok) {
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = 0u;
        }
        // 128-byte swizzle: 16-byte chunk j of row r lives at chunk j ^ (r & 7)
        float* orow = obuf + lane * OUT_COLS;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int pj = j ^ (lane & 7);
          float4 v = make_float4(-__uint_as_float(r[4 * j]), -__uint_as_float(r[4 * j + 1]),
                                 -__uint_as_float(r[4 * j + 2]), -__uint_as_float(r[4 * j + 3]));
          *reinterpret_cast<float4*>(orow + 4 * pj) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && ok && row0 < p.M) {
          tma_reduce_add_2d(&tm_w, obuf_s, p.n0 + tn * BN + c * OUT_COLS, row0);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8u * acc);
     }
    }
    if (lane == 0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// x_hi = x with the low 13 mantissa bits cleared (a TF32 value), x_lo = x - x_hi.
__global__ void split_tf32_kernel(const float* __restrict__ x, float* __restrict__ hi,
                                  float* __restrict__ lo, size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    const float h = __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    hi[i] = h;
    lo[i] = v - h;
  }
}

}  // namespace trail
}  // namespace gptq
