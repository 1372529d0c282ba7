// Matmul with the packed 4-bit layer: Y[b][r] = sum_k X[b][k] W^[r][k],
// W^[r][k] = s[r][g(k)] (q[r][k] - z[r][g(k)]), X bf16 (up to 8 activation
// rows), Y fp32.  The consumer the quantized layer exists for
// (dingiv.github.io "量化" page, section GPTQ: 4-bit weights speed up
// memory-bound batch-1 decoding).
//
// The pass is bound by reading the packed weights once (d_row d_col / 2
// bytes), so two things decide its speed: enough bytes in flight to cover
// HBM latency, and per-code arithmetic far below the SM's issue rate.
//
// Arithmetic.  Converting each code with I2F (a quarter-rate pipe) and doing
// one FMA per code and activation row would be ALU-bound well below HBM
// bandwidth.  Instead the contraction runs on mma.sync m16n8k16 (bf16 in,
// fp32 accumulate) with the activation rows as the N = 8 side:
//   - a code q becomes the bf16 value 128 + q with one LOP3 (OR-ing the
//     nibble into the mantissa of 128.0: bf16 keeps 8 significant bits, so
//     128..143 are exact), two codes per 32-bit op; subtracting 128 + z
//     with one bf16x2 subtraction leaves q - z exactly;
//   - the products (q - z) x are exact in fp32 (8-bit by 5-bit
//     significands); only the fp32 accumulation rounds;
//   - the scale multiplies an fp32 partial sum once per region of 32 V
//     columns (all inside one group), or once per row when scales are
//     per channel.
// The k order inside one mma is free as long as A and B agree on it, so the
// row-major GPTQ words are used as they are (no repacking): lane (g, t)
// holds for rows g and g + 8 the word w(t) and for activation row g the
// same 8 columns; one word feeds two mma steps, slots (2t, 2t+1, 2t+8,
// 2t+9) taking codes (0, 4, 1, 5) of the word and then (2, 6, 3, 7).  The
// activations are permuted to match with two PRMTs per register pair.
//
// Memory.  A CTA owns 16-row tiles (persistent: tile = blockIdx.x + i
// gridDim.x); its 8 warps split each tile's columns into work items of 16
// rows x 128 CPI columns (warp w: items w, w + 8, ...; CPI = 2 where the
// scale regions are whole chunks and the batch is at most 4, else 1), and a
// shared-memory sum over the warps at the end of the tile gives Y.  Each
// warp streams its own items through a private ring of D shared-memory slots
// with 16-byte cp.async copies (an item's weights and activation rows), D - 1
// items ahead of the one it computes (D from 2 to 8, sized to 13.5 KB per
// warp), so no other warp and no barrier sits on its path; at batch 1 the 16
// warps of an SM keep 96 KB of weights in flight.  The slots' row pitches
// make every shared-memory read below free of bank conflicts: lane t of a
// quad holds word 4 j + t of each 128-column chunk (j = 0..3), so mma pair j
// covers 32 consecutive columns; the weight pitch is an odd number of
// 16-byte units (the 32-bit reads of 8 rows fall in 8 distinct groups of 4
// banks) and the activation pitch is 4 mod 8 units (the 16-byte reads of 2
// rows fall in distinct halves).  Scales and zero points of the next item
// are loaded into registers one item ahead.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace gptq {
namespace w4a16 {



constexpr int WARPS = 8;
constexpr int THREADS = WARPS * 32;
constexpr int ROWS = 16;     // rows per tile (one mma M tile)
constexpr int CHUNK_W = 16;  // words per chunk: 128 columns
constexpr int MAX_DEPTH = 8;
constexpr int WARP_BUDGET = 13824;  // ring bytes per warp: 2 CTAs of 8 warps per SM
constexpr int RED_BYTES = WARPS * 32 * 4 * 4;

// An item is CPI chunks of 16 rows.  Pitches in 16-byte units: odd for the
// weights (8 rows x 16 B per 32-bit read phase land in distinct bank
// groups), = 4 mod 8 for the activations (2 rows x 64 B per 16-byte read
// phase).
template <int CPI>
struct Geom {
  static constexpr int ITEM_W = CPI * CHUNK_W;  // words per item row
  static constexpr int PITCH_A = ITEM_W * 4 + 16;
  static constexpr int PITCH_X = ITEM_W * 16 + 64;
  static constexpr int A_SLOT = ROWS * PITCH_A;
  static_assert((PITCH_A / 16) % 2 == 1 && (PITCH_X / 16) % 8 == 4, "bank-conflict-free pitches");
};

__host__ __device__ constexpr int slot_bytes(int cpi, int batch) {
  return ROWS * (cpi * CHUNK_W * 4 + 16) + batch * (cpi * CHUNK_W * 16 + 64);
}
__host__ __device__ constexpr int ring_depth(int cpi, int batch) {
  return WARP_BUDGET / slot_bytes(cpi, batch) > MAX_DEPTH
             ? MAX_DEPTH
             : (WARP_BUDGET / slot_bytes(cpi, batch) < 2 ? 2 : WARP_BUDGET / slot_bytes(cpi, batch));
}
__host__ __device__ constexpr int smem_bytes(int cpi, int batch) {
  return WARPS * ring_depth(cpi, batch) * slot_bytes(cpi, batch) + RED_BYTES;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most n of this thread's copy groups are pending (n < 8).
__device__ __forceinline__ void cp_async_wait(int n) {
  switch (n) {
    case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
    case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
    case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
    case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
    case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
    default: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
  }
}

__device__ __forceinline__ uint32_t code_pair(uint32_t v) {
  // lo = 128 + code at bits 0..3, hi = 128 + code at bits 16..19, both bf16
  return (v & 0x000F000Fu) | 0x43004300u;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                             *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t zero_pair(int z) {
  const uint32_t b = 0x4300u | static_cast<uint32_t>(z);  // bf16 128 + z
  return b | (b << 16);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One word of rows g, g+8 (vg, vh) and the matching 8 activations xv of
// activation row g: two mma steps into d.
__device__ __forceinline__ void word_mma(float (&d)[4], uint32_t vg, uint32_t vh, uint32_t zg,
                                         uint32_t zh, const uint4& xv) {
  const uint32_t g0 = bf16x2_sub(code_pair(vg), zg), h0 = bf16x2_sub(code_pair(vh), zh);
  const uint32_t g1 = bf16x2_sub(code_pair(vg >> 4), zg), h1 = bf16x2_sub(code_pair(vh >> 4), zh);
  mma_bf16_16816(d, g0, h0, g1, h1, __byte_perm(xv.x, xv.z, 0x5410),
                 __byte_perm(xv.x, xv.z, 0x7632));
  const uint32_t g2 = bf16x2_sub(code_pair(vg >> 8), zg), h2 = bf16x2_sub(code_pair(vh >> 8), zh);
  const uint32_t g3 = bf16x2_sub(code_pair(vg >> 12), zg),
                 h3 = bf16x2_sub(code_pair(vh >> 12), zh);
  mma_bf16_16816(d, g2, h2, g3, h3, __byte_perm(xv.y, xv.w, 0x5410),
                 __byte_perm(xv.y, xv.w, 0x7632));
}

// The copies a lane issues for its warp's items.  Lane l copies, of each
// item, the 16-byte weight piece l % PPR of rows l / PPR + RPP k (k <
// 16 / RPP) and the activation word l % ITEM_W of rows l / ITEM_W + XPP k:
// fixed per lane, so an item costs a pointer offset and the copies.  Rows
// past d_row and words past the row end are not copied; what the slot holds
// there is never used for a written output.
template <int CPI>
struct Fetcher {
  using Gm = Geom<CPI>;
  static constexpr int PPR = Gm::ITEM_W / 4;  // weight pieces per row
  static constexpr int RPP = 32 / PPR;        // weight rows per pass
  static constexpr int XPP = 32 / Gm::ITEM_W;  // activation rows per pass
  const uint32_t* wrow;                        // row l / PPR of the tile, piece l % PPR
  const __nv_bfloat16* xrow;                   // activation row l / ITEM_W, word l % ITEM_W
  uint32_t rows_ok;                            // bit k: row l / PPR + RPP k < d_row
  int wstride;                                 // RPP rows, in words
  uint32_t dst_a, dst_x;                       // offsets inside a slot

  __device__ __forceinline__ void init(const __nv_bfloat16* X, int lane, int d_col) {
    xrow = X + static_cast<size_t>(lane / Gm::ITEM_W) * d_col + (lane % Gm::ITEM_W) * 8;
    dst_a = (lane / PPR) * Gm::PITCH_A + (lane % PPR) * 16;
    dst_x = Gm::A_SLOT + (lane / Gm::ITEM_W) * Gm::PITCH_X + (lane % Gm::ITEM_W) * 16;
  }
  __device__ __forceinline__ void tile(const uint32_t* qweight, int row0, int d_row, int words,
                                       int lane) {
    const int r = row0 + lane / PPR;
    wrow = qweight + static_cast<size_t>(min(r, d_row - 1)) * words + (lane % PPR) * 4;
    wstride = RPP * words;
    rows_ok = 0;
#pragma unroll
    for (int k = 0; k < ROWS / RPP; ++k) rows_ok |= (r + RPP * k < d_row ? 1u : 0u) << k;
  }
  __device__ __forceinline__ void item(uint32_t slot, int w0, int words, int d_col, int batch,
                                       int lane) const {
    const bool full = w0 + Gm::ITEM_W <= words;
    const bool a_in = full || 4 * (lane % PPR) < words - w0;
    const uint32_t* src = wrow + w0;
#pragma unroll
    for (int k = 0; k < ROWS / RPP; ++k)
      if (a_in && ((rows_ok >> k) & 1u))
        cp_async16(slot + dst_a + k * RPP * Gm::PITCH_A, src + static_cast<size_t>(k) * wstride);
    if (full || lane % Gm::ITEM_W < words - w0) {
      const __nv_bfloat16* xs = xrow + static_cast<size_t>(w0) * 8;
      for (int n = lane / Gm::ITEM_W, k = 0; n < batch; n += XPP, ++k)
        cp_async16(slot + dst_x + k * XPP * Gm::PITCH_X, xs + static_cast<size_t>(k) * XPP * d_col);
    }
  }
};

// Scale and zero point of rows g and g + 8 for each scale region of one
// item: NS = CPI 4 / GJ regions of 32 GJ columns (GJ = 0: one per row).
template <int GJ, int CPI>
struct RowParams {
  static constexpr int NS = GJ ? CPI * 4 / GJ : 1;
  float sg[NS], sh[NS];
  uint32_t zg[NS], zh[NS];
};

// Rows g and g + 8 of a tile, clamped into the layer (rows past d_row are
// computed on a real row's parameters and never written).
struct RowPtrs {
  const float *sg, *sh;
  const uint8_t *zg, *zh;
};

__device__ __forceinline__ RowPtrs row_ptrs(const float* __restrict__ scales,
                                            const uint8_t* __restrict__ zeros, int tile, int g,
                                            int d_row, int n_groups) {
  const int rg = min(tile * ROWS + g, d_row - 1), rh = min(tile * ROWS + g + 8, d_row - 1);
  const size_t og = static_cast<size_t>(rg) * n_groups, oh = static_cast<size_t>(rh) * n_groups;
  return RowPtrs{scales + og, scales + oh, zeros + og, zeros + oh};
}

// Parameters of the item starting at word w0.  gmagic = ceil(2^32 / group):
// umulhi(k, gmagic) is k / group exactly for k, group < 2^16.
template <int GJ, int CPI>
__device__ __forceinline__ void load_params(RowParams<GJ, CPI>& p, const RowPtrs& rp, int w0,
                                            int last_group, uint32_t gmagic) {
#pragma unroll
  for (int m = 0; m < RowParams<GJ, CPI>::NS; ++m) {
    int gi = 0;
    if (GJ) {
      const uint32_t k0 = static_cast<uint32_t>((w0 + 4 * GJ * m) * 8);
      gi = min(static_cast<int>(__umulhi(k0, gmagic)), last_group);  // past the end: clamped
    }
    p.sg[m] = __ldg(rp.sg + gi);
    p.sh[m] = __ldg(rp.sh + gi);
    p.zg[m] = zero_pair(__ldg(rp.zg + gi));
    p.zh[m] = zero_pair(__ldg(rp.zh + gi));
  }
}

// GJ: mma pairs (32 columns each) per scale region: 1 (groups of 32 k),
// 2 (64 k), 4 (multiples of 128 k); 0 for one scale per output channel.
// CPI: 128-column chunks per work item.  depth: ring slots per warp.
template <int GJ, int CPI>
__global__ void __launch_bounds__(THREADS, 2)
w4a16_matmul_kernel(const uint32_t* __restrict__ qweight, const float* __restrict__ scales,
                    const uint8_t* __restrict__ zeros, const __nv_bfloat16* __restrict__ X,
                    float* __restrict__ Y, int d_row, int d_col, int batch, uint32_t gmagic,
                    int n_groups, int depth) {
  using Gm = Geom<CPI>;
  using Params = RowParams<GJ, CPI>;
  constexpr int NSC = GJ ? 4 / GJ : 1;  // scale regions per chunk
  extern __shared__ __align__(128) uint8_t w4sm[];
  const int SB = Gm::A_SLOT + batch * Gm::PITCH_X;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  uint8_t* ring = w4sm + warp * depth * SB;
  const uint32_t ring_s = smem_u32(ring);
  float(*red)[32][4] = reinterpret_cast<float(*)[32][4]>(w4sm + WARPS * depth * SB);

  const int words = d_col / 8;
  const int nchunks = (words + CHUNK_W - 1) / CHUNK_W;
  const int nitems = (words + Gm::ITEM_W - 1) / Gm::ITEM_W;  // per tile, over all warps
  const int ntiles = (d_row + ROWS - 1) / ROWS;
  const int last_group = n_groups - 1;

  // fetch cursor: the warp's items in order (tile, item = warp, warp + 8, ...)
  int f_tile = warp < nitems ? static_cast<int>(blockIdx.x) : ntiles, f_item = warp;
  uint32_t f_slot = ring_s;
  const uint32_t ring_end = ring_s + depth * SB;
  Fetcher<CPI> fe;
  fe.init(X, lane, d_col);
  if (f_tile < ntiles) fe.tile(qweight, f_tile * ROWS, d_row, words, lane);
#define W4_FETCH_NEXT()                                                       \
  do {                                                                        \
    if (f_tile < ntiles) {                                                    \
      fe.item(f_slot, f_item * Gm::ITEM_W, words, d_col, batch, lane);        \
      f_item += WARPS;                                                        \
      if (f_item >= nitems) {                                                 \
        f_item = warp;                                                        \
        f_tile += gridDim.x;                                                  \
        if (f_tile < ntiles) fe.tile(qweight, f_tile * ROWS, d_row, words, lane); \
      }                                                                       \
    }                                                                         \
    cp_async_commit();                                                        \
    f_slot += SB;                                                             \
    if (f_slot == ring_end) f_slot = ring_s;                                  \
  } while (0)

  for (int k = 0; k < depth - 1; ++k) W4_FETCH_NEXT();

  // activation lanes past the batch read row 0: their output columns are
  // never written (an mma output column depends only on its own B column)
  const int xr = g < batch ? g : 0;
  const int a_off = g * Gm::PITCH_A + t * 4;
  const int x_off = Gm::A_SLOT + xr * Gm::PITCH_X + t * 16;
  int c_slot = 0;
  RowPtrs rp = row_ptrs(scales, zeros, blockIdx.x, g, d_row, n_groups);
  Params nxt;
  load_params<GJ, CPI>(nxt, rp, warp * Gm::ITEM_W, last_group, gmagic);
  Params cur = nxt;

  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
    for (int item = warp; item < nitems; item += WARPS) {
      W4_FETCH_NEXT();  // depth - 1 items ahead
      cur = nxt;        // scales and zero points one item ahead
      {
        int ntile = tile, nitem = item + WARPS;
        if (nitem >= nitems) {
          nitem = warp;
          ntile += gridDim.x;
          if (ntile < ntiles) rp = row_ptrs(scales, zeros, ntile, g, d_row, n_groups);
        }
        // one scale per row: loaded when the next item starts a new tile
        if (ntile < ntiles && (GJ != 0 || ntile != tile))
          load_params<GJ, CPI>(nxt, rp, nitem * Gm::ITEM_W, last_group, gmagic);
      }
      cp_async_wait(depth - 1);
      __syncwarp();
      const uint8_t* sl = ring + c_slot * SB;
#pragma unroll
      for (int ch = 0; ch < CPI; ++ch) {
        const int c = item * CPI + ch;  // chunk index in the row
        if (c >= nchunks) break;
        uint32_t vg[4], vh[4];
        uint4 xv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          vg[j] = *reinterpret_cast<const uint32_t*>(sl + a_off + ch * 64 + 16 * j);
          vh[j] = *reinterpret_cast<const uint32_t*>(sl + a_off + 8 * Gm::PITCH_A + ch * 64 + 16 * j);
          xv[j] = *reinterpret_cast<const uint4*>(sl + x_off + (ch * CHUNK_W + 4 * j) * 16);
        }
        // a partial last chunk: 32-column runs past the row end are skipped
        // (the slot holds stale words and activations there)
        const int runs = min(4, (words - c * CHUNK_W) / 4);
        if (GJ == 0) {
          if (runs == 4) {
            word_mma(acc0, vg[0], vh[0], cur.zg[0], cur.zh[0], xv[0]);
            word_mma(acc1, vg[1], vh[1], cur.zg[0], cur.zh[0], xv[1]);
            word_mma(acc0, vg[2], vh[2], cur.zg[0], cur.zh[0], xv[2]);
            word_mma(acc1, vg[3], vh[3], cur.zg[0], cur.zh[0], xv[3]);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              if (j < runs) word_mma(acc0, vg[j], vh[j], cur.zg[0], cur.zh[0], xv[j]);
          }
        } else {
#pragma unroll
          for (int m = 0; m < NSC; ++m) {
            const int sm_ = ch * NSC + m;
            float p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < GJ; ++i) {
              const int j = m * GJ + i;
              if (j < runs) word_mma((i & 1) ? p1 : p0, vg[j], vh[j], cur.zg[sm_], cur.zh[sm_], xv[j]);
            }
            acc0[0] = fmaf(cur.sg[sm_], p0[0] + p1[0], acc0[0]);
            acc0[1] = fmaf(cur.sg[sm_], p0[1] + p1[1], acc0[1]);
            acc0[2] = fmaf(cur.sh[sm_], p0[2] + p1[2], acc0[2]);
            acc0[3] = fmaf(cur.sh[sm_], p0[3] + p1[3], acc0[3]);
          }
        }
      }
      __syncwarp();  // the slot is refilled by the next fetch
      if (++c_slot == depth) c_slot = 0;
    }

    // end of the tile: sum over the warps.  Fragment element i of lane l is
    // row (l >> 2) + 8 (i >> 1), activation row 2 (l & 3) + (i & 1).
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = acc0[i] + acc1[i];
    if (GJ == 0) {  // one scale per row: this tile's, held since its first item
      v[0] *= cur.sg[0];
      v[1] *= cur.sg[0];
      v[2] *= cur.sh[0];
      v[3] *= cur.sh[0];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][lane][i] = v[i];
    __syncthreads();
    if (threadIdx.x < 128) {
      const int l = threadIdx.x >> 2, i = threadIdx.x & 3;
      float y = 0.f;
#pragma unroll
      for (int w = 0; w < WARPS; ++w) y += red[w][l][i];
      const int r = tile * ROWS + (l >> 2) + 8 * (i >> 1), n = 2 * (l & 3) + (i & 1);
      if (r < d_row && n < batch) Y[static_cast<size_t>(n) * d_row + r] = y;
    }
    __syncthreads();
  }
#undef W4_FETCH_NEXT
  cp_async_wait(0);
}

// ------------------------------------------------------------------------
// Layers with one scale per output channel, or per group of a multiple of
// 128 columns (the common GPTQ settings): a leaner layout with no staging.
//
// A CTA owns 32 rows (two 16-row mma tiles per warp) and its 8 warps split
// the 128-column chunks of the row (warp w: chunks w, w + 8, ...); one
// shared-memory sum over the warps at the end gives Y.  Lane (g, t) loads,
// for rows g and g + 8 of each tile, the 16 bytes holding words 4t..4t+3 of
// the chunk (columns 32t..32t+31): a quad reads 64 contiguous bytes of a row
// with one 128-bit load each, straight into registers, and the next chunk's
// loads are issued before the current chunk is computed.  Within a chunk the
// k order is free (A and B agree on it): mma pair j takes word 4t + j of
// every lane, slots (2t, 2t+1, 2t+8, 2t+9) holding codes (0, 4, 1, 5) of the
// word and then (2, 6, 3, 7), so a pair spans the whole chunk, which is why
// a scale region must cover whole chunks here.  The activations of those
// columns (batch row g) are loaded and permuted once per chunk and serve
// both tiles.  Decoding a word: code c of the word becomes the bf16 128 + c
// with one LOP3 per pair of codes (three shifts per word), and one bf16x2
// subtraction of 128 + z gives c - z exactly.
constexpr int WT = 2;             // 16-row tiles per warp
constexpr int W_ROWS = ROWS * WT;  // rows per CTA

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t word_at(const uint4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// Rows g, g + 8 of one tile, word j of the lane's piece: two mma steps.
__device__ __forceinline__ void tile_word_mma(float (&d)[4], uint32_t vg, uint32_t vh,
                                              uint32_t zg, uint32_t zh, const uint32_t (&b)[4]) {
  const uint32_t g0 = bf16x2_sub(code_pair(vg), zg), h0 = bf16x2_sub(code_pair(vh), zh);
  const uint32_t g1 = bf16x2_sub(code_pair(vg >> 4), zg), h1 = bf16x2_sub(code_pair(vh >> 4), zh);
  mma_bf16_16816(d, g0, h0, g1, h1, b[0], b[1]);
  const uint32_t g2 = bf16x2_sub(code_pair(vg >> 8), zg), h2 = bf16x2_sub(code_pair(vh >> 8), zh);
  const uint32_t g3 = bf16x2_sub(code_pair(vg >> 12), zg), h3 = bf16x2_sub(code_pair(vh >> 12), zh);
  mma_bf16_16816(d, g2, h2, g3, h3, b[2], b[3]);
}

template <bool PER_CHANNEL>
__global__ void __launch_bounds__(THREADS, 2)
w4a16_wide_kernel(const uint32_t* __restrict__ qweight, const float* __restrict__ scales,
                  const uint8_t* __restrict__ zeros, const __nv_bfloat16* __restrict__ X,
                  float* __restrict__ Y, int d_row, int d_col, int batch, int group,
                  int n_groups) {
  __shared__ float red[WARPS][WT][32][4];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int words = d_col >> 3;
  const int nchunks = (d_col + 127) >> 7;
  const int row0 = blockIdx.x * W_ROWS;
  // the lane's rows, clamped into the layer for the loads (rows past d_row
  // are computed on a real row and never written)
  const uint4* wrow[WT][2];
  int prow[WT][2];
#pragma unroll
  for (int i = 0; i < WT; ++i)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = min(row0 + ROWS * i + g + 8 * h, d_row - 1);
      prow[i][h] = r;
      wrow[i][h] = reinterpret_cast<const uint4*>(qweight + static_cast<size_t>(r) * words) + t;
    }
  const bool xrow_ok = g < batch;
  const uint4* xrow = reinterpret_cast<const uint4*>(X + static_cast<size_t>(xrow_ok ? g : 0) * d_col) + 4 * t;

  // one chunk's inputs: the lane's weight pieces, its activations, and (for
  // groups) the scales and zero points of its rows
  struct In {
    uint4 w[WT][2];
    uint4 x[4];
    float s[WT][2];
    uint32_t z[WT][2];
  };
  auto load = [&](int cc, In& in) {
    const bool lv = 128 * cc + 32 * t < d_col;  // this lane's 32 columns exist
#pragma unroll
    for (int i = 0; i < WT; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        in.w[i][h] = lv ? ld_stream_v4(wrow[i][h] + 4 * cc) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      in.x[j] = (lv && xrow_ok) ? __ldg(xrow + 16 * cc + j) : make_uint4(0u, 0u, 0u, 0u);
    if (!PER_CHANNEL) {
      const int gi = (128 * cc) / group;
#pragma unroll
      for (int i = 0; i < WT; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const size_t o = static_cast<size_t>(prow[i][h]) * n_groups + gi;
          in.s[i][h] = __ldg(scales + o);
          in.z[i][h] = zero_pair(__ldg(zeros + o));
        }
    }
  };

  uint32_t zc[WT][2];
  if (PER_CHANNEL) {
#pragma unroll
    for (int i = 0; i < WT; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) zc[i][h] = zero_pair(__ldg(zeros + prow[i][h]));
  }
  float acc[WT][4];
#pragma unroll
  for (int i = 0; i < WT; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.0f;

  In cur, nxt;
  if (warp < nchunks) load(warp, cur);
  for (int c = warp; c < nchunks; c += WARPS) {
    if (c + WARPS < nchunks) load(c + WARPS, nxt);  // in flight while this chunk computes
    // B fragments of the chunk's 4 words: (x0, x4), (x1, x5), (x2, x6), (x3, x7)
    uint32_t b[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      b[j][0] = __byte_perm(cur.x[j].x, cur.x[j].z, 0x5410);
      b[j][1] = __byte_perm(cur.x[j].x, cur.x[j].z, 0x7632);
      b[j][2] = __byte_perm(cur.x[j].y, cur.x[j].w, 0x5410);
      b[j][3] = __byte_perm(cur.x[j].y, cur.x[j].w, 0x7632);
    }
#pragma unroll
    for (int i = 0; i < WT; ++i) {
      if (PER_CHANNEL) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tile_word_mma(acc[i], word_at(cur.w[i][0], j), word_at(cur.w[i][1], j), zc[i][0],
                        zc[i][1], b[j]);
      } else {
        float part[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tile_word_mma(part, word_at(cur.w[i][0], j), word_at(cur.w[i][1], j), cur.z[i][0],
                        cur.z[i][1], b[j]);
        acc[i][0] = fmaf(cur.s[i][0], part[0], acc[i][0]);
        acc[i][1] = fmaf(cur.s[i][0], part[1], acc[i][1]);
        acc[i][2] = fmaf(cur.s[i][1], part[2], acc[i][2]);
        acc[i][3] = fmaf(cur.s[i][1], part[3], acc[i][3]);
      }
    }
    cur = nxt;
  }
  if (PER_CHANNEL) {
#pragma unroll
    for (int i = 0; i < WT; ++i) {
      const float sg = __ldg(scales + prow[i][0]), sh = __ldg(scales + prow[i][1]);
      acc[i][0] *= sg; acc[i][1] *= sg; acc[i][2] *= sh; acc[i][3] *= sh;
    }
  }
  // sum over the warps.  Fragment element e of lane l is row (l >> 2) +
  // 8 (e >> 1) of the tile, activation row 2 (l & 3) + (e & 1).
#pragma unroll
  for (int i = 0; i < WT; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) red[warp][i][lane][e] = acc[i][e];
  __syncthreads();
  {
    const int i = threadIdx.x >> 7, l = (threadIdx.x >> 2) & 31, e = threadIdx.x & 3;
    float y = 0.0f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) y += red[w][i][l][e];
    const int r = row0 + ROWS * i + (l >> 2) + 8 * (e >> 1), n = 2 * (l & 3) + (e & 1);
    if (r < d_row && n < batch) Y[static_cast<size_t>(n) * d_row + r] = y;
  }
}

}  // namespace w4a16
}  // namespace gptq
