// extern "C" entry points of libgptq.so (declared in include/gptq.h): argument
// validation, workspace layout, TMA descriptor encoding and the launch
// sequences of the GPTQ stages.  All device kernels are in the .cuh files
// included below, compiled as one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/gptq.h"
#include "chol_fp64.cuh"
#include "common.cuh"
#include "quantize.cuh"
#include "syrk_tcgen05.cuh"
#include "trailing_tf32.cuh"
#include "w4a16.cuh"
#include "awq.cuh"

namespace {

using namespace gptq;

// Shape of the factorization's trailing-update DGEMM (U_k): TM, WGM, warps
// per group, tile columns, groups, K slice, stages.
#ifndef GPTQ_UK_SHAPE
#define GPTQ_UK_SHAPE 128, 4, 8, 64, 2, 16, 3
#endif
template <int TM, int WGM, int NW, int TNG, int NG, int TKG, int STG>
constexpr int gemm_smem_of() { return chol::gemm_smem<TM, TNG, NG, TKG, STG>(); }

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

#define GPTQ_CUDA_TRY(expr)                          \
  do {                                               \
    cudaError_t e_ = (expr);                         \
    if (e_ != cudaSuccess) {                         \
      std::fprintf(stderr, "gptq: %s failed: %s\n", #expr, cudaGetErrorString(e_)); \
      return GPTQ_ERR_CUDA;                          \
    }                                                \
  } while (0)

std::atomic<uint64_t> g_launches{0};

// Fault injection for the failure-detection tests (gptq_fault_inject): which
// kernel's producer stalls, and the limit of every bounded wait.
std::atomic<int> g_fault{GPTQ_FAULT_NONE};
std::atomic<uint64_t> g_wait_ns{gptq::kWaitLimitNs};

#define GPTQ_LAUNCH_CHECK()                          \
  do {                                               \
    g_launches.fetch_add(1, std::memory_order_relaxed); \
    cudaError_t e_ = cudaGetLastError();             \
    if (e_ != cudaSuccess) {                         \
      std::fprintf(stderr, "gptq: launch failed at %s:%d: %s\n", __FILE__, __LINE__, \
                   cudaGetErrorString(e_));          \
      return GPTQ_ERR_CUDA;                          \
    }                                                \
  } while (0)

// ------------------------------------------------------------ device setup
constexpr int kEvents = 10;  // fork, join, 4 block-step and 4 trailing-update events

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  // The column sweep runs the block steps on the caller's stream and the
  // trailing updates on this auxiliary stream, joined by events; qmu keeps
  // calls from several host threads from interleaving on them.
  cudaStream_t aux = nullptr;
  cudaEvent_t ev[kEvents] = {};
  std::mutex qmu;
};

std::mutex g_mu;
DeviceInfo g_dev[64];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

DeviceInfo* current_device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  return &g_dev[dev];
}

gptq_status device_setup(int* num_sms) {
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.ready) {
    GPTQ_CUDA_TRY(cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, dev));
    for (const void* f : {reinterpret_cast<const void*>(w4a16::w4a16_matmul_kernel<0, 1>),
                          reinterpret_cast<const void*>(w4a16::w4a16_matmul_kernel<0, 2>),
                          reinterpret_cast<const void*>(w4a16::w4a16_matmul_kernel<4, 1>),
                          reinterpret_cast<const void*>(w4a16::w4a16_matmul_kernel<4, 2>),
                          reinterpret_cast<const void*>(w4a16::w4a16_matmul_kernel<2, 1>),
                          reinterpret_cast<const void*>(w4a16::w4a16_matmul_kernel<1, 1>)})
      GPTQ_CUDA_TRY(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         w4a16::WARPS * w4a16::WARP_BUDGET + w4a16::RED_BYTES));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(syrk::syrk_bf16_tcgen05_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       syrk::SMEM_BYTES));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(chol::dgemm_nt_kernel<GPTQ_UK_SHAPE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       gemm_smem_of<GPTQ_UK_SHAPE>()));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(chol::dgemm_nt_kernel<64, 2>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       chol::gemm_smem<64>()));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(chol::dgemm_nt_kernel<32, 1>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       chol::gemm_smem<32>()));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(chol::leaf_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       chol::LEAF_SMEM));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(quant::block_step_kernel<128>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       quant::block_step_smem<128>()));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(quant::block_step_kernel<64>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       quant::block_step_smem<64>()));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(quant::block_step_kernel<32>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       quant::block_step_smem<32>()));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(quant::block_step_kernel<128, true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       quant::block_step_smem<128>()));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(trail::trailing_tf32x3_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       trail::SMEM_BYTES));
    // The column sweep runs a step CTA and a trailing-update CTA side by side
    // on each SM (two streams).  Their shared memory only fits together with
    // the largest shared-memory carveout; left to itself the driver may size
    // an SM's carveout for the first kernel alone, and the other then waits
    // for that SM to drain.
    for (const void* f : {reinterpret_cast<const void*>(quant::block_step_kernel<128>),
                          reinterpret_cast<const void*>(quant::block_step_kernel<64>),
                          reinterpret_cast<const void*>(quant::block_step_kernel<32>),
                          reinterpret_cast<const void*>(quant::block_step_kernel<128, true>),
                          reinterpret_cast<const void*>(trail::trailing_tf32x3_kernel)})
      GPTQ_CUDA_TRY(cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         cudaSharedmemCarveoutMaxShared));
    GPTQ_CUDA_TRY(cudaStreamCreateWithFlags(&di.aux, cudaStreamNonBlocking));
    for (int i = 0; i < kEvents; ++i)
      GPTQ_CUDA_TRY(cudaEventCreateWithFlags(&di.ev[i], cudaEventDisableTiming));
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      GPTQ_CUDA_TRY(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
      if (q != cudaDriverEntryPointSuccess || !fn) return GPTQ_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    di.ready = true;
  }
  if (num_sms) *num_sms = di.num_sms;
  return GPTQ_OK;
}

bool config_ok(const gptq_config* c, int64_t d_col) {
  if (!c) return false;
  if (c->bits < 2 || c->bits > 8) return false;
  if (c->block != 32 && c->block != 64 && c->block != 128) return false;
  if (c->sym != 0 && c->sym != 1) return false;
  if (!(c->damp_rel >= 0.0) || !std::isfinite(c->damp_rel)) return false;
  const int g = c->group_size;
  if (g < 0) return false;
  if (g > 0) {
    if (g % 32 != 0) return false;
    if (d_col % g != 0) return false;
    if (!(c->block % g == 0 || g % c->block == 0)) return false;
  }
  return true;
}

// ---------------------------------------------------------- workspace map
struct PrepareWs {
  size_t stats, istat, pivot, A, Mt, Xd, total;
};
PrepareWs prepare_layout(int64_t d) {
  PrepareWs w{};
  size_t off = 0;
  w.stats = off; off = align_up(off + 8);
  w.istat = off; off = align_up(off + 8);
  w.pivot = off; off = align_up(off + 8);
  w.A = off; off = align_up(off + static_cast<size_t>(d) * d * 8);
  w.Mt = off; off = align_up(off + static_cast<size_t>(d) * d * 8);
  const int64_t nt = (d + chol::NB - 1) / chol::NB;
  w.Xd = off; off = align_up(off + static_cast<size_t>(nt) * chol::NB * chol::NB * 8);
  w.total = off;
  return w;
}

struct QuantWs {
  size_t Wk, E[2][3], Ghi, Glo, total;  // E[window buffer][hi / lo / as it is]
  int lde;                              // E row stride: one window of blocks
};
QuantWs quant_layout(int64_t d_row, int64_t d_col, int block) {
  QuantWs w{};
  w.lde = quant::sweep_window_blocks(d_col) * block;
  size_t off = 0;
  w.Wk = off; off = align_up(off + static_cast<size_t>(d_row) * d_col * 4);
  for (int b = 0; b < 2; ++b)
    for (int h = 0; h < 3; ++h) {
      w.E[b][h] = off;
      off = align_up(off + static_cast<size_t>(d_row) * w.lde * 4);
    }
  w.Ghi = off; off = align_up(off + static_cast<size_t>(d_col) * d_col * 4);
  w.Glo = off; off = align_up(off + static_cast<size_t>(d_col) * d_col * 4);
  w.total = off;
  return w;
}

struct CheckWs {
  size_t partials, loss, total;
};
CheckWs check_layout(int64_t d_row, int64_t d_col) {
  CheckWs w{};
  const size_t tiles = static_cast<size_t>((d_row + 127) / 128) * ((d_col + 127) / 128);
  size_t off = 0;
  w.partials = off; off = align_up(off + tiles * 8);
  w.loss = off; off = align_up(off + 8);
  w.total = off;
  return w;
}

// ------------------------------------------------------------------ AWQ
struct AwqWs {
  size_t Hhi, Hlo, Ehi, Elo, T, s, partials, total;
};
AwqWs awq_layout(int64_t d_row, int64_t d_col) {
  AwqWs w{};
  size_t off = 0;
  const size_t hh = static_cast<size_t>(d_col) * d_col * 4, ww = static_cast<size_t>(d_row) * d_col * 4;
  w.Hhi = off; off = align_up(off + hh);
  w.Hlo = off; off = align_up(off + hh);
  w.Ehi = off; off = align_up(off + ww);
  w.Elo = off; off = align_up(off + ww);
  w.T = off; off = align_up(off + ww);
  w.s = off; off = align_up(off + static_cast<size_t>(d_col) * 4);
  w.partials = off; off = align_up(off + awq::DOT_BLOCKS * 8);
  w.total = off;
  return w;
}

bool awq_config_ok(const gptq_config* cfg, int64_t d_row, int64_t d_col) {
  // the per-(row, group) work items are counted in int
  return config_ok(cfg, d_col) && cfg->bits == 4 && cfg->sym == 0 && d_row >= 1 &&
         d_row <= (int64_t(1) << 24) && d_col >= 32 && d_col % 32 == 0 && d_col <= 65536 &&
         d_row * d_col <= int64_t(INT32_MAX);
}

// 2D fp32 tensor map: dims {inner, outer}, row stride in elements, box {bx, by}.
gptq_status encode_f32_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer,
                          uint64_t row_stride, uint32_t bx, uint32_t by,
                          CUtensorMapSwizzle swz) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride * 4};
  const cuuint32_t box[2] = {bx, by};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) {
    std::fprintf(stderr, "gptq: cuTensorMapEncodeTiled (f32) failed (%d)\n", static_cast<int>(cr));
    return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

// A row-major fp32 matrix (rows x cols, cols a multiple of 32) seen as 3-D
// for TMA: x = the 32 columns of one 128-byte chunk, y = the row, z = the
// chunk.  One box of 32 x by x nz lands in shared memory as nz chunks of
// by rows of 128 bytes, each chunk by * 128 bytes after the previous: the
// layout of an MN-major operand in 128-byte-swizzled atoms, fetched with one
// copy instead of nz.
gptq_status encode_f32_chunks(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                              uint64_t row_stride, uint32_t by, uint32_t nz,
                              CUtensorMapSwizzle swz) {
  const cuuint64_t dims[3] = {32, rows, cols / 32};
  const cuuint64_t strides[2] = {row_stride * 4, 128};
  const cuuint32_t box[3] = {32, by, nz};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult cr = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) {
    std::fprintf(stderr, "gptq: cuTensorMapEncodeTiled (f32 chunks) failed (%d)\n",
                 static_cast<int>(cr));
    return GPTQ_ERR_CUDA;
  }
  return GPTQ_OK;
}

// --------------------------------------------------------- SYRK launching
void choose_split(int ntiles, int n, int num_sms, int* split_tokens, int* nsplit) {
  const int nkb = (n + syrk::BK - 1) / syrk::BK;
  double best = 1e300;
  int best_s = 1;
  const int max_s = std::max(1, std::min(64, nkb));
  for (int s = 1; s <= max_s; ++s) {
    const int kb_per = (nkb + s - 1) / s;
    const int s_eff = (nkb + kb_per - 1) / kb_per;
    const long long units = static_cast<long long>(ntiles) * s_eff;
    const long long waves = (units + num_sms - 1) / num_sms;
    // a unit costs its k-stages plus a fixed ramp/epilogue share
    const double cost = static_cast<double>(waves) * (kb_per + 6);
    if (cost < best * 0.999) { best = cost; best_s = s; }
  }
  const int kb_per = (nkb + best_s - 1) / best_s;
  *split_tokens = kb_per * syrk::BK;
  *nsplit = (nkb + kb_per - 1) / kb_per;
}

}  // namespace

namespace {

// Launch the grouped NT DGEMM with TM-row tiles: persistent CTAs, at most
// one per SM, leaving `reserve_sms` SMs free for work that must run beside
// it (a persistent grid on every SM would keep a later kernel on another
// stream from starting until it exits).  Problems with an empty output are
// dropped.
template <int TM, int WGM, int NW = 8, int TNG = chol::TN, int NG = 1, int TKG = chol::TK,
          int STG = chol::GSTAGES>
gptq_status launch_nt(const std::vector<chol::GemmProblem>& probs, cudaStream_t s,
                      int reserve_sms = 0) {
  int num_sms = 148;
  gptq_status st = device_setup(&num_sms);
  if (st != GPTQ_OK) return st;
  size_t i = 0;
  while (i < probs.size()) {
    chol::GemmBatch b{};
    int tiles = 0;
    while (i < probs.size() && b.count < chol::MAXP) {
      const chol::GemmProblem& q = probs[i++];
      if (q.M <= 0 || q.N <= 0) continue;
      const int tm = (q.M + TM - 1) / TM, tn = (q.N + TNG - 1) / TNG;
      b.tile_start[b.count] = tiles;
      b.p[b.count++] = q;
      tiles += q.lower_only ? chol::lower_tiles<TM, TNG>(q.M, q.N) : tm * tn;
    }
    b.tile_start[b.count] = tiles;
    const int grid = std::min((tiles + NG - 1) / NG, std::max(1, num_sms - reserve_sms));
    if (grid > 0) {
      chol::dgemm_nt_kernel<TM, WGM, NW, TNG, NG, TKG, STG>
          <<<grid, NG * NW * 32, chol::gemm_smem<TM, TNG, NG, TKG, STG>(), s>>>(b);
      GPTQ_LAUNCH_CHECK();
    }
  }
  return GPTQ_OK;
}

}  // namespace

extern "C" {

const char* gptq_status_string(gptq_status s) {
  switch (s) {
    case GPTQ_OK: return "GPTQ_OK";
    case GPTQ_ERR_INVALID: return "GPTQ_ERR_INVALID";
    case GPTQ_ERR_NOT_SPD: return "GPTQ_ERR_NOT_SPD";
    case GPTQ_ERR_NONFINITE: return "GPTQ_ERR_NONFINITE";
    case GPTQ_ERR_WORKSPACE: return "GPTQ_ERR_WORKSPACE";
    case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA";
    case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT";
  }
  return "GPTQ_ERR_UNKNOWN";
}

uint64_t gptq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t gptq_workspace_size(int64_t d_row, int64_t d_col, const gptq_config* cfg) {
  if (d_row < 1 || d_col < 32 || d_col % 32 != 0 || d_col > 65536 || !config_ok(cfg, d_col))
    return 0;
  const size_t a = prepare_layout(d_col).total;
  const size_t b = quant_layout(d_row, d_col, cfg->block).total;
  const size_t c = check_layout(d_row, d_col).total;
  return std::max(a, std::max(b, c));
}

gptq_status gptq_w4a16_matmul(const uint32_t* qweight, const float* scales,
                              const uint8_t* zeros, int64_t d_row, int64_t d_col,
                              const gptq_config* cfg, const void* X, int64_t batch,
                              float* Y, void* stream) {
  if (!qweight || !scales || !zeros || !X || !Y) return GPTQ_ERR_INVALID;
  if (d_row < 1 || d_row > (int64_t(1) << 24) || d_col < 32 || d_col % 32 != 0 ||
      d_col > 65536)
    return GPTQ_ERR_INVALID;
  if (!config_ok(cfg, d_col) || cfg->bits != 4) return GPTQ_ERR_INVALID;
  if (batch < 1 || batch > 8 || !aligned(X, 16) || !aligned(qweight, 16) || !aligned(scales, 4) ||
      !aligned(Y, 4))
    return GPTQ_ERR_INVALID;
  int num_sms = 148;
  gptq_status st = device_setup(&num_sms);
  if (st != GPTQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dr = static_cast<int>(d_row), dc = static_cast<int>(d_col), nb = static_cast<int>(batch);
  const int g = cfg->group_size, n_groups = g ? dc / g : 1;
  if (g == 0 || g % 128 == 0) {
    // scale regions of whole 128-column chunks: the unstaged layout
    const int grid = (dr + w4a16::W_ROWS - 1) / w4a16::W_ROWS;
    if (g == 0)
      w4a16::w4a16_wide_kernel<true><<<grid, w4a16::THREADS, 0, s>>>(
          qweight, scales, zeros, static_cast<const __nv_bfloat16*>(X), Y, dr, dc, nb, g, n_groups);
    else
      w4a16::w4a16_wide_kernel<false><<<grid, w4a16::THREADS, 0, s>>>(
          qweight, scales, zeros, static_cast<const __nv_bfloat16*>(X), Y, dr, dc, nb, g, n_groups);
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
  }
  const int tiles = (dr + w4a16::ROWS - 1) / w4a16::ROWS;
  // two 128-column chunks per work item where the scale regions are whole
  // chunks and the activations leave room for a deep ring; one otherwise
  const int cpi = (g == 0 || g % 128 == 0) && nb <= 4 ? 2 : 1;
  const int depth = w4a16::ring_depth(cpi, nb), smem = w4a16::smem_bytes(cpi, nb);
  const int per_sm = std::max(1, std::min(2, (228 * 1024) / (smem + 1024)));
  const int grid = std::min(tiles, per_sm * num_sms);  // persistent CTAs
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(X);
  // ceil(2^32 / group): umulhi(k, gmagic) == k / group for k, group < 2^16
  const uint32_t gmagic = g ? static_cast<uint32_t>(((uint64_t(1) << 32) + g - 1) / g) : 0u;
#define GPTQ_W4(GJ, CPI)                                                                   \
  w4a16::w4a16_matmul_kernel<GJ, CPI><<<grid, w4a16::THREADS, smem, s>>>(                  \
      qweight, scales, zeros, xb, Y, dr, dc, nb, gmagic, n_groups, depth)
  // a scale region of 32 GJ columns must lie inside one group
  if (g == 0) {
    if (cpi == 2) GPTQ_W4(0, 2);
    else GPTQ_W4(0, 1);
  } else if (g % 128 == 0) {
    if (cpi == 2) GPTQ_W4(4, 2);
    else GPTQ_W4(4, 1);
  } else if (g % 64 == 0) {
    GPTQ_W4(2, 1);
  } else {
    GPTQ_W4(1, 1);
  }
#undef GPTQ_W4
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

gptq_status gptq_awq_channel_scale(const void* X, int64_t n, int64_t d, int64_t ldx, double* sx,
                                   void* stream) {
  if (!X || !sx) return GPTQ_ERR_INVALID;
  if (n < 1 || n > (int64_t(1) << 31) - 1 || d < 8 || d % 8 != 0 || d > 65536) return GPTQ_ERR_INVALID;
  if (ldx < d || ldx % 8 != 0 || !aligned(X, 16) || !aligned(sx, 8)) return GPTQ_ERR_INVALID;
  int num_sms = 148;
  gptq_status st = device_setup(&num_sms);
  if (st != GPTQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dn = static_cast<int>(d), nn = static_cast<int>(n);
  GPTQ_CUDA_TRY(cudaMemsetAsync(sx, 0, static_cast<size_t>(d) * 8, s));
  const int tpb = std::max(256, (nn + 65534) / 65535);  // tokens per block (grid.y <= 65535)
  const dim3 grid((dn + awq::COLS_PER_BLOCK - 1) / awq::COLS_PER_BLOCK, (nn + tpb - 1) / tpb);
  awq::absum_kernel<<<grid, awq::THREADS, 0, s>>>(static_cast<const __nv_bfloat16*>(X), nn, dn,
                                                  ldx, tpb, sx);
  GPTQ_LAUNCH_CHECK();
  awq::mean_kernel<<<(dn + 255) / 256, 256, 0, s>>>(sx, dn, nn);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

size_t gptq_awq_workspace_size(int64_t d_row, int64_t d_col, const gptq_config* cfg) {
  if (!awq_config_ok(cfg, d_row, d_col)) return 0;
  return awq_layout(d_row, d_col).total;
}

gptq_status gptq_awq_search(const float* W, const float* H, const double* sx, int64_t d_row,
                            int64_t d_col, const gptq_config* cfg, int n_grid, double* losses,
                            int32_t* best, float* s_out, uint32_t* qweight, float* scales,
                            uint8_t* zeros, void* ws, size_t ws_bytes, void* stream) {
  if (!W || !H || !sx || !losses || !best || !s_out || !qweight || !scales || !zeros)
    return GPTQ_ERR_INVALID;
  if (!awq_config_ok(cfg, d_row, d_col) || n_grid < 2 || n_grid > 64) return GPTQ_ERR_INVALID;
  if (!aligned(W, 16) || !aligned(H, 16) || !aligned(sx, 8) || !aligned(losses, 8) ||
      !aligned(best, 4) || !aligned(s_out, 4) || !aligned(qweight, 4) || !aligned(scales, 4))
    return GPTQ_ERR_INVALID;
  const AwqWs L = awq_layout(d_row, d_col);
  if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return GPTQ_ERR_WORKSPACE;
  int num_sms = 148;
  gptq_status st = device_setup(&num_sms);
  if (st != GPTQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* Hhi = reinterpret_cast<float*>(base + L.Hhi);
  float* Hlo = reinterpret_cast<float*>(base + L.Hlo);
  float* Ehi = reinterpret_cast<float*>(base + L.Ehi);
  float* Elo = reinterpret_cast<float*>(base + L.Elo);
  float* T = reinterpret_cast<float*>(base + L.T);
  float* sv = reinterpret_cast<float*>(base + L.s);
  double* partials = reinterpret_cast<double*>(base + L.partials);
  const int dr = static_cast<int>(d_row), dc = static_cast<int>(d_col);
  const int gw = cfg->group_size ? cfg->group_size : dc;
  // the contraction T -= dW H on the split-TF32 tcgen05 kernel: E = dW
  // (K-major, K = d_col), G = H (all d_col rows), output T
  CUtensorMap tm_ehi, tm_elo, tm_hhi, tm_hlo, tm_t;
  if ((st = encode_f32_2d(&tm_ehi, Ehi, dc, dr, dc, trail::BK, trail::BM, CU_TENSOR_MAP_SWIZZLE_64B)) != GPTQ_OK ||
      (st = encode_f32_2d(&tm_elo, Elo, dc, dr, dc, trail::BK, trail::BM, CU_TENSOR_MAP_SWIZZLE_64B)) != GPTQ_OK ||
      (st = encode_f32_chunks(&tm_hhi, Hhi, dc, dc, dc, trail::BK, trail::BN / trail::B_BOX,
                          CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B)) != GPTQ_OK ||
      (st = encode_f32_chunks(&tm_hlo, Hlo, dc, dc, dc, trail::BK, trail::BN / trail::B_BOX,
                          CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B)) != GPTQ_OK ||
      (st = encode_f32_2d(&tm_t, T, dc, dr, dc, trail::OUT_COLS, trail::OUT_ROWS, CU_TENSOR_MAP_SWIZZLE_128B)) != GPTQ_OK)
    return st;
  trail::Params tp{};
  tp.M = dr; tp.N = dc; tp.K = dc; tp.n0 = 0; tp.j0 = 0;
  tp.wait_ns = g_wait_ns.load();
  tp.stall = g_fault.load() == GPTQ_FAULT_TRAILING_STALL;
  tp.tiles_m = (dr + trail::BM - 1) / trail::BM;
  tp.tiles_n = (dc + trail::BN - 1) / trail::BN;
  tp.tiles = tp.tiles_m * tp.tiles_n;
  const int tgrid = std::min(tp.tiles, num_sms);
  const int units = dr * (dc / gw);
  const int qgrid = std::max(1, std::min((units + 7) / 8, num_sms * 8));
  const size_t nel = static_cast<size_t>(dr) * dc;

  awq::sym_split_kernel<<<num_sms * 4, 256, 0, s>>>(H, dc, Hhi, Hlo);
  GPTQ_LAUNCH_CHECK();
  for (int a = 0; a < n_grid; ++a) {
    const double alpha = static_cast<double>(a) / static_cast<double>(n_grid - 1);
    awq::scales_kernel<<<(dc + 255) / 256, 256, 0, s>>>(sx, dc, alpha, sv);
    GPTQ_LAUNCH_CHECK();
    awq::delta_kernel<<<qgrid, awq::THREADS, 0, s>>>(W, sv, dr, dc, gw, Ehi, Elo);
    GPTQ_LAUNCH_CHECK();
    GPTQ_CUDA_TRY(cudaMemsetAsync(T, 0, nel * 4, s));
    trail::trailing_tf32x3_kernel<<<tgrid, trail::NUM_THREADS, trail::SMEM_BYTES, s>>>(
        tm_ehi, tm_elo, tm_hhi, tm_hlo, tm_t, tp);
    GPTQ_LAUNCH_CHECK();
    awq::dot_kernel<<<awq::DOT_BLOCKS, awq::THREADS, 0, s>>>(Ehi, Elo, T, nel / 4, partials);
    GPTQ_LAUNCH_CHECK();
    awq::finalize_kernel<<<1, 1024, 0, s>>>(partials, awq::DOT_BLOCKS, losses + a);
    GPTQ_LAUNCH_CHECK();
  }
  awq::argmin_kernel<<<1, 256, 0, s>>>(losses, n_grid, sx, dc, best, s_out);
  GPTQ_LAUNCH_CHECK();
  awq::pack_kernel<<<qgrid, awq::THREADS, 0, s>>>(W, s_out, dr, dc, gw, qweight, scales, zeros);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

gptq_status gptq_device_status(void* stream) {
  GPTQ_CUDA_TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int v = 0, zero = 0;
  GPTQ_CUDA_TRY(cudaMemcpyFromSymbol(&v, gptq::g_device_status, sizeof(int)));
  GPTQ_CUDA_TRY(cudaMemcpyToSymbol(gptq::g_device_status, &zero, sizeof(int)));
  return static_cast<gptq_status>(v);
}

}  // extern "C"

namespace {

gptq_status hessian_accumulate(float* H, const void* X, int64_t n, int64_t d, int64_t ldx,
                               float scale, bool ordered, void* stream) {
  if (!H) return GPTQ_ERR_INVALID;
  if (d < 8 || d > 65536 || d % 8 != 0) return GPTQ_ERR_INVALID;
  // token offsets and a chunk's length rounded up to BK stay below 2^31
  if (n < 0 || n > (int64_t(1) << 31) - 1 - syrk::BK) return GPTQ_ERR_INVALID;
  if (ldx < d || ldx % 8 != 0) return GPTQ_ERR_INVALID;
  if (!std::isfinite(scale) || !aligned(H, 16)) return GPTQ_ERR_INVALID;
  if (n == 0) return GPTQ_OK;  // X may be NULL for an empty chunk
  if (!X || !aligned(X, 16)) return GPTQ_ERR_INVALID;
  int num_sms = 0;
  gptq_status st = device_setup(&num_sms);
  if (st != GPTQ_OK) return st;

  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldx) * 2};
  const cuuint32_t box[2] = {syrk::BOX, syrk::BK};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = g_encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) {
    std::fprintf(stderr, "gptq: cuTensorMapEncodeTiled failed (%d)\n", static_cast<int>(cr));
    return GPTQ_ERR_CUDA;
  }

  CUtensorMap tmap_h;  // H as the reduce-add target: 128 rows x 32 fp32 pieces
  st = encode_f32_2d(&tmap_h, H, d, d, d, syrk::OUT_COLS, syrk::BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != GPTQ_OK) return st;

  syrk::Params p{};
  p.H = H;
  p.d = static_cast<int>(d);
  p.n = static_cast<int>(n);
  p.scale = scale;
  p.nti = static_cast<int>((d + syrk::BM - 1) / syrk::BM);
  p.ntj = static_cast<int>((d + syrk::BN - 1) / syrk::BN);
  {
    const int h = p.nti >> 1;
    p.ntiles = p.nti * p.ntj - (h * (h - 1) + (p.nti & 1) * h);
  }
  if (ordered) {  // one chunk: each element of H gets exactly one add
    p.split_tokens = (p.n + syrk::BK - 1) / syrk::BK * syrk::BK;
    p.nsplit = 1;
  } else {
    choose_split(p.ntiles, p.n, num_sms, &p.split_tokens, &p.nsplit);
  }
  p.units = p.ntiles * p.nsplit;
  p.wait_ns = g_wait_ns.load();
  p.stall = g_fault.load() == GPTQ_FAULT_SYRK_STALL;
  const int grid = std::min(p.units, num_sms);
  syrk::syrk_bf16_tcgen05_kernel<<<grid, syrk::NUM_THREADS, syrk::SMEM_BYTES,
                                   static_cast<cudaStream_t>(stream)>>>(tmap, tmap_h, p);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace

extern "C" {

gptq_status gptq_hessian_accumulate(float* H, const void* X, int64_t n, int64_t d, int64_t ldx,
                                    float scale, void* stream) {
  return hessian_accumulate(H, X, n, d, ldx, scale, false, stream);
}

gptq_status gptq_hessian_accumulate_ordered(float* H, const void* X, int64_t n, int64_t d,
                                            int64_t ldx, float scale, void* stream) {
  return hessian_accumulate(H, X, n, d, ldx, scale, true, stream);
}

gptq_status gptq_fault_inject(int where, int64_t wait_limit_ns) {
  if (where != GPTQ_FAULT_NONE && where != GPTQ_FAULT_SYRK_STALL &&
      where != GPTQ_FAULT_TRAILING_STALL)
    return GPTQ_ERR_INVALID;
  if (wait_limit_ns != 0 && (wait_limit_ns < 1000000 || wait_limit_ns > 10000000000ll))
    return GPTQ_ERR_INVALID;
  g_wait_ns.store(wait_limit_ns ? static_cast<uint64_t>(wait_limit_ns) : gptq::kWaitLimitNs);
  g_fault.store(where);
  return GPTQ_OK;
}


}  // extern "C"

namespace {

// The factorization behind gptq_prepare_hinv (factor = false: G = V^-1) and
// gptq_prepare_factor (factor = true: F, see prepare_factor below).
gptq_status prepare_impl(const float* H, int64_t d, double damp_rel, float* G,
                         uint8_t* dead_mask, void* ws, size_t ws_bytes, int64_t* bad_pivot,
                         void* stream, bool factor) {
  if (bad_pivot) *bad_pivot = -1;
  if (!H || !G || !dead_mask) return GPTQ_ERR_INVALID;
  if (d < 8 || d > 65536 || d % 8 != 0) return GPTQ_ERR_INVALID;
  if (!(damp_rel >= 0.0) || !std::isfinite(damp_rel)) return GPTQ_ERR_INVALID;
  const PrepareWs L = prepare_layout(d);
  if (!ws || !aligned(ws, kAlign) || ws_bytes < L.total) return GPTQ_ERR_WORKSPACE;
  gptq_status st = device_setup(nullptr);
  if (st != GPTQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  double* stats = reinterpret_cast<double*>(base + L.stats);
  int* istat = reinterpret_cast<int*>(base + L.istat);
  long long* pivot = reinterpret_cast<long long*>(base + L.pivot);
  double* A = reinterpret_cast<double*>(base + L.A);
  double* Mt = reinterpret_cast<double*>(base + L.Mt);
  double* Xd = reinterpret_cast<double*>(base + L.Xd);
  const int di = static_cast<int>(d);
  const int NB = chol::NB;
  // Block k covers [bstart(k), bstart(k+1)).  For F the blocks of the
  // reversed matrix must map onto the sweep's blocks [128 b, 128 b + 128) of
  // the original order, so a ragged block (d % 128 != 0) comes first rather
  // than last.
  const int shift = factor ? di % NB : 0;
  const int nt = shift ? 1 + (di - shift) / NB : (di + NB - 1) / NB;
  auto bstart = [&](int k) {
    if (k >= nt) return di;
    return shift ? (k == 0 ? 0 : shift + (k - 1) * NB) : k * NB;
  };
  auto at = [&](double* m, int r, int c) { return m + static_cast<size_t>(r) * di + c; };

  GPTQ_CUDA_TRY(cudaMemsetAsync(pivot, 0xFF, 8, s));
  // M^T accumulates its off-diagonal blocks from zero (F reads only the
  // blocks it writes)
  if (!factor) GPTQ_CUDA_TRY(cudaMemsetAsync(Mt, 0, static_cast<size_t>(d) * d * 8, s));
  chol::diag_stats_kernel<<<1, 1024, 0, s>>>(H, di, damp_rel, dead_mask, stats, istat);
  GPTQ_LAUNCH_CHECK();
  {
    dim3 grid((di + 255) / 256, std::min(di, 65535));
    chol::reverse_damp_fill_kernel<<<grid, 256, 0, s>>>(H, di, stats, A);
    GPTQ_LAUNCH_CHECK();
  }
  DeviceInfo* dinfo = current_device_info();
  if (!dinfo) return GPTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(dinfo->qmu);
  cudaStream_t aux = dinfo->aux;
  cudaEvent_t evP[2] = {dinfo->ev[2], dinfo->ev[3]};
  cudaEvent_t evL[2] = {dinfo->ev[4], dinfo->ev[5]};
  auto leaf = [&](int k, cudaStream_t st) {
    const int off = bstart(k);
    chol::leaf_kernel<<<1, chol::LEAF_THREADS, chol::LEAF_SMEM, st>>>(
        A, Mt, Xd + static_cast<size_t>(k) * NB * NB, di, off, bstart(k + 1) - off, pivot);
  };
  leaf(0, s);
  GPTQ_LAUNCH_CHECK();
  // Step k: P_k (caller's stream) forms the panel and rescales M's column
  // block k; then the auxiliary stream updates the next diagonal block (D_k)
  // and factors it (leaf k+1) while the caller's stream runs the rest of the
  // update U_k; P_{k+1} waits for both.  The trailing updates are lazy over
  // windows of m panels: inside a window, U_k only updates the window's
  // remaining columns (K = one panel); the window's last panel updates every
  // column to its right with all m panels at once (K = 128 m), so most of the
  // d^3 work runs with long K.  m = 1 is the plain right-looking sweep.
  // For F, M is not formed: its products are dropped, and U_k also writes
  // the block row F_k = L_{>k,k} X_kk (see prepare_factor).
  const int m = chol::window_panels(di);
  for (int k = 0; k < nt; ++k) {
    const int k0 = bstart(k), k1 = bstart(k + 1), nk = k1 - k0, rest = di - k1;
    double* Xk = Xd + static_cast<size_t>(k) * NB * NB;
    std::vector<chol::GemmProblem> pk;
    if (rest > 0) {
      chol::GemmProblem q{};  // L21 = A21 X_kk^T
      q.A = at(A, k1, k0); q.lda = di; q.B = Xk; q.ldb = NB; q.C = at(A, k1, k0); q.ldc = di;
      q.M = rest; q.N = nk; q.K = nk; q.alpha = 1.0; q.beta = 0.0;
      pk.push_back(q);
    }
    if (k0 > 0 && !factor) {
      chol::GemmProblem q{};  // Mt[:k0, block k] <- Mt[:k0, block k] X_kk^T
      q.A = at(Mt, 0, k0); q.lda = di; q.B = Xk; q.ldb = NB; q.C = at(Mt, 0, k0); q.ldc = di;
      q.M = k0; q.N = nk; q.K = nk; q.alpha = 1.0; q.beta = 0.0;
      pk.push_back(q);
    }
    // 64-row tiles from about one wave of them up: the panel is K = 128
    // deep, so finer tiles balance the SMs better than 128-row ones (at
    // d = 22016, 342 tiles against 171 on 148 SMs)
    const int prow = rest + (factor ? 0 : k0);
    if (prow >= 148 * 64) st = launch_nt<64, 2>(pk, s);
    else st = launch_nt<32, 1>(pk, s);
    if (st != GPTQ_OK) return st;
    if (rest <= 0) break;
    const int n1 = bstart(k + 2) - k1;  // next diagonal block
    // window of this panel: columns [e0, e1); the panels applied now are
    // [ka, k1) with K = kK, to the columns [k1, w1)
    const int e0 = bstart((k / m) * m), e1 = bstart((k / m) * m + m);
    const bool last = k1 >= e1;
    const int ka = last ? e0 : k0, kK = k1 - ka, w1 = last ? di : e1;
    GPTQ_CUDA_TRY(cudaEventRecord(evP[k & 1], s));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(aux, evP[k & 1], 0));
    {
      std::vector<chol::GemmProblem> dk(1);
      chol::GemmProblem& q = dk[0];  // D_k: A_{k+1,k+1} -= L_{k+1,[ka,k1)} L_{k+1,[ka,k1)}^T
      q = chol::GemmProblem{};
      q.A = at(A, k1, ka); q.lda = di; q.B = at(A, k1, ka); q.ldb = di;
      q.C = at(A, k1, k1); q.ldc = di;
      q.M = n1; q.N = n1; q.K = kK; q.alpha = -1.0; q.beta = 1.0;
      st = launch_nt<32, 1>(dk, aux);
      if (st != GPTQ_OK) return st;
      leaf(k + 1, aux);
      GPTQ_LAUNCH_CHECK();
      GPTQ_CUDA_TRY(cudaEventRecord(evL[k & 1], aux));
    }
    std::vector<chol::GemmProblem> uk;
    if (rest > n1) {
      chol::GemmProblem q{};  // rows below the next diagonal block, its columns
      q.A = at(A, k1 + n1, ka); q.lda = di; q.B = at(A, k1, ka); q.ldb = di;
      q.C = at(A, k1 + n1, k1); q.ldc = di;
      q.M = rest - n1; q.N = n1; q.K = kK; q.alpha = -1.0; q.beta = 1.0;
      uk.push_back(q);
      const int c2 = w1 - (k1 + n1);  // the further columns to update
      if (c2 > 0) {
        chol::GemmProblem r{};  // their square part, lower tiles
        r.A = at(A, k1 + n1, ka); r.lda = di; r.B = at(A, k1 + n1, ka); r.ldb = di;
        r.C = at(A, k1 + n1, k1 + n1); r.ldc = di;
        r.M = c2; r.N = c2; r.K = kK; r.lower_only = 1; r.alpha = -1.0; r.beta = 1.0;
        uk.push_back(r);
        if (di > w1) {
          chol::GemmProblem t{};  // the rows under the window's square part
          t.A = at(A, w1, ka); t.lda = di; t.B = at(A, k1 + n1, ka); t.ldb = di;
          t.C = at(A, w1, k1 + n1); t.ldc = di;
          t.M = di - w1; t.N = c2; t.K = kK; t.alpha = -1.0; t.beta = 1.0;
          uk.push_back(t);
        }
      }
    }
    if (!factor) {
      chol::GemmProblem q{};  // Mt[:k1, k1:w1] -= Mt[:k1, ka:k1] L[k1:w1, ka:k1]^T
      q.A = at(Mt, 0, ka); q.lda = di; q.B = at(A, k1, ka); q.ldb = di;
      q.C = at(Mt, 0, k1); q.ldc = di;
      q.M = k1; q.N = w1 - k1; q.K = kK; q.alpha = -1.0; q.beta = 1.0;
      uk.push_back(q);
    } else {
      chol::GemmProblem q{};  // F_k = L[k1:, k0:k1] X_kk into Mt's lower part
      q.A = at(A, k1, k0); q.lda = di; q.B = at(Mt, k0, k0); q.ldb = di;  // X_kk^T
      q.C = at(Mt, k1, k0); q.ldc = di;
      q.M = rest; q.N = nk; q.K = nk; q.alpha = 1.0; q.beta = 0.0;
      uk.push_back(q);
    }
    // two SMs stay free for D_k and leaf k+1 on the auxiliary stream (the
    // leaf's 141 KB of shared memory cannot share an SM with a U_k CTA)
    st = launch_nt<GPTQ_UK_SHAPE>(uk, s, 2);
    if (st != GPTQ_OK) return st;
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, evL[k & 1], 0));  // X_{k+1} for P_{k+1}
  }
  {
    dim3 grid((di + 31) / 32, (di + 31) / 32);
    if (factor) chol::write_f_kernel<<<grid, dim3(32, 8), 0, s>>>(Mt, di, G);
    else chol::write_g_kernel<<<grid, dim3(32, 8), 0, s>>>(Mt, di, G);
    GPTQ_LAUNCH_CHECK();
  }
  long long host_pivot = -1;
  int host_istat = 0;
  GPTQ_CUDA_TRY(cudaMemcpyAsync(&host_pivot, pivot, 8, cudaMemcpyDeviceToHost, s));
  GPTQ_CUDA_TRY(cudaMemcpyAsync(&host_istat, istat, 4, cudaMemcpyDeviceToHost, s));
  GPTQ_CUDA_TRY(cudaStreamSynchronize(s));
  if (bad_pivot) *bad_pivot = host_pivot;
  if (host_istat) return GPTQ_ERR_NONFINITE;
  if (host_pivot >= 0) return GPTQ_ERR_NOT_SPD;
  return GPTQ_OK;
}

}  // namespace

extern "C" {

gptq_status gptq_prepare_hinv(const float* H, int64_t d, double damp_rel, float* G,
                              uint8_t* dead_mask, void* ws, size_t ws_bytes,
                              int64_t* bad_pivot, void* stream) {
  return prepare_impl(H, d, damp_rel, G, dead_mask, ws, ws_bytes, bad_pivot, stream, false);
}

gptq_status gptq_prepare_factor(const float* H, int64_t d, double damp_rel, float* F,
                                uint8_t* dead_mask, void* ws, size_t ws_bytes,
                                int64_t* bad_pivot, void* stream) {
  return prepare_impl(H, d, damp_rel, F, dead_mask, ws, ws_bytes, bad_pivot, stream, true);
}

}  // extern "C"

namespace {

// The sweep behind gptq_quantize_layer (factor = false, G) and
// gptq_quantize_layer_factor (factor = true, F).
gptq_status quantize_impl(const float* W, int64_t d_row, int64_t d_col, const float* G,
                          const uint8_t* dead_mask, const gptq_config* cfg, uint32_t* qweight,
                          float* scales, uint8_t* zeros, void* ws, size_t ws_bytes, void* stream,
                          bool factor) {
  if (!W || !G || !qweight || !scales || !zeros) return GPTQ_ERR_INVALID;
  if (d_row < 1 || d_row > (int64_t(1) << 24) || d_col < 32 || d_col % 32 != 0 ||
      d_col > 65536)
    return GPTQ_ERR_INVALID;
  if (!config_ok(cfg, d_col)) return GPTQ_ERR_INVALID;
  // F's blocks are 128 wide, and a group's parameters must be taken inside
  // one block (F gives the exact running weights only at block starts)
  if (factor && (cfg->block != 128 || (cfg->group_size && 128 % cfg->group_size != 0)))
    return GPTQ_ERR_INVALID;
  if (!aligned(W, 16) || !aligned(G, 16) || !aligned(qweight, 4) || !aligned(scales, 4))
    return GPTQ_ERR_INVALID;
  if (dead_mask && !aligned(dead_mask, 4)) return GPTQ_ERR_INVALID;
  const QuantWs L = quant_layout(d_row, d_col, cfg->block);
  if (!ws || !aligned(ws, kAlign) || ws_bytes < L.total) return GPTQ_ERR_WORKSPACE;
  gptq_status st = device_setup(nullptr);
  if (st != GPTQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* Wk = reinterpret_cast<float*>(base + L.Wk);
  float* Eb[2][3];
  for (int b = 0; b < 2; ++b)
    for (int h = 0; h < 3; ++h) Eb[b][h] = reinterpret_cast<float*>(base + L.E[b][h]);
  float* Ghi = reinterpret_cast<float*>(base + L.Ghi);
  float* Glo = reinterpret_cast<float*>(base + L.Glo);
  const int dr = static_cast<int>(d_row), dc = static_cast<int>(d_col);
  const int B = cfg->block, g = cfg->group_size;
  const int n_groups = g ? dc / g : 1;
  const int per_channel = g == 0;
  int num_sms = 148;
  st = device_setup(&num_sms);
  if (st != GPTQ_OK) return st;
  // tensor maps of the trailing update: E splits (K-major, one window of
  // blocks per row), G splits, W
  const int lde = L.lde, mw = lde / B;
  CUtensorMap tm_e[2][2], tm_ghi, tm_glo, tm_w;
  for (int b = 0; b < 2; ++b)
    for (int h = 0; h < 2; ++h) {
      st = encode_f32_2d(&tm_e[b][h], Eb[b][h], lde, dr, lde, trail::BK, trail::BM,
                         CU_TENSOR_MAP_SWIZZLE_64B);
      if (st != GPTQ_OK) return st;
    }
  if ((st = encode_f32_chunks(&tm_ghi, Ghi, dc, dc, dc, trail::BK, trail::BN / trail::B_BOX,
                          CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B)) != GPTQ_OK) return st;
  if ((st = encode_f32_chunks(&tm_glo, Glo, dc, dc, dc, trail::BK, trail::BN / trail::B_BOX,
                          CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B)) != GPTQ_OK) return st;
  if ((st = encode_f32_2d(&tm_w, Wk, dc, dr, dc, trail::OUT_COLS, trail::OUT_ROWS,
                          CU_TENSOR_MAP_SWIZZLE_128B)) != GPTQ_OK) return st;
  DeviceInfo* di = current_device_info();
  if (!di) return GPTQ_ERR_CUDA;

  quant::prepare_rows_kernel<<<(dr + 7) / 8, 256, 0, s>>>(W, Wk, dead_mask, dr, dc, cfg->bits,
                                                           cfg->sym, per_channel, scales, zeros);
  GPTQ_LAUNCH_CHECK();
  trail::split_tf32_kernel<<<4 * num_sms, 256, 0, s>>>(G, Ghi, Glo, static_cast<size_t>(dc) * dc);
  GPTQ_LAUNCH_CHECK();
  // Block j: the step kernel Q_j (caller's stream) applies E_{j-1} to block j
  // and quantizes it; the trailing kernel T_j (auxiliary stream) applies E_j
  // to the columns right of block j+1.  Q_j needs T_{j-2} (it finished
  // block j's earlier updates); T_j needs Q_j.  So Q_{j+1} overlaps T_j.
  // The updates are lazy over windows of mw blocks: inside a window, T_j
  // reaches only the window's remaining columns; the window's last block
  // applies all the window's errors (K = mw B) to everything right of the
  // next block, and the next window's first step applies them to itself.
  // The errors of a window stay in one of two E buffers (row stride lde).
  std::lock_guard<std::mutex> lk(di->qmu);
  cudaEvent_t ev_fork = di->ev[0], ev_join = di->ev[1];
  cudaEvent_t* evQ = di->ev + 2;
  cudaEvent_t* evT = di->ev + 6;
  GPTQ_CUDA_TRY(cudaEventRecord(ev_fork, s));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(di->aux, ev_fork, 0));
  const int nblk = (dc + B - 1) / B;
  const dim3 qgrid((dr + quant::QROWS - 1) / quant::QROWS);
  // W[:, n0:n1] -= E[buf][:, ek0:ek0+K] * G[gj0:gj0+K, n0:n1]
  auto trailing = [&](int buf, int ek0, int K, int gj0, int n0, int n1) -> gptq_status {
    if (n0 % trail::B_BOX != 0) return GPTQ_ERR_INVALID;  // G is fetched in 32-column chunks
    trail::Params tp{};
    tp.M = dr; tp.N = n1 - n0; tp.K = K; tp.n0 = n0; tp.j0 = gj0; tp.ek0 = ek0;
    tp.chain = 256 / trail::BK;  // a window's update is summed 256 columns at a time
    tp.wait_ns = g_wait_ns.load();
    tp.stall = g_fault.load() == GPTQ_FAULT_TRAILING_STALL;
    tp.tiles_m = (dr + trail::BM - 1) / trail::BM;
    tp.tiles_n = (tp.N + trail::BN - 1) / trail::BN;
    tp.tiles = tp.tiles_m * tp.tiles_n;
    const int grid = std::min(tp.tiles, num_sms);
    trail::trailing_tf32x3_kernel<<<grid, trail::NUM_THREADS, trail::SMEM_BYTES, di->aux>>>(
        tm_e[buf][0], tm_e[buf][1], tm_ghi, tm_glo, tm_w, tp);
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
  };
  for (int jb = 0; jb < nblk; ++jb) {
    const int j0 = jb * B, ncols = std::min(B, dc - j0);
    const int win = jb / mw, pos = jb % mw, e0 = win * mw * B, e1 = std::min(dc, e0 + mw * B);
    const int cb = win & 1, pb = (win - 1) & 1;
    if (jb >= 2) GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, evT[(jb - 2) % 4], 0));
    if (g > B && j0 % g == 0 && jb >= 1)  // group params read columns ahead
      GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, evT[(jb - 1) % 4], 0));
    // the previous block, or at a window's first block the whole previous window
    const float* Ep = nullptr;
    int jp0 = -1, nprev = 0;
    if (jb > 0 && pos > 0) {
      Ep = Eb[cb][2] + (pos - 1) * B;
      jp0 = j0 - B; nprev = B;
    } else if (jb > 0) {
      Ep = Eb[pb][2];
      jp0 = e0 - mw * B; nprev = mw * B;
    }
    float* Ecf = Eb[cb][2] + pos * B;
    float* Ech = Eb[cb][0] + pos * B;
    float* Ecl = Eb[cb][1] + pos * B;
#define GPTQ_STEP(BB, FAC)                                                                 \
  quant::block_step_kernel<BB, FAC>                                                        \
      <<<qgrid, quant::QTHREADS, quant::block_step_smem<BB>(), s>>>(                       \
          Wk, dr, dc, j0, ncols, G, Ep, jp0, nprev, lde, Ecf, Ech, Ecl, qweight, scales,  \
          zeros, cfg->bits, cfg->sym, g, n_groups, per_channel, W, dead_mask)
    if (factor) GPTQ_STEP(128, true);
    else if (B == 128) GPTQ_STEP(128, false);
    else if (B == 64) GPTQ_STEP(64, false);
    else GPTQ_STEP(32, false);
#undef GPTQ_STEP
    GPTQ_LAUNCH_CHECK();
    GPTQ_CUDA_TRY(cudaEventRecord(evQ[jb % 4], s));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(di->aux, evQ[jb % 4], 0));
    if (pos < mw - 1 && j0 + ncols < dc) {
      // inside the window: this block's errors on the window's remaining
      // columns (block jb+1 takes them in its own step)
      if (e1 > j0 + 2 * B && (st = trailing(cb, pos * B, ncols, j0, j0 + 2 * B, e1)) != GPTQ_OK)
        return st;
    } else if (e1 + B < dc) {
      // the window's last block: all its errors on everything right of the
      // next block (which takes them in its own step)
      if ((st = trailing(cb, 0, e1 - e0, e0, e1 + B, dc)) != GPTQ_OK) return st;
    }
    GPTQ_CUDA_TRY(cudaEventRecord(evT[jb % 4], di->aux));
  }
  GPTQ_CUDA_TRY(cudaEventRecord(ev_join, di->aux));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, ev_join, 0));
  return GPTQ_OK;
}

}  // namespace

extern "C" {

gptq_status gptq_quantize_layer(const float* W, int64_t d_row, int64_t d_col, const float* G,
                                const uint8_t* dead_mask, const gptq_config* cfg,
                                uint32_t* qweight, float* scales, uint8_t* zeros, void* ws,
                                size_t ws_bytes, void* stream) {
  return quantize_impl(W, d_row, d_col, G, dead_mask, cfg, qweight, scales, zeros, ws, ws_bytes,
                       stream, false);
}

gptq_status gptq_quantize_layer_factor(const float* W, int64_t d_row, int64_t d_col,
                                       const float* F, const uint8_t* dead_mask,
                                       const gptq_config* cfg, uint32_t* qweight, float* scales,
                                       uint8_t* zeros, void* ws, size_t ws_bytes, void* stream) {
  return quantize_impl(W, d_row, d_col, F, dead_mask, cfg, qweight, scales, zeros, ws, ws_bytes,
                       stream, true);
}

gptq_status gptq_dequant_check(const uint32_t* qweight, const float* scales, const uint8_t* zeros,
                               const float* W, const float* H, int64_t d_row, int64_t d_col,
                               const gptq_config* cfg, float* W_hat, double* loss, void* ws,
                               size_t ws_bytes, void* stream) {
  if (!qweight || !scales || !zeros) return GPTQ_ERR_INVALID;
  if (d_row < 1 || d_row > (int64_t(1) << 24) || d_col < 32 || d_col % 32 != 0 ||
      d_col > 65536)
    return GPTQ_ERR_INVALID;
  if (!config_ok(cfg, d_col)) return GPTQ_ERR_INVALID;
  if (loss && (!W || !H)) return GPTQ_ERR_INVALID;
  const CheckWs L = check_layout(d_row, d_col);
  if (loss && (!ws || !aligned(ws, kAlign) || ws_bytes < L.total)) return GPTQ_ERR_WORKSPACE;
  gptq_status st = device_setup(nullptr);
  if (st != GPTQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dr = static_cast<int>(d_row), dc = static_cast<int>(d_col);
  const int g = cfg->group_size;
  const int n_groups = g ? dc / g : 1;
  if (W_hat) {
    quant::dequant_kernel<<<1184, 256, 0, s>>>(qweight, scales, zeros, dr, dc, cfg->bits, g,
                                               n_groups, W_hat);
    GPTQ_LAUNCH_CHECK();
  }
  if (loss) {
    uint8_t* base = static_cast<uint8_t*>(ws);
    double* partials = reinterpret_cast<double*>(base + L.partials);
    double* dloss = reinterpret_cast<double*>(base + L.loss);
    const dim3 grid((dr + 127) / 128, (dc + 127) / 128);
    quant::loss_tiles_kernel<<<grid, 256, 0, s>>>(qweight, scales, zeros, W, H, dr, dc,
                                                  cfg->bits, g, n_groups, partials);
    GPTQ_LAUNCH_CHECK();
    quant::sum_partials_kernel<<<1, 1024, 0, s>>>(partials, static_cast<int>(grid.x * grid.y),
                                                  dloss);
    GPTQ_LAUNCH_CHECK();
    GPTQ_CUDA_TRY(cudaMemcpyAsync(loss, dloss, 8, cudaMemcpyDeviceToHost, s));
  }
  GPTQ_CUDA_TRY(cudaStreamSynchronize(s));
  return GPTQ_OK;
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Loss check without a caller workspace: its scratch is this fixed device
// array.  Host code must not pass g_noalloc_scratch itself to a kernel (on
// the host the name is only a stand-in); it uses the device address that
// cudaGetSymbolAddress returns, looked up once per device.
static __device__ __align__(256) double g_noalloc_scratch[GPTQ_NOALLOC_MAX_TILES + 32];

namespace {
std::mutex g_noalloc_mu;
// Per device: the array's device address and the context it was looked up
// in.  A device reset (cudaDeviceReset, or a framework that resets the
// device) makes a new primary context with a new copy of the array, so the
// address is looked up again whenever the current context differs.
double* g_noalloc_ptr[64] = {};
CUcontext g_noalloc_ctx[64] = {};
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;

gptq_status noalloc_scratch(double** out) {
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_ctx_current) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    GPTQ_CUDA_TRY(cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q));
    if (q != cudaDriverEntryPointSuccess || !fn) return GPTQ_ERR_CUDA;
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  }
  // No context current on this thread yet (or another one): look the
  // address up, which also makes the device's primary context current.
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return GPTQ_ERR_CUDA;
  if (!ctx || !g_noalloc_ptr[dev] || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      std::fprintf(stderr, "gptq: cudaGetSymbolAddress(no-alloc scratch) failed: %s\n",
                   cudaGetErrorString(e));
      return GPTQ_ERR_CUDA;
    }
    if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return GPTQ_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<double*>(p);
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_ptr[dev];
  return GPTQ_OK;
}
}  // namespace

extern "C" gptq_status gptq_dequant_check_noalloc(const uint32_t* qweight, const float* scales,
                                                  const uint8_t* zeros, const float* W,
                                                  const float* H, int64_t d_row, int64_t d_col,
                                                  const gptq_config* cfg, float* W_hat,
                                                  double* loss, void* stream) {
  if (!qweight || !scales || !zeros) return GPTQ_ERR_INVALID;
  if (d_row < 1 || d_row > (int64_t(1) << 24) || d_col < 32 || d_col % 32 != 0 ||
      d_col > 65536)
    return GPTQ_ERR_INVALID;
  if (!config_ok(cfg, d_col)) return GPTQ_ERR_INVALID;
  if (loss && (!W || !H)) return GPTQ_ERR_INVALID;
  const int64_t tiles = ((d_row + 127) / 128) * ((d_col + 127) / 128);
  if (tiles > GPTQ_NOALLOC_MAX_TILES) {
    std::fprintf(stderr,
                 "gptq: gptq_dequant_check_noalloc: %lld x %lld needs %lld tiles, more than "
                 "GPTQ_NOALLOC_MAX_TILES (%d)\n",
                 static_cast<long long>(d_row), static_cast<long long>(d_col),
                 static_cast<long long>(tiles), GPTQ_NOALLOC_MAX_TILES);
    return GPTQ_ERR_INVALID;
  }
  gptq_status st = device_setup(nullptr);
  if (st != GPTQ_OK) return st;
  double* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != GPTQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dr = static_cast<int>(d_row), dc = static_cast<int>(d_col);
  const int g = cfg->group_size;
  const int n_groups = g ? dc / g : 1;
  if (W_hat) {
    quant::dequant_kernel<<<1184, 256, 0, s>>>(qweight, scales, zeros, dr, dc, cfg->bits, g,
                                               n_groups, W_hat);
    GPTQ_LAUNCH_CHECK();
  }
  if (loss) {
    double* partials = scratch;                        // one slot per tile, all rewritten
    double* dloss = scratch + GPTQ_NOALLOC_MAX_TILES;  // written by the final sum
    const dim3 grid((dr + 127) / 128, (dc + 127) / 128);
    quant::loss_tiles_kernel<<<grid, 256, 0, s>>>(qweight, scales, zeros, W, H, dr, dc,
                                                  cfg->bits, g, n_groups, partials);
    GPTQ_LAUNCH_CHECK();
    quant::sum_partials_kernel<<<1, 1024, 0, s>>>(partials, static_cast<int>(grid.x * grid.y),
                                                  dloss);
    GPTQ_LAUNCH_CHECK();
    GPTQ_CUDA_TRY(cudaMemcpyAsync(loss, dloss, 8, cudaMemcpyDeviceToHost, s));
  }
  GPTQ_CUDA_TRY(cudaStreamSynchronize(s));
  return GPTQ_OK;
}
