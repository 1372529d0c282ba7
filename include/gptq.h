/*
 * gptq.h -- C ABI of the B200 (sm_100a) GPTQ layer quantizer, libgptq.so.
 *
 * The method is GPTQ as described on the dingiv.github.io quantization page,
 * section GPTQ: for one linear layer W (d_row x d_col, out x in) and
 * calibration inputs X (d_col x n), find quantized W^ minimising
 * ||W X - W^ X||_F^2 using the Hessian H = 2 X X^T, the upper Cholesky factor
 * of H^-1, a fixed left-to-right column order, and blocks of B columns with
 * immediate in-block error updates and one lazy batched update of the columns
 * to the right after each block.  Output is b-bit codes (b = 2, 3, 4) with a
 * scale and zero point per output channel or per group of input columns
 * (granularity as on the psvmc.cn page, section 按量化粒度划分).  Widths 5 to 8
 * use the same path (section AWQ vs GPTQ names 8-bit GPTQ).
 *
 * Around the quantizer, the same library serves two steps the pages name:
 *  - gptq_w4a16_matmul multiplies activations by a packed 4-bit layer
 *    without writing the dequantized weights (section GPTQ: 4-bit weights
 *    for memory-bound decoding);
 *  - gptq_awq_channel_scale and gptq_awq_search run the AWQ scale search
 *    (section AWQ) on the same calibration Hessian and produce 4-bit output
 *    in the same format.
 *
 * Conventions for every call:
 *  - All array pointers are DEVICE pointers owned by the caller; the library
 *    allocates no device memory.  Scratch space comes from a caller-provided
 *    workspace of gptq_workspace_size() bytes, 256-byte aligned.
 *  - Matrices are dense row-major with the leading dimension stated.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *  - Calls validate their arguments first; on GPTQ_ERR_INVALID or
 *    GPTQ_ERR_WORKSPACE nothing is launched and no output is written.
 *  - gptq_hessian_accumulate, gptq_quantize_layer, gptq_w4a16_matmul and the
 *    AWQ calls are asynchronous and do not synchronize.  gptq_prepare_hinv
 *    and gptq_dequant_check synchronize `stream` once to return a status /
 *    value.
 *  - Kernels never spin without bound.  A kernel whose internal wait runs out
 *    records GPTQ_ERR_TIMEOUT in a device status word, frees what it holds
 *    and returns; gptq_device_status() reports it.  gptq_quantize_layer
 *    reports a non-finite weight through the same word.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID = 1,    /* bad argument: null pointer, size, alignment, config */
  GPTQ_ERR_NOT_SPD = 2,    /* damped H is not positive definite (see bad_pivot) */
  GPTQ_ERR_NONFINITE = 3,  /* NaN or Inf found in H (prepare) or in W (quantize) */
  GPTQ_ERR_WORKSPACE = 4,  /* workspace null, misaligned or smaller than required */
  GPTQ_ERR_CUDA = 5,       /* a CUDA runtime call or launch failed */
  GPTQ_ERR_TIMEOUT = 6     /* a kernel's bounded internal wait ran out */
} gptq_status;

/* Quantizer settings.
 *  bits        2 to 8 (the pages' INT2/3/4 outputs and INT8; every width
 *              packs into the same little-endian bit stream, codes may
 *              straddle 32-bit words).
 *  group_size  0 = one scale/zero per output channel, computed from the
 *              original row of W; otherwise the number of consecutive input
 *              columns sharing a scale/zero, computed from the current
 *              (error-updated) weights when the group's first column is
 *              reached.  Must be a multiple of 32 that divides d_col, with
 *              block % group_size == 0 or group_size % block == 0.
 *  sym         0: asymmetric, codes q = clip(rint(w/s) + z, 0, 2^b-1) with
 *                 s = (max(0,max w) - min(0,min w)) / (2^b-1), z = rint(-min(0,min w)/s)
 *                 where the quotient is formed with s exact (one fp64
 *                 division), so an exact tie rounds half to even;
 *              1: symmetric, s = max|w| / (2^(b-1)-1), z = 2^(b-1) (codes
 *                 stored offset-binary, i.e. signed code + 2^(b-1)).
 *              Dequantized value: s * (q - z).  (dingiv.github.io page,
 *              section 量化基础; youleyou.com page, sections 二 and 四.)
 *  block       B, columns per lazy-update block: 32, 64 or 128.
 *  damp_rel    relative damping: lambda = damp_rel * mean(diag H).
 */
typedef struct {
  int bits;
  int group_size;
  int sym;
  int block;
  double damp_rel;
} gptq_config;

/* Bytes of workspace needed by gptq_prepare_hinv (d = d_col),
 * gptq_quantize_layer and gptq_dequant_check for this layer shape: the
 * maximum over the three.  Returns 0 if the arguments are invalid. */
size_t gptq_workspace_size(int64_t d_row, int64_t d_col, const gptq_config* cfg);

/* H += scale * X^T X over n calibration tokens  (dingiv.github.io page,
 * section GPTQ: H = 2 X X^T, so scale = 2 for that definition).
 *  H      fp32, d x d row-major (leading dimension d), accumulated in place:
 *         the caller zeroes it before the first chunk.  Only the upper
 *         triangle including the diagonal (H[i][j], i <= j) is written; the
 *         strict lower triangle is never touched.
 *  X      bf16 token-major activations, n rows of d values, row stride ldx
 *         elements (ldx >= d, ldx % 8 == 0, X 16-byte aligned).  This is
 *         X^T of the page's d x n matrix, the layout a model's activations
 *         have.  Chunks of any size may be accumulated by repeated calls.
 *  d      % 8 == 0, 8 <= d <= 65536.   0 <= n < 2^31 - 64 (n == 0 is a
 *         no-op and X may then be NULL).
 * Each 128 x 256 tile of H sums its tokens on the tensor cores (fp32
 * accumulation, restarted every 1024 tokens and folded with round-to-nearest
 * adds).  When the tiles are too few to fill the GPU, the tokens are split
 * into chunks whose partial sums meet in H through TMA reduce-adds in L2,
 * in an order that varies between runs, so H may then differ in the last
 * bits from run to run (gptq_hessian_accumulate_ordered fixes the order).
 * Asynchronous. */
gptq_status gptq_hessian_accumulate(float* H, const void* X, int64_t n,
                                    int64_t d, int64_t ldx, float scale,
                                    void* stream);

/* gptq_hessian_accumulate with a fixed summation order: the tokens of a call
 * are never split, so every element of H receives exactly one add per call
 * and, for the same H, X and chunking, H is bitwise reproducible.  Same
 * arguments and errors.  It costs up to about 10% of the Hessian stage where
 * the tile count leaves the last wave of SMs part-empty (d = 4096: 272 tiles
 * on 148 SMs) and nothing where the tiles fill the GPU anyway (d >= 11008).
 * Asynchronous. */
gptq_status gptq_hessian_accumulate_ordered(float* H, const void* X, int64_t n,
                                            int64_t d, int64_t ldx, float scale,
                                            void* stream);

/* From H (upper triangle, as left by gptq_hessian_accumulate) compute the
 * damped H' = H + lambda I, lambda = damp_rel * mean(diag H), with a dead
 * input channel (H_ii == 0) given H'_ii = 1 and flagged in dead_mask, and
 * then G = the upper triangular U with U^T U = H'^-1 (dingiv.github.io page,
 * section GPTQ: the Cholesky factor of H^-1 through which all updates go).
 * Computed in fp64 as U = V^-1 where H' = V V^T with V upper triangular
 * (a Cholesky factorisation taken from the last row upward).
 *  H          fp32 d x d, read-only; only the upper triangle is read.
 *  G          fp32 d x d output; upper triangle = U, strict lower = 0.
 *  dead_mask  uint8[d] output, 1 for a dead channel.
 *  bad_pivot  host int64 out (may be NULL): -1, or the first column (in the
 *             original order) whose pivot was not positive and finite.
 *  ws         workspace of at least gptq_workspace_size(?, d, cfg) bytes.
 * Returns GPTQ_ERR_NOT_SPD if a pivot fails, GPTQ_ERR_NONFINITE if H has a
 * NaN/Inf on its diagonal.  Synchronizes `stream` once. */
gptq_status gptq_prepare_hinv(const float* H, int64_t d, double damp_rel,
                              float* G, uint8_t* dead_mask,
                              void* ws, size_t ws_bytes,
                              int64_t* bad_pivot, void* stream);

/* Quantize W column by column, left to right, in blocks of cfg->block
 * columns (dingiv.github.io page, section GPTQ, and its three refinements:
 * fixed order, Cholesky factor, lazy batched updates):
 *   for column q: code it, e = (w_q - w^_q) / G_qq, subtract e * G[q][k]
 *   from every later column k of the block at once; after the block,
 *   W[:, right] -= E * G[block, right].
 *  W          fp32 d_row x d_col input weights, read-only (a working copy
 *             is kept in the workspace).  Columns flagged in dead_mask are
 *             zeroed before quantization.
 *  G          fp32 d_col x d_col from gptq_prepare_hinv (upper triangle read).
 *  dead_mask  uint8[d_col] or NULL (no dead channels).
 *  qweight    uint32 d_row x (d_col*bits/32) output: row r's codes as a
 *             little-endian bit stream, code k at bits [bits*k, bits*k+bits),
 *             word w holding bits [32w, 32w+32).
 *  scales     fp32 d_row x n_groups output (n_groups = 1 when group_size is
 *             0, else d_col / group_size), row-major.
 *  zeros      uint8 d_row x n_groups output (integer zero points).
 *  Shapes: d_row >= 1, d_col % 32 == 0, d_col >= 32.  Asynchronous.
 * A NaN or Inf in W (outside dead columns) sets the device status word to
 * GPTQ_ERR_NONFINITE, reported by the next gptq_device_status(); the outputs
 * of that call are then meaningless. */
gptq_status gptq_quantize_layer(const float* W, int64_t d_row, int64_t d_col,
                                const float* G, const uint8_t* dead_mask,
                                const gptq_config* cfg, uint32_t* qweight,
                                float* scales, uint8_t* zeros,
                                void* ws, size_t ws_bytes, void* stream);

/* The same quantized layer with half of the fp64 work of gptq_prepare_hinv:
 * the column sweep never needs G = V^-1 outside its 128x128 diagonal
 * blocks.  From the sweep's recurrence (dingiv.github.io page, section
 * GPTQ: each column's error e_q = (w_q - w^_q)/G_qq is subtracted times row q
 * of G), W = W^ + E G, so E = (W - W^) V.  The running weights at the start
 * of 128-column block b are therefore
 *   W_b + sum_{a<b} (W - W^)_a V_ab G_bb,
 * the same values the sweep through G reaches there (the same sums in
 * another order), and inside the block the sweep runs through G_bb as
 * before.
 * gptq_prepare_factor takes the arguments of gptq_prepare_hinv and writes
 *  F  fp32 d x d: F_bb = G_bb on the diagonal 128-blocks (block b covers
 *     columns [128 b, 128 b + 128), the last one ragged), F_ab = V_ab G_bb
 *     for blocks a < b, 0 below the diagonal.
 * It factors H' once (d^3/3 flops) and forms no inverse beyond the diagonal
 * blocks; errors, pivots and synchronization as gptq_prepare_hinv.
 * gptq_quantize_layer_factor takes the arguments of gptq_quantize_layer
 * with F in place of G and writes the same outputs.  It needs
 * cfg->block == 128 and group_size 0 or a divisor of 128 (a group's
 * parameters are read from the running weights, which F gives exactly at
 * block starts only); otherwise GPTQ_ERR_INVALID.  Asynchronous. */
gptq_status gptq_prepare_factor(const float* H, int64_t d, double damp_rel,
                                float* F, uint8_t* dead_mask,
                                void* ws, size_t ws_bytes,
                                int64_t* bad_pivot, void* stream);
gptq_status gptq_quantize_layer_factor(const float* W, int64_t d_row, int64_t d_col,
                                       const float* F, const uint8_t* dead_mask,
                                       const gptq_config* cfg, uint32_t* qweight,
                                       float* scales, uint8_t* zeros,
                                       void* ws, size_t ws_bytes, void* stream);

/* Dequantize the packed output and measure the layer loss of the page's
 * objective through the Hessian: loss = 1/2 * sum_r dW_r H dW_r^T with
 * dW = W - W^, which equals ||W X - W^ X||_F^2 for H = 2 X X^T
 * (dingiv.github.io page, section GPTQ, the per-layer objective).
 *  qweight, scales, zeros  as written by gptq_quantize_layer.
 *  W       fp32 d_row x d_col, the original weights.
 *  H       fp32 d_col x d_col, the UNdamped Hessian (upper triangle read).
 *  W_hat   fp32 d_row x d_col output of dequantized weights, or NULL.
 *  loss    host double out (may be NULL).
 * Synchronizes `stream` once. */
gptq_status gptq_dequant_check(const uint32_t* qweight, const float* scales,
                               const uint8_t* zeros, const float* W,
                               const float* H, int64_t d_row, int64_t d_col,
                               const gptq_config* cfg, float* W_hat,
                               double* loss, void* ws, size_t ws_bytes,
                               void* stream);

/* Largest number of 128x128 tiles, ceil(d_row/128) * ceil(d_col/128), that
 * gptq_dequant_check_noalloc accepts (e.g. 16384 x 65536 or 65536 x 16384). */
#define GPTQ_NOALLOC_MAX_TILES 65536

/* gptq_dequant_check without a workspace argument, for callers that cannot
 * allocate device memory: for example a process whose device memory is all
 * reserved up front by its own pool, or a code path where the device-wide
 * synchronization of cudaMalloc is not allowed, and that has no workspace to
 * pass.  The paper has no counterpart; this is an interface variant, not part
 * of the method.
 *  Same arguments, outputs and synchronization as gptq_dequant_check, minus
 *  ws / ws_bytes.  Its scratch (one fp64 partial sum per 128x128 tile plus the
 *  loss) lives in a fixed array of (GPTQ_NOALLOC_MAX_TILES + 32) doubles,
 *  512 KB, in the library's device image: every GPU that loads the library
 *  holds it until the process exits.  The call itself allocates nothing (no
 *  cudaMalloc, cudaFree or allocating library routine).
 *  Layers with more tiles than GPTQ_NOALLOC_MAX_TILES are rejected with
 *  GPTQ_ERR_INVALID (and a message on stderr) before anything is launched.
 *  The first call on a device looks up that array's device address (once per
 *  device and CUDA context, with that device current); make that first call
 *  before any stream capture.  After a device reset (cudaDeviceReset, or a
 *  framework that resets the device) the new context holds a new copy of the
 *  array, and the next call looks its address up again.
 *  All calls share the one array, which keeps the last call's contents; each
 *  call overwrites every entry it later reads, so nothing needs clearing, but
 *  calls that overlap on the GPU (other streams, other host threads) race on
 *  it and must be serialized by the caller. */
gptq_status gptq_dequant_check_noalloc(const uint32_t* qweight, const float* scales,
                                       const uint8_t* zeros, const float* W,
                                       const float* H, int64_t d_row, int64_t d_col,
                                       const gptq_config* cfg, float* W_hat,
                                       double* loss, void* stream);

/* Y = X W^T with the packed layer dequantized on the fly (dingiv.github.io
 * "量化" page, section GPTQ: the quantized weights serve inference, where
 * batch-1 decoding is memory-bound and 4-bit weights cut the bytes read):
 *   Y[b][r] = sum_k X[b][k] * s[r][g(k)] * (q[r][k] - z[r][g(k)]).
 *  qweight, scales, zeros  the output of gptq_quantize_layer for a
 *             d_row x d_col layer with cfg (device, read-only): qweight
 *             16-byte aligned, scales 4-byte aligned, zero points 0..15.
 *             cfg->bits must be 4; group_size as in the quantize call.
 *  X          bf16 batch x d_col, row-major, 16-byte aligned (device).
 *  batch      1 to 8 activation rows.
 *  Y          fp32 batch x d_row, row-major (device, every element written).
 * The products (q - z) x are formed exactly and summed in fp32 (tensor-core
 * accumulation), so |Y - exact| <= (8 ceil(d_col / 1024) + 32) 2^-23
 * sum_k |X[b][k]| |W^[r][k]|.
 * Asynchronous on `stream`; allocates nothing.  Returns GPTQ_ERR_INVALID for
 * other widths, batches, misaligned pointers or a d_col that is not a
 * multiple of 32; nothing is launched then. */
gptq_status gptq_w4a16_matmul(const uint32_t* qweight, const float* scales,
                              const uint8_t* zeros, int64_t d_row, int64_t d_col,
                              const gptq_config* cfg, const void* X, int64_t batch,
                              float* Y, void* stream);

/* AWQ channel scale (dingiv.github.io "量化" page, section AWQ: salient
 * input channels are found by their mean activation magnitude):
 *   sx[k] = (1/n) sum_t |X[t][k]|.
 *  X    bf16 calibration tokens, token-major: token t at X + t*ldx
 *       (device, 16-byte aligned; ldx >= d, ldx % 8 == 0).
 *  n    tokens, >= 1.   d  channels, a multiple of 8, <= 65536.
 *  sx   fp64[d] (device, written).  The sums are exact in fp64 for bf16
 *       inputs, so the result does not depend on the order of summation.
 * Asynchronous on `stream`.  GPTQ_ERR_INVALID for bad sizes or pointers. */
gptq_status gptq_awq_channel_scale(const void* X, int64_t n, int64_t d, int64_t ldx, double* sx,
                                   void* stream);

/* Workspace bytes for gptq_awq_search: 2 d_col^2 + 3 d_row d_col floats and a
 * few KB.  0 for an unsupported configuration. */
size_t gptq_awq_workspace_size(int64_t d_row, int64_t d_col, const gptq_config* cfg);

/* AWQ scale search (dingiv.github.io "量化" page, section AWQ): for each
 * alpha_a = a / (n_grid - 1), s = sx^alpha (s = 1 where sx = 0), W diag(s)
 * is quantized to 4 bits with the min-max quantizer of this library and
 * divided by s again, and the loss is the layer's output error
 *   L(alpha) = ||W X - Q(W diag(s)) diag(s)^-1 X||_F^2
 *            = 1/2 sum_r dW_r H dW_r^T,   H = 2 X X^T.
 * The best alpha (the first smallest loss) is then applied: the outputs are
 * the codes, scales and zero points of W diag(s*) and s* itself (the
 * activations, or the previous layer's output, are divided by s*).
 *  W        fp32 d_row x d_col, row-major (device, 16-byte aligned, read).
 *  H        fp32 d_col x d_col upper triangle as gptq_hessian_accumulate
 *           writes it (device, 16-byte aligned, read).
 *  sx       fp64[d_col] from gptq_awq_channel_scale (device).
 *  cfg      bits 4, sym 0, group_size 0 (one scale per row) or a multiple of
 *           32 dividing d_col; d_col a multiple of 32, <= 65536;
 *           d_row * d_col < 2^31.
 *  n_grid   grid points, 2 to 64 (the AWQ section uses 20).
 *  losses   fp64[n_grid] (device, written): L(alpha_a).
 *  best     int32 (device, written): a of the best alpha.
 *  s_out    fp32[d_col] (device, written): s*.
 *  qweight, scales, zeros  as written by gptq_quantize_layer for 4 bits
 *           (device, written), here for W diag(s*).
 *  ws       >= gptq_awq_workspace_size bytes (device, 256-byte aligned).
 * The contraction dW H runs on the tensor cores as three TF32 products of
 * hi/lo splits (about fp32 accuracy); the loss is summed in fp64.
 * Asynchronous on `stream`; allocates nothing.  GPTQ_ERR_INVALID for bad
 * sizes, configurations or pointers, GPTQ_ERR_WORKSPACE for a short or
 * misaligned workspace; nothing is launched then. */
gptq_status gptq_awq_search(const float* W, const float* H, const double* sx, int64_t d_row,
                            int64_t d_col, const gptq_config* cfg, int n_grid, double* losses,
                            int32_t* best, float* s_out, uint32_t* qweight, float* scales,
                            uint8_t* zeros, void* ws, size_t ws_bytes, void* stream);

/* Synchronize `stream`, then return and clear the device status word that
 * kernels set when a bounded internal wait runs out (GPTQ_ERR_TIMEOUT) or
 * when gptq_quantize_layer meets a non-finite weight (GPTQ_ERR_NONFINITE).
 * The first such event since the last call is kept. */
gptq_status gptq_device_status(void* stream);

/* Fault injection for testing the failure detection; the paper has no
 * counterpart.  Off (GPTQ_FAULT_NONE) unless set, process-wide, and applied
 * to every later launch until changed:
 *  where          GPTQ_FAULT_SYRK_STALL: the producer warp of the Hessian
 *                 kernel issues no loads, so the MMA thread's first bounded
 *                 wait runs out; GPTQ_FAULT_TRAILING_STALL: the same in the
 *                 trailing-update kernel of gptq_quantize_layer and
 *                 gptq_awq_search.  Nothing is in flight when the waits give
 *                 up; the kernel records GPTQ_ERR_TIMEOUT, frees its tensor
 *                 memory and returns, and the context stays usable.  The
 *                 outputs of a stalled call are meaningless.
 *  wait_limit_ns  the limit of every bounded wait in every kernel, 1 ms to
 *                 10 s; 0 restores the default of 2 s.
 * Returns GPTQ_ERR_INVALID for other values (nothing changes then).  Not
 * thread-safe against launches in flight on other host threads. */
enum { GPTQ_FAULT_NONE = 0, GPTQ_FAULT_SYRK_STALL = 1, GPTQ_FAULT_TRAILING_STALL = 2 };
gptq_status gptq_fault_inject(int where, int64_t wait_limit_ns);

/* Number of kernels this library has launched in this process (all devices,
 * all streams).  Instrumentation for benchmarks: the difference across a
 * timed region is the launch count of that region.  The paper has no
 * counterpart; it is not part of the method. */
uint64_t gptq_launch_count(void);

/* Static, human-readable name of a status code. */
const char* gptq_status_string(gptq_status s);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
