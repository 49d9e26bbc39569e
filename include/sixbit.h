/*
 * sixbit.h -- C ABI of the B200 (sm_100a) hot path of 6Bit-Diffusion.
 *
 * 6Bit-Diffusion (arXiv:2603.18742, as described by the write-up "6Bit-Diffusion: dynamic
 * quantization ..." and the explainer "6Bit-Diffusion: Inference-Time Mixed-Precision
 * Quantization for Video Diffusion Models") runs every linear layer of a video diffusion
 * transformer in NVFP4 or INT8, chosen per layer and per denoising step from the previous step's
 * input/output difference, rotates activations with a block Hadamard transform first, skips whole
 * modules whose outputs barely change (Temporal Delta Cache, TDC), and computes in full precision
 * when the input's outlier ratio is too large (Purified Delta Refresh, PDR).
 *
 * Conventions (apply to every entry point):
 *  - Pointers are DEVICE pointers unless the parameter is marked "host". Structs passed by
 *    pointer (sb_config, sb_rule, sb_weight, sb_fp4, sb_i8) are HOST structs whose pointer
 *    fields are device pointers; sb_module_state and sb_stats live in DEVICE memory.
 *  - The caller owns all memory. The library allocates no device memory; scratch lives in the
 *    caller's workspace `ws` (sb_workspace_size). The one exception is sb_prepass_static, whose
 *    scratch is a fixed array compiled into the library (see there); no other call keeps device
 *    state between calls.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; 0 = legacy default stream).
 *    Calls that share a workspace must be ordered on one stream.
 *  - Arguments are validated synchronously; on failure nothing is launched, the status is
 *    returned and sb_last_error() describes it. Device-side faults of the method (a bounded wait
 *    that gave up, non-finite input) set an error word inside `ws`; sb_check() reads and clears it.
 *  - Every device pointer must be 16-byte aligned (SB_EALIGN otherwise).
 *  - Shapes: activations are [M][K] row-major bf16 (M tokens, K channels); weights are [N][K]
 *    row-major (row = output channel, the PyTorch Linear layout); outputs are [M][N].
 *  - No C++ exception crosses this boundary.
 */
#ifndef SIXBIT_H
#define SIXBIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* sb_stream; /* identical to cudaStream_t */

typedef enum {
  SB_OK = 0,
  SB_EINVAL = 1,        /* null pointer where one is required, bad enum value */
  SB_ESHAPE = 2,        /* inconsistent or out-of-range sizes */
  SB_EALIGN = 3,        /* a device pointer is not 16-byte aligned */
  SB_EUNSUPPORTED = 4,  /* block not in {16,32,64,128,256}, K % block, K % 64, N % 32, K > 16384 */
  SB_ECUDA = 5,         /* a CUDA runtime call failed (launch, attribute, tensor map) */
  SB_ETIMEOUT = 6,      /* device: a bounded wait inside a kernel gave up (reported by sb_check) */
  SB_ENONFINITE = 7     /* device: a pre-pass input held Inf/NaN (reported by sb_check) */
} sb_status;

/* Precision of one layer at one step ("write-up" section 一: NVFP4 is the fast, coarse format,
 * INT8 the precise one; section 三: full precision when PDR fires; section 二: skip). */
typedef enum { SB_NVFP4 = 0, SB_INT8 = 1, SB_BF16 = 2, SB_SKIP = 3 } sb_prec;

enum { SB_OUT_BF16 = 0, SB_OUT_F32 = 1, SB_OUT_RAW = 2 };   /* sb_linear out_dtype */
enum { SB_EPI_NONE = 0, SB_EPI_GELU_TANH = 1 };             /* sb_linear epilogue  */
enum { SB_PREPASS_QUANT = 0, SB_PREPASS_STATS = 1 };        /* sb_prepass mode     */

/* NVFP4 tensor: E2M1 codes packed two per byte along K (element 2i in the low nibble), one E4M3
 * scale per 16 consecutive elements of a row stored in the tensor-core block-scale layout
 * (sb_fp4_sf_bytes), one FP32 tensor scale s_g. value = e2m1 * e4m3 * s_g. */
typedef struct {
  uint8_t* codes;   /* [rows][cols/2] */
  uint8_t* sf;      /* sb_fp4_sf_bytes(rows, cols) bytes; rows padded to 128 with zero scales */
  float* gscale;    /* 1 float */
  int64_t rows, cols;
} sb_fp4;

/* INT8 tensor, symmetric, one FP32 scale per row: value = code * scale[row]. */
typedef struct {
  int8_t* codes;    /* [rows][cols] */
  float* scale;     /* [rows] */
  int64_t rows, cols;
} sb_i8;

/* A prepared linear layer. w4 and w8 hold the Hadamard-rotated weight (rows rotated along K with
 * the same block as the activations) quantized to NVFP4 (tensor scale) and INT8 (per output
 * channel); w_bf16 is the original weight kept for the PDR full-precision path. */
typedef struct {
  const void* w_bf16;     /* [N][K] bf16, original */
  const void* bias_bf16;  /* [N] bf16 or NULL */
  sb_fp4 w4;
  sb_i8 w8;
  int64_t N, K;
  int32_t block;
} sb_weight;

/* Per-layer linear rule ("write-up" section 一 and 六: a simple linear model of the previous
 * step's difference predicts the need for precision): INT8 iff a * d_prev + b > tau. */
typedef struct { double a, b, tau; } sb_rule;

typedef struct {
  double rho;         /* PDR outlier-ratio threshold (max|x| / mean|x|), e.g. 64 */
  double tdc_thresh;  /* TDC accumulator threshold, e.g. 0.1 */
  int32_t block;      /* Hadamard block B (16..256, power of two), default 128 */
  int32_t force_prec; /* -1: decide; 0/1/2 force NVFP4/INT8/BF16 (benchmarks, tests) */
} sb_config;

/* Per-module decision state (device memory, 64 bytes). */
typedef struct {
  double prev_d;        /* d of the last computed step */
  double acc;           /* accumulated delta since the last computed step */
  double delta;         /* relative L1 change between the last two computed outputs */
  int32_t have_d;       /* prev_d belongs to the step just before the current one */
  int32_t n_out;        /* computed outputs so far */
  int32_t last_skipped; /* the previous step was skipped */
  int32_t skip;         /* decision of the current step (1 = reuse the cache) */
  int32_t steps;        /* sb_tdc_step calls so far */
  int32_t reserved[3];
} sb_module_state;

/* Pre-pass statistics (device memory, 88 bytes; the Python binding allocates 96). Sums are the
 * deterministic pairwise reductions (FP32 per row, FP64 across rows) so that every decision is
 * reproducible bit for bit. */
typedef struct {
  double sum_abs;   /* sum |x| */
  double sum_d2;    /* sum (x - x_ref)^2 (0 without x_ref) */
  double sum_ref2;  /* sum x_ref^2 (0 without x_ref) */
  double max_abs;   /* max |x| */
  double amax_rot;  /* max |H x| over the tensor: the NVFP4 tensor amax */
  double ratio;     /* PDR outlier ratio max|x| / (sum|x| / numel); +inf when sum|x| = 0 */
  double d;         /* sqrt(sum_d2) / sqrt(sum_ref2) (relative input/output difference) */
  double numel;
  int32_t has_ref;  /* d is valid */
  int32_t prec_in;  /* precision on entry */
  int32_t prec_out; /* precision after PDR */
  int32_t nonfinite; /* the input X held Inf or NaN (a row's max |x| is Inf or its sum |x| NaN) */
  int32_t error;     /* written by sb_prepass_static only: the device error word of its call */
  int32_t reserved;
} sb_stats;

const char* sb_version(void);

/* Thread-local description of the last failed call of this thread ("" if none). */
const char* sb_last_error(void);

/* Bytes of workspace needed by calls with at most max_M rows (tokens or weight rows N) of at most
 * max_K columns: a 256-byte header and two arrays of one 48-byte slot per 16 rows. `bytes` is a
 * host pointer. */
sb_status sb_workspace_size(int64_t max_M, int64_t max_K, size_t* bytes);

/* Zero a workspace (counters and error word) before its first use. */
sb_status sb_workspace_init(void* ws, size_t bytes, sb_stream stream);

/* Bytes of the block-scale array of an NVFP4 tensor: ceil(rows/128)*128 * cols/16. */
int64_t sb_fp4_sf_bytes(int64_t rows, int64_t cols);

/* Reset a module state (n_out = 0, no difference, nothing accumulated). */
sb_status sb_state_init(sb_module_state* state, sb_stream stream);

/* Block Hadamard rotation only (utility and test hook): Y[m][k] = (H_B X[m][block(k)])[k] in FP32,
 * H_B the unnormalised Sylvester matrix, butterfly stages h = 1, 2, ..., B/2 ascending.
 * X bf16 [M][K], Y float [M][K]. ("write-up" section 一: block Hadamard transform.) */
sb_status sb_rotate(const void* X, float* Y, int64_t M, int64_t K, int32_t block, sb_stream stream);

/* Offline weight preparation (untimed): rotate each row of W [N][K] along K in blocks of
 * `block`, write the INT8 copy (per-row scale) into w->w8 and the NVFP4 copy (tensor scale from
 * the rotated amax) into w->w4. The caller sets w->w_bf16, w->bias_bf16 and the device buffers of
 * w->w4 (codes N*K/2, sf sb_fp4_sf_bytes(N,K), gscale 1 float) and w->w8 (codes N*K, scale N);
 * this call fills N, K and block. ("write-up" section 四: W4A6, weights pre-quantized.) */
sb_status sb_prepare_weight(const void* W, const void* bias, int64_t N, int64_t K, int32_t block,
                            sb_weight* w /* host */, void* ws, sb_stream stream);

/* TDC check of one module for the current step ("write-up" section 二): the first two steps are
 * computed; afterwards acc += delta and the module is skipped while acc <= cfg->tdc_thresh. A skip
 * clears have_d (the next computed step is a restart). Writes state->skip. */
sb_status sb_tdc_step(sb_module_state* state, const sb_config* cfg /* host */, sb_stream stream);

/* Precision of one layer for the current step ("write-up" sections 一 and 三): SB_SKIP if the
 * module is skipped; cfg->force_prec if >= 0; INT8 if no previous difference exists (first step or
 * restart after skips); else INT8 iff rule->a * prev_d + rule->b > rule->tau, NVFP4 otherwise.
 * Writes *prec (device int32). */
sb_status sb_select_precision(const sb_module_state* state, const sb_rule* rule /* host */,
                              const sb_config* cfg /* host */, int32_t* prec, sb_stream stream);

/* sb_tdc_step followed by sb_select_precision for each of a module's n layers (1 <= n <= 8), in
 * one launch: rules[i] (host array) decides *precs[i] (host array of device int32 pointers, 4-byte
 * aligned) from the state the TDC check leaves. Same results as the separate calls. */
sb_status sb_module_decide(sb_module_state* state, const sb_config* cfg /* host */, int32_t n,
                           const sb_rule* rules /* host */, int32_t* const* precs /* host */,
                           sb_stream stream);

/* Activation pre-pass of one layer input X [M][K] bf16 ("write-up" sections 一, 三, 四).
 * One pass computes the statistics record *stats (PDR ratio on the raw X; d against X_ref when
 * given) and, in SB_PREPASS_QUANT mode, the block-Hadamard-rotated quantized activations for the
 * precision in *prec: INT8 into a8 (codes [M][K], per-token scales [M]) or NVFP4 into a4 (codes,
 * block scales, tensor scale; a second streaming kernel, which needs the tensor amax first).
 * In SB_PREPASS_QUANT mode PDR is applied: a quantized *prec becomes SB_BF16 when
 * stats->ratio > cfg->rho (unless cfg->force_prec >= 0). *prec == SB_SKIP makes every kernel exit
 * at once. SB_PREPASS_STATS computes the record only and leaves *prec unchanged (prec may be
 * NULL) and does not rotate (stats->amax_rot is then 0). a4/a8 may be NULL in STATS mode; in QUANT
 * mode both must be given (the precision is only known on the device). Requires M*K > 0,
 * K % block == 0, K % 64 == 0, K <= 16384. */
sb_status sb_prepass(const void* X, const void* X_ref, int64_t M, int64_t K,
                     const sb_config* cfg /* host */, int32_t mode, int32_t* prec,
                     const sb_fp4* a4 /* host */, const sb_i8* a8 /* host */, sb_stats* stats,
                     void* ws, sb_stream stream);

/* sb_prepass for a tensor whose per-chunk statistics its producer already computed (FFN-pair
 * fusion: the layer that writes X hands these over, so the pre-pass does not read X for them).
 * chunks: device float4 records [M][K/128], one per aligned 128-channel chunk of a row:
 * x = max |H_B x| over the chunk (B = cfg->block <= 128), y = the canonical pairwise sum of |x|
 * over its 128 values, z = max |x|; w is scratch: the call leaves the row's rotated amax in the
 * w of its first record. The records fold into the same statistics record, PDR verdict and INT8
 * scales as sb_prepass computes from X; in QUANT mode X is then read once for the codes (INT8
 * when *prec said INT8 at the start, NVFP4 when it says NVFP4 after PDR). X_ref is not
 * supported. Requires K % 128 == 0 and block <= 128 (SB_EUNSUPPORTED), else as sb_prepass. */
sb_status sb_prepass_chunks(const void* X, float* chunks, int64_t M, int64_t K,
                            const sb_config* cfg /* host */, int32_t mode, int32_t* prec,
                            const sb_fp4* a4 /* host */, const sb_i8* a8 /* host */, sb_stats* stats,
                            void* ws, sb_stream stream);

/* The producer of those records (FFN-pair fusion, "write-up" section 四): sb_linear with bf16
 * output Y [M][N] that also writes, from its epilogue, the chunk records of Y as it stores it
 * (float4 [M][N/128]; x = max |H_B y| over the chunk, y = the canonical pairwise sum of |y|,
 * z = max |y|, w = 0), for a next pre-pass whose cfg->block is `block`, which must be 128 here
 * (SB_EUNSUPPORTED otherwise; sb_chunk_records covers the smaller blocks). The records describe
 * the bf16 values Y holds, whatever precision *prec
 * selects; under SB_SKIP neither Y nor the records are written. records: 16-byte aligned device
 * memory (SB_EALIGN), owned by the caller; requires N % 256 == 0 (SB_EUNSUPPORTED), else as
 * sb_linear (whose out_dtype is SB_OUT_BF16 here). */
sb_status sb_linear_records(const void* X, const sb_fp4* a4 /* host */, const sb_i8* a8 /* host */,
                            const int32_t* prec, const sb_weight* w /* host */, int32_t epilogue, void* Y,
                            int64_t M, int32_t block, float* records, void* ws, sb_stream stream);

/* The same chunk records computed from a bf16 tensor X [M][K] in device memory (K % 128 == 0,
 * K <= 16384, block in {16, 32, 64, 128}, else SB_EUNSUPPORTED; M >= 1, else SB_ESHAPE; X and
 * records 16-byte aligned, else SB_EALIGN), with the arithmetic of sb_linear_records' epilogue:
 * a stand-alone producer for tensors that no GEMM of this library wrote. */
sb_status sb_chunk_records(const void* X, int64_t M, int64_t K, int32_t block, float* records, sb_stream stream);

/* Quantized linear layer Y = X W^T + bias ("write-up" section 四; tcgen05 tensor cores):
 *   NVFP4: Y = acc * s_gx * s_gw / B + bias, acc = sum of block-scaled E2M1 products
 *          (tcgen05.mma kind::mxf4nvf4, UE4M3 scales per 16);
 *   INT8:  Y = acc * s_x[m] * s_w[n] / B + bias, acc exact int32 (kind::i8);
 *   BF16:  Y = X W^T + bias on the raw X and original W (kind::f16), the PDR path.
 * The kind is read from *prec on the device (SB_SKIP: nothing is written). 1/B undoes the
 * unnormalised rotation of both operands. epilogue SB_EPI_GELU_TANH applies the tanh GELU.
 * out_dtype: SB_OUT_BF16 / SB_OUT_F32 write the result; SB_OUT_RAW writes the raw accumulator
 * (int32 for INT8, FP32 otherwise; test hook). X (bf16 [M][K]) may be NULL if the BF16 path is
 * never taken; a4/a8 may be NULL if that precision is never taken (the kernel then reports
 * SB_EINVAL through sb_check). Requires K % 128 == 0, N % 32 == 0. */
sb_status sb_linear(const void* X, const sb_fp4* a4 /* host */, const sb_i8* a8 /* host */,
                    const int32_t* prec, const sb_weight* w /* host */, int32_t epilogue,
                    int32_t out_dtype, void* Y, int64_t M, void* ws, sb_stream stream);

/* TDC record after a computed step ("write-up" section 二; explainer section 3): y_new and
 * y_cache are bf16 [M][C]; y_cache holds the last computed output. If at least one output was
 * recorded before, delta = sum|y_new - y_cache| / sum|y_cache| (pairwise FP32 rows, FP64 across
 * rows; +inf when sum|y_cache| = 0) is stored. Then n_out += 1, acc = 0, and d is taken from
 * d_src (if non-NULL and d_src->has_ref) as prev_d with have_d = 1, else have_d = 0. With
 * update_cache != 0 the same pass refreshes y_cache with y_new. Does nothing if state->skip. */
sb_status sb_tdc_record(const void* y_new, void* y_cache, int64_t M, int64_t C,
                        const sb_stats* d_src, int32_t update_cache, sb_module_state* state,
                        void* ws, sb_stream stream);

/* The module's output record in one pass ("write-up" sections 一 and 二): the difference statistic
 * of the module output y against its input x, then the TDC record of y against the cached last
 * output, reading y once. Bit for bit the same results (stats, state, cache) as
 *   sb_prepass(y, x, M, C, cfg, SB_PREPASS_STATS, prec, NULL, NULL, stats, ws) followed by
 *   sb_tdc_record(y, cache, M, C, stats, update_cache, state, ws),
 * each part with its own gate: the statistics are skipped when *prec == SB_SKIP (prec may be
 * NULL: never skipped; *prec is not modified), the record when state->skip; the record takes its d
 * from the stats this call writes. y, x, cache: bf16 [M][C] row-major, 16-byte aligned
 * (SB_EALIGN); stats: device sb_stats; state: device sb_module_state; C a multiple of 64 in
 * [64, 16384] (SB_EUNSUPPORTED); M in [1, 2^30] (SB_ESHAPE). The call uses two group-slot arrays
 * of ws, so ws must come from sb_workspace_size with max_M >= M. */
sb_status sb_module_record(const void* y, const void* x, void* cache, int64_t M, int64_t C, int32_t* prec,
                           int32_t update_cache, sb_stats* stats, sb_module_state* state, void* ws,
                           sb_stream stream);

/* sb_linear (bf16 output, the module's output Y [M][N]) fused with sb_module_record(Y, x, cache,
 * M, N, prec, update_cache, stats, state, ws): the GEMM's epilogue computes, for every row and
 * aligned 128-column chunk of the bf16 values it stores, the partial sums of the difference
 * statistic (sum |y|, sum (y - x)^2, sum x^2, max |y|) and of the TDC record (sum |y - c|, sum |c|;
 * c, the cached output, reads as zero while state->n_out == 0), and stores the output to the cache
 * as well when update_cache is set and state->skip == 0; a second kernel folds the partial sums into
 * the rows' canonical sums, the group slots and both finishes ("write-up" sections 三 and 四). Stats,
 * state and cache come out bit for bit as from the two separate calls whenever *prec != SB_SKIP;
 * under SB_SKIP nothing runs (the separate record would still record the stale Y when the module's
 * own skip flag is clear, which sb_module_decide never leaves so). records: caller-owned device
 * scratch of M * (N / 128) * 8 floats, 16-byte aligned. x, cache: bf16 [M][N], 16-byte aligned.
 * Requires N % 256 == 0 and N <= 16384 (SB_EUNSUPPORTED), else as sb_linear. ws holds two slot
 * arrays for M rows (sb_workspace_size). */
sb_status sb_linear_module_record(const void* X, const sb_fp4* a4 /* host */, const sb_i8* a8 /* host */,
                                  int32_t* prec, const sb_weight* w /* host */, int32_t epilogue, void* Y, int64_t M,
                                  const void* x, void* cache, int32_t update_cache, float* records, sb_stats* stats,
                                  sb_module_state* state, void* ws, sb_stream stream);

/* sb_prepass without a caller workspace. The paper has no counterpart: this exists for callers
 * that cannot allocate device memory -- e.g. a plugin inside a host program that owns the whole
 * device-memory pool and forbids other allocations, or a latency-critical loop that must never
 * call cudaMalloc/cudaFree because they can synchronise the device. The scratch that sb_prepass
 * keeps in `ws` lives instead in a 256 KiB array compiled into the library (present on every GPU
 * that loads it, until the process exits); this call allocates nothing. Arguments and results are
 * exactly those of sb_prepass; M may be at most SB_STATIC_MAX_ROWS (SB_ESHAPE otherwise, nothing
 * launched). The first call on a device looks up the array's device address with
 * cudaGetSymbolAddress (that device must be current), so make that first call before any stream
 * capture. Every call on a device shares the one array: calls that can overlap on the GPU (other
 * streams, other host threads) race and must be serialised by the caller. There is no workspace
 * for sb_check to read, so the call ends by copying the array's device error word into
 * stats->error: SB_OK, SB_ETIMEOUT (a bounded wait gave up; codes and statistics are then
 * undefined), SB_ENONFINITE (X held Inf/NaN; also in stats->nonfinite) or SB_EINVAL. The next
 * call clears the word, so read stats->error after each call. */
#define SB_STATIC_MAX_ROWS 65536
sb_status sb_prepass_static(const void* X, const void* X_ref, int64_t M, int64_t K,
                            const sb_config* cfg /* host */, int32_t mode, int32_t* prec,
                            const sb_fp4* a4 /* host */, const sb_i8* a8 /* host */, sb_stats* stats,
                            sb_stream stream);

/* Temporal Delta Cache, reuse path ("write-up" section 二: a skipped module reuses the cached
 * result; explainer section 3: the old outcome is used and adjusted very slightly). The cache
 * keeps the module's residual D = y - x of its last computed step:
 *   sb_tdc_refresh: if the module computed this step (state->skip == 0), delta = bf16(y - x);
 *   sb_tdc_reuse:   if the module is skipped this step (state->skip == 1), y = bf16(x + delta);
 * each element as the FP32 difference / sum of the bf16 values, rounded to nearest even. The other
 * case writes nothing, so both calls can be enqueued every step after sb_tdc_step. x, y, delta:
 * bf16 [M][C] row-major, caller-owned, 16-byte aligned (SB_EALIGN); C a multiple of 8
 * (SB_EUNSUPPORTED); state: device sb_module_state. */
sb_status sb_tdc_refresh(const void* x, const void* y, void* delta, int64_t M, int64_t C, const sb_module_state* state,
                         sb_stream stream);
sb_status sb_tdc_reuse(const void* x, const void* delta, void* y, int64_t M, int64_t C, const sb_module_state* state,
                       sb_stream stream);

/* ---- Token sharding: several GPUs each own a contiguous range of a tensor's rows ----
 * Every step of the path works row by row except the reductions of the pre-pass and of the TDC
 * record, which span all rows. A shard runs the row work of its rows and writes its FP64 group
 * partials (one 48-byte slot per aligned 16-row group) into a slot array covering the whole tensor.
 * Shards write disjoint ranges of that array, so gathering them is exact: e.g. an int64 all-reduce
 * SUM of zero-filled copies. Every GPU then runs the same final reduction over the gathered array
 * and obtains the statistics record, PDR verdict or module-state update of the whole tensor, bit
 * for bit those of the unsharded call, because the group slots are aligned subtrees of the same
 * FP64 tree. The weights are replicated, so the GEMMs need no exchange. ("write-up" sections 一,
 * 二, 三: the difference, the TDC change and the outlier ratio are statistics of whole tensors.)
 * Shard rules: row0 % 16 == 0, and M % 16 == 0 unless the shard ends the tensor. */

/* Bytes of the slot array of an M_total-row tensor (48 per 16-row group), or -1 if M_total < 1. */
int64_t sb_group_slots_bytes(int64_t M_total);

/* The row work of sb_prepass on rows [row0, row0 + M) of an M_total-row tensor: X, X_ref and a8
 * hold only these M rows ([M][K] bf16; a8 codes [M][K], scales [M]). Writes the shard's group
 * slots at slots + (row0 / 16) * 48 and, in SB_PREPASS_QUANT mode when *prec says INT8, the INT8
 * codes and per-token scales. Writes no statistics record and leaves *prec unchanged; the NVFP4
 * codes need the whole tensor's amax (sb_nvfp4_encode after sb_prepass_finish). slots: device,
 * 16-byte aligned, sb_group_slots_bytes(M_total) bytes. Validation as sb_prepass (SB_ESHAPE for
 * the shard rules). */
sb_status sb_prepass_partial(const void* X, const void* X_ref, int64_t M, int64_t K, int64_t row0,
                             int64_t M_total, const sb_config* cfg /* host */, int32_t mode,
                             int32_t* prec, const sb_i8* a8 /* host */, void* slots, void* ws,
                             sb_stream stream);

/* The final reduction of a sharded pre-pass of an M_total x K tensor over the gathered slots:
 * writes *stats and, in SB_PREPASS_QUANT mode, applies PDR to *prec, as sb_prepass does. has_ref:
 * whether the shards were given X_ref. */
sb_status sb_prepass_finish(const void* slots, int64_t M_total, int64_t K, int32_t has_ref,
                            const sb_config* cfg /* host */, int32_t mode, int32_t* prec,
                            sb_stats* stats, void* ws, sb_stream stream);

/* NVFP4 codes of the rows X [M][K] (a shard, or a whole tensor) from finished statistics: tensor
 * scale from stats->amax_rot (the whole tensor's), E4M3 block scales in the tiled layout of these
 * M rows. Writes a4 only when *prec is SB_NVFP4 (prec NULL: always). */
sb_status sb_nvfp4_encode(const void* X, int64_t M, int64_t K, const sb_config* cfg /* host */,
                          const int32_t* prec, const sb_stats* stats, const sb_fp4* a4 /* host */,
                          void* ws, sb_stream stream);

/* The row work of sb_tdc_record on rows [row0, row0 + M) of an M_total-row module output: the
 * shard's sums of |y_new - y_cache| and |y_cache| into the slot array, and the cache refresh with
 * update_cache. The module state is read (skip, whether an output was recorded), not written. */
sb_status sb_tdc_record_partial(const void* y_new, void* y_cache, int64_t M, int64_t C, int64_t row0,
                                int64_t M_total, int32_t update_cache,
                                const sb_module_state* state, void* slots, void* ws, sb_stream stream);

/* The final TDC reduction over the gathered slots: delta and the state update of sb_tdc_record
 * (d from d_src when given). Does nothing if state->skip. */
sb_status sb_tdc_finish(const void* slots, int64_t M_total, int64_t C, const sb_stats* d_src,
                        sb_module_state* state, void* ws, sb_stream stream);

/* ---- Delta tokens ("DeltaQuant: 4-bit Video Diffusion Models with Spatiotemporal Delta
 * Smoothing", abstract): the activations of the latent video grid are grouped into local 3D
 * spatiotemporal cubes; each cube's mean token (its core token) is kept in FP8 and only the
 * differences of the cube's tokens from it (delta tokens) take the 4-bit path. A linear layer is
 * then Y = GEMM(delta) + core W^T (+ bias), the core product computed once per cube and added to
 * each of its tokens. With these calls the caller runs: sb_delta_split; sb_prepass and sb_linear
 * on the delta tokens (SB_OUT_F32, no bias, no epilogue); sb_linear in BF16 on the core tokens
 * (SB_OUT_F32, with the bias); sb_delta_combine (adds them, optional GELU, bf16 output). */

/* Token layout: tokens [0, text) are text tokens, one cube each; token text + (f*height + h)*width
 * + w is position (f, h, w) of the frames x height x width latent grid, in cube (f/ct, h/ch, w/cw)
 * (edge cubes are smaller). Cubes are numbered text first, then grid cubes in (f, h, w) order. */
typedef struct {
  int64_t text, frames, height, width;
  int32_t ct, ch, cw; /* cube extent; ct*ch*cw <= 32 */
} sb_cubes;

/* Number of cubes of M tokens, or -1 when M != text + frames*height*width or a size is invalid. */
int64_t sb_cube_count(const sb_cubes* cubes /* host */, int64_t M);

/* Split X [M][K] bf16 into core and delta tokens. Per cube and channel: the pairwise FP32 sum of
 * the cube's tokens (token order, zero-padded to a power of two) divided by the token count; per
 * core token a = max |mean|, scale s = a / 448, codes E4M3(RN(mean * (448 / a))) (satfinite;
 * a = 0: s = 0, zero codes; if 448 / a overflows, nonzero means take +-448), dequantized core
 * dec = E4M3 value * s. Writes core_codes [ncube][K] (E4M3 bytes), core_scale [ncube] (FP32),
 * core_bf16 [ncube][K] (bf16(dec), the operand of the core GEMM) and delta [M][K] (bf16 of the
 * FP32 difference x - dec). K % 64 == 0, K <= 16384 (SB_EUNSUPPORTED); pointers 16-byte aligned
 * (SB_EALIGN); the cube layout must cover M tokens (SB_ESHAPE). */
sb_status sb_delta_split(const void* X, int64_t M, int64_t K, const sb_cubes* cubes /* host */,
                         uint8_t* core_codes, float* core_scale, void* core_bf16, void* delta,
                         sb_stream stream);

/* Y [M][N] bf16 = act(Y_delta[t] + Y_core[cube(t)]) with Y_delta FP32 [M][N] and Y_core FP32
 * [ncube][N] (the core GEMM's output, which carries the bias); epilogue SB_EPI_NONE or
 * SB_EPI_GELU_TANH (tanh GELU with the hardware tanh approximation). N % 8 == 0. */
sb_status sb_delta_combine(const float* y_delta, const float* y_core, int64_t M, int64_t N,
                           const sb_cubes* cubes /* host */, int32_t epilogue, void* Y, sb_stream stream);

/* The delta tokens' linear layer with the combine fused into the GEMM epilogue: as sb_linear on
 * the delta tokens (delta, a4, a8, prec, w, epilogue, out_dtype, Y, M, ws as there), except that
 * every output row t adds, before the activation, row cube(t) of y_core (FP32 [cubes][N], the
 * cores' product with W without bias, e.g. from sb_linear on the cores with SB_OUT_F32):
 *   Y[t] = act(linear(delta)[t] + bias + y_core[cube(t)]).
 * The same result as sb_linear with SB_OUT_F32 and no bias followed by sb_delta_combine, within
 * FP32 rounding (the bias enters the sum at another place), without the FP32 round trip. y_core:
 * 16-byte aligned (SB_EALIGN); cubes: as for sb_delta_split, covering the M tokens (SB_ESHAPE);
 * out_dtype SB_OUT_BF16 or SB_OUT_F32 (SB_EINVAL otherwise). */
sb_status sb_delta_linear(const void* delta, const sb_fp4* a4 /* host */, const sb_i8* a8 /* host */,
                          const int32_t* prec, const sb_weight* w /* host */, const float* y_core,
                          const sb_cubes* cubes /* host */, int32_t epilogue, int32_t out_dtype, void* Y, int64_t M,
                          void* ws, sb_stream stream);

/* The same reuse path with the residual kept in FP8 ("write-up" section 七: the cache's history
 * may be stored in low-precision formats): half the bytes of the bf16 residual.
 *   sb_tdc_refresh_fp8: if the module computed this step (state->skip == 0), per token row m:
 *     d = RN(y - x) in FP32, a = max |d| over the row, scale[m] = a / 448, codes E4M3(RN(d * (448 /
 *     a))) with round to nearest even and saturation to +-448; a = 0 gives scale 0 and zero codes;
 *     448 / a overflowing FP32 gives +-448 (0x7e / 0xfe) for nonzero d and 0 for zeros;
 *   sb_tdc_reuse_fp8: if the module is skipped this step (state->skip == 1),
 *     y = bf16(x + RN(E4M3(code) * scale[m])).
 * The other case writes nothing. x, y: bf16 [M][C]; codes: E4M3 [M][C]; scale: FP32 [M]; all
 * row-major, caller-owned device memory; x, y, codes 16-byte aligned, scale 4-byte aligned
 * (SB_EALIGN); C a multiple of 16 (SB_EUNSUPPORTED); M in [1, 2^30] (SB_ESHAPE). */
sb_status sb_tdc_refresh_fp8(const void* x, const void* y, uint8_t* codes, float* scale, int64_t M, int64_t C,
                             const sb_module_state* state, sb_stream stream);
sb_status sb_tdc_reuse_fp8(const void* x, const uint8_t* codes, const float* scale, void* y, int64_t M, int64_t C,
                           const sb_module_state* state, sb_stream stream);

/* Bounded device-side wait, the library's failure-detection primitive (the pages have no
 * counterpart). Enqueues on `stream` a one-thread kernel that polls the device int32 at `flag`
 * (acquire loads, ~1 us apart) until it equals `value`. If `limit_ns` nanoseconds of device time
 * (%globaltimer) pass first, the kernel records SB_ETIMEOUT in `ws` and returns, so the stream and
 * the context stay usable; sb_check() reports the timeout. The flag must be written by something
 * that does not need this kernel to finish or to be co-scheduled with it: the host (mapped or
 * managed memory), a copy or kernel that completes before this launch, or another device -- never
 * a kernel launched later on the same GPU. flag: 4-byte aligned device pointer (SB_EALIGN);
 * limit_ns in [1, 1e10] (SB_EINVAL otherwise). */
sb_status sb_wait_flag(const int32_t* flag, int32_t value, uint64_t limit_ns, void* ws, sb_stream stream);

/* Stall drill of the quantized linear layer (testing only; the pages have no counterpart). Arms
 * the next sb_linear launch of this process, on any stream or host thread, as follows: in every
 * CTA pair of the GEMM the leader CTA's TMA producer skips the copies of its `withhold_stage`-th
 * K-block stage (counted from 0 over all the pair's tiles) but still announces their bytes, so that
 * stage never completes. The MMA issuer's wait for it gives up after `limit_ns` of device time
 * (%globaltimer); the abort flag and the same limit end every other wait of both CTAs, in-flight
 * copies and MMAs are drained, tensor memory is freed, and the launch records SB_ETIMEOUT in its
 * workspace (read by sb_check). Its output is undefined; the stream and context stay usable. The
 * launch that takes the drill disarms it; a stage index past the pair's last K-block leaves that
 * launch unaffected. A layer whose precision flag reads SB_SKIP also takes (and drops) the drill.
 * withhold_stage >= 0 and limit_ns in [1e5, 1e10], else SB_EINVAL. */
sb_status sb_drill_gemm_stall(int64_t withhold_stage, uint64_t limit_ns);

/* Synchronise `stream`, read and clear the device error word of `ws`. Returns SB_OK,
 * SB_ETIMEOUT, SB_ENONFINITE, SB_EINVAL or SB_ECUDA. */
sb_status sb_check(void* ws, sb_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* SIXBIT_H */
