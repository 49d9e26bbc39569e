// api.cu -- the C ABI declared in include/sixbit.h: argument validation and kernel dispatch.
//
// No entry point allocates device memory; scratch lives in the caller's workspace:
//   [0, 128)    WsHeader (device error word, last-CTA tickets)
//   [128, 224)  sb_stats scratch (weight preparation)
//   [224, 228)  int32 precision scratch (weight preparation)
//   [256, ...)  one 48-byte GroupSlot per aligned group of 16 rows (kGroupRows), then (for
//               sb_module_record) a second such array right after the call's own groups
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "sb_device.cuh"
#include "sb_kernels.h"

namespace {

thread_local std::string g_err;

sb_status fail(sb_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

sb_status ok() {
  g_err.clear();
  return SB_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_block(int b) { return b == 16 || b == 32 || b == 64 || b == 128 || b == 256; }

constexpr size_t kOffStats = 128;
constexpr size_t kOffGroups = 256;

void* ws_groups(void* ws) { return static_cast<char*>(ws) + kOffGroups; }
sb_stats* ws_stats(void* ws) { return reinterpret_cast<sb_stats*>(static_cast<char*>(ws) + kOffStats); }

sb_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SB_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define SB_REQUIRE(cond, status, ...) \
  do {                                \
    if (!(cond)) return fail(status, __VA_ARGS__); \
  } while (0)

#define SB_ALIGNED(p, name) SB_REQUIRE(aligned16(p), SB_EALIGN, "%s is not 16-byte aligned", name)

sb_status check_rows_cols(int64_t M, int64_t K, int32_t block) {
  SB_REQUIRE(M >= 1, SB_ESHAPE, "M must be >= 1 (got %lld)", (long long)M);
  SB_REQUIRE(M <= (int64_t)1 << 30, SB_ESHAPE, "M too large (%lld)", (long long)M);
  SB_REQUIRE(valid_block(block), SB_EUNSUPPORTED, "block must be 16, 32, 64, 128 or 256 (got %d)", block);
  SB_REQUIRE(K >= 64 && K % 64 == 0, SB_EUNSUPPORTED, "K must be a positive multiple of 64 (got %lld)",
             (long long)K);
  SB_REQUIRE(K % block == 0, SB_EUNSUPPORTED, "K (%lld) must be a multiple of the block (%d)", (long long)K, block);
  SB_REQUIRE(K <= sb::kMaxK, SB_EUNSUPPORTED, "K must be <= %d (got %lld)", sb::kMaxK, (long long)K);
  return SB_OK;
}

}  // namespace

namespace sb {
// Lets other translation units of the library report a failure through sb_last_error().
sb_status report_error(sb_status st, const char* msg) { return fail(st, "%s", msg); }
}  // namespace sb

extern "C" {

const char* sb_version(void) { return "sixbit 0.1 (sm_100a)"; }

const char* sb_last_error(void) { return g_err.c_str(); }

sb_status sb_workspace_size(int64_t max_M, int64_t max_K, size_t* bytes) {
  SB_REQUIRE(bytes != nullptr, SB_EINVAL, "bytes is NULL");
  SB_REQUIRE(max_M >= 0 && max_K >= 0, SB_ESHAPE, "negative size");
  const size_t groups = (size_t)sb::ceil_div(max_M > 0 ? max_M : 1, sb::kGroupRows);
  size_t b = kOffGroups + 2 * groups * sizeof(sb::GroupSlot);  // two slot arrays (sb_module_record)
  *bytes = (b + 255) & ~(size_t)255;
  return ok();
}

sb_status sb_workspace_init(void* ws, size_t bytes, sb_stream stream) {
  SB_REQUIRE(ws != nullptr, SB_EINVAL, "ws is NULL");
  SB_ALIGNED(ws, "ws");
  SB_REQUIRE(bytes >= kOffGroups, SB_ESHAPE, "workspace smaller than %zu bytes", kOffGroups);
  cudaError_t e = sb::launch_ws_init(ws, bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_workspace_init");
  return ok();
}

int64_t sb_fp4_sf_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return -1;
  return ((rows + 127) / 128) * 128 * (cols / 16);
}

sb_status sb_state_init(sb_module_state* state, sb_stream stream) {
  SB_REQUIRE(state != nullptr, SB_EINVAL, "state is NULL");
  SB_ALIGNED(state, "state");
  cudaError_t e = sb::launch_state_init(state, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_state_init");
  return ok();
}

sb_status sb_rotate(const void* X, float* Y, int64_t M, int64_t K, int32_t block, sb_stream stream) {
  SB_REQUIRE(X && Y, SB_EINVAL, "X and Y are required");
  SB_ALIGNED(X, "X");
  SB_ALIGNED(Y, "Y");
  sb_status st = check_rows_cols(M, K, block);
  if (st != SB_OK) return st;
  cudaError_t e = sb::launch_rotate(X, Y, M, K, block, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_rotate");
  return ok();
}

static sb_status check_fp4(const sb_fp4* t, int64_t rows, int64_t cols, const char* name) {
  SB_REQUIRE(t->codes && t->sf && t->gscale, SB_EINVAL, "%s: codes, sf and gscale are required", name);
  SB_ALIGNED(t->codes, name);
  SB_ALIGNED(t->sf, name);
  SB_REQUIRE((reinterpret_cast<uintptr_t>(t->gscale) & 3u) == 0, SB_EALIGN, "%s.gscale misaligned", name);
  SB_REQUIRE(t->rows == rows && t->cols == cols, SB_ESHAPE, "%s is [%lld x %lld], expected [%lld x %lld]", name,
             (long long)t->rows, (long long)t->cols, (long long)rows, (long long)cols);
  return SB_OK;
}

static sb_status check_i8(const sb_i8* t, int64_t rows, int64_t cols, const char* name) {
  SB_REQUIRE(t->codes && t->scale, SB_EINVAL, "%s: codes and scale are required", name);
  SB_ALIGNED(t->codes, name);
  SB_ALIGNED(t->scale, name);
  SB_REQUIRE(t->rows == rows && t->cols == cols, SB_ESHAPE, "%s is [%lld x %lld], expected [%lld x %lld]", name,
             (long long)t->rows, (long long)t->cols, (long long)rows, (long long)cols);
  return SB_OK;
}

sb_status sb_prepare_weight(const void* W, const void* bias, int64_t N, int64_t K, int32_t block, sb_weight* w,
                            void* ws, sb_stream stream) {
  SB_REQUIRE(W && w && ws, SB_EINVAL, "W, w and ws are required");
  SB_ALIGNED(W, "W");
  SB_ALIGNED(ws, "ws");
  if (bias) SB_ALIGNED(bias, "bias");
  sb_status st = check_rows_cols(N, K, block);
  if (st != SB_OK) return st;
  if ((st = check_fp4(&w->w4, N, K, "w->w4")) != SB_OK) return st;
  if ((st = check_i8(&w->w8, N, K, "w->w8")) != SB_OK) return st;
  w->w_bf16 = W;
  w->bias_bf16 = bias;
  w->N = N;
  w->K = K;
  w->block = block;
  cudaStream_t s = (cudaStream_t)stream;
  sb::PrepassLaunch p{};
  p.finish = 1;
  p.X = W;
  p.R = nullptr;
  p.M = N;
  p.K = K;
  p.B = block;
  p.mode = SB_PREPASS_QUANT;
  p.prec = nullptr;
  p.force_int8 = 1;
  p.q8 = w->w8.codes;
  p.s8 = w->w8.scale;
  p.rho = 0.0;
  p.force = -1;
  p.groups = ws_groups(ws);
  p.hdr = ws;
  p.stats = ws_stats(ws);
  cudaError_t e = sb::launch_prepass(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "sb_prepare_weight (rotation, INT8)");
  sb::Nvfp4Launch q{};
  q.X = W;
  q.M = N;
  q.K = K;
  q.B = block;
  q.prec = nullptr;
  q.stats = ws_stats(ws);
  q.codes = w->w4.codes;
  q.sf = w->w4.sf;
  q.gscale = w->w4.gscale;
  q.hdr = ws;
  e = sb::launch_nvfp4(q, s);
  if (e != cudaSuccess) return cuda_fail(e, "sb_prepare_weight (NVFP4)");
  return ok();
}

sb_status sb_tdc_step(sb_module_state* state, const sb_config* cfg, sb_stream stream) {
  SB_REQUIRE(state && cfg, SB_EINVAL, "state and cfg are required");
  SB_ALIGNED(state, "state");
  cudaError_t e = sb::launch_tdc_step(state, cfg->tdc_thresh, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_tdc_step");
  return ok();
}

sb_status sb_select_precision(const sb_module_state* state, const sb_rule* rule, const sb_config* cfg,
                              int32_t* prec, sb_stream stream) {
  SB_REQUIRE(state && rule && cfg && prec, SB_EINVAL, "state, rule, cfg and prec are required");
  SB_ALIGNED(state, "state");
  SB_REQUIRE((reinterpret_cast<uintptr_t>(prec) & 3u) == 0, SB_EALIGN, "prec misaligned");
  SB_REQUIRE(cfg->force_prec >= -1 && cfg->force_prec <= 2, SB_EINVAL, "force_prec must be -1, 0, 1 or 2");
  cudaError_t e = sb::launch_select(state, rule->a, rule->b, rule->tau, cfg->force_prec, prec, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_select_precision");
  return ok();
}

sb_status sb_prepass_chunks(const void* X, float* chunks, int64_t M, int64_t K, const sb_config* cfg, int32_t mode,
                            int32_t* prec, const sb_fp4* a4, const sb_i8* a8, sb_stats* stats, void* ws,
                            sb_stream stream) {
  SB_REQUIRE(X && chunks && cfg && stats && ws, SB_EINVAL, "X, chunks, cfg, stats and ws are required");
  SB_ALIGNED(X, "X");
  SB_ALIGNED(chunks, "chunks");
  SB_ALIGNED(stats, "stats");
  SB_ALIGNED(ws, "ws");
  SB_REQUIRE(mode == SB_PREPASS_QUANT || mode == SB_PREPASS_STATS, SB_EINVAL, "mode must be QUANT or STATS");
  SB_REQUIRE(cfg->force_prec >= -1 && cfg->force_prec <= 2, SB_EINVAL, "force_prec must be -1, 0, 1 or 2");
  sb_status st = check_rows_cols(M, K, cfg->block);
  if (st != SB_OK) return st;
  SB_REQUIRE(cfg->block <= 128 && K % 128 == 0, SB_EUNSUPPORTED,
             "chunk records need block <= 128 and K a multiple of 128 (got block %d, K %lld)", (int)cfg->block,
             (long long)K);
  if (mode == SB_PREPASS_QUANT) {
    SB_REQUIRE(prec && a4 && a8, SB_EINVAL, "QUANT mode needs prec, a4 and a8");
    if ((st = check_fp4(a4, M, K, "a4")) != SB_OK) return st;
    if ((st = check_i8(a8, M, K, "a8")) != SB_OK) return st;
  }
  if (prec) SB_REQUIRE((reinterpret_cast<uintptr_t>(prec) & 3u) == 0, SB_EALIGN, "prec misaligned");
  cudaStream_t s = (cudaStream_t)stream;
  sb::PrepassLaunch p{};
  p.finish = 1;
  p.X = X;
  p.M = M;
  p.K = K;
  p.B = cfg->block;
  p.mode = mode;
  p.prec = prec;
  p.q8 = (mode == SB_PREPASS_QUANT) ? a8->codes : nullptr;
  p.s8 = (mode == SB_PREPASS_QUANT) ? a8->scale : nullptr;
  p.rho = cfg->rho;
  p.force = cfg->force_prec;
  p.groups = ws_groups(ws);
  p.hdr = ws;
  p.stats = stats;
  cudaError_t e = sb::launch_prepass_chunks(p, chunks, s);
  if (e != cudaSuccess) return cuda_fail(e, "sb_prepass_chunks");
  if (mode == SB_PREPASS_QUANT) {
    sb::Nvfp4Launch q{};
    q.X = X;
    q.M = M;
    q.K = K;
    q.B = cfg->block;
    q.prec = prec;
    q.stats = stats;
    q.codes = a4->codes;
    q.sf = a4->sf;
    q.gscale = a4->gscale;
    q.hdr = ws;
    e = sb::launch_nvfp4(q, s);
    if (e != cudaSuccess) return cuda_fail(e, "sb_prepass_chunks (NVFP4 encode)");
  }
  return ok();
}

sb_status sb_module_decide(sb_module_state* state, const sb_config* cfg, int32_t n, const sb_rule* rules,
                           int32_t* const* precs, sb_stream stream) {
  SB_REQUIRE(state && cfg && rules && precs, SB_EINVAL, "state, cfg, rules and precs are required");
  SB_ALIGNED(state, "state");
  SB_REQUIRE(n >= 1 && n <= sb::kDecideMax, SB_EINVAL, "n must be in [1, %d] (got %d)", sb::kDecideMax, (int)n);
  SB_REQUIRE(cfg->force_prec >= -1 && cfg->force_prec <= 2, SB_EINVAL, "force_prec must be -1, 0, 1 or 2");
  sb::DecideLayers L{};
  L.n = n;
  for (int i = 0; i < n; ++i) {
    SB_REQUIRE(precs[i] != nullptr, SB_EINVAL, "precs[%d] is NULL", i);
    SB_REQUIRE((reinterpret_cast<uintptr_t>(precs[i]) & 3u) == 0, SB_EALIGN, "precs[%d] misaligned", i);
    L.a[i] = rules[i].a;
    L.b[i] = rules[i].b;
    L.tau[i] = rules[i].tau;
    L.prec[i] = precs[i];
  }
  cudaError_t e = sb::launch_decide(state, cfg->tdc_thresh, cfg->force_prec, L, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_module_decide");
  return ok();
}

sb_status sb_prepass(const void* X, const void* X_ref, int64_t M, int64_t K, const sb_config* cfg, int32_t mode,
                     int32_t* prec, const sb_fp4* a4, const sb_i8* a8, sb_stats* stats, void* ws,
                     sb_stream stream) {
  SB_REQUIRE(X && cfg && stats && ws, SB_EINVAL, "X, cfg, stats and ws are required");
  SB_ALIGNED(X, "X");
  if (X_ref) SB_ALIGNED(X_ref, "X_ref");
  SB_ALIGNED(stats, "stats");
  SB_ALIGNED(ws, "ws");
  SB_REQUIRE(mode == SB_PREPASS_QUANT || mode == SB_PREPASS_STATS, SB_EINVAL, "mode must be QUANT or STATS");
  SB_REQUIRE(cfg->force_prec >= -1 && cfg->force_prec <= 2, SB_EINVAL, "force_prec must be -1, 0, 1 or 2");
  sb_status st = check_rows_cols(M, K, cfg->block);
  if (st != SB_OK) return st;
  if (mode == SB_PREPASS_QUANT) {
    SB_REQUIRE(prec && a4 && a8, SB_EINVAL, "QUANT mode needs prec, a4 and a8");
    if ((st = check_fp4(a4, M, K, "a4")) != SB_OK) return st;
    if ((st = check_i8(a8, M, K, "a8")) != SB_OK) return st;
  }
  if (prec) SB_REQUIRE((reinterpret_cast<uintptr_t>(prec) & 3u) == 0, SB_EALIGN, "prec misaligned");
  cudaStream_t s = (cudaStream_t)stream;
  sb::PrepassLaunch p{};
  p.finish = 1;
  p.X = X;
  p.R = X_ref;
  p.M = M;
  p.K = K;
  p.B = cfg->block;
  p.mode = mode;
  p.prec = prec;
  p.force_int8 = 0;
  p.q8 = (mode == SB_PREPASS_QUANT) ? a8->codes : nullptr;
  p.s8 = (mode == SB_PREPASS_QUANT) ? a8->scale : nullptr;
  p.rho = cfg->rho;
  p.force = cfg->force_prec;
  p.groups = ws_groups(ws);
  p.hdr = ws;
  p.stats = stats;
  cudaError_t e = sb::launch_prepass(p, s);
  if (e != cudaSuccess) return cuda_fail(e, "sb_prepass (statistics)");
  if (mode == SB_PREPASS_QUANT) {
    sb::Nvfp4Launch q{};
    q.X = X;
    q.M = M;
    q.K = K;
    q.B = cfg->block;
    q.prec = prec;
    q.stats = stats;
    q.codes = a4->codes;
    q.sf = a4->sf;
    q.gscale = a4->gscale;
    q.hdr = ws;
    e = sb::launch_nvfp4(q, s);
    if (e != cudaSuccess) return cuda_fail(e, "sb_prepass (NVFP4 encode)");
  }
  return ok();
}

// sb_linear's validation and launch; `row` (may be NULL) adds a gathered row to each output row.
static sb_status linear_impl(const void* X, const sb_fp4* a4, const sb_i8* a8, const int32_t* prec,
                             const sb_weight* w, int32_t epilogue, int32_t out_dtype, void* Y, int64_t M, void* ws,
                             sb_stream stream, const sb::GemmLaunch* row) {
  SB_REQUIRE(prec && w && Y && ws, SB_EINVAL, "prec, w, Y and ws are required");
  SB_ALIGNED(Y, "Y");
  SB_ALIGNED(ws, "ws");
  SB_REQUIRE(epilogue == SB_EPI_NONE || epilogue == SB_EPI_GELU_TANH, SB_EINVAL, "bad epilogue");
  SB_REQUIRE(out_dtype == SB_OUT_BF16 || out_dtype == SB_OUT_F32 || out_dtype == SB_OUT_RAW, SB_EINVAL,
             "bad out_dtype");
  const int64_t N = w->N, K = w->K;
  SB_REQUIRE(M >= 1 && M <= (int64_t)1 << 30, SB_ESHAPE, "M out of range (%lld)", (long long)M);
  SB_REQUIRE(N >= 32 && N % 32 == 0 && N <= (int64_t)1 << 20, SB_EUNSUPPORTED, "N must be a multiple of 32 (got %lld)",
             (long long)N);
  SB_REQUIRE(K >= 128 && K % 128 == 0 && K <= (int64_t)1 << 20, SB_EUNSUPPORTED,
             "K must be a positive multiple of 128 (got %lld)", (long long)K);
  SB_REQUIRE(valid_block(w->block), SB_EUNSUPPORTED, "weight block %d unsupported", w->block);
  if (w->bias_bf16) SB_ALIGNED(w->bias_bf16, "bias");
  sb::GemmLaunch L{};
  L.M = M;
  L.N = N;
  L.K = K;
  L.B = w->block;
  L.prec = prec;
  if (X && w->w_bf16) {
    SB_ALIGNED(X, "X");
    SB_ALIGNED(w->w_bf16, "w->w_bf16");
    L.X = X;
    L.W16 = w->w_bf16;
  }
  sb_status st;
  if (a8 && a8->codes) {
    if ((st = check_i8(a8, M, K, "a8")) != SB_OK) return st;
    if ((st = check_i8(&w->w8, N, K, "w->w8")) != SB_OK) return st;
    L.A8 = a8->codes;
    L.sA8 = a8->scale;
    L.B8 = w->w8.codes;
    L.sB8 = w->w8.scale;
  }
  if (a4 && a4->codes) {
    if ((st = check_fp4(a4, M, K, "a4")) != SB_OK) return st;
    if ((st = check_fp4(&w->w4, N, K, "w->w4")) != SB_OK) return st;
    L.A4 = a4->codes;
    L.sfA4 = a4->sf;
    L.gA4 = a4->gscale;
    L.B4 = w->w4.codes;
    L.sfB4 = w->w4.sf;
    L.gB4 = w->w4.gscale;
  }
  SB_REQUIRE(L.X || L.A8 || L.A4, SB_EINVAL, "no operand set given (X+w_bf16, a8 or a4)");
  L.bias = w->bias_bf16;
  L.epilogue = epilogue;
  L.out_dtype = out_dtype;
  L.Y = Y;
  L.hdr = ws;
  if (row) {
    L.records = row->records;
    L.mr_x = row->mr_x;
    L.mr_c = row->mr_c;
    L.mr_rec = row->mr_rec;
    L.mr_st = row->mr_st;
    L.mr_update = row->mr_update;
    L.rowadd = row->rowadd;
    L.ra_T = row->ra_T;
    L.ra_H = row->ra_H;
    L.ra_W = row->ra_W;
    L.ra_ct = row->ra_ct;
    L.ra_ch = row->ra_ch;
    L.ra_cw = row->ra_cw;
  }
  const char* why = "kernel launch";
  cudaError_t e = sb::launch_gemm(L, (cudaStream_t)stream, &why);
  if (e != cudaSuccess) return cuda_fail(e, why);
  return ok();
}

sb_status sb_linear(const void* X, const sb_fp4* a4, const sb_i8* a8, const int32_t* prec, const sb_weight* w,
                    int32_t epilogue, int32_t out_dtype, void* Y, int64_t M, void* ws, sb_stream stream) {
  return linear_impl(X, a4, a8, prec, w, epilogue, out_dtype, Y, M, ws, stream, nullptr);
}

sb_status sb_linear_records(const void* X, const sb_fp4* a4, const sb_i8* a8, const int32_t* prec,
                            const sb_weight* w, int32_t epilogue, void* Y, int64_t M, int32_t block, float* records,
                            void* ws, sb_stream stream) {
  SB_REQUIRE(records && w, SB_EINVAL, "records and w are required");
  SB_ALIGNED(records, "records");
  SB_REQUIRE(block == 128, SB_EUNSUPPORTED, "the GEMM's chunk records are for block 128 (got %d)", (int)block);
  SB_REQUIRE(w->N % 256 == 0, SB_EUNSUPPORTED, "chunk records need N a multiple of 256 (got %lld)", (long long)w->N);
  sb::GemmLaunch rec{};
  rec.records = records;
  return linear_impl(X, a4, a8, prec, w, epilogue, SB_OUT_BF16, Y, M, ws, stream, &rec);
}

sb_status sb_linear_module_record(const void* X, const sb_fp4* a4, const sb_i8* a8, int32_t* prec,
                                  const sb_weight* w, int32_t epilogue, void* Y, int64_t M, const void* x, void* cache,
                                  int32_t update_cache, float* records, sb_stats* stats, sb_module_state* state,
                                  void* ws, sb_stream stream) {
  SB_REQUIRE(w && x && cache && records && stats && state && ws, SB_EINVAL,
             "w, x, cache, records, stats, state and ws are required");
  SB_ALIGNED(x, "x");
  SB_ALIGNED(cache, "cache");
  SB_ALIGNED(records, "records");
  SB_ALIGNED(stats, "stats");
  SB_ALIGNED(state, "state");
  SB_REQUIRE(w->N % 256 == 0 && w->N <= sb::kMaxK, SB_EUNSUPPORTED,
             "the fused module record needs N a multiple of 256 up to %d (got %lld)", sb::kMaxK, (long long)w->N);
  SB_REQUIRE(M >= 1 && M <= (int64_t)1 << 30, SB_ESHAPE, "M out of range (%lld)", (long long)M);
  sb::GemmLaunch rec{};
  rec.mr_x = x;
  rec.mr_c = cache;
  rec.mr_rec = records;
  rec.mr_st = state;
  rec.mr_update = update_cache ? 1 : 0;
  const sb_status st = linear_impl(X, a4, a8, prec, w, epilogue, SB_OUT_BF16, Y, M, ws, stream, &rec);
  if (st != SB_OK) return st;
  sb::RecordLaunch p{};
  p.Y = Y;
  p.X = x;
  p.Cache = cache;
  p.M = M;
  p.C = w->N;
  p.prec = prec;
  p.rho = 0.0;
  p.force = -1;
  p.update = update_cache ? 1 : 0;
  p.stats = stats;
  p.st = state;
  p.groups = ws_groups(ws);
  p.groups2 = static_cast<char*>(ws_groups(ws)) + sb::ceil_div(M, sb::kGroupRows) * sizeof(sb::GroupSlot);
  p.hdr = ws;
  cudaError_t e = sb::launch_fold_modrec(p, records, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "k_fold_modrec launch");
  return ok();
}

sb_status sb_chunk_records(const void* X, int64_t M, int64_t K, int32_t block, float* records, sb_stream stream) {
  SB_REQUIRE(X && records, SB_EINVAL, "X and records are required");
  SB_ALIGNED(X, "X");
  SB_ALIGNED(records, "records");
  SB_REQUIRE(M >= 1 && M <= (int64_t)1 << 30, SB_ESHAPE, "M out of range (%lld)", (long long)M);
  SB_REQUIRE(K >= 128 && K % 128 == 0 && K <= sb::kMaxK, SB_EUNSUPPORTED, "K must be a multiple of 128 in [128, %d]",
             sb::kMaxK);
  SB_REQUIRE(block == 16 || block == 32 || block == 64 || block == 128, SB_EUNSUPPORTED,
             "chunk records need block in {16, 32, 64, 128} (got %d)", (int)block);
  cudaError_t e = sb::launch_chunk_records(X, M, K, block, records, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "k_chunk_records launch");
  return ok();
}

sb_status sb_tdc_record(const void* y_new, void* y_cache, int64_t M, int64_t C, const sb_stats* d_src,
                        int32_t update_cache, sb_module_state* state, void* ws, sb_stream stream) {
  SB_REQUIRE(y_new && y_cache && state && ws, SB_EINVAL, "y_new, y_cache, state and ws are required");
  SB_ALIGNED(y_new, "y_new");
  SB_ALIGNED(y_cache, "y_cache");
  SB_ALIGNED(state, "state");
  SB_ALIGNED(ws, "ws");
  if (d_src) SB_ALIGNED(d_src, "d_src");
  SB_REQUIRE(M >= 1 && M <= (int64_t)1 << 30, SB_ESHAPE, "M out of range (%lld)", (long long)M);
  SB_REQUIRE(C >= 8 && C % 8 == 0 && C <= sb::kMaxK, SB_EUNSUPPORTED, "C must be a multiple of 8 in [8, %d]",
             sb::kMaxK);
  sb::TdcLaunch p{};
  p.finish = 1;
  p.Y = y_new;
  p.Cache = y_cache;
  p.M = M;
  p.C = C;
  p.update = update_cache ? 1 : 0;
  p.dsrc = d_src;
  p.st = state;
  p.groups = ws_groups(ws);
  p.hdr = ws;
  cudaError_t e = sb::launch_tdc_record(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_tdc_record");
  return ok();
}

// ---------------------------------------------------------------------------------------------
// Token sharding: partial row work into a slot array, gathered elsewhere, then the final reduction
// ---------------------------------------------------------------------------------------------

int64_t sb_group_slots_bytes(int64_t M_total) {
  if (M_total < 1) return -1;
  return sb::ceil_div(M_total, sb::kGroupRows) * (int64_t)sizeof(sb::GroupSlot);
}

static sb_status check_shard(int64_t M, int64_t row0, int64_t M_total, const void* slots) {
  SB_REQUIRE(slots != nullptr, SB_EINVAL, "slots is NULL");
  SB_ALIGNED(slots, "slots");
  SB_REQUIRE(M >= 1 && row0 >= 0 && M_total <= (int64_t)1 << 30 && row0 + M <= M_total, SB_ESHAPE,
             "shard rows [%lld, %lld) outside the tensor's %lld rows", (long long)row0, (long long)(row0 + M),
             (long long)M_total);
  SB_REQUIRE(row0 % sb::kGroupRows == 0, SB_ESHAPE, "row0 (%lld) must be a multiple of %d", (long long)row0,
             sb::kGroupRows);
  SB_REQUIRE(row0 + M == M_total || M % sb::kGroupRows == 0, SB_ESHAPE,
             "a shard that does not end the tensor must hold a multiple of %d rows (got %lld)", sb::kGroupRows,
             (long long)M);
  return SB_OK;
}

static char* shard_slots(void* slots, int64_t row0) {
  return static_cast<char*>(slots) + (row0 / sb::kGroupRows) * (int64_t)sizeof(sb::GroupSlot);
}

sb_status sb_prepass_partial(const void* X, const void* X_ref, int64_t M, int64_t K, int64_t row0, int64_t M_total,
                             const sb_config* cfg, int32_t mode, int32_t* prec, const sb_i8* a8, void* slots, void* ws,
                             sb_stream stream) {
  SB_REQUIRE(X && cfg && ws, SB_EINVAL, "X, cfg and ws are required");
  SB_ALIGNED(X, "X");
  if (X_ref) SB_ALIGNED(X_ref, "X_ref");
  SB_ALIGNED(ws, "ws");
  SB_REQUIRE(mode == SB_PREPASS_QUANT || mode == SB_PREPASS_STATS, SB_EINVAL, "mode must be QUANT or STATS");
  SB_REQUIRE(cfg->force_prec >= -1 && cfg->force_prec <= 2, SB_EINVAL, "force_prec must be -1, 0, 1 or 2");
  sb_status st = check_rows_cols(M, K, cfg->block);
  if (st != SB_OK) return st;
  if ((st = check_shard(M, row0, M_total, slots)) != SB_OK) return st;
  if (mode == SB_PREPASS_QUANT) {
    SB_REQUIRE(prec && a8, SB_EINVAL, "QUANT mode needs prec and a8");
    if ((st = check_i8(a8, M, K, "a8")) != SB_OK) return st;
  }
  if (prec) SB_REQUIRE((reinterpret_cast<uintptr_t>(prec) & 3u) == 0, SB_EALIGN, "prec misaligned");
  sb::PrepassLaunch p{};
  p.finish = 0;
  p.X = X;
  p.R = X_ref;
  p.M = M;
  p.K = K;
  p.B = cfg->block;
  p.mode = mode;
  p.prec = prec;
  p.q8 = (mode == SB_PREPASS_QUANT) ? a8->codes : nullptr;
  p.s8 = (mode == SB_PREPASS_QUANT) ? a8->scale : nullptr;
  p.rho = cfg->rho;
  p.force = cfg->force_prec;
  p.groups = shard_slots(slots, row0);
  p.hdr = ws;
  cudaError_t e = sb::launch_prepass(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_prepass_partial");
  return ok();
}

sb_status sb_prepass_finish(const void* slots, int64_t M_total, int64_t K, int32_t has_ref, const sb_config* cfg,
                            int32_t mode, int32_t* prec, sb_stats* stats, void* ws, sb_stream stream) {
  SB_REQUIRE(slots && cfg && stats && ws, SB_EINVAL, "slots, cfg, stats and ws are required");
  SB_ALIGNED(slots, "slots");
  SB_ALIGNED(stats, "stats");
  SB_ALIGNED(ws, "ws");
  SB_REQUIRE(mode == SB_PREPASS_QUANT || mode == SB_PREPASS_STATS, SB_EINVAL, "mode must be QUANT or STATS");
  SB_REQUIRE(mode == SB_PREPASS_STATS || prec, SB_EINVAL, "QUANT mode needs prec");
  sb_status st = check_rows_cols(M_total, K, cfg->block);
  if (st != SB_OK) return st;
  if (prec) SB_REQUIRE((reinterpret_cast<uintptr_t>(prec) & 3u) == 0, SB_EALIGN, "prec misaligned");
  sb::FinishLaunch f{};
  f.op = 0;
  f.has_ref = has_ref ? 1 : 0;
  f.M = M_total;
  f.K = K;
  f.mode = mode;
  f.prec = prec;
  f.rho = cfg->rho;
  f.force = cfg->force_prec;
  f.groups = slots;
  f.hdr = ws;
  f.stats = stats;
  cudaError_t e = sb::launch_finish(f, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_prepass_finish");
  return ok();
}

sb_status sb_nvfp4_encode(const void* X, int64_t M, int64_t K, const sb_config* cfg, const int32_t* prec,
                          const sb_stats* stats, const sb_fp4* a4, void* ws, sb_stream stream) {
  SB_REQUIRE(X && cfg && stats && a4 && ws, SB_EINVAL, "X, cfg, stats, a4 and ws are required");
  SB_ALIGNED(X, "X");
  SB_ALIGNED(stats, "stats");
  SB_ALIGNED(ws, "ws");
  sb_status st = check_rows_cols(M, K, cfg->block);
  if (st != SB_OK) return st;
  if ((st = check_fp4(a4, M, K, "a4")) != SB_OK) return st;
  if (prec) SB_REQUIRE((reinterpret_cast<uintptr_t>(prec) & 3u) == 0, SB_EALIGN, "prec misaligned");
  sb::Nvfp4Launch q{};
  q.X = X;
  q.M = M;
  q.K = K;
  q.B = cfg->block;
  q.prec = prec;
  q.stats = stats;
  q.codes = a4->codes;
  q.sf = a4->sf;
  q.gscale = a4->gscale;
  q.hdr = ws;
  cudaError_t e = sb::launch_nvfp4(q, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_nvfp4_encode");
  return ok();
}

sb_status sb_tdc_record_partial(const void* y_new, void* y_cache, int64_t M, int64_t C, int64_t row0, int64_t M_total,
                                int32_t update_cache, const sb_module_state* state, void* slots, void* ws,
                                sb_stream stream) {
  SB_REQUIRE(y_new && y_cache && state && ws, SB_EINVAL, "y_new, y_cache, state and ws are required");
  SB_ALIGNED(y_new, "y_new");
  SB_ALIGNED(y_cache, "y_cache");
  SB_ALIGNED(state, "state");
  SB_ALIGNED(ws, "ws");
  SB_REQUIRE(C >= 8 && C % 8 == 0 && C <= sb::kMaxK, SB_EUNSUPPORTED, "C must be a multiple of 8 in [8, %d]",
             sb::kMaxK);
  sb_status st = check_shard(M, row0, M_total, slots);
  if (st != SB_OK) return st;
  sb::TdcLaunch p{};
  p.finish = 0;
  p.Y = y_new;
  p.Cache = y_cache;
  p.M = M;
  p.C = C;
  p.update = update_cache ? 1 : 0;
  p.st = const_cast<sb_module_state*>(state);
  p.groups = shard_slots(slots, row0);
  p.hdr = ws;
  cudaError_t e = sb::launch_tdc_record(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_tdc_record_partial");
  return ok();
}

sb_status sb_tdc_finish(const void* slots, int64_t M_total, int64_t C, const sb_stats* d_src, sb_module_state* state,
                        void* ws, sb_stream stream) {
  SB_REQUIRE(slots && state && ws, SB_EINVAL, "slots, state and ws are required");
  SB_ALIGNED(slots, "slots");
  SB_ALIGNED(state, "state");
  SB_ALIGNED(ws, "ws");
  if (d_src) SB_ALIGNED(d_src, "d_src");
  SB_REQUIRE(M_total >= 1 && M_total <= (int64_t)1 << 30, SB_ESHAPE, "M_total out of range (%lld)",
             (long long)M_total);
  SB_REQUIRE(C >= 8 && C % 8 == 0 && C <= sb::kMaxK, SB_EUNSUPPORTED, "C must be a multiple of 8 in [8, %d]",
             sb::kMaxK);
  sb::FinishLaunch f{};
  f.op = 2;
  f.has_ref = 1;
  f.M = M_total;
  f.K = C;
  f.dsrc = d_src;
  f.st = state;
  f.groups = slots;
  f.hdr = ws;
  cudaError_t e = sb::launch_finish(f, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_tdc_finish");
  return ok();
}

static sb_status tdc_combine_args(const void* a, const void* b, const void* out, int64_t M, int64_t C,
                                  const sb_module_state* state) {
  SB_REQUIRE(a && b && out && state, SB_EINVAL, "x, the residual, the output and state are required");
  SB_ALIGNED(a, "x");
  SB_ALIGNED(b, "second input");
  SB_ALIGNED(out, "output");
  SB_REQUIRE(M >= 1 && M <= (int64_t)1 << 30, SB_ESHAPE, "M out of range (%lld)", (long long)M);
  SB_REQUIRE(C >= 8 && C % 8 == 0 && C <= (int64_t)1 << 20, SB_EUNSUPPORTED, "C must be a multiple of 8 (got %lld)",
             (long long)C);
  return SB_OK;
}

sb_status sb_tdc_refresh(const void* x, const void* y, void* delta, int64_t M, int64_t C, const sb_module_state* state,
                         sb_stream stream) {
  const sb_status st = tdc_combine_args(x, y, delta, M, C, state);
  if (st != SB_OK) return st;
  cudaError_t e = sb::launch_tdc_refresh(x, y, delta, M * C, state, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "k_tdc_combine (refresh) launch");
  return ok();
}

sb_status sb_tdc_reuse(const void* x, const void* delta, void* y, int64_t M, int64_t C, const sb_module_state* state,
                       sb_stream stream) {
  const sb_status st = tdc_combine_args(x, delta, y, M, C, state);
  if (st != SB_OK) return st;
  cudaError_t e = sb::launch_tdc_reuse(x, delta, y, M * C, state, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "k_tdc_combine (reuse) launch");
  return ok();
}

static sb_status tdc_fp8_args(const void* x, const void* yd, const void* codes, const float* scale, int64_t M,
                              int64_t C, const sb_module_state* state) {
  SB_REQUIRE(x && yd && codes && scale && state, SB_EINVAL, "x, y, codes, scale and state are required");
  SB_ALIGNED(x, "x");
  SB_ALIGNED(yd, "y");
  SB_ALIGNED(codes, "codes");
  SB_REQUIRE((reinterpret_cast<uintptr_t>(scale) & 3u) == 0, SB_EALIGN, "scale misaligned");
  SB_REQUIRE(M >= 1 && M <= (int64_t)1 << 30, SB_ESHAPE, "M out of range (%lld)", (long long)M);
  SB_REQUIRE(C >= 16 && C % 16 == 0 && C <= (int64_t)1 << 20, SB_EUNSUPPORTED,
             "C must be a multiple of 16 (got %lld)", (long long)C);
  return SB_OK;
}

sb_status sb_tdc_refresh_fp8(const void* x, const void* y, uint8_t* codes, float* scale, int64_t M, int64_t C,
                             const sb_module_state* state, sb_stream stream) {
  const sb_status st = tdc_fp8_args(x, y, codes, scale, M, C, state);
  if (st != SB_OK) return st;
  cudaError_t e = sb::launch_tdc_refresh8(x, y, codes, scale, M, C, state, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "k_tdc_refresh8 launch");
  return ok();
}

sb_status sb_tdc_reuse_fp8(const void* x, const uint8_t* codes, const float* scale, void* y, int64_t M, int64_t C,
                           const sb_module_state* state, sb_stream stream) {
  const sb_status st = tdc_fp8_args(x, y, codes, scale, M, C, state);
  if (st != SB_OK) return st;
  cudaError_t e = sb::launch_tdc_reuse8(x, codes, scale, y, M, C, state, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "k_tdc_reuse8 launch");
  return ok();
}

sb_status sb_module_record(const void* y, const void* x, void* cache, int64_t M, int64_t C, int32_t* prec,
                           int32_t update_cache, sb_stats* stats, sb_module_state* state, void* ws,
                           sb_stream stream) {
  SB_REQUIRE(y && x && cache && stats && state && ws, SB_EINVAL, "y, x, cache, stats, state and ws are required");
  SB_ALIGNED(y, "y");
  SB_ALIGNED(x, "x");
  SB_ALIGNED(cache, "cache");
  SB_ALIGNED(stats, "stats");
  SB_ALIGNED(state, "state");
  SB_ALIGNED(ws, "ws");
  if (prec) SB_REQUIRE((reinterpret_cast<uintptr_t>(prec) & 3u) == 0, SB_EALIGN, "prec misaligned");
  SB_REQUIRE(M >= 1 && M <= (int64_t)1 << 30, SB_ESHAPE, "M out of range (%lld)", (long long)M);
  SB_REQUIRE(C >= 64 && C % 64 == 0 && C <= sb::kMaxK, SB_EUNSUPPORTED, "C must be a multiple of 64 in [64, %d]",
             sb::kMaxK);
  sb::RecordLaunch p{};
  p.Y = y;
  p.X = x;
  p.Cache = cache;
  p.M = M;
  p.C = C;
  p.prec = prec;
  p.rho = 0.0;
  p.force = -1;
  p.update = update_cache ? 1 : 0;
  p.stats = stats;
  p.st = state;
  p.groups = ws_groups(ws);
  p.groups2 = static_cast<char*>(ws_groups(ws)) + sb::ceil_div(M, sb::kGroupRows) * sizeof(sb::GroupSlot);
  p.hdr = ws;
  cudaError_t e = sb::launch_module_record(p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_module_record");
  return ok();
}

sb_status sb_wait_flag(const int32_t* flag, int32_t value, uint64_t limit_ns, void* ws, sb_stream stream) {
  SB_REQUIRE(flag && ws, SB_EINVAL, "flag and ws are required");
  SB_REQUIRE((reinterpret_cast<uintptr_t>(flag) & 3u) == 0, SB_EALIGN, "flag misaligned");
  SB_REQUIRE(limit_ns >= 1 && limit_ns <= 10000000000ull, SB_EINVAL, "limit_ns must be in [1, 1e10] (got %llu)",
             (unsigned long long)limit_ns);
  cudaError_t e = sb::launch_wait_flag(flag, value, limit_ns, ws, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "k_wait_flag launch");
  return ok();
}

sb_status sb_drill_gemm_stall(int64_t withhold_stage, uint64_t limit_ns) {
  SB_REQUIRE(withhold_stage >= 0, SB_EINVAL, "withhold_stage must be >= 0 (got %lld)", (long long)withhold_stage);
  SB_REQUIRE(limit_ns >= 100000ull && limit_ns <= 10000000000ull, SB_EINVAL,
             "limit_ns must be in [1e5, 1e10] (got %llu)", (unsigned long long)limit_ns);
  sb::arm_gemm_stall_drill(withhold_stage, limit_ns);
  return ok();
}

static bool cubes_geom(const sb_cubes* c, int64_t M, sb::DeltaCubes* g, int64_t* ncube) {
  if (!c || c->text < 0 || c->frames < 1 || c->height < 1 || c->width < 1 || c->ct < 1 || c->ch < 1 || c->cw < 1)
    return false;
  if ((int64_t)c->ct * c->ch * c->cw > sb::kDeltaMaxCube) return false;
  if (c->frames > ((int64_t)1 << 30) / c->height / c->width) return false;
  if (M != c->text + c->frames * c->height * c->width) return false;
  g->T = c->text;
  g->F = c->frames;
  g->H = c->height;
  g->W = c->width;
  g->ct = c->ct;
  g->ch = c->ch;
  g->cw = c->cw;
  *ncube = c->text + sb::ceil_div(c->frames, c->ct) * sb::ceil_div(c->height, c->ch) * sb::ceil_div(c->width, c->cw);
  return true;
}

int64_t sb_cube_count(const sb_cubes* cubes, int64_t M) {
  sb::DeltaCubes g;
  int64_t n = -1;
  if (!cubes_geom(cubes, M, &g, &n)) return -1;
  return n;
}

sb_status sb_delta_linear(const void* delta, const sb_fp4* a4, const sb_i8* a8, const int32_t* prec,
                          const sb_weight* w, const float* y_core, const sb_cubes* cubes, int32_t epilogue,
                          int32_t out_dtype, void* Y, int64_t M, void* ws, sb_stream stream) {
  SB_REQUIRE(y_core && cubes, SB_EINVAL, "y_core and cubes are required");
  SB_ALIGNED(y_core, "y_core");
  SB_REQUIRE(out_dtype == SB_OUT_BF16 || out_dtype == SB_OUT_F32, SB_EINVAL, "out_dtype must be BF16 or F32");
  sb::DeltaCubes g;
  int64_t ncube = 0;
  SB_REQUIRE(cubes_geom(cubes, M, &g, &ncube), SB_ESHAPE, "the cube layout does not cover the %lld tokens",
             (long long)M);
  sb::GemmLaunch row{};
  row.rowadd = y_core;
  row.ra_T = g.T;
  row.ra_H = g.H;
  row.ra_W = g.W;
  row.ra_ct = g.ct;
  row.ra_ch = g.ch;
  row.ra_cw = g.cw;
  return linear_impl(delta, a4, a8, prec, w, epilogue, out_dtype, Y, M, ws, stream, &row);
}

sb_status sb_delta_split(const void* X, int64_t M, int64_t K, const sb_cubes* cubes, uint8_t* core_codes,
                         float* core_scale, void* core_bf16, void* delta, sb_stream stream) {
  SB_REQUIRE(X && cubes && core_codes && core_scale && core_bf16 && delta, SB_EINVAL,
             "X, cubes, core_codes, core_scale, core_bf16 and delta are required");
  SB_ALIGNED(X, "X");
  SB_ALIGNED(core_codes, "core_codes");
  SB_ALIGNED(core_scale, "core_scale");
  SB_ALIGNED(core_bf16, "core_bf16");
  SB_ALIGNED(delta, "delta");
  SB_REQUIRE(K >= 64 && K % 64 == 0 && K <= sb::kMaxK, SB_EUNSUPPORTED, "K must be a multiple of 64 in [64, %d]",
             sb::kMaxK);
  sb::DeltaCubes g;
  int64_t ncube = 0;
  SB_REQUIRE(M >= 1 && cubes_geom(cubes, M, &g, &ncube), SB_ESHAPE,
             "the cube layout must cover the M = %lld tokens (text + frames*height*width) with cubes of at most %d "
             "tokens",
             (long long)M, sb::kDeltaMaxCube);
  cudaError_t e = sb::launch_delta_split(X, K, g, ncube, core_codes, core_scale, core_bf16, delta, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_delta_split");
  return ok();
}

sb_status sb_delta_combine(const float* y_delta, const float* y_core, int64_t M, int64_t N, const sb_cubes* cubes,
                           int32_t epilogue, void* Y, sb_stream stream) {
  SB_REQUIRE(y_delta && y_core && cubes && Y, SB_EINVAL, "y_delta, y_core, cubes and Y are required");
  SB_ALIGNED(y_delta, "y_delta");
  SB_ALIGNED(y_core, "y_core");
  SB_ALIGNED(Y, "Y");
  SB_REQUIRE(epilogue == SB_EPI_NONE || epilogue == SB_EPI_GELU_TANH, SB_EINVAL, "bad epilogue");
  SB_REQUIRE(N >= 8 && N % 8 == 0 && N <= (int64_t)1 << 20, SB_EUNSUPPORTED, "N must be a multiple of 8");
  sb::DeltaCubes g;
  int64_t ncube = 0;
  SB_REQUIRE(M >= 1 && cubes_geom(cubes, M, &g, &ncube), SB_ESHAPE,
             "the cube layout must cover the M = %lld tokens", (long long)M);
  cudaError_t e = sb::launch_delta_combine(y_delta, y_core, M, N, g, epilogue == SB_EPI_GELU_TANH ? 1 : 0, Y,
                                           (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sb_delta_combine");
  return ok();
}

sb_status sb_check(void* ws, sb_stream stream) {
  SB_REQUIRE(ws != nullptr, SB_EINVAL, "ws is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "sb_check (stream synchronize)");
  uint32_t err = 0;
  e = cudaMemcpy(&err, ws, sizeof(err), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "sb_check (read error word)");
  if (err != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "sb_check (clear error word)");
    return fail((sb_status)err, "device reported status %u", err);
  }
  return ok();
}

}  // extern "C"
