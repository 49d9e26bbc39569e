// sb_kernels.h -- internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sixbit.h"

namespace sb {

struct PrepassLaunch {
  const void* X;
  const void* R;
  int64_t M, K;
  int B;
  int mode;
  int32_t* prec;
  int force_int8;
  int8_t* q8;
  float* s8;
  double rho;
  int force;
  void* groups;
  void* hdr;
  sb_stats* stats;
  int finish;  // 1: reduce the slots in the last CTA; 0: write this launch's group slots only
};

struct Nvfp4Launch {
  const void* X;
  int64_t M, K;
  int B;
  const int32_t* prec;
  const sb_stats* stats;
  uint8_t* codes;
  uint8_t* sf;
  float* gscale;
  void* hdr;  // workspace header: error word
};

struct TdcLaunch {
  const void* Y;
  void* Cache;
  int64_t M, C;
  int update;
  const sb_stats* dsrc;
  sb_module_state* st;
  void* groups;
  void* hdr;
  int finish;
};

// The final reduction over gathered group slots: op 0 pre-pass (mode, has_ref as in
// PrepassLaunch), op 2 TDC record. The row kernels' arguments carry M = the whole tensor's rows.
struct FinishLaunch {
  int op;
  int has_ref;
  int64_t M, K;
  int mode;
  int32_t* prec;
  double rho;
  int force;
  const sb_stats* dsrc;
  sb_module_state* st;
  const void* groups;
  void* hdr;
  sb_stats* stats;
};

struct GemmLaunch {
  int64_t M, N, K;
  int B;
  const int32_t* prec;
  // BF16 path
  const void* X;
  const void* W16;
  // INT8 path
  const int8_t* A8;
  const float* sA8;
  const int8_t* B8;
  const float* sB8;
  // NVFP4 path
  const uint8_t* A4;
  const uint8_t* sfA4;
  const float* gA4;
  const uint8_t* B4;
  const uint8_t* sfB4;
  const float* gB4;
  const void* bias;
  int epilogue;
  int out_dtype;
  void* Y;
  void* hdr;
  // delta tokens: output row t adds row cube(t) of rowadd (FP32 [cubes][N]) before the activation
  const float* rowadd;
  int64_t ra_T, ra_H, ra_W;
  int ra_ct, ra_ch, ra_cw;
  // FFN-pair fusion: the output's chunk records (float4 [M][N/128], rotated amax over Hadamard
  // blocks of 128 columns; needs 256-wide tiles)
  float* records;
  // Module record fused into the GEMM (the output is the module's output; needs 256-wide tiles):
  // the module input, the cached output (read, then refreshed), the per-chunk partial sums
  // (float4 [M][N/128][2]) and the module state that gates the cache's part
  const void* mr_x;
  void* mr_c;
  float* mr_rec;
  const sb_module_state* mr_st;
  int mr_update;
};

cudaError_t launch_prepass(const PrepassLaunch& p, cudaStream_t s);
cudaError_t launch_nvfp4(const Nvfp4Launch& p, cudaStream_t s);
cudaError_t launch_rotate(const void* X, float* Y, int64_t M, int64_t K, int B, cudaStream_t s);
cudaError_t launch_tdc_record(const TdcLaunch& p, cudaStream_t s);

// The module's output record: the difference statistic of Y against X and the TDC record of Y
// against the cache, one pass (OP_REC).
struct RecordLaunch {
  const void* Y;
  const void* X;
  void* Cache;
  int64_t M, C;
  int32_t* prec;
  double rho;
  int force;
  int update;
  sb_stats* stats;
  sb_module_state* st;
  void* groups;
  void* groups2;
  void* hdr;
};
cudaError_t launch_module_record(const RecordLaunch& p, cudaStream_t s);
cudaError_t launch_finish(const FinishLaunch& p, cudaStream_t s);
cudaError_t launch_prepass_chunks(const PrepassLaunch& p, float* chunks, cudaStream_t s);

// The decision of one module step: its layers' rules and precision flags (at most kDecideMax).
constexpr int kDecideMax = 8;
struct DecideLayers {
  int n;
  double a[kDecideMax], b[kDecideMax], tau[kDecideMax];
  int32_t* prec[kDecideMax];
};
cudaError_t launch_decide(sb_module_state* st, double thr, int force, const DecideLayers& L, cudaStream_t s);
cudaError_t launch_gemm(const GemmLaunch& p, cudaStream_t s, const char** why);
// Chunk records of a bf16 tensor (sb_chunk_records).
// The module record from the GEMM's per-chunk partial sums (sb_linear_module_record): the rows'
// sums, the group slots and both finishes of the fused record.
cudaError_t launch_fold_modrec(const RecordLaunch& p, const float* rec, cudaStream_t s);
cudaError_t launch_chunk_records(const void* X, int64_t M, int64_t K, int B, float* out, cudaStream_t s);
// Arms the stall drill for the next launch_gemm (sb_drill_gemm_stall).
void arm_gemm_stall_drill(int64_t withhold_stage, uint64_t wait_ns);

cudaError_t launch_state_init(sb_module_state* st, cudaStream_t s);
cudaError_t launch_tdc_step(sb_module_state* st, double thr, cudaStream_t s);
cudaError_t launch_select(const sb_module_state* st, double a, double b, double tau, int force, int32_t* prec,
                          cudaStream_t s);
cudaError_t launch_set_i32(int32_t* p, int32_t v, cudaStream_t s);
cudaError_t launch_wait_flag(const int32_t* flag, int32_t value, uint64_t limit_ns, void* hdr, cudaStream_t s);
cudaError_t launch_tdc_refresh(const void* x, const void* y, void* d, int64_t n, const sb_module_state* st,
                               cudaStream_t s);
cudaError_t launch_tdc_reuse(const void* x, const void* d, void* y, int64_t n, const sb_module_state* st,
                             cudaStream_t s);
cudaError_t launch_tdc_refresh8(const void* x, const void* y, uint8_t* codes, float* scale, int64_t M, int64_t C,
                                const sb_module_state* st, cudaStream_t s);
cudaError_t launch_tdc_reuse8(const void* x, const uint8_t* codes, const float* scale, void* y, int64_t M, int64_t C,
                              const sb_module_state* st, cudaStream_t s);
cudaError_t launch_ws_init(void* ws, size_t bytes, cudaStream_t s);

// Delta tokens: the cube geometry (text tokens, grid F x H x W, cube ct x ch x cw).
struct DeltaCubes {
  int64_t T, F, H, W;
  int ct, ch, cw;
};
constexpr int kDeltaMaxCube = 32;  // tokens per cube
cudaError_t launch_delta_split(const void* X, int64_t K, const DeltaCubes& c, int64_t ncube, uint8_t* codes,
                               float* scale, void* core16, void* delta, cudaStream_t s);
cudaError_t launch_delta_combine(const float* Yd, const float* Yc, int64_t M, int64_t N, const DeltaCubes& c,
                                 int gelu, void* Y, cudaStream_t s);

sb_status report_error(sb_status st, const char* msg);

}  // namespace sb
