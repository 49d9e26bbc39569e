// decide.cu -- single-thread decision kernels: TDC skip check and per-layer precision choice.
//
// They run on the device so that a whole denoising step can be enqueued without host round trips;
// the FP64 arithmetic is written with explicit round-to-nearest operations (no fused
// multiply-add) so every decision is reproducible bit for bit.
#include "sb_device.cuh"
#include "sb_kernels.h"

namespace sb {

__global__ void k_state_init(sb_module_state* st) {
  if (threadIdx.x != 0) return;
  st->prev_d = 0.0;
  st->acc = 0.0;
  st->delta = 0.0;
  st->have_d = 0;
  st->n_out = 0;
  st->last_skipped = 0;
  st->skip = 0;
  st->steps = 0;
  st->reserved[0] = st->reserved[1] = st->reserved[2] = 0;
}

// "write-up" section 二: two outputs are needed before the change can be predicted; after that
// the per-step change delta accumulates and the module is skipped while the sum stays within the
// threshold. A skipped step leaves no input/output difference for the next step (section 三).
__device__ __forceinline__ void tdc_step(sb_module_state* st, double thr) {
  int skip = 0;
  if (st->n_out >= 2) {
    const double acc = __dadd_rn(st->acc, st->delta);
    st->acc = acc;
    skip = (acc <= thr) ? 1 : 0;
  }
  st->skip = skip;
  if (skip) {
    st->have_d = 0;
    st->last_skipped = 1;
  }
  st->steps += 1;
}

// "write-up" sections 一 and 三: INT8 for a changing module (linear rule on the previous step's
// difference), NVFP4 for a stable one, INT8 after a restart or at the first step.
__device__ __forceinline__ int32_t select_precision(const sb_module_state* st, double a, double b, double tau,
                                                    int force) {
  if (st->skip) return SB_SKIP;
  if (force >= 0) return force;
  if (!st->have_d) return SB_INT8;
  const double v = __dadd_rn(__dmul_rn(a, st->prev_d), b);
  return (v > tau) ? SB_INT8 : SB_NVFP4;
}

__global__ void k_tdc_step(sb_module_state* st, double thr) {
  if (threadIdx.x == 0) tdc_step(st, thr);
}

__global__ void k_select(const sb_module_state* st, double a, double b, double tau, int force, int32_t* prec) {
  if (threadIdx.x == 0) *prec = select_precision(st, a, b, tau, force);
}

// Both in one launch: the module's TDC check, then the precision of each of its layers.
__global__ void k_decide(sb_module_state* st, double thr, int force, DecideLayers L) {
  if (threadIdx.x != 0) return;
  tdc_step(st, thr);
  for (int i = 0; i < L.n; ++i) *L.prec[i] = select_precision(st, L.a[i], L.b[i], L.tau[i], force);
}

__global__ void k_set_i32(int32_t* p, int32_t v) {
  if (threadIdx.x == 0) *p = v;
}

__global__ void k_zero(uint32_t* p, size_t words) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < words; i += (size_t)gridDim.x * blockDim.x)
    p[i] = 0u;
}

cudaError_t launch_state_init(sb_module_state* st, cudaStream_t s) {
  k_state_init<<<1, 32, 0, s>>>(st);
  return cudaGetLastError();
}

cudaError_t launch_tdc_step(sb_module_state* st, double thr, cudaStream_t s) {
  k_tdc_step<<<1, 32, 0, s>>>(st, thr);
  return cudaGetLastError();
}

cudaError_t launch_select(const sb_module_state* st, double a, double b, double tau, int force, int32_t* prec,
                          cudaStream_t s) {
  k_select<<<1, 32, 0, s>>>(st, a, b, tau, force, prec);
  return cudaGetLastError();
}

cudaError_t launch_decide(sb_module_state* st, double thr, int force, const DecideLayers& L, cudaStream_t s) {
  k_decide<<<1, 32, 0, s>>>(st, thr, force, L);
  return cudaGetLastError();
}

// Bounded wait for *flag == value: acquire loads, a short sleep between polls, %globaltimer for
// the deadline. On timeout the workspace error word records SB_ETIMEOUT and the kernel returns.
__global__ void k_wait_flag(const int32_t* flag, int32_t value, uint64_t limit_ns, WsHeader* hdr) {
  const uint64_t t0 = globaltimer();
  while (true) {
    int32_t v;
    asm volatile("ld.acquire.sys.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v == value) return;
    if (globaltimer() - t0 > limit_ns) {
      set_error(hdr, SB_ETIMEOUT);
      return;
    }
    __nanosleep(1000);
  }
}

cudaError_t launch_wait_flag(const int32_t* flag, int32_t value, uint64_t limit_ns, void* hdr, cudaStream_t s) {
  k_wait_flag<<<1, 1, 0, s>>>(flag, value, limit_ns, reinterpret_cast<WsHeader*>(hdr));
  return cudaGetLastError();
}

cudaError_t launch_set_i32(int32_t* p, int32_t v, cudaStream_t s) {
  k_set_i32<<<1, 32, 0, s>>>(p, v);
  return cudaGetLastError();
}

cudaError_t launch_ws_init(void* ws, size_t bytes, cudaStream_t s) {
  const size_t words = bytes / 4;
  const unsigned grid = (unsigned)((words + 255) / 256 < 1024 ? (words + 255) / 256 : 1024);
  k_zero<<<grid > 0 ? grid : 1, 256, 0, s>>>(reinterpret_cast<uint32_t*>(ws), words);
  return cudaGetLastError();
}

}  // namespace sb
