// prepass_static.cu -- sb_prepass_static: the activation pre-pass with library-owned scratch.
//
// sb_prepass needs a caller-allocated workspace for its cross-CTA partial sums, tickets and
// error word. Some callers cannot allocate device memory at all: a plugin running inside a host
// application that owns the whole device-memory pool and forbids any other allocation, or a
// latency-critical loop that must never call cudaMalloc / cudaFree (they can synchronise the
// device). For them this entry point keeps the scratch in a fixed array compiled into the library
// (kScratchBytes on every GPU that loads it, held until the process exits) and allocates nothing.
//
// In host code the array's name is only a stand-in, never a device address: the address is
// looked up with cudaGetSymbolAddress, once per device, with that device current, on the first
// call made on that device; later calls reuse it.
//
// Device-side errors (a bounded wait that gave up, non-finite input) land in the array's error
// word, which no caller can read; the call therefore ends with a one-thread kernel that copies
// that word into stats->error.
#include <mutex>

#include "sb_device.cuh"
#include "sb_kernels.h"

namespace {

constexpr size_t kScratchBytes = 256 * 1024;  // the workspace of up to SB_STATIC_MAX_ROWS rows
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// The scratch's device error word (the first word of its header) into the caller's statistics
// record, after the pre-pass kernels on the same stream.
__global__ void k_copy_error(const uint32_t* err, sb_stats* stats) { stats->error = (int32_t)*err; }

}  // namespace

extern "C" sb_status sb_prepass_static(const void* X, const void* X_ref, int64_t M, int64_t K,
                                       const sb_config* cfg, int32_t mode, int32_t* prec, const sb_fp4* a4,
                                       const sb_i8* a8, sb_stats* stats, sb_stream stream) {
  if (M > SB_STATIC_MAX_ROWS)
    return sb::report_error(SB_ESHAPE, "sb_prepass_static: M exceeds SB_STATIC_MAX_ROWS (65536 rows)");
  size_t need = 0;
  const sb_status st = sb_workspace_size(M > 0 ? M : 1, K > 0 ? K : 1, &need);
  if (st != SB_OK) return st;
  if (need > kScratchBytes)
    return sb::report_error(SB_ESHAPE, "sb_prepass_static: problem needs more scratch than the static array");
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return sb::report_error(SB_ECUDA, "sb_prepass_static: no current CUDA device (or device index >= 64)");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr)
        return sb::report_error(SB_ECUDA, "sb_prepass_static: cudaGetSymbolAddress of the scratch array failed");
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  // The array keeps what the previous call left there; its counters and error word must start at
  // zero, so they are cleared on the stream before the kernels run.
  if (cudaMemsetAsync(scratch, 0, 256, (cudaStream_t)stream) != cudaSuccess)
    return sb::report_error(SB_ECUDA, "sb_prepass_static: clearing the scratch header failed");
  const sb_status ps = sb_prepass(X, X_ref, M, K, cfg, mode, prec, a4, a8, stats, scratch, stream);
  if (ps != SB_OK) return ps;
  k_copy_error<<<1, 1, 0, (cudaStream_t)stream>>>(static_cast<const uint32_t*>(scratch), stats);
  if (cudaGetLastError() != cudaSuccess)
    return sb::report_error(SB_ECUDA, "sb_prepass_static: launching the error-word copy failed");
  return SB_OK;
}
