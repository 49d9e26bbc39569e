// reuse.cu -- the Temporal Delta Cache's reuse path ("write-up" section 二: a skipped module
// reuses the cached result; explainer section 3: the old outcome is used and adjusted very
// slightly). At a computed step the module's residual is kept, D = bf16(y - x); at a skipped step
// the output is y = bf16(x + D). Both are streaming kernels gated on the device by the module's
// skip decision, so a whole step stays enqueued without host round trips.
#include "sb_device.cuh"
#include "sb_kernels.h"

namespace sb {

// 8 bf16 of a and b -> 8 bf16 of round_to_nearest_even(fp32(a) op fp32(b)), op = b - a or a + b.
template <bool SUB>
__device__ __forceinline__ uint4 combine8(const uint4& a, const uint4& b) {
  float fa[8], fb[8];
  unpack8(a, fa);
  unpack8(b, fb);
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float r0 = SUB ? __fsub_rn(fb[2 * i], fa[2 * i]) : __fadd_rn(fa[2 * i], fb[2 * i]);
    const float r1 = SUB ? __fsub_rn(fb[2 * i + 1], fa[2 * i + 1]) : __fadd_rn(fa[2 * i + 1], fb[2 * i + 1]);
    const __nv_bfloat162 h = __floats2bfloat162_rn(r0, r1);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// out = combine(a, b) over n8 16-byte vectors when the module's skip flag equals `when_skip`.
template <bool SUB>
__global__ void __launch_bounds__(256) k_tdc_combine(const uint4* a, const uint4* b, uint4* out, int64_t n8,
                                                     const sb_module_state* st, int when_skip) {
  if ((st->skip != 0) != (when_skip != 0)) return;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  // two vectors per iteration: both loads are in flight before either result is needed
  for (; i + stride < n8; i += 2 * stride) {
    const uint4 a0 = ldg_nc_v4(a + i), b0 = ldg_nc_v4(b + i);
    const uint4 a1 = ldg_nc_v4(a + i + stride), b1 = ldg_nc_v4(b + i + stride);
    out[i] = combine8<SUB>(a0, b0);
    out[i + stride] = combine8<SUB>(a1, b1);
  }
  if (i < n8) out[i] = combine8<SUB>(ldg_nc_v4(a + i), ldg_nc_v4(b + i));
}

static unsigned combine_grid(int64_t n8) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  const int64_t want = ceil_div(n8, 256);
  const int64_t cap = (int64_t)sms * 8;  // 8 CTAs of 256 threads per SM
  return (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
}

cudaError_t launch_tdc_refresh(const void* x, const void* y, void* d, int64_t n, const sb_module_state* st,
                               cudaStream_t s) {
  const int64_t n8 = n / 8;
  k_tdc_combine<true><<<combine_grid(n8), 256, 0, s>>>(reinterpret_cast<const uint4*>(x),
                                                        reinterpret_cast<const uint4*>(y), reinterpret_cast<uint4*>(d),
                                                        n8, st, 0);
  return cudaGetLastError();
}

cudaError_t launch_tdc_reuse(const void* x, const void* d, void* y, int64_t n, const sb_module_state* st,
                             cudaStream_t s) {
  const int64_t n8 = n / 8;
  k_tdc_combine<false><<<combine_grid(n8), 256, 0, s>>>(reinterpret_cast<const uint4*>(x),
                                                         reinterpret_cast<const uint4*>(d), reinterpret_cast<uint4*>(y),
                                                         n8, st, 1);
  return cudaGetLastError();
}

}  // namespace sb
