// reuse.cu -- the Temporal Delta Cache's reuse path ("write-up" section 二: a skipped module
// reuses the cached result; explainer section 3: the old outcome is used and adjusted very
// slightly). At a computed step the module's residual is kept, D = bf16(y - x); at a skipped step
// the output is y = bf16(x + D). Both are streaming kernels gated on the device by the module's
// skip decision, so a whole step stays enqueued without host round trips.
//
// The residual may also be kept in FP8 ("write-up" section 七: history in low-precision
// formats): E4M3 codes with one FP32 scale per token, s = max|d| / 448, codes E4M3(RN(d * 448 /
// max|d|)) saturating, d = RN(y - x); a skipped step returns bf16(x + RN(E4M3(code) * s)).
#include <cfloat>

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

// ---- FP8 residual -------------------------------------------------------------------------

__device__ __forceinline__ void residual8(const uint4& xa, const uint4& ya, float (&d)[8]) {
  float fx[8], fy[8];
  unpack8(xa, fx);
  unpack8(ya, fy);
#pragma unroll
  for (int i = 0; i < 8; ++i) d[i] = __fsub_rn(fy[i], fx[i]);
}

// E4M3 codes of 8 residuals with the row's scale decision (a = max |d| of the row).
__device__ __forceinline__ uint2 residual_codes8(const float (&d)[8], float a, float inv, bool finite) {
  uint32_t q[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    if (a == 0.0f) {
      q[i] = q[i + 1] = 0u;
    } else if (!finite) {  // 448 / a overflowed: nonzero residuals take +-448, zeros 0
      q[i] = (d[i] == 0.0f) ? 0u : ((d[i] < 0.0f ? 0x80u : 0u) | 0x7eu);
      q[i + 1] = (d[i + 1] == 0.0f) ? 0u : ((d[i + 1] < 0.0f ? 0x80u : 0u) | 0x7eu);
    } else {
      uint16_t c16;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c16) : "f"(__fmul_rn(d[i + 1], inv)), "f"(__fmul_rn(d[i], inv)));
      q[i] = c16 & 0xffu;
      q[i + 1] = c16 >> 8;
    }
  }
  return make_uint2(q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24), q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24));
}

// The row's max over the CTA (blockDim.x a multiple of 32, at most 1024).
__device__ __forceinline__ float row_max_cta(float am, float* s_wmax) {
  am = warp_max_f32(am);
  if ((threadIdx.x & 31) == 0) s_wmax[threadIdx.x >> 5] = am;
  __syncthreads();
  float a = 0.0f;
  const int nw = (int)(blockDim.x >> 5);
  for (int w = 0; w < nw; ++w) a = fmaxf(a, s_wmax[w]);
  return a;
}

// One CTA per token row, each thread GPT groups of 8 channels held in registers: one read of x
// and y. Rows wider than GPT * 8 * 1024 channels take k_tdc_refresh8_2pass. (One warp per row,
// with the row's max by shuffles only, measured slower: 12 groups per lane held too many
// registers for enough warps per SM.)
template <int GPT>
__global__ void __launch_bounds__(1024) k_tdc_refresh8(const uint4* x, const uint4* y, uint2* codes, float* scale, int C,
                                                       const sb_module_state* st) {
  if (st->skip != 0) return;
  __shared__ float s_wmax[32];
  const int64_t m = blockIdx.x;
  const int G = C / 8;
  const uint4* xr = x + m * G;
  const uint4* yr = y + m * G;
  float d[GPT][8];
  float am = 0.0f;
#pragma unroll
  for (int k = 0; k < GPT; ++k) {
    const int g = threadIdx.x + k * (int)blockDim.x;
    if (g < G) {
      residual8(ldg_nc_v4(xr + g), ldg_nc_v4(yr + g), d[k]);
#pragma unroll
      for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(d[k][i]));
    }
  }
  const float a = row_max_cta(am, s_wmax);
  const float s = (a == 0.0f) ? 0.0f : __fdiv_rn(a, 448.0f);
  const float inv = (a == 0.0f) ? 0.0f : __fdiv_rn(448.0f, a);
  if (threadIdx.x == 0) scale[m] = s;
#pragma unroll
  for (int k = 0; k < GPT; ++k) {
    const int g = threadIdx.x + k * (int)blockDim.x;
    if (g < G) codes[m * G + g] = residual_codes8(d[k], a, inv, inv <= FLT_MAX);
  }
}

// Any row width: the row's max first, then a second read of x and y (from L1 or L2) for the codes.
__global__ void __launch_bounds__(256) k_tdc_refresh8_2pass(const uint4* x, const uint4* y, uint2* codes, float* scale,
                                                            int C, const sb_module_state* st) {
  if (st->skip != 0) return;
  __shared__ float s_wmax[32];
  const int64_t m = blockIdx.x;
  const int G = C / 8;
  const uint4* xr = x + m * G;
  const uint4* yr = y + m * G;
  float am = 0.0f;
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    float d[8];
    residual8(ldg_nc_v4(xr + g), ldg_nc_v4(yr + g), d);
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(d[i]));
  }
  const float a = row_max_cta(am, s_wmax);
  const float s = (a == 0.0f) ? 0.0f : __fdiv_rn(a, 448.0f);
  const float inv = (a == 0.0f) ? 0.0f : __fdiv_rn(448.0f, a);
  if (threadIdx.x == 0) scale[m] = s;
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    float d[8];
    residual8(xr[g], yr[g], d);
    codes[m * G + g] = residual_codes8(d, a, inv, inv <= FLT_MAX);
  }
}

// y = bf16(x + RN(E4M3(code) * s_row)), 16 elements per thread and step (C % 16 == 0).
__global__ void __launch_bounds__(256) k_tdc_reuse8(const uint4* x, const uint4* codes, const float* scale, uint4* y,
                                                    int64_t n16, int C16, const sb_module_state* st) {
  if (st->skip == 0) return;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) {
    const float s = __ldg(scale + i / C16);
    const uint4 q = ldg_nc_v4(codes + i);
    const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float fx[8];
      unpack8(ldg_nc_v4(x + 2 * i + h), fx);
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t word = qw[2 * h + (k >> 1)];
        const uint32_t c0 = (word >> (16 * (k & 1))) & 0xffu, c1 = (word >> (16 * (k & 1) + 8)) & 0xffu;
        const float r0 = __fadd_rn(fx[2 * k], __fmul_rn(e4m3_to_f32(c0), s));
        const float r1 = __fadd_rn(fx[2 * k + 1], __fmul_rn(e4m3_to_f32(c1), s));
        const __nv_bfloat162 b = __floats2bfloat162_rn(r0, r1);
        w[k] = *reinterpret_cast<const uint32_t*>(&b);
      }
      y[2 * i + h] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

cudaError_t launch_tdc_refresh8(const void* x, const void* y, uint8_t* codes, float* scale, int64_t M, int64_t C,
                                const sb_module_state* st, cudaStream_t s) {
  const uint4* xv = reinterpret_cast<const uint4*>(x);
  const uint4* yv = reinterpret_cast<const uint4*>(y);
  uint2* cv = reinterpret_cast<uint2*>(codes);
  constexpr int GPT = 4;
  const int64_t threads = ((ceil_div(C / 8, GPT) + 31) / 32) * 32;
  if (threads <= 1024)
    k_tdc_refresh8<GPT><<<(unsigned)M, (unsigned)threads, 0, s>>>(xv, yv, cv, scale, (int)C, st);
  else
    k_tdc_refresh8_2pass<<<(unsigned)M, 256, 0, s>>>(xv, yv, cv, scale, (int)C, st);
  return cudaGetLastError();
}

cudaError_t launch_tdc_reuse8(const void* x, const uint8_t* codes, const float* scale, void* y, int64_t M, int64_t C,
                              const sb_module_state* st, cudaStream_t s) {
  const int64_t n16 = M * C / 16;
  k_tdc_reuse8<<<combine_grid(n16), 256, 0, s>>>(reinterpret_cast<const uint4*>(x), reinterpret_cast<const uint4*>(codes),
                                                  scale, reinterpret_cast<uint4*>(y), n16, (int)(C / 16), st);
  return cudaGetLastError();
}

}  // namespace sb
