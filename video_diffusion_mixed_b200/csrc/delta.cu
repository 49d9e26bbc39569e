// delta.cu -- delta tokens ("DeltaQuant: 4-bit Video Diffusion Models with Spatiotemporal Delta
// Smoothing", abstract): the tokens of the latent video grid are grouped into local 3D
// spatiotemporal cubes; each cube's mean token is its core token, kept in FP8 (E4M3 codes with one
// FP32 scale per core token); the differences of the cube's tokens from their core (delta tokens,
// bf16) go through the 4-bit path of this library like any activation. The linear layer is then
// the delta tokens' GEMM plus, once per cube, the core token's product with the weight, added to
// every token of the cube.
//
//  k_delta_split    one CTA per cube: per channel the pairwise FP32 sum over the cube's tokens
//                   (token order, zero-padded to a power of two), the mean, the core's amax and
//                   scale, its E4M3 codes, its dequantized value (kept as bf16 for the core GEMM),
//                   and the cube's delta tokens bf16(x - core).
//  k_delta_combine  Y[t] = act(Yd[t] + Yc[cube(t)]) in FP32, stored as bf16.
#include <cfloat>

#include "launch_util.h"
#include "sb_device.cuh"
#include "sb_kernels.h"

namespace sb {

constexpr int kDqThreads = 256;
constexpr int kDqMaxCube = kDeltaMaxCube;  // tokens per cube

struct CubeGeom {
  int64_t T, F, H, W;
  int ct, ch, cw;
  int64_t nh, nw;  // cubes along h and w
};

__host__ __device__ inline int64_t cube_of(const CubeGeom& g, int64_t t) {
  if (t < g.T) return t;
  const int64_t p = t - g.T;
  const int64_t f = p / (g.H * g.W), h = (p / g.W) % g.H, w = p % g.W;
  return g.T + ((f / g.ct) * g.nh + h / g.ch) * g.nw + w / g.cw;
}

// The tokens of cube k in index order; returns their count.
__device__ __forceinline__ int cube_tokens(const CubeGeom& g, int64_t k, int64_t (&tok)[kDqMaxCube]) {
  if (k < g.T) {
    tok[0] = k;
    return 1;
  }
  const int64_t q = k - g.T;
  const int64_t a = q / (g.nh * g.nw), b = (q / g.nw) % g.nh, c = q % g.nw;
  int n = 0;
  for (int64_t f = a * g.ct; f < g.F && f < (a + 1) * g.ct; ++f)
    for (int64_t h = b * g.ch; h < g.H && h < (b + 1) * g.ch; ++h)
      for (int64_t w = c * g.cw; w < g.W && w < (c + 1) * g.cw; ++w) tok[n++] = g.T + (f * g.H + h) * g.W + w;
  return n;
}

// Pairwise FP32 tree over v[0 .. N) (N a power of two), in place.
template <int N>
__device__ __forceinline__ float2 tree_pair2(float2 (&v)[kDqMaxCube]) {
#pragma unroll
  for (int len = N; len > 1; len >>= 1) {
#pragma unroll
    for (int i = 0; i < len / 2; ++i) v[i] = make_float2(__fadd_rn(v[2 * i].x, v[2 * i + 1].x), __fadd_rn(v[2 * i].y, v[2 * i + 1].y));
  }
  return v[0];
}

__global__ void __launch_bounds__(kDqThreads) k_delta_split(const __nv_bfloat16* X, int K, CubeGeom g,
                                                           uint8_t* codes, float* scale, __nv_bfloat16* core16,
                                                           __nv_bfloat16* delta) {
  extern __shared__ float s_mean[];  // K means of this cube
  __shared__ float s_wmax[kDqThreads / 32];
  __shared__ int64_t tok[kDqMaxCube];  // the cube's tokens, index order
  __shared__ int s_n;
  const int64_t k = blockIdx.x;
  if (threadIdx.x == 0) {
    int64_t t[kDqMaxCube];
    const int nn = cube_tokens(g, k, t);
    for (int j = 0; j < nn; ++j) tok[j] = t[j];
    s_n = nn;
  }
  __syncthreads();
  const int n = s_n;
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  const float fn = (float)n;
  // ---- pass 1: means of channel pairs (one 32-bit word of bf16 per token)
  float am = 0.0f;
  for (int c2 = threadIdx.x; c2 < K / 2; c2 += kDqThreads) {
    float2 v[kDqMaxCube];
#pragma unroll
    for (int j = 0; j < kDqMaxCube; ++j) {
      if (j < n) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(X + tok[j] * K) + c2);
        v[j] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
      } else {
        v[j] = make_float2(0.0f, 0.0f);
      }
    }
    float2 s;
    switch (n2) {  // the canonical tree over exactly n2 leaves (padding with +0 beyond n)
      case 1: s = v[0]; break;
      case 2: s = tree_pair2<2>(v); break;
      case 4: s = tree_pair2<4>(v); break;
      case 8: s = tree_pair2<8>(v); break;
      case 16: s = tree_pair2<16>(v); break;
      default: s = tree_pair2<32>(v); break;
    }
    const float m0 = __fdiv_rn(s.x, fn), m1 = __fdiv_rn(s.y, fn);
    s_mean[2 * c2] = m0;
    s_mean[2 * c2 + 1] = m1;
    am = fmaxf(am, fmaxf(fabsf(m0), fabsf(m1)));
  }
  am = warp_max_f32(am);
  if ((threadIdx.x & 31) == 0) s_wmax[threadIdx.x >> 5] = am;
  __syncthreads();
  float a = 0.0f;
#pragma unroll
  for (int w = 0; w < kDqThreads / 32; ++w) a = fmaxf(a, s_wmax[w]);
  // ---- the core's scale and codes, its dequantized value, the delta tokens
  const float s = (a == 0.0f) ? 0.0f : __fdiv_rn(a, 448.0f);
  const float inv = (a == 0.0f) ? 0.0f : __fdiv_rn(448.0f, a);
  const bool finite = inv <= FLT_MAX;
  if (threadIdx.x == 0) scale[k] = s;
  for (int c2 = threadIdx.x; c2 < K / 2; c2 += kDqThreads) {
    const float m0 = s_mean[2 * c2], m1 = s_mean[2 * c2 + 1];
    uint32_t q0, q1;
    if (a == 0.0f) {
      q0 = q1 = 0u;
    } else if (!finite) {  // 448 / a overflowed: nonzero means take +-448, zeros 0
      q0 = (m0 == 0.0f) ? 0u : ((m0 < 0.0f ? 0x80u : 0u) | 0x7eu);
      q1 = (m1 == 0.0f) ? 0u : ((m1 < 0.0f ? 0x80u : 0u) | 0x7eu);
    } else {
      uint16_t c16;
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c16) : "f"(__fmul_rn(m1, inv)), "f"(__fmul_rn(m0, inv)));
      q0 = c16 & 0xffu;
      q1 = c16 >> 8;
    }
    reinterpret_cast<uint16_t*>(codes + k * K)[c2] = (uint16_t)(q0 | (q1 << 8));
    const float d0 = __fmul_rn(e4m3_to_f32(q0), s), d1 = __fmul_rn(e4m3_to_f32(q1), s);
    reinterpret_cast<__nv_bfloat162*>(core16 + k * K)[c2] = __floats2bfloat162_rn(d0, d1);
    for (int j = 0; j < n; ++j) {
      const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(X + tok[j] * K) + c2);
      const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xffff0000u);
      reinterpret_cast<__nv_bfloat162*>(delta + tok[j] * K)[c2] =
          __floats2bfloat162_rn(__fsub_rn(x0, d0), __fsub_rn(x1, d1));
    }
  }
}

__device__ __forceinline__ float gelu_tanh_f(float v) {
  float t;
  const float u = __fmul_rn(0.7978845608028654f, __fmaf_rn(0.044715f, __fmul_rn(__fmul_rn(v, v), v), v));
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(u));
  const float h = __fmul_rn(0.5f, v);
  return __fmaf_rn(h, t, h);
}

// Y[t][n] = act(Yd[t][n] + Yc[cube(t)][n]) as bf16; 8 columns per thread (N % 8 == 0).
__global__ void __launch_bounds__(256) k_delta_combine(const float* Yd, const float* Yc, int64_t M, int N, CubeGeom g,
                                                      int gelu, __nv_bfloat16* Y) {
  const int n8 = N / 8;
  const int64_t total = M * n8;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / n8;
    const int c = (int)(i - t * n8) * 8;
    const int64_t cube = cube_of(g, t);
    const float4* pd = reinterpret_cast<const float4*>(Yd + t * N + c);
    const float4* pc = reinterpret_cast<const float4*>(Yc + cube * N + c);
    float v[8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float4 a = __ldcs(pd + h), b = __ldg(pc + h);
      v[4 * h] = __fadd_rn(a.x, b.x);
      v[4 * h + 1] = __fadd_rn(a.y, b.y);
      v[4 * h + 2] = __fadd_rn(a.z, b.z);
      v[4 * h + 3] = __fadd_rn(a.w, b.w);
    }
    if (gelu) {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = gelu_tanh_f(v[j]);
    }
    uint4 o;
    __nv_bfloat162 p0 = __floats2bfloat162_rn(v[0], v[1]), p1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 p2 = __floats2bfloat162_rn(v[4], v[5]), p3 = __floats2bfloat162_rn(v[6], v[7]);
    o.x = *reinterpret_cast<uint32_t*>(&p0);
    o.y = *reinterpret_cast<uint32_t*>(&p1);
    o.z = *reinterpret_cast<uint32_t*>(&p2);
    o.w = *reinterpret_cast<uint32_t*>(&p3);
    *reinterpret_cast<uint4*>(Y + t * N + c) = o;
  }
}

static CubeGeom geom_from(const DeltaCubes& c) {
  CubeGeom g;
  g.T = c.T;
  g.F = c.F;
  g.H = c.H;
  g.W = c.W;
  g.ct = c.ct;
  g.ch = c.ch;
  g.cw = c.cw;
  g.nh = ceil_div(c.H, c.ch);
  g.nw = ceil_div(c.W, c.cw);
  return g;
}

cudaError_t launch_delta_split(const void* X, int64_t K, const DeltaCubes& c, int64_t ncube, uint8_t* codes,
                               float* scale, void* core16, void* delta, cudaStream_t s) {
  const int dsm = (int)(K * sizeof(float));
  static std::atomic<uint64_t> attr{0};
  if (dsm > 48 * 1024) {
    const cudaError_t e = smem_attr_once(k_delta_split, 64 * 1024, attr);
    if (e != cudaSuccess) return e;
  }
  k_delta_split<<<(unsigned)ncube, kDqThreads, dsm, s>>>(reinterpret_cast<const __nv_bfloat16*>(X), (int)K,
                                                         geom_from(c), codes, scale,
                                                         reinterpret_cast<__nv_bfloat16*>(core16),
                                                         reinterpret_cast<__nv_bfloat16*>(delta));
  return cudaGetLastError();
}

cudaError_t launch_delta_combine(const float* Yd, const float* Yc, int64_t M, int64_t N, const DeltaCubes& c,
                                 int gelu, void* Y, cudaStream_t s) {
  const int64_t total = M * (N / 8);
  const int64_t want = ceil_div(total, 256);
  const int64_t cap = (int64_t)device_sm_count() * 8;
  k_delta_combine<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(Yd, Yc, M, (int)N, geom_from(c), gelu,
                                                                     reinterpret_cast<__nv_bfloat16*>(Y));
  return cudaGetLastError();
}

}  // namespace sb
