// delta.cu -- delta tokens ("DeltaQuant: 4-bit Video Diffusion Models with Spatiotemporal Delta
// Smoothing", abstract): the tokens of the latent video grid are grouped into local 3D
// spatiotemporal cubes; each cube's mean token is its core token, kept in FP8 (E4M3 codes with one
// FP32 scale per core token); the differences of the cube's tokens from their core (delta tokens,
// bf16) go through the 4-bit path of this library like any activation. The linear layer is then
// the delta tokens' GEMM plus, once per cube, the core token's product with the weight, added to
// every token of the cube.
//
//  k_delta_split    one CTA per cube, 8 channels per thread and step: per channel the pairwise
//                   FP32 sum over the cube's tokens (token order, zero-padded to a power of two),
//                   the mean, the core's amax and scale, its E4M3 codes, its dequantized value
//                   (kept as bf16 for the core GEMM), and the cube's delta tokens bf16(x - core).
//                   Instantiated for cubes of up to 8 tokens and of up to 32.
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

// Sum of the leaves v[0 .. n2) by the canonical pairwise tree (n2 a power of two <= NMAX; the
// leaves in [n, n2) are +0). The levels are formed for all NMAX leaves and the level of n2 is
// returned, so every index is a compile-time constant and the leaves stay in registers.
template <int NMAX>
__device__ __forceinline__ float tree_sum(float (&v)[NMAX], int n2) {
  float r = v[0];
#pragma unroll
  for (int len = 2; len <= NMAX; len <<= 1) {
#pragma unroll
    for (int i = 0; i < NMAX / len; ++i) v[i] = __fadd_rn(v[2 * i], v[2 * i + 1]);
    if (n2 == len) r = v[0];
  }
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float (&f)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

// One CTA per cube; each thread takes groups of 8 channels (16-byte loads of every token of the
// cube). Pass 1: the channel means (into shared memory) and the core's amax; pass 2: codes, the
// bf16 core, and the delta tokens from a second read of the cube's rows (L1-resident by then).
template <int NMAX>
__global__ void __launch_bounds__(kDqThreads) k_delta_split(const __nv_bfloat16* X, int K, CubeGeom g,
                                                           uint8_t* codes, float* scale, __nv_bfloat16* core16,
                                                           __nv_bfloat16* delta) {
  extern __shared__ float s_mean[];  // K means of this cube
  __shared__ float s_wmax[kDqThreads / 32];
  __shared__ int64_t s_tok[kDqMaxCube];  // the cube's tokens, index order
  __shared__ int s_n;
  const int64_t k = blockIdx.x;
  if (threadIdx.x == 0) s_n = cube_tokens(g, k, s_tok);
  __syncthreads();
  const int n = s_n;
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  const float fn = (float)n;
  const int G = K / 8;  // 8-channel groups per token
  const uint4* rows[NMAX];
#pragma unroll
  for (int j = 0; j < NMAX; ++j) rows[j] = reinterpret_cast<const uint4*>(X + (j < n ? s_tok[j] : s_tok[0]) * K);
  // ---- pass 1: means and amax
  float am = 0.0f;
  for (int gi = threadIdx.x; gi < G; gi += kDqThreads) {
    uint4 raw[NMAX];
#pragma unroll
    for (int j = 0; j < NMAX; ++j) raw[j] = (j < n) ? __ldg(rows[j] + gi) : make_uint4(0u, 0u, 0u, 0u);
    float m[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float v[NMAX];
#pragma unroll
      for (int j = 0; j < NMAX; ++j) {
        float f[8];
        bf16x8_to_f32(raw[j], f);
        v[j] = f[c];
      }
      m[c] = __fdiv_rn(tree_sum<NMAX>(v, n2), fn);
      am = fmaxf(am, fabsf(m[c]));
    }
    float4* sm = reinterpret_cast<float4*>(s_mean + 8 * gi);
    sm[0] = make_float4(m[0], m[1], m[2], m[3]);
    sm[1] = make_float4(m[4], m[5], m[6], m[7]);
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
  for (int gi = threadIdx.x; gi < G; gi += kDqThreads) {
    const float4* sm = reinterpret_cast<const float4*>(s_mean + 8 * gi);
    const float4 m0 = sm[0], m1 = sm[1];
    const float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    uint32_t q[8];
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
      if (a == 0.0f) {
        q[c] = q[c + 1] = 0u;
      } else if (!finite) {  // 448 / a overflowed: nonzero means take +-448, zeros 0
        q[c] = (m[c] == 0.0f) ? 0u : ((m[c] < 0.0f ? 0x80u : 0u) | 0x7eu);
        q[c + 1] = (m[c + 1] == 0.0f) ? 0u : ((m[c + 1] < 0.0f ? 0x80u : 0u) | 0x7eu);
      } else {
        uint16_t c16;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
            : "=h"(c16)
            : "f"(__fmul_rn(m[c + 1], inv)), "f"(__fmul_rn(m[c], inv)));
        q[c] = c16 & 0xffu;
        q[c + 1] = c16 >> 8;
      }
    }
    reinterpret_cast<uint2*>(codes + k * K)[gi] =
        make_uint2(q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24), q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24));
    float d[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) d[c] = __fmul_rn(e4m3_to_f32(q[c]), s);
    uint32_t cw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(d[2 * i], d[2 * i + 1]);
      cw[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(core16 + k * K)[gi] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
#pragma unroll
    for (int j = 0; j < NMAX; ++j) {
      if (j < n) {
        float x[8];
        bf16x8_to_f32(__ldg(rows[j] + gi), x);
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(__fsub_rn(x[2 * i], d[2 * i]), __fsub_rn(x[2 * i + 1], d[2 * i + 1]));
          o[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        reinterpret_cast<uint4*>(delta + s_tok[j] * K)[gi] = make_uint4(o[0], o[1], o[2], o[3]);
      }
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
  const bool small = (int64_t)c.ct * c.ch * c.cw <= 8;
  static std::atomic<uint64_t> attr8{0}, attr32{0};
  if (dsm > 48 * 1024) {
    const cudaError_t e = small ? smem_attr_once(k_delta_split<8>, 64 * 1024, attr8)
                                : smem_attr_once(k_delta_split<kDqMaxCube>, 64 * 1024, attr32);
    if (e != cudaSuccess) return e;
  }
  const CubeGeom g = geom_from(c);
  const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(X);
  __nv_bfloat16* c16 = reinterpret_cast<__nv_bfloat16*>(core16);
  __nv_bfloat16* d16 = reinterpret_cast<__nv_bfloat16*>(delta);
  if (small)
    k_delta_split<8><<<(unsigned)ncube, kDqThreads, dsm, s>>>(x, (int)K, g, codes, scale, c16, d16);
  else
    k_delta_split<kDqMaxCube><<<(unsigned)ncube, kDqThreads, dsm, s>>>(x, (int)K, g, codes, scale, c16, d16);
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
