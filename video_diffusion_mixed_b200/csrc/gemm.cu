// gemm.cu -- quantized linear layer on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent, warp-specialised kernel serves the three precisions of a layer; the precision
// is read from the device flag written by the decision/pre-pass kernels, so no host round trip
// is needed ("write-up" section 一: NVFP4 or INT8 per layer and step; section 三: full precision
// under PDR; section 四: 4-bit weights).
//
//   NVFP4  tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16  K-block 256 elements
//   INT8   tcgen05.mma.cta_group::2.kind::i8 (s32 accumulators)          K-block 128 elements
//   BF16   tcgen05.mma.cta_group::2.kind::f16 (fp32 accumulators)        K-block  64 elements
//
// The kernel runs as clusters of two CTAs on the two SMs of a pair. A cluster owns a 256 x BN
// output tile (BN = 256, or 128 when N is not a multiple of 256): each CTA loads its own 128 rows
// of A and one half of B -- and, for NVFP4, the E4M3 scales of its rows and of all BN columns --
// with TMA (no multicast) into its own shared memory; the even CTA (the leader) issues MMAs with
// M = 256 that read both CTAs' operands, and each CTA's tensor memory receives its 128 rows. Per
// SM this halves the B traffic through shared memory, whose port is shared by the TMA writes and
// the MMA reads and otherwise limits the MMA rate.
//
// Every K-block is one 128-byte-wide row slab (128B swizzle), consumed by four MMAs of 32 bytes
// of K. Warp roles (384 threads = 3 warpgroups per CTA):
//   warp 0      TMA producer (one lane), in both CTAs
//   warp 1      TMEM allocation (both CTAs); scale copies to TMEM and MMA issue (leader only)
//   warps 2-3   idle
//   warps 4-11  epilogue: TMEM -> registers, release the accumulator, then dequant scale, bias,
//               optional GELU, store
// The first warpgroup gives registers up (setmaxnreg) so that each epilogue thread can hold 128
// accumulator values: 72 x 128 + 216 x 256 registers, exactly the 168 x 384 of the launch.
// Accumulators: two buffers of BN columns when they fit next to the NVFP4 scale columns (the
// epilogue of tile i then overlaps the mainloop of tile i + 1), else one; either way the
// epilogue drains its columns into registers and releases the buffer before computing, so the
// next tile's MMAs start after the drain. Every wait is bounded; a wait that gives up records
// SB_ETIMEOUT.
#include <cudaTypedefs.h>

#include <mutex>

#include "launch_util.h"
#include "sb_device.cuh"
#include "sb_kernels.h"
#include "tmap.h"

namespace sb {

// Per-stage shared memory of one CTA: A 128 rows x 128 B | B half (BN/2 rows) x 128 B | NVFP4
// only: SFA 4 atoms x 512 B | SFB 2 column tiles x 4 atoms x 512 B. Stage sizes are multiples
// of 1024 B (the 128B-swizzle atom).
constexpr int kOffB = 16384;
constexpr int kOffSFA = 32768;
constexpr int kOffSFB = 34816;
constexpr int kStageBytesQ = 32768;  // INT8 / BF16
constexpr int kStagesQ = 6;
constexpr int kStageBytesF = 38912;  // NVFP4
constexpr int kStagesF = 5;
constexpr int kMaxStages = 6;
constexpr int kStageArea = kStagesQ * kStageBytesQ;
constexpr int kThreads = 384;
constexpr int kEpiWarp0 = 4;  // first epilogue warp
constexpr int kEpiWarps = 8;
constexpr uint32_t kRegsCtl = 72;   // producer / MMA warpgroup
constexpr uint32_t kRegsEpi = 216;  // epilogue warpgroups
constexpr int kRegsNeeded = (int)(kRegsCtl * 128 + kRegsEpi * 256);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCols = 48;             // NVFP4: 16 SFA + 32 SFB columns per K-block
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s: far above any legitimate wait (the default limit)
constexpr uint64_t kDrainNs = 20000000ull;   // 20 ms to let in-flight copies land after an abort
// After the stages: 1 KB of barriers, then the epilogue's output staging (bf16 output): two
// 32 x 32 bf16 boxes (2 KB each, 64B swizzle) per epilogue warp.
constexpr int kBarBytes = 1024;
constexpr int kOutOff = kStageArea + kBarBytes;
constexpr int kOutBox = 2048;
constexpr int kOutBytes = 8 * 2 * kOutBox;
constexpr int kStoreLane = 31;  // epilogue lane that issues a warp's TMA stores
constexpr int kSmemBytes = kOutOff + kOutBytes + 1024;  // + alignment of the dynamic base to 1 KB
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(kStagesF * kStageBytesF <= kStageArea, "NVFP4 stages exceed the stage area");
// NVFP4 leaves the end of the stage area free: each epilogue warp's 128-column bias slice (bf16).
constexpr int kBiasOffF = kStagesF * kStageBytesF;
static_assert(kBiasOffF + 8 * 256 <= kStageArea, "NVFP4 bias slices");
static_assert(kOffSFB + 2 * 2048 <= kStageBytesF, "NVFP4 stage layout");

enum { KIND_FP4 = 0, KIND_I8 = 1, KIND_BF16 = 2 };

struct TMaps {
  CUtensorMap a[3];
  CUtensorMap b[3];
  CUtensorMap sfa;  // NVFP4 scales of A, 3-D: 128 words x K/64 atoms x 128-row tiles
  CUtensorMap sfb;  // NVFP4 scales of B, same shape over the N rows of the weight
  CUtensorMap y;    // bf16 output, box 32 columns x 32 rows, 64B swizzle
  CUtensorMap yc;   // k_gemm<kEpiModRec>: the module's cached output, same boxes (c := y is stored there)
};

struct GemmParams {
  int M, N, K;
  int bn[3];  // tile width per precision: 256, 192 (NVFP4) or 128
  float invB;
  const int32_t* prec;
  int have[3];
  const float* sA8;
  const float* sB8;
  const float* gA4;
  const float* gB4;
  const __nv_bfloat16* bias;
  void* Y;
  int out_dtype;
  int epilogue;
  int tma_store;  // bf16 output through shared memory and TMA stores
  int group_m;    // M-tiles per raster group (tile_coords)
  uint64_t wait_ns;  // limit of the pipeline waits (kWaitNs unless a stall drill is armed)
  int64_t withhold;  // stall drill: the leader's producer skips the loads of this stage (-1: none)
  // Row addend (delta tokens, k_gemm<kEpiRowAdd> only): output row t adds the FP32 row ra_row(t)
  // of rowadd ([cubes][N]) before the activation; rows map to the cubes of a T + F x H x W grid.
  const float* rowadd;
  int64_t ra_T, ra_H, ra_W, ra_nh, ra_nw;
  int ra_ct, ra_ch, ra_cw;
  // Chunk records (k_gemm<kEpiRecord> only): per row and aligned 128-column chunk of the bf16
  // output, {max |H_128 y|, canonical pairwise sum |y|, max |y|, 0}, float4 [M][N / 128].
  float4* records;
  int rec_nc;  // chunks per row
  // Module record (k_gemm<kEpiModRec> only; the output y is the module's output): per row and
  // aligned 128-column chunk, from the bf16 values y holds, the module input x (mr_x) and the cached
  // output c (mr_c, read as zero while the module has no cached output), the partial sums
  // {sum |y|, sum (y - x)^2, sum x^2, sum |y - c|} and {sum |c|, max |y|, 0, 0} (two float4 per
  // chunk, mr_rec [M][N / 128][2]); each sum is the balanced tree over the chunk's columns. When
  // the module's TDC record runs and mr_update is set, the staged output is stored to the cache too.
  const __nv_bfloat16* mr_x;
  const __nv_bfloat16* mr_c;
  float4* mr_rec;
  const sb_module_state* mr_st;
  int mr_update;
  WsHeader* hdr;
};

// Epilogue forms, one k_gemm instantiation each (the plain one is what every ordinary launch runs).
enum { kEpiPlain = 0, kEpiRowAdd = 1, kEpiRecord = 2, kEpiModRec = 3 };


// The cube of token t (text tokens first, one cube each; then the grid in (f, h, w) order).
__device__ __forceinline__ int64_t ra_row(const GemmParams& p, int64_t t) {
  if (t < p.ra_T) return t;
  const int64_t q = t - p.ra_T;
  const int64_t f = q / (p.ra_H * p.ra_W), h = (q / p.ra_W) % p.ra_H, w = q % p.ra_W;
  return p.ra_T + ((f / p.ra_ct) * p.ra_nh + h / p.ra_ch) * p.ra_nw + w / p.ra_cw;
}

__device__ __forceinline__ uint32_t idesc_for(int kind, int BM, int BN) {
  const uint32_t n = (uint32_t)(BN >> 3) << 17;
  const uint32_t m = (uint32_t)(BM >> 4) << 24;
  switch (kind) {
    case KIND_FP4:  // block-scaled: A,B = E2M1 (1), scale type UE4M3 (bit 23 = 0), K = 64
      return (1u << 7) | (1u << 10) | n | m;
    case KIND_I8:  // D = S32 (2), A,B signed 8-bit (1)
      return (2u << 4) | (1u << 7) | (1u << 10) | n | m;
    default:  // D = F32 (1), A,B = BF16 (1)
      return (1u << 4) | (1u << 7) | (1u << 10) | n | m;
  }
}

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// FP32x2 arithmetic for the epilogue (one instruction, two lanes of FP32 work; the epilogue's
// outputs are compared with a tolerance, so contraction is allowed here).
__device__ __forceinline__ uint64_t ep_bits(float2 a) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a.x), "f"(a.y));
  return r;
}
__device__ __forceinline__ float2 ep_f2(uint64_t r) {
  float2 a;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a.x), "=f"(a.y) : "l"(r));
  return a;
}
__device__ __forceinline__ float2 ep_mul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ep_bits(a)), "l"(ep_bits(b)));
  return ep_f2(r);
}
__device__ __forceinline__ float2 ep_fma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(ep_bits(a)), "l"(ep_bits(b)), "l"(ep_bits(c)));
  return ep_f2(r);
}
__device__ __forceinline__ float2 ep_add2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(ep_bits(a)), "l"(ep_bits(b)));
  return ep_f2(r);
}

// tanh-form GELU, 0.5 v (1 + tanh(sqrt(2/pi) (v + 0.044715 v^3))), with the SFU's tanh
// approximation (relative error about 2^-11, below the 2^-9 rounding of the bf16 output), on two
// values at a time.
__device__ __forceinline__ float2 gelu_tanh2(float2 v) {
  const float2 c1 = make_float2(0.7978845608028654f * 0.044715f, 0.7978845608028654f * 0.044715f);
  const float2 c0 = make_float2(0.7978845608028654f, 0.7978845608028654f);
  const float2 u = ep_mul2(v, ep_fma2(c1, ep_mul2(v, v), c0));
  const float2 h = ep_mul2(make_float2(0.5f, 0.5f), v);
  return ep_fma2(h, make_float2(tanh_approx(u.x), tanh_approx(u.y)), h);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Grouped tile order: group_m consecutive M-tiles are swept across all N-tiles before the next
// group starts (M-tile fastest inside a group), so the A rows of a group stay in L2 while every
// N-tile reuses them (A of the second FFN layer is larger than L2 and would otherwise be re-read
// from HBM for each N-tile). The host picks group_m (pick_group_m).
__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles, int group_m, int* mt, int* nt) {
  const int group = group_m * n_tiles;
  const int g = t / group, r = t - g * group;
  const int first = g * group_m;
  const int gm = min(group_m, m_tiles - first);
  *mt = first + r % gm;
  *nt = r / gm;
}

// Per-column epilogue operands of a 32-column chunk: bias (bf16) and, for INT8, the weight's
// per-output-channel scale. They are loaded a chunk ahead of their use (the shared-memory stages
// leave little L1, so they come from L2).
template <int KIND>
struct ColOps {
  uint4 b[4];
  float4 s[KIND == KIND_I8 ? 8 : 1];
};

template <int KIND>
__device__ __forceinline__ void load_colops(const GemmParams& p, int n, ColOps<KIND>& o) {
  if (p.bias) {
    const uint4* bp = reinterpret_cast<const uint4*>(p.bias + n);
#pragma unroll
    for (int i = 0; i < 4; ++i) o.b[i] = __ldg(bp + i);
  }
  if constexpr (KIND == KIND_I8) {
    const float4* sp = reinterpret_cast<const float4*>(p.sB8 + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) o.s[i] = __ldg(sp + i);
  }
}

// Epilogue arithmetic of 32 accumulator columns of one row, in place: the accumulator words become
// the FP32 outputs. Dequant scale and bias are one FMA, then the optional GELU; columns go in
// pairs through FP32x2 arithmetic.
template <int KIND, bool ROWADD = false>
__device__ __forceinline__ void epilogue_math(const GemmParams& p, const ColOps<KIND>& o, float sxb, float alpha,
                                              uint32_t (&r)[32], const float* rowp = nullptr) {
  const bool has_bias = p.bias != nullptr, gelu = p.epilogue == SB_EPI_GELU_TANH;
  float4 ra[ROWADD ? 8 : 1];  // the row addend's 32 columns (zero for rows past M)
  if constexpr (ROWADD) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      ra[i] = rowp ? __ldg(reinterpret_cast<const float4*>(rowp) + i) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {  // columns 2j, 2j + 1
    const uint4 bq = o.b[j >> 2];
    const uint32_t w = (j & 3) == 0 ? bq.x : (j & 3) == 1 ? bq.y : (j & 3) == 2 ? bq.z : bq.w;
    const float2 bias = has_bias ? make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u))
                                 : make_float2(0.0f, 0.0f);
    float2 y;
    if constexpr (KIND == KIND_I8) {
      const float4 sc = o.s[j >> 1];
      const float2 c = (j & 1) ? make_float2(sc.z, sc.w) : make_float2(sc.x, sc.y);
      const float2 acc = make_float2(__int2float_rn((int)r[2 * j]), __int2float_rn((int)r[2 * j + 1]));
      y = ep_fma2(acc, ep_mul2(make_float2(sxb, sxb), c), bias);
    } else if constexpr (KIND == KIND_FP4) {
      y = ep_fma2(make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1])), make_float2(alpha, alpha),
                  bias);
    } else {
      y = make_float2(__uint_as_float(r[2 * j]) + bias.x, __uint_as_float(r[2 * j + 1]) + bias.y);
    }
    if constexpr (ROWADD) {
      const float4 q = ra[j >> 1];
      y = make_float2(y.x + ((j & 1) ? q.z : q.x), y.y + ((j & 1) ? q.w : q.y));
    }
    if (gelu) y = gelu_tanh2(y);
    r[2 * j] = __float_as_uint(y.x);
    r[2 * j + 1] = __float_as_uint(y.y);
  }
}

// Direct global stores of one row's 32 columns (FP32 / raw outputs, or bf16 without TMA).
template <int KIND, bool ROWADD = false>
__device__ __forceinline__ void store_direct(const GemmParams& p, int m, int n, float sxb, float alpha,
                                             uint32_t (&r)[32], const float* rowp = nullptr) {
  if (p.out_dtype == SB_OUT_RAW) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint32_t*>(p.Y) + (int64_t)m * p.N + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
    return;
  }
  ColOps<KIND> o;
  load_colops<KIND>(p, n, o);
  epilogue_math<KIND, ROWADD>(p, o, sxb, alpha, r, rowp);
  if (p.out_dtype == SB_OUT_F32) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<float*>(p.Y) + (int64_t)m * p.N + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.Y) + (int64_t)m * p.N + n);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = make_uint4(pack_bf16(__uint_as_float(r[8 * i]), __uint_as_float(r[8 * i + 1])),
                          pack_bf16(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3])),
                          pack_bf16(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5])),
                          pack_bf16(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7])));
  }
}

// bf16 row chunk into a 32 x 32 staging box (row = lane, 64 bytes): 16-byte granule g of row r
// sits at granule g ^ ((r >> 1) & 3), the TMA 64B swizzle, so the 32 lanes' writes hit distinct
// banks in groups of eight.
__device__ __forceinline__ void stage_bf16_row(uint32_t box, int lane, const uint32_t (&y)[32]) {
  const uint32_t row = box + 64u * (uint32_t)lane;
  const uint32_t sw = ((uint32_t)lane >> 1) & 3u;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const float* v = reinterpret_cast<const float*>(&y[8 * g]);
    st_shared_v4(row + 16u * ((uint32_t)g ^ sw), pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                 pack_bf16(v[6], v[7]));
  }
}

// stage_bf16_row for columns already packed as bf16 pairs (word i: columns 2i, 2i + 1).
__device__ __forceinline__ void stage_packed_row(uint32_t box, int lane, const uint32_t (&w)[16]) {
  const uint32_t row = box + 64u * (uint32_t)lane;
  const uint32_t sw = ((uint32_t)lane >> 1) & 3u;
#pragma unroll
  for (int g = 0; g < 4; ++g) st_shared_v4(row + 16u * ((uint32_t)g ^ sw), w[4 * g], w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]);
}

// What the epilogue warps of one CTA share.
struct EpiCtx {
  uint64_t* tfull;
  uint32_t tempty_leader;  // shared::cluster address of the leader's tempty[0]
  volatile int* abort;
  uint32_t tmem;
  int unit, tiles, nunits, m_tiles, n_tiles, group_m, nacc, BN, M, N, row_off, q, half, lane;
  uint64_t wait_ns;
  uint32_t out_box;  // this warp's two staging boxes
  uint32_t bias_s;   // NVFP4: this warp's bias slice in shared memory (past the NVFP4 stages)
  float alpha;
  const CUtensorMap* tyc;  // kEpiModRec: where the refreshed cache goes (null: no refresh)
  bool have_prev;          // kEpiModRec: the module has a cached output (else c reads as zero)
  uint64_t pol;            // kEpiModRec: L2 evict-first policy of the record's streams
};

// The module record's streams (x and the old cache read once, the new cache written once) go
// through L2 as evict-first lines, so they do not push out the GEMM's operands, which the tile
// order keeps in L2 for reuse.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// 16-byte read-only load with an L2 policy, kept in program order (volatile): the record's loads of
// one chunk must not be hoisted above the previous chunk's stores, or their registers pile up.
__device__ __forceinline__ uint4 ld_nc_hint(const uint4* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.b32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}
__device__ __forceinline__ void tma_store_2d_hint(const void* tmap, uint32_t smem_src, int x, int y, uint64_t pol) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%1, %2}], [%3], %4;" ::"l"(tmap),
               "r"(x), "r"(y), "r"(smem_src), "l"(pol)
               : "memory");
}

// One 32 x 32 bf16 chunk (a row per lane) through a staging box and one TMA store; rows past M
// are clipped by the store. Lane kStoreLane issues the stores and owns their bulk groups, so lane
// 0's release-arrive on the accumulator barrier never waits for them.
template <bool MR = false, int NW = 32>
__device__ __forceinline__ void store_chunk_tma(const CUtensorMap* ty, const EpiCtx& e, const uint32_t (&r)[NW],
                                                int n, int m_warp, uint32_t& oc) {
  const uint32_t box = e.out_box + (oc & 1u) * (uint32_t)kOutBox;
  if (e.lane == kStoreLane) bulk_wait_read<1>();  // the store issued from this box before has read it
  __syncwarp();
  if constexpr (NW == 32)
    stage_bf16_row(box, e.lane, r);  // FP32 values, packed here
  else
    stage_packed_row(box, e.lane, r);  // bf16 pairs
  fence_proxy_async_smem();
  __syncwarp();
  if (e.lane == kStoreLane) {
    tma_store_2d(ty, box, n, m_warp);
    if (MR && e.tyc) tma_store_2d_hint(e.tyc, box, n, m_warp, e.pol);  // the module's cache refresh, same group
    bulk_commit();
  }
  ++oc;
}


// bf16 pair k of 32 packed columns (16 words; word i holds columns 2i and 2i + 1): columns k and
// k + 16 as FP32, the pairing of the row engine's statistics.
__device__ __forceinline__ float2 mr_pair(const uint32_t (&w)[16], int k) {
  const uint32_t lo = w[k >> 1], hi = w[8 + (k >> 1)];
  return (k & 1) ? make_float2(__uint_as_float(lo & 0xffff0000u), __uint_as_float(hi & 0xffff0000u))
                 : make_float2(__uint_as_float(lo << 16), __uint_as_float(hi << 16));
}

// Balanced tree over the 32 columns held as 16 pairs (column k, column k + 16): adjacent columns
// first, as the row engine sums a lane's run.
__device__ __forceinline__ float mr_tree(float2 (&t)[16]) {
#pragma unroll
  for (int len = 16; len > 1; len >>= 1) {
#pragma unroll
    for (int i = 0; i < len / 2; ++i) t[i] = ep_add2(t[2 * i], t[2 * i + 1]);
  }
  return __fadd_rn(t[0].x, t[0].y);
}

// Module record of one row's 32 output columns n .. n + 31 (kEpiModRec), yw the bf16 outputs: the
// terms are those of the row engine's fused record, on the bf16 values the output holds
// (|y|; (y - x)^2 and x^2 with the difference and the squares each rounded once; |y - c|; |c|),
// q[s] the balanced tree of term s over the 32 columns, rmx the running max |y|.
__device__ __forceinline__ void modrec_chunk(const GemmParams& p, const EpiCtx& e, int m, int n,
                                             const uint32_t (&yw)[16], float (&q)[5], float& rmx) {
  uint32_t xw[16], cw[16];
  const uint4* xp = reinterpret_cast<const uint4*>(p.mr_x + (int64_t)m * e.N + n);
  const uint4* cp = reinterpret_cast<const uint4*>(p.mr_c + (int64_t)m * e.N + n);
  // x and c together, so that one memory round trip serves both; each element of c is read here
  // before this thread's own chunk is stored to the cache, so the read-only path never serves a
  // value this kernel has overwritten
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = ld_nc_hint(xp + i, e.pol);
    xw[4 * i] = v.x, xw[4 * i + 1] = v.y, xw[4 * i + 2] = v.z, xw[4 * i + 3] = v.w;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = e.have_prev ? ld_nc_hint(cp + i, e.pol) : make_uint4(0u, 0u, 0u, 0u);
    cw[4 * i] = v.x, cw[4 * i + 1] = v.y, cw[4 * i + 2] = v.z, cw[4 * i + 3] = v.w;
  }
  float2 t[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float2 y = mr_pair(yw, k);
    t[k] = make_float2(fabsf(y.x), fabsf(y.y));
    rmx = max3(rmx, t[k].x, t[k].y);
  }
  q[0] = mr_tree(t);
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float2 y = mr_pair(yw, k), x = mr_pair(xw, k);
    const float dx = __fsub_rn(y.x, x.x), dy = __fsub_rn(y.y, x.y);
    t[k] = make_float2(__fmul_rn(dx, dx), __fmul_rn(dy, dy));
  }
  q[1] = mr_tree(t);
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float2 x = mr_pair(xw, k);
    t[k] = make_float2(__fmul_rn(x.x, x.x), __fmul_rn(x.y, x.y));
  }
  q[2] = mr_tree(t);
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float2 y = mr_pair(yw, k), c = mr_pair(cw, k);
    t[k] = make_float2(fabsf(__fsub_rn(y.x, c.x)), fabsf(__fsub_rn(y.y, c.y)));
  }
  q[3] = mr_tree(t);
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float2 c = mr_pair(cw, k);
    t[k] = make_float2(fabsf(c.x), fabsf(c.y));
  }
  q[4] = mr_tree(t);
}

// The epilogue of every tile of this CTA. DRAIN_ALL (one accumulator buffer, and the record form
// in every precision): the warp's columns are moved to registers and the buffer released before
// any arithmetic, so the next tile's MMAs can start. Otherwise (two buffers) 32-column chunks are
// loaded as they are processed and the buffer is released after the last load.
template <int KIND, bool DRAIN_ALL, int EPI>
__device__ __forceinline__ void epilogue_loop(const GemmParams& p, const CUtensorMap* ty, const EpiCtx& e) {
  constexpr bool ROWADD = EPI == kEpiRowAdd, RECORD = EPI == kEpiRecord, MODREC = EPI == kEpiModRec;
  const int nch = e.BN / 64;  // 32-column chunks per warp: 2 or 4
  const int row = 32 * e.q + e.lane;
  uint32_t oc = 0;
  int it = 0;
  for (int tile = e.unit; tile < e.tiles; tile += e.nunits, ++it) {
    int mt, nt;
    tile_coords(tile, e.m_tiles, e.n_tiles, e.group_m, &mt, &nt);
    const int m = mt * 256 + e.row_off + row;
    const int m_warp = mt * 256 + e.row_off + 32 * e.q;
    const int n0 = nt * e.BN + e.half * (e.BN / 2);
    const int b = it % e.nacc;
    const uint32_t tph = (uint32_t)((it / e.nacc) & 1);
    const bool tma = p.tma_store && m_warp < e.M;
    // operands that do not depend on the accumulator are loaded before waiting for it
    const float sxb = (KIND == KIND_I8 && m < e.M) ? __fmul_rn(__ldg(p.sA8 + m), p.invB) : 0.0f;
    const float* rrow = (ROWADD && m < e.M) ? p.rowadd + ra_row(p, m) * (int64_t)e.N : nullptr;
    ColOps<KIND> ops;
    float mq[MODREC ? 4 : 1][5], mrx = 0.0f;  // MODREC: per 32-column chunk partial sums, max |y|
    if constexpr (DRAIN_ALL) {
      // NVFP4: the warp's bias slice (128 columns, 256 bytes) goes to shared memory asynchronously
      // (the INT8 / BF16 stages fill the whole stage area, so their drained form reads it per chunk)
      if constexpr (KIND == KIND_FP4) {
        if (tma && p.bias && e.lane < 16) cp_async16(e.bias_s + 16u * (uint32_t)e.lane, p.bias + n0 + 8 * e.lane);
      }
      cp_async_commit();
    } else {
      if (tma) load_colops<KIND>(p, n0, ops);
    }
    if (!mbar_wait_bounded(&e.tfull[b], tph, e.abort, e.wait_ns)) {
      set_error(p.hdr, SB_ETIMEOUT);
      *e.abort = 1;
      break;
    }
    tc_fence_after();
    const uint32_t tcol = e.tmem + ((uint32_t)(32 * e.q) << 16) + (uint32_t)(b * e.BN + e.half * (e.BN / 2));
    if constexpr (DRAIN_ALL) {
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < nch) tmem_ld32(tcol + 32u * c, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (e.lane == 0) mbar_arrive_cluster(e.tempty_leader + 8u * b);  // the leader waits for both CTAs
      cp_async_wait_all();
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n = n0 + 32 * c;
        if (c < nch && n < e.N) {
          if (tma) {
            if constexpr (KIND == KIND_FP4) {
              if (p.bias) {
#pragma unroll
                for (int i = 0; i < 4; ++i) ops.b[i] = ld_shared_v4(e.bias_s + 64u * c + 16u * i);
              }
            } else {  // the record form drains INT8 / BF16 tiles too: bias (and scales) from L1
              load_colops<KIND>(p, n, ops);
            }
            epilogue_math<KIND, ROWADD>(p, ops, sxb, e.alpha, r[c], rrow ? rrow + n : nullptr);
            if constexpr (MODREC) {  // packed now; recorded and stored below, once every chunk is
#pragma unroll
              for (int i = 0; i < 16; ++i)
                r[c][i] = pack_bf16(__uint_as_float(r[c][2 * i]), __uint_as_float(r[c][2 * i + 1]));
            } else {
              store_chunk_tma(ty, e, r[c], n, m_warp, oc);
            }
          } else if (m < e.M) {
            store_direct<KIND, ROWADD>(p, m, n, sxb, e.alpha, r[c], rrow ? rrow + n : nullptr);
          }
        }
      }
      if constexpr (MODREC) {  // each chunk's record reads the old cache before the chunk is stored there
        if (tma) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t yw[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) yw[i] = r[c][i];
            if (m < e.M) modrec_chunk(p, e, m, n0 + 32 * c, yw, mq[c], mrx);
            store_chunk_tma<true, 16>(ty, e, yw, n0 + 32 * c, m_warp, oc);
          }
        }
      }
      if constexpr (RECORD) {  // 256-wide tiles: the warp's 128 columns are one aligned chunk
        if (m < e.M) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {  // the values the bf16 output holds
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const uint32_t w = pack_bf16(__uint_as_float(r[c][2 * i]), __uint_as_float(r[c][2 * i + 1]));
              r[c][2 * i] = w << 16;
              r[c][2 * i + 1] = w & 0xffff0000u;
            }
          }
          p.records[(int64_t)m * p.rec_nc + (n0 >> 7)] = chunk_record<128>(r);
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (c < nch) {
          uint32_t r[32];
          tmem_ld32(tcol + 32u * c, r);
          tmem_ld_wait();
          if (c == nch - 1) {
            tc_fence_before();
            __syncwarp();
            if (e.lane == 0) mbar_arrive_cluster(e.tempty_leader + 8u * b);
          }
          const int n = n0 + 32 * c;
          if (n < e.N) {
            if (tma) {
              ColOps<KIND> next;
              if (c + 1 < nch && n + 32 < e.N) load_colops<KIND>(p, n + 32, next);
              epilogue_math<KIND, ROWADD>(p, ops, sxb, e.alpha, r, rrow ? rrow + n : nullptr);
              if constexpr (MODREC) {
                uint32_t yw[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) yw[i] = pack_bf16(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                if (m < e.M) modrec_chunk(p, e, m, n, yw, mq[c], mrx);
                store_chunk_tma<true, 16>(ty, e, yw, n, m_warp, oc);
              } else {
                store_chunk_tma(ty, e, r, n, m_warp, oc);
              }
              ops = next;
            } else if (m < e.M) {
              store_direct<KIND, ROWADD>(p, m, n, sxb, e.alpha, r, rrow ? rrow + n : nullptr);
            }
          }
        }
      }
    }
    if constexpr (MODREC) {  // 256-wide tiles: the warp's 128 columns are one aligned chunk
      if (tma && m < e.M) {
        float q[5];
#pragma unroll
        for (int k = 0; k < 5; ++k) q[k] = __fadd_rn(__fadd_rn(mq[0][k], mq[1][k]), __fadd_rn(mq[2][k], mq[3][k]));
        float4* dst = p.mr_rec + 2 * ((int64_t)m * p.rec_nc + (n0 >> 7));
        dst[0] = make_float4(q[0], q[1], q[2], q[3]);
        dst[1] = make_float4(q[4], mrx, 0.0f, 0.0f);
      }
    }
  }
  if (e.lane == kStoreLane) bulk_wait_all();  // staged outputs are read and written before the CTA exits
  __syncwarp();
}

// ---------------------------------------------------------------------------------------------
// MMA issue (one thread of the leader CTA). The loop is instantiated per precision and number of
// 128-column scale tiles so that a full K-block is straight-line code: shared-memory descriptors
// are advanced by adding to their 14-bit start-address field (addresses stay below 256 KB), and
// TMEM addresses are precomputed.
// ---------------------------------------------------------------------------------------------

struct Issuer {
  uint64_t* full;
  uint64_t* empty;
  uint64_t* tfull;
  uint64_t* tempty;
  volatile int* abort;
  uint32_t smem;      // shared address of stage 0
  uint32_t stage16;   // stage size in 16-byte units
  int stages, nkb, tail_nk, tiles, unit, nunits, BN, nacc, m_tiles, n_tiles, group_m;
  uint64_t wait_ns;
  uint32_t tmem, sfa, sfb, idesc;  // TMEM base, scale columns (absolute), instruction descriptor
};

template <int KIND>
__device__ __forceinline__ void mma_one(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t sfa,
                                        uint32_t sfb, uint32_t acc) {
  if constexpr (KIND == KIND_FP4)
    mma_fp4_pair(d, ad, bd, idesc, sfa, sfb, acc);
  else if constexpr (KIND == KIND_I8)
    mma_i8_pair(d, ad, bd, idesc, acc);
  else
    mma_bf16_pair(d, ad, bd, idesc, acc);
}

// One K-block: NVFP4 scale copies (SFA atom j -> 4 columns at 4j; SFB atom j of column tile t ->
// 4 columns at 8j + 4t), then the nk MMAs of 32 bytes of K each. The MMA reads the scales of
// output column n from column (n / 32) of its SFB columns, so a tile that starts 64 columns into
// a 128-column scale tile (192-wide tiles) passes its SFB address advanced by `shift` = 2.
template <int KIND, int SFT>
__device__ __forceinline__ void issue_kblock(const Issuer& c, uint32_t d, uint64_t ad, uint64_t bd, uint64_t fa,
                                             uint64_t fb, int nk, bool first, uint32_t shift) {
  if (nk == 4) {
    if constexpr (KIND == KIND_FP4) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        tmem_cp_sf_pair(c.sfa + 4u * j, fa + 32u * j);
#pragma unroll
        for (int t = 0; t < SFT; ++t) tmem_cp_sf_pair(c.sfb + 8u * j + 4u * t, fb + 128u * t + 32u * j);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      mma_one<KIND>(d, ad + 2u * j, bd + 2u * j, c.idesc, c.sfa + 4u * j, c.sfb + 8u * j + shift,
                    (first && j == 0) ? 0u : 1u);
  } else {
    if constexpr (KIND == KIND_FP4) {
      for (int j = 0; j < nk; ++j) {
        tmem_cp_sf_pair(c.sfa + 4u * j, fa + 32u * j);
#pragma unroll
        for (int t = 0; t < SFT; ++t) tmem_cp_sf_pair(c.sfb + 8u * j + 4u * t, fb + 128u * t + 32u * j);
      }
    }
    for (int j = 0; j < nk; ++j)
      mma_one<KIND>(d, ad + 2u * j, bd + 2u * j, c.idesc, c.sfa + 4u * j, c.sfb + 8u * j + shift,
                    (first && j == 0) ? 0u : 1u);
  }
}

// Returns false when a wait gave up.
template <int KIND, int SFT>
__device__ __noinline__ bool issue_all(const Issuer c) {
  const uint64_t dsw = desc_sw128(c.smem);
  const uint64_t dsf = desc_sf(c.smem);
  int s = 0;
  uint32_t ph = 0;
  int it = 0;
  for (int tile = c.unit; tile < c.tiles; tile += c.nunits, ++it) {
    const int b = (c.nacc == 1) ? 0 : (it & 1);
    const uint32_t tph = (uint32_t)(((c.nacc == 1) ? it : (it >> 1)) & 1);
    if (!mbar_wait_bounded(&c.tempty[b], tph ^ 1u, c.abort, c.wait_ns)) return false;
    tc_fence_after();
    const uint32_t d = c.tmem + (uint32_t)(b * c.BN);
    uint32_t shift = 0;
    if (KIND == KIND_FP4) {
      int mt, nt;
      tile_coords(tile, c.m_tiles, c.n_tiles, c.group_m, &mt, &nt);
      shift = (uint32_t)(((nt * c.BN) & 127) >> 5);
    }
    for (int kb = 0; kb < c.nkb; ++kb) {
      if (!mbar_wait_bounded(&c.full[s], ph, c.abort, c.wait_ns)) return false;
      tc_fence_after();
      const uint32_t so = (uint32_t)s * c.stage16;
      const uint64_t ad = dsw + so;
      issue_kblock<KIND, SFT>(c, d, ad, ad + (kOffB >> 4), dsf + so + (kOffSFA >> 4), dsf + so + (kOffSFB >> 4),
                              (kb == c.nkb - 1) ? c.tail_nk : 4, kb == 0, shift);
      mma_commit_pair(&c.empty[s], (uint16_t)3);  // frees the stage in both CTAs
      if (++s == c.stages) {
        s = 0;
        ph ^= 1u;
      }
    }
    mma_commit_pair(&c.tfull[b], (uint16_t)3);  // both CTAs' accumulators are ready
  }
  return true;
}

// EPI: kEpiPlain; kEpiRowAdd, the delta-token form, whose epilogue adds each output row's cube row
// of p.rowadd; kEpiRecord, which also writes the output's chunk records. Separate instantiations,
// so the plain kernel's code and registers do not change.
template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_gemm(const __grid_constant__ TMaps tm, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStageArea);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kind = *p.prec;
  if (kind < 0 || kind > 2) return;  // skipped module: nothing to compute (uniform)
  if (!p.have[kind]) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_error(p.hdr, SB_EINVAL);
    return;
  }
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const bool fp4 = (kind == KIND_FP4);
  const int M = p.M, N = p.N, K = p.K, BN = p.bn[kind];
  const int kb_elems = fp4 ? 256 : (kind == KIND_I8 ? 128 : 64);
  const int mma_k = kb_elems >> 2;
  const int nkb = (K + kb_elems - 1) / kb_elems;
  const int m_tiles = (M + 255) / 256;
  const int n_tiles = (N + BN - 1) / BN;
  const int tiles = m_tiles * n_tiles;
  const int unit = (int)(blockIdx.x >> 1);
  const int nunits = (int)(gridDim.x >> 1);
  if (unit >= tiles) return;  // both CTAs of the cluster leave together
  const int stages = fp4 ? kStagesF : kStagesQ;
  const int stage_bytes = fp4 ? kStageBytesF : kStageBytesQ;
  const int row_off = 128 * (int)rank;  // this CTA's rows inside the 256-row tile
  const int sf_tiles = (BN + 127) / 128;  // NVFP4: 128-column scale tiles of B per output tile
  const int nacc = (2 * BN + (fp4 ? (int)kSfCols : 0) <= (int)kTmemCols) ? 2 : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  cluster_sync();  // the peer's barriers exist before any remote arrive or copy
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t sfa_col = (uint32_t)(nacc * BN);  // NVFP4: 4 columns per MMA (128 rows x 4 scales)
  const uint32_t sfb_col = sfa_col + 16u;          // NVFP4: 8 columns per MMA (up to 2 column tiles)

  if (warp < kEpiWarp0) {
    setmaxnreg_dec<kRegsCtl>();  // one instruction for the whole first warpgroup
    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer (both CTAs)
      if (elect_one()) {
        prefetch_tmap(&tm.a[kind]);
        prefetch_tmap(&tm.b[kind]);
        if (fp4) {
          prefetch_tmap(&tm.sfa);
          prefetch_tmap(&tm.sfb);
        }
        const uint32_t full_leader = cluster_addr(&full[0], 0);
        // bytes both CTAs deliver to the leader's barrier per stage
        const uint32_t stage_tx = 2u * (16384u + (uint32_t)(BN / 2) * 128u + (fp4 ? 2048u * (1u + sf_tiles) : 0u));
        int s = 0;
        uint32_t ph = 0;
        int64_t issued = 0;
        bool ok = true;
        for (int tile = unit; ok && tile < tiles; tile += nunits) {
          int mt, nt;
          tile_coords(tile, m_tiles, n_tiles, p.group_m, &mt, &nt);
          const int m0 = mt * 256 + row_off, n0 = nt * BN;
          for (int kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, p.wait_ns)) {
              ok = false;
              break;
            }
            uint8_t* st = smem + s * stage_bytes;
            const uint32_t fb = full_leader + 8u * s;
            if (leader) mbar_arrive_expect_tx(&full[s], stage_tx);
            const int x = (kind == KIND_BF16) ? kb * 64 : kb * 128;  // 128-byte column slab
            if (leader && issued == p.withhold) {  // stall drill: announced bytes that never come
              ++issued;
              if (++s == stages) {
                s = 0;
                ph ^= 1u;
              }
              continue;
            }
            tma_load_2d_pair(st, &tm.a[kind], fb, x, m0);
            tma_load_2d_pair(st + kOffB, &tm.b[kind], fb, x, n0 + (BN / 2) * (int)rank);
            if (fp4) {
              // 4 scale atoms (64 K-elements each) of this CTA's 128 rows and of every 128-column
              // tile of B; atoms past K and rows past M read as zero
              tma_load_3d_pair(st + kOffSFA, &tm.sfa, fb, 0, 4 * kb, m0 >> 7);
              for (int t = 0; t < sf_tiles; ++t)
                tma_load_3d_pair(st + kOffSFB + 2048 * t, &tm.sfb, fb, 0, 4 * kb, (n0 >> 7) + t);
            }
            ++issued;
            if (++s == stages) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) {
          set_error(p.hdr, SB_ETIMEOUT);
          *abort_flag = 1;
          if (leader) {  // both CTAs' copies complete on the leader's barriers: let them land
            const int64_t first = issued > stages ? issued - stages : 0;
            for (int64_t k = first; k < issued; ++k)
              mbar_wait_bounded(&full[k % stages], (uint32_t)((k / stages) & 1), nullptr, kDrainNs);
          }
        }
      }
      __syncwarp();
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issue (leader)
      if (leader && elect_one()) {
        Issuer c;
        c.full = full;
        c.empty = empty;
        c.tfull = tfull;
        c.tempty = tempty;
        c.abort = abort_flag;
        c.smem = smem_u32(smem);
        c.stage16 = (uint32_t)stage_bytes >> 4;
        c.stages = stages;
        c.nkb = nkb;
        c.tail_nk = min(4, (K - (nkb - 1) * kb_elems) / mma_k);
        c.tiles = tiles;
        c.unit = unit;
        c.nunits = nunits;
        c.BN = BN;
        c.m_tiles = m_tiles;
        c.n_tiles = n_tiles;
        c.group_m = p.group_m;
        c.wait_ns = p.wait_ns;
        c.nacc = nacc;
        c.tmem = tmem_base;
        c.sfa = tmem_base + sfa_col;
        c.sfb = tmem_base + sfb_col;
        c.idesc = idesc_for(kind, 256, BN);
        bool ok;
        if (fp4)
          ok = (sf_tiles == 2) ? issue_all<KIND_FP4, 2>(c) : issue_all<KIND_FP4, 1>(c);
        else if (kind == KIND_I8)
          ok = issue_all<KIND_I8, 0>(c);
        else
          ok = issue_all<KIND_BF16, 0>(c);
        if (!ok) {
          set_error(p.hdr, SB_ETIMEOUT);
          *abort_flag = 1;
        }
        // wait for every MMA issued by this thread before TMEM is released
        mma_commit_pair(drain, (uint16_t)1);
        mbar_wait_bounded(drain, 0u, nullptr, kWaitNs);
      }
      __syncwarp();
    }
  } else {
    setmaxnreg_inc<kRegsEpi>();
    // ------------------------------------------------------------------ epilogue (both CTAs)
    EpiCtx e;
    e.tfull = tfull;
    e.tempty_leader = cluster_addr(&tempty[0], 0);
    e.abort = abort_flag;
    e.tmem = tmem_base;
    e.unit = unit;
    e.tiles = tiles;
    e.nunits = nunits;
    e.m_tiles = m_tiles;
    e.n_tiles = n_tiles;
    e.group_m = p.group_m;
    e.wait_ns = p.wait_ns;
    e.nacc = nacc;
    e.BN = BN;
    e.M = M;
    e.N = N;
    e.row_off = row_off;
    e.q = warp & 3;                    // TMEM lane quadrant this warp may access
    e.half = (warp - kEpiWarp0) >> 2;  // two warps per quadrant split the tile's columns
    e.lane = lane;
    e.out_box = smem_u32(smem + kOutOff) + (uint32_t)(2 * (warp - kEpiWarp0) * kOutBox);
    e.bias_s = smem_u32(smem + kBiasOffF) + 256u * (uint32_t)(warp - kEpiWarp0);
    e.alpha = fp4 ? __fmul_rn(__fmul_rn(*p.gA4, *p.gB4), p.invB) : 1.0f;
    e.tyc = nullptr;
    e.have_prev = false;
    e.pol = 0;
    if (EPI == kEpiModRec) {  // the module state decides the cache's part: read as zero, refreshed
      e.have_prev = p.mr_st->n_out >= 1;
      e.pol = l2_evict_first_policy();
      if (p.mr_update && p.mr_st->skip == 0) e.tyc = &tm.yc;
    }
    if (fp4) {
      // with two accumulators the row-addend form streams its chunks (one chunk of accumulators
      // and addends live at a time); the plain form drains every column first
      if (EPI == kEpiRowAdd && nacc == 2)
        epilogue_loop<KIND_FP4, false, EPI>(p, &tm.y, e);
      else
        epilogue_loop<KIND_FP4, true, EPI>(p, &tm.y, e);
    } else if (kind == KIND_I8) {  // the record form drains every column first in all precisions
      epilogue_loop<KIND_I8, EPI == kEpiRecord, EPI>(p, &tm.y, e);
    } else {
      epilogue_loop<KIND_BF16, EPI == kEpiRecord, EPI>(p, &tm.y, e);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer is done with this pair's TMEM, barriers and shared memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() { return tmap_encoder(); }

// 2-D row-major map: `inner` elements per row, `outer` rows; box = 128 bytes x box_rows, SW128.
static bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t inner,
                     uint64_t outer, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over an NVFP4 block-scale array in the tensor-core layout (512-byte atoms of 128 rows x
// 4 groups, K/64 atoms per 128-row tile): 128 32-bit words per atom x K/64 atoms x row tiles;
// box = 4 atoms of one row tile (2 KB), no swizzle.
static bool make_sf_map(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, K / 64, (rows + 127) / 128};
  cuuint64_t strides[2] = {512, (K / 64) * 512};
  cuuint32_t box[3] = {128, 4, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int device_sms() { return device_sm_count(); }

// M-tiles per raster group: 8, so a group's A rows stay in L2 across its N sweep. Groups sized
// to one wave of the persistent grid for narrow outputs (every N-tile of 6 M-tiles for the
// 3072-wide second FFN layer) measured the same within run-to-run noise (+-4%) on the DiT shapes.
static int pick_group_m(int64_t m_tiles, int64_t n_tiles, int64_t units) {
  (void)m_tiles;
  (void)n_tiles;
  (void)units;
  return 8;
}

// Stall drill (sb_drill_gemm_stall): armed by the host, taken by the next launch.
static std::atomic<int64_t> g_drill_withhold{-1};
static std::atomic<uint64_t> g_drill_wait_ns{0};

void arm_gemm_stall_drill(int64_t withhold_stage, uint64_t wait_ns) {
  g_drill_wait_ns.store(wait_ns);
  g_drill_withhold.store(withhold_stage);
}

// Shared-memory attribute and register-split check of one k_gemm instantiation.
template <int EPI>
static cudaError_t gemm_ready(const char** why) {
  static std::atomic<uint64_t> attr{0};  // one bit per device
  const cudaError_t attr_err = smem_attr_once(k_gemm<EPI>, kSmemBytes, attr);
  if (attr_err != cudaSuccess) {
    *why = "cudaFuncSetAttribute(max dynamic shared memory) failed";
    return attr_err;
  }
  // The register split of the kernel must fit what a CTA is launched with, or the epilogue's
  // setmaxnreg.inc would wait for registers that never come free.
  static std::atomic<int> regs{-1};
  if (regs.load() < 0) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, k_gemm<EPI>) != cudaSuccess) {
      *why = "cudaFuncGetAttributes(k_gemm) failed";
      return cudaErrorInvalidValue;
    }
    regs.store(fa.numRegs);
  }
  if (regs.load() * kThreads < kRegsNeeded) {
    *why = "k_gemm was compiled with fewer registers per thread than its warpgroup split needs";
    return cudaErrorInvalidConfiguration;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t s, const char** why) {
  const bool rowadd = L.rowadd != nullptr, record = L.records != nullptr, modrec = L.mr_rec != nullptr;
  const cudaError_t ready = modrec ? gemm_ready<kEpiModRec>(why)
                                   : (record ? gemm_ready<kEpiRecord>(why)
                                             : (rowadd ? gemm_ready<kEpiRowAdd>(why) : gemm_ready<kEpiPlain>(why)));
  if (ready != cudaSuccess) return ready;
  TMaps tm;
  memset(&tm, 0, sizeof(tm));
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = (int)L.M;
  p.N = (int)L.N;
  p.K = (int)L.K;
  // Tile width per precision: 256, or 128 when N is not a multiple of 256. NVFP4 takes 192-wide
  // tiles (two accumulators next to the scale columns) when N is a multiple of 192 but not of 256:
  // measured on B200, 16% and 10% faster than 128-wide tiles on 1920-wide layers, while on the FFN
  // shapes one 256-wide accumulator beats two 192-wide ones by 5-12% (the narrower tile reads more
  // shared memory per MMA flop).
  const int bn_q = (L.N % 256 == 0) ? 256 : 128;
  const int bn_f = (L.N % 256 != 0 && L.N % 192 == 0) ? 192 : bn_q;
  p.bn[KIND_FP4] = bn_f;
  p.bn[KIND_I8] = p.bn[KIND_BF16] = bn_q;
  p.invB = 1.0f / (float)L.B;
  p.prec = L.prec;
  p.sA8 = L.sA8;
  p.sB8 = L.sB8;
  p.gA4 = L.gA4;
  p.gB4 = L.gB4;
  p.bias = reinterpret_cast<const __nv_bfloat16*>(L.bias);
  p.Y = L.Y;
  p.out_dtype = L.out_dtype;
  p.epilogue = L.epilogue;
  p.hdr = reinterpret_cast<WsHeader*>(L.hdr);
  p.rowadd = L.rowadd;
  if (rowadd) {
    p.ra_T = L.ra_T;
    p.ra_H = L.ra_H;
    p.ra_W = L.ra_W;
    p.ra_ct = L.ra_ct;
    p.ra_ch = L.ra_ch;
    p.ra_cw = L.ra_cw;
    p.ra_nh = ceil_div(L.ra_H, L.ra_ch > 0 ? L.ra_ch : 1);
    p.ra_nw = ceil_div(L.ra_W, L.ra_cw > 0 ? L.ra_cw : 1);
  }
  p.records = reinterpret_cast<float4*>(L.records);
  p.rec_nc = (int)(L.N / 128);
  p.mr_x = reinterpret_cast<const __nv_bfloat16*>(L.mr_x);
  p.mr_c = reinterpret_cast<const __nv_bfloat16*>(L.mr_c);
  p.mr_rec = reinterpret_cast<float4*>(L.mr_rec);
  p.mr_st = L.mr_st;
  p.mr_update = L.mr_update;
  p.withhold = g_drill_withhold.exchange(-1);
  const uint64_t drill_ns = g_drill_wait_ns.exchange(0);
  p.wait_ns = (p.withhold >= 0 && drill_ns != 0) ? drill_ns : kWaitNs;
  // bf16 output through TMA stores when the output satisfies their alignment (else direct stores)
  if (L.out_dtype == SB_OUT_BF16 && (reinterpret_cast<uintptr_t>(L.Y) & 15) == 0) {
    auto fn = encode_fn();
    cuuint64_t dims[2] = {(cuuint64_t)L.N, (cuuint64_t)L.M};
    cuuint64_t strides[1] = {(cuuint64_t)L.N * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    p.tma_store = fn && fn(&tm.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L.Y, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    if (modrec && p.tma_store)
      p.tma_store = fn(&tm.yc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, L.mr_c, dims, strides, box, estr,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  if (modrec && !p.tma_store) {  // the record form stores the output and the cache through TMA only
    *why = "cuTensorMapEncodeTiled failed (output or cache of the module record)";
    return cudaErrorInvalidValue;
  }
  const uint64_t M = (uint64_t)L.M, N = (uint64_t)L.N, K = (uint64_t)L.K;
  const uint32_t half = (uint32_t)bn_q / 2;  // B rows each CTA of the pair loads (INT8 / BF16)
  if (L.A4 && L.B4 && L.sfA4 && L.sfB4 && L.gA4 && L.gB4) {
    if (!make_map(&tm.a[KIND_FP4], L.A4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, M, 128) ||
        !make_map(&tm.b[KIND_FP4], L.B4, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K / 2, N, (uint32_t)bn_f / 2) ||
        !make_sf_map(&tm.sfa, L.sfA4, K, M) || !make_sf_map(&tm.sfb, L.sfB4, K, N)) {
      *why = "cuTensorMapEncodeTiled failed (NVFP4 operands)";
      return cudaErrorInvalidValue;
    }
    p.have[KIND_FP4] = 1;
  }
  if (L.A8 && L.B8 && L.sA8 && L.sB8) {
    if (!make_map(&tm.a[KIND_I8], L.A8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, M, 128) ||
        !make_map(&tm.b[KIND_I8], L.B8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, K, N, half)) {
      *why = "cuTensorMapEncodeTiled failed (INT8 operands)";
      return cudaErrorInvalidValue;
    }
    p.have[KIND_I8] = 1;
  }
  if (L.X && L.W16) {
    if (!make_map(&tm.a[KIND_BF16], L.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, M, 128) ||
        !make_map(&tm.b[KIND_BF16], L.W16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, K, N, half)) {
      *why = "cuTensorMapEncodeTiled failed (BF16 operands)";
      return cudaErrorInvalidValue;
    }
    p.have[KIND_BF16] = 1;
  }
  // one cluster of two CTAs per 256 x BN tile, at most one CTA per SM
  const int64_t want = 2 * ceil_div(L.M, 256) * ceil_div(L.N, bn_q < bn_f ? bn_q : bn_f);
  const int sms = device_sms() & ~1;
  const unsigned grid = (unsigned)(want < sms ? want : sms);
  p.group_m = pick_group_m(ceil_div(L.M, 256), ceil_div(L.N, bn_q), grid / 2);
  if (modrec)
    k_gemm<kEpiModRec><<<grid, kThreads, kSmemBytes, s>>>(tm, p);
  else if (record)
    k_gemm<kEpiRecord><<<grid, kThreads, kSmemBytes, s>>>(tm, p);
  else if (rowadd)
    k_gemm<kEpiRowAdd><<<grid, kThreads, kSmemBytes, s>>>(tm, p);
  else
    k_gemm<kEpiPlain><<<grid, kThreads, kSmemBytes, s>>>(tm, p);
  return cudaGetLastError();
}

}  // namespace sb
