// prepass.cu -- streaming kernels of the activation pre-pass and of the Temporal Delta Cache.
//
//  k_rows<.., OP_PREPASS>  one pass over X (and X_ref): block Hadamard rotation, per-token rotated
//                 amax, deterministic statistics (|x|, (x - x_ref)^2, x_ref^2), per-token INT8
//                 codes when the layer runs in INT8; the last CTA reduces the groups, writes the
//                 statistics record and applies Purified Delta Refresh to the precision flag.
//                 ("write-up" sections 一 (difference statistic, block Hadamard), 三 (outlier
//                 ratio max / mean), 四 (quantization fused with the Hadamard transform).)
//  k_rows<.., OP_STATS>    the same statistics without rotation (the d of a module output).
//  k_rows<.., OP_TDC>      relative L1 change between a module's new output and its cached last
//                 output, cache refresh in the same pass, module-state update by the last CTA.
//                 ("write-up" section 二; explainer section 3.)
//  k_rows<.., OP_REC>      OP_STATS (with the module input as x_ref) and OP_TDC over one read of
//                 the module output: both statistics records, the cache refresh, the state.
//  k_nvfp4        re-reads X once the tensor amax is known, rotates again and writes E2M1 codes,
//                 E4M3 block scales in the tensor-core layout and the FP32 tensor scale.
//  k_rotate       rotation only (test hook).
#include "launch_util.h"
#include "prepass_blk.cuh"
#include "rows.cuh"
#include "tmap.h"

namespace sb {

static int sm_count() { return device_sm_count(); }

static RowArgs row_args_from(const PrepassLaunch& p) {
  RowArgs a{};
  a.X = reinterpret_cast<const __nv_bfloat16*>(p.X);
  a.R = const_cast<__nv_bfloat16*>(reinterpret_cast<const __nv_bfloat16*>(p.R));
  a.M = p.M;
  a.K = (int)p.K;
  a.B = p.B;
  a.mode = p.mode;
  a.prec = p.prec;
  a.force_int8 = p.force_int8;
  a.q8 = p.q8;
  a.s8 = p.s8;
  a.rho = p.rho;
  a.force = p.force;
  a.groups = reinterpret_cast<GroupSlot*>(p.groups);
  a.hdr = reinterpret_cast<WsHeader*>(p.hdr);
  a.stats = p.stats;
  a.finish = p.finish;
  return a;
}

// TMA maps of a row kernel's tensors; a.tma stays 0 (direct loads) when a row is not a whole
// number of 128-byte chunks or a map cannot be built.
static void row_maps(RowArgs& a, RowMaps& mp, const void* X, const void* R) {
  memset(&mp, 0, sizeof(mp));
  a.tma = make_row_segment_map(&mp.x, X, a.M, a.K) && (!R || make_row_segment_map(&mp.r, R, a.M, a.K)) ? 1 : 0;
}

template <int B>
static cudaError_t launch_pb(const RowArgs& a, const PbGeom& gm, const CUtensorMap& mx, unsigned grid, cudaStream_t s) {
  constexpr int dsm = kPbRing + 1024;
  static std::atomic<uint64_t> attr{0};  // per instantiation, one bit per device
  const cudaError_t e = smem_attr_once(k_prepass_blk<B>, dsm, attr);
  if (e != cudaSuccess) return e;
  k_prepass_blk<B><<<grid, kPbThreads, dsm, s>>>(a, gm, mx);
  return cudaGetLastError();
}

// The block-per-lane pre-pass (k_prepass_blk): no x_ref, B <= 128, whole 128-channel blocks and a
// team shape and tensor map that fit. Returns false (nothing launched) otherwise.
static bool launch_prepass_blk(const RowArgs& a, cudaStream_t s, int sms, cudaError_t* err) {
  if (a.R || a.B > 128 || a.K % 128 != 0) return false;
  PbGeom gm;
  if (!pick_pb_geom(a.K / 128, &gm)) return false;
  CUtensorMap mx;
  if (!make_halfblock_map(&mx, a.X, a.M, a.K)) return false;
  const int64_t groups = ceil_div(a.M, kG);  // a team's unit of work
  const unsigned grid = (unsigned)(groups < sms ? groups : sms);
  switch (a.B) {
    case 16: *err = launch_pb<16>(a, gm, mx, grid, s); return true;
    case 32: *err = launch_pb<32>(a, gm, mx, grid, s); return true;
    case 64: *err = launch_pb<64>(a, gm, mx, grid, s); return true;
    case 128: *err = launch_pb<128>(a, gm, mx, grid, s); return true;
    default: return false;
  }
}

cudaError_t launch_prepass(const PrepassLaunch& p, cudaStream_t s) {
  RowArgs a = row_args_from(p);
  const int sms = sm_count();
  if (!(p.mode == SB_PREPASS_STATS && !p.force_int8) && !p.R) {
    cudaError_t e;
    if (launch_prepass_blk(a, s, sms, &e)) return e;
  }
  RowMaps mp;
  row_maps(a, mp, p.X, p.R);
  if (p.mode == SB_PREPASS_STATS && !p.force_int8)
    return p.R ? launch_rows_t<OP_STATS, true>(a, mp, s, sms) : launch_rows_t<OP_STATS, false>(a, mp, s, sms);
  return p.R ? launch_rows_t<OP_PREPASS, true>(a, mp, s, sms) : launch_rows_t<OP_PREPASS, false>(a, mp, s, sms);
}

cudaError_t launch_tdc_record(const TdcLaunch& p, cudaStream_t s) {
  RowArgs a{};
  a.X = reinterpret_cast<const __nv_bfloat16*>(p.Y);
  a.R = reinterpret_cast<__nv_bfloat16*>(p.Cache);
  a.M = p.M;
  a.K = (int)p.C;
  a.B = 0;
  a.update = p.update;
  a.dsrc = p.dsrc;
  a.st = p.st;
  a.groups = reinterpret_cast<GroupSlot*>(p.groups);
  a.hdr = reinterpret_cast<WsHeader*>(p.hdr);
  a.finish = p.finish;
  RowMaps mp;
  row_maps(a, mp, p.Y, p.Cache);
  return launch_rows_t<OP_TDC, true>(a, mp, s, sm_count());
}

cudaError_t launch_module_record(const RecordLaunch& p, cudaStream_t s) {
  RowArgs a{};
  a.X = reinterpret_cast<const __nv_bfloat16*>(p.Y);
  a.R = const_cast<__nv_bfloat16*>(reinterpret_cast<const __nv_bfloat16*>(p.X));
  a.C3 = reinterpret_cast<__nv_bfloat16*>(p.Cache);
  a.M = p.M;
  a.K = (int)p.C;
  a.B = 0;
  a.mode = SB_PREPASS_STATS;
  a.prec = p.prec;
  a.rho = p.rho;
  a.force = p.force;
  a.update = p.update;
  a.st = p.st;
  a.stats = p.stats;
  a.groups = reinterpret_cast<GroupSlot*>(p.groups);
  a.groups2 = reinterpret_cast<GroupSlot*>(p.groups2);
  a.hdr = reinterpret_cast<WsHeader*>(p.hdr);
  a.finish = 1;
  RowMaps mp;
  memset(&mp, 0, sizeof(mp));
  a.tma = (make_row_segment_map(&mp.x, p.Y, a.M, a.K) && make_row_segment_map(&mp.r, p.X, a.M, a.K) &&
           make_row_segment_map(&mp.c, p.Cache, a.M, a.K))
              ? 1
              : 0;
  return launch_rows_rec(a, mp, s, sm_count());
}

cudaError_t launch_finish(const FinishLaunch& p, cudaStream_t s) {
  RowArgs a{};
  a.M = p.M;
  a.K = (int)p.K;
  a.mode = p.mode;
  a.prec = p.prec;
  a.rho = p.rho;
  a.force = p.force;
  a.dsrc = p.dsrc;
  a.st = p.st;
  a.groups = const_cast<GroupSlot*>(reinterpret_cast<const GroupSlot*>(p.groups));
  a.hdr = reinterpret_cast<WsHeader*>(p.hdr);
  a.stats = p.stats;
  a.finish = 1;
  const int64_t G = ceil_div(p.M, kG);
  if (p.op == 2) {
    k_finish<OP_TDC, true><<<1, 256, 0, s>>>(a, G);
  } else if (p.mode == SB_PREPASS_STATS) {
    if (p.has_ref) k_finish<OP_STATS, true><<<1, 256, 0, s>>>(a, G);
    else k_finish<OP_STATS, false><<<1, 256, 0, s>>>(a, G);
  } else {
    if (p.has_ref) k_finish<OP_PREPASS, true><<<1, 256, 0, s>>>(a, G);
    else k_finish<OP_PREPASS, false><<<1, 256, 0, s>>>(a, G);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// NVFP4 encode: one warp per 1024-element segment of a row; a lane's 32 values are two 16-value
// scale groups, so group maxima need no shuffle.
// ---------------------------------------------------------------------------------------------

struct Nvfp4Args {
  const __nv_bfloat16* X;
  int64_t M;
  int K, B;
  const int32_t* prec;  // null: always encode
  const sb_stats* stats;
  uint8_t* codes;
  uint8_t* sf;
  float* gscale;
  WsHeader* hdr;
};

__device__ __forceinline__ int64_t sf_offset(int64_t m, int64_t g, int64_t K) {
  return ((m >> 7) * (K >> 6) + (g >> 2)) * 512 + (m & 31) * 16 + ((m & 127) >> 5) * 4 + (g & 3);
}

// E4M3 block scale of one 16-value group and the reciprocal used for its codes.
__device__ __forceinline__ void group_scale(float amax, float s_g, uint32_t* sb, float* inv, bool* zero) {
  const float sfv = __fdiv_rn(__fdiv_rn(amax, 6.0f), s_g);
  *sb = cvt_e4m3(sfv);
  const float den = __fmul_rn(e4m3_to_f32(*sb), s_g);
  *inv = (den == 0.0f) ? 0.0f : __fdiv_rn(1.0f, den);
  *zero = (den == 0.0f) || !(*inv <= FLT_MAX);
}

__global__ void __launch_bounds__(256) k_nvfp4(Nvfp4Args a) {
  if (a.prec && *a.prec != SB_NVFP4) return;
  const int lane = threadIdx.x & 31;
  const int K = a.K;
  const int nseg = (K + 1023) >> 10;
  const int64_t Mpad = (a.M + 127) & ~(int64_t)127;
  const float A = (float)a.stats->amax_rot;  // exact: a float widened to double
  const float s_g = (A == 0.0f) ? 1.0f : __fdiv_rn(A, 2688.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.gscale = s_g;
  const int64_t units = Mpad * nseg;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t u = warp0; u < units; u += nwarps) {
    const int64_t m = u / nseg;
    const int sgi = (int)(u - m * nseg);
    const int e0 = sgi * 1024 + lane * 32;
    const bool in_row = e0 < K;
    Raw32 raw;
    load_raw(raw, a.X + m * K, e0, K, in_row && m < a.M);
    float2 p[16];
    unpack_pairs(raw, p);
    fwht_pairs(p, lane, a.B);
    // group 0 = elements 0..15 = the x halves, group 1 = elements 16..31 = the y halves
    float am0 = 0.0f, am1 = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; k += 2) {
      am0 = max3(am0, fabsf(p[k].x), fabsf(p[k + 1].x));
      am1 = max3(am1, fabsf(p[k].y), fabsf(p[k + 1].y));
    }
    uint32_t sb0, sb1;
    float inv0, inv1;
    bool z0, z1;
    group_scale(am0, s_g, &sb0, &inv0, &z0);
    group_scale(am1, s_g, &sb1, &inv1, &z1);
    const float2 inv2 = make_float2(inv0, inv1);
#pragma unroll
    for (int k = 0; k < 16; ++k) p[k] = mul2(p[k], inv2);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // word q = elements 8q..8q+7 (group 0 for q < 2)
      const bool hi = q >= 2;
      const bool z = hi ? z1 : z0;
      uint32_t word = 0;
      if (!z) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int k = 8 * (q & 1) + 2 * b;
          word |= cvt_e2m1x2(hi ? p[k].y : p[k].x, hi ? p[k + 1].y : p[k + 1].x) << (8 * b);
        }
      }
      w[q] = word;
    }
    if (m < a.M && in_row)
      *reinterpret_cast<uint4*>(a.codes + m * (K >> 1) + (e0 >> 1)) = make_uint4(w[0], w[1], w[2], w[3]);
    // scale word of groups 4j..4j+3 = lanes 2j (groups 4j, 4j+1) and 2j+1 (4j+2, 4j+3)
    const uint32_t mine = sb0 | (sb1 << 8);
    const uint32_t other = __shfl_down_sync(0xffffffffu, mine, 1);
    if ((lane & 1) == 0 && in_row)
      *reinterpret_cast<uint32_t*>(a.sf + sf_offset(m, e0 >> 4, K)) = mine | (other << 16);
  }
}

// ---------------------------------------------------------------------------------------------
// NVFP4 encode with one 128-channel block per lane (B <= 128, K a multiple of 128): a lane's 8
// scale groups are its own, so warps never meet. A warp encodes 32 consecutive blocks of the
// row-padded tensor per task (TMA ring as in k_prepass_blk; rows past M read as zero, which writes
// the zero scale factors of the padding rows).
// ---------------------------------------------------------------------------------------------

// Eight values -> one word of E2M1 codes: byte t holds values 2t (low nibble) and 2t + 1.
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                           float v7) {
  uint32_t w;
  asm("{\n\t.reg .b8 c0, c1, c2, c3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n\t"
      "mov.b32 %0, {c0, c1, c2, c3};\n\t}"
      : "=r"(w)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return w;
}

// Per-tensor tables of the block-scale arithmetic, built by every CTA from the tensor scale s_g
// (a few hundred IEEE divisions per CTA, overlapped with its first loads). The block scale of a
// 16-value group is sb(amax) = E4M3(RN(RN(amax / 6) / s_g)), a monotone step function of amax,
// and its codes use inv(sb) = RN(1 / RN(dec(sb) s_g)):
//   thr[c]  the smallest amax with sb(amax) >= c (NaN when no amax reaches c, so that every
//           comparison with it is false); thr[0] = 0
//   inv[c]  inv(c), or 0 when the group's codes are all zero (dec(c) s_g = 0, or 1 / den
//           overflows)
// In the encode, c0 = E4M3(RN(amax K)) with K = RN(1 / RN(6 s_g)) is within one code of sb(amax):
// the two arguments differ by a few FP32 ulps, and E4M3 rounding boundaries are more than 2^-5
// apart relatively (2^-9 absolutely among its subnormals), so at most one boundary lies between
// them. Two comparisons with thr then give sb(amax) exactly: three instructions and two
// shared-memory loads instead of three IEEE divisions per group.
constexpr int kScaleCodes = 128;

__device__ __forceinline__ uint32_t block_scale_code(float amax, float s_g) {
  return cvt_e4m3(__fdiv_rn(__fdiv_rn(amax, 6.0f), s_g));
}

__device__ __forceinline__ void build_scale_tables(float s_g, float* inv, float* thr) {
  const int t = (int)threadIdx.x;
  if (t < kScaleCodes) {
    const float den = __fmul_rn(e4m3_to_f32((uint32_t)t), s_g);
    float r = (den == 0.0f) ? 0.0f : __fdiv_rn(1.0f, den);
    if (!(r <= FLT_MAX)) r = 0.0f;  // 1 / den overflowed (or the NaN code): zero codes
    inv[t] = r;
  } else if (t < 2 * kScaleCodes + 1) {
    const uint32_t c = (uint32_t)(t - kScaleCodes);  // 0 .. 128
    float v;
    if (c == 0) {
      v = 0.0f;
    } else if (block_scale_code(__uint_as_float(0x7f800000u), s_g) < c) {
      v = __uint_as_float(0x7fc00000u);  // unreachable code: NaN, never <= amax
    } else {
      // smallest non-negative float bit pattern b with sb(b) >= c (non-negative floats order
      // like their bit patterns, and sb is monotone): invariant sb(lo) < c <= sb(hi). The search
      // starts from a bracket of +-2^-14 around the estimate 6 s_g m (m: the E4M3 rounding
      // midpoint below code c) and falls back to the whole range when the bracket misses.
      const float m = 0.5f * (e4m3_to_f32(c - 1u) + e4m3_to_f32(c < 127u ? c : 126u));
      const float est = __fmul_rn(__fmul_rn(m, 6.0f), s_g);
      uint32_t lo = __float_as_uint(__fmul_rn(est, 1.0f - 0x1p-14f));
      uint32_t hi = __float_as_uint(__fmul_rn(est, 1.0f + 0x1p-14f));
      if (!(hi <= 0x7f800000u && block_scale_code(__uint_as_float(lo), s_g) < c &&
            block_scale_code(__uint_as_float(hi), s_g) >= c)) {
        lo = 0u;
        hi = 0x7f800000u;
      }
      if (block_scale_code(0.0f, s_g) >= c) hi = 0u;
      while (lo + 1u < hi) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (block_scale_code(__uint_as_float(mid), s_g) >= c) hi = mid;
        else lo = mid;
      }
      v = __uint_as_float(hi);
    }
    thr[c] = v;
  }
}

// Block scale code of one group from its candidate c0 and the thresholds (see above).
__device__ __forceinline__ uint32_t scale_from_tables(float amax, const float* thr, uint32_t c0) {
  uint32_t c = c0;
  if (amax >= thr[c0 + 1]) c = c0 + 1;
  else if (amax < thr[c0]) c = c0 - 1;
  return c;
}

template <int B>
__global__ void __launch_bounds__(kPbThreads, 1) k_nvfp4_blk(Nvfp4Args a, int NB, const __grid_constant__ CUtensorMap mx) {
  extern __shared__ uint8_t pb_dsm[];
  __shared__ uint64_t s_bar[kPbWarps][kPbD];
  __shared__ float s_inv[kScaleCodes];
  __shared__ float s_thr[kScaleCodes + 1];
  if (a.prec && *a.prec != SB_NVFP4) return;
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pb_dsm) + 1023) & ~(uintptr_t)1023);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = a.K;
  const float A = (float)a.stats->amax_rot;  // exact: a float widened to double
  const float s_g = (A == 0.0f) ? 1.0f : __fdiv_rn(A, 2688.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.gscale = s_g;
  const int64_t Mpad = (a.M + 127) & ~(int64_t)127;
  const int64_t nblk = Mpad * NB;
  const int ntask = (int)ceil_div(nblk, 32);
  const int nw = (int)gridDim.x * kPbWarps;
  const uint32_t ring_w = smem_u32(ring) + (uint32_t)(warp * kPbD * kPbSlot);
  // Tasks run from the end of the tensor backwards: the statistics pass that ran just before
  // read the end last, so that part is still in L2 (all of a tensor that fits).
  auto issue = [&](int t, int slot) {  // lane 0
    if (t >= ntask) return;
    const uint32_t bar = smem_u32(&s_bar[warp][slot]);
    mbar_arrive_expect_tx_u32(bar, (uint32_t)kPbSlot);
    tma_load_2d_u32(ring_w + (uint32_t)(slot * kPbSlot), &mx, bar, 0, 64 * (ntask - 1 - t));
  };
  const int t0 = (int)blockIdx.x * kPbWarps + warp;
  if (lane == 0) {
    mbar_init(&s_bar[warp][0], 1);
    mbar_init(&s_bar[warp][1], 1);
    fence_barrier_init();
    issue(t0, 0);
    issue(t0 + nw, 1);
  }
  build_scale_tables(s_g, s_inv, s_thr);
  __syncthreads();
  const float kmul = __fdiv_rn(1.0f, __fmul_rn(6.0f, s_g));
  int bad_it = -1;
  for (int it = 0, t = t0; t < ntask; ++it, t += nw) {
    const int slot = it & 1;
    __syncwarp();  // every lane has read the previous task's slot (lanes may drift apart)
    if (lane == 0 && it > 0) issue(t + nw, slot ^ 1);  // the previous task's slot, read there
    if (!mbar_wait_bounded(&s_bar[warp][slot], (uint32_t)((it >> 1) & 1), nullptr, kRowWaitNs)) {
      if (lane == 0) set_error(a.hdr, SB_ETIMEOUT);
      bad_it = it;
    }
    float2 P[64];
    pb_load_block(ring_w + (uint32_t)(slot * kPbSlot), lane, P);
#pragma unroll
    for (int k = 0; k < 64; k += 2) {
      const float2 x = P[k], y = P[k + 1];
      P[k] = add2(x, y);
      P[k + 1] = sub2(x, y);
    }
    (void)pb_stages_rest<B>(P, pb_swap(lane) ? -1.0f : 1.0f);
    const int64_t f = (int64_t)(ntask - 1 - t) * 32 + lane;
    if (f >= nblk) continue;
    const int64_t m = f / NB;
    const int blk = (int)(f - m * NB);
    // groups i (elements 16i.., the x halves of P[16i..16i+15]) and i + 4 (the y halves); a
    // swapped lane's halves are the other way round, which only moves where they are stored
    uint32_t w[16];
    uint32_t sbx = 0, sby = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float ax0 = 0.0f, ay0 = 0.0f, ax1 = 0.0f, ay1 = 0.0f;  // two chains per half
#pragma unroll
      for (int u = 0; u < 8; u += 2) {
        ax0 = max3(ax0, fabsf(P[16 * i + u].x), fabsf(P[16 * i + u + 1].x));
        ay0 = max3(ay0, fabsf(P[16 * i + u].y), fabsf(P[16 * i + u + 1].y));
        ax1 = max3(ax1, fabsf(P[16 * i + 8 + u].x), fabsf(P[16 * i + 8 + u + 1].x));
        ay1 = max3(ay1, fabsf(P[16 * i + 8 + u].y), fabsf(P[16 * i + 8 + u + 1].y));
      }
      const float ax = fmaxf(ax0, ax1), ay = fmaxf(ay0, ay1);
      uint16_t c2;  // candidate codes of both groups in one conversion: x in the low byte
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c2) : "f"(__fmul_rn(ay, kmul)), "f"(__fmul_rn(ax, kmul)));
      const uint32_t bx = scale_from_tables(ax, s_thr, (uint32_t)c2 & 0xffu);
      const uint32_t by = scale_from_tables(ay, s_thr, (uint32_t)c2 >> 8);
      const float ix = s_inv[bx], iy = s_inv[by];
      sbx |= bx << (8 * i);
      sby |= by << (8 * i);
      const float2 inv2 = make_float2(ix, iy);
      float2 q[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) q[u] = mul2(P[16 * i + u], inv2);
      w[2 * i] = (ix == 0.0f) ? 0u : e2m1x8(q[0].x, q[1].x, q[2].x, q[3].x, q[4].x, q[5].x, q[6].x, q[7].x);
      w[2 * i + 1] = (ix == 0.0f) ? 0u : e2m1x8(q[8].x, q[9].x, q[10].x, q[11].x, q[12].x, q[13].x, q[14].x, q[15].x);
      w[8 + 2 * i] = (iy == 0.0f) ? 0u : e2m1x8(q[0].y, q[1].y, q[2].y, q[3].y, q[4].y, q[5].y, q[6].y, q[7].y);
      w[9 + 2 * i] = (iy == 0.0f) ? 0u : e2m1x8(q[8].y, q[9].y, q[10].y, q[11].y, q[12].y, q[13].y, q[14].y, q[15].y);
    }
    const int hx = (int)pb_swap(lane), hy = 1 - hx;  // which half of the block x and y are
    if (m < a.M) {
      uint8_t* dst = a.codes + m * (K >> 1) + (int64_t)blk * 64;
      if (aligned32(dst)) {
        stg_v8(dst + 32 * hx, make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]));
        stg_v8(dst + 32 * hy, make_uint4(w[8], w[9], w[10], w[11]), make_uint4(w[12], w[13], w[14], w[15]));
      } else {
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          *reinterpret_cast<uint4*>(dst + 32 * hx + 16 * v) =
              make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          *reinterpret_cast<uint4*>(dst + 32 * hy + 16 * v) =
              make_uint4(w[8 + 4 * v], w[9 + 4 * v], w[10 + 4 * v], w[11 + 4 * v]);
        }
      }
    }
    *reinterpret_cast<uint32_t*>(a.sf + sf_offset(m, 8 * (int64_t)blk + 4 * hx, K)) = sbx;
    *reinterpret_cast<uint32_t*>(a.sf + sf_offset(m, 8 * (int64_t)blk + 4 * hy, K)) = sby;
  }
  if (bad_it >= 0 && lane == 0)
    mbar_wait_bounded(&s_bar[warp][bad_it & 1], (uint32_t)((bad_it >> 1) & 1), nullptr, kRowDrainNs);
}

// ---------------------------------------------------------------------------------------------
// Rotation only
// ---------------------------------------------------------------------------------------------

__global__ void __launch_bounds__(256) k_rotate(const __nv_bfloat16* X, float* Y, int64_t M, int K, int B) {
  const int lane = threadIdx.x & 31;
  const int nseg = (K + 1023) >> 10;
  const int64_t units = M * nseg;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t u = warp0; u < units; u += nwarps) {
    const int64_t m = u / nseg;
    const int e0 = (int)(u - m * nseg) * 1024 + lane * 32;
    const bool ok = e0 < K;
    Raw32 raw;
    load_raw(raw, X + m * K, e0, K, ok);
    float2 p[16];
    unpack_pairs(raw, p);
    fwht_pairs(p, lane, B);
    if (ok) {
      float4* dst = reinterpret_cast<float4*>(Y + m * K + e0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        dst[q] = make_float4(p[4 * q].x, p[4 * q + 1].x, p[4 * q + 2].x, p[4 * q + 3].x);
        dst[4 + q] = make_float4(p[4 * q].y, p[4 * q + 1].y, p[4 * q + 2].y, p[4 * q + 3].y);
      }
    }
  }
}

static unsigned stream_grid(int64_t units) {
  const int64_t want = ceil_div(units, 8);  // 8 warps per CTA, one unit each
  const int64_t cap = (int64_t)sm_count() * 8;
  return (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
}

template <int B>
static cudaError_t launch_nvfp4_blk(const Nvfp4Args& a, int NB, const CUtensorMap& mx, unsigned grid, cudaStream_t s) {
  constexpr int dsm = kPbRing + 1024;
  static std::atomic<uint64_t> attr{0};  // per instantiation, one bit per device
  const cudaError_t e = smem_attr_once(k_nvfp4_blk<B>, dsm, attr);
  if (e != cudaSuccess) return e;
  k_nvfp4_blk<B><<<grid, kPbThreads, dsm, s>>>(a, NB, mx);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4(const Nvfp4Launch& p, cudaStream_t s) {
  Nvfp4Args a{};
  a.X = reinterpret_cast<const __nv_bfloat16*>(p.X);
  a.M = p.M;
  a.K = (int)p.K;
  a.B = p.B;
  a.prec = p.prec;
  a.stats = p.stats;
  a.codes = p.codes;
  a.sf = p.sf;
  a.gscale = p.gscale;
  a.hdr = reinterpret_cast<WsHeader*>(p.hdr);
  const int64_t Mpad = (p.M + 127) & ~(int64_t)127;
  CUtensorMap mx;
  if (p.B <= 128 && p.K % 128 == 0 && p.B >= 16 && Mpad * (p.K / 64) < (int64_t(1) << 31) &&
      make_halfblock_map(&mx, p.X, p.M, p.K)) {
    const int NB = (int)(p.K / 128);
    const int64_t tasks = ceil_div(Mpad * NB, 32);
    const int64_t want = ceil_div(tasks, kPbWarps);
    const unsigned grid = (unsigned)(want < sm_count() ? want : sm_count());
    switch (p.B) {
      case 16: return launch_nvfp4_blk<16>(a, NB, mx, grid, s);
      case 32: return launch_nvfp4_blk<32>(a, NB, mx, grid, s);
      case 64: return launch_nvfp4_blk<64>(a, NB, mx, grid, s);
      case 128: return launch_nvfp4_blk<128>(a, NB, mx, grid, s);
      default: break;
    }
  }
  const int64_t units = Mpad * ceil_div(p.K, 1024);
  k_nvfp4<<<stream_grid(units), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rotate(const void* X, float* Y, int64_t M, int64_t K, int B, cudaStream_t s) {
  const int64_t units = M * ceil_div(K, 1024);
  k_rotate<<<stream_grid(units), 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(X), Y, M, (int)K, B);
  return cudaGetLastError();
}

}  // namespace sb
