// rows.cuh -- the row engine behind the pre-pass, the difference statistic and the TDC record.
//
// Layout: a lane owns 32 contiguous elements of a 1024-element row segment (four 16-byte loads),
// so a warp-wide access covers one segment and a Hadamard block of B <= 256 channels spans B/32
// neighbouring lanes. The block FWHT runs its stages h = 1..16 inside the lane and h = 32..128 with
// one shuffle + one FMA (by +-1) per element per stage. A "team" of T warps owns one row at a time
// (T*SPW segments, segment c*T + w for the w-th warp of the team); with T = 1 a row needs no
// barrier at all, with T > 1 the team meets once per row at a named barrier.
//
// Reductions follow the canonical pairwise tree of the oracle: 32 terms inside a lane, lanes
// 1..16 apart inside a segment, then a tree over the (zero-padded) segments of the row; rows meet
// in FP64 over aligned groups of kG rows (warp 0 of the CTA), groups in FP64 in the last CTA.
//
// Loads: every warp keeps a ring of D row slots in shared memory, filled by TMA a few rows ahead of
// the row it processes (one 2 KB box per 1024-element segment and tensor, 128B swizzle), so that
// enough bytes are in flight to cover the memory latency with only 8 warps per SM. Each lane then
// reads its 64 bytes from the slot without bank conflicts. Rows whose length is not a multiple of
// 64 elements (possible for the TDC record) use direct global loads instead.
#pragma once

#include <cudaTypedefs.h>

#include <cfloat>

#include "launch_util.h"
#include "sb_device.cuh"
#include "sb_kernels.h"

namespace sb {

constexpr int kRowWarps = 8;  // warps per CTA
constexpr int kG = kGroupRows;  // rows per FP64 group

enum { OP_PREPASS = 0, OP_STATS = 1, OP_TDC = 2, OP_REC = 3 };  // OP_REC: OP_STATS (x_ref) + OP_TDC in one pass

struct RowArgs {
  const __nv_bfloat16* X;  // PREPASS / STATS: the tensor; TDC, REC: the new module output
  __nv_bfloat16* R;        // PREPASS / STATS: x_ref (may be null); TDC: the cached last output; REC: x_ref
  __nv_bfloat16* C3;       // REC: the cached last output
  int64_t M;
  int K, B;
  int mode;         // SB_PREPASS_QUANT / SB_PREPASS_STATS
  int32_t* prec;    // layer precision flag (may be null)
  int force_int8;   // weight preparation: always write INT8 codes, never touch *prec
  int8_t* q8;
  float* s8;
  double rho;
  int force;
  int update;             // TDC: refresh the cache with the new output
  const sb_stats* dsrc;   // TDC: where d comes from
  sb_module_state* st;    // TDC: module state
  GroupSlot* groups;
  GroupSlot* groups2;     // REC: the TDC record's group slots (groups: the statistics')
  WsHeader* hdr;
  sb_stats* stats;
  int tma;  // rows arrive through the TMA rings (the maps below are valid)
  int finish;  // 1: the last CTA reduces the group slots; 0: only this launch's slots are written
               // (one shard of a token-sharded tensor; the slots are folded later)
};

// TMA maps of the row tensors (make_row_segment_map): x = X (TDC: the new output), r = x_ref
// (TDC: the cache).
struct RowMaps {
  CUtensorMap x;
  CUtensorMap r;
  CUtensorMap c;  // REC: the cache
};

constexpr uint64_t kRowWaitNs = 2000000000ull;  // 2 s: far above any legitimate wait
constexpr uint64_t kRowDrainNs = 20000000ull;

// Ring geometry of one k_rows instantiation: NT tensors per row, SPW 2 KB segments per tensor and
// warp, D slots per warp (2..4, about 200 KB per CTA at most).
template <int SPW, int OP, bool REF>
struct RowRing {
  static constexpr int NT = (OP == OP_REC) ? 3 : ((OP == OP_TDC || REF) ? 2 : 1);
  static constexpr int SEG = 2048;
  static constexpr int SLOT = NT * SPW * SEG;
  static constexpr int D0 = (200 * 1024) / (kRowWarps * SLOT);
  // two rows in flight per warp; the fused record (three tensors) may keep one: its slot is read
  // into registers before the next row is issued into it, so that row's load still overlaps the
  // current row's arithmetic
  static constexpr int DMIN = (OP == OP_REC) ? 1 : 2;
  static constexpr int D = D0 < DMIN ? DMIN : (D0 > 4 ? 4 : D0);
  static constexpr int BYTES = kRowWarps * D * SLOT;
};

struct Raw32 {
  uint4 q[4];
};

// The lane's 32 elements start at element e0 of a row of K elements: two 32-byte loads where the
// address is 32-byte aligned (16-byte loads otherwise); 16-byte chunks at or past the row end read
// as zero (K is a multiple of 8).
__device__ __forceinline__ bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

__device__ __forceinline__ void load_raw(Raw32& r, const __nv_bfloat16* row, int e0, int K, bool ok) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int e = e0 + 16 * h;
    if (ok && e + 16 <= K && aligned32(row + e)) {
      ldg_nc_v8(row + e, r.q[2 * h], r.q[2 * h + 1]);
    } else {
      r.q[2 * h] = (ok && e < K) ? ldg_nc_v4(row + e) : make_uint4(0, 0, 0, 0);
      r.q[2 * h + 1] = (ok && e + 8 < K) ? ldg_nc_v4(row + e + 8) : make_uint4(0, 0, 0, 0);
    }
  }
}

// The lane's 64 bytes of a 2 KB segment box written by TMA with 128B swizzle: lane l owns bytes
// [64 l, 64 l + 64), i.e. granules 4 (l & 1) .. +3 of 128-byte chunk l / 2, stored at granule
// g ^ (chunk & 7). In each load the 8 lanes of a quarter-warp touch 8 distinct granules.
__device__ __forceinline__ void read_seg_sw128(Raw32& r, uint32_t seg, int lane) {
  const uint32_t ch = (uint32_t)lane >> 1, h = (uint32_t)lane & 1u;
  const uint32_t base = seg + 128u * ch;
#pragma unroll
  for (int j = 0; j < 4; ++j) r.q[j] = ld_shared_v4(base + 16u * ((4u * h + (uint32_t)j) ^ (ch & 7u)));
}

__device__ __forceinline__ void load_raw_coherent(Raw32& r, const __nv_bfloat16* row, int e0, int K, bool ok) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int e = e0 + 16 * h;
    if (ok && e + 16 <= K && aligned32(row + e)) {
      ldg_v8(row + e, r.q[2 * h], r.q[2 * h + 1]);
    } else {
      r.q[2 * h] = (ok && e < K) ? ldg_v4(row + e) : make_uint4(0, 0, 0, 0);
      r.q[2 * h + 1] = (ok && e + 8 < K) ? ldg_v4(row + e + 8) : make_uint4(0, 0, 0, 0);
    }
  }
}

// A lane's 32 values live as 16 packed pairs p[k] = (v[k], v[k + 16]) so that FP32x2 arithmetic
// (one instruction, two independently rounded results) covers the butterflies and tree levels that
// pair elements differing in bits 0..3 of their index.
__device__ __forceinline__ uint32_t raw_word(const Raw32& r, int i) {
  const uint4 q = r.q[i >> 2];
  return (i & 3) == 0 ? q.x : (i & 3) == 1 ? q.y : (i & 3) == 2 ? q.z : q.w;
}

__device__ __forceinline__ void unpack_pairs(const Raw32& r, float2 (&p)[16]) {
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t lo = raw_word(r, k >> 1), hi = raw_word(r, 8 + (k >> 1));
    p[k] = (k & 1) ? make_float2(__uint_as_float(lo & 0xffff0000u), __uint_as_float(hi & 0xffff0000u))
                   : make_float2(__uint_as_float(lo << 16), __uint_as_float(hi << 16));
  }
}

// FP32x2 arithmetic in PTX. Each half is rounded exactly like the scalar operation, with one
// caveat measured on this toolchain: an FP32x2 multiply whose result feeds an FP32x2 add can be
// fused into one rounding even with .rn (an INT8 rounding through RN(RN(y * inv) + 1.5 2^23),
// written with the CUDA 12.9 paired-FP32 built-ins, also came out off by one against the oracle).
// So mul2 is only used where its product goes to a conversion; products that are summed are
// formed with scalar mul.rn (sq2).
__device__ __forceinline__ uint64_t f2_bits(float2 a) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a.x), "f"(a.y));
  return r;
}
__device__ __forceinline__ float2 bits_f2(uint64_t r) {
  float2 a;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a.x), "=f"(a.y) : "l"(r));
  return a;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {  // a * b + c, one rounding
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
  return bits_f2(r);
}
__device__ __forceinline__ float2 abs2(float2 a) { return make_float2(fabsf(a.x), fabsf(a.y)); }
__device__ __forceinline__ float2 sq2(float2 a) { return make_float2(__fmul_rn(a.x, a.x), __fmul_rn(a.y, a.y)); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {  // a - b = fma(b, -1, a): one rounding
  return fma2(b, make_float2(-1.0f, -1.0f), a);
}
__device__ __forceinline__ float sign127(float v) { return v > 0.0f ? 127.0f : (v < 0.0f ? -127.0f : 0.0f); }

// Pairwise tree over the lane's 32 terms t (packed like p): levels 1..4 pair indices differing in
// bits 0..3 (one FP32x2 add each), the last level adds the two halves. Destroys t.
__device__ __forceinline__ float tree_pairs(float2 (&t)[16]) {
#pragma unroll
  for (int len = 16; len > 1; len >>= 1) {
#pragma unroll
    for (int i = 0; i < len / 2; ++i) t[i] = add2(t[2 * i], t[2 * i + 1]);
  }
  return __fadd_rn(t[0].x, t[0].y);
}

// Pairwise tree over N (a power of two) values (destroys t).
template <int N>
__device__ __forceinline__ float tree_n(float (&t)[N]) {
#pragma unroll
  for (int len = N; len > 1; len >>= 1) {
#pragma unroll
    for (int i = 0; i < len / 2; ++i) t[i] = __fadd_rn(t[2 * i], t[2 * i + 1]);
  }
  return t[0];
}

__host__ __device__ constexpr int pow2_at_least(int n) { return n <= 1 ? 1 : 2 * pow2_at_least((n + 1) / 2); }

// Block FWHT of the lane's 32 values: stages h = 1, 2, 4, 8 (pairs p[k], p[k+h]), h = 16 (the two
// halves of each pair), then h = 32, 64, 128 across lanes 1, 2, 4 apart -- each while h < B.
// Lower element: a + b; upper element: a - b; every result rounded once (FP32, nearest-even).
__device__ __forceinline__ void fwht_pairs(float2 (&p)[16], int lane, int B) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
    if (h < B) {
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        if ((k & h) == 0) {
          const float2 x = p[k], y = p[k + h];
          p[k] = add2(x, y);
          p[k + h] = sub2(x, y);
        }
      }
    }
  }
  if (16 < B) {
#pragma unroll
    for (int k = 0; k < 16; ++k) p[k] = make_float2(__fadd_rn(p[k].x, p[k].y), __fsub_rn(p[k].x, p[k].y));
  }
#pragma unroll
  for (int s = 1; s < 8; s <<= 1) {
    if (32 * s < B) {
      const float sg = (lane & s) ? -1.0f : 1.0f;  // upper lane: other - own = a - b
      const float2 sg2 = make_float2(sg, sg);
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float2 o = make_float2(__shfl_xor_sync(0xffffffffu, p[k].x, s), __shfl_xor_sync(0xffffffffu, p[k].y, s));
        p[k] = fma2(sg2, p[k], o);
      }
    }
  }
}

constexpr int kFinChunk = 4096;  // group sums reduced per pass of the last CTA

// Pairwise FP64 tree over n strided values zero-padded to a power of two P >= 256, by the first
// 256 threads of the CTA (every thread calls it: it holds CTA barriers). Chunks of up to 4096 values are staged in shared memory; thread t reduces the
// aligned run [t*R, (t+1)*R) of its chunk (R = chunk/256 <= 16, zero-padded to 16, which leaves a
// power-of-two run's sum unchanged), the warps combine 32 runs, thread 0 combines the 8 warps and
// then, in order, the chunk sums with a stack of partial sums. Every addition is one of the
// halving tree S(lo,n) = S(lo,n/2) + S(lo+n/2,n/2). The result is valid in thread 0.
__device__ inline double cta_pairwise_f64(const double* p, int64_t stride, int64_t n, double* sbuf,
                                          double* swarp) {
  int64_t P = 256;
  while (P < n) P <<= 1;
  const int L = (int)(P < kFinChunk ? P : kFinChunk);
  const int R = L / 256;
  const int64_t nchunks = P / L;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool act = tid < 256;
  double stack[40];
  int sp = 0;
  for (int64_t b = 0; b < nchunks; ++b) {
    const int64_t lo = b * L;
    for (int i = tid; act && i < L; i += 256) {
      const int64_t idx = lo + i;
      sbuf[i] = (idx < n) ? __ldcg(p + idx * stride) : 0.0;
    }
    __syncthreads();
    double t[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) t[k] = (act && k < R) ? sbuf[tid * R + k] : 0.0;
#pragma unroll
    for (int len = 16; len > 1; len >>= 1) {
#pragma unroll
      for (int i = 0; i < len / 2; ++i) t[i] = __dadd_rn(t[2 * i], t[2 * i + 1]);
    }
    const double wsum = warp_pairwise_f64(t[0]);
    if (act && lane == 0) swarp[warp] = wsum;
    __syncthreads();
    if (tid == 0) {
      double u[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) u[k] = swarp[k];
#pragma unroll
      for (int len = 8; len > 1; len >>= 1) {
#pragma unroll
        for (int i = 0; i < len / 2; ++i) u[i] = __dadd_rn(u[2 * i], u[2 * i + 1]);
      }
      double x = u[0];
      for (int64_t k = b; k & 1; k >>= 1) x = __dadd_rn(stack[--sp], x);
      stack[sp++] = x;
    }
    __syncthreads();
  }
  return stack[0];
}

// The last CTA to finish reduces the group slots (FP64, the canonical halving tree over the groups
// zero-padded to a power of two), writes the statistics record or the module state and applies
// Purified Delta Refresh to the precision flag. Every thread of the CTA calls it (it holds CTA
// barriers); the first 256 threads do the work. s_fin: at least kFinChunk doubles of shared memory
// that nothing else uses any more.
template <int OP, bool REF>
__device__ void rows_finish(const RowArgs& a, int64_t ngroups, int prec, bool have_prev, double* s_fin) {
  constexpr int NST = (OP == OP_TDC) ? 2 : 3;
  constexpr int NW = 8;  // working warps
  __shared__ int s_last;
  __shared__ double s_fwarp[NW];
  __shared__ float s_fmax[NW][2];
  __shared__ int s_fnf[NW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool act = threadIdx.x < NW * 32;
  const int K = a.K;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t tk = atomicAdd(&a.hdr->ticket[OP == OP_TDC ? TICKET_TDC : TICKET_PREPASS], 1u);
    s_last = (tk == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int64_t G = ngroups;
  double S[NST];
  float mx = 0.0f, ar = 0.0f;
  int nf = 0;
  int64_t P = 256;
  while (P < G) P <<= 1;
  if (P <= 256 * 16) {
    // One pass over the group slots for every statistic and maximum: thread t owns the aligned
    // run [t R, (t + 1) R) of the zero-padded slots (R = P / 256 <= 16, padded to 16 with zeros),
    // then the warp trees and the tree of the 8 warp sums -- the same halving tree as
    // cta_pairwise_f64 with a single chunk.
    const int R = (int)(P / 256);
    double t3[NST][16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int64_t gi = (int64_t)threadIdx.x * R + k;
      const bool in = act && k < R && gi < G;
      const GroupSlot* gs = a.groups + (in ? gi : 0);
#pragma unroll
      for (int st = 0; st < NST; ++st) t3[st][k] = in ? __ldcg(&gs->s[st]) : 0.0;
      if (in) {
        mx = fmaxf(mx, __ldcg(&gs->max_abs));
        ar = fmaxf(ar, __ldcg(&gs->amax_rot));
        nf |= __ldcg(&gs->nonfinite);
      }
    }
    double* s_w3 = s_fin;  // [warp][statistic]
#pragma unroll
    for (int st = 0; st < NST; ++st) {
#pragma unroll
      for (int len = 16; len > 1; len >>= 1) {
#pragma unroll
        for (int i = 0; i < len / 2; ++i) t3[st][i] = __dadd_rn(t3[st][2 * i], t3[st][2 * i + 1]);
      }
      const double wsum = warp_pairwise_f64(t3[st][0]);
      if (act && lane == 0) s_w3[warp * NST + st] = wsum;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
#pragma unroll
      for (int st = 0; st < NST; ++st) {
        double u[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) u[w] = s_w3[w * NST + st];
#pragma unroll
        for (int len = 8; len > 1; len >>= 1) {
#pragma unroll
          for (int i = 0; i < len / 2; ++i) u[i] = __dadd_rn(u[2 * i], u[2 * i + 1]);
        }
        S[st] = u[0];
      }
    }
  } else {
#pragma unroll
    for (int st = 0; st < NST; ++st)
      S[st] = cta_pairwise_f64(&a.groups[0].s[st], sizeof(GroupSlot) / 8, G, s_fin, s_fwarp);
    for (int64_t gg = threadIdx.x; act && gg < G; gg += NW * 32) {
      const GroupSlot* gs = a.groups + gg;
      mx = fmaxf(mx, __ldcg(&gs->max_abs));
      ar = fmaxf(ar, __ldcg(&gs->amax_rot));
      nf |= __ldcg(&gs->nonfinite);
    }
  }
  mx = warp_max_f32(mx);
  ar = warp_max_f32(ar);
  nf = __any_sync(0xffffffffu, nf);
  if (act && lane == 0) {
    s_fmax[warp][0] = mx;
    s_fmax[warp][1] = ar;
    s_fnf[warp] = nf;
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  for (int w = 1; w < NW; ++w) {
    mx = fmaxf(mx, s_fmax[w][0]);
    ar = fmaxf(ar, s_fmax[w][1]);
    nf |= s_fnf[w];
  }
  const double inf = __longlong_as_double(0x7ff0000000000000ll);
  if (OP == OP_TDC) {
    sb_module_state* st = a.st;
    if (have_prev) st->delta = (S[1] == 0.0) ? inf : __ddiv_rn(S[0], S[1]);
    st->n_out += 1;
    st->acc = 0.0;
    st->last_skipped = 0;
    if (a.dsrc && a.dsrc->has_ref) {
      st->prev_d = a.dsrc->d;
      st->have_d = 1;
    } else {
      st->have_d = 0;
    }
    a.hdr->ticket[TICKET_TDC] = 0u;
  } else {
    const double numel = (double)a.M * (double)K;
    const double ratio = (S[0] == 0.0) ? inf : __ddiv_rn((double)mx, __ddiv_rn(S[0], numel));
    double d = 0.0;
    if (REF) {
      const double num = __dsqrt_rn(S[1]);
      const double den = __dsqrt_rn(S[2]);
      d = (den == 0.0) ? (num == 0.0 ? 0.0 : inf) : __ddiv_rn(num, den);
    }
    int pout = prec;
    if (OP == OP_PREPASS && !a.force_int8 && a.mode == SB_PREPASS_QUANT && a.force < 0 &&
        (prec == SB_NVFP4 || prec == SB_INT8) && ratio > a.rho)
      pout = SB_BF16;
    if (a.stats) {
      sb_stats* so = a.stats;
      so->sum_abs = S[0];
      so->sum_d2 = S[1];
      so->sum_ref2 = S[2];
      so->max_abs = (double)mx;
      so->amax_rot = (double)ar;
      so->ratio = ratio;
      so->d = d;
      so->numel = numel;
      so->has_ref = REF ? 1 : 0;
      so->prec_in = prec;
      so->prec_out = pout;
      so->nonfinite = nf;
    }
    if (pout != prec && a.prec) *a.prec = pout;
    if (nf) set_error(a.hdr, SB_ENONFINITE);
    a.hdr->ticket[TICKET_PREPASS] = 0u;
  }
  __threadfence();
}

__device__ __forceinline__ void team_sync(int team, int T) {
  if (T > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(T * 32) : "memory");
}

template <int T, int SPW, int OP, bool REF>
__global__ void __launch_bounds__(256) k_rows(RowArgs a, const __grid_constant__ RowMaps mp) {
  using RG = RowRing<SPW, OP, REF>;
  constexpr int NTEAM = kRowWarps / T;
  constexpr int NSEG = T * SPW;
  constexpr int NSEG2 = pow2_at_least(NSEG);
  // statistics per row; REC: |y|, (y - x)^2, x^2 of the difference statistic, then |y - c|, |c|
  constexpr int NST = (OP == OP_TDC) ? 2 : (OP == OP_REC ? 5 : 3);
  static_assert(RG::BYTES + 1024 <= 227 * 1024, "row ring exceeds shared memory");
  __shared__ float s_seg[NTEAM][2][NST][NSEG];  // team exchange (T > 1), by row parity
  __shared__ float s_wmax[NTEAM][2][T];        // per-warp rotated amax
  __shared__ float s_wraw[NTEAM][2][T];        // per-warp raw max |x|
  __shared__ float s_rowpart[2][NST][kG];      // by group parity
  __shared__ float s_rowamax[2][kG];
  __shared__ float s_rowmax[2][kG];
  __shared__ int s_rownf[2][kG];
  __shared__ uint64_t s_bar[kRowWarps][4];
  extern __shared__ uint8_t dsm_raw[];
  // dynamic shared memory: the rings (1024-byte aligned for the swizzled boxes); the last CTA
  // reuses it for the final reduction
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~(uintptr_t)1023);
  double* s_fin = reinterpret_cast<double*>(ring);
  static_assert(RG::BYTES >= kFinChunk * 8, "final-reduction buffer");

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int team = warp / T, wt = warp % T;

  int prec = -1;
  bool have_prev = true;
  bool do_stats = OP != OP_TDC, do_tdc = OP == OP_TDC;  // REC: each part keeps its own gate
  if (OP == OP_TDC) {
    if (a.st->skip) return;  // the module reuses its cache at this step
    have_prev = a.st->n_out >= 1;
  } else if (OP == OP_REC) {
    prec = a.prec ? *a.prec : -1;
    do_stats = prec != SB_SKIP;
    do_tdc = a.st->skip == 0;
    if (!do_stats && !do_tdc) return;
    have_prev = a.st->n_out >= 1;
  } else {
    prec = a.force_int8 ? SB_INT8 : (a.prec ? *a.prec : -1);
    if (prec == SB_SKIP) return;
  }
  const bool do_int8 = (OP == OP_PREPASS) && (a.force_int8 || (a.mode == SB_PREPASS_QUANT && prec == SB_INT8));
  const int K = a.K;
  const int64_t ngroups = ceil_div(a.M, kG);

  // A team walks its rows of the CTA's groups in order: row i = team + NTEAM * j (j < RPT) of
  // group g = blockIdx.x + n * gridDim.x. The difference statistic (OP_STATS) walks the groups from
  // the end of the tensor instead: its input is usually a GEMM output whose last rows were written
  // last and are still in L2, and the TDC record that follows it (forward) then finds the first
  // rows, which this pass read last. Returns false past the last group.
  constexpr int RPT = kG / NTEAM;
  auto row_of = [&](int64_t it, int64_t* g, int* i) -> bool {
    const int64_t g0 = blockIdx.x + (it / RPT) * (int64_t)gridDim.x;
    *g = (OP == OP_STATS) ? ngroups - 1 - g0 : g0;
    *i = team + (int)(it % RPT) * NTEAM;
    return g0 < ngroups;
  };
  // this warp's ring: slot s holds, per tensor t and segment c, the box of segment c*T + wt
  const uint32_t ring_w = smem_u32(ring) + (uint32_t)(warp * RG::D * RG::SLOT);
  const bool use_tma = a.tma != 0;
  auto issue_row = [&](int64_t it) {  // lane 0
    int64_t g;
    int i;
    if (!row_of(it, &g, &i)) return;
    const int m = (int)(g * kG + i);  // rows past M read as zero
    const int slot = (int)(it % RG::D);
    const uint32_t bar = smem_u32(&s_bar[warp][slot]);
    mbar_arrive_expect_tx_u32(bar, (uint32_t)RG::SLOT);
#pragma unroll
    for (int t = 0; t < RG::NT; ++t) {
#pragma unroll
      for (int c = 0; c < SPW; ++c)
        tma_load_3d(ring_w + (uint32_t)(slot * RG::SLOT + (t * SPW + c) * RG::SEG),
                    t == 0 ? &mp.x : (t == 1 ? &mp.r : &mp.c), bar, 0, (c * T + wt) * 16, m);
    }
  };
  int64_t bad_it = -1;  // last row whose wait gave up (its copy may still be in flight)
  if (use_tma) {
    if (lane == 0) {
#pragma unroll
      for (int d = 0; d < RG::D; ++d) mbar_init(&s_bar[warp][d], 1);
      fence_barrier_init();
      for (int d = 0; d < RG::D; ++d) issue_row(d);
    }
    __syncwarp();
  }

  for (int64_t it = 0;; ++it) {
    int64_t g;
    int i;
    if (!row_of(it, &g, &i)) break;
    const int gpar = (int)((it / RPT) & 1);
    const int rpar = (int)(it & 1);
    const bool group_end = (it % RPT) == RPT - 1;
    const int64_t m = g * kG + i;
    Raw32 xr[SPW], rr[SPW], cr[OP == OP_REC ? SPW : 1];
    if (use_tma) {
      // this row's slot: wait for its boxes, copy the lane's part to registers, refill the slot
      // with the row D steps ahead
      const int slot = (int)(it % RG::D);
      if (!mbar_wait_bounded(&s_bar[warp][slot], (uint32_t)((it / RG::D) & 1), nullptr, kRowWaitNs)) {
        if (lane == 0) set_error(a.hdr, SB_ETIMEOUT);
        bad_it = it;
      }
      const uint32_t sl = ring_w + (uint32_t)(slot * RG::SLOT);
#pragma unroll
      for (int c = 0; c < SPW; ++c) read_seg_sw128(xr[c], sl + (uint32_t)(c * RG::SEG), lane);
      if (RG::NT >= 2) {
#pragma unroll
        for (int c = 0; c < SPW; ++c) read_seg_sw128(rr[c], sl + (uint32_t)((SPW + c) * RG::SEG), lane);
      }
      if (OP == OP_REC) {
#pragma unroll
        for (int c = 0; c < SPW; ++c) read_seg_sw128(cr[c], sl + (uint32_t)((2 * SPW + c) * RG::SEG), lane);
      }
      __syncwarp();
      if (lane == 0) issue_row(it + RG::D);
      if (OP == OP_TDC && !have_prev) {  // no cached output yet: it reads as zero
#pragma unroll
        for (int c = 0; c < SPW; ++c) rr[c].q[0] = rr[c].q[1] = rr[c].q[2] = rr[c].q[3] = make_uint4(0, 0, 0, 0);
      }
      if (OP == OP_REC && !have_prev) {
#pragma unroll
        for (int c = 0; c < SPW; ++c) cr[c].q[0] = cr[c].q[1] = cr[c].q[2] = cr[c].q[3] = make_uint4(0, 0, 0, 0);
      }
    }
    if (m < a.M) {
      const __nv_bfloat16* xrow = a.X + m * K;
      __nv_bfloat16* rrow = (OP == OP_TDC || REF) ? a.R + m * K : nullptr;
      __nv_bfloat16* crow = (OP == OP_REC) ? a.C3 + m * K : nullptr;
      if (!use_tma) {
#pragma unroll
        for (int c = 0; c < SPW; ++c) {
          const int e0 = (c * T + wt) * 1024 + lane * 32;
          load_raw(xr[c], xrow, e0, K, true);
          if (OP == OP_TDC) load_raw_coherent(rr[c], rrow, e0, K, have_prev);
          else if (REF) load_raw(rr[c], rrow, e0, K, true);
          if (OP == OP_REC) load_raw_coherent(cr[c], crow, e0, K, have_prev);
        }
      }
      float seg[NST][SPW];
      float2 vr[OP == OP_PREPASS ? SPW : 1][16];
      float am = 0.0f, rawmax = 0.0f;
#pragma unroll
      for (int c = 0; c < SPW; ++c) {
        float2 p[16], t[16];
        unpack_pairs(xr[c], p);
        if (OP == OP_TDC) {
          float2 r[16];
          unpack_pairs(rr[c], r);
#pragma unroll
          for (int k = 0; k < 16; ++k) t[k] = abs2(sub2(p[k], r[k]));
          seg[0][c] = warp_pairwise_f32(tree_pairs(t));
#pragma unroll
          for (int k = 0; k < 16; ++k) t[k] = abs2(r[k]);
          seg[1][c] = warp_pairwise_f32(tree_pairs(t));
          const int e0 = (c * T + wt) * 1024 + lane * 32;
          if (a.update) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int e = e0 + 16 * h;
              if (e + 16 <= K && aligned32(rrow + e)) {
                stg_v8(rrow + e, xr[c].q[2 * h], xr[c].q[2 * h + 1]);
              } else {
                if (e < K) *reinterpret_cast<uint4*>(rrow + e) = xr[c].q[2 * h];
                if (e + 8 < K) *reinterpret_cast<uint4*>(rrow + e + 8) = xr[c].q[2 * h + 1];
              }
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            t[k] = abs2(p[k]);
            rawmax = max3(rawmax, t[k].x, t[k].y);
          }
          seg[0][c] = warp_pairwise_f32(tree_pairs(t));
          if (REF) {
            float2 r[16], t2[16];
            unpack_pairs(rr[c], r);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              t[k] = sq2(sub2(p[k], r[k]));
              t2[k] = sq2(r[k]);
            }
            seg[1][c] = warp_pairwise_f32(tree_pairs(t));
            seg[2][c] = warp_pairwise_f32(tree_pairs(t2));
          } else {
            seg[1][c] = 0.0f;
            seg[2][c] = 0.0f;
          }
          if (OP == OP_REC) {  // the TDC record's |y - c| and |c|, and the cache refresh
            float2 r[16];
            unpack_pairs(cr[c], r);
#pragma unroll
            for (int k = 0; k < 16; ++k) t[k] = abs2(sub2(p[k], r[k]));
            seg[NST == 5 ? 3 : 0][c] = warp_pairwise_f32(tree_pairs(t));
#pragma unroll
            for (int k = 0; k < 16; ++k) t[k] = abs2(r[k]);
            seg[NST == 5 ? 4 : 0][c] = warp_pairwise_f32(tree_pairs(t));
            const int e0 = (c * T + wt) * 1024 + lane * 32;
            if (do_tdc && a.update) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int e = e0 + 16 * h;
                if (e + 16 <= K && aligned32(crow + e)) {
                  stg_v8(crow + e, xr[c].q[2 * h], xr[c].q[2 * h + 1]);
                } else {
                  if (e < K) *reinterpret_cast<uint4*>(crow + e) = xr[c].q[2 * h];
                  if (e + 8 < K) *reinterpret_cast<uint4*>(crow + e + 8) = xr[c].q[2 * h + 1];
                }
              }
            }
          }
          if (OP == OP_PREPASS) {
            fwht_pairs(p, lane, a.B);
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              am = max3(am, fabsf(p[k].x), fabsf(p[k].y));
              vr[c][k] = p[k];
            }
          }
        }
      }
      // ---- combine the row across the team
      float part[NST];
      float a_m = 0.0f, rmax = 0.0f;
      if (OP == OP_PREPASS) am = warp_max_f32(am);
      if (OP != OP_TDC) rawmax = warp_max_f32(rawmax);
      if (T == 1) {
#pragma unroll
        for (int s = 0; s < NST; ++s) {
          float t[NSEG2];
#pragma unroll
          for (int k = 0; k < NSEG2; ++k) t[k] = (k < NSEG) ? seg[s][k] : 0.0f;
          part[s] = tree_n<NSEG2>(t);
        }
        a_m = am;
        rmax = rawmax;
      } else {
        if (lane == 0) {
#pragma unroll
          for (int s = 0; s < NST; ++s) {
#pragma unroll
            for (int c = 0; c < SPW; ++c) s_seg[team][rpar][s][c * T + wt] = seg[s][c];
          }
          s_wmax[team][rpar][wt] = am;
          s_wraw[team][rpar][wt] = rawmax;
        }
        team_sync(team, T);
#pragma unroll
        for (int s = 0; s < NST; ++s) {
          float t[NSEG2];
#pragma unroll
          for (int k = 0; k < NSEG2; ++k) t[k] = (k < NSEG) ? s_seg[team][rpar][s][k] : 0.0f;
          part[s] = tree_n<NSEG2>(t);
        }
#pragma unroll
        for (int w = 0; w < T; ++w) {
          a_m = fmaxf(a_m, s_wmax[team][rpar][w]);
          rmax = fmaxf(rmax, s_wraw[team][rpar][w]);
        }
      }
      if (wt == 0 && lane == 0) {
#pragma unroll
        for (int s = 0; s < NST; ++s) s_rowpart[gpar][s][i] = part[s];
        s_rowamax[gpar][i] = a_m;
        s_rowmax[gpar][i] = rmax;
        s_rownf[gpar][i] = (isnan(part[0]) || isinf(rmax)) ? 1 : 0;  // Inf or NaN in the row
      }
      // ---- per-token INT8 of the rotated row held in registers
      if (OP == OP_PREPASS && do_int8) {
        const float inv = (a_m == 0.0f) ? 0.0f : __fdiv_rn(127.0f, a_m);
#pragma unroll
        for (int c = 0; c < SPW; ++c) {
          const int e0 = (c * T + wt) * 1024 + lane * 32;
          if (e0 < K) {
            // q = rne(RN(y * inv)): FP32x2 product, then a round-to-nearest-even conversion
            const float2 inv2 = make_float2(inv, inv);
            float2 f[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) f[k] = mul2(vr[c][k], inv2);
            if (!(inv <= FLT_MAX)) {  // 127 / a_m overflowed: +-inf * y clamps to +-127, y = 0 gives 0
#pragma unroll
              for (int k = 0; k < 16; ++k) f[k] = make_float2(sign127(vr[c][k].x), sign127(vr[c][k].y));
            }
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {  // word i = elements 4i..4i+3 (x halves for i < 4)
              const int k0 = 4 * (i & 3);
              const bool hi = i >= 4;
              const uint32_t q0 = (uint32_t)__float2int_rn(hi ? f[k0].y : f[k0].x);
              const uint32_t q1 = (uint32_t)__float2int_rn(hi ? f[k0 + 1].y : f[k0 + 1].x);
              const uint32_t q2 = (uint32_t)__float2int_rn(hi ? f[k0 + 2].y : f[k0 + 2].x);
              const uint32_t q3 = (uint32_t)__float2int_rn(hi ? f[k0 + 3].y : f[k0 + 3].x);
              w[i] = __byte_perm(__byte_perm(q0, q1, 0x0040), __byte_perm(q2, q3, 0x0040), 0x5410);
            }
            int8_t* dst = a.q8 + m * K + e0;
            if (aligned32(dst)) {
              stg_v8(dst, make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]));
            } else {
              reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
              reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
          }
        }
        if (wt == 0 && lane == 0) a.s8[m] = (a_m == 0.0f) ? 0.0f : __fdiv_rn(a_m, 127.0f);
      }
    } else if (wt == 0 && lane == 0) {
#pragma unroll
      for (int s = 0; s < NST; ++s) s_rowpart[gpar][s][i] = 0.0f;
      s_rowamax[gpar][i] = 0.0f;
      s_rowmax[gpar][i] = 0.0f;
      s_rownf[gpar][i] = 0;
    }
    if (!group_end) continue;
    // ---- the group's FP64 partials
    __syncthreads();
    if (warp == 0) {
      const bool in = lane < kG;
      double gs[NST];
#pragma unroll
      for (int s = 0; s < NST; ++s) gs[s] = warp_pairwise_f64(in ? (double)s_rowpart[gpar][s][lane] : 0.0);
      const float gam = warp_max_f32(in ? s_rowamax[gpar][lane] : 0.0f);
      const float gmx = warp_max_f32(in ? s_rowmax[gpar][lane] : 0.0f);
      const int gnf = __any_sync(0xffffffffu, in ? s_rownf[gpar][lane] : 0);
      if (lane == 0) {
        GroupSlot* slot = a.groups + g;
#pragma unroll
        for (int s = 0; s < (NST < 3 ? NST : 3); ++s) slot->s[s] = gs[s];
        slot->max_abs = gmx;
        slot->amax_rot = gam;
        slot->nonfinite = gnf;
        if (OP == OP_REC) {
          GroupSlot* slot2 = a.groups2 + g;
          slot2->s[0] = gs[NST == 5 ? 3 : 0];
          slot2->s[1] = gs[NST == 5 ? 4 : 0];
          slot2->s[2] = 0.0;
          slot2->max_abs = 0.0f;
          slot2->amax_rot = 0.0f;
          slot2->nonfinite = 0;
        }
      }
    }
  }
  // a copy whose wait gave up may still be in flight: give it a bounded chance to land before the
  // ring is reused or the CTA exits
  if (use_tma && bad_it >= 0 && lane == 0)
    mbar_wait_bounded(&s_bar[warp][bad_it % RG::D], (uint32_t)((bad_it / RG::D) & 1), nullptr, kRowDrainNs);
  if (OP == OP_REC) {
    // the statistics record first: the TDC record takes its d (the last CTA of the second ticket
    // runs after every CTA has passed the first finish, which wrote the record)
    if (a.finish && do_stats) rows_finish<OP_STATS, true>(a, ngroups, prec, true, s_fin);
    if (a.finish && do_tdc) {
      RowArgs t = a;
      t.groups = a.groups2;
      t.dsrc = a.stats;
      rows_finish<OP_TDC, true>(t, ngroups, prec, have_prev, s_fin);
    }
  } else if (a.finish) {
    rows_finish<OP, REF>(a, ngroups, prec, have_prev, s_fin);
  }
}

// The final reduction alone, over group slots written by earlier launches (the shards of a
// token-sharded tensor, gathered): one CTA runs rows_finish over a.groups[0 .. ngroups).
template <int OP, bool REF>
__global__ void __launch_bounds__(256) k_finish(RowArgs a, int64_t ngroups) {
  __shared__ double s_fin[kFinChunk];
  int prec = -1;
  bool have_prev = true;
  if (OP == OP_TDC) {
    if (a.st->skip) return;
    have_prev = a.st->n_out >= 1;
  } else {
    prec = a.force_int8 ? SB_INT8 : (a.prec ? *a.prec : -1);
    if (prec == SB_SKIP) return;
  }
  rows_finish<OP, REF>(a, ngroups, prec, have_prev, s_fin);
}

// Team size T and segments per warp SPW for a row of K elements: T*SPW >= ceil(K/1024), SPW <= 3.
inline void pick_row_tiling(int K, int* T, int* SPW) {
  const int S = (K + 1023) / 1024;
  int t = 1;
  while ((S + t - 1) / t > 3 && t < 8) t <<= 1;
  *T = t;
  *SPW = (S + t - 1) / t;
}

template <int OP, bool REF>
cudaError_t launch_rows_t(const RowArgs& a, const RowMaps& mp, cudaStream_t s, int sms) {
  int T, SPW;
  pick_row_tiling(a.K, &T, &SPW);
  const int64_t ngroups = ceil_div(a.M, kG);
#define SB_ROWS_CASE(TT, SS)                                                                              \
  if (T == TT && SPW == SS) {                                                                             \
    constexpr int dsm = RowRing<SS, OP, REF>::BYTES + 1024;                                               \
    static std::atomic<uint64_t> attr{0}; /* one bit per device */                                      \
    const cudaError_t ae = smem_attr_once(k_rows<TT, SS, OP, REF>, dsm, attr);                            \
    if (ae != cudaSuccess) return ae;                                                                     \
    int occ = 0;                                                                                          \
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_rows<TT, SS, OP, REF>, kRowWarps * 32, dsm);   \
    if (occ <= 0) occ = 1;                                                                                \
    const int64_t cap = (int64_t)sms * occ; /* persistent: one wave of resident CTAs */                   \
    const unsigned grid = (unsigned)(ngroups < cap ? ngroups : cap);                                      \
    k_rows<TT, SS, OP, REF><<<grid, kRowWarps * 32, dsm, s>>>(a, mp);                                     \
    return cudaGetLastError();                                                                            \
  }
  SB_ROWS_CASE(1, 1)
  SB_ROWS_CASE(1, 2)
  SB_ROWS_CASE(1, 3)
  SB_ROWS_CASE(2, 2)
  SB_ROWS_CASE(2, 3)
  SB_ROWS_CASE(4, 2)
  SB_ROWS_CASE(4, 3)
  SB_ROWS_CASE(8, 2)
#undef SB_ROWS_CASE
  return cudaErrorInvalidValue;
}

// The fused record (OP_REC) rings three tensors per row; it takes the tiling of the other row
// kernels (with one row in flight per warp at SPW = 3).
inline void pick_rec_tiling(int K, int* T, int* SPW) { pick_row_tiling(K, T, SPW); }

inline cudaError_t launch_rows_rec(const RowArgs& a, const RowMaps& mp, cudaStream_t s, int sms) {
  int T, SPW;
  pick_rec_tiling(a.K, &T, &SPW);
  const int64_t ngroups = ceil_div(a.M, kG);
#define SB_REC_CASE(TT, SS)                                                                               \
  if (T == TT && SPW == SS) {                                                                             \
    constexpr int dsm = RowRing<SS, OP_REC, true>::BYTES + 1024;                                          \
    static std::atomic<uint64_t> attr{0};                                                                 \
    const cudaError_t ae = smem_attr_once(k_rows<TT, SS, OP_REC, true>, dsm, attr);                       \
    if (ae != cudaSuccess) return ae;                                                                     \
    int occ = 0;                                                                                          \
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_rows<TT, SS, OP_REC, true>, kRowWarps * 32, dsm); \
    if (occ <= 0) occ = 1;                                                                                \
    const int64_t cap = (int64_t)sms * occ;                                                               \
    const unsigned grid = (unsigned)(ngroups < cap ? ngroups : cap);                                      \
    k_rows<TT, SS, OP_REC, true><<<grid, kRowWarps * 32, dsm, s>>>(a, mp);                                \
    return cudaGetLastError();                                                                            \
  }
  SB_REC_CASE(1, 1)
  SB_REC_CASE(1, 2)
  SB_REC_CASE(1, 3)
  SB_REC_CASE(2, 2)
  SB_REC_CASE(2, 3)
  SB_REC_CASE(4, 2)
  SB_REC_CASE(4, 3)
  SB_REC_CASE(8, 2)
#undef SB_REC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sb
