// prepass_blk.cuh -- the pre-pass with one 128-channel Hadamard block per lane.
//
// It computes what k_rows<.., OP_PREPASS, false> computes -- the block FWHT of every token, the
// raw statistics (sum |x| in the canonical pairwise order, max |x|), the per-token rotated amax,
// the per-token INT8 codes when the layer runs in INT8, the group slots and, in the last CTA, the
// statistics record and the Purified Delta Refresh verdict ("write-up" sections 一, 三, 四) -- for
// Hadamard blocks of B <= 128 channels and rows of K = 128 NB channels.
//
// Layout: a lane owns one whole 128-element block, so all butterfly stages run inside its
// registers and no value crosses lanes. Its 128 values live as 64 packed pairs
// P[k] = (v[k], v[k + 64]): FP32x2 arithmetic covers the stages h = 1..32, the stage h = 64 pairs
// the two halves of each P[k]. Lanes 4..7 of every eight hold the halves the other way round,
// P[k] = (v[k + 64], v[k]) (see pb_load_block); every step but the stage h = 64 and the final
// stores treats the two halves alike.
//
// Teams: T warps (T | 12) own R rows at a time (R | kG), their R NB blocks laid out flat over the
// team's 32 T lanes (a row may straddle warps; idle lanes compute on whatever the box holds and
// write nothing). Row maxima go through shared-memory atomics, sums of aligned runs of blocks
// through a shared buffer that one warp of the team (rotating) folds into row sums. In the INT8
// pass the team meets once per task at a named barrier, since every lane needs its row's amax;
// in a statistics-only pass only the folding warp waits for the others (mbarriers). A team walks
// whole groups of kG rows and writes each group's FP64 slot itself; the last CTA finishes as
// k_rows does.
//
// Loads: every warp keeps a ring of kPbD slots, each one TMA box of 32 consecutive blocks (8 KB,
// 128B swizzle); a slot is refilled at the start of the task after the one that read it, so one
// load is always in flight while a task computes.
#pragma once

#include <type_traits>

#include "rows.cuh"

namespace sb {

constexpr int kPbWarps = 12;
constexpr int kPbThreads = kPbWarps * 32;
constexpr int kPbSlot = 8192;                        // 32 blocks of 128 bf16
constexpr int kPbD = 2;                              // ring slots per warp
constexpr int kPbRing = kPbWarps * kPbD * kPbSlot;  // 192 KB
constexpr int kPbSumPerWarp = 64;                    // block-sum floats per team warp (R NB2 < 64 T)
constexpr int kPbMaxNB = 32 * kPbWarps;              // blocks per row (K <= 49152)

struct PbGeom {
  int NB;   // blocks per row
  int NB2;  // NB rounded up to a power of two (the row tree's padding)
  int T;    // warps per team
  int R;    // rows per task
  int SUB;  // largest power of two <= 32 dividing NB: aligned runs of SUB blocks of a row sit on
            // aligned lane groups of one warp, so each warp sums them before the team meets
};

// Team shape for rows of NB blocks: T | 12, R | kG, R NB <= 32 T; the most busy lanes, then the
// fewest warps per team, then the most rows per task. False when no shape fits.
inline bool pick_pb_geom(int NB, PbGeom* g) {
  if (NB < 1 || NB > kPbMaxNB) return false;
  static const int kTs[] = {1, 2, 3, 4, 6, 12};
  double best = 0.0;
  for (int T : kTs) {
    for (int R = kG; R >= 1; R >>= 1) {
      if (R * NB > 32 * T) continue;
      const double eff = (double)(R * NB) / (32.0 * T);
      if (eff > best + 1e-12) {
        best = eff;
        g->T = T;
        g->R = R;
      }
      break;  // the largest R that fits is the best for this T
    }
  }
  if (best <= 0.0) return false;
  g->NB = NB;
  int p = 1;
  while (p < NB) p <<= 1;
  g->NB2 = p;
  g->SUB = 1;
  while (g->SUB < 32 && NB % (2 * g->SUB) == 0) g->SUB <<= 1;
  return true;
}

// The lane's 128 values from its two swizzled half blocks in the slot: half block r = 2 lane + h
// holds elements 64 h .. 64 h + 63; its 16-byte chunk c sits at chunk position c ^ (r & 7).
// Lanes with swp = 1 (lanes 4..7 of every eight) read their upper half first, so the eight lanes
// of each 128-bit load phase touch half blocks with eight different (r & 7): no bank conflicts.
// Their pairs come out as (v[k + 64], v[k]).
__device__ __forceinline__ uint32_t pb_swap(int lane) { return ((uint32_t)lane >> 2) & 1u; }

__device__ __forceinline__ void pb_load_block(uint32_t slot, int lane, float2 (&P)[64]) {
  const uint32_t swp = pb_swap(lane);
  const uint32_t r0 = 2u * (uint32_t)lane + swp, r1 = 2u * (uint32_t)lane + 1u - swp;
  const uint32_t b0 = slot + 128u * r0, b1 = slot + 128u * r1;
  const uint32_t sw0 = r0 & 7u, sw1 = r1 & 7u;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 u0 = ld_shared_v4(b0 + 16u * ((uint32_t)c ^ sw0));
    const uint4 u1 = ld_shared_v4(b1 + 16u * ((uint32_t)c ^ sw1));
    const uint32_t w0[4] = {u0.x, u0.y, u0.z, u0.w};
    const uint32_t w1[4] = {u1.x, u1.y, u1.z, u1.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // word i of chunk c = elements 8c + 2i (low half), 8c + 2i + 1
      P[8 * c + 2 * i] = make_float2(__uint_as_float(w0[i] << 16), __uint_as_float(w1[i] << 16));
      P[8 * c + 2 * i + 1] = make_float2(__uint_as_float(w0[i] & 0xffff0000u), __uint_as_float(w1[i] & 0xffff0000u));
    }
  }
}

__device__ __forceinline__ float2 abs_max2(float2 a, float2 b) {
  return make_float2(fmaxf(fabsf(a.x), fabsf(b.x)), fmaxf(fabsf(a.y), fabsf(b.y)));
}

// Stage h = 1 of the block FWHT fused with the raw statistics of the block: max |x| and the
// canonical pairwise sum of |x| over its 128 elements. For a butterfly pair (a, b),
// max(|a + b|, |a - b|) equals the correctly rounded |a| + |b| -- the tree's first addition -- so
// that level costs one max per pair instead of two absolute values and an add.
__device__ __forceinline__ float pb_stage1_raw(float2 (&P)[64], float* rmax) {
  float2 c8[8];
  float mx[2] = {0.0f, 0.0f};  // two independent chains (max is exact in any order)
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float2 l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int k = 8 * c + 2 * u;
      const float2 a = P[k], b = P[k + 1];
      mx[u & 1] = max3(mx[u & 1], fabsf(a.x), fabsf(b.x));
      mx[u & 1] = max3(mx[u & 1], fabsf(a.y), fabsf(b.y));
      P[k] = add2(a, b);
      P[k + 1] = sub2(a, b);
      l[u] = abs_max2(P[k], P[k + 1]);  // elements 8c + 2u, +1 of each half
    }
    c8[c] = add2(add2(l[0], l[1]), add2(l[2], l[3]));  // 8 elements of each half
  }
  const float2 s16a = add2(c8[0], c8[1]), s16b = add2(c8[2], c8[3]);
  const float2 s16c = add2(c8[4], c8[5]), s16d = add2(c8[6], c8[7]);
  const float2 s64 = add2(add2(s16a, s16b), add2(s16c, s16d));  // each half: 64 elements
  *rmax = fmaxf(mx[0], mx[1]);
  return __fadd_rn(s64.x, s64.y);
}

// Stages h = 2 .. 64 (each while h < B) and the block's rotated amax. B is a template argument:
// stages chosen at run time would force the compiler to reconcile the pairs' registers at every
// join and spill. The stage h = 64 adds and subtracts the halves of each pair as one fused
// multiply-add by +-1 each (exact product, one rounding): (x + y, x - y) for a pair (lower, upper)
// and (y - x, y + x) for a swapped pair (upper, lower) -- the same two results in swapped places.
// Without Y (the rotated values are not needed, only their amax) that stage is not formed: the
// larger magnitude of RN(x + y) and RN(x - y) is RN(|x| + |y|) (rounding is monotone and
// symmetric), NaN and infinities included, so a pair costs one add.
template <int B, bool Y = true>
__device__ __forceinline__ float pb_stages_rest(float2 (&P)[64], float cx) {  // cx = -1: swapped pairs
#pragma unroll
  for (int h = 2; h <= 32; h <<= 1) {
    if (h < B) {
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        if ((k & h) == 0) {
          const float2 x = P[k], y = P[k + h];
          P[k] = add2(x, y);
          P[k + h] = sub2(x, y);
        }
      }
    }
  }
  float am[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four independent chains
  if (64 < B && !Y) {
#pragma unroll
    for (int k = 0; k < 64; k += 2) {
      const float t0 = __fadd_rn(fabsf(P[k].x), fabsf(P[k].y)), t1 = __fadd_rn(fabsf(P[k + 1].x), fabsf(P[k + 1].y));
      am[(k >> 1) & 3] = max3(am[(k >> 1) & 3], t0, t1);
    }
  } else if (64 < B) {
    const float cy = -cx;
#pragma unroll
    for (int k = 0; k < 64; ++k) {
      const float s = __fmaf_rn(cx, P[k].x, P[k].y), d = __fmaf_rn(cy, P[k].y, P[k].x);
      P[k] = make_float2(s, d);
      am[k & 3] = max3(am[k & 3], fabsf(s), fabsf(d));
    }
  } else {
#pragma unroll
    for (int k = 0; k < 64; ++k) am[k & 3] = max3(am[k & 3], fabsf(P[k].x), fabsf(P[k].y));
  }
  return fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
}

// Per-token INT8 codes of the lane's rotated block, q = rne(RN(y * inv)) with inv = RN(127 / a_m),
// clamped to +-127, stored at dst (128 bytes). When 127 / a_m overflows (a_m below 127 / FLT_MAX)
// the product is +-inf for every nonzero y and the clamp gives +-127; y = 0 gives 0. The codes go
// out in two halves (pairs P[0..31], then P[32..63]) so that few words are live at a time. The
// rounding stays a float-to-integer conversion: the cheaper RN(v + 1.5 2^23) needs the product
// and the addition rounded apart, and the compiler fuses an FP32x2 multiply with the FP32x2 add
// that consumes it (measured: codes off by one against the oracle).
__device__ __forceinline__ uint32_t pb_pack4(float a, float b, float c, float d) {
  const uint32_t q0 = (uint32_t)__float2int_rn(a), q1 = (uint32_t)__float2int_rn(b);
  const uint32_t q2 = (uint32_t)__float2int_rn(c), q3 = (uint32_t)__float2int_rn(d);
  return __byte_perm(__byte_perm(q0, q1, 0x0040), __byte_perm(q2, q3, 0x0040), 0x5410);
}

__device__ __forceinline__ uint32_t pb_sign_code(float v) { return v > 0.0f ? 127u : (v < 0.0f ? 0x81u : 0u); }

__device__ __forceinline__ void pb_store_int8(float2 (&P)[64], float a_m, int8_t* dst, int lane) {
  const float inv = (a_m == 0.0f) ? 0.0f : __fdiv_rn(127.0f, a_m);
  const int64_t ox = pb_swap(lane) ? 64 : 0, oy = 64 - ox;  // where the x and y halves go
  const bool finite = inv <= FLT_MAX;
  const float2 inv2 = make_float2(inv, inv);
#pragma unroll
  for (int i = 0; i < 16; i += 4) {  // pairs P[4i .. 4i + 15]: elements 4i.. (x halves) and 64 + 4i.. (y)
    uint32_t wx[4], wy[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int k = 4 * (i + v);
      if (finite) {
        float2 f[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) f[u] = mul2(P[k + u], inv2);
        wx[v] = pb_pack4(f[0].x, f[1].x, f[2].x, f[3].x);
        wy[v] = pb_pack4(f[0].y, f[1].y, f[2].y, f[3].y);
      } else {
        uint32_t x = 0, y = 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          x |= pb_sign_code(P[k + u].x) << (8 * u);
          y |= pb_sign_code(P[k + u].y) << (8 * u);
        }
        wx[v] = x;
        wy[v] = y;
      }
    }
    *reinterpret_cast<uint4*>(dst + ox + 4 * i) = make_uint4(wx[0], wx[1], wx[2], wx[3]);
    *reinterpret_cast<uint4*>(dst + oy + 4 * i) = make_uint4(wy[0], wy[1], wy[2], wy[3]);
  }
}

__device__ __forceinline__ void pb_team_sync(int team, int T) {
  if (T > 1)
    asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(T * 32) : "memory");
  else
    __syncwarp();
}

// Pairwise tree of the C values at p (C a power of two <= 16).
template <int C>
__device__ __forceinline__ float pb_run_sum(const float* p) {
  float t[C];
#pragma unroll
  for (int i = 0; i < C; ++i) t[i] = p[i];
  return tree_n<C>(t);
}

template <int B>
__global__ void __launch_bounds__(kPbThreads, 1) k_prepass_blk(RowArgs a, PbGeom gm, const __grid_constant__ CUtensorMap mx) {
  extern __shared__ uint8_t pb_dsm[];
  __shared__ uint64_t s_bar[kPbWarps][kPbD];
  __shared__ float s_bsum[2][kPbWarps * kPbSumPerWarp];  // block sums by task parity, team regions
  __shared__ uint32_t s_ram[3][kPbWarps][kG];              // row rotated amax (float bits), 3 tasks
  __shared__ uint32_t s_rmx[3][kPbWarps][kG];              // row raw max |x|
  __shared__ float s_gsum[kPbWarps][kG];                   // per row of the current group
  __shared__ float s_gam[kPbWarps][kG];
  __shared__ float s_grm[kPbWarps][kG];
  __shared__ uint64_t s_full[kPbWarps][2];   // statistics-only pass: the team's task buffers
  __shared__ uint64_t s_empty[kPbWarps][2];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pb_dsm) + 1023) & ~(uintptr_t)1023);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int T = gm.T, R = gm.R, NB = gm.NB, NB2 = gm.NB2;
  const int team = warp / T, wt = warp - team * T;
  const int nteam = kPbWarps / T;

  const int prec = a.force_int8 ? SB_INT8 : (a.prec ? *a.prec : -1);
  if (prec == SB_SKIP) return;
  const bool do_int8 = a.force_int8 || (a.mode == SB_PREPASS_QUANT && prec == SB_INT8);
  const int G = (int)ceil_div(a.M, kG);  // M <= 2^30
  const int TPG = kG / R;                 // tasks per group
  const int gteam = team * (int)gridDim.x + (int)blockIdx.x;  // consecutive groups on different CTAs
  const int nteams = (int)gridDim.x * nteam;

  // this lane's block of every task: flat index q of the team's R NB blocks
  const int q = wt * 32 + lane;
  const bool qv = q < R * NB;
  const int rl = qv ? q / NB : R;  // row within the task (R: idle lane)
  const int blk = q - (q / NB) * NB;
  const unsigned rowmask = __match_any_sync(0xffffffffu, rl);
  const bool leader = (__ffs(rowmask) - 1) == lane;
  const int sbase = team * T * kPbSumPerWarp;

  for (int i = threadIdx.x; i < 2 * kPbWarps * kPbSumPerWarp; i += kPbThreads) (&s_bsum[0][0])[i] = 0.0f;
  for (int i = threadIdx.x; i < 3 * kPbWarps * kG; i += kPbThreads) {
    (&s_ram[0][0][0])[i] = 0u;
    (&s_rmx[0][0][0])[i] = 0u;
  }

  const uint32_t ring_w = smem_u32(ring) + (uint32_t)(warp * kPbD * kPbSlot);
  // task (g, j): rows g kG + j R .. + R - 1; the team's tasks run j = 0..TPG-1 over its groups
  // g = gteam, gteam + nteams, ...
  auto issue = [&](int g, int j, int slot) {  // lane 0
    if (g >= G) return;
    const int m0 = g * kG + j * R;
    const uint32_t bar = smem_u32(&s_bar[warp][slot]);
    mbar_arrive_expect_tx_u32(bar, (uint32_t)kPbSlot);
    tma_load_2d_u32(ring_w + (uint32_t)(slot * kPbSlot), &mx, bar, 0, 2 * (m0 * NB + 32 * wt));
  };
  if (lane == 0) {
#pragma unroll
    for (int d = 0; d < kPbD; ++d) mbar_init(&s_bar[warp][d], 1);
    if (wt == 0) {
      mbar_init(&s_full[team][0], (uint32_t)T);
      mbar_init(&s_full[team][1], (uint32_t)T);
      mbar_init(&s_empty[team][0], 1);
      mbar_init(&s_empty[team][1], 1);
    }
    fence_barrier_init();
  }
  __syncthreads();  // zeroed buffers and initialised barriers
  if (lane == 0) {
    issue(gteam, 0, 0);
    issue(TPG == 1 ? gteam + nteams : gteam, TPG == 1 ? 0 : 1, 1);
  }
  __syncwarp();
  static_assert(kPbD == 2, "ring of two slots");

  const int SUB = gm.SUB, NBS = NB2 / SUB;  // per row: NBS aligned run sums (zero-padded)
  int bad_it = -1;
  auto bounded = [&](uint64_t* bar, uint32_t parity, int it) {
    if (!mbar_wait_bounded(bar, parity, nullptr, kRowWaitNs)) {
      if (lane == 0) set_error(a.hdr, SB_ETIMEOUT);
      bad_it = it;
    }
  };
  // Q: the INT8 pass. Every lane needs its row's amax before it quantizes, so the team meets at a
  // named barrier each task, and the maxima are triple-buffered. Otherwise (statistics only) just
  // the warp that folds the task's rows waits for the others: every warp arrives on
  // s_full[team][t & 1] and goes on; the folding warp waits there, folds, clears the task's
  // buffers and arrives on s_empty[team][t & 1]; a warp waits on s_empty only before it writes the
  // buffers again two tasks later.
  auto run = [&](auto qtag) {
    constexpr bool Q = decltype(qtag)::value;
    int g = gteam, j = 0, tb = 0, dw = 0;  // group, task in group, maxima buffer (Q), folding warp
    for (int it = 0; g < G; ++it) {
      const int m0 = g * kG + j * R;
      const int slot = it & 1, pb = it & 1;
      const int ab = Q ? tb : pb;  // maxima buffer of this task
      const int jn = (j + 1 == TPG) ? 0 : j + 1, gn = (j + 1 == TPG) ? g + nteams : g;  // next task
      // the slot of the previous task was read into registers (and used) there: refill it with the
      // task after this one
      if (lane == 0 && it > 0) issue(gn, jn, slot ^ 1);
      bounded(&s_bar[warp][slot], (uint32_t)((it >> 1) & 1), it);
      float2 P[64];
      pb_load_block(ring_w + (uint32_t)(slot * kPbSlot), lane, P);

      float rmax;
      const float bsum = pb_stage1_raw(P, &rmax);
      const float am = pb_stages_rest<B, Q>(P, pb_swap(lane) ? -1.0f : 1.0f);  // Q: the codes need y

      // ---- row maxima and sums of aligned runs of SUB blocks, then the team meets
      if (!Q && it >= 2) bounded(&s_empty[team][pb], (uint32_t)(((it >> 1) & 1) ^ 1), it);
      const uint32_t amb = __reduce_max_sync(rowmask, __float_as_uint(am));
      const uint32_t rmb = __reduce_max_sync(rowmask, __float_as_uint(rmax));
      if (qv && leader) {
        atomicMax(&s_ram[ab][team][rl], amb);
        atomicMax(&s_rmx[ab][team][rl], rmb);
      }
      float run = bsum;
      for (int sh = 1; sh < SUB; sh <<= 1) run = __fadd_rn(run, __shfl_xor_sync(0xffffffffu, run, sh));
      if (qv && (blk & (SUB - 1)) == 0) s_bsum[pb][sbase + rl * NBS + blk / SUB] = run;
      if (Q) {
        pb_team_sync(team, T);
        const int m = m0 + rl;
        if (qv && m < a.M)
          pb_store_int8(P, __uint_as_float(s_ram[ab][team][rl]), a.q8 + ((int64_t)m * NB + blk) * 128, lane);
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_full[team][pb]);
      }

      // ---- one warp of the team: row sums, the task's rows into the group, the group's slot
      if (wt == dw) {
        if (!Q) bounded(&s_full[team][pb], (uint32_t)((it >> 1) & 1), it);
        const int n = R * NBS;
        const int c = n >= 32 ? n / 32 : 1;
        const float* bs = &s_bsum[pb][sbase + lane * c];
        float v;
        if (c == 1) v = (lane < n) ? bs[0] : 0.0f;
        else if (c == 2) v = pb_run_sum<2>(bs);
        else if (c == 4) v = pb_run_sum<4>(bs);
        else if (c == 8) v = pb_run_sum<8>(bs);
        else v = pb_run_sum<16>(bs);
        const int span = NBS / c;  // lanes per row
        for (int s = 1; s < span; s <<= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, s));
        const int r = lane / span;
        if ((lane & (span - 1)) == 0 && r < R) {
          const int gi = j * R + r;
          const float a_m = __uint_as_float(s_ram[ab][team][r]);
          s_gsum[team][gi] = v;
          s_gam[team][gi] = a_m;
          s_grm[team][gi] = __uint_as_float(s_rmx[ab][team][r]);
          if (Q && m0 + r < a.M) a.s8[m0 + r] = (a_m == 0.0f) ? 0.0f : __fdiv_rn(a_m, 127.0f);
        }
        // the maxima buffer used next starts from zero: Q, the one two tasks ahead (the others
        // have read this task's already); otherwise this task's own, read above
        if (!Q) __syncwarp();
        if (lane < R) {
          const int tz = Q ? (tb == 0 ? 2 : tb - 1) : ab;
          s_ram[tz][team][lane] = 0u;
          s_rmx[tz][team][lane] = 0u;
        }
        if (j == TPG - 1) {
          __syncwarp();
          const bool in = lane < kG;
          const float rs = in ? s_gsum[team][lane] : 0.0f;
          const double gs = warp_pairwise_f64((double)rs);
          const float gam = warp_max_f32(in ? s_gam[team][lane] : 0.0f);
          const float rm = in ? s_grm[team][lane] : 0.0f;
          const float gmx = warp_max_f32(rm);
          // non-finite input: an infinite |x| makes the row max infinite, a NaN makes the row sum
          // NaN (a finite row whose sum overflows to +inf is not flagged)
          const int gnf = __any_sync(0xffffffffu, isnan(rs) || isinf(rm));
          if (lane == 0) {
            GroupSlot* gsl = a.groups + g;
            gsl->s[0] = gs;
            gsl->s[1] = 0.0;
            gsl->s[2] = 0.0;
            gsl->max_abs = gmx;
            gsl->amax_rot = gam;
            gsl->nonfinite = gnf;
          }
        }
        if (!Q) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_empty[team][pb]);
        }
      }
      g = gn;
      j = jn;
      tb = tb == 2 ? 0 : tb + 1;
      dw = dw + 1 == T ? 0 : dw + 1;
    }
  };
  if (do_int8)
    run(std::true_type{});
  else
    run(std::false_type{});
  if (bad_it >= 0 && lane == 0)
    mbar_wait_bounded(&s_bar[warp][bad_it & 1], (uint32_t)((bad_it >> 1) & 1), nullptr, kRowDrainNs);
  if (a.finish) rows_finish<OP_PREPASS, false>(a, G, prec, true, reinterpret_cast<double*>(ring));
}

}  // namespace sb
