// chunks.cu -- the pre-pass of a tensor whose per-chunk statistics are already known.
//
// The second linear layer of an FFN reads the tensor the first one wrote. If that layer's
// producer also hands over, for every aligned 128-channel chunk of every row, the chunk's rotated
// amax, its canonical pairwise sum of |x| and its max |x|, the pre-pass no longer needs a
// statistics pass over the tensor: the records fold into the row statistics (a chunk is an
// aligned subtree of its row's sum tree), the group slots and, in the last CTA, the statistics
// record and the Purified Delta Refresh verdict ("write-up" sections 一, 三, 四). Only the
// quantization pass reads the tensor: the NVFP4 encode as in sb_prepass, or a streaming INT8
// pass that knows every row's amax in advance and so needs no team of warps per row.
//
//  k_fold_chunks   one warp per 16-row group, a lane per row: the tree over the chunk sums and
//                  the chunk maxima; INT8 scales; the group's FP64 slot; rows_finish in the last CTA.
//                  The row's rotated amax is left in the fourth float of its first record.
//  k_int8_blk      INT8 codes, one 128-channel block per lane (as the NVFP4 encode).
#include "launch_util.h"
#include "prepass_blk.cuh"
#include "tmap.h"

namespace sb {

constexpr int kFoldWarps = 8;

// Canonical pairwise tree over 16 values whose tail is zero.
__device__ __forceinline__ float tree16(float (&t)[16]) {
#pragma unroll
  for (int len = 16; len > 1; len >>= 1) {
#pragma unroll
    for (int i = 0; i < len / 2; ++i) t[i] = __fadd_rn(t[2 * i], t[2 * i + 1]);
  }
  return t[0];
}


__global__ void __launch_bounds__(kFoldWarps * 32) k_fold_chunks(RowArgs a, float4* chunks, int NB) {
  __shared__ double s_fin[kFinChunk];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int prec = a.prec ? *a.prec : -1;
  if (prec == SB_SKIP) return;
  const bool do_int8 = a.mode == SB_PREPASS_QUANT && prec == SB_INT8;
  const int64_t G = ceil_div(a.M, kG);
  for (int64_t g = (int64_t)blockIdx.x * kFoldWarps + warp; g < G; g += (int64_t)gridDim.x * kFoldWarps) {
    // lane i < kG: row i of the group, its chunks read in order
    const int64_t m = g * kG + lane;
    const bool row = lane < kG && m < a.M;
    const float4* rc = chunks + (row ? m : 0) * NB;
    // the row's tree in two levels: aligned runs of 8 chunks in registers, then the 16 run sums
    float runs[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) runs[k] = 0.0f;
    float ram = 0.0f, rmx = 0.0f;
    if (row) {
#pragma unroll 4
      for (int b0 = 0; b0 < NB; b0 += 8) {  // several runs' loads in flight at once
        float t[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          t[u] = 0.0f;
          if (b0 + u < NB) {
            const float4 r = rc[b0 + u];
            t[u] = r.y;
            ram = fmaxf(ram, r.x);
            rmx = fmaxf(rmx, r.z);
          }
        }
        const float s8 = __fadd_rn(__fadd_rn(__fadd_rn(t[0], t[1]), __fadd_rn(t[2], t[3])),
                                   __fadd_rn(__fadd_rn(t[4], t[5]), __fadd_rn(t[6], t[7])));
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (k == (b0 >> 3)) runs[k] = s8;  // a register per run: no indexed local array
      }
    }
    const float rs = tree16(runs);
    if (row) {
      chunks[m * NB].w = ram;
      if (do_int8) a.s8[m] = (ram == 0.0f) ? 0.0f : __fdiv_rn(ram, 127.0f);
    }
    const bool in = lane < kG;
    const double gs = warp_pairwise_f64(in ? (double)rs : 0.0);
    const float gam = warp_max_f32(in ? ram : 0.0f);
    const float gmx = warp_max_f32(in ? rmx : 0.0f);
    const int gnf = __any_sync(0xffffffffu, in && (isnan(rs) || isinf(rmx)));  // Inf or NaN in a row
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
  rows_finish<OP_PREPASS, false>(a, G, prec, true, s_fin);
}

// INT8 codes of the rows, with every row's amax known: a warp streams 32 consecutive blocks per
// task through a two-slot TMA ring, a lane rotates its block and writes its 128 codes. Written
// when the flag said INT8 when the pre-pass began (stats->prec_in), as sb_prepass writes them.
template <int B>
__global__ void __launch_bounds__(kPbThreads, 1) k_int8_blk(RowArgs a, const float4* chunks, int NB,
                                                           const __grid_constant__ CUtensorMap mx) {
  extern __shared__ uint8_t pb_dsm[];
  __shared__ uint64_t s_bar[kPbWarps][kPbD];
  const int p = a.prec ? *a.prec : -1;
  if (p == SB_SKIP || a.mode != SB_PREPASS_QUANT || a.stats->prec_in != SB_INT8) return;
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pb_dsm) + 1023) & ~(uintptr_t)1023);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t nblk = a.M * NB;
  const int ntask = (int)ceil_div(nblk, 32);
  const int nw = (int)gridDim.x * kPbWarps;
  const uint32_t ring_w = smem_u32(ring) + (uint32_t)(warp * kPbD * kPbSlot);
  auto issue = [&](int t, int slot) {  // lane 0
    if (t >= ntask) return;
    const uint32_t bar = smem_u32(&s_bar[warp][slot]);
    mbar_arrive_expect_tx_u32(bar, (uint32_t)kPbSlot);
    tma_load_2d_u32(ring_w + (uint32_t)(slot * kPbSlot), &mx, bar, 0, 64 * t);
  };
  const int t0 = (int)blockIdx.x * kPbWarps + warp;
  if (lane == 0) {
    mbar_init(&s_bar[warp][0], 1);
    mbar_init(&s_bar[warp][1], 1);
    fence_barrier_init();
    issue(t0, 0);
    issue(t0 + nw, 1);
  }
  __syncwarp();
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
    const int64_t f = (int64_t)t * 32 + lane;
    if (f >= nblk) continue;
    const int64_t m = f / NB;
    pb_store_int8(P, chunks[m * NB].w, a.q8 + f * 128, lane);
  }
  if (bad_it >= 0 && lane == 0)
    mbar_wait_bounded(&s_bar[warp][bad_it & 1], (uint32_t)((bad_it >> 1) & 1), nullptr, kRowDrainNs);
}

static int chunks_sms() { return device_sm_count(); }

template <int B>
static cudaError_t launch_int8_blk(const RowArgs& a, const float4* chunks, int NB, const CUtensorMap& mx,
                                   cudaStream_t s) {
  constexpr int dsm = kPbRing + 1024;
  static std::atomic<uint64_t> attr{0};  // per instantiation, one bit per device
  const cudaError_t e = smem_attr_once(k_int8_blk<B>, dsm, attr);
  if (e != cudaSuccess) return e;
  const int64_t want = ceil_div(ceil_div(a.M * NB, 32), kPbWarps);
  const int sms = chunks_sms();
  const unsigned grid = (unsigned)(want < sms ? want : sms);
  k_int8_blk<B><<<grid, kPbThreads, dsm, s>>>(a, chunks, NB, mx);
  return cudaGetLastError();
}

cudaError_t launch_prepass_chunks(const PrepassLaunch& p, float* chunks, cudaStream_t s) {
  RowArgs a{};
  a.X = reinterpret_cast<const __nv_bfloat16*>(p.X);
  a.M = p.M;
  a.K = (int)p.K;
  a.B = p.B;
  a.mode = p.mode;
  a.prec = p.prec;
  a.q8 = p.q8;
  a.s8 = p.s8;
  a.rho = p.rho;
  a.force = p.force;
  a.groups = reinterpret_cast<GroupSlot*>(p.groups);
  a.hdr = reinterpret_cast<WsHeader*>(p.hdr);
  a.stats = p.stats;
  a.finish = 1;
  const int NB = (int)(p.K / 128);
  float4* c4 = reinterpret_cast<float4*>(chunks);
  const int64_t G = ceil_div(p.M, kG);
  const int64_t want = ceil_div(G, kFoldWarps);
  const int sms = chunks_sms();
  k_fold_chunks<<<(unsigned)(want < sms ? want : sms), kFoldWarps * 32, 0, s>>>(a, c4, NB);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || p.mode != SB_PREPASS_QUANT) return e;
  CUtensorMap mx;
  if (!make_halfblock_map(&mx, p.X, p.M, p.K)) return cudaErrorInvalidValue;
  switch (p.B) {
    case 16: return launch_int8_blk<16>(a, c4, NB, mx, s);
    case 32: return launch_int8_blk<32>(a, c4, NB, mx, s);
    case 64: return launch_int8_blk<64>(a, c4, NB, mx, s);
    case 128: return launch_int8_blk<128>(a, c4, NB, mx, s);
    default: return cudaErrorInvalidValue;
  }
}

// The fused module record from the GEMM's per-chunk partial sums (two float4 per row and
// 128-column chunk: {sum |y|, sum (y - x)^2, sum x^2, sum |y - c|}, {sum |c|, max |y|, 0, 0}). A
// chunk's sums are aligned subtrees of the row's canonical tree, so one warp per 16-row group (a
// lane per row) rebuilds each row's five sums as the row engine does (the chunks zero-padded),
// then writes the group's two FP64 slots; the last CTA runs the record's two finishes: the
// difference statistic into *stats, then the TDC record with d from it, as k_rows<.., OP_REC>.
__global__ void __launch_bounds__(kFoldWarps * 32) k_fold_modrec(RowArgs a, const float4* rec, int NB) {
  __shared__ double s_fin[kFinChunk];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int prec = a.prec ? *a.prec : -1;
  if (prec == SB_SKIP) return;  // the GEMM did not run: no output to record
  const bool do_tdc = a.st->skip == 0;
  const bool have_prev = a.st->n_out >= 1;
  const int64_t G = ceil_div(a.M, kG);
  int NB2 = 1;
  while (NB2 < NB) NB2 <<= 1;
  const int c = NB2 >= 32 ? NB2 / 32 : 1;  // chunks per lane (a power of two <= 16)
  const int span = NB2 / c;                // lanes covering one row
  for (int64_t g = (int64_t)blockIdx.x * kFoldWarps + warp; g < G; g += (int64_t)gridDim.x * kFoldWarps) {
    // lane i < kG: row i of the group, its chunks read in order
    const int64_t m = g * kG + lane;
    const bool row = lane < kG && m < a.M;
    const float4* rc = rec + 2 * (row ? m : 0) * NB;
    // each row's trees in two levels: aligned runs of 8 chunks in registers, then the 16 run sums
    float runs[5][16];
#pragma unroll
    for (int st = 0; st < 5; ++st)
#pragma unroll
      for (int k = 0; k < 16; ++k) runs[st][k] = 0.0f;
    float rmx = 0.0f;
    if (row) {
#pragma unroll 2
      for (int b0 = 0; b0 < NB; b0 += 8) {  // two runs' loads in flight at once
        float t[5][8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
#pragma unroll
          for (int st = 0; st < 5; ++st) t[st][u] = 0.0f;
          if (b0 + u < NB) {
            const float4 r0 = rc[2 * (b0 + u)], r1 = rc[2 * (b0 + u) + 1];
            t[0][u] = r0.x;
            t[1][u] = r0.y;
            t[2][u] = r0.z;
            t[3][u] = r0.w;
            t[4][u] = r1.x;
            rmx = fmaxf(rmx, r1.y);
          }
        }
#pragma unroll
        for (int st = 0; st < 5; ++st) {
          const float s8 = __fadd_rn(__fadd_rn(__fadd_rn(t[st][0], t[st][1]), __fadd_rn(t[st][2], t[st][3])),
                                     __fadd_rn(__fadd_rn(t[st][4], t[st][5]), __fadd_rn(t[st][6], t[st][7])));
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (k == (b0 >> 3)) runs[st][k] = s8;  // a register per run: no indexed local array
        }
      }
    }
    float rs[5];
#pragma unroll
    for (int st = 0; st < 5; ++st) rs[st] = tree16(runs[st]);
    const bool in = lane < kG;
    double gs[5];
#pragma unroll
    for (int st = 0; st < 5; ++st) gs[st] = warp_pairwise_f64(in ? (double)rs[st] : 0.0);
    const float gmx = warp_max_f32(in ? rmx : 0.0f);
    const int gnf = __any_sync(0xffffffffu, in && (isnan(rs[0]) || isinf(rmx)));  // Inf or NaN in a row
    if (lane == 0) {
      GroupSlot* slot = a.groups + g;
      slot->s[0] = gs[0];
      slot->s[1] = gs[1];
      slot->s[2] = gs[2];
      slot->max_abs = gmx;
      slot->amax_rot = 0.0f;
      slot->nonfinite = gnf;
      GroupSlot* slot2 = a.groups2 + g;
      slot2->s[0] = gs[3];
      slot2->s[1] = gs[4];
      slot2->s[2] = 0.0;
      slot2->max_abs = 0.0f;
      slot2->amax_rot = 0.0f;
      slot2->nonfinite = 0;
    }
  }
  rows_finish<OP_STATS, true>(a, G, prec, true, s_fin);
  if (do_tdc) {
    RowArgs t = a;
    t.groups = a.groups2;
    t.dsrc = a.stats;
    rows_finish<OP_TDC, true>(t, G, prec, have_prev, s_fin);
  }
}

cudaError_t launch_fold_modrec(const RecordLaunch& p, const float* rec, cudaStream_t s) {
  RowArgs a{};
  a.M = p.M;
  a.K = (int)p.C;
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
  const int NB = (int)(p.C / 128);
  const int64_t G = ceil_div(p.M, kG);
  const int64_t want = ceil_div(G, kFoldWarps);
  const int sms = chunks_sms();
  k_fold_modrec<<<(unsigned)(want < sms ? want : sms), kFoldWarps * 32, 0, s>>>(a, reinterpret_cast<const float4*>(rec),
                                                                                  NB);
  return cudaGetLastError();
}

// Chunk records of a bf16 tensor [M][K] (K % 128 == 0) with the same arithmetic the GEMM's
// record epilogue uses: one thread per (row, 128-channel chunk).
__global__ void __launch_bounds__(128) k_chunk_records(const __nv_bfloat16* X, int64_t M, int K, int B,
                                                        float4* out) {
  const int nc = K / 128;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M * nc) return;
  const int64_t m = i / nc;
  const int c = (int)(i - m * nc);
  const uint4* src = reinterpret_cast<const uint4*>(X + m * K + 128 * c);
  uint32_t v[4][32];
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const uint4 w = src[q];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int k = 8 * q + 2 * t;
      v[k >> 5][k & 31] = ws[t] << 16;
      v[(k + 1) >> 5][(k + 1) & 31] = ws[t] & 0xffff0000u;
    }
  }
  out[i] = chunk_record(v, B);
}

cudaError_t launch_chunk_records(const void* X, int64_t M, int64_t K, int B, float* out, cudaStream_t s) {
  const int64_t n = M * (K / 128);
  k_chunk_records<<<(unsigned)ceil_div(n, 128), 128, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(X), M, (int)K,
                                                             B, reinterpret_cast<float4*>(out));
  return cudaGetLastError();
}

}  // namespace sb
