// sb_device.cuh -- device helpers shared by the sm_100a kernels of libsixbit.
//
// bf16 unpacking, the warp-level block Hadamard butterfly, deterministic pairwise reductions,
// NVFP4/E4M3 hardware conversions and thin inline-PTX wrappers for mbarriers, TMA and the
// tcgen05 tensor-core / tensor-memory instructions. Written for sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sixbit.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libsixbit is written for sm_100a (B200) only"
#endif

namespace sb {

// ---------------------------------------------------------------------------------------------
// Workspace layout (caller-owned memory; see sb_workspace_size)
// ---------------------------------------------------------------------------------------------

// One slot per aligned group of kGroupRows (16) rows: FP64 pairwise partial sums of the group,
// maxima.
struct GroupSlot {
  double s[3];       // per-statistic group sum (pre-pass: |x|, (x-r)^2, r^2; TDC: |a-b|, |b|)
  float max_abs;     // max |x| of the group (raw)
  float amax_rot;    // max |Hx| of the group (rotated)
  int32_t nonfinite; // a row held Inf/NaN: its max |x| is Inf or its sum |x| NaN
  int32_t pad[3];
};
static_assert(sizeof(GroupSlot) == 48, "GroupSlot layout");

struct WsHeader {
  uint32_t err;         // first device error (sb_status), 0 = none
  uint32_t ticket[7];   // last-CTA tickets, one per kernel family; self-resetting
  uint32_t pad[24];
};
static_assert(sizeof(WsHeader) == 128, "WsHeader layout");

enum { TICKET_PREPASS = 0, TICKET_TDC = 1 };

constexpr int kGroupRows = 16;  // rows per FP64 group partial
constexpr int kMaxK = 16384;

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---------------------------------------------------------------------------------------------
// Errors
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ void set_error(WsHeader* h, uint32_t code) {
  if (h) atomicCAS(&h->err, 0u, code);
}

// ---------------------------------------------------------------------------------------------
// bf16 <-> f32, exact widening
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ void unpack8(const uint4& u, float (&v)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// 32-byte (256-bit) accesses, sm_100: one full sector per lane per instruction.
__device__ __forceinline__ void ldg_nc_v8(const void* p, uint4& a, uint4& b) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
               : "l"(p));
}

__device__ __forceinline__ void ldg_v8(const void* p, uint4& a, uint4& b) {
  asm volatile("ld.global.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
               : "l"(p));
}

__device__ __forceinline__ void stg_v8(void* p, const uint4& a, const uint4& b) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w),
               "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

__device__ __forceinline__ uint4 ldg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------------------------
// Block Hadamard (unnormalised Sylvester), 8 contiguous elements per lane.
// Stage h pairs (j, j+h) with bit h of j clear: (a, b) -> (a + b, a - b), FP32 RN, h ascending.
// Stages h = 1, 2, 4 run inside the lane; h = 8 .. B/2 pair lane l with lane l ^ (h/8).
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ void fwht8_in_lane(float (&v)[8]) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if ((j & h) == 0) {
        const float a = v[j], b = v[j + h];
        v[j] = __fadd_rn(a, b);
        v[j + h] = __fsub_rn(a, b);
      }
    }
  }
}

// lanes_per_block = B / 8 (2 .. 32). Inactive lanes must still execute (full-warp shuffles).
__device__ __forceinline__ void fwht_across_lanes(float (&v)[8], int lane, int lanes_per_block) {
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    if (s >= lanes_per_block) break;
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float other = __shfl_xor_sync(0xffffffffu, v[j], s);
      // lower element keeps a + b, upper keeps a - b with a = the lower lane's value
      v[j] = upper ? __fsub_rn(other, v[j]) : __fadd_rn(v[j], other);
    }
  }
}

// Pairwise sum of the 8 lane-local terms: ((t0+t1)+(t2+t3))+((t4+t5)+(t6+t7)).
__device__ __forceinline__ float pairwise8(const float (&t)[8]) {
  const float a = __fadd_rn(__fadd_rn(t[0], t[1]), __fadd_rn(t[2], t[3]));
  const float b = __fadd_rn(__fadd_rn(t[4], t[5]), __fadd_rn(t[6], t[7]));
  return __fadd_rn(a, b);
}

// Pairwise tree across the 32 lanes (lane-aligned subtrees of 2, 4, .., 32), every lane gets it.
__device__ __forceinline__ float warp_pairwise_f32(float x) {
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, s));
  return x;
}

__device__ __forceinline__ double warp_pairwise_f64(double x) {
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) x = __dadd_rn(x, __shfl_xor_sync(0xffffffffu, x, s));
  return x;
}

__device__ __forceinline__ float warp_max_f32(float x) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, s));
  return x;
}

// Pairwise FP64 sum of the aligned run [lo, lo + R) of a strided array (R a power of two;
// entries at or beyond n count as zero), evaluated with a stack of partial sums so the additions
// follow the same tree as halving the run recursively: S(lo,R) = S(lo,R/2) + S(lo+R/2,R/2).
__device__ inline double run_pairwise_f64(const double* p, int64_t stride, int64_t lo, int64_t R, int64_t n) {
  double stack[40];
  int sp = 0;
  for (int64_t i = 0; i < R; ++i) {
    const int64_t idx = lo + i;
    double x = (idx < n) ? __ldcg(p + idx * stride) : 0.0;
    for (int64_t k = i; k & 1; k >>= 1) x = __dadd_rn(stack[--sp], x);
    stack[sp++] = x;
  }
  return stack[0];
}

// Pairwise FP64 tree over n strided values zero-padded to a power of two P >= 32, by one warp:
// lane l reduces the run [l*P/32, (l+1)*P/32), then the 32 run sums meet in the warp tree.
__device__ inline double warp_pairwise_f64_global(const double* p, int64_t stride, int64_t n, int lane) {
  int64_t P = 32;
  while (P < n) P <<= 1;
  const int64_t R = P / 32;
  return warp_pairwise_f64(run_pairwise_f64(p, stride, (int64_t)lane * R, R, n));
}

// ---------------------------------------------------------------------------------------------
// Number-format conversions (PTX cvt, round-to-nearest-even, satfinite)
// ---------------------------------------------------------------------------------------------

// Two floats -> one byte of two E2M1 codes: `lo` in bits 0-3, `hi` in bits 4-7.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// float -> E4M3 byte (RN, satfinite)
__device__ __forceinline__ uint32_t cvt_e4m3(float v) {
  uint16_t r;
  asm volatile("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return (uint32_t)(r & 0xffu);
}

// E4M3 byte -> float (exact)
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  uint32_t h2;
  const uint16_t in = (uint16_t)(b & 0xffu);
  asm volatile("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  const __half h = __ushort_as_half((unsigned short)(h2 & 0xffffu));
  return __half2float(h);
}

// ---------------------------------------------------------------------------------------------
// Shared-memory addresses, mbarriers, bounded waits
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with parity `parity` to complete. Gives up after `limit_ns` (or when
// *abort is raised by another role; abort may be null), returning false; the caller then records
// SB_ETIMEOUT.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t it = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++it & 63u) == 0) {
      if (abort && *abort) return false;
      if (globaltimer() - t0 > limit_ns) return false;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// TMA (no multicast anywhere) and bulk copies
// ---------------------------------------------------------------------------------------------

// 3-D TMA tile load into this CTA's shared memory (shared address), completing on a local barrier.
__device__ __forceinline__ void tma_load_3d(uint32_t smem_dst, const void* tmap, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_dst),
      "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx_u32(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// The same with shared-memory addresses already in the shared window.
__device__ __forceinline__ void tma_load_2d_u32(uint32_t smem_dst, const void* tmap, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_dst),
      "l"(tmap), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// TMA tile store from this CTA's shared memory, tracked by the issuing thread's bulk groups.
// Rows or columns of the box outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t smem_src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tmap), "r"(x),
               "r"(y), "r"(smem_src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N bulk groups of this thread still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 16-byte asynchronous global -> shared copy (cp.async), completed by cp_async_wait_all.
__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ---------------------------------------------------------------------------------------------
// Clusters of two CTAs (the tcgen05 CTA pair)
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// shared::cluster address of the variable at `smem_ptr` in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t cluster_addr(const void* smem_ptr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(smem_ptr)), "r"(rank));
  return r;
}

// Arrive on a barrier of any CTA of the cluster (shared::cluster address), with the default CTA-
// scope release. Used to hand tensor memory back: that ordering comes from tcgen05.wait::ld and
// tcgen05.fence::before_thread_sync, not from this arrive (a cluster-scope release here waited
// for the thread's outstanding memory traffic and cost about a microsecond per tile).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar_addr) : "memory");
}

// TMA tile load of one CTA of the pair; completion bytes go to the barrier at `bar_cluster`
// (a shared::cluster address, here the leader CTA's barrier). No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const void* tmap, uint32_t bar_cluster, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const void* tmap, uint32_t bar_cluster, int x, int y,
                                                 int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(z), "r"(bar_cluster)
      : "memory");
}

// ---------------------------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, commit, loads
// ---------------------------------------------------------------------------------------------

__device__ __forceinline__ void mma_fp4_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                             uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}

// Scale factors of one 32-row x 16-byte slice from each CTA's shared memory into the same columns
// of its own tensor memory, replicated to the four 32-lane quadrants (issued by the leader).
__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Arrive (once each) on the barrier at the same offset in every CTA of `mask` when all earlier
// tcgen05 operations of this thread have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle, 8-row core groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3ffffu) >> 4);      // start address
  d |= (uint64_t)1 << 16;                         // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024 >> 4) << 32;               // stride byte offset
  d |= (uint64_t)1 << 46;                         // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                         // SWIZZLE_128B
  return d;
}

// Descriptor of a 32-row x 16-byte scale-factor atom slice (no swizzle, 8-row groups 128 B apart)
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3ffffu) >> 4);
  d |= (uint64_t)(128 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                        uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}

__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 columns of 32-bit words: lane i gets columns [col, col+32) of TMEM lane (base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Per-warpgroup register budget (all warps of the warpgroup execute it). An increase waits until
// other warpgroups have released enough of the registers the CTA was launched with, so the
// launcher checks that the final split fits the launch allocation.
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// max(a, b, c) in one instruction, with fmaxf's rule for NaN (a NaN input is ignored unless all
// three are NaN).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// ---------------------------------------------------------------------------------------------
// Chunk records (FFN-pair fusion)
// ---------------------------------------------------------------------------------------------

// FP32x2 butterfly of two adjacent pairs: (a0, a1) <- (a0 + b0, a1 + b1), (b0, b1) <- (a0 - b0,
// a1 - b1), every lane rounded to nearest as the scalar sum and difference are.
__device__ __forceinline__ void bfly2(uint32_t& a0, uint32_t& a1, uint32_t& b0, uint32_t& b1) {
  uint64_t a, b, s, d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "r"(a0), "r"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "r"(b0), "r"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(s) : "l"(a), "l"(b));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a0), "=r"(a1) : "l"(s));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(b0), "=r"(b1) : "l"(d));
}


// The chunk record of one row's 128 output columns, in place on v[c][j] = column 32 c + j (FP32
// bit patterns of the values the bf16 output holds), B the Hadamard block (16, 32, 64 or 128):
//  - max |v|;
//  - the canonical pairwise sum of |v|, whose first level RN(|a| + |b|) = max(|a + b|, |a - b|)
//    comes out of the first butterfly;
//  - the unnormalised FWHT stages h = 1 .. B/4 in ascending order (a + b, a - b rounded to
//    nearest), one transform per aligned block of B columns; the last stage h = B/2 is not
//    formed: its outputs' largest magnitude is max(|RN(a + b)|, |RN(a - b)|) = RN(|a| + |b|);
//  - the rotated amax.
template <int B>
__device__ __forceinline__ float4 chunk_record(uint32_t (&v)[4][32]) {
#define SB_V(k) v[(k) >> 5][(k) & 31]
  float mx = 0.0f, part[16];  // part[g]: the tree sum of elements 8 g .. 8 g + 7
#pragma unroll
  for (int g = 0; g < 16; ++g) {
    float l[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int k = 8 * g + 2 * u;
      const float a = __uint_as_float(SB_V(k)), b = __uint_as_float(SB_V(k + 1));
      mx = max3(mx, fabsf(a), fabsf(b));
      const float s = __fadd_rn(a, b), d = __fsub_rn(a, b);
      SB_V(k) = __float_as_uint(s);
      SB_V(k + 1) = __float_as_uint(d);
      l[u] = fmaxf(fabsf(s), fabsf(d));
    }
    part[g] = __fadd_rn(__fadd_rn(l[0], l[1]), __fadd_rn(l[2], l[3]));
  }
#pragma unroll
  for (int len = 16; len > 1; len >>= 1) {
#pragma unroll
    for (int i = 0; i < len / 2; ++i) part[i] = __fadd_rn(part[2 * i], part[2 * i + 1]);
  }
  float am = 0.0f;
#pragma unroll
  for (int h = 2; h <= B / 2; h <<= 1) {
    if (2 * h < B) {
#pragma unroll
      for (int k = 0; k < 128; k += 2) {
        if ((k & h) == 0) bfly2(SB_V(k), SB_V(k + 1), SB_V(k + h), SB_V(k + h + 1));
      }
    } else {
#pragma unroll
      for (int k = 0; k < 128; k += 2) {
        if ((k & h) == 0) {
          const float t0 = __fadd_rn(fabsf(__uint_as_float(SB_V(k))), fabsf(__uint_as_float(SB_V(k + h))));
          const float t1 = __fadd_rn(fabsf(__uint_as_float(SB_V(k + 1))), fabsf(__uint_as_float(SB_V(k + h + 1))));
          am = max3(am, t0, t1);
        }
      }
    }
  }
#undef SB_V
  return make_float4(am, part[0], mx, 0.0f);
}

// chunk_record for a block size known at run time (one instantiation per supported block).
__device__ __forceinline__ float4 chunk_record(uint32_t (&v)[4][32], int B) {
  switch (B) {
    case 16: return chunk_record<16>(v);
    case 32: return chunk_record<32>(v);
    case 64: return chunk_record<64>(v);
    default: return chunk_record<128>(v);
  }
}

}  // namespace sb
