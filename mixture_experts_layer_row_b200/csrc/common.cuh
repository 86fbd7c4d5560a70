// Device-side building blocks shared by the kernels of the MoE layer library (sm_100a only).
//
// - the sticky error flag that device code sets instead of trapping;
// - bounded mbarrier waits: every wait gives up after a time limit (read from %globaltimer), sets
//   MOE_DEVERR_TIMEOUT and lets the kernel return;
// - thin inline-PTX wrappers for mbarrier, TMA tile loads, and the tcgen05 tensor-core family
//   (TMEM allocation, MMA, commit, TMEM loads), written from the PTX ISA's descriptions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_b200.h"

namespace moe {

// Layout of the workspace head: the sticky error flag, then a few reserved words.
constexpr size_t kWsHeadBytes = 256;

__device__ __forceinline__ void set_error(uint32_t* flag, uint32_t bits) {
  if (flag) atomicOr(flag, bits);
}

// Division by a loop-invariant divisor d >= 1 through a precomputed multiplier (T. Granlund and
// P. Montgomery, "Division by invariant integers using multiplication", 1994, the round-up variant):
// with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1, floor(n / d) = (mulhi(m, n) + n) >> l
// for every 0 <= n < 2^32 (the sum taken in 64 bits).
struct FastDiv {
  uint32_t m, l;
  int d;
  __host__ __device__ FastDiv() : m(1), l(0), d(1) {}
  __host__ __device__ explicit FastDiv(int div) : d(div) {
    l = 0;
    while ((1ull << l) < (uint64_t)div) ++l;
    m = (uint32_t)((((1ull << 32) * ((1ull << l) - (uint64_t)div)) / (uint64_t)div) + 1);
  }
  __device__ __forceinline__ int div(int n) const {
    return (int)(((uint64_t)__umulhi((uint32_t)n, m) + (uint32_t)n) >> l);
  }
};

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete. Returns false -- after setting
// MOE_DEVERR_TIMEOUT and the CTA-wide abort word -- if it did not within `limit_ns`, or if another
// role of the CTA has already aborted.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                                  volatile int* abort_word, uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort_word && *abort_word) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      if (abort_word) *abort_word = 1;
      set_error(err, MOE_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, completion counted on an mbarrier)
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// 3-D tiled load (coordinates innermost first).
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Bring a tile into L2 ahead of its shared-memory load (no completion tracking, no smem).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1)
               : "memory");
}

// TMA tile store shared -> global, tracked as one bulk group per call.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t c0,
                                             int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all of this thread's bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Make this thread's generic-proxy shared-memory writes visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(void* p, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p)), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_u32(p))
               : "memory");
  return v;
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16), counted on an mbarrier.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, commit, loads
// ---------------------------------------------------------------------------------------------
// Allocation is a warp-wide operation; the TMEM base address is written to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, shapes and types in the instruction descriptor.
template <int KIND>  // 0: kind::f16 (bf16/fp16 inputs), 1: kind::tf32
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                     uint32_t accumulate) {
  if constexpr (KIND == 0) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// MXFP8 block-scaled MMA: E4M3 A/B from shared memory, one UE8M0 scale per 32 K-elements per row
// of A and of B read from TMEM (scale columns at sfa/sfb; the byte of each 32-bit column that holds
// this MMA's K-block is selected by the instruction descriptor's scale-factor ids).
__device__ __forceinline__ void umma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p; }" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Copy 32 rows x 16 bytes from shared memory (described by a no-swizzle K-major descriptor) into 32
// TMEM lanes x 4 columns, replicated to all four 32-lane quadrants.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Instruction descriptor for kind::mxf8f6f4.block_scale: E4M3 x E4M3, UE8M0 scales, fp32 accumulate.
__host__ __device__ constexpr uint32_t instr_desc_mx(bool a_mn, bool b_mn, int M, int N) {
  return (0u << 7) | (0u << 10)  // A, B: E4M3
         | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         (1u << 23)  // scale format: UE8M0
         | ((uint32_t)(M >> 4) << 24);
}

// Make the mbarrier track completion of all tcgen05 operations this thread issued before.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets row (lane base + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Wait for this thread's outstanding tcgen05.ld and pass `r` through the wait, so that no use of
// those registers can be scheduled ahead of it. tmem_regs_after then orders a further set of
// registers after the same wait.
__device__ __forceinline__ void tmem_ld_wait_regs(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_regs_after(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// ---------------------------------------------------------------------------------------------
// Programmatic dependent launch. Every kernel of this library is launched with the stream's
// programmatic serialisation allowed, so it may be scheduled while the previous kernel in the stream
// is still finishing. pdl_trigger lets the next kernel be scheduled; pdl_wait blocks until the previous
// kernel has completed and its memory is visible. Each kernel calls pdl_wait before its first global
// memory access (read or write).
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_enter() {
  pdl_trigger();
  pdl_wait();
}

// ---------------------------------------------------------------------------------------------
// CTA pairs (thread-block cluster of 2, tcgen05 cta_group::2): the leader (rank 0) issues MMAs with
// M = 256 whose A rows 0-127 and 128-255 and whose two halves of B sit in the two CTAs' shared
// memory at the same offsets; each CTA's tensor memory holds its 128 accumulator rows.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void fence_barrier_init_cluster() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Shared::cluster address of the object at the same offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrive (release at cluster scope) on an mbarrier given by its shared::cluster address.
// The arrive keeps the default CTA-scope release: the barriers that cross the pair only hand over
// tensor memory, whose accesses the tcgen05 fences on either side of the arrive / wait order. A
// cluster-scope release would add a fence at that scope to every handover.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// try_wait with acquire at cluster scope (for barriers that the peer CTA arrives on).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2; "
      "selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_bounded_cluster(uint64_t* bar, uint32_t parity,
                                                          uint64_t limit_ns, volatile int* abort_word,
                                                          uint32_t* err) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (abort_word && *abort_word) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      if (abort_word) *abort_word = 1;
      set_error(err, MOE_DEVERR_TIMEOUT);
      return false;
    }
  }
}
// TMA loads issued by either CTA of a pair into its own shared memory, completing on the leader's
// mbarrier (shared::cluster address). No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// Tensor memory of a CTA pair: the same warp of both CTAs allocates, relinquishes and frees.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// M = 256 MMA of a CTA pair (issued by the leader); KIND 0: kind::f16, 1: kind::tf32.
template <int KIND>
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  if constexpr (KIND == 0) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}
// Arrive on the mbarrier at this offset in every CTA of `mask` once the pair's earlier MMAs finish.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// Shared-memory matrix descriptor for tcgen05 (version 1 for sm_100).
//   start: byte address in shared memory; lbo/sbo: leading / stride byte offsets;
//   layout: 2 = 128-byte swizzle (16-byte chunks, 8-row atoms), 1 = 128-byte swizzle with 32-byte
//   chunks and 4-row atoms (the layout MN-major 32-bit operands need).
constexpr uint32_t kLayoutSW128 = 2;
constexpr uint32_t kLayoutSW128Atom32 = 1;
__device__ __forceinline__ uint64_t smem_desc(uint32_t start, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((start >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

// Instruction descriptor for kind::f16 / kind::tf32 dense MMA with fp32 accumulation.
//   fmt: 1 = bf16 (kind::f16), 2 = tf32; a_mn / b_mn: operand is MN-major (else K-major).
__host__ __device__ constexpr uint32_t instr_desc(uint32_t fmt, bool a_mn, bool b_mn, int M, int N) {
  return (1u << 4)                    // D format: fp32
         | (fmt << 7) | (fmt << 10)   // A, B formats
         | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------------------------------------
// small numeric helpers
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}


// ---------------------------------------------------------------------------------------------
// MXFP8 encoding (OCP Microscaling Formats v1.0: E4M3 elements, one UE8M0 scale per 32-element block)
//   block exponent e = floor(log2(amax)) - 8 (8 = E4M3's largest exponent), clamped to [-127, 127];
//   scale byte = e + 127; code = round-to-nearest-even(x * 2^-e) saturated to +-448;
//   an all-zero block gets scale byte 0 and zero codes.
// ---------------------------------------------------------------------------------------------
// floor(log2(a)) for a finite a > 0 given as fp32 bits.
__device__ __forceinline__ int floor_log2_bits(uint32_t bits) {
  const int ex = (int)((bits >> 23) & 0xFFu);
  if (ex != 0) return ex - 127;
  const uint32_t man = bits & 0x7FFFFFu;  // subnormal: man * 2^-149
  return -149 + (31 - __clz(man));
}

// 2^k as an fp32 value for k in [-127, 127] (2^-127 is subnormal, still exact).
__device__ __forceinline__ float exp2_exact(int k) {
  return k >= -126 ? __int_as_float((k + 127) << 23) : __int_as_float(1 << (k + 149));
}

// Block exponent and scale byte for a block with maximum magnitude amax (>= 0).
__device__ __forceinline__ int block_exponent(float amax, uint8_t* scale_byte) {
  if (!(amax > 0.f)) {
    *scale_byte = 0;
    return 127;  // unused: all codes are zero
  }
  int e = floor_log2_bits(__float_as_uint(amax)) - 8;
  e = e < -127 ? -127 : (e > 127 ? 127 : e);
  *scale_byte = (uint8_t)(e + 127);
  return e;
}

// Two floats -> two E4M3 codes (round to nearest even, saturate to finite), packed lo | hi << 8.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Byte mask over four packed column codes that clears the codes of all-zero column blocks (whose
// values, +0 or -0, would otherwise convert to +0 or -0 codes; an all-zero block has zero codes).
__device__ __forceinline__ uint32_t zero_block_mask(const float (&amax)[4]) {
  return (amax[0] > 0.f ? 0x000000FFu : 0u) | (amax[1] > 0.f ? 0x0000FF00u : 0u) |
         (amax[2] > 0.f ? 0x00FF0000u : 0u) | (amax[3] > 0.f ? 0xFF000000u : 0u);
}

// Byte offset of the scale of (MN index i, K-block b) in the tiled layout with KB K-blocks per MN index.
__device__ __forceinline__ int64_t tiled_sf_offset(int64_t i, int64_t b, int64_t KB) {
  return ((i >> 7) * (KB >> 2) + (b >> 2)) * 512 + (i & 31) * 16 + ((i >> 5) & 3) * 4 + (b & 3);
}

// The MXFP8 quantisations of a warp's 32 rows x 32 columns, one row per lane (v = this lane's row,
// already rounded to the stored precision).
// Row block: the lane's 32 values -> 32 codes (8 words, column order) and the block's scale byte.
__device__ __forceinline__ uint8_t mx_row_block(const float (&v)[32], uint32_t (&c)[8]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
  uint8_t sb;
  const float ir = exp2_exact(-block_exponent(m, &sb));
#pragma unroll
  for (int i = 0; i < 8; ++i)
    c[i] = m > 0.f ? ((uint32_t)cvt_e4m3x2(v[4 * i] * ir, v[4 * i + 1] * ir) |
                      ((uint32_t)cvt_e4m3x2(v[4 * i + 2] * ir, v[4 * i + 3] * ir) << 16))
                   : 0u;
  return sb;
}
// Column blocks: column j of the warp's 32 rows is one block. The 32 column maxima come out of a
// transposing butterfly (lane L ends with column L's maximum), the scales are broadcast back, and
// each lane converts its own row; returns the scale byte of column `lane`.
__device__ __forceinline__ uint8_t mx_col_blocks(const float (&v)[32], int lane, uint32_t (&c)[8]) {
  float m[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) m[i] = fabsf(v[i]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;  // keep columns [off, 2off) of the current range, else [0, off)
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? m[i] : m[i + off];
      const float keep = upper ? m[i + off] : m[i];
      m[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
    }
  }
  uint8_t sb;
  const int e = block_exponent(m[0], &sb);
  const float inv_mine = m[0] > 0.f ? exp2_exact(-e) : 0.f;
  const uint32_t nz = __ballot_sync(0xffffffffu, m[0] > 0.f);  // columns whose block is not all zero
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = v[4 * i + q] * __shfl_sync(0xffffffffu, inv_mine, 4 * i + q);
    uint32_t word = (uint32_t)cvt_e4m3x2(w[0], w[1]) | ((uint32_t)cvt_e4m3x2(w[2], w[3]) << 16);
    const uint32_t keep = ((nz >> (4 * i)) & 1u ? 0x000000FFu : 0u) | ((nz >> (4 * i + 1)) & 1u ? 0x0000FF00u : 0u) |
                          ((nz >> (4 * i + 2)) & 1u ? 0x00FF0000u : 0u) | ((nz >> (4 * i + 3)) & 1u ? 0xFF000000u : 0u);
    c[i] = word & keep;
  }
  return sb;
}

}  // namespace moe
