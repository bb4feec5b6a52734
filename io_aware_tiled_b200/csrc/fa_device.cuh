// fa_device.cuh -- sm_100a device primitives used by the attention kernels:
// mbarriers with bounded waits, TMA tensor loads, tcgen05 (TMEM allocation,
// MMA issue/commit, TMEM loads/stores) and the shared-memory / instruction
// descriptors the tensor cores read.
//
// Every wait on an mbarrier is bounded by a wall-clock limit (the %globaltimer
// register).  When the limit passes, the waiting thread records an error code
// in the library's device error word and returns false; the kernel then
// leaves its loops, frees its tensor memory and exits.  Nothing here traps.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// ---------------------------------------------------------------------------
// error word (one per device, read and cleared by fa_sync_status)
// ---------------------------------------------------------------------------
__device__ unsigned int g_error_word = 0u;   // 0 = ok; else (where << 8) | code
constexpr unsigned int kErrTimeout = 1u;

// Wall-clock limit of one mbarrier wait, in nanoseconds.  Correct code waits
// microseconds; the limit only ends a kernel whose pipeline has stalled.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_error(unsigned int code, unsigned int where) {
  atomicCAS(&g_error_word, 0u, (where << 8) | code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0u;
}

// Wait for the phase of parity `parity` to complete, at most kWaitLimitNs.
// `where` identifies the wait site in the error word.
__device__ __forceinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, unsigned int where,
                                            unsigned long long limit_ns) {
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) {
      record_error(kErrTimeout, where);
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned int where) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, where, kWaitLimitNs);
}

// ---------------------------------------------------------------------------
// clusters of two CTAs (the 2-SM tensor-core form)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared_to_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t cluster_addr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(cluster_addr),
               "r"(bytes)
               : "memory");
}
// Non-blocking test (test_wait): a thread suspended in try_wait is not woken
// promptly by an arrival from the peer CTA, so cluster-scope waits poll.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0u;
}
// Bounded wait on a local barrier that the peer CTA also arrives on.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, unsigned int where) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      record_error(kErrTimeout, where);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// register reallocation between warpgroups (warpgroup-wide; the sum over the
// CTA must stay within the registers it was launched with)
// ---------------------------------------------------------------------------
template <uint32_t R>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}

// ---------------------------------------------------------------------------
// named barriers (a subset of the CTA's warps)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// TMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 3-D tiled load (no multicast) completing on an mbarrier.  c0 is the
// innermost coordinate (elements), c1 the row, c2 the head.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 3-D tiled load issued by either CTA of a pair, completing on the barrier at
// `bar_cluster_addr` (the leader CTA's barrier); no multicast.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster_addr,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory
// ---------------------------------------------------------------------------
// Allocation and deallocation are warp-wide (.sync.aligned): call from one full warp.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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
// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]; kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]; A is K-major in tensor memory (lane = row).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-wide forms: every lane of the warp executes the call with the same
// (warp-uniform) operands and one elected lane issues the instruction.  Keeping
// the issuing loop warp-uniform lets the descriptors live in uniform registers.
__device__ __forceinline__ void mma_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit_warp(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

// Grouped issue: one elect.sync, then the MMAs of a whole K loop.  A shared-
// memory descriptor advances along K by adding to its start-address field
// (16-byte units): +2 per K step of 16 bf16 inside a 128-byte row, and a new
// 64-column chunk starts from its own base descriptor.  All lanes call these
// with warp-uniform operands; the elected lane issues.
//
// K = 128, A and B K-major in shared memory (two 64-column chunks each).
__device__ __forceinline__ void mma_ss_k128(uint32_t d_tmem, uint64_t a0, uint64_t a1, uint64_t b0, uint64_t b1,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b64 ax, bx;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "setp.eq.b32 t, %5, %5;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %3, %5, p;\n\t"
      "add.s64 ax, %1, 2;\n\tadd.s64 bx, %3, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "add.s64 ax, %1, 4;\n\tadd.s64 bx, %3, 4;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "add.s64 ax, %1, 6;\n\tadd.s64 bx, %3, 6;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %4, %5, t;\n\t"
      "add.s64 ax, %2, 2;\n\tadd.s64 bx, %4, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "add.s64 ax, %2, 4;\n\tadd.s64 bx, %4, 4;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "add.s64 ax, %2, 6;\n\tadd.s64 bx, %4, 6;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %5, t;\n\t}" ::"r"(d_tmem),
      "l"(a0), "l"(a1), "l"(b0), "l"(b1), "r"(idesc), "r"(accumulate)
      : "memory");
}
// K = 64, A and B K-major in shared memory (one 64-column chunk).
__device__ __forceinline__ void mma_ss_k64(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b64 ax, bx;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %3, %3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "add.s64 ax, %1, 2;\n\tadd.s64 bx, %2, 2;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 4;\n\tadd.s64 bx, %2, 4;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 6;\n\tadd.s64 bx, %2, 6;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t}" ::"r"(d_tmem),
      "l"(a0), "l"(b0), "r"(idesc), "r"(accumulate)
      : "memory");
}
// K = 64, A K-major (+32 B per K step) and B MN-major (16 rows of 128 bytes =
// +2048 B per K step), both in shared memory.
__device__ __forceinline__ void mma_ss_k64_bmn(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b64 ax, bx;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %3, %3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "add.s64 ax, %1, 2;\n\tadd.s64 bx, %2, 128;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 4;\n\tadd.s64 bx, %2, 256;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 6;\n\tadd.s64 bx, %2, 384;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t}" ::"r"(d_tmem),
      "l"(a0), "l"(b0), "r"(idesc), "r"(accumulate)
      : "memory");
}
// A from tensor memory (K-major, 8 columns of packed bf16 per K step of 16),
// B MN-major in shared memory (16 rows of 128 bytes = +128 per K step).
// K = 128 (8 steps).
__device__ __forceinline__ void mma_ts_k128(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b64 bx;\n\t.reg .b32 ax;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %3, %3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "add.s32 ax, %1, 8;\n\tadd.s64 bx, %2, 128;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 16;\n\tadd.s64 bx, %2, 256;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 24;\n\tadd.s64 bx, %2, 384;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 32;\n\tadd.s64 bx, %2, 512;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 40;\n\tadd.s64 bx, %2, 640;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 48;\n\tadd.s64 bx, %2, 768;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 56;\n\tadd.s64 bx, %2, 896;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b0), "r"(idesc), "r"(accumulate)
      : "memory");
}
// K = 64 (4 steps).
__device__ __forceinline__ void mma_ts_k64(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b64 bx;\n\t.reg .b32 ax;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %3, %3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "add.s32 ax, %1, 8;\n\tadd.s64 bx, %2, 128;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 16;\n\tadd.s64 bx, %2, 256;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 24;\n\tadd.s64 bx, %2, 384;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [ax], bx, %3, t;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b0), "r"(idesc), "r"(accumulate)
      : "memory");
}

// K = 128, A and B both MN-major in shared memory (16 rows of 128 bytes =
// +2048 B per K step for each): D^T-style products whose contraction runs
// over the rows of both staged tiles.
__device__ __forceinline__ void mma_ss_k128_mnmn(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b64 ax, bx;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %3, %3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "add.s64 ax, %1, 128;\n\tadd.s64 bx, %2, 128;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 256;\n\tadd.s64 bx, %2, 256;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 384;\n\tadd.s64 bx, %2, 384;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 512;\n\tadd.s64 bx, %2, 512;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 640;\n\tadd.s64 bx, %2, 640;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 768;\n\tadd.s64 bx, %2, 768;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t"
      "add.s64 ax, %1, 896;\n\tadd.s64 bx, %2, 896;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ax, bx, %3, t;\n\t}" ::"r"(d_tmem),
      "l"(a0), "l"(b0), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ---------------------------------------------------------------------------
// bulk (non-tensor) copies between shared and global memory
// ---------------------------------------------------------------------------
// Makes this thread's ordinary shared-memory stores visible to the async
// proxy (the tensor core's operand reads, bulk copies) once a barrier orders
// them before the consumer.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// global[dst .. dst+bytes) += shared[src .. src+bytes) as fp32, element-wise,
// performed by the bulk-copy engine; both addresses 16-byte aligned, bytes a
// multiple of 16.  Tracked by the issuing thread's bulk groups.
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
               "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every bulk group of this thread has completed (writes performed).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 2-SM forms (cta_group::2): issued by the leader CTA of a pair; A and D rows
// are split between the two CTAs (M/2 each), B's N columns likewise.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Arrive once on the barrier at this offset in every CTA of `cta_mask` when all
// prior tcgen05 operations of this thread complete.
__device__ __forceinline__ void tc_commit_pair_warp(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}" ::"r"(
          bar),
      "h"(cta_mask)
      : "memory");
}
__device__ __forceinline__ void mma2_ss_k128(uint32_t d_tmem, uint64_t a0, uint64_t a1, uint64_t b0, uint64_t b1,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b64 ax, bx;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "setp.eq.b32 t, %5, %5;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %3, %5, p;\n\t"
      "add.s64 ax, %1, 2;\n\tadd.s64 bx, %3, 2;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "add.s64 ax, %1, 4;\n\tadd.s64 bx, %3, 4;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "add.s64 ax, %1, 6;\n\tadd.s64 bx, %3, 6;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %2, %4, %5, t;\n\t"
      "add.s64 ax, %2, 2;\n\tadd.s64 bx, %4, 2;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "add.s64 ax, %2, 4;\n\tadd.s64 bx, %4, 4;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], ax, bx, %5, t;\n\t"
      "add.s64 ax, %2, 6;\n\tadd.s64 bx, %4, 6;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], ax, bx, %5, t;\n\t}" ::"r"(d_tmem),
      "l"(a0), "l"(a1), "l"(b0), "l"(b1), "r"(idesc), "r"(accumulate)
      : "memory");
}
// K = 64 (4 steps): A from each CTA's tensor memory, B MN-major in each CTA's
// shared memory (+2048 B per step of 16 rows).
__device__ __forceinline__ void mma2_ts_k64(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b64 bx;\n\t.reg .b32 ax;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %3, %3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "add.s32 ax, %1, 8;\n\tadd.s64 bx, %2, 128;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 16;\n\tadd.s64 bx, %2, 256;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 24;\n\tadd.s64 bx, %2, 384;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b0), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma2_ts_k128(uint32_t d_tmem, uint32_t a_tmem, uint64_t b0, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred e, p, t;\n\t.reg .b64 bx;\n\t.reg .b32 ax;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 t, %3, %3;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "add.s32 ax, %1, 8;\n\tadd.s64 bx, %2, 128;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 16;\n\tadd.s64 bx, %2, 256;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 24;\n\tadd.s64 bx, %2, 384;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 32;\n\tadd.s64 bx, %2, 512;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 40;\n\tadd.s64 bx, %2, 640;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 48;\n\tadd.s64 bx, %2, 768;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t"
      "add.s32 ax, %1, 56;\n\tadd.s64 bx, %2, 896;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ax], bx, %3, t;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b0), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-collective TMEM load, shape 32x32b: thread t of the warp reads lane
// (32 * (warp % 4) + t) of the address's lane window, 32 consecutive columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Keeps the compiler from using registers filled by tcgen05.ld before the wait.
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
                 "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
                 "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor, 128-byte swizzle (the layout TMA writes
// with CU_TENSOR_MAP_SWIZZLE_128B).  Fields: start address >> 4 (bits 0-13),
// leading-dimension byte offset >> 4 (16-29), stride-dimension byte offset
// >> 4 (32-45), descriptor version 1 (46-47), base offset 0 (49-51; every
// swizzle atom is 1024-byte aligned), layout type 2 = SWIZZLE_128B (61-63).
//
// K-major operand (rows of 64 bf16 = 128 B, 8-row atoms of 1024 B): LBO is
// unused (encoded 16 B), SBO = 1024 B between 8-row groups.  One MMA step of
// K = 16 elements advances the start address by 32 B inside the atom; the
// next 64-element K chunk is a separate block of rows.
//
// MN-major operand (the same smem image read transposed): LBO = byte
// distance between 64-element MN chunks, SBO = 1024 B between 8-row K groups;
// one MMA step of K = 16 rows advances the start address by 16 * 128 B.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(lbo_bytes >> 4) << 16) |
         (static_cast<uint64_t>(sbo_bytes >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// The same descriptor split into its two 32-bit halves: the low half holds the
// start address and LBO (changes per MMA step), the high half SBO, version and
// swizzle mode (constant per operand).
__device__ __forceinline__ uint32_t sdesc_lo(uint32_t saddr, uint32_t lbo_bytes) {
  return ((saddr & 0x3FFFFu) >> 4) | ((lbo_bytes >> 4) << 16);
}
__host__ __device__ constexpr uint32_t sdesc_hi(uint32_t sbo_bytes) {
  return (sbo_bytes >> 4) | (1u << 14) | (2u << 29);
}
__device__ __forceinline__ uint64_t sdesc_make(uint32_t lo, uint32_t hi) {
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A bf16 (7-9 = 1),
// B bf16 (10-12 = 1), A major (15; 0 = K, 1 = MN), B major (16), N >> 3
// (17-22), M >> 4 (24-28); dense, no negation, no saturation.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// arithmetic helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^t on the FMA and integer pipes instead of the MUFU, for t <= 8 (the
// softmax arguments; -inf included).  Cody-Waite range reduction: 2^t =
// 2^j 2^f with j = rint(t) (added 1.5 * 2^23 leaves j in the low mantissa
// bits of r) and f = t - j in [-1/2, 1/2]; 2^f from the degree-3 polynomial of
// least maximum relative error on that interval (Remez exchange, fitted by
// fit_exp2_poly.py); j is added to the exponent field.  Relative error
// <= 7.5e-5 on [-125, 8], below bf16's rounding of P (2^-9).  t is clamped at
// -126 so the exponent field never wraps: smaller arguments (masked scores
// are -inf) give a positive value <= 2^-125 (not 0), which no fp32 sum or
// bf16 product can register.
// The softmax sends a fixed share of its exponentials here so that the MUFU
// and the FMA pipes finish together.
__device__ __forceinline__ float exp2_poly3(float t) {
  t = fmaxf(t, -126.f);
  const float r = t + 12582912.f;
  const float f = t - (r - 12582912.f);
  const float p = fmaf(fmaf(fmaf(0.05517166853f, f, 0.2426111251f), f, 0.6932609677f), f, 0.9999280572f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(r) << 23));
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of the NC (a multiple of 8, >= 32) values of s: 8 independent
// chains of three-input maxima, then a three-input tree.
template <int NC>
__device__ __forceinline__ float row_max(const float (&s)[NC]) {
  static_assert(NC % 8 == 0 && NC >= 32, "row_max expects a multiple of 8 columns, at least 32");
  float pm[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) pm[e] = fmax3(s[e], s[8 + e], s[16 + e]);
  int c = 24;
#pragma unroll
  for (; c + 16 <= NC; c += 16)
#pragma unroll
    for (int e = 0; e < 8; ++e) pm[e] = fmax3(pm[e], s[c + e], s[c + 8 + e]);
  if (c < NC) {
#pragma unroll
    for (int e = 0; e < 8; ++e) pm[e] = fmaxf(pm[e], s[c + e]);
  }
  return fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
}

// Two fp32 values in one 64-bit register for the paired fp32 instructions
// (fma.rn.f32x2, add.rn.f32x2): one instruction for two elements.
__device__ __forceinline__ uint64_t f2_make(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// Multiply 32 fp32 values (raw bits, in place) by `mul`, two per instruction.
__device__ __forceinline__ void scale32(uint32_t (&a)[32], float mul) {
  const uint64_t m2 = f2_make(mul, mul);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float lo, hi;
    f2_split(f2_mul(f2_make(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1])), m2), lo, hi);
    a[2 * i] = __float_as_uint(lo);
    a[2 * i + 1] = __float_as_uint(hi);
  }
}

// exp2_poly3 of the two values of a pair, on the paired fp32 instructions:
// the same operations lane by lane (the same results), half the FMA-pipe
// instructions.
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ void exp2_poly3_x2(uint64_t t2, float& p0, float& p1) {
  float t0, t1;
  f2_split(t2, t0, t1);
  const uint64_t t = f2_make(fmaxf(t0, -126.f), fmaxf(t1, -126.f));
  const uint64_t magic = f2_make(12582912.f, 12582912.f);
  const uint64_t r = f2_add(t, magic);
  const uint64_t f = f2_sub(t, f2_sub(r, magic));
  const uint64_t c3 = f2_make(0.05517166853f, 0.05517166853f), c2 = f2_make(0.2426111251f, 0.2426111251f);
  const uint64_t c1 = f2_make(0.6932609677f, 0.6932609677f), c0 = f2_make(0.9999280572f, 0.9999280572f);
  const uint64_t p = f2_fma(f2_fma(f2_fma(c3, f, c2), f, c1), f, c0);
  float q0, q1, r0, r1;
  f2_split(p, q0, q1);
  f2_split(r, r0, r1);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(r0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(r1) << 23));
}


__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
  return *reinterpret_cast<uint32_t*>(&v);
}

// 32 fp32 values (as raw bits) times `mul`, as 32 bf16 (64 bytes) at `dst`
// (16-byte aligned): two 32-byte stores when `dst` is 32-byte aligned, so each
// writes whole 32-byte sectors, else four 16-byte stores.
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const uint32_t (&a)[32], float mul) {
  uint32_t w[16];
  const uint64_t m2 = f2_make(mul, mul);
#pragma unroll
  for (int i = 0; i < 16; ++i) {  // two products per paired multiply
    float lo, hi;
    f2_split(f2_mul(f2_make(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1])), m2), lo, hi);
    w[i] = pack_bf16(lo, hi);
  }
  if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 16), "r"(w[8]), "r"(w[9]),
                 "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]), "r"(w[15])
                 : "memory");
  } else {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int v = 0; v < 4; ++v) d4[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
  }
}

// Index of the k-th work unit of a persistent worker w out of W: units are
// dealt in rounds of W, left to right on even rounds and right to left on odd
// ones ("serpentine").  With units sorted longest first this balances the
// per-worker sums far better than plain round robin.
__device__ __forceinline__ int serpentine_unit(int k, int w, int W) {
  return k * W + ((k & 1) ? (W - 1 - w) : w);
}

// Causal block orders of the backward launch the longest blocks first so the
// last wave is short; across all heads at once, that keeps every head's K and
// V (or Q and dO) in flight.  Heads therefore go in groups whose K and V
// (bf16) fit in 32 MiB of the 126 MB L2 (all heads when they fit), longest
// blocks first inside each group.  Returns the group size.
__host__ __device__ __forceinline__ int causal_head_group(int BH, int N, int D) {
  const long long per_head = 4ll * N * D;
  const long long g = (32ll << 20) / per_head;
  return g >= BH ? BH : (g < 1 ? 1 : static_cast<int>(g));
}
// Unit u of that order for units of NR ranks per head (rank 0 = longest):
// head bh and rank r.
__host__ __device__ __forceinline__ void causal_grouped_unit(int u, int BH, int NR, int G, int& bh, int& r) {
  const int per_group = G * NR;
  const int g = u / per_group;
  const int v = u - g * per_group;
  const int gh = G < BH - g * G ? G : BH - g * G;  // heads in this group (the last may be short)
  r = v / gh;
  bh = g * G + (v - r * gh);
}

// Per-CTA work lists of the persistent kernels, computed on the host (a
// longest-processing-time assignment) and passed by value: CTA c runs the
// units order[start[c] .. start[c + 1]) in that order.  n = 0: no list.
struct UnitList {
  static constexpr int kMaxCtas = 160;
  static constexpr int kMaxUnits = 4096;
  int n;                                   // units in `order`
  unsigned short start[kMaxCtas + 1];
  unsigned short order[kMaxUnits];         // unit indices, in each kernel's own numbering
};
struct NoUnitList {
  int n;
};
template <bool WITH_LIST>
struct UnitListOf {
  using type = NoUnitList;
};
template <>
struct UnitListOf<true> {
  using type = UnitList;
};

// The k-th unit of worker w (of W) in `list` (>= units when it has no more);
// without a list, the units dealt in serpentine order over the W workers.
template <typename L>
__device__ __forceinline__ int worker_unit(const L& list, int k, int units, int w, int W) {
  if constexpr (sizeof(L) > sizeof(NoUnitList)) {
    if (list.n > 0) {
      const int i = list.start[w] + k;
      return i < list.start[w + 1] ? static_cast<int>(list.order[i]) : units;
    }
  }
  return serpentine_unit(k, w, W);
}
// The same with one worker per CTA.
template <typename L>
__device__ __forceinline__ int list_unit(const L& list, int k, int units) {
  return worker_unit(list, k, units, static_cast<int>(blockIdx.x), static_cast<int>(gridDim.x));
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace fa
