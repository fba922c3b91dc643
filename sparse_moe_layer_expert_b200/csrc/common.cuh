// common.cuh -- sm_100a building blocks shared by the kernels of libmoefp8:
// mbarrier waits with a time limit, TMA tile loads, tcgen05 (TMEM allocation,
// MMA issue, commit, TMEM loads) and UMMA descriptor construction.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_fp8.h"  // include/ is on the include path (build.py)

namespace moe {

// Every mbarrier wait gives up after this long (unless a kernel is given a
// shorter limit) and reports MOE_DEVERR_TIMEOUT instead of spinning forever.
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

// The suspend-time hint lets the hardware park a waiting thread until the
// phase completes (or the hint expires) instead of spinning through issue
// slots that the working warps of the same SM sub-partition need.
constexpr uint32_t kSuspendHintNs = 1000000;  // 1 ms

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Shared state for bounded waits inside one CTA: once any wait of the CTA
// times out, `abort` is set and all later waits return false at once, so
// every role drains quickly and the kernel ends.
struct WaitCtl {
  volatile int *abort;  // in shared memory
  int32_t *err;         // global error word
  uint64_t limit_ns;
};

// Wait for phase `parity` of `bar` to complete.  Returns false (and records
// a timeout) if it does not within ctl.limit_ns, or if the CTA is aborting.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const WaitCtl &ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*ctl.abort) return false;
    if (global_timer_ns() - t0 > ctl.limit_ns) {
      *ctl.abort = 1;
      if (ctl.err) atomicOr(ctl.err, MOE_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// Non-blocking probe of phase `parity` (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for two phases.  Both are probed before either result is used, so the
// two round trips to the barriers overlap when both phases are already
// complete (the common case on the critical path); otherwise each is waited
// for in turn with the bounded wait above.
__device__ __forceinline__ bool mbar_wait2(uint64_t *bar1, uint32_t parity1, uint64_t *bar2, uint32_t parity2,
                                           const WaitCtl &ctl) {
  const bool a = mbar_test_wait(bar1, parity1);
  const bool b = mbar_test_wait(bar2, parity2);
  if (a && b) return true;
  return (a || mbar_wait(bar1, parity1, ctl)) && (b || mbar_wait(bar2, parity2, ctl));
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy reads of them (TMA, tcgen05.cp, tcgen05.mma operands).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2D tiled bulk copy global -> shared; completes `bytes` on `bar`.
// x (innermost coordinate, in elements) must keep x * elem_size a multiple
// of 16; callers only pass multiples of 128.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Same with an L2 eviction-priority hint (a createpolicy value).
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *map, uint64_t *bar, int32_t x,
                                                 int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, "
      "{%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ------------------------------------------------------------- cp.async (4 B)
// Asynchronous 4-byte global -> shared copy (no register holds the data).
__device__ __forceinline__ void cp_async4(void *dst_smem, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst_smem)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's committed groups are still pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 1D bulk copy global -> shared of `bytes` (multiple of 16; both addresses
// 16-byte aligned), completing `bytes` on `bar`.
// 2D tiled bulk copy shared -> global (the box of the tensor map at
// coordinates x, y; x * elem_size a multiple of 16, x and y >= 0), tracked by
// the issuing thread's bulk groups: commit, then wait until the shared-memory
// source has been read (wait_read) or the copy is complete (wait_all).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// -------------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
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

// D[tmem] (+)= A[smem desc] x B[smem desc]^T, E4M3 x E4M3 -> F32.
__device__ __forceinline__ void umma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A x B^T, BF16 x BF16 -> F32.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread
// has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// columns [col, col+32) of TMEM lane (lane_base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// 32 lanes x 64 consecutive 32-bit columns (one register per column).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row (1024-byte) swizzle atoms
// stacked contiguously (stride 1024 B between atoms), tile base 1024-aligned.
// Advancing the K position inside the 128-byte row adds bytes/16 to the
// start-address field.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4)  // start address
         | (static_cast<uint64_t>(1) << 16)              // leading byte offset (unused here)
         | (static_cast<uint64_t>(1024 >> 4) << 32)      // stride byte offset: 8 rows x 128 B
         | (static_cast<uint64_t>(1) << 46)              // descriptor version (sm_100)
         | (static_cast<uint64_t>(2) << 61);             // layout: 128-byte swizzle
}

// Instruction descriptors (dense, K-major A and B, FP32 accumulate).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4)                                    // D format F32
         | (0u << 7) | (0u << 10)                     // A, B format E4M3
         | (static_cast<uint32_t>(N >> 3) << 17)      // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);     // M / 16
}
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                    // D format F32
         | (1u << 7) | (1u << 10)                     // A, B format BF16
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------ CTA pairs (clusters of 2)
// Rank of this CTA inside its cluster.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The shared::cluster address of the variable at shared::cta address `saddr`
// in the CTA of cluster rank `rank` (same offset in that CTA's shared memory).
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}

// Arrive on an mbarrier given by its shared::cluster address (this CTA's or
// another CTA's of the cluster) with the default release semantics at CTA
// scope.  These arrivals carry no generic-memory data between the CTAs: they
// order TMEM reads (with the tcgen05 fences around them) and count TMA bytes,
// so no cluster-wide fence is needed -- and one costs about a microsecond on
// the critical path of the pair GEMM.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t caddr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cluster.b64 _, [%0], %1;" ::"r"(caddr), "r"(bytes) : "memory");
}

// Barrier over every thread of the cluster (all threads of both CTAs of a
// pair execute it, convergently).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 2D tiled bulk copy global -> this CTA's shared memory whose completion is
// counted on an mbarrier of either CTA of the pair (given by its
// shared::cluster address): the pair's MMA issuer waits on one barrier for
// the operands of both CTAs.
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar_caddr, int32_t x,
                                                 int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_caddr), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// TMEM allocation shared by the two CTAs of a pair: one warp of each CTA
// (the same warp index) executes these; both get the same columns.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Pair MMA, E4M3 x E4M3 -> F32, issued by one thread of the even CTA: M is
// split over the two CTAs (rows 0..M/2-1 from the even CTA's A tile, the rest
// from the odd CTA's at the same shared-memory offset), N likewise (B rows
// 0..N/2-1 from the even CTA), and each CTA's TMEM receives its M/2 rows x N.
__device__ __forceinline__ void umma_f8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at the same shared-memory offset in every CTA
// of `cta_mask` when all pair MMAs issued so far by this thread completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Barrier over `nthreads` that also returns the OR of `pred` over them.
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// a / b rounded to nearest from y = RN(1/b): q0 = RN(a*y), the exact residual
// r = a - b*q0 (one FMA), then RN(q0 + r*y).  One residual correction of the
// quotient (Markstein's division by reciprocal, as presented in Muller et al.,
// "Handbook of Floating-Point Arithmetic", chapter on division) -- used where
// many values share one divisor; b > 0 normal, a/b far from over/underflow.
// With b > 0 the quotient carries a's sign; copysignf keeps it for a = -0,
// where the residual step would otherwise return +0 (-0 + +0 = +0).
__device__ __forceinline__ float div_by_recip(float a, float b, float y) {
  const float q0 = a * y;
  const float r = fmaf(-b, q0, a);
  return copysignf(fmaf(r, y, q0), a);
}

// Two independent FP32 fused multiply-adds in one instruction:
// (lo, hi) <- (p_lo * s + c_lo, p_hi * s + c_hi), each rounded to nearest
// like fmaf.
__device__ __forceinline__ void ffma2_scalar(float &c_lo, float &c_hi, float p_lo, float p_hi, float s) {
  uint64_t c, p, ss;
  asm("mov.b64 %0, {%1, %2};" : "=l"(c) : "f"(c_lo), "f"(c_hi));
  asm("mov.b64 %0, {%1, %2};" : "=l"(p) : "f"(p_lo), "f"(p_hi));
  asm("mov.b64 %0, {%1, %1};" : "=l"(ss) : "f"(s));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(c) : "l"(p), "l"(ss));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(c_lo), "=f"(c_hi) : "l"(c));
}

// (lo, hi) <- (p_lo * s_lo + c_lo, p_hi * s_hi + c_hi): two FMAs with their
// own multipliers, one instruction.
__device__ __forceinline__ void ffma2_vec(float &c_lo, float &c_hi, float p_lo, float p_hi, float s_lo, float s_hi) {
  uint64_t c, p, ss;
  asm("mov.b64 %0, {%1, %2};" : "=l"(c) : "f"(c_lo), "f"(c_hi));
  asm("mov.b64 %0, {%1, %2};" : "=l"(p) : "f"(p_lo), "f"(p_hi));
  asm("mov.b64 %0, {%1, %2};" : "=l"(ss) : "f"(s_lo), "f"(s_hi));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(c) : "l"(p), "l"(ss));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(c_lo), "=f"(c_hi) : "l"(c));
}

// Power-of-two scale, the variant whose scale factors a tensor core applies
// itself (block-scaled MMA with 8-bit exponent scale factors): S = 2^e with e
// the smallest integer for which amax <= 448 * 2^e, held at 2^-127 or above;
// amax == 0 gives 0.  With amax = 1.m * 2^E and 448 = 1.75 * 2^8, e = E - 8
// when 1.m <= 1.75 and E - 7 otherwise.  The exponent byte of the returned
// float is the scale factor's 8-bit code (2^-127 is the float subnormal with
// exponent byte 0).
__device__ __forceinline__ float pow2_scale(float amax) {
  if (!(amax > 0.0f)) return 0.0f;
  uint32_t b = __float_as_uint(amax);
  int E = static_cast<int>(b >> 23) - 127;
  uint32_t m = b & 0x7FFFFFu;
  if ((b >> 23) == 0) {  // subnormal: amax = m * 2^-149, leading bit at p
    const int p = 31 - __clz(m);
    E = p - 149;
    m = (m << (23 - p)) & 0x7FFFFFu;
  }
  int e = (m <= 0x600000u) ? E - 8 : E - 7;
  if (e < -127) e = -127;
  return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// Two E4M3 codes (round to nearest even, saturating) packed low = a, high = b.
__device__ __forceinline__ uint32_t e4m3x2_rn_sat(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// E4M3 code of v (round to nearest even, saturating at +-448).
__device__ __forceinline__ uint8_t e4m3_rn_sat(float v) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

}  // namespace moe

// Host-side helpers (defined in api.cu).
namespace moe_host {
int encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner,
                   uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);
int sm_count();
}  // namespace moe_host
