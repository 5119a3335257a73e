// Shared device helpers of the NOSA sparse-decode kernels (sm_100a).
//
// mbarrier + bulk-copy (TMA, cp.async.bulk) wrappers written as inline PTX,
// with every wait bounded: a wait that does not complete within
// kWaitLimitNs of %globaltimer (or kWaitLimitIters polls) sets
// NOSA_DEV_TIMEOUT in the device status word and returns false, so a kernel
// never spins forever and never traps.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nosa.h"

namespace nosa {

constexpr int kHeadDim = 128;
constexpr int kPoolKernel = 32;
constexpr int kPoolStride = 16;
constexpr int kBlock = 64;
constexpr int kWindowsPerBlock = kBlock / kPoolStride;  // 4
// A scoring chunk covers 15 blocks [b0, b0+15), i.e. pooled windows
// [4*b0-1, 4*b0+60): 61 rows, fetched as TMA boxes of 32 fp32 columns
// (128 bytes) each, so that a chunk's four boxes fill one 32 KB ring stage.
constexpr int kChunkBlocks = 15;
constexpr int kChunkWindows = kChunkBlocks * kWindowsPerBlock + 1;  // 61
constexpr int kBoxCols = 32;
constexpr int kBoxRows = kChunkWindows;
constexpr int kMaxCluster = 16;  // CTAs per (sequence, KV head) cluster, at most
constexpr int kMaxGroup = 16;
constexpr int kMaxLocalBlocks = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr uint32_t kWaitLimitIters = 1u << 30;

__host__ __device__ inline int64_t n_windows(int64_t L) {
  return L >= kPoolKernel ? (L - kPoolKernel) / kPoolStride + 1 : 0;
}
__host__ __device__ inline int64_t n_blocks(int64_t L) { return (L + kBlock - 1) / kBlock; }
__host__ __device__ inline int64_t n_candidates(int64_t L, int local_blocks) {
  int64_t c = n_blocks(L) - local_blocks;
  return c > 0 ? c : 0;
}

__device__ inline void set_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

__device__ inline uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ inline uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the async (TMA) proxy.
__device__ inline void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ inline void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ inline void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Tests whether the phase with the given parity has completed.  A waiting
// thread is suspended (it takes no issue slots) until the phase completes
// or `suspend_ns` pass, so polling warps do not slow down the other warps
// of their SM.
__device__ inline bool mbar_test_parity(uint64_t* bar, uint32_t parity, uint32_t suspend_ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(suspend_ns)
      : "memory");
  return done != 0;
}

// Waits until the phase with the given parity has completed.  Bounded by
// `max_iters` suspended polls of at most `suspend_ns` each and by
// kWaitLimitNs of wall time; on giving up it sets NOSA_DEV_TIMEOUT and
// returns false.
__device__ inline bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                 uint32_t max_iters = kWaitLimitIters, uint32_t suspend_ns = 100000u) {
  if (mbar_test_parity(bar, parity, suspend_ns)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; it < max_iters; ++it) {
    if (mbar_test_parity(bar, parity, suspend_ns)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) break;
  }
  set_status(status, NOSA_DEV_TIMEOUT);
  return false;
}

// L2 policy for data read once per step (KV tiles, pooled keys): evict it
// first, so streaming it does not push the kernels' code and small metadata
// out of L2.
__device__ inline uint64_t l2_evict_first_policy() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}

// 1-D bulk copy global -> shared through the TMA unit, completing on `bar`,
// with the evict-first L2 policy.  dst, src and bytes must be multiples of 16.
__device__ inline void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(l2_evict_first_policy())
      : "memory");
}

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start while its predecessor on the stream is finishing:
// it must not touch global memory before grid_dependency_wait(), which returns
// once the predecessor grid has completed and its writes are visible.
// allow_dependents() lets the next kernel on the stream start its own
// prologue early.  Both are no-ops without a programmatic predecessor.
__device__ inline void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ inline void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- KV rows
// Where the tokens of one sequence live in the K/V caches: contiguous rows
// from `base` (seq_start[i]), or 64-token pages through the sequence's row
// of a page table (token t in row pages[t / 64] * 64 + t % 64).  The page
// size equals the block size, so an attention tile is exactly one page.
constexpr int kPageTokens = kBlock;

struct KvRows {
  int64_t base;          // contiguous: the sequence's first row
  const int32_t* pages;  // paged: the sequence's page-table row (nullptr: contiguous)
  int64_t num_pages;     // paged: valid page indices are [0, num_pages)
  __device__ int64_t row(int64_t t) const {
    return pages ? static_cast<int64_t>(pages[t / kPageTokens]) * kPageTokens + t % kPageTokens : base + t;
  }
  // Whether token t's page index is valid (always, for contiguous caches,
  // whose range the caller checks once).
  __device__ bool page_ok(int64_t t) const {
    if (!pages) return true;
    const int32_t pg = pages[t / kPageTokens];
    return pg >= 0 && pg < num_pages;
  }
};

// ---------------------------------------------------------------- clusters
// Thread-block cluster primitives (distributed shared memory).  Addresses
// of another CTA's shared memory are 32-bit shared::cluster addresses from
// mapa.

__device__ inline uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ inline uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

__device__ inline uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

// The address of the same shared-memory location in CTA `rank` of the cluster.
__device__ inline uint32_t map_shared_rank(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}

__device__ inline void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ inline void st_cluster_f32x4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

// Asynchronous store of one fp32 into another CTA's shared memory that
// completes `bytes` (4) of transaction count on that CTA's mbarrier (both
// addresses are shared::cluster addresses): the receiver's wait on the
// barrier then sees the value, with no fence on the sender's side.
__device__ inline void st_async_f32(uint32_t addr, float v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(addr),
               "r"(__float_as_uint(v)), "r"(remote_bar)
               : "memory");
}

// As st_async_f32, four fp32 (16 bytes, 16-byte aligned address).
__device__ inline void st_async_f32x4(uint32_t addr, float4 v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
               "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)), "r"(__float_as_uint(v.z)),
               "r"(__float_as_uint(v.w)), "r"(remote_bar)
               : "memory");
}

__device__ inline float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ inline float4 ld_cluster_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Split cluster barrier: every thread of every CTA of the cluster arrives
// once and waits once per phase (arrive publishes this thread's earlier
// writes, wait acquires everyone's).
__device__ inline void cluster_arrive() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ inline void cluster_wait() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }

__device__ inline void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }

// Arrive on an mbarrier of another CTA of the cluster, releasing this
// thread's earlier writes at cluster scope.
__device__ inline void mbar_remote_arrive(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}

// As mbar_wait, acquiring at cluster scope: for phases completed by other
// CTAs' remote arrivals.
__device__ inline bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t* status,
                                         uint32_t max_iters = kWaitLimitIters, uint32_t suspend_ns = 100000u) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0; it < max_iters; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(suspend_ns)
        : "memory");
    if (done) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) break;
  }
  set_status(status, NOSA_DEV_TIMEOUT);
  return false;
}

// Order-preserving map of an fp32 score to uint32, with -0.0 == +0.0 and NaN
// ranked as -inf (ties are then broken by index by the caller).
__device__ inline uint32_t order_key(float f) {
  if (f != f) f = -INFINITY;
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace nosa
