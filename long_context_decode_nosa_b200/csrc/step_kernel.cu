// Kernels for selection, sparse attention and the fused decode step.
//
// One persistent kernel, `step_kernel<G>`, runs any mix of two kinds of work
// items from an atomic work queue held in the workspace:
//   * scoring items (sequence i, KV head g, chunk of 16 blocks): compressed
//     scores and block scores of the chunk; the last chunk of a pair (atomic
//     ticket) selects its top-k ("NOSA-1B 性能基准全解析" §三.2/§三.3);
//   * decode items (i, g, split): exact attention over that split of the
//     pair's tiles (§三.3 / §三.2 local window).
// Scoring items are handed out first.  In the fused decode step the first
// scoring item of each pair also appends the new token's K/V rows and pools
// the window the token completes ("从论文到代码…" item 2), and each decode
// item streams its local-window tiles at once but waits -- a bounded spin on
// the pair's ready flag, published with a release store by the CTA that
// selected the pair's blocks -- before its first tile that depends on the
// selection or on the appended token.  Items are dispensed in index order to
// resident CTAs only (the grid never exceeds what fits on the GPU), so every
// scoring item a decode item waits for is already running: no deadlock.
// The last CTA to leave resets the queue; tickets and flags are reset by
// their last users, so the workspace is ready for the next launch.
#include "decode_device.cuh"
#include "nosa_common.cuh"
#include "nosa_kernels.h"
#include "pool_device.cuh"
#include "select_device.cuh"

namespace nosa {

#ifdef NOSA_TRACE
// Instrumented builds only (-DNOSA_TRACE): one record per work item of the
// step kernel -- CTA, SM, item, start / selection-seen / end globaltimer.
struct TraceRecord {
  uint32_t cta, smid, item, clk_delta;  // clk_delta: SM clock cycles spent in the item
  uint64_t t_start, t_flag, t_end;
  uint32_t issue[8], full[8], done[8];  // per tile, ns after t_start
  uint32_t merge[6];                     // decode merge phase, ns after t_start
};
constexpr int kTraceCapacity = 1 << 16;
__device__ TraceRecord g_trace[kTraceCapacity];
__device__ uint32_t g_trace_count;
#endif

namespace {

constexpr int kSelOnlyThreads = 256;
constexpr int kCtasPerSm = 2;

__device__ void write_empty_selection(const SelectArgs& a, int pair, int nthreads) {
  for (int t = threadIdx.x; t < a.topk; t += nthreads) a.sel_idx[static_cast<int64_t>(pair) * a.topk + t] = -1;
  if (threadIdx.x == 0) a.sel_cnt[pair] = 0;
}

// Append the new token's K/V rows and pool the window it completes, for one
// (sequence, KV head) of length L (the new token is token L-1).  Warp 0
// stores the rows, warp 1 pools (reading the new K row from k_new).
__device__ void append_and_pool(const PoolArgs& p, int pair, int L) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = pair / p.hkv, h = pair % p.hkv;
  const int64_t base = p.seq_start[i];
  if (base < 0 || base + L > p.cache_rows) {
    if (threadIdx.x == 0) set_status(p.status, NOSA_DEV_CACHE_ROWS);
    return;
  }
  const int64_t len_old = L - 1;
  const uint2* knew =
      p.k_new ? reinterpret_cast<const uint2*>(p.k_new + (static_cast<int64_t>(i) * p.hkv + h) * kHeadDim) : nullptr;
  if (warp == 0 && knew) {
    const int64_t row = (base + len_old) * p.hkv + h;
    const uint2* vnew = reinterpret_cast<const uint2*>(p.v_new + (static_cast<int64_t>(i) * p.hkv + h) * kHeadDim);
    reinterpret_cast<uint2*>(p.k_cache + row * kHeadDim)[lane] = knew[lane];
    reinterpret_cast<uint2*>(p.v_cache + row * kHeadDim)[lane] = vnew[lane];
  }
  const int64_t j = n_windows(L) - 1;
  if (warp == 1 && j >= 0 && j >= n_windows(len_old)) {
    if (j >= p.nc_cap) {
      if (lane == 0) set_status(p.status, NOSA_DEV_NC_CAP);
    } else {
      pool_window_warp(p.k_cache, p.hkv, base, h, j, knew ? len_old : -1, knew,
                       p.pooled + ((static_cast<int64_t>(i) * p.hkv + h) * p.nc_cap + j) * kHeadDim, lane);
    }
  }
}

#ifdef NOSA_TRACE
#define NOSA_STAMP(slot)                                      \
  do {                                                        \
    if (threadIdx.x == 0) stamps[slot] = global_timer_ns();   \
  } while (0)
#else
#define NOSA_STAMP(slot) \
  do {                   \
  } while (0)
#endif

template <int G>
__device__ void score_item(const StepArgs& a, int item, uint8_t* smem, uint64_t* key_bar, uint32_t& key_phase,
                           TopkShared& tsh, int* sh_last, uint64_t* stamps) {
  const SelectArgs& s = a.sel;
  const int pair = item % a.pairs, chunk = item / a.pairs;
  const int i = pair / s.hkv, g = pair % s.hkv;
  const int tid = threadIdx.x;
  const int L = s.seq_len[i];
  NOSA_STAMP(0);
  if (L < 1 || L > s.max_seq_len) {
    if (chunk == 0) {
      if (tid == 0) set_status(s.status, L < 1 ? NOSA_DEV_BAD_LENGTH : NOSA_DEV_MAX_LEN);
      write_empty_selection(s, pair, kDecThreads);
    }
    return;
  }
  const ScoreGeometry geo = score_geometry(L, s.nc_cap, s.local_blocks, s.comp_out != nullptr, chunk);
  if (chunk >= geo.nchunks) return;
  if (chunk == 0 && n_windows(L) > s.nc_cap && tid == 0) set_status(s.status, NOSA_DEV_NC_CAP);
  if ((a.mode & kStepAppend) && chunk == 0) append_and_pool(a.pool, pair, L);
  const bool uses_keys = geo.b1 > geo.b0 && geo.jhi > geo.jlo;
  score_chunk<G, kDecThreads>(s.q, s.pooled, s.nc_cap, s.hq, s.hkv, i, g, s.scale, geo,
                              s.bscratch + static_cast<int64_t>(pair) * s.nb_ws, s.comp_out,
                              s.bs_out ? s.bs_out + static_cast<int64_t>(pair) * s.nb_out : nullptr, smem, key_bar,
                              key_phase, s.status, stamps ? stamps + 1 : nullptr);
  if (uses_keys) key_phase ^= 1u;
  __syncthreads();
  NOSA_STAMP(2);
  if (tid == 0) {
    __threadfence();
    const uint32_t t = atomicAdd(&s.tickets[pair], 1u);
    *sh_last = (t == static_cast<uint32_t>(geo.nchunks - 1));
  }
  __syncthreads();
  NOSA_STAMP(3);
  if (!*sh_last) return;
  if (tid == 0) __threadfence();  // acquire: the other chunks' block scores
  __syncthreads();
  NOSA_STAMP(7);
  // The pair's last chunk: every block score is written; select.
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  select_topk<kDecThreads>(s.bscratch + static_cast<int64_t>(pair) * s.nb_ws, true, geo.ncand, s.topk,
                           s.sel_idx + static_cast<int64_t>(pair) * s.topk, s.sel_cnt + pair,
                           reinterpret_cast<uint32_t*>(smem), tsh, stamps ? stamps + 4 : nullptr);
  __syncthreads();
  if (tid == 0) {
    s.tickets[pair] = 0u;
    if (a.mode & kStepDecode) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __threadfence();
      asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a.ready + pair), "r"(1u) : "memory");
    }
  }
}

template <int G>
__global__ void __launch_bounds__(kDecThreads, kCtasPerSm)
    step_kernel(const StepArgs a, const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzled TMA boxes want 1024-byte aligned destinations.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ DecodeShared dsh;
  __shared__ TopkShared tsh;
  __shared__ __align__(8) uint64_t key_bar;
  __shared__ int sh_item;
  __shared__ int sh_last;
  const int tid = threadIdx.x;
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&dsh.full_bar[s], 1);
      mbar_init(&dsh.empty_bar[s], kDecConsumerWarps);
    }
    mbar_init(&key_bar, 1);
    mbar_init(&dsh.merge_bar, 1);
    dsh.merge_phase = 0;
    fence_barrier_init();
  }
  if (tid == kDecConsumerWarps * 32 && (a.mode & kStepDecode)) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_k) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_v) : "memory");
  }
#ifdef NOSA_TRACE
  if (tid == 0) {
    dsh.t_flag = 0;
    for (int n = 0; n < 8; ++n) dsh.t_issue[n] = dsh.t_full[n] = dsh.t_done[n] = 0;
    for (int n = 0; n < 6; ++n) dsh.t_merge[n] = 0;
  }
#endif
  grid_dependency_wait();
  allow_dependents();
  __syncthreads();
  uint32_t ring_n = 0, key_phase = 0;
  for (;;) {
    if (tid == 0) sh_item = static_cast<int>(atomicAdd(a.work, 1u));
    __syncthreads();
    const int item = sh_item;
    if (item >= a.n_items) break;
#ifdef NOSA_TRACE
    const uint64_t tr_start = global_timer_ns();
    const long long tr_clk0 = clock64();
#endif
    if (item < a.n_score_items) {
#ifdef NOSA_TRACE
      score_item<G>(a, item, smem, &key_bar, key_phase, tsh, &sh_last, dsh.t_issue);
#else
      score_item<G>(a, item, smem, &key_bar, key_phase, tsh, &sh_last, nullptr);
#endif
    } else {
      const int d = item - a.n_score_items;
      decode_item(a.dec, &tm_k, &tm_v, d % a.pairs, d / a.pairs, (a.mode & kStepScore) ? a.ready + d % a.pairs : nullptr,
                  ring_n, smem, dsh);
    }
    // Shared memory written by this item's threads may next be written by TMA.
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
#ifdef NOSA_TRACE
    if (tid == 0) {
      const uint32_t k = atomicAdd(&g_trace_count, 1u);
      if (k < kTraceCapacity) {
        uint32_t smid;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
        TraceRecord rec{blockIdx.x, smid, static_cast<uint32_t>(item), static_cast<uint32_t>(clock64() - tr_clk0),
                        tr_start, dsh.t_flag, global_timer_ns()};
        for (int n = 0; n < 8; ++n) {
          rec.issue[n] = dsh.t_issue[n] ? static_cast<uint32_t>(dsh.t_issue[n] - tr_start) : 0u;
          rec.full[n] = dsh.t_full[n] ? static_cast<uint32_t>(dsh.t_full[n] - tr_start) : 0u;
          rec.done[n] = dsh.t_done[n] ? static_cast<uint32_t>(dsh.t_done[n] - tr_start) : 0u;
          dsh.t_issue[n] = dsh.t_full[n] = dsh.t_done[n] = 0;
        }
        for (int n = 0; n < 6; ++n) {
          rec.merge[n] = dsh.t_merge[n] ? static_cast<uint32_t>(dsh.t_merge[n] - tr_start) : 0u;
          dsh.t_merge[n] = 0;
        }
        g_trace[k] = rec;
      }
      dsh.t_flag = 0;
    }
#endif
  }
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(a.work + 1, 1u) == gridDim.x - 1) {
      a.work[0] = 0u;
      a.work[1] = 0u;
    }
  }
}

// Selection only, from caller-provided block scores: one CTA per pair.
__global__ void __launch_bounds__(kSelOnlyThreads) select_only_kernel(const SelectArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ TopkShared sh;
  const int pair = blockIdx.y;
  const int i = pair / a.hkv;
  grid_dependency_wait();
  allow_dependents();
  const int L = a.seq_len[i];
  if (L < 1 || L > a.max_seq_len) {
    if (threadIdx.x == 0) set_status(a.status, L < 1 ? NOSA_DEV_BAD_LENGTH : NOSA_DEV_MAX_LEN);
    write_empty_selection(a, pair, kSelOnlyThreads);
    return;
  }
  const int ncand = static_cast<int>(n_candidates(L, a.local_blocks));
  select_topk<kSelOnlyThreads>(a.bs_in + static_cast<int64_t>(pair) * a.nb_in, false, ncand, a.topk,
                               a.sel_idx + static_cast<int64_t>(pair) * a.topk, a.sel_cnt + pair,
                               reinterpret_cast<uint32_t*>(smem), sh);
}

// A bounded wait on an mbarrier that nothing ever arrives on: exercises the
// timeout path (status bit set, kernel returns) without faulting or hanging.
__global__ void wait_selftest_kernel(uint32_t* status, uint32_t max_iters) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, status, max_iters, 1000u);
}

constexpr int kStepSmem = kRingBytes + 1024;

template <int G>
int resident_ctas() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int per_sm = 0, sms = 0;
    cudaFuncSetAttribute(step_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kStepSmem);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, step_kernel<G>, kDecThreads, kStepSmem) != cudaSuccess ||
        per_sm < 1)
      per_sm = 1;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 1;
    cached[dev] = per_sm * sms;
  }
  return cached[dev];
}

template <int G>
cudaError_t launch_step_g(const StepArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v, cudaStream_t stream) {
  if (a.n_items <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(step_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kStepSmem);
  if (e != cudaSuccess) return e;
  const int grid = min(a.n_items, resident_ctas<G>());
  return launch_overlapped(step_kernel<G>, dim3(grid), dim3(kDecThreads), kStepSmem, stream, a, tm_k, tm_v);
}

}  // namespace

int step_resident_ctas(int group) {
  switch (group) {
    case 1: return resident_ctas<1>();
    case 2: return resident_ctas<2>();
    case 4: return resident_ctas<4>();
    case 8: return resident_ctas<8>();
    case 16: return resident_ctas<16>();
    default: return 0;
  }
}

cudaError_t launch_step(const StepArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v, cudaStream_t stream) {
  switch (a.dec.group) {
    case 1: return launch_step_g<1>(a, tm_k, tm_v, stream);
    case 2: return launch_step_g<2>(a, tm_k, tm_v, stream);
    case 4: return launch_step_g<4>(a, tm_k, tm_v, stream);
    case 8: return launch_step_g<8>(a, tm_k, tm_v, stream);
    case 16: return launch_step_g<16>(a, tm_k, tm_v, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_select_only(const SelectArgs& a, cudaStream_t stream) {
  if (a.batch * a.hkv == 0) return cudaSuccess;
  const int smem = ((a.nb_in * 4 + 127) / 128) * 128;
  cudaError_t e = cudaFuncSetAttribute(select_only_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_overlapped(select_only_kernel, dim3(1, a.batch * a.hkv), dim3(kSelOnlyThreads), smem, stream, a);
}

void decode_split_plan(int pairs, int max_tiles, int num_ctas, int* nsplit) {
  if (max_tiles < 1) max_tiles = 1;
  int ns = pairs > 0 ? num_ctas / pairs : 1;
  if (ns > max_tiles) ns = max_tiles;
  if (ns > kMaxSplits) ns = kMaxSplits;
  if (ns < 1) ns = 1;
  *nsplit = ns;
}

#ifdef NOSA_TRACE
extern "C" __attribute__((visibility("default"))) int nosa_trace_read(void* host, int max_records) {
  uint32_t n = 0;
  if (cudaMemcpyFromSymbol(&n, g_trace_count, sizeof n) != cudaSuccess) return -1;
  if (n > static_cast<uint32_t>(max_records)) n = static_cast<uint32_t>(max_records);
  if (n > kTraceCapacity) n = kTraceCapacity;
  if (n && cudaMemcpyFromSymbol(host, g_trace, n * sizeof(TraceRecord)) != cudaSuccess) return -1;
  const uint32_t zero = 0;
  cudaMemcpyToSymbol(g_trace_count, &zero, sizeof zero);
  return static_cast<int>(n);
}
#endif

cudaError_t launch_wait_selftest(uint32_t* status, uint32_t max_iters, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, max_iters);
  return cudaGetLastError();
}

}  // namespace nosa
