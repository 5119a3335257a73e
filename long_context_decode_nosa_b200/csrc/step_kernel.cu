// The decode step: one kernel launch, one thread-block cluster of C CTAs per
// (sequence, KV head) pair.
//
// What a step computes ("NOSA-1B 性能基准全解析" (wmrh.cn) §三.2 / §三.3;
// "从论文到代码：手把手教你理解NOSA-8B的高效注意力机制实现" (nzsm.cn) item 2):
// append the new token's K/V rows and pool the window it completes; score
// the pooled keys with the group's queries and reduce them to block scores;
// select the top-k blocks; attend exactly over the selected blocks and the
// local window.  Any subset of the three parts runs (kStepScore,
// kStepDecode, kStepAppend), so the same kernel serves the fused step and
// the separate selection / attention entry points.
//
// Work split inside a cluster (rank r of C):
//   * scoring chunks k = r, r + C, ... (15 blocks = 61 pooled rows each);
//   * attention tiles t = r, r + C, ... of the pair's tile list (the local
//     blocks, then the selected blocks in ascending order).
// Roles inside a CTA (192 threads):
//   * warps 0-3, consumers: tensor-core scoring of a staged chunk (block
//     rule, block scores sent to every CTA of the cluster through
//     distributed shared memory), then the attention tiles (online softmax
//     per warp);
//   * warp 4, producer: issues every TMA copy of the CTA in job order --
//     scoring chunks, local tiles, selected tiles (after the selection) --
//     into a ring of 32 KB stages (full / empty mbarriers); with INT8 caches
//     a stage carries two tiles (half the bytes each) and their scale rows;
//   * warp 5, selector: pools the window completed by the new token (rank
//     0), waits until the block scores of the whole pair have arrived, runs
//     the exact top-k with the consumers (the selection group: a bucket
//     select with the keys in registers -- up to 7 per thread, 13 with one
//     CTA per SM -- or a radix select above that; alone when the block
//     scores are kept in global memory) -- every CTA computes the same
//     selection, so no second exchange is needed -- and hands the selected
//     blocks to the producer; rank 0 writes the selection out.
// Merge: each CTA merges its four warps into one partial (O, m, l) and
// pushes it, slice by slice, into the receive buffers of the cluster's CTAs
// (CTA r owns output slice r) with st.async, whose bytes complete on the
// receiver's mbarrier; once its slice has arrived, CTA r combines the C
// partials from its own shared memory, in rank order.  No cluster barrier
// ends the kernel: a CTA only waits for what is pushed into it.
//
// No global-memory flags, tickets or work queues: the only cross-CTA
// traffic is inside the cluster, and every wait is bounded (status bit
// NOSA_DEV_TIMEOUT), so a launch always finishes.
#include "decode_device.cuh"
#include "kv_int8.cuh"
#include "nosa_common.cuh"
#include "nosa_kernels.h"
#include "pool_device.cuh"
#include "select_device.cuh"

#include <cstdio>
#include <cstdlib>
#include <mutex>

namespace nosa {

#ifdef NOSA_TRACE
// Instrumented builds only (-DNOSA_TRACE): one record per CTA of the step
// kernel with %globaltimer stamps of its phases.
struct TraceRecord {
  uint32_t pair, rank, smid, csize;
  uint64_t t[24];  // see the NOSA_STAMP call sites
};
constexpr int kTraceCapacity = 1 << 16;
__device__ TraceRecord g_trace[kTraceCapacity];
__device__ uint32_t g_trace_count;
#define NOSA_STAMP(k) (sh.tr[k] = global_timer_ns())
#else
#define NOSA_STAMP(k) ((void)0)
#endif

namespace {

constexpr int kProducerWarp = kConsumerWarps;            // 4
constexpr int kSelectorWarp = kConsumerWarps + 1;        // 5
constexpr int kStepThreads = (kConsumerWarps + 2) * 32;  // 192
constexpr int kConsumerThreads = kConsumerWarps * 32;    // 128
constexpr int kCtasPerSm = 2;
constexpr int kSelOnlyThreads = 256;

// Paths of the step kernel kept out of line, so that they do not sit in the
// middle of the code every launch runs: the selector's top-k over block
// scores in global memory (very long sequences only), the selection group's
// radix select and the bucket selects of more than two keys per thread (the
// two-key one, the small-batch case, stays inline), and the pooling of the
// window the new token completes (one warp of one CTA per pair, once per
// launch, off the scoring chain).  Each runs at most once per launch.
__device__ __noinline__ void select_spilled(const float* scores, int ncand, int topk, int32_t* sel_row,
                                            int32_t* sel_cnt, int lane) {
  warp_topk_mem(scores, true, ncand, topk, sel_row, sel_cnt, lane);
}
__device__ __noinline__ void select_radix(const float* scores, int ncand, int topk, int32_t* sel_row,
                                          int32_t* sel_cnt, int gtid, GroupTopkShared& gtk, int bar_id) {
  group_topk<kConsumerThreads + 32>(scores, false, ncand, topk, sel_row, sel_cnt, gtid, gtk, bar_id);
}
template <int M>
__device__ __noinline__ void select_bucket(float* scores, int ncand, int topk, int32_t* sel_row, int32_t* sel_cnt,
                                           int gtid, GroupTopkShared& gtk, int bar_id, uint64_t* stamps) {
  bucket_topk<kConsumerThreads + 32, M>(scores, ncand, topk, sel_row, sel_cnt, gtid, gtk, bar_id, stamps);
}
__device__ __noinline__ void pool_new_window(const __nv_bfloat16* k_cache, int hkv, const KvRows& kv, int g,
                                             int64_t j, int64_t new_row, const uint2* knew, void* dst, bool bf16,
                                             int lane) {
  pool_window_warp(k_cache, hkv, kv, g, j, new_row, knew, dst, bf16, lane);
}

struct StepShared {
  uint64_t full_bar[kMaxStages];
  uint64_t empty_bar[kMaxStages];
  uint64_t scores_bar;  // completes when every CTA of the cluster has sent its block scores
  uint64_t sel_bar;     // completes when the selection is in shared memory (selector -> producer)
  uint64_t recv_bar;    // completes when every CTA of the cluster has pushed its share of this CTA's output slice
  int stage_blk[kMaxStages][2];   // the stage's tiles (second: kAbsentTile when one)
  int stage_soff[kMaxStages][2];  // INT8: position of the tile's first scale in its scale slot
  int sel_count;
  GroupTopkShared gtk;      // the selection group's exchange (consumers + selector)
#ifdef NOSA_TRACE
  uint64_t tr[24];
#endif
};

// A stage slot left empty (INT8 caches: a job with one tile).
constexpr int kAbsentTile = -2;

// Shared memory of the step kernel (dynamic, from a 1024-byte aligned base):
//   ring  kRingBytes                      kStages stages of 32 KB
//   sel   round16(4 * topk) bytes         the pair's selection (ascending block indices)
//   bsm   4 * ncand_max bytes             the pair's block scores (unless kept in global memory)
//   recv  recv_bytes<G>(C)                the partials the cluster's CTAs push for this CTA's
//                                         share of the output (see the merge); before that,
//                                         two G x kScoreStride float buffers of window scores
//                                         (chunks alternate between them)
//   scl   S x kScaleStageBytes            INT8 caches: the scale rows of each stage's tiles
// The window-score buffers can share the receive buffer: another CTA pushes
// into it only after its selection, i.e. after every CTA of the cluster --
// this one too -- has sent its last block score, the last use of them.
template <int G>
__host__ __device__ constexpr int ssm_floats() {
  return G * kScoreStride;
}
__host__ __device__ constexpr int round16(int x) { return (x + 15) & ~15; }
// Output float4s of a pair and the receive buffer of a cluster of C CTAs:
// C x ceil(items / C) pushed float4s plus C x G row maxima and C x G row
// sums, and at least the two window-score buffers.  Sized for the launch's
// own cluster size (the host sizes shared memory for an upper bound of it).
template <int G>
__host__ __device__ constexpr int out_items() {
  return G * kHeadDim / 4;
}
template <int G>
__host__ __device__ constexpr int recv_bytes(int C) {
  return (out_items<G>() + C) * 16 + 2 * C * G * 4 > 8 * ssm_floats<G>()
             ? (out_items<G>() + C) * 16 + 2 * C * G * 4
             : 8 * ssm_floats<G>();
}

// Output float4s [f0, f1) of CTA `rank`'s slice of a pair's output.
template <int G>
__host__ __device__ inline void out_slice(int rank, int C, int* f0, int* f1) {
  const int slice = (out_items<G>() + C - 1) / C;
  *f0 = rank * slice < out_items<G>() ? rank * slice : out_items<G>();
  *f1 = *f0 + slice < out_items<G>() ? *f0 + slice : out_items<G>();
}
// Bytes the cluster's CTAs push into CTA `rank` in the merge.
template <int G>
__device__ inline uint32_t recv_slice_bytes(int rank, int C) {
  int f0, f1;
  out_slice<G>(rank, C, &f0, &f1);
  if (f1 <= f0) return 0u;
  constexpr int kVec = kHeadDim / 4;
  const int rows = (f1 - 1) / kVec - f0 / kVec + 1;
  return static_cast<uint32_t>(C * (16 * (f1 - f0) + 8 * rows));
}

// Offset (from the aligned base) of the INT8 scale slots: after the receive
// buffer of a cluster of C CTAs, 128-byte aligned.
template <int G, int S>
__host__ __device__ inline int step_scale_offset(const StepArgs& a, int C) {
  const int end = S * kStageBytes + round16(4 * a.topk) + (a.bs_spill ? 0 : round16(4 * max(a.ncand_max, 1))) +
                  recv_bytes<G>(C);
  return (end + 127) & ~127;
}

// Named barrier of the four consumer warps.
__device__ inline void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory"); }

// Named barrier of the consumer warps that also returns whether `v` holds in
// all of them (so that they leave a loop together).
__device__ inline bool consumer_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kConsumerThreads)
      : "memory");
  return r != 0;
}

// The selection group: the consumer warps and the selector warp (160
// threads, named barrier 2) select together once the block scores are in.
constexpr int kSelectThreads = kConsumerThreads + 32;
constexpr int kSelectBar = 2;

__device__ inline bool select_group_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kSelectBar), "n"(kSelectThreads)
      : "memory");
  return r != 0;
}

// Cross-warp merge scratch (in the drained ring): per warp O rows with a
// padded stride (bank-conflict free float2 stores), row max and row sum.
constexpr int kMoStride = kHeadDim + 8;
template <int G>
struct MergeLayout {
  static constexpr int kMo = 0;                                      // [4][G][kMoStride]
  static constexpr int kMm = kMo + kConsumerWarps * G * kMoStride;   // [4][G]
  static constexpr int kMl = kMm + kConsumerWarps * G;               // [4][G]
};
static_assert((MergeLayout<kMaxGroup>::kMl + kConsumerWarps * kMaxGroup) * 4 <= 2 * kStageBytes,
              "merge scratch must fit in the smallest ring (2 stages)");

// Ring depths of a launch: the smaller one for two CTAs per SM, the larger
// for one.  An INT8 stage carries two tiles plus their scale rows, so its
// rings are 2 and 4 stages (4 and 8 tiles in flight): a 3-stage INT8 ring
// with the scale slots no longer fits two CTAs per SM at long contexts.
template <bool Q8>
struct Rings {
  static constexpr int kLo = Q8 ? 2 : kMinStages;
  static constexpr int kHi = Q8 ? 4 : kMaxStages;
};

// S = ring stages: 3 (two CTAs per SM) or 6 (one CTA per SM, twice the
// bytes in flight per CTA); with INT8 caches (Q8) 2 or 4 stages of two tiles.
// Q8: the K/V caches are INT8 (codes + per-row scales).
// P: fp32 pooled keys scored two chunks per pass after the first (the deep
// ring, for CTAs with many scoring chunks).
template <int G, int S, bool Q8, bool P = false>
__global__ void __launch_bounds__(kStepThreads, S == Rings<Q8>::kHi ? 1 : kCtasPerSm)
    step_kernel(const StepArgs a, const __grid_constant__ StepMaps maps) {
  constexpr int kRing = S * kStageBytes;
  const CUtensorMap* tm_k = &maps.k;
  const CUtensorMap* tm_v = &maps.v;
  const CUtensorMap* tm_p = &maps.p;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzled TMA boxes want 1024-byte aligned destinations.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int32_t* sel_list = reinterpret_cast<int32_t*>(smem + kRing);
  float* bsm = reinterpret_cast<float*>(smem + kRing + round16(4 * a.topk));
  float* recv = reinterpret_cast<float*>(smem + kRing + round16(4 * a.topk) +
                                         (a.bs_spill ? 0 : round16(4 * max(a.ncand_max, 1))));
  __shared__ StepShared sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t C = cluster_nctarank(), rank = cluster_ctarank();
  const int pair = static_cast<int>(cluster_id_x());
  const bool scoring = (a.mode & kStepScore) != 0;
  const bool decoding = (a.mode & kStepDecode) != 0;
  const bool appending = (a.mode & kStepAppend) != 0;
  const bool spill = a.bs_spill != nullptr;

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) {
      mbar_init(&sh.full_bar[s], 1);
      mbar_init(&sh.empty_bar[s], kConsumerWarps);
    }
    // Block scores in shared memory arrive as st.async transactions counted
    // in bytes against the selector's one arrival; in global memory (spill)
    // every CTA of the cluster arrives once.
    mbar_init(&sh.scores_bar, spill ? C : 1);
    mbar_init(&sh.sel_bar, 1);
    mbar_init(&sh.recv_bar, 1);
    fence_barrier_init();
#ifdef NOSA_TRACE
    for (int k = 0; k < 24; ++k) sh.tr[k] = 0;
    NOSA_STAMP(0);
#endif
  }
  __syncthreads();
  if (warp == kProducerWarp && lane == 0) {
    if (scoring) asm volatile("prefetch.tensormap [%0];" ::"l"(tm_p) : "memory");
    if (decoding) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(tm_k) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(tm_v) : "memory");
      if (Q8) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.ks) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&maps.vs) : "memory");
      }
    }
  }
  grid_dependency_wait();
  allow_dependents();
#ifdef NOSA_TRACE
  if (tid == 0) NOSA_STAMP(6);
#endif
  const int i = pair / a.hkv, g = pair % a.hkv;
  const __nv_bfloat16* q_group = a.q + (static_cast<int64_t>(i) * a.hq + static_cast<int64_t>(g) * G) * kHeadDim;
  // This CTA's first scoring chunk goes out before the sequence length is
  // read: its rows depend only on the pair, so chunk `rank` is issued
  // whenever a sequence of max_seq_len tokens has it; if the sequence turns
  // out shorter the consumers release the stage unscored.  Meanwhile the
  // selector warp pulls the group's queries into L1.
  const int nchunks_max =
      scoring && a.comp_out == nullptr && a.seq_of == nullptr ? (a.ncand_max + kChunkBlocks - 1) / kChunkBlocks : 0;
  const bool early_chunk = static_cast<int>(rank) < nchunks_max;
  if (early_chunk && warp == kProducerWarp && lane == 0) {
    const int row0 = (i * a.hkv + g) * a.nc_cap + kChunkBlocks * kWindowsPerBlock * static_cast<int>(rank) - 1;
    const uint64_t policy = l2_evict_first_policy();
    if (a.pooled_bf16) {
      mbar_arrive_expect_tx(&sh.full_bar[0], kScoreTxBytesBf16);
      tma_load_keys(smem, tm_p, 0, row0, &sh.full_bar[0], policy);
      tma_load_keys(smem + kScoreSlotBytes, tm_p, 64, row0, &sh.full_bar[0], policy);
    } else {
      mbar_arrive_expect_tx(&sh.full_bar[0], kScoreTxBytes);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tma_load_keys(smem + c * kScoreSlotBytes, tm_p, c * kBoxCols, row0, &sh.full_bar[0], policy);
    }
#ifdef NOSA_TRACE
    NOSA_STAMP(13);
#endif
  }
  if (warp == kSelectorWarp && lane < 2 * G)
    asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const uint8_t*>(q_group) + 128 * lane) : "memory");

  // ---------------------------------------------------------------- geometry
  // (identical in every CTA of the cluster)
  // Entry i is one query (its own length L, q, selection and output); si is
  // the sequence whose cache and pooled keys it reads (si = i except for
  // the multi-query prefill, where many entries share one sequence).
  const bool uses_cache = decoding || appending;
  const int L = a.seq_len[i];
  const int si = a.seq_of ? a.seq_of[i] : i;
  const bool paged = a.page_table != nullptr;
  const int64_t start_i = uses_cache && !paged ? a.seq_start[si] : 0;  // issued with the length load
  const bool bad_len = L < 1 || L > a.max_seq_len;
#ifdef NOSA_TRACE
  if (warp == kProducerWarp && lane == 0 && !bad_len) NOSA_STAMP(8);
#endif
  const int64_t seq_base = bad_len ? 0 : start_i;
  KvRows kv;
  kv.base = seq_base;
  kv.pages = paged ? a.page_table + static_cast<int64_t>(si) * a.max_pages : nullptr;
  kv.num_pages = a.cache_rows / kPageTokens;
  const bool bad_rows = uses_cache && !bad_len &&
                        (paged ? static_cast<int64_t>(L) > static_cast<int64_t>(a.max_pages) * kPageTokens
                               : seq_base < 0 || seq_base + L > a.cache_rows);
  const int Lv = bad_len ? 0 : L;
  const int nb = static_cast<int>(n_blocks(Lv));
  const int ncand = static_cast<int>(n_candidates(Lv, a.local_blocks));
  const int nloc = nb - ncand;
  const int64_t nc_all = n_windows(Lv);
  const int64_t nc = nc_all < a.nc_cap ? nc_all : a.nc_cap;
  const int cnt_max = min(a.topk, ncand);
  const int nchunks = scoring ? ((a.comp_out ? nb : ncand) + kChunkBlocks - 1) / kChunkBlocks : 0;
  int cnt = cnt_max;
  if (decoding && !scoring && !bad_len) {
    cnt = a.sel_cnt[pair];
    if (cnt < 0 || cnt > cnt_max) {
      if (rank == 0 && tid == 0) set_status(a.status, NOSA_DEV_BAD_COUNT);
      cnt = cnt < 0 ? 0 : cnt_max;
    }
  }
  const int ntiles = decoding && !bad_rows ? nloc + cnt : 0;
  if (rank == 0 && tid == 0) {
    if (bad_len) set_status(a.status, L < 1 ? NOSA_DEV_BAD_LENGTH : NOSA_DEV_MAX_LEN);
    if (bad_rows) set_status(a.status, NOSA_DEV_CACHE_ROWS);
    if (scoring && nc_all > a.nc_cap) set_status(a.status, NOSA_DEV_NC_CAP);
  }
  // The selector expects the pair's block-score bytes before this CTA joins
  // cluster barrier phase 1, so no other CTA can send one before.
  if (scoring && !spill && warp == kSelectorWarp && lane == 0)
    mbar_arrive_expect_tx(&sh.scores_bar, 4u * static_cast<uint32_t>(ncand));
  // The same for this CTA's output slice: C x (16 bytes per float4 of the
  // slice + 8 bytes (row max, row sum) per row the slice touches).
  if (decoding && warp == kSelectorWarp && lane == 0)
    mbar_arrive_expect_tx(&sh.recv_bar, recv_slice_bytes<G>(static_cast<int>(rank), static_cast<int>(C)));
  // Cluster barrier phase 1: this CTA's barriers exist (and expect their
  // bytes).  Each thread waits on it before its first access to another
  // CTA's shared memory.
  cluster_arrive();
#ifdef NOSA_TRACE
  if (warp == kProducerWarp && lane == 0) NOSA_STAMP(23);
#endif

  // Who selects: the selection group when the block scores are in shared
  // memory, else (block scores in global memory) the selector alone.
  const bool group_selects = scoring && !spill;
  // Top-k of the pair by the selection group, from the block scores in
  // shared memory; every member calls it (gtid = its index in the group).
  // The decision to give up after a timed-out wait is taken together.
  auto group_select = [&](int gtid) {
    bool ok = mbar_wait_cluster(&sh.scores_bar, 0, a.status);
    ok = select_group_all(ok);
#ifdef NOSA_TRACE
    if (gtid == kConsumerThreads) NOSA_STAMP(3);
#endif
    if (ok) {
#ifdef NOSA_TRACE
      uint64_t* stamps = &sh.tr[14];
#else
      uint64_t* stamps = nullptr;
#endif
      // Bucket select, the candidates held in registers: up to 7 per thread,
      // and with one CTA per SM (registers to spare) up to 13, every count
      // shared memory holds; the radix select beyond.
      if (ncand <= 2 * kSelectThreads)
        bucket_topk<kSelectThreads, 2>(bsm, ncand, a.topk, sel_list, &sh.sel_count, gtid, sh.gtk, kSelectBar, stamps);
      else if (ncand <= 7 * kSelectThreads)
        select_bucket<7>(bsm, ncand, a.topk, sel_list, &sh.sel_count, gtid, sh.gtk, kSelectBar, stamps);
      else if constexpr (S == Rings<Q8>::kHi)
        select_bucket<13>(bsm, ncand, a.topk, sel_list, &sh.sel_count, gtid, sh.gtk, kSelectBar, stamps);
      else
        select_radix(bsm, ncand, a.topk, sel_list, &sh.sel_count, gtid, sh.gtk, kSelectBar);
    } else {
      for (int x = gtid; x < a.topk; x += kSelectThreads) sel_list[x] = -1;
      if (gtid == 0) sh.sel_count = 0;
    }
    group_bar(kSelectBar, kSelectThreads);
  };

  AttnState att;
  if (warp == kProducerWarp) {
    // ---------------------------------------------------------------- producer
    const uint64_t policy = l2_evict_first_policy();
    uint32_t r = early_chunk ? 1u : 0u;  // jobs issued
    bool ok = true;
    // Lane 0 waits for the stage, then issues the job's boxes.
    auto issue = [&](auto&& body) {
      int good = 1;
      if (lane == 0) {
        const int s = static_cast<int>(r % S);
        if (r >= static_cast<uint32_t>(S) && !mbar_wait(&sh.empty_bar[s], ((r / S) - 1) & 1u, a.status))
          good = 0;
        else
          body(s, smem + s * kStageBytes);
      }
      ok = __shfl_sync(0xffffffffu, good, 0) != 0;
      if (ok) ++r;
    };
    const int row_base = (si * a.hkv + g) * a.nc_cap;  // first pooled row of the pair (host: rows < 2^31)
    for (int k = static_cast<int>(rank) + (early_chunk ? static_cast<int>(C) : 0); k < nchunks && ok;
         k += static_cast<int>(C)) {
      issue([&](int s, uint8_t* st) {
        const int row0 = row_base + kChunkBlocks * kWindowsPerBlock * k - 1;
        if (a.pooled_bf16) {
          mbar_arrive_expect_tx(&sh.full_bar[s], kScoreTxBytesBf16);
          tma_load_keys(st, tm_p, 0, row0, &sh.full_bar[s], policy);
          tma_load_keys(st + kScoreSlotBytes, tm_p, 64, row0, &sh.full_bar[s], policy);
        } else {
          mbar_arrive_expect_tx(&sh.full_bar[s], kScoreTxBytes);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tma_load_keys(st + c * kScoreSlotBytes, tm_p, c * kBoxCols, row0, &sh.full_bar[s], policy);
        }
      });
    }
#ifdef NOSA_TRACE
    if (lane == 0) NOSA_STAMP(1);
#endif
    // The first row of a tile: in a paged cache its page's, read from the
    // page table (an invalid page rejects the tile).  Resolved by the whole
    // warp, 32 tiles at a time (one parallel round trip for the table).
    auto tile_row = [&](int blk, int& out_blk) -> int {
      out_blk = blk;
      if (blk < 0) return 0;
      if (!paged) return static_cast<int>(seq_base + static_cast<int64_t>(blk) * kBlock);
      const int32_t pg = kv.pages[blk];
      if (pg < 0 || pg >= kv.num_pages) {
        set_status(a.status, NOSA_DEV_BAD_INDEX);
        out_blk = -1;
        return 0;
      }
      return pg * kPageTokens;
    };
    // One job: a tile (bf16: four {64 dims, 1 head, 64 tokens} boxes), or
    // with INT8 caches up to two tiles (a {128 bytes, 1 head, 64 tokens} box
    // of K and of V each, plus their 68-scale rows).
    auto issue_job = [&](int blk0, int row0, int blk1, int row1) {
      issue([&](int s, uint8_t* st) {
        sh.stage_blk[s][0] = blk0;
        sh.stage_blk[s][1] = blk1;
        if constexpr (Q8) {
          uint8_t* scl = smem + step_scale_offset<G, S>(a, static_cast<int>(C)) + s * kScaleStageBytes;
          const int n = blk1 == kAbsentTile ? 1 : 2;
          mbar_arrive_expect_tx(&sh.full_bar[s], n * kTileTxBytesInt8);
          for (int x = 0; x < n; ++x) {
            const int row = x ? row1 : row0;
            sh.stage_soff[s][x] = row & 3;
            tma_load_box(st + 2 * x * kTileBytesInt8, tm_k, 0, g, row, &sh.full_bar[s], policy);
            tma_load_box(st + (2 * x + 1) * kTileBytesInt8, tm_v, 0, g, row, &sh.full_bar[s], policy);
            tma_load_keys(scl + 2 * x * kScaleSlot, &maps.ks, row & ~3, g, &sh.full_bar[s], policy);
            tma_load_keys(scl + (2 * x + 1) * kScaleSlot, &maps.vs, row & ~3, g, &sh.full_bar[s], policy);
          }
        } else {
          (void)blk1;
          (void)row1;
          mbar_arrive_expect_tx(&sh.full_bar[s], kTileTxBytes);
          tma_load_box(st, tm_k, 0, g, row0, &sh.full_bar[s], policy);
          tma_load_box(st + kHalfBytes, tm_k, 64, g, row0, &sh.full_bar[s], policy);
          tma_load_box(st + 2 * kHalfBytes, tm_v, 0, g, row0, &sh.full_bar[s], policy);
          tma_load_box(st + 3 * kHalfBytes, tm_v, 64, g, row0, &sh.full_bar[s], policy);
        }
      });
    };
    constexpr int kPerJob = Q8 ? 2 : 1;
    const int Ci = static_cast<int>(C), ri = static_cast<int>(rank);
    // Local tiles t = rank, rank + C, ... < nloc: known at once.
    {
      const int tend = min(nloc, ntiles);
      int my_blk = -1, my_row = 0, n = 0;
      for (int t = ri; t < tend && ok; t += kPerJob * Ci, n += kPerJob) {
        if ((n & 31) == 0) {
          const int tl = t + Ci * lane;
          my_row = tile_row(tl < tend ? ncand + tl : -1, my_blk);
        }
        const int blk = __shfl_sync(0xffffffffu, my_blk, n & 31);
        const int row = __shfl_sync(0xffffffffu, my_row, n & 31);
        const bool two = Q8 && t + Ci < tend;
        int blk1 = kAbsentTile, row1 = 0;
        if constexpr (Q8) {
          blk1 = __shfl_sync(0xffffffffu, my_blk, (n + 1) & 31);
          row1 = __shfl_sync(0xffffffffu, my_row, (n + 1) & 31);
        }
        if (appending && a.k_new != nullptr && (t == nloc - 1 || (two && t + Ci == nloc - 1))) {
          // This job holds token L-1: write the new K/V rows first and order
          // them before the tile's TMA read (same CTA, async proxy).
          if (kv.page_ok(L - 1)) {
            const int64_t src = static_cast<int64_t>(i) * a.hkv + g;
            if constexpr (Q8) {
              const int64_t r = kv.row(L - 1);
              store_int8_row_warp(Int8Cache{reinterpret_cast<int8_t*>(a.k_cache), a.k_scale, a.scale_stride}, a.hkv,
                                  r, g, reinterpret_cast<const uint2*>(a.k_new + src * kHeadDim), lane);
              store_int8_row_warp(Int8Cache{reinterpret_cast<int8_t*>(a.v_cache), a.v_scale, a.scale_stride}, a.hkv,
                                  r, g, reinterpret_cast<const uint2*>(a.v_new + src * kHeadDim), lane);
            } else {
              const int64_t row_w = kv.row(L - 1) * a.hkv + g;
              reinterpret_cast<uint2*>(a.k_cache + row_w * kHeadDim)[lane] =
                  reinterpret_cast<const uint2*>(a.k_new + src * kHeadDim)[lane];
              reinterpret_cast<uint2*>(a.v_cache + row_w * kHeadDim)[lane] =
                  reinterpret_cast<const uint2*>(a.v_new + src * kHeadDim)[lane];
            }
            asm volatile("fence.proxy.async.global;" ::: "memory");
          }
          __syncwarp();
        }
        issue_job(blk, row, two ? blk1 : kAbsentTile, row1);
      }
    }
    // Selected tiles t = nloc + x, t = rank (mod C): after the selection.
    {
      const int t0 = nloc + ((ri - nloc % Ci) % Ci + Ci) % Ci;
      if (t0 < ntiles && ok) {
        int got = 0;
        if (lane == 0) got = mbar_wait(&sh.sel_bar, 0, a.status) ? 1 : 0;
        const bool sel_ok = __shfl_sync(0xffffffffu, got, 0) != 0;
        int my_blk = -1, my_row = 0, n = 0;
        for (int t = t0; t < ntiles && ok; t += kPerJob * Ci, n += kPerJob) {
          if ((n & 31) == 0) {
            const int tl = t + Ci * lane;
            int blk = -1;
            if (tl < ntiles && sel_ok) {
              blk = sel_list[tl - nloc];
              if (blk < 0 || blk >= ncand) {
                set_status(a.status, NOSA_DEV_BAD_INDEX);
                blk = -1;
              }
            }
            my_row = tile_row(blk, my_blk);
          }
          const bool two = Q8 && t + Ci < ntiles;
          const int blk0 = __shfl_sync(0xffffffffu, my_blk, n & 31);
          const int row0 = __shfl_sync(0xffffffffu, my_row, n & 31);
          int blk1 = kAbsentTile, row1 = 0;
          if constexpr (Q8) {
            blk1 = __shfl_sync(0xffffffffu, my_blk, (n + 1) & 31);
            row1 = __shfl_sync(0xffffffffu, my_row, (n + 1) & 31);
          }
          issue_job(blk0, row0, two ? blk1 : kAbsentTile, row1);
        }
      }
    }
    // Every copy issued has landed before the ring is reused for the merge.
    if (lane == 0) {
      const uint32_t first = r > static_cast<uint32_t>(S) ? r - S : 0u;
      for (uint32_t n = first; n < r; ++n) mbar_wait(&sh.full_bar[n % S], (n / S) & 1u, a.status);
    }
    __syncwarp();
    cluster_wait();
  } else if (warp == kSelectorWarp) {
    // ---------------------------------------------------------------- selector
    cluster_wait();
    if (appending && rank == 0 && !bad_len && !bad_rows) {
      // Pool the window that token L-1 completes (it lies in the local
      // window, so this step's selection never reads it).
      const int64_t j = n_windows(L) - 1;
      if (j >= 0 && j >= n_windows(L - 1)) {
        if (j >= a.nc_cap) {
          if (lane == 0) set_status(a.status, NOSA_DEV_NC_CAP);
        } else {
          const uint2* knew = a.k_new ? reinterpret_cast<const uint2*>(
                                            a.k_new + (static_cast<int64_t>(i) * a.hkv + g) * kHeadDim)
                                      : nullptr;
          const int64_t at = ((static_cast<int64_t>(si) * a.hkv + g) * a.nc_cap + j) * kHeadDim;
          void* dst = a.pooled_bf16 ? static_cast<void*>(static_cast<__nv_bfloat16*>(a.pooled) + at)
                                    : static_cast<void*>(static_cast<float*>(a.pooled) + at);
          if (kv.page_ok(j * kPoolStride) && kv.page_ok(j * kPoolStride + kPoolKernel - 1)) {
            if constexpr (Q8)
              pool_window_warp_int8(Int8Cache{reinterpret_cast<int8_t*>(a.k_cache), a.k_scale, a.scale_stride}, a.hkv,
                                    kv, g, j, knew ? L - 1 : -1, knew, dst, a.pooled_bf16 != 0, lane);
            else
              pool_new_window(a.k_cache, a.hkv, kv, g, j, knew ? L - 1 : -1, knew, dst, a.pooled_bf16 != 0, lane);
          } else if (lane == 0)
            set_status(a.status, NOSA_DEV_BAD_INDEX);
        }
      }
    }
    if (scoring) {
      if (group_selects) {
        group_select(kConsumerThreads + lane);
      } else {
        const bool ok = mbar_wait_cluster(&sh.scores_bar, 0, a.status);
#ifdef NOSA_TRACE
        if (lane == 0) NOSA_STAMP(3);
#endif
        if (ok) {
          // Block scores in global memory: beyond the group's shared memory, so
          // more than any register-resident selection holds.
          select_spilled(a.bs_spill + static_cast<int64_t>(pair) * a.nb_spill, ncand, a.topk, sel_list,
                         &sh.sel_count, lane);
        } else {
          for (int t = lane; t < a.topk; t += 32) sel_list[t] = -1;
          if (lane == 0) sh.sel_count = 0;
        }
        __syncwarp();
      }
      if (rank == 0) {
        int32_t* dst = a.sel_idx + static_cast<int64_t>(pair) * a.topk;
        for (int t = lane; t < a.topk; t += 32) dst[t] = sel_list[t];
        if (lane == 0) a.sel_cnt[pair] = sh.sel_count;
      }
    } else if (decoding) {
      const int32_t* src = a.sel_idx + static_cast<int64_t>(pair) * a.topk;
      for (int t = lane; t < cnt; t += 32) sel_list[t] = src[t];
    }
    __syncwarp();
#ifdef NOSA_TRACE
    if (lane == 0) NOSA_STAMP(4);
#endif
    if (lane == 0) mbar_arrive(&sh.sel_bar);
  } else {
    // ---------------------------------------------------------------- consumers
    // Cluster barrier phase 1 is awaited just before the first access to
    // another CTA's shared memory (the first block-score send), so that the
    // first chunk is scored meanwhile.
    bool joined = false;
    auto join_cluster = [&] {
      if (!joined) cluster_wait();
      joined = true;
    };
    uint32_t r = 0;  // jobs consumed
    bool ok = true;
    if (scoring) {
      // Chunk jobs of this CTA: its chunks of the pair, or the early chunk
      // alone when the sequence is too short to have it.
      const int chunk_end = max(nchunks, early_chunk ? static_cast<int>(rank) + 1 : 0);
      if (static_cast<int>(rank) < chunk_end) {
        const bool bf16 = a.pooled_bf16 != 0;
        ScoreQ<G> qf;
        ScoreQBf16<G> qfb;
        if (bf16)
          load_score_q_bf16<G>(qfb, q_group, lane);
        else
          load_score_q<G>(qf, q_group, lane);
        if constexpr (!P) {
          for (int k = static_cast<int>(rank); k < chunk_end; k += static_cast<int>(C)) {
            const int s = static_cast<int>(r % S);
            const bool landed = consumer_all(mbar_wait(&sh.full_bar[s], (r / S) & 1u, a.status));
            if (!landed) {
              ok = false;
              break;
            }
            if (k >= nchunks) {  // the early chunk of a short sequence
              __syncwarp();
              if (lane == 0) mbar_arrive(&sh.empty_bar[s]);
              ++r;
              continue;
            }
#ifdef NOSA_TRACE
            if (tid == 0 && k == static_cast<int>(rank)) NOSA_STAMP(9);
            if (tid == 0 && k == static_cast<int>(rank + C)) NOSA_STAMP(20);
#endif
            // Chunks alternate between two window-score buffers: a buffer is
            // rewritten two chunks later, after every warp has passed the
            // next chunk's barrier and so has finished reading it.
            float* ssm = recv + ((k - static_cast<int>(rank)) / static_cast<int>(C) & 1) * ssm_floats<G>();
            if (bf16)
              score_stage_bf16<G>(qfb, smem_addr(smem + s * kStageBytes), ssm, a.scale, warp, lane);
            else
              score_stage<G>(qf, smem_addr(smem + s * kStageBytes), ssm, a.scale, warp, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.empty_bar[s]);
            ++r;
            consumer_sync();  // the chunk's window scores are complete
#ifdef NOSA_TRACE
            if (tid == 0 && k == static_cast<int>(rank)) NOSA_STAMP(10);
            if (tid == 0 && k == static_cast<int>(rank + C)) NOSA_STAMP(21);
#endif
            const int b0 = kChunkBlocks * k;
            const int nblk = min(kChunkBlocks, ncand - b0);
            if (a.comp_out) {
              // windows [60k, min(60k + 60, nc)); the row of window j is j - 60k + 1
              const int64_t j0 = static_cast<int64_t>(kChunkBlocks) * kWindowsPerBlock * k;
              constexpr int kWin = kChunkBlocks * kWindowsPerBlock;
              for (int t = tid; t < G * kWin; t += kConsumerThreads) {
                const int h = t / kWin, x = t % kWin;
                if (j0 + x < nc)
                  a.comp_out[(static_cast<int64_t>(i) * a.hq + static_cast<int64_t>(g) * G + h) * a.nc_cap + j0 + x] =
                      ssm[h * kScoreStride + x + 1];
              }
            }
            join_cluster();
            {
              // Every lane of block t's group holds its score: lane hl sends it
              // to CTAs hl, hl + kLanes, ... of the cluster.
              constexpr int kLanes = G < 8 ? G : 8;
              const int t = tid / kLanes, hl = tid % kLanes;
              float bscore;
              if (block_rule<G>(ssm, k, nblk, nc, tid, &bscore)) {
                if (!spill)
                  for (int d = hl; d < static_cast<int>(C); d += kLanes)
                    st_async_f32(map_shared_rank(smem_addr(bsm + b0 + t), static_cast<uint32_t>(d)), bscore,
                                 map_shared_rank(smem_addr(&sh.scores_bar), static_cast<uint32_t>(d)));
                if (hl == 0 && a.bs_out) a.bs_out[static_cast<int64_t>(pair) * a.nb_out + b0 + t] = bscore;
                if (hl == 0 && spill) a.bs_spill[static_cast<int64_t>(pair) * a.nb_spill + b0 + t] = bscore;
              }
            }
#ifdef NOSA_TRACE
            if (tid == 0 && k == static_cast<int>(rank)) NOSA_STAMP(19);
#endif
          }
        } else {
          // The block rule and the sends of chunk k from its window scores
          // (as in the single-chunk loop above).
          auto send_chunk = [&](int k, const float* ssm) {
            const int b0 = kChunkBlocks * k;
            const int nblk = min(kChunkBlocks, ncand - b0);
            if (a.comp_out) {
              const int64_t j0 = static_cast<int64_t>(kChunkBlocks) * kWindowsPerBlock * k;
              constexpr int kWin = kChunkBlocks * kWindowsPerBlock;
              for (int t = tid; t < G * kWin; t += kConsumerThreads) {
                const int h = t / kWin, x = t % kWin;
                if (j0 + x < nc)
                  a.comp_out[(static_cast<int64_t>(i) * a.hq + static_cast<int64_t>(g) * G + h) * a.nc_cap + j0 +
                             x] = ssm[h * kScoreStride + x + 1];
              }
            }
            join_cluster();
            constexpr int kLanes = G < 8 ? G : 8;
            const int t = tid / kLanes, hl = tid % kLanes;
            float bscore;
            if (block_rule<G>(ssm, k, nblk, nc, tid, &bscore)) {
              if (!spill)
                for (int d = hl; d < static_cast<int>(C); d += kLanes)
                  st_async_f32(map_shared_rank(smem_addr(bsm + b0 + t), static_cast<uint32_t>(d)), bscore,
                               map_shared_rank(smem_addr(&sh.scores_bar), static_cast<uint32_t>(d)));
              if (hl == 0 && a.bs_out) a.bs_out[static_cast<int64_t>(pair) * a.nb_out + b0 + t] = bscore;
              if (hl == 0 && spill) a.bs_spill[static_cast<int64_t>(pair) * a.nb_spill + b0 + t] = bscore;
            }
          };
          // The first chunk alone (scored as soon as it lands), then pairs of
          // chunks k, k + C into the two window-score buffers.  Every pass
          // starts with the consumers' barrier, after every warp has finished
          // reading the buffers of the pass before.
          float* const ssm2[2] = {recv, recv + ssm_floats<G>()};
          for (int k = static_cast<int>(rank); k < chunk_end;) {
            const bool two = k != static_cast<int>(rank) && k + static_cast<int>(C) < nchunks;
            const int s = static_cast<int>(r % S), s1 = static_cast<int>((r + 1) % S);
            bool landed = mbar_wait(&sh.full_bar[s], (r / S) & 1u, a.status);
            if (two) landed = mbar_wait(&sh.full_bar[s1], ((r + 1) / S) & 1u, a.status) && landed;
            if (!consumer_all(landed)) {
              ok = false;
              break;
            }
            if (k >= nchunks) {  // the early chunk of a short sequence
              __syncwarp();
              if (lane == 0) mbar_arrive(&sh.empty_bar[s]);
              ++r;
              k += static_cast<int>(C);
              continue;
            }
            if (two) {
              const uint32_t st[2] = {smem_addr(smem + s * kStageBytes), smem_addr(smem + s1 * kStageBytes)};
              score_stage_pair<G>(qf, st, ssm2, a.scale, warp, lane);
            } else {
              score_stage<G>(qf, smem_addr(smem + s * kStageBytes), ssm2[0], a.scale, warp, lane);
            }
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&sh.empty_bar[s]);
              if (two) mbar_arrive(&sh.empty_bar[s1]);
            }
            r += two ? 2u : 1u;
            consumer_sync();  // the chunks' window scores are complete
            send_chunk(k, ssm2[0]);
            if (two) send_chunk(k + static_cast<int>(C), ssm2[1]);
            k += (two ? 2 : 1) * static_cast<int>(C);
          }
        }
      }
      join_cluster();
      if (spill) {
        // Block scores in global memory: tell every CTA of the cluster (this
        // one included) that this CTA's are in place.
        fence_acq_rel_cluster();
        consumer_sync();
        if (tid == 0)
          for (uint32_t d = 0; d < C; ++d) mbar_remote_arrive(map_shared_rank(smem_addr(&sh.scores_bar), d));
      }
#ifdef NOSA_TRACE
      if (tid == 0) NOSA_STAMP(2);
#endif
      if (group_selects) group_select(tid);
    }
    join_cluster();
    attn_init(att);
    if (decoding && ok) {
      // This CTA's tiles: local t = rank, rank + C, ... < min(nloc, ntiles),
      // then selected t = rank (mod C) in [nloc, ntiles); with INT8 caches
      // each phase is issued two tiles per job.
      const int Ci = static_cast<int>(C), ri = static_cast<int>(rank);
      const int tend = min(nloc, ntiles);
      const int my_local = tend > ri ? (tend - ri + Ci - 1) / Ci : 0;
      const int t0 = nloc + ((ri - nloc % Ci) % Ci + Ci) % Ci;
      const int my_sel = ntiles > t0 ? (ntiles - t0 + Ci - 1) / Ci : 0;
      const int my_tiles = Q8 ? (my_local + 1) / 2 + (my_sel + 1) / 2 : my_local + my_sel;
      if (my_tiles > 0) {
        uint32_t qa[8][4];
        float qpow = 1.0f;
        if constexpr (Q8)
          qpow = load_attn_q_int8(qa, q_group, G, lane);
        else
          load_attn_q(qa, q_group, G, lane);
        // Tiles start once the selection is known (the consumers took part
        // in it, or wait for the selector): the selection runs on a quiet
        // SM, and the local tiles, already staged, are consumed while the
        // first selected tiles are in flight.
        if (scoring && !group_selects) mbar_wait(&sh.sel_bar, 0, a.status);
        for (int n = 0; n < my_tiles; ++n) {
          const int s = static_cast<int>(r % S);
          if (!mbar_wait(&sh.full_bar[s], (r / S) & 1u, a.status)) break;
#ifdef NOSA_TRACE
          if (tid == 0 && n == 0) NOSA_STAMP(22);
#endif
          if constexpr (Q8) {
            const uint8_t* st = smem + s * kStageBytes;
            const float* scl = reinterpret_cast<const float*>(smem + step_scale_offset<G, S>(a, static_cast<int>(C)) + s * kScaleStageBytes);
            const int blk[2] = {sh.stage_blk[s][0], sh.stage_blk[s][1]};
            const float* const ksc[2] = {scl + sh.stage_soff[s][0], scl + 2 * (kScaleSlot / 4) + sh.stage_soff[s][1]};
            const float* const vsc[2] = {scl + (kScaleSlot / 4) + sh.stage_soff[s][0],
                                         scl + 3 * (kScaleSlot / 4) + sh.stage_soff[s][1]};
#ifdef NOSA_TRACE
            uint64_t* stamps = tid == 0 && n == 1 ? &sh.tr[14] : nullptr;
#else
            uint64_t* stamps = nullptr;
#endif
            if (blk[1] == kAbsentTile)
              attend_stage_int8<1>(att, qa, qpow, st, ksc, vsc, blk, L, a.scale_log2, warp, lane, stamps);
            else
              attend_stage_int8<2>(att, qa, qpow, st, ksc, vsc, blk, L, a.scale_log2, warp, lane, stamps);
          } else {
            attend_tile(att, qa, smem + s * kStageBytes, sh.stage_blk[s][0], L, a.scale_log2, warp, lane);
          }
          if (lane == 0) mbar_arrive(&sh.empty_bar[s]);
          ++r;
        }
      }
      attn_finish(att);
    }
  }
  __syncthreads();  // the ring is drained: reuse it for the merge
#ifdef NOSA_TRACE
  if (tid == 0) NOSA_STAMP(5);
#endif

  // ---------------------------------------------------------------- merge
  using ML = MergeLayout<G>;
  float* mf = reinterpret_cast<float*>(smem);

  if (decoding) {
    // The four warps' states, in warp order, into this CTA's partial.
    if (warp < kConsumerWarps) {
      const int grp = lane >> 2, tig = lane & 3;
#pragma unroll
      for (int d = 0; d < 16; ++d) {
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int row = grp + h2 * 8;
          if (row < G) {
            float* o = mf + ML::kMo + (warp * G + row) * kMoStride;
            if constexpr (Q8) {  // acc[d][e]: dim 32 tig + 16 (e & 1) + d, scaled by 1 / U
              o[32 * tig + d] = att.acc[d][2 * h2] * att.vscale;
              o[32 * tig + 16 + d] = att.acc[d][2 * h2 + 1] * att.vscale;
            } else {
              *reinterpret_cast<float2*>(o + d * 8 + 2 * tig) = make_float2(att.acc[d][2 * h2], att.acc[d][2 * h2 + 1]);
            }
          }
        }
      }
      if (tig == 0) {
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int row = grp + rr * 8;
          if (row < G) {
            mf[ML::kMm + warp * G + row] = att.m[rr];
            mf[ML::kMl + warp * G + row] = att.l[rr];
          }
        }
      }
    }
    __syncthreads();
    // Push: output float4 f of this CTA's partial (its four warps combined,
    // weights 2^(m_w - M)) goes to CTA f / slice of the cluster (slot
    // [rank][f % slice] of its receive buffer), and the first float4 of each
    // row in a slice also carries the row's max and sum.  st.async completes
    // the bytes on the receiver's recv_bar: no cluster barrier.
    constexpr int kVec = kHeadDim / 4;
    const int slice = (out_items<G>() + static_cast<int>(C) - 1) / static_cast<int>(C);
    float* recv_m = recv + 4 * static_cast<int>(C) * slice;  // [C][G]
    float* recv_l = recv_m + static_cast<int>(C) * G;         // [C][G]
    for (int f = tid; f < out_items<G>(); f += kStepThreads) {
      const int row = f / kVec, d4 = f % kVec;
      float mw[kConsumerWarps];
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        mw[w] = mf[ML::kMm + w * G + row];
        M = fmaxf(M, mw[w]);
      }
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      float lsum = 0.0f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float fw = mw[w] == -INFINITY ? 0.0f : fast_exp2(mw[w] - M);
        const float4 x = *reinterpret_cast<const float4*>(mf + ML::kMo + (w * G + row) * kMoStride + 4 * d4);
        o.x = fmaf(fw, x.x, o.x);
        o.y = fmaf(fw, x.y, o.y);
        o.z = fmaf(fw, x.z, o.z);
        o.w = fmaf(fw, x.w, o.w);
        lsum = fmaf(fw, mf[ML::kMl + w * G + row], lsum);
      }
      const int dst = f / slice;
      const uint32_t bar = map_shared_rank(smem_addr(&sh.recv_bar), static_cast<uint32_t>(dst));
      st_async_f32x4(map_shared_rank(smem_addr(recv + 4 * (static_cast<int>(rank) * slice + (f - dst * slice))),
                                     static_cast<uint32_t>(dst)),
                     o, bar);
      if (f == max(row * kVec, dst * slice)) {
        st_async_f32(map_shared_rank(smem_addr(recv_m + static_cast<int>(rank) * G + row), static_cast<uint32_t>(dst)),
                     M, bar);
        st_async_f32(map_shared_rank(smem_addr(recv_l + static_cast<int>(rank) * G + row), static_cast<uint32_t>(dst)),
                     lsum, bar);
      }
    }
#ifdef NOSA_TRACE
    if (tid == 0) NOSA_STAMP(11);
#endif
    // This CTA's slice of the output, once all C partials have arrived:
    // combined in rank order.
    int f0, f1;
    out_slice<G>(static_cast<int>(rank), static_cast<int>(C), &f0, &f1);
    const bool arrived = tid < f1 - f0 && mbar_wait(&sh.recv_bar, 0, a.status);
#ifdef NOSA_TRACE
    if (tid == 0) NOSA_STAMP(12);
#endif
    for (int f = f0 + tid; f < f1; f += kStepThreads) {
      const int row = f / kVec, d4 = f % kVec;
      float M = -INFINITY;
      for (int k = 0; k < static_cast<int>(C); ++k) M = fmaxf(M, recv_m[k * G + row]);
      float lsum = 0.0f;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k = 0; k < static_cast<int>(C); ++k) {
        const float mk = recv_m[k * G + row];
        const float w = mk == -INFINITY ? 0.0f : fast_exp2(mk - M);
        lsum = fmaf(recv_l[k * G + row], w, lsum);
        const float4 x = *reinterpret_cast<const float4*>(recv + 4 * (k * slice + (f - f0)));
        o.x = fmaf(w, x.x, o.x);
        o.y = fmaf(w, x.y, o.y);
        o.z = fmaf(w, x.z, o.z);
        o.w = fmaf(w, x.w, o.w);
      }
      if (!arrived) {  // a push never came (status bit set): write zeros
        o = make_float4(0.f, 0.f, 0.f, 0.f);
        lsum = 0.0f;
        M = -INFINITY;
      }
      const int64_t orow = static_cast<int64_t>(i) * a.hq + static_cast<int64_t>(g) * G + row;
      const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(a.out + orow * kHeadDim + 4 * d4);
      dst[0] = __floats2bfloat162_rn(o.x * inv, o.y * inv);
      dst[1] = __floats2bfloat162_rn(o.z * inv, o.w * inv);
      if (a.lse && d4 == 0) a.lse[orow] = lsum > 0.0f ? (M + log2f(lsum)) * kLn2 : -INFINITY;
    }
  }
#ifdef NOSA_TRACE
  if (tid == 0) {
    NOSA_STAMP(7);
    const uint32_t k = atomicAdd(&g_trace_count, 1u);
    if (k < kTraceCapacity) {
      uint32_t smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      TraceRecord rec;
      rec.pair = pair;
      rec.rank = rank;
      rec.smid = smid;
      rec.csize = C | (S << 8);
      for (int n = 0; n < 24; ++n) rec.t[n] = sh.tr[n];
      g_trace[k] = rec;
    }
  }
#endif
}

__device__ void write_empty_selection(const SelectArgs& a, int pair, int nthreads) {
  for (int t = threadIdx.x; t < a.topk; t += nthreads) a.sel_idx[static_cast<int64_t>(pair) * a.topk + t] = -1;
  if (threadIdx.x == 0) a.sel_cnt[pair] = 0;
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

// Shared memory of a launch whose clusters have at most C CTAs.
template <int G, int S, bool Q8>
size_t step_smem_bytes(const StepArgs& a, int C) {
  return 1024 + step_scale_offset<G, S>(a, C) + (Q8 ? static_cast<size_t>(S) * kScaleStageBytes : 0);
}

// Residency of the step kernel at a given shared-memory size: resident
// CTAs and co-resident clusters of each size (cached per kernel and size).
struct Capacity {
  int dev = -1;
  size_t smem = 0;
  int slots = 0, sms = 0;
  int max_clusters[kMaxCluster + 1] = {};  // C = 1..16
};
std::mutex g_plan_mu;
// [group size][ring: 3 or 6 stages][bf16 / INT8 caches][receive buffer for
// clusters of up to 16 / up to kSmallCluster CTAs]
Capacity g_cap[5][2][2][2];
constexpr int kSmallCluster = 4;

template <int G, int S, bool Q8>
cudaError_t capacity(size_t smem, bool small_recv, const Capacity** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  constexpr int gi = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : G == 8 ? 3 : 4;
  Capacity& c = g_cap[gi][S == Rings<Q8>::kLo ? 0 : 1][Q8 ? 1 : 0][small_recv ? 1 : 0];
  if (c.dev != dev || c.smem != smem) {
    // The attribute is an upper bound: set to the largest size the device
    // allows next to the kernel's static shared memory, so that concurrent
    // launches of different sizes never undercut each other.
    int optin = 0;
    cudaFuncAttributes fa;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
    if ((e = cudaFuncGetAttributes(&fa, step_kernel<G, S, Q8>)) != cudaSuccess) return e;
    const int max_dyn = optin - static_cast<int>(fa.sharedSizeBytes);
    if (static_cast<int>(smem) > max_dyn) return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(step_kernel<G, S, Q8>, cudaFuncAttributeMaxDynamicSharedMemorySize, max_dyn)) !=
        cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(step_kernel<G, S, Q8>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) !=
        cudaSuccess)
      return e;
    int per_sm = 0, sms = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, step_kernel<G, S, Q8>, kStepThreads, smem)) !=
        cudaSuccess)
      return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    c.slots = per_sm * sms;
    c.sms = sms;
    for (int cs = 1; cs <= kMaxCluster; ++cs) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(cs);
      cfg.blockDim = dim3(kStepThreads);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, step_kernel<G, S, Q8>, &cfg) != cudaSuccess) {
        cudaGetLastError();  // a size the device cannot co-schedule: never chosen
        n = 0;
      }
      c.max_clusters[cs] = n;
    }
    c.dev = dev;
    c.smem = smem;
  }
  *out = &c;
  return cudaSuccess;
}

// Among the cluster sizes up to max_c whose pairs x C CTAs are all resident
// at once, the smallest C with the fewest scoring chunks per CTA (`units` of
// the longest pair): a larger cluster would not shorten the longest CTA's
// scoring and only costs wider exchanges.  1 when no larger cluster fits
// (then clusters run in waves).
int choose_cluster(const Capacity& c, int pairs, int units, int max_c) {
  int best = 1, best_units = units;
  for (int cs = 2; cs <= max_c; ++cs) {
    if (static_cast<int64_t>(pairs) * cs > c.slots || c.max_clusters[cs] < pairs) continue;
    const int per_cta = (units + cs - 1) / cs;
    if (per_cta < best_units) {
      best = cs;
      best_units = per_cta;
    }
  }
  return best;
}

template <int G, int S, bool Q8, bool P = false>
cudaError_t launch_with(const StepArgs& a, const StepMaps& maps, size_t smem, int csize, bool pdl,
                        cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.batch * a.hkv) * csize);
  cfg.blockDim = dim3(kStepThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, step_kernel<G, S, Q8, P>, a, maps);
}

// The pair-scoring instance of the deep ring: the same shared-memory
// attributes as its base instance (set once per device), and the same
// residency (one CTA per SM, equal shared memory).
template <int G, bool Q8>
cudaError_t prepare_pairs() {
  static int prepared_dev = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || prepared_dev == dev) return e;
  constexpr int kHi = Rings<Q8>::kHi;
  int optin = 0;
  cudaFuncAttributes fa;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  if ((e = cudaFuncGetAttributes(&fa, step_kernel<G, kHi, Q8, true>)) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(step_kernel<G, kHi, Q8, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                optin - static_cast<int>(fa.sharedSizeBytes))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(step_kernel<G, kHi, Q8, true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) !=
      cudaSuccess)
    return e;
  prepared_dev = dev;
  return cudaSuccess;
}

// Launch plan: the cluster size (choose_cluster) on the 3-stage ring, two
// CTAs per SM.  When the whole grid then fits one CTA per SM, the 6-stage
// ring (one CTA per SM, twice the bytes in flight) runs instead, if the
// same cluster size is still co-resident.  Programmatic dependent launch
// only when the grid leaves at least half of the resident slots free: the
// next launch's clusters then become resident and run their prologue early;
// when the grid fills the GPU, early-resident clusters of the next launch
// only skew where the rest are placed.  NOSA_CLUSTER_SIZE (1..16),
// NOSA_RING_STAGES (the smaller or the larger ring: 3 / 6, INT8 2 / 4) and
// NOSA_PDL (0 / 1) override the choices.  With the deep ring, fp32 pooled
// keys and at least kPairChunks scoring chunks per CTA, chunks after the
// first are scored two per pass (NOSA_PAIRS 0 / 1 overrides): the scoring of
// long contexts is bound by the consumers' tensor-core chains, while with
// few chunks per CTA a pair would hold the second chunk's scores back.
constexpr int kPairChunks = 8;

template <int G, bool Q8>
cudaError_t launch_step_g(const StepArgs& a, const StepMaps& maps, cudaStream_t stream) {
  const int pairs = a.batch * a.hkv;
  if (pairs <= 0) return cudaSuccess;
  // Work units of the longest pair: its selection's scoring chunks.  The
  // same in every mode, so the separate selection and attention launches
  // split a pair's tiles exactly as the fused step does (bit-identical
  // results).
  const int units = max((a.ncand_max + kChunkBlocks - 1) / kChunkBlocks, 1);
  static const int forced_c = [] {
    const char* v = getenv("NOSA_CLUSTER_SIZE");
    const int n = v ? atoi(v) : 0;
    return n >= 1 && n <= kMaxCluster ? n : 0;
  }();
  static const int forced_s = [] {
    const char* v = getenv("NOSA_RING_STAGES");
    return v ? atoi(v) : 0;
  }();
  static const int forced_pdl = [] {
    const char* v = getenv("NOSA_PDL");
    return v && (atoi(v) == 0 || atoi(v) == 1) ? atoi(v) : -1;
  }();
  static const int forced_pairs = [] {
    const char* v = getenv("NOSA_PAIRS");
    return v && (atoi(v) == 0 || atoi(v) == 1) ? atoi(v) : -1;
  }();
  constexpr int kLo = Rings<Q8>::kLo, kHi = Rings<Q8>::kHi;
  const size_t smem6 = step_smem_bytes<G, kHi, Q8>(a, kMaxCluster);
  size_t smem3 = step_smem_bytes<G, kLo, Q8>(a, kMaxCluster);
  const size_t smem3_small = step_smem_bytes<G, kLo, Q8>(a, kSmallCluster);
  int csize, stages = kLo;
  bool pdl;
  {
    std::lock_guard<std::mutex> lock(g_plan_mu);
    const Capacity* c3 = nullptr;
    cudaError_t e = capacity<G, kLo, Q8>(smem3, false, &c3);
    if (e != cudaSuccess) return e;
    csize = choose_cluster(*c3, pairs, units, kMaxCluster);
    if (forced_c && c3->max_clusters[forced_c] > 0) {
      csize = forced_c;
    } else if (smem3_small < smem3 && c3->slots <= c3->sms) {
      // The receive buffer of 16-CTA clusters keeps the 3-stage ring at one
      // CTA per SM (long contexts: the block scores take the room); sized for
      // clusters of at most kSmallCluster CTAs it may fit two.  That plan is
      // taken when it gives fewer scoring chunks per CTA.
      const Capacity* c3s = nullptr;
      if (capacity<G, kLo, Q8>(smem3_small, true, &c3s) == cudaSuccess && c3s->slots > c3->slots) {
        const int cs = choose_cluster(*c3s, pairs, units, kSmallCluster);
        if ((units + cs - 1) / cs < (units + csize - 1) / csize) {
          csize = cs;
          c3 = c3s;
          smem3 = smem3_small;
        }
      }
      cudaGetLastError();
    }
    pdl = forced_pdl >= 0 ? forced_pdl != 0 : static_cast<int64_t>(pairs) * csize * 2 <= c3->slots;
    const Capacity* c6 = nullptr;
    const bool forced = forced_s == kLo || forced_s == kHi;
    const bool want6 = forced ? forced_s == kHi : static_cast<int64_t>(pairs) * csize <= c3->sms;
    if (want6 && capacity<G, kHi, Q8>(smem6, false, &c6) == cudaSuccess && c6->max_clusters[csize] >= pairs) {
      stages = kHi;
      pdl = forced_pdl >= 0 ? forced_pdl != 0 : static_cast<int64_t>(pairs) * csize * 2 <= c6->slots;
    }
    cudaGetLastError();  // a 6-stage ring the device cannot host is simply not used
#ifdef NOSA_TRACE
    fprintf(stderr, "plan G=%d pairs=%d units=%d -> C=%d stages=%d pdl=%d (3-stage slots %d, 6-stage clusters of C: %d)\n",
            G, pairs, units, csize, stages, static_cast<int>(pdl), c3->slots, c6 ? c6->max_clusters[csize] : -1);
#endif
  }
  if (stages == kHi) {
    if constexpr (!Q8 && G <= 8) {
      const bool pairs_mode =
          !a.pooled_bf16 && (forced_pairs >= 0 ? forced_pairs == 1 : (units + csize - 1) / csize >= kPairChunks);
      if (pairs_mode) {
        cudaError_t e;
        {
          std::lock_guard<std::mutex> lock(g_plan_mu);
          e = prepare_pairs<G, Q8>();
        }
        if (e != cudaSuccess) return e;
        return launch_with<G, kHi, Q8, true>(a, maps, smem6, csize, pdl, stream);
      }
    }
    return launch_with<G, kHi, Q8>(a, maps, smem6, csize, pdl, stream);
  }
  return launch_with<G, kLo, Q8>(a, maps, smem3, csize, pdl, stream);
}

template <int G>
cudaError_t launch_step_q(const StepArgs& a, const StepMaps& maps, cudaStream_t stream) {
  // The INT8 kernels only differ in what the attention tiles hold: scoring
  // and selection alone use the bf16 instance.
  if (a.kv_int8 && (a.mode & (kStepDecode | kStepAppend))) return launch_step_g<G, true>(a, maps, stream);
  return launch_step_g<G, false>(a, maps, stream);
}

}  // namespace

cudaError_t launch_step(const StepArgs& a, const StepMaps& maps, cudaStream_t stream) {
  switch (a.hq / a.hkv) {
    case 1: return launch_step_q<1>(a, maps, stream);
    case 2: return launch_step_q<2>(a, maps, stream);
    case 4: return launch_step_q<4>(a, maps, stream);
    case 8: return launch_step_q<8>(a, maps, stream);
    case 16: return launch_step_q<16>(a, maps, stream);
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
