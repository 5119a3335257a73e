// Compressed scores, block scores and top-k selection: device routines of the
// selection-only kernel and the decode-step kernel.
//
// "NOSA-1B 模型家族全景" (demingchina.com), 核心原理: compressed attention
// screens the history for the TopK blocks; "NOSA-1B 性能基准全解析" (wmrh.cn)
// §三.2 (block 64, 16 local blocks, TopK 64) and §三.3 (scores of the
// kernel-32 / stride-16 pooled keys, then TopK).
//
//   s[h][j] = scale * q[h] . pooled[j]                        (j < nc)
//   S[b]    = sum_{h in group, ascending} max_{j in J(b)} s[h][j],
//             J(b) = {4b-1, ..., 4b+3} n [0, nc)               (b < ncand)
//   sel     = the min(topk, ncand) largest S, ties to the lower index,
//             ascending, -1 padded.
#pragma once

#include <cuda.h>

#include "decode_device.cuh"
#include "nosa_common.cuh"

namespace nosa {

struct TopkShared {
  uint32_t hist[256];
  uint32_t warp_eq[32];
  uint32_t warp_take[32];
  uint32_t prefix, need, run_eq, run_pos;
};

// Exact top-k by one warp, for up to 32 * KPL candidates (candidate b lives
// in lane b % 32, register b / 32).  The k-th largest order-preserving key T
// is found bit by bit from the top (T = the largest value with at least k
// keys >= T; each step counts with ballots), then an index-ordered ballot
// compaction writes every key above T plus the lowest-index keys equal to T.
// No block-wide barriers; the other warps are not involved.
template <int KPL>
__device__ void warp_topk(const float* scores, bool coherent, int ncand, int topk, int32_t* sel_row,
                          int32_t* sel_cnt, int lane, uint64_t* trace_stamps = nullptr) {
  const int k_eff = ncand < topk ? ncand : topk;
  uint32_t key[KPL];
#pragma unroll
  for (int m = 0; m < KPL; ++m) {
    const int b = m * 32 + lane;
    key[m] = b < ncand ? order_key(coherent ? __ldcg(scores + b) : scores[b]) : 0u;  // valid keys are > 0
  }
#ifdef NOSA_TRACE
  if (trace_stamps && lane == 0) trace_stamps[0] = global_timer_ns() + (key[0] & 0u);
#endif
  uint32_t T = 0u;
  int need = 0;
  if (k_eff < ncand) {
    // The k-th largest key lies in [min, max]: its bits above their highest
    // differing bit are theirs.  The rest is found two bits per step --
    // count the keys >= each of T|01, T|10, T|11 (warp sums, redux.sync) and
    // keep the largest threshold that still has at least k keys at or above.
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
    for (int m = 0; m < KPL; ++m) {
      if (m * 32 + lane < ncand) {
        lo = min(lo, key[m]);
        hi = max(hi, key[m]);
      }
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t k = static_cast<uint32_t>(k_eff);
    if (lo != hi) {
      const int top = 31 - __clz(lo ^ hi);                // highest differing bit
      T = hi & ~((2u << top) - 1u);                       // common prefix (top == 31: shift by 32 avoided)
      if (top == 31) T = 0u;
      int bit = top;
      if ((top & 1) == 0) {                               // odd number of bits left: one single-bit step
        const uint32_t c1 = T | (1u << bit);
        uint32_t n1 = 0;
#pragma unroll
        for (int m = 0; m < KPL; ++m) n1 += key[m] >= c1;
        if (__reduce_add_sync(0xffffffffu, n1) >= k) T = c1;
        --bit;
      }
#pragma unroll 1
      for (bit -= 1; bit >= 0; bit -= 2) {
        const uint32_t c1 = T | (1u << bit), c2 = T | (2u << bit), c3 = T | (3u << bit);
        uint32_t n1 = 0, n2 = 0, n3 = 0;
#pragma unroll
        for (int m = 0; m < KPL; ++m) {
          n1 += key[m] >= c1;
          n2 += key[m] >= c2;
          n3 += key[m] >= c3;
        }
        n1 = __reduce_add_sync(0xffffffffu, n1);
        n2 = __reduce_add_sync(0xffffffffu, n2);
        n3 = __reduce_add_sync(0xffffffffu, n3);
        T = n3 >= k ? c3 : n2 >= k ? c2 : n1 >= k ? c1 : T;
      }
    } else {
      T = hi;
    }
    uint32_t above = 0;
#pragma unroll
    for (int m = 0; m < KPL; ++m) above += key[m] > T;
    need = k_eff - static_cast<int>(__reduce_add_sync(0xffffffffu, above));
  }
#ifdef NOSA_TRACE
  if (trace_stamps && lane == 0) trace_stamps[1] = global_timer_ns() + (T & 0u);
#endif
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t n_eq = 0;
#pragma unroll
  for (int m = 0; m < KPL; ++m) n_eq += (m * 32 + lane < ncand) && key[m] == T;
  n_eq = __reduce_add_sync(0xffffffffu, n_eq);
  int pos = 0;
  if (k_eff == ncand || static_cast<uint32_t>(need) == n_eq) {
    // Every key tied with the threshold is taken: key >= T decides alone.
#pragma unroll
    for (int m = 0; m < KPL; ++m) {
      const int b = m * 32 + lane;
      const bool take = b < ncand && key[m] >= T;
      const uint32_t tb = __ballot_sync(0xffffffffu, take);
      const int p = pos + __popc(tb & lt_mask);
      if (take && p < topk) sel_row[p] = b;
      pos += __popc(tb);
    }
  } else {
    int eq_seen = 0;
#pragma unroll
    for (int m = 0; m < KPL; ++m) {
      const int b = m * 32 + lane;
      const bool valid = b < ncand;
      const bool eq = valid && key[m] == T;
      const uint32_t eb = __ballot_sync(0xffffffffu, eq);
      const bool take = valid && (key[m] > T || (eq && eq_seen + __popc(eb & lt_mask) < need));
      const uint32_t tb = __ballot_sync(0xffffffffu, take);
      const int p = pos + __popc(tb & lt_mask);
      if (take && p < topk) sel_row[p] = b;
      eq_seen += __popc(eb);
      pos += __popc(tb);
    }
  }
  for (int t = k_eff + lane; t < topk; t += 32) sel_row[t] = -1;
  if (lane == 0) *sel_cnt = k_eff;
#ifdef NOSA_TRACE
  if (trace_stamps && lane == 0) trace_stamps[2] = global_timer_ns();
#endif
}

// Candidates up to which one warp selects (warp_topk); larger sets use the
// block-wide radix select.
constexpr int kWarpTopkMax = 1024;

// Top-k of `ncand` scores (global; read with ld.global.cg when `coherent`) by
// NT threads: one warp (warp_topk) for up to kWarpTopkMax candidates, else an
// exact 4 x 8-bit radix select of the k-th largest order-preserving key and
// an index-ordered ballot compaction (every key above it plus the
// lowest-index keys equal to it).  Writes the pair's sel_idx row (ascending,
// -1 padded) and its count.  `ords` is shared memory for ncand keys.
template <int NT>
__device__ void select_topk(const float* scores, bool coherent, int ncand, int topk, int32_t* sel_row,
                            int32_t* sel_cnt, uint32_t* ords, TopkShared& sh, uint64_t* trace_stamps = nullptr) {
  constexpr int kWarpsNT = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (ncand <= kWarpTopkMax) {
    if (warp == 0) {
      if (ncand <= 256)
        warp_topk<8>(scores, coherent, ncand, topk, sel_row, sel_cnt, lane, trace_stamps);
      else
        warp_topk<32>(scores, coherent, ncand, topk, sel_row, sel_cnt, lane, trace_stamps);
    }
    return;
  }
  const int k_eff = ncand < topk ? ncand : topk;
  for (int b = tid; b < ncand; b += NT) ords[b] = order_key(coherent ? __ldcg(scores + b) : scores[b]);
  if (tid == 0) {
    sh.prefix = 0;
    sh.need = 0;
    sh.run_eq = 0;
    sh.run_pos = 0;
  }
  __syncthreads();
  uint32_t T = 0, need = 0;  // T = 0: take every key (all keys are > 0)
  if (k_eff < ncand) {
    uint32_t prefix = 0;
    need = static_cast<uint32_t>(k_eff);
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
      for (int t = tid; t < 256; t += NT) sh.hist[t] = 0;
      __syncthreads();
      for (int b = tid; b < ncand; b += NT) {
        const uint32_t key = ords[b];
        if ((key & hi_mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (warp == 0) {
        uint32_t c[8], sum = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          c[k] = sh.hist[8 * lane + k];
          sum += c[k];
        }
        uint32_t suf = sum;  // sum over lanes >= this lane
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t x = __shfl_down_sync(0xffffffffu, suf, o);
          if (lane + o < 32) suf += x;
        }
        const uint32_t above = suf - sum;
        if (above < need && need <= suf) {
          uint32_t acc = above;
#pragma unroll
          for (int k = 7; k >= 0; --k) {
            if (acc + c[k] >= need) {
              sh.prefix = prefix | (static_cast<uint32_t>(8 * lane + k) << shift);
              sh.need = need - acc;
              break;
            }
            acc += c[k];
          }
        }
      }
      __syncthreads();
      prefix = sh.prefix;
      need = sh.need;
    }
    T = prefix;
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < ncand; base += NT) {
    const int b = base + tid;
    const uint32_t key = b < ncand ? ords[b] : 0u;
    const bool gt = b < ncand && key > T;
    const bool eq = b < ncand && key == T && k_eff < ncand;
    uint32_t ball = __ballot_sync(0xffffffffu, eq);
    const uint32_t eq_in_warp = __popc(ball & lt_mask);
    if (lane == 0) sh.warp_eq[warp] = __popc(ball);
    __syncthreads();
    uint32_t eq_before = sh.run_eq + eq_in_warp;
    for (int w = 0; w < warp; ++w) eq_before += sh.warp_eq[w];
    const bool take = gt || (eq && eq_before < need);
    ball = __ballot_sync(0xffffffffu, take);
    if (lane == 0) sh.warp_take[warp] = __popc(ball);
    __syncthreads();
    uint32_t pos = sh.run_pos + __popc(ball & lt_mask);
    for (int w = 0; w < warp; ++w) pos += sh.warp_take[w];
    if (take && pos < static_cast<uint32_t>(topk)) sel_row[pos] = b;
    __syncthreads();
    if (tid == 0) {
      for (int w = 0; w < kWarpsNT; ++w) {
        sh.run_eq += sh.warp_eq[w];
        sh.run_pos += sh.warp_take[w];
      }
    }
    __syncthreads();
  }
  for (int t = k_eff + tid; t < topk; t += NT) sel_row[t] = -1;
  if (tid == 0) *sel_cnt = k_eff;
}

// Exact top-k by one warp over any number of candidates held in memory
// (shared, or global when `coherent`): warp_topk's threshold search and
// compaction, with the keys re-read on every step instead of kept in
// registers.  For candidate sets beyond warp_topk's register capacity.
__device__ inline void warp_topk_mem(const float* scores, bool coherent, int ncand, int topk, int32_t* sel_row,
                                     int32_t* sel_cnt, int lane) {
  auto key_at = [&](int b) { return order_key(coherent ? __ldcg(scores + b) : scores[b]); };
  const int k_eff = ncand < topk ? ncand : topk;
  uint32_t T = 0u;
  uint32_t need = 0u;
  if (k_eff < ncand) {
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (int b = lane; b < ncand; b += 32) {
      const uint32_t k = key_at(b);
      lo = min(lo, k);
      hi = max(hi, k);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t k = static_cast<uint32_t>(k_eff);
    if (lo != hi) {
      const int top = 31 - __clz(lo ^ hi);
      T = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
      int bit = top;
      if ((top & 1) == 0) {
        const uint32_t c1 = T | (1u << bit);
        uint32_t n1 = 0;
        for (int b = lane; b < ncand; b += 32) n1 += key_at(b) >= c1;
        if (__reduce_add_sync(0xffffffffu, n1) >= k) T = c1;
        --bit;
      }
      for (bit -= 1; bit >= 0; bit -= 2) {
        const uint32_t c1 = T | (1u << bit), c2 = T | (2u << bit), c3 = T | (3u << bit);
        uint32_t n1 = 0, n2 = 0, n3 = 0;
        for (int b = lane; b < ncand; b += 32) {
          const uint32_t key = key_at(b);
          n1 += key >= c1;
          n2 += key >= c2;
          n3 += key >= c3;
        }
        n1 = __reduce_add_sync(0xffffffffu, n1);
        n2 = __reduce_add_sync(0xffffffffu, n2);
        n3 = __reduce_add_sync(0xffffffffu, n3);
        T = n3 >= k ? c3 : n2 >= k ? c2 : n1 >= k ? c1 : T;
      }
    } else {
      T = hi;
    }
    uint32_t above = 0;
    for (int b = lane; b < ncand; b += 32) above += key_at(b) > T;
    need = k - __reduce_add_sync(0xffffffffu, above);
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  int pos = 0;
  uint32_t eq_seen = 0;
  for (int base = 0; base < ncand; base += 32) {
    const int b = base + lane;
    const bool valid = b < ncand;
    const uint32_t key = valid ? key_at(b) : 0u;
    const bool eq = valid && k_eff < ncand && key == T;
    const uint32_t eb = __ballot_sync(0xffffffffu, eq);
    const bool take = valid && (key > T || (k_eff == ncand) || (eq && eq_seen + __popc(eb & lt_mask) < need));
    const uint32_t tb = __ballot_sync(0xffffffffu, take);
    const int p = pos + __popc(tb & lt_mask);
    if (take && p < topk) sel_row[p] = b;
    eq_seen += __popc(eb);
    pos += __popc(tb);
  }
  for (int t = k_eff + lane; t < topk; t += 32) sel_row[t] = -1;
  if (lane == 0) *sel_cnt = k_eff;
}

// Exact top-k by a group of NT threads (a multiple of 32, synchronised with
// named barrier `bar_id`) over up to NT * kGroupKeys candidates in memory
// (shared, or global when `coherent`).  Thread t holds the contiguous keys
// [t * kpt, (t + 1) * kpt).  The k-th largest order-preserving key T is
// found by a radix select on 8-bit digits (a shared-memory histogram per
// pass) below the common prefix of the min and max keys; one prefix scan of
// the per-thread (greater, equal) counts then places every key above T and
// the lowest-index keys equal to T in ascending order.  Same result as
// warp_topk.  Every thread of the group must call it with the same
// arguments; `tid` is the thread's index in the group.
constexpr int kGroupKeys = 16;

// Survivors the bucket select ranks in shared memory (more fall back to the
// radix select), and its taken-bit words (32 candidate slots each).
constexpr int kSurvivorCap = 128;
constexpr int kTakeWords = 80;

struct alignas(16) GroupTopkShared {
  uint32_t hist[256];             // radix select: digit histogram; bucket select: bucket counts
  uint64_t surv[kSurvivorCap];    // bucket select: survivors, key << 32 | ~index
  uint32_t take[kTakeWords];      // bucket select: taken bits
  uint32_t red[2][8][2];  // per-warp partials, double-buffered
  uint32_t prefix, need, nsurv;
};

__device__ inline void group_bar(int bar_id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthreads) : "memory");
}

template <int NT, bool kKeys = false>
__device__ void group_topk(const float* scores, bool coherent, int ncand, int topk, int32_t* sel_row,
                           int32_t* sel_cnt, int tid, GroupTopkShared& sh, int bar_id,
                           uint64_t* trace_stamps = nullptr) {
#ifdef NOSA_TRACE
#define GTK_STAMP(k) \
  if (trace_stamps && tid == 0) trace_stamps[k] = global_timer_ns()
#else
#define GTK_STAMP(k)
#endif
  constexpr int kWarps = NT / 32;
  const int lane = tid & 31, warp = tid >> 5;
  const int k_eff = ncand < topk ? ncand : topk;
  const int kpt = (ncand + NT - 1) / NT;
  const int b0 = tid * kpt;
  uint32_t key[kGroupKeys];
#pragma unroll
  for (int m = 0; m < kGroupKeys; ++m) {
    const int b = b0 + m;
    if (m < kpt && b < ncand)  // valid keys are > 0
      key[m] = kKeys ? reinterpret_cast<const uint32_t*>(scores)[b]
                     : order_key(coherent ? __ldcg(scores + b) : scores[b]);
    else
      key[m] = 0u;
  }
  GTK_STAMP(0);
  uint32_t T = 0u, need = 0u;
  if (k_eff < ncand) {
    // Common prefix of the min and max valid keys.
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
#pragma unroll
    for (int m = 0; m < kGroupKeys; ++m)
      if (m < kpt && b0 + m < ncand) {
        lo = min(lo, key[m]);
        hi = max(hi, key[m]);
      }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if (lane == 0) {
      sh.red[0][warp][0] = lo;
      sh.red[0][warp][1] = hi;
    }
    group_bar(bar_id, NT);
    GTK_STAMP(1);
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      lo = min(lo, sh.red[0][w][0]);
      hi = max(hi, sh.red[0][w][1]);
    }
    need = static_cast<uint32_t>(k_eff);
    if (lo == hi) {
      T = hi;
    } else {
      const int top = 31 - __clz(lo ^ hi);
      uint32_t P = top == 31 ? 0u : (hi & ~((2u << top) - 1u));
      int r = top + 1;  // bits of T still open: [0, r)
      while (r > 0) {   // the same pass count in every thread
        const int w = r < 8 ? r : 8;
        const int shift = r - w;
        for (int x = tid; x < 256; x += NT) sh.hist[x] = 0u;
        group_bar(bar_id, NT);
#pragma unroll
        for (int m = 0; m < kGroupKeys; ++m) {
          const uint32_t kk = key[m];
          if (m < kpt && b0 + m < ncand && (r == 32 || (kk >> r) == (P >> r)))
            atomicAdd(&sh.hist[(kk >> shift) & ((1u << w) - 1u)], 1u);
        }
        group_bar(bar_id, NT);
        if (warp == 0) {
          // Lane l owns digits [8l, 8l+8); the digit holding the need-th
          // largest key is where the count from the top first reaches need.
          uint32_t c[8], sum = 0;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            c[q] = sh.hist[8 * lane + q];
            sum += c[q];
          }
          uint32_t suf = sum;  // sum over lanes >= this lane
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
            if (lane + o < 32) suf += y;
          }
          const uint32_t above = suf - sum;
          if (above < need && need <= suf) {
            uint32_t acc = above;
#pragma unroll
            for (int q = 7; q >= 0; --q) {
              if (acc + c[q] >= need) {
                sh.prefix = P | (static_cast<uint32_t>(8 * lane + q) << shift);
                sh.need = need - acc;
                break;
              }
              acc += c[q];
            }
          }
        }
        group_bar(bar_id, NT);
        P = sh.prefix;
        need = sh.need;
        r = shift;
        GTK_STAMP(2);
      }
      T = P;
    }
  }
  // Placement: keys above T, then the first `need` keys equal to T in index
  // order.  (gt << 16 | eq) per thread, scanned over the group.
  uint32_t gt = 0, eq = 0;
#pragma unroll
  for (int m = 0; m < kGroupKeys; ++m)
    if (m < kpt && b0 + m < ncand) {
      gt += key[m] > T;
      eq += key[m] == T;
    }
  if (k_eff == ncand) {  // everything is taken
    gt += eq;
    eq = 0;
    need = 0;
  }
  const uint32_t mine = (gt << 16) | eq;
  uint32_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sh.red[1][warp][0] = incl;
  GTK_STAMP(3);
  group_bar(bar_id, NT);
  GTK_STAMP(4);
  uint32_t before = incl - mine;
  for (int w = 0; w < warp; ++w) before += sh.red[1][w][0];
  const uint32_t gt_before = before >> 16, eq_before = before & 0xFFFFu;
  int pos = static_cast<int>(gt_before + min(eq_before, need));
  uint32_t eq_take = min(eq_before + eq, need) - min(eq_before, need);
#pragma unroll
  for (int m = 0; m < kGroupKeys; ++m) {
    const int b = b0 + m;
    if (m < kpt && b < ncand) {
      bool take = key[m] > T || k_eff == ncand;
      if (!take && key[m] == T && eq_take > 0) {
        take = true;
        --eq_take;
      }
      if (take) {
        if (pos < topk) sel_row[pos] = b;
        ++pos;
      }
    }
  }
  for (int x = k_eff + tid; x < topk; x += NT) sel_row[x] = -1;
  if (tid == 0) *sel_cnt = k_eff;
  GTK_STAMP(5);
#undef GTK_STAMP
}

// The bucket select's hand-over to the radix select (more survivors in the
// k-th bucket than its list holds: ties, or a range the buckets cannot
// split).  Out of line: it almost never runs, and inlined it would sit in
// the middle of the bucket select's code.
template <int NT>
__device__ __noinline__ void group_topk_from_keys(float* scores, int ncand, int topk, int32_t* sel_row,
                                                  int32_t* sel_cnt, int tid, GroupTopkShared& sh, int bar_id) {
  group_topk<NT, true>(scores, false, ncand, topk, sel_row, sel_cnt, tid, sh, bar_id);
}

// The fp32 score an order-preserving key stands for (order_key's inverse;
// -0.0 and NaN come back as +0.0 and -inf).
__device__ inline float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Exact top-k of the selection group by bucket select: NT threads (a
// multiple of 32, at most 8 warps; `tid` is the thread's index in the
// group) and up to NT * M candidates, candidate b held by thread b mod NT in
// register b / NT.  `scores` is the pair's block scores in shared memory;
// they are overwritten by their order-preserving keys.
//   1. Keys in registers and in place of the scores; the smallest and
//      largest key over the group.
//   2. Each key falls into one of 256 equal-width buckets of its score
//      between the smallest and the largest, bucket(x) = floor((x - lo) *
//      256 / (hi - lo)) clamped to 255: a non-decreasing function of the
//      score (an fp32 subtraction and a multiplication by a positive
//      constant never reverse an order), counted in a shared histogram.
//   3. Every warp scans the histogram from the top for the bucket B that
//      holds the k-th largest key; the keys of higher buckets are taken (one
//      bit each in the taken-bit words, word q = candidates [32q, 32q + 32)),
//      the keys of bucket B are listed as key << 32 | ~index.
//   4. Each listed key is ranked among the list (key descending, then index
//      ascending); the first k - (keys above B) set their taken bits.
//   5. Placement in ascending index order: a candidate's position is the
//      number of taken bits below its own.
// One pass over the keys and four barriers; more than kSurvivorCap keys in
// bucket B (many equal keys, or a range the buckets cannot split: an
// infinite score, all scores equal) hand over to the radix select.
template <int NT, int M>
__device__ void bucket_topk(float* scores, int ncand, int topk, int32_t* sel_row, int32_t* sel_cnt, int tid,
                            GroupTopkShared& sh, int bar_id, uint64_t* trace_stamps = nullptr) {
#ifdef NOSA_TRACE
#define BKT_STAMP(k) \
  if (trace_stamps && tid == 0) trace_stamps[k] = global_timer_ns()
#else
#define BKT_STAMP(k)
#endif
  constexpr int kW = NT / 32;
  constexpr int kQ = M * kW;  // taken-bit words of the NT * M candidate slots
  static_assert(NT % 32 == 0 && kW <= 8, "the group is 1..8 whole warps");
  static_assert(M >= 1 && kQ <= kTakeWords, "one taken-bit word per 32 candidate slots");
  constexpr uint32_t kFull = 0xffffffffu;
  const int lane = tid & 31, w = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int k_eff = ncand < topk ? ncand : topk;
  if (k_eff == ncand) {  // every candidate is taken
    for (int b = tid; b < topk; b += NT) sel_row[b] = b < ncand ? b : -1;
    if (tid == 0) *sel_cnt = k_eff;
    return;
  }
  uint32_t* ords = reinterpret_cast<uint32_t*>(scores);
  uint32_t key[M];
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int b = tid + m * NT;
    const float f = scores[b < ncand ? b : 0];  // loads issued unconditionally
    key[m] = b < ncand ? order_key(f) : 0u;     // valid keys are > 0
    if (b < ncand) {
      ords[b] = key[m];
      kmin = min(kmin, key[m]);
      kmax = max(kmax, key[m]);
    }
  }
  for (int x = tid; x < 256; x += NT) sh.hist[x] = 0u;
  if (tid == 0) sh.nsurv = 0u;
  kmin = __reduce_min_sync(kFull, kmin);
  kmax = __reduce_max_sync(kFull, kmax);
  if (lane == 0) {
    sh.red[0][w][0] = kmin;
    sh.red[0][w][1] = kmax;
  }
  group_bar(bar_id, NT);
  BKT_STAMP(0);
#pragma unroll
  for (int x = 0; x < kW; ++x) {
    kmin = min(kmin, sh.red[0][x][0]);
    kmax = max(kmax, sh.red[0][x][1]);
  }
  const float lo = key_float(kmin), range = key_float(kmax) - lo;
  // range is +inf or NaN when a score is infinite: one bucket for all.
  const float scale = range > 0.0f && range <= 3.0e38f ? 256.0f / range : 0.0f;
  auto bucket = [&](uint32_t kk) -> int {
    const float d = (key_float(kk) - lo) * scale;
    return d >= 255.0f ? 255 : d > 0.0f ? static_cast<int>(d) : 0;
  };
#pragma unroll
  for (int m = 0; m < M; ++m)
    if (tid + m * NT < ncand) atomicAdd(&sh.hist[bucket(key[m])], 1u);
  group_bar(bar_id, NT);
  BKT_STAMP(1);
  // Lane l owns buckets [8l, 8l + 8); the bucket holding the k-th largest
  // key is where the count from the top first reaches k.  Every warp finds
  // it, so no barrier is needed to share it.
  const uint32_t k = static_cast<uint32_t>(k_eff);
  uint32_t c[8], sum = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    c[q] = sh.hist[8 * lane + q];
    sum += c[q];
  }
  uint32_t suf = sum;  // sum over lanes >= this lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(kFull, suf, o);
    if (lane + o < 32) suf += y;
  }
  int my_b = -1;
  uint32_t my_above = 0;
  if (suf - sum < k && k <= suf) {
    uint32_t acc = suf - sum;
#pragma unroll
    for (int q = 7; q >= 0; --q) {
      if (my_b < 0 && acc + c[q] >= k) {
        my_b = 8 * lane + q;
        my_above = acc;
      }
      acc += c[q];
    }
  }
  const int src = __ffs(__ballot_sync(kFull, my_b >= 0)) - 1;  // exactly one lane
  const int B = __shfl_sync(kFull, my_b, src);
  const uint32_t c_above = __shfl_sync(kFull, my_above, src);
  const uint32_t nsurv = sh.hist[B], need = k - c_above;
  if (nsurv > static_cast<uint32_t>(kSurvivorCap)) {  // uniform over the group
    group_topk_from_keys<NT>(scores, ncand, topk, sel_row, sel_cnt, tid, sh, bar_id);
    return;
  }
  const uint32_t nsurv4 = (nsurv + 3u) & ~3u;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int b = tid + m * NT;
    const int bkm = b < ncand ? bucket(key[m]) : -1;
    if (bkm == B) {
      const uint32_t slot = atomicAdd(&sh.nsurv, 1u);
      if (slot < nsurv) sh.surv[slot] = (static_cast<uint64_t>(key[m]) << 32) | ~static_cast<uint32_t>(b);
    }
    const uint32_t hb = __ballot_sync(kFull, bkm > B);
    if (lane == 0) sh.take[m * kW + w] = hb;
  }
  if (tid < 4 && nsurv + tid < nsurv4) sh.surv[nsurv + tid] = 0u;  // below every entry
  group_bar(bar_id, NT);
  BKT_STAMP(2);
  for (int t = tid; t < static_cast<int>(nsurv); t += NT) {
    const uint64_t ct = sh.surv[t];
    uint32_t r0 = 0, r1 = 0;
#pragma unroll 4
    for (uint32_t s2 = 0; s2 < nsurv4; s2 += 2) {
      const ulonglong2 e = *reinterpret_cast<const ulonglong2*>(&sh.surv[s2]);
      r0 += e.x > ct;
      r1 += e.y > ct;
    }
    if (r0 + r1 < need) {
      const uint32_t b = ~static_cast<uint32_t>(ct);
      atomicOr(&sh.take[b >> 5], 1u << (b & 31u));
    }
  }
  group_bar(bar_id, NT);
  BKT_STAMP(3);
  // Exclusive prefix of the words' bit counts, by every warp: lane j scans
  // words [kPer j, kPer j + kPer).
  constexpr int kPer = (kQ + 31) / 32;
  uint32_t pe[kPer];
  uint32_t tot = 0;
#pragma unroll
  for (int x = 0; x < kPer; ++x) {
    const int qq = lane * kPer + x;
    pe[x] = tot;
    const uint32_t wd = sh.take[qq < kQ ? qq : 0];
    tot += qq < kQ ? __popc(wd) : 0u;
  }
  uint32_t inc = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, inc, o);
    if (lane >= o) inc += y;
  }
#pragma unroll
  for (int x = 0; x < kPer; ++x) pe[x] += inc - tot;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int q = m * kW + w;  // this thread's word (uniform over the warp)
    uint32_t v = pe[0];
#pragma unroll
    for (int x = 1; x < kPer; ++x)
      if (q % kPer == x) v = pe[x];
    const uint32_t pre = __shfl_sync(kFull, v, q / kPer);
    const uint32_t word = sh.take[q];
    if ((word >> lane) & 1u) sel_row[pre + __popc(word & lt_mask)] = tid + m * NT;
  }
  for (int x = k_eff + tid; x < topk; x += NT) sel_row[x] = -1;
  if (tid == 0) *sel_cnt = k_eff;
  BKT_STAMP(4);
#undef BKT_STAMP
}

// ---------------------------------------------------------------- scoring
// A scoring chunk k of a (sequence, KV head) covers blocks [15k, 15k+15)
// and pooled windows [60k-1, 60k+60) (61 rows; row r is window 60k-1+r).
// Its rows arrive as four 2-D TMA boxes of {32 fp32 columns, 61 rows}
// (128-byte swizzle), box c holding dimensions [32c, 32c+32), each in an
// 8 KB slot (64 rows) of one ring stage.
constexpr int kScoreSlotBytes = 64 * 128;                          // 8 KB
constexpr uint32_t kScoreTxBytes = 4u * kBoxRows * kBoxCols * 4u;  // bytes landed per chunk
constexpr int kScoreStride = 64 + 4;                               // floats per head row of window scores

__device__ inline void mma_tf32_1688(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 2-D tiled TMA load of one {32 columns, 61 rows} fp32 box of the pooled keys.
__device__ inline void tma_load_keys(void* dst, const CUtensorMap* map, int col, int row, uint64_t* bar,
                                     uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(col), "r"(row), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

template <int G>
struct ScoreQ {
  static constexpr int kNTiles = G > 8 ? 2 : 1;  // n-tiles of 8 heads
  uint32_t b[kNTiles][16][2];
};

// The group's queries as TF32 B fragments of mma m16n8k8 (n = head; heads
// >= G are zero), bf16 widened exactly.  The k slots of each k-step are
// permuted so that a lane's A values are four consecutive dimensions of a
// row (one 16-byte load; see score_stage): with d(u, t) = 32 (u / 2) +
// 4 (2t + u % 2), k-step 2u covers dimensions d + {0, 1} in slots t and
// t + 4, k-step 2u + 1 dimensions d + {2, 3} (t = the lane's quad
// position).  A dot product does not depend on the order of its terms.
template <int G>
__device__ inline void load_score_q(ScoreQ<G>& f, const __nv_bfloat16* __restrict__ q_group, int lane) {
  const int grp = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int nt = 0; nt < ScoreQ<G>::kNTiles; ++nt) {
    const int head = nt * 8 + grp;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int d = 32 * (u >> 1) + 4 * (2 * tig + (u & 1));
      const uint2 w = head < G ? __ldg(reinterpret_cast<const uint2*>(q_group + head * kHeadDim + d)) : make_uint2(0u, 0u);
      f.b[nt][2 * u][0] = w.x << 16;
      f.b[nt][2 * u][1] = w.x & 0xFFFF0000u;
      f.b[nt][2 * u + 1][0] = w.y << 16;
      f.b[nt][2 * u + 1][1] = w.y & 0xFFFF0000u;
    }
  }
}

// Compressed scores of one chunk on the tensor cores: consumer warp w
// computes rows [16w, 16w+16) of S^T = K * Q^T (mma.sync m16n8k8, TF32
// inputs, fp32 accumulation) and stores scale * s into ssm[head][row] for
// rows < 61.  Each fp32 pooled value x is split into hi (x with its low 13
// mantissa bits cleared, exact in TF32) and lo = x - hi (exact in fp32, of
// which the tensor core reads the TF32 part); the hi and lo products go to
// separate fp32 accumulators that are added at the end, so the only input
// rounding is that of lo, below 2^-20 of |x| ("NOSA-1B 性能基准全解析" §三.3:
// scores of the pooled keys).  A lane reads its four dimensions of a row
// (see load_score_q) with one 16-byte load per row and k-step pair: 16-byte
// unit 2t + u % 2 of the row's 128-byte box row, so that the two rows a
// quarter warp reads (their row indices differ in the lowest bit, which the
// 128-byte swizzle XORs into the unit) fall on disjoint banks.
template <int G>
__device__ inline void score_stage(const ScoreQ<G>& qf, uint32_t stage, float* __restrict__ ssm, float scale,
                                   int warp, int lane) {
  constexpr int NT = ScoreQ<G>::kNTiles;
  const int grp = lane >> 2, tig = lane & 3;
  const int r0 = warp * 16;
  const int ra = r0 + grp, rb = ra + 8;
  // Four independent accumulation chains per n-tile (hi / lo x even / odd
  // k-step) keep the tensor pipe busy instead of waiting on one chain.
  float acc_hi[2][NT][4], acc_lo[2][NT][4];
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc_hi[c][nt][e] = acc_lo[c][nt][e] = 0.0f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {  // k-steps 2u, 2u + 1
    const uint32_t box = stage + (u >> 1) * kScoreSlotBytes;
    const int unit = 2 * tig + (u & 1);  // dimensions d(u, tig) .. + 3 of the box row
    uint32_t va[4], vb[4];
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(va[0]), "=r"(va[1]), "=r"(va[2]), "=r"(va[3])
                 : "r"(box + ra * 128 + ((unit ^ (ra & 7)) << 4)));
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(vb[0]), "=r"(vb[1]), "=r"(vb[2]), "=r"(vb[3])
                 : "r"(box + rb * 128 + ((unit ^ (rb & 7)) << 4)));
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // k-step 2u + h: dimensions d(u, tig) + 2h + {0, 1}
      const uint32_t x[4] = {va[2 * h], vb[2 * h], va[2 * h + 1], vb[2 * h + 1]};
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hi[e] = x[e] & 0xffffe000u;
        lo[e] = __float_as_uint(__uint_as_float(x[e]) - __uint_as_float(hi[e]));
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_tf32_1688(acc_hi[h][nt], hi, qf.b[nt][2 * u + h][0], qf.b[nt][2 * u + h][1]);
        mma_tf32_1688(acc_lo[h][nt], lo, qf.b[nt][2 * u + h][0], qf.b[nt][2 * u + h][1]);
      }
    }
  }
  // acc[nt][0..1]: row ra, heads nt*8 + 2*tig + {0,1}; [2..3]: row rb.
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int head = nt * 8 + 2 * tig + (e & 1);
      const int row = (e >> 1) ? rb : ra;
      if (head < G && row < kChunkWindows)
        ssm[head * kScoreStride + row] =
            ((acc_hi[0][nt][e] + acc_hi[1][nt][e]) + (acc_lo[0][nt][e] + acc_lo[1][nt][e])) * scale;
    }
  }
}

// Two chunks in one pass (stage[c] -> ssm[c]), each scored exactly as
// score_stage scores it: the chunks' products are independent accumulation
// chains, so the pass keeps twice as many tensor-core operations in flight.
template <int G>
__device__ inline void score_stage_pair(const ScoreQ<G>& qf, const uint32_t (&stage)[2], float* const (&ssm)[2],
                                        float scale, int warp, int lane) {
  constexpr int NT = ScoreQ<G>::kNTiles;
  const int grp = lane >> 2, tig = lane & 3;
  const int r0 = warp * 16;
  const int ra = r0 + grp, rb = ra + 8;
  float acc_hi[2][2][NT][4], acc_lo[2][2][NT][4];  // [chunk][k-step parity][n-tile][fragment]
#pragma unroll
  for (int x = 0; x < 2; ++x)
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc_hi[x][c][nt][e] = acc_lo[x][c][nt][e] = 0.0f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {  // k-steps 2u, 2u + 1
    const int unit = 2 * tig + (u & 1);
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      const uint32_t box = stage[x] + (u >> 1) * kScoreSlotBytes;
      uint32_t va[4], vb[4];
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(va[0]), "=r"(va[1]), "=r"(va[2]), "=r"(va[3])
                   : "r"(box + ra * 128 + ((unit ^ (ra & 7)) << 4)));
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(vb[0]), "=r"(vb[1]), "=r"(vb[2]), "=r"(vb[3])
                   : "r"(box + rb * 128 + ((unit ^ (rb & 7)) << 4)));
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t xv[4] = {va[2 * h], vb[2 * h], va[2 * h + 1], vb[2 * h + 1]};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = xv[e] & 0xffffe000u;
          lo[e] = __float_as_uint(__uint_as_float(xv[e]) - __uint_as_float(hi[e]));
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_tf32_1688(acc_hi[x][h][nt], hi, qf.b[nt][2 * u + h][0], qf.b[nt][2 * u + h][1]);
          mma_tf32_1688(acc_lo[x][h][nt], lo, qf.b[nt][2 * u + h][0], qf.b[nt][2 * u + h][1]);
        }
      }
    }
  }
#pragma unroll
  for (int x = 0; x < 2; ++x)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int head = nt * 8 + 2 * tig + (e & 1);
        const int row = (e >> 1) ? rb : ra;
        if (head < G && row < kChunkWindows)
          ssm[x][head * kScoreStride + row] =
              ((acc_hi[x][0][nt][e] + acc_hi[x][1][nt][e]) + (acc_lo[x][0][nt][e] + acc_lo[x][1][nt][e])) * scale;
      }
    }
}

// bf16 pooled keys: a chunk's rows arrive as two 2-D TMA boxes of {64 bf16
// columns, 61 rows} (128-byte swizzle), box c holding dimensions
// [64c, 64c+64), in the first two 8 KB slots of the stage.
constexpr uint32_t kScoreTxBytesBf16 = 2u * kBoxRows * 128u;  // bytes landed per chunk

template <int G>
struct ScoreQBf16 {
  static constexpr int kNTiles = G > 8 ? 2 : 1;  // n-tiles of 8 heads
  uint32_t b[kNTiles][8][2];
};

// The group's queries as bf16 B fragments of mma m16n8k16 (k = dimension,
// n = head; heads >= G are zero).
template <int G>
__device__ inline void load_score_q_bf16(ScoreQBf16<G>& f, const __nv_bfloat16* __restrict__ q_group, int lane) {
  const int grp = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int nt = 0; nt < ScoreQBf16<G>::kNTiles; ++nt) {
    const int head = nt * 8 + grp;
    const uint32_t* row = reinterpret_cast<const uint32_t*>(q_group + head * kHeadDim);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      f.b[nt][ks][0] = head < G ? __ldg(row + ks * 8 + tig) : 0u;      // dims 16ks + 2tig, +1
      f.b[nt][ks][1] = head < G ? __ldg(row + ks * 8 + tig + 4) : 0u;  // dims 16ks + 2tig + 8, +9
    }
  }
}

// Compressed scores of one chunk of bf16 pooled keys: S^T = K * Q^T on
// mma.sync m16n8k16 (bf16 inputs, exact products, fp32 accumulation), the A
// fragments read with ldmatrix from the swizzled boxes.  Warp w computes rows
// [16w, 16w+16) and stores scale * s into ssm[head][row] for rows < 61, as
// score_stage does.
template <int G>
__device__ inline void score_stage_bf16(const ScoreQBf16<G>& qf, uint32_t stage, float* __restrict__ ssm, float scale,
                                        int warp, int lane) {
  constexpr int NT = ScoreQBf16<G>::kNTiles;
  const int grp = lane >> 2, tig = lane & 3;
  const int r0 = warp * 16;
  const int mat = lane >> 3;                             // ldmatrix: which 8x8 matrix this lane addresses
  const int arow = r0 + (mat & 1) * 8 + (lane & 7);
  float acc[2][NT][4];
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[c][nt][e] = 0.0f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int k8 = 2 * ks + (mat >> 1);                  // 8-dimension chunk 0..15
    uint32_t a[4];
    ldsm_x4(swz(stage + (k8 >> 3) * kScoreSlotBytes, arow, k8 & 7), a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[ks & 1][nt], a, qf.b[nt][ks][0], qf.b[nt][ks][1]);
  }
  const int ra = r0 + grp, rb = ra + 8;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int head = nt * 8 + 2 * tig + (e & 1);
      const int row = (e >> 1) ? rb : ra;
      if (head < G && row < kChunkWindows) ssm[head * kScoreStride + row] = (acc[0][nt][e] + acc[1][nt][e]) * scale;
    }
  }
}

// Block rule for the blocks of chunk k, from the chunk's window scores:
// S[b] = sum over the group's heads of the max of s over windows
// 4b-1 .. 4b+3 that exist (0 <= j < nc), i.e. rows 4t .. 4t+4 for block
// b = 15k + t.  Spread over the consumer threads: min(G, 8) lanes per block,
// each taking the window max of G / min(G, 8) heads, then a fixed shuffle
// tree sums the heads.  Every thread of the (full) warps calls it; every
// lane of block t's lanes gets S[b] in *out (the butterfly adds the same
// operands in every lane, so they agree bit for bit) and true.
template <int G>
__device__ inline bool block_rule(const float* __restrict__ ssm, int k, int nblk, int64_t nc, int tid, float* out) {
  constexpr int kLanes = G < 8 ? G : 8;   // lanes per block
  constexpr int kHeads = G / kLanes;      // heads per lane
  const int t = tid / kLanes, hl = tid % kLanes;
  const int64_t jb = static_cast<int64_t>(kWindowsPerBlock) * (kChunkBlocks * k + t) - 1;
  float part = 0.0f;
  if (t < nblk) {
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh) {
      const int h = hl * kHeads + hh;
      float m = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWindowsPerBlock + 1; ++w) {
        const int64_t j = jb + w;
        if (j >= 0 && j < nc) m = fmaxf(m, ssm[h * kScoreStride + 4 * t + w]);
      }
      part += m;
    }
  }
#pragma unroll
  for (int o = kLanes / 2; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  *out = part;
  return t < nblk;
}

}  // namespace nosa
