// Exact attention over the selected blocks plus the local window: the decode
// work item shared by the standalone attention launch and the persistent
// decode-step kernel.
//
// "NOSA-1B 性能基准全解析" (wmrh.cn) §三.3: the TopK blocks chosen from the
// compressed scores get exact attention; §三.2: every query also attends to
// its fixed local window (1024 tokens = 16 blocks of 64).
//
//   T   = (U_{b in sel} [64b, 64b+64) U [64*ncand, L)) n [0, L)
//   out = sum_{t in T} softmax_t(scale * q . k_t) v_t
//
// One item = (sequence i, KV head g, split s).  The pair's tile list is the
// local blocks [ncand, nb) followed by the selected blocks; split s takes the
// balanced range [s*n/S, (s+1)*n/S).  Every tile is read once for all G query
// heads of the group.
//
// Data movement: one producer thread issues, per 64-token tile, four 3-D
// tensor-TMA boxes {64 dims, 1 head, 64 tokens} (K low/high dims, V low/high
// dims; cp.async.bulk.tensor with the 128-byte swizzle) into a 3-stage ring,
// one mbarrier per stage (expect_tx) plus empty barriers for reuse; the ring
// position carries over from item to item.  Rows past the cache allocation
// are zero-filled by the TMA unit; rows past the sequence end are masked out
// of the softmax and their V rows zeroed in shared memory (then a proxy fence
// before the stage is reused), so stale or garbage rows cannot produce NaN.
//
// Math: four consumer warps each own 16 of the tile's 64 tokens.  With the
// group's queries as the A operand (16 rows, heads >= G zero) a warp runs
// S = Q K^T and O += P V on bf16 tensor cores (mma.sync m16n8k16, fp32
// accumulate); the S accumulator is re-packed in registers as the A operand
// of P V.  Each warp keeps its own online softmax (row max m, row sum l, O)
// in the exp2 domain.  The four warps merge in fixed order in shared memory;
// with several splits the partial (O, m, l) goes to the workspace and the
// last item of the pair (atomic ticket, no spinning) merges the splits in
// split order, so results are bit-reproducible.
#pragma once

#include <cuda.h>

#include "nosa_common.cuh"
#include "nosa_kernels.h"

namespace nosa {

constexpr int kDecConsumerWarps = 4;
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;  // 160
constexpr int kStages = 3;
constexpr int kHalfBytes = kBlock * 128;                   // one 64-token x 64-dim box: 8 KB
constexpr int kStageBytes = 4 * kHalfBytes;                // K lo/hi, V lo/hi: 32 KB
constexpr int kRingBytes = kStages * kStageBytes;          // 96 KB
constexpr uint32_t kTileTxBytes = kStageBytes;
constexpr float kLn2 = 0.69314718055994530942f;

__device__ inline void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ inline void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                     uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ inline void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ inline uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// 3-D tiled TMA load of one {64 dims, 1 head, 64 tokens} box, completing on
// `bar`, with the given L2 cache policy.
__device__ inline void tma_load_box(void* dst, const CUtensorMap* map, int dim0, int head, int row,
                                    uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(dim0), "r"(head), "r"(row), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Address of 16-byte chunk `chunk` (0..7) of row `row` in a box written with
// the 128-byte swizzle: chunks are permuted by XOR with (row mod 8).
__device__ inline uint32_t swz(uint32_t box_base, int row, int chunk) {
  return box_base + row * 128 + ((chunk ^ (row & 7)) << 4);
}

// Bounded wait for a pair's selection, published by another CTA of the same
// launch with a release store; on giving up sets NOSA_DEV_TIMEOUT.
__device__ inline bool wait_ready(const uint32_t* flag, uint32_t* status) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0; it < kWaitLimitIters; ++it) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0u) {
      // Make the generic-proxy writes published with the flag (the appended
      // K/V row) visible to this thread's following TMA reads.
      asm volatile("fence.proxy.async.global;" ::: "memory");
      return true;
    }
    __nanosleep(200);
    if ((it & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) break;
  }
  set_status(status, NOSA_DEV_TIMEOUT);
  return false;
}

constexpr int kSelList = 128;  // selected block indices a split stages in shared memory

struct DecodeShared {
  uint64_t full_bar[kStages];
  uint64_t empty_bar[kStages];
  uint64_t merge_bar;     // bulk copies of the split partials (final merge)
  uint32_t merge_phase;   // its current parity
  int stage_blk[kStages];
  int last;
  int sel_list[kSelList];
#ifdef NOSA_TRACE
  uint64_t t_flag;  // instrumented builds: when the producer saw the selection
  uint64_t t_issue[8], t_full[8], t_done[8];  // per tile: TMA issued, landed, consumed (warp 0)
  uint64_t t_merge[6];  // drained, warps merged, partial written, ticket taken, splits loaded, done
#endif
};

// One decode item with 160 threads (4 consumer warps + 1 producer warp).
// `ready` (nullable): the pair's selection flag, waited on before the first
// tile that depends on the selection or on the appended token; when given,
// the tile count is the selector's (min(topk, ncand)) rather than sel_cnt.
// `ring_n` is the CTA's running tile count (uniform), advanced by the item.
__device__ inline void decode_item(const DecodeArgs& a, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                   int pair, int split, uint32_t* ready, uint32_t& ring_n, uint8_t* smem,
                                   DecodeShared& sh) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = pair / a.hkv, g = pair % a.hkv;
  const int G = a.group;
  const int L = a.seq_len[i];
  const int64_t seq_base = a.seq_start[i];
  const int64_t out_row0 = static_cast<int64_t>(i) * a.hq + static_cast<int64_t>(g) * G;
  const bool bad_len = L < 1 || L > a.max_seq_len;
  const bool bad_rows = !bad_len && (seq_base < 0 || seq_base + L > a.cache_rows);
  if (bad_len || bad_rows) {
    if (split == 0) {
      if (tid == 0)
        set_status(a.status, bad_rows ? NOSA_DEV_CACHE_ROWS : (L < 1 ? NOSA_DEV_BAD_LENGTH : NOSA_DEV_MAX_LEN));
      for (int t = tid; t < G * kHeadDim; t += kDecThreads)
        a.out[out_row0 * kHeadDim + t] = __float2bfloat16_rn(0.0f);
      if (a.lse)
        for (int t = tid; t < G; t += kDecThreads) a.lse[out_row0 + t] = -INFINITY;
    }
    return;
  }
  const int nb = static_cast<int>(n_blocks(L));
  const int ncand = static_cast<int>(n_candidates(L, a.local_blocks));
  const int n_local = nb - ncand;
  const int cnt_max = min(a.topk, ncand);
  int cnt = cnt_max;
  if (ready == nullptr) {
    cnt = a.sel_cnt[pair];
    if (cnt < 0 || cnt > cnt_max) {
      if (split == 0 && tid == 0) set_status(a.status, NOSA_DEV_BAD_COUNT);
      cnt = cnt < 0 ? 0 : cnt_max;
    }
  }
  const int ntiles = n_local + cnt;
  const int t_begin = static_cast<int>((static_cast<int64_t>(split) * ntiles) / a.nsplit);
  const int t_end = static_cast<int>((static_cast<int64_t>(split + 1) * ntiles) / a.nsplit);
  const int my_n = t_end - t_begin;
  const int32_t* sel = a.sel_idx + static_cast<int64_t>(pair) * a.topk;

  float acc[16][4];
  float m_r[2] = {-INFINITY, -INFINITY};
  float l_r[2] = {0.0f, 0.0f};
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;

  if (warp == kDecConsumerWarps) {
    // ---------------------------------------------------------------- producer
    // The whole warp walks the tiles; lane 0 waits and issues the copies.
    // Once the selection is known, the warp fetches this split's selected
    // block indices into shared memory in one parallel round trip.
    const uint64_t policy = l2_evict_first_policy();
    const int first_sel = max(t_begin, n_local);
    const int n_sel = max(0, t_end - first_sel);
    bool have_sel = ready == nullptr;
    bool sel_ok = have_sel;
    auto load_sel_list = [&]() {
      for (int x = lane; x < min(n_sel, kSelList); x += 32) sh.sel_list[x] = __ldcg(sel + (first_sel - n_local) + x);
      __syncwarp();
    };
    if (have_sel) load_sel_list();
    int issued = 0;
    for (int n = 0; n < my_n; ++n) {
      const int t = t_begin + n;
      // The selected tiles and the last local block (it holds the token
      // appended by this launch) wait for the pair's selection flag.
      if (!have_sel && t >= n_local - 1) {
        int ok = 0;
        if (lane == 0) {
          ok = wait_ready(ready, a.status) ? 1 : 0;
#ifdef NOSA_TRACE
          sh.t_flag = global_timer_ns();
#endif
          if (ok && __ldcg(a.sel_cnt + pair) != cnt) set_status(a.status, NOSA_DEV_BAD_COUNT);
        }
        sel_ok = __shfl_sync(0xffffffffu, ok, 0) != 0;
        have_sel = true;
        if (sel_ok) load_sel_list();
      }
      int stop = 0;
      if (lane == 0) {
        int blk;
        if (t < n_local) {
          blk = ncand + t;
        } else if (!sel_ok) {
          blk = -1;
        } else {
          const int x = t - first_sel;
          blk = x < kSelList ? sh.sel_list[x] : __ldcg(sel + (t - n_local));
          if (blk < 0 || blk >= ncand) {
            set_status(a.status, NOSA_DEV_BAD_INDEX);
            blk = -1;
          }
        }
        const uint32_t r = ring_n + static_cast<uint32_t>(n);
        const int s = static_cast<int>(r % kStages);
        if (r >= static_cast<uint32_t>(kStages) &&
            !mbar_wait(&sh.empty_bar[s], ((r / kStages) - 1) & 1u, a.status)) {
          stop = 1;
        } else {
          sh.stage_blk[s] = blk;
          const int row = static_cast<int>(seq_base + (blk < 0 ? 0 : static_cast<int64_t>(blk) * kBlock));
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&sh.full_bar[s], kTileTxBytes);
          tma_load_box(st, tm_k, 0, g, row, &sh.full_bar[s], policy);
          tma_load_box(st + kHalfBytes, tm_k, 64, g, row, &sh.full_bar[s], policy);
          tma_load_box(st + 2 * kHalfBytes, tm_v, 0, g, row, &sh.full_bar[s], policy);
          tma_load_box(st + 3 * kHalfBytes, tm_v, 64, g, row, &sh.full_bar[s], policy);
#ifdef NOSA_TRACE
          if (n < 8) sh.t_issue[n] = global_timer_ns();
#endif
          issued = n + 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) break;
    }
    // Every copy issued has landed before shared memory is reused.
    if (lane == 0) {
      for (int n = max(0, issued - kStages); n < issued; ++n) {
        const uint32_t r = ring_n + static_cast<uint32_t>(n);
        mbar_wait(&sh.full_bar[r % kStages], (r / kStages) & 1u, a.status);
      }
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int grp = lane >> 2, tig = lane & 3;
    // Q as the A operand: rows = heads of the group (zero past G), 8 k-steps of 16 dims.
    uint32_t qa[8][4];
    const __nv_bfloat16* qbase = a.q + out_row0 * kHeadDim;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = grp + (r & 1) * 8;
        const int col = ks * 16 + 2 * tig + (r >> 1) * 8;
        qa[ks][r] = row < G ? __ldg(reinterpret_cast<const uint32_t*>(qbase + row * kHeadDim + col)) : 0u;
      }
    }
    const int wrow = warp * 16;  // this warp's 16 tokens of the tile
    for (int n = 0; n < my_n; ++n) {
      const uint32_t r = ring_n + static_cast<uint32_t>(n);
      const int s = static_cast<int>(r % kStages);
      if (!mbar_wait(&sh.full_bar[s], (r / kStages) & 1u, a.status)) break;
#ifdef NOSA_TRACE
      if (warp == 0 && lane == 0 && n < 8) sh.t_full[n] = global_timer_ns();
#endif
      const int blk = sh.stage_blk[s];
      uint8_t* st = smem + s * kStageBytes;
      const uint32_t k_lo = smem_addr(st);
      const uint32_t v_lo = k_lo + 2 * kHalfBytes;
      const int64_t tok0 = static_cast<int64_t>(blk) * kBlock + wrow;
      // Rows of this warp past the sequence end (or of a rejected tile) may
      // hold anything; zero their V rows so that P = 0 cannot meet a NaN.
      const bool partial = blk < 0 || tok0 + 16 > L;
      if (partial) {
        for (int idx = lane; idx < 16 * 16; idx += 32) {
          const int rr = idx >> 4, c16 = idx & 15;
          if (blk < 0 || tok0 + rr >= L) {
            const int row = wrow + rr;
            *reinterpret_cast<uint4*>(st + 2 * kHalfBytes + (c16 >> 3) * kHalfBytes + row * 128 +
                                      (((c16 & 7) ^ (row & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        __syncwarp();
      }
      // S = Q K^T over this warp's 16 tokens (two n-tiles of 8).
      float sc[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
        const int row = wrow + nt * 8 + (lane & 7);
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(swz(k_lo + (kp >> 1) * kHalfBytes, row, (kp & 1) * 4 + (lane >> 3)), b0, b1, b2, b3);
          mma_bf16_16816(sc[nt], qa[2 * kp], b0, b1);
          mma_bf16_16816(sc[nt], qa[2 * kp + 1], b2, b3);
        }
      }
      // Scale into the exp2 domain and mask tokens outside [0, L) / rejected tiles.
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t tok = tok0 + nt * 8 + 2 * tig + (e & 1);
          const bool valid = blk >= 0 && tok < L;
          sc[nt][e] = valid ? sc[nt][e] * a.scale_log2 : -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], sc[nt][e]);
        }
      }
      float alpha[2], m_use[2];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
        mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
        const float m_new = fmaxf(m_r[rr], mx[rr]);
        m_use[rr] = m_new == -INFINITY ? 0.0f : m_new;
        alpha[rr] = exp2f(m_r[rr] - m_use[rr]);
        m_r[rr] = m_new;
      }
      float rs[2] = {0.0f, 0.0f};
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sc[nt][e] = exp2f(sc[nt][e] - m_use[e >> 1]);
          rs[e >> 1] += sc[nt][e];
        }
      }
      l_r[0] = l_r[0] * alpha[0] + rs[0];
      l_r[1] = l_r[1] * alpha[1] + rs[1];
#pragma unroll
      for (int d = 0; d < 16; ++d) {
        acc[d][0] *= alpha[0];
        acc[d][1] *= alpha[0];
        acc[d][2] *= alpha[1];
        acc[d][3] *= alpha[1];
      }
      // P as the A operand (m16 x k16 over the warp's 16 tokens).
      const uint32_t pa[4] = {pack_bf16x2(sc[0][0], sc[0][1]), pack_bf16x2(sc[0][2], sc[0][3]),
                              pack_bf16x2(sc[1][0], sc[1][1]), pack_bf16x2(sc[1][2], sc[1][3])};
      // O += P V: V^T fragments via transposed ldmatrix, 16 dims per load.
      const int vrow = wrow + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(swz(v_lo + (dp >> 2) * kHalfBytes, vrow, (dp & 3) * 2 + (lane >> 4)), b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * dp], pa, b0, b1);
        mma_bf16_16816(acc[2 * dp + 1], pa, b2, b3);
      }
      if (partial) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.empty_bar[s]);
#ifdef NOSA_TRACE
      if (warp == 0 && lane == 0 && n < 8) sh.t_done[n] = global_timer_ns();
#endif
    }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 1);
      l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 2);
    }
  }
  ring_n += static_cast<uint32_t>(my_n);
  __syncthreads();  // ring drained: reuse it for the cross-warp merge
#ifdef NOSA_TRACE
#define NOSA_MSTAMP(k) \
  if (tid == 0) sh.t_merge[k] = global_timer_ns()
#else
#define NOSA_MSTAMP(k)
#endif
  NOSA_MSTAMP(0);

  // Cross-warp merge in fixed warp order.  Each warp's O goes to shared
  // memory as float2 pairs with a padded row stride (bank-conflict free);
  // per-row weights are computed once.
  constexpr int kMoStride = kHeadDim + 8;                         // floats per merge row
  float* mo = reinterpret_cast<float*>(smem);                     // [4][G][kMoStride]
  float* mm = mo + kDecConsumerWarps * G * kMoStride;             // [4][G] row max
  float* ml = mm + kDecConsumerWarps * G;                         // [4][G] row sum
  float* mw = ml + kDecConsumerWarps * G;                         // [4][G] weights
  float* mrow = mw + kDecConsumerWarps * G;                       // [G] M, then [G] L
  if (warp < kDecConsumerWarps) {
    const int grp = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int d = 0; d < 16; ++d) {
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int row = grp + h2 * 8;
        if (row < G)
          *reinterpret_cast<float2*>(mo + (warp * G + row) * kMoStride + d * 8 + 2 * tig) =
              make_float2(acc[d][2 * h2], acc[d][2 * h2 + 1]);
      }
    }
    if (tig == 0) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int row = grp + rr * 8;
        if (row < G) {
          mm[warp * G + row] = m_r[rr];
          ml[warp * G + row] = l_r[rr];
        }
      }
    }
  }
  __syncthreads();
  for (int row = tid; row < G; row += kDecThreads) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecConsumerWarps; ++w) M = fmaxf(M, mm[w * G + row]);
    float lsum = 0.0f;
#pragma unroll
    for (int w = 0; w < kDecConsumerWarps; ++w) {
      const float m_w = mm[w * G + row];
      const float f = m_w == -INFINITY ? 0.0f : exp2f(m_w - M);
      mw[w * G + row] = f;
      lsum += ml[w * G + row] * f;
    }
    mrow[row] = M;
    mrow[G + row] = lsum;
  }
  __syncthreads();
  NOSA_MSTAMP(1);

  const bool single = a.nsplit == 1;
  const int stride = part_stride(G);
  float* part = a.part + (static_cast<int64_t>(pair) * kMaxSplits + split) * stride;
  constexpr int kVec = kHeadDim / 4;
  for (int t = tid; t < G * kVec; t += kDecThreads) {
    const int row = t / kVec, d4 = t % kVec;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kDecConsumerWarps; ++w) {
      const float f = mw[w * G + row];
      const float4 x = *reinterpret_cast<const float4*>(mo + (w * G + row) * kMoStride + 4 * d4);
      o.x = fmaf(f, x.x, o.x);
      o.y = fmaf(f, x.y, o.y);
      o.z = fmaf(f, x.z, o.z);
      o.w = fmaf(f, x.w, o.w);
    }
    if (single) {
      const float lsum = mrow[G + row];
      const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(a.out + (out_row0 + row) * kHeadDim + 4 * d4);
      dst[0] = __floats2bfloat162_rn(o.x * inv, o.y * inv);
      dst[1] = __floats2bfloat162_rn(o.z * inv, o.w * inv);
      if (a.lse && d4 == 0) a.lse[out_row0 + row] = lsum > 0.0f ? (mrow[row] + log2f(lsum)) * kLn2 : -INFINITY;
    } else {
      reinterpret_cast<float4*>(part + row * kHeadDim)[d4] = o;
    }
  }
  if (!single)
    for (int row = tid; row < G; row += kDecThreads) {
      part[G * kHeadDim + row] = mrow[row];
      part[G * kHeadDim + G + row] = mrow[G + row];
    }
  if (single) {
    if (ready != nullptr && tid == 0) *ready = 0u;  // the pair's only item: re-arm the flag
    return;
  }

  // Publish this split's partial, then take a ticket; the last split of the
  // pair merges all of them.
  __threadfence();
  __syncthreads();
  NOSA_MSTAMP(2);
  if (tid == 0) {
    const uint32_t t = atomicAdd(&a.tickets[pair], 1u);
    sh.last = (t == static_cast<uint32_t>(a.nsplit - 1));
  }
  __syncthreads();
  NOSA_MSTAMP(3);
  if (!sh.last) return;
  if (tid == 0) __threadfence();  // acquire: the other splits' partials
  __syncthreads();
  // Merge the splits in split order.  The partials (O, m, l of every split)
  // are staged in shared memory by 1-D bulk (TMA) copies -- all of them in
  // one copy when they fit -- then the weights and the weighted sums are
  // computed from there.
  const float* pbase = a.part + static_cast<int64_t>(pair) * kMaxSplits * stride;
  float* sm_w = reinterpret_cast<float*>(smem + kRingBytes - (kMaxSplits * kMaxGroup + 2 * kMaxGroup) * 4);
  float* sm_L = sm_w + kMaxSplits * kMaxGroup;                    // [G]
  float* sm_M = sm_L + kMaxGroup;                                 // [G]
  const int stage_bytes_max = kRingBytes - (kMaxSplits * kMaxGroup + 2 * kMaxGroup) * 4;
  const int per_copy = max(1, stage_bytes_max / (stride * 4));
  const bool one_copy = a.nsplit <= per_copy;
  // The TMA unit reads next the other splits' partials (published by their
  // tickets) and writes shared memory this CTA wrote with plain stores.
  asm volatile("fence.proxy.async;" ::: "memory");
  __syncthreads();
  const float* stg = reinterpret_cast<const float*>(smem);
  if (one_copy && tid == 0) {
    const uint32_t bytes = static_cast<uint32_t>(a.nsplit * stride * 4);
    mbar_arrive_expect_tx(&sh.merge_bar, bytes);
    bulk_copy_g2s(smem, pbase, bytes, &sh.merge_bar);
  }
  // (m, l) of split sp, row r: from the staged copy, or from global memory.
  auto m_of = [&](int sp, int r) {
    return one_copy ? stg[sp * stride + G * kHeadDim + r] : __ldcg(pbase + sp * stride + G * kHeadDim + r);
  };
  auto l_of = [&](int sp, int r) {
    return one_copy ? stg[sp * stride + G * kHeadDim + G + r] : __ldcg(pbase + sp * stride + G * kHeadDim + G + r);
  };
  if (one_copy) mbar_wait(&sh.merge_bar, sh.merge_phase, a.status);
  for (int row = tid; row < G; row += kDecThreads) {
    float M = -INFINITY;
    for (int sp = 0; sp < a.nsplit; ++sp) M = fmaxf(M, m_of(sp, row));
    sm_M[row] = M;
  }
  __syncthreads();
  for (int t = tid; t < a.nsplit * G; t += kDecThreads) {
    const int sp = t / G, row = t % G;
    const float ms = m_of(sp, row);
    sm_w[t] = ms == -INFINITY ? 0.0f : exp2f(ms - sm_M[row]);
  }
  __syncthreads();
  for (int row = tid; row < G; row += kDecThreads) {
    float lsum = 0.0f;
    for (int sp = 0; sp < a.nsplit; ++sp) lsum += l_of(sp, row) * sm_w[sp * G + row];
    sm_L[row] = lsum;
  }
  NOSA_MSTAMP(4);
  // Each thread owns output float4s t = tid, tid + 160, ... (at most 4).
  constexpr int kOwn = (kMaxGroup * kVec + kDecThreads - 1) / kDecThreads;
  float4 o[kOwn];
#pragma unroll
  for (int k = 0; k < kOwn; ++k) o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sp0 = 0; sp0 < a.nsplit; sp0 += per_copy) {
    const int nsp = min(per_copy, a.nsplit - sp0);
    if (!one_copy) {
      if (tid == 0) {
        const uint32_t bytes = static_cast<uint32_t>(nsp * stride * 4);
        mbar_arrive_expect_tx(&sh.merge_bar, bytes);
        bulk_copy_g2s(smem, pbase + static_cast<int64_t>(sp0) * stride, bytes, &sh.merge_bar);
      }
      mbar_wait(&sh.merge_bar, sh.merge_phase, a.status);
    }
#pragma unroll
    for (int k = 0; k < kOwn; ++k) {
      const int t = tid + k * kDecThreads;
      if (t < G * kVec) {
        const int row = t / kVec, d4 = t % kVec;
        for (int sp = 0; sp < nsp; ++sp) {
          const float w = sm_w[(sp0 + sp) * G + row];
          const float4 x = *reinterpret_cast<const float4*>(stg + sp * stride + row * kHeadDim + 4 * d4);
          o[k].x = fmaf(w, x.x, o[k].x);
          o[k].y = fmaf(w, x.y, o[k].y);
          o[k].z = fmaf(w, x.z, o[k].z);
          o[k].w = fmaf(w, x.w, o[k].w);
        }
      }
    }
    __syncthreads();  // everyone is done with the staged splits
    if (tid == 0) sh.merge_phase ^= 1u;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
  }
#pragma unroll
  for (int k = 0; k < kOwn; ++k) {
    const int t = tid + k * kDecThreads;
    if (t < G * kVec) {
      const int row = t / kVec, d4 = t % kVec;
      const float lsum = sm_L[row];
      const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(a.out + (out_row0 + row) * kHeadDim + 4 * d4);
      dst[0] = __floats2bfloat162_rn(o[k].x * inv, o[k].y * inv);
      dst[1] = __floats2bfloat162_rn(o[k].z * inv, o[k].w * inv);
      if (a.lse && d4 == 0) a.lse[out_row0 + row] = lsum > 0.0f ? (sm_M[row] + log2f(lsum)) * kLn2 : -INFINITY;
    }
  }
  if (tid == 0) {
    a.tickets[pair] = 0u;
    if (ready != nullptr) *ready = 0u;  // every item of the pair has passed its wait
  }
  NOSA_MSTAMP(5);
}

}  // namespace nosa
