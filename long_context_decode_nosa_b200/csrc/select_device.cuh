// Compressed scores, block scores and top-k selection: device routines shared
// by the selection-only kernel and the persistent decode-step kernel.
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

#include "nosa_common.cuh"

namespace nosa {

constexpr int kChunkBlocks = 16;                                     // blocks per scoring item
constexpr int kChunkWindows = kChunkBlocks * kWindowsPerBlock + 1;   // 65 pooled rows
constexpr int kScoreStride = 68;                                     // floats per head row
constexpr int kKeyBytes = kHeadDim * 4;                              // one fp32 pooled key
constexpr int kScoreKeysBytes = kChunkWindows * kKeyBytes;           // 33,280
constexpr int kScoreSmemBytes = kScoreKeysBytes + kMaxGroup * kScoreStride * 4;

// Exchange half of `v` (N values) with lane ^ off; keep the half this lane's
// side owns, added to the partner's copy of it.
template <int N>
__device__ inline void xpose_step(float* v, int lane, int off) {
  const bool upper = (lane & off) != 0;
#pragma unroll
  for (int k = 0; k < N / 2; ++k) {
    const float send = upper ? v[k] : v[k + N / 2];
    const float keep = upper ? v[k + N / 2] : v[k];
    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
  }
}

template <int G>
__host__ __device__ constexpr int log2_of() {
  return G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : G == 8 ? 3 : 4;
}

// Sum over the 32 lanes of v[h] for the head h this lane ends up owning:
// log2(G) halving exchanges, then 5 - log2(G) plain butterfly steps.
template <int G>
__device__ inline float group_warp_sum(float (&v)[G], int lane, int* head) {
  int h = 0;
  if constexpr (G >= 2) {
    xpose_step<G>(v, lane, 16);
    h += (lane & 16) ? G / 2 : 0;
  }
  if constexpr (G >= 4) {
    xpose_step<G / 2>(v, lane, 8);
    h += (lane & 8) ? G / 4 : 0;
  }
  if constexpr (G >= 8) {
    xpose_step<G / 4>(v, lane, 4);
    h += (lane & 4) ? G / 8 : 0;
  }
  if constexpr (G >= 16) {
    xpose_step<G / 8>(v, lane, 2);
    h += (lane & 2) ? G / 16 : 0;
  }
  float s = v[0];
#pragma unroll
  for (int o = 16 >> log2_of<G>(); o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  *head = h;
  return s;
}

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

struct ScoreGeometry {
  int L, nb, ncand, nchunks, b0, b1, jlo, jhi;
  int64_t nc;
};

// Scores one chunk of 16 blocks of one (sequence i, KV head g) with NT
// threads: one 1-D bulk (TMA) copy stages the chunk's pooled rows
// [4*b0-1, 4*b1) in shared memory (`keys`), each warp scores one window at a
// time with the group's queries in registers, and the block rule runs from
// shared memory (`ssm`).  Writes block scores to `bscratch` (and the optional
// outputs).  `bar` is this CTA's key barrier, `phase` its current parity.
// Returns false when a bounded wait gave up.
template <int G, int NT>
__device__ bool score_chunk(const __nv_bfloat16* __restrict__ q, const float* __restrict__ pooled,
                            int nc_cap, int hq, int hkv, int i, int g, float scale, const ScoreGeometry& geo,
                            float* __restrict__ bscratch_row, float* __restrict__ comp_out,
                            float* __restrict__ bs_out_row, uint8_t* smem, uint64_t* bar, uint32_t phase,
                            uint32_t* status, uint64_t* trace_landed = nullptr) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float* keys = reinterpret_cast<float*>(smem);
  float* ssm = reinterpret_cast<float*>(smem + kScoreKeysBytes);
  const int nwin = geo.jhi - geo.jlo;
  if (geo.b1 <= geo.b0 || nwin <= 0) return true;
  if (tid == 0) {
    const uint32_t bytes = static_cast<uint32_t>(nwin) * kKeyBytes;
    mbar_arrive_expect_tx(bar, bytes);
    const float* src = pooled + ((static_cast<int64_t>(i) * hkv + g) * nc_cap + geo.jlo) * kHeadDim;
    bulk_copy_g2s(keys, src, bytes, bar);
  }
  // The group's queries, dims 4*lane .. 4*lane+3, widened to fp32.
  float4 qv[G];
  const __nv_bfloat16* qbase = q + (static_cast<int64_t>(i) * hq + g * G) * kHeadDim;
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qbase + hh * kHeadDim) + lane);
    qv[hh] = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                         __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u));
  }
  const bool ok = mbar_wait(bar, phase, status);
#ifdef NOSA_TRACE
  if (tid == 0 && trace_landed) *trace_landed = global_timer_ns();
  if (lane == 0 && trace_landed) atomicMax(reinterpret_cast<unsigned long long*>(trace_landed + 3),
                                           static_cast<unsigned long long>(global_timer_ns()));
#endif
  if (ok) {
    // Four windows per warp and iteration: four independent reduction chains
    // keep the shuffle pipeline busy.
    constexpr int kWin = 4;
    const int writer_mask = 32 / G - 1;
    for (int j0 = warp * kWin; j0 < nwin; j0 += (NT / 32) * kWin) {
      float v[kWin][G];
#pragma unroll
      for (int w = 0; w < kWin; ++w) {
        const int jj = min(j0 + w, nwin - 1);
        const float4 kv = reinterpret_cast<const float4*>(keys + jj * kHeadDim)[lane];
        if constexpr (G >= 2) {
          // Two heads per packed fp32x2 FMA; each head's sum keeps the order
          // x, y, z, w of the scalar form (same rounding).
#pragma unroll
          for (int hh = 0; hh < G; hh += 2) {
            float2 d = __fmul2_rn(make_float2(qv[hh].x, qv[hh + 1].x), make_float2(kv.x, kv.x));
            d = __ffma2_rn(make_float2(qv[hh].y, qv[hh + 1].y), make_float2(kv.y, kv.y), d);
            d = __ffma2_rn(make_float2(qv[hh].z, qv[hh + 1].z), make_float2(kv.z, kv.z), d);
            d = __ffma2_rn(make_float2(qv[hh].w, qv[hh + 1].w), make_float2(kv.w, kv.w), d);
            v[w][hh] = d.x;
            v[w][hh + 1] = d.y;
          }
        } else {
          float d = qv[0].x * kv.x;
          d = fmaf(qv[0].y, kv.y, d);
          d = fmaf(qv[0].z, kv.z, d);
          d = fmaf(qv[0].w, kv.w, d);
          v[w][0] = d;
        }
      }
#pragma unroll
      for (int w = 0; w < kWin; ++w) {
        int head;
        const float s = group_warp_sum<G>(v[w], lane, &head);
        if ((lane & writer_mask) == 0 && j0 + w < nwin) ssm[head * kScoreStride + j0 + w] = s * scale;
      }
    }
#ifdef NOSA_TRACE
    if (lane == 0 && trace_landed) atomicMax(reinterpret_cast<unsigned long long*>(trace_landed + 4),
                                             static_cast<unsigned long long>(global_timer_ns()));
#endif
  }
  __syncthreads();
  if (ok) {
    if (comp_out) {
      const int jo0 = kWindowsPerBlock * geo.b0, jo1 = geo.jhi;
      const int span = jo1 - jo0;
      for (int t = tid; t < G * span; t += NT) {
        const int hh = t / span, j = jo0 + t % span;
        comp_out[(static_cast<int64_t>(i) * hq + g * G + hh) * nc_cap + j] = ssm[hh * kScoreStride + (j - geo.jlo)];
      }
    }
    const int bend = min(geo.b1, geo.ncand);
    for (int t = tid; t < bend - geo.b0; t += NT) {
      const int b = geo.b0 + t;
      // J(b) = {4b-1, ..., 4b+3} clipped to [0, nc): a fixed 5-step loop with
      // predication keeps the shared-memory loads independent.
      const int jb = kWindowsPerBlock * b - 1;
      float S = 0.0f;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        float m = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWindowsPerBlock + 1; ++w) {
          const int j = jb + w;
          if (j >= 0 && j < geo.nc) m = fmaxf(m, ssm[hh * kScoreStride + (j - geo.jlo)]);
        }
        S += m;
      }
      bscratch_row[b] = S;
      if (bs_out_row) bs_out_row[b] = S;
    }
  }
  return ok;
}

// Geometry of scoring item `chunk` of a sequence of length L (L valid).
// `full` = scores wanted for every window (comp_out) rather than only the
// windows the selection reads.
__device__ inline ScoreGeometry score_geometry(int L, int nc_cap, int local_blocks, bool full, int chunk) {
  ScoreGeometry g;
  g.L = L;
  g.nc = n_windows(L);
  if (g.nc > nc_cap) g.nc = nc_cap;
  g.nb = static_cast<int>(n_blocks(L));
  g.ncand = static_cast<int>(n_candidates(L, local_blocks));
  const int nbw = full ? g.nb : g.ncand;
  g.nchunks = nbw > 0 ? (nbw + kChunkBlocks - 1) / kChunkBlocks : 1;
  g.b0 = chunk * kChunkBlocks;
  g.b1 = min(g.b0 + kChunkBlocks, nbw);
  g.jlo = max(0, kWindowsPerBlock * g.b0 - 1);
  const int64_t jh = static_cast<int64_t>(kWindowsPerBlock) * g.b1;
  g.jhi = static_cast<int>(g.nc < jh ? g.nc : jh);
  return g;
}

}  // namespace nosa
