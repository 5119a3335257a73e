// Attention of the sparse prefill, query rows grouped so that K/V tiles are
// shared.
//
// What it computes is step 4 of the decode step for every prefill token
// ("NOSA 技术架构解析" (devpress.csdn.net) §1.3, NOSAS: sparse prefill; the
// token at position t attends, over its prefix L = t + 1, to its selected
// blocks and its local window):
//     out[e][h] = sum_{k in T_e} softmax_k(scale * q[e][h] . k_k) v_k
//     T_e = (U_{b in sel[e]} [64b, 64b+64) U [64 ncand(L_e), L_e)) n [0, L_e)
// The selections come from the step kernel (scoring + top-k per entry).
//
// One CTA per group of 64/G consecutive entries (query rows) of one
// sequence: its 4 consumer warps own 16 (token, head) rows each, so the CTA
// holds 64 rows.  The CTA walks the union of its tokens' selected and local
// blocks once, in ascending order; the producer warp stages each 64-token
// tile with the tensor copies of the decode kernel (four {64 dims, 1 head,
// 64 tokens} boxes, 128-byte swizzle) into a 3-stage ring, and every warp
// runs the whole tile against its rows on bf16 tensor cores
// (S = Q K^T: 16 x 64, O += P V: 16 x 128), masking rows whose token did not
// select the block and keys past a token's length (causal).  A warp skips a
// tile no row of it needs.  Entries of different sequences in one group are
// handled as consecutive segments.  Each warp's rows are complete at the end
// (no cross-warp merge).
#include <cstdlib>

#include "decode_device.cuh"
#include "nosa_common.cuh"
#include "nosa_kernels.h"
#include "umma.cuh"

namespace nosa {

namespace {

constexpr int kPfWarps = 4;                     // consumer warps
constexpr int kPfThreads = (kPfWarps + 1) * 32;  // + the producer warp
constexpr int kPfStages = 3;
constexpr int kPfRing = kPfStages * kStageBytes;
constexpr int kNoBlock = -0x7fffffff;  // no selection in this slot

// Named barrier 1 of the consumer warps; pf_all also returns whether `v`
// holds in all of them (so that a timed-out wait is given up together).
__device__ inline void pf_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kPfWarps * 32) : "memory"); }
__device__ inline bool pf_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kPfWarps * 32)
      : "memory");
  return r != 0;
}

// One warp's 16 rows against one staged tile of block `blk`: rows grp
// (accumulator elements 0, 1) and grp + 8 (elements 2, 3) of this lane attend
// to the tile when need0 / need1, to keys below L0 / L1.
__device__ inline void attend_rows(AttnState& s, const uint32_t (&qa)[8][4], const uint8_t* st, int blk, bool need0,
                                   bool need1, int L0, int L1, float scale_log2, int lane) {
  const int tig = lane & 3;
  const uint32_t k_lo = smem_addr(st);
  const uint32_t v_lo = k_lo + 2 * kHalfBytes;
  const int64_t kb0 = static_cast<int64_t>(blk) * kBlock;
  float sc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    float s0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int row = nt * 8 + (lane & 7);
#pragma unroll
    for (int kp = 0; kp < 4; ++kp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(swz(k_lo + (kp >> 1) * kHalfBytes, row, (kp & 1) * 4 + (lane >> 3)), b0, b1, b2, b3);
      mma_bf16_16816(s0, qa[2 * kp], b0, b1);
      mma_bf16_16816(s1, qa[2 * kp + 1], b2, b3);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) sc[nt][e] = s0[e] + s1[e];
  }
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int64_t key = kb0 + nt * 8 + 2 * tig + (e & 1);
      const bool valid = (e >> 1) ? (need1 && key < L1) : (need0 && key < L0);
      sc[nt][e] = valid ? sc[nt][e] * scale_log2 : -INFINITY;
      mx[e >> 1] = fmaxf(mx[e >> 1], sc[nt][e]);
    }
  }
  float alpha[2], m_use[2];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
    mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
    const float m_new = fmaxf(s.m[rr], mx[rr]);
    m_use[rr] = m_new == -INFINITY ? 0.0f : m_new;
    alpha[rr] = fast_exp2(s.m[rr] - m_use[rr]);
    s.m[rr] = m_new;
  }
  float rs[2] = {0.0f, 0.0f};
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      sc[nt][e] = fast_exp2(sc[nt][e] - m_use[e >> 1]);
      rs[e >> 1] += sc[nt][e];
    }
  }
  s.l[0] = s.l[0] * alpha[0] + rs[0];
  s.l[1] = s.l[1] * alpha[1] + rs[1];
#pragma unroll
  for (int d = 0; d < 16; ++d) {
    s.acc[d][0] *= alpha[0];
    s.acc[d][1] *= alpha[0];
    s.acc[d][2] *= alpha[1];
    s.acc[d][3] *= alpha[1];
  }
  // O += P V over the tile's four 16-key chunks.
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t pa[4] = {pack_bf16x2(sc[2 * c][0], sc[2 * c][1]), pack_bf16x2(sc[2 * c][2], sc[2 * c][3]),
                            pack_bf16x2(sc[2 * c + 1][0], sc[2 * c + 1][1]),
                            pack_bf16x2(sc[2 * c + 1][2], sc[2 * c + 1][3])};
    const int vrow = c * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_trans(swz(v_lo + (dp >> 2) * kHalfBytes, vrow, (dp & 3) * 2 + (lane >> 4)), b0, b1, b2, b3);
      mma_bf16_16816(s.acc[2 * dp], pa, b0, b1);
      mma_bf16_16816(s.acc[2 * dp + 1], pa, b2, b3);
    }
  }
}

template <int G>
__global__ void __launch_bounds__(kPfThreads, 2)
    prefill_attn_kernel(const PrefillAttnArgs a, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v) {
  constexpr int kTokens = kBlock / G;             // entries per CTA (64 rows)
  constexpr int kTokPerWarp = kTokens / kPfWarps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nbw = a.nb_words;
  uint32_t* sel_bm = reinterpret_cast<uint32_t*>(smem + kPfRing);  // [kTokens][nbw]: blocks each token selected
  uint32_t* uni_bm = sel_bm + kTokens * nbw;                       // [nbw]: union of the tiles to stage
  __shared__ uint64_t full_bar[kPfStages], empty_bar[kPfStages];
  __shared__ int tok_len[kTokens], tok_ncand[kTokens], tok_nb[kTokens];
  __shared__ unsigned char tok_in[kTokens];  // the token belongs to the current segment
  __shared__ int tok_seq[kTokens], tok_raw[kTokens], tok_raw_cnt[kTokens];  // loaded once per CTA
  __shared__ int tok_cnt[kTokens];  // selections used in the current segment
  __shared__ int seg_lo_blk, seg_hi_blk, seg_len;
  __shared__ int sh_bad[kPfStages];  // the stage holds a tile whose page was invalid (masked)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y;
  const int e_begin = blockIdx.x * kTokens;
  const int e_end = min(e_begin + kTokens, a.total_q);
  if (tid == 0) {
    for (int x = 0; x < kPfStages; ++x) {
      mbar_init(&full_bar[x], 1);
      mbar_init(&empty_bar[x], kPfWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  grid_dependency_wait();
  allow_dependents();
  if (e_begin >= e_end) return;
  // The group's entries: sequence, length and selection count (one parallel load).
  if (tid < kTokens) {
    const int e = e_begin + tid;
    const bool in = e < e_end;
    tok_seq[tid] = in ? a.entry_seq[e] : -1;
    tok_raw[tid] = in ? a.entry_len[e] : 0;
    tok_raw_cnt[tid] = in ? a.sel_cnt[static_cast<int64_t>(e) * a.hkv + g] : 0;
  }
  __syncthreads();

  uint32_t jobs = 0;  // tiles staged (producer) / consumed (consumers) so far, in every segment
  AttnState att;
  int e_lo = e_begin;
  while (e_lo < e_end) {
    // ------------------------------------------------------------ segment
    const int sq = tok_seq[e_lo - e_begin];
    int e_hi = e_lo + 1;
    while (e_hi < e_end && tok_seq[e_hi - e_begin] == sq) ++e_hi;
    // contiguous rows from seq_start, or 64-token pages through the table
    const int64_t base = a.page_table ? 0 : a.seq_start[sq];
    const int32_t* pages = a.page_table ? a.page_table + static_cast<int64_t>(sq) * a.max_pages : nullptr;
    const int num_pages = static_cast<int>(a.cache_rows / kBlock);
    for (int x = tid; x < (kTokens + 1) * nbw; x += kPfThreads) sel_bm[x] = 0u;
    if (tid < kTokens) {
      const int e = e_begin + tid;
      int L = e >= e_lo && e < e_hi ? tok_raw[tid] : 0;
      if (e >= e_lo && e < e_hi) {
        if (L < 1 || L > a.max_seq_len) {
          set_status(a.status, L < 1 ? NOSA_DEV_BAD_LENGTH : NOSA_DEV_MAX_LEN);
          L = 0;
        } else if (pages ? static_cast<int64_t>(L) > static_cast<int64_t>(a.max_pages) * kBlock
                         : base < 0 || base + L > a.cache_rows) {
          set_status(a.status, NOSA_DEV_CACHE_ROWS);
          L = 0;
        }
      }
      tok_len[tid] = L;
      tok_in[tid] = e >= e_lo && e < e_hi;
      tok_nb[tid] = static_cast<int>(n_blocks(L));
      tok_ncand[tid] = static_cast<int>(n_candidates(L, a.local_blocks));
      int cnt = tok_raw_cnt[tid];
      if (L > 0 && (cnt < 0 || cnt > a.topk)) {
        set_status(a.status, NOSA_DEV_BAD_COUNT);
        cnt = cnt < 0 ? 0 : a.topk;
      }
      tok_cnt[tid] = L > 0 ? cnt : 0;
    }
    __syncthreads();
    if (tid == 0) {
      int lo = 1 << 30, hi = 0, len = 0;
      for (int t = 0; t < kTokens; ++t)
        if (tok_len[t] > 0) {
          lo = min(lo, tok_ncand[t]);
          hi = max(hi, tok_nb[t]);
          len = max(len, tok_len[t]);
        }
      seg_lo_blk = lo;
      seg_hi_blk = hi;
      seg_len = len;
    }
    // selected blocks of every token (sel_idx written by the selection
    // launch), eight independent loads in flight per thread
    {
      constexpr int kU = 8;
      const int n = kTokens * a.topk;
      for (int x0 = tid; x0 < n; x0 += kPfThreads * kU) {
        int v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const int x = x0 + u * kPfThreads;
          const int t = x / a.topk, j = x - (x / a.topk) * a.topk;
          v[u] = x < n && j < tok_cnt[t]
                     ? a.sel_idx[(static_cast<int64_t>(e_begin + t) * a.hkv + g) * a.topk + j]
                     : kNoBlock;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          if (v[u] == kNoBlock) continue;
          const int t = (x0 + u * kPfThreads) / a.topk;
          const int b = v[u];
          if (b < 0 || b >= tok_ncand[t]) {
            set_status(a.status, NOSA_DEV_BAD_INDEX);
            continue;
          }
          atomicOr(&sel_bm[t * nbw + (b >> 5)], 1u << (b & 31));
          atomicOr(&uni_bm[b >> 5], 1u << (b & 31));
        }
      }
    }
    __syncthreads();
    // the local windows: blocks [min ncand, max nb) of the segment's tokens
    for (int b = seg_lo_blk + tid; b < seg_hi_blk; b += kPfThreads) atomicOr(&uni_bm[b >> 5], 1u << (b & 31));
    __syncthreads();
    const int hi_blk = seg_hi_blk;

    if (warp == kPfWarps) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        const uint64_t policy = l2_evict_first_policy();
        bool ok = true;
        for (int w = 0; w < nbw && ok; ++w) {
          uint32_t bits = uni_bm[w];
          while (bits && ok) {
            const int b = w * 32 + __ffs(bits) - 1;
            bits &= bits - 1u;
            if (b >= hi_blk) continue;
            const int x = static_cast<int>(jobs % kPfStages);
            if (jobs >= kPfStages && !mbar_wait(&empty_bar[x], ((jobs / kPfStages) - 1) & 1u, a.status)) {
              ok = false;
              break;
            }
            uint8_t* st = smem + x * kStageBytes;
            int row = static_cast<int>(base + static_cast<int64_t>(b) * kBlock);
            if (pages) {
              const int32_t pg = pages[b];
              if (pg < 0 || pg >= num_pages) {
                // an invalid page: stage the first page and mask the whole tile
                set_status(a.status, NOSA_DEV_BAD_INDEX);
                sh_bad[x] = 1;
                row = 0;
              } else {
                sh_bad[x] = 0;
                row = pg * kBlock;
              }
            }
            mbar_arrive_expect_tx(&full_bar[x], kTileTxBytes);
            tma_load_box(st, &tm_k, 0, g, row, &full_bar[x], policy);
            tma_load_box(st + kHalfBytes, &tm_k, 64, g, row, &full_bar[x], policy);
            tma_load_box(st + 2 * kHalfBytes, &tm_v, 0, g, row, &full_bar[x], policy);
            tma_load_box(st + 3 * kHalfBytes, &tm_v, 64, g, row, &full_bar[x], policy);
            ++jobs;
          }
        }
        // every copy issued has landed before the segment's bitmaps are reused
        const uint32_t first = jobs > kPfStages ? jobs - kPfStages : 0u;
        for (uint32_t n = first; n < jobs; ++n) mbar_wait(&full_bar[n % kPfStages], (n / kPfStages) & 1u, a.status);
      }
      jobs = __shfl_sync(0xffffffffu, jobs, 0);
    } else {
      // ---------------------------------------------------------- consumers
      const int grp = lane >> 2, tig = lane & 3;
      const int t0 = warp * kTokPerWarp + grp / G, t1 = warp * kTokPerWarp + (grp + 8) / G;
      const int L0 = tok_len[t0], L1 = tok_len[t1];
      const bool live = __any_sync(0xffffffffu, L0 > 0 || L1 > 0);
      uint32_t qa[8][4];
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int rowr = grp + (r & 1) * 8;
          const int t = warp * kTokPerWarp + rowr / G;
          const int col = ks * 16 + 2 * tig + (r >> 1) * 8;
          const __nv_bfloat16* qrow =
              a.q + (static_cast<int64_t>(e_begin + t) * a.hq + static_cast<int64_t>(g) * G + rowr % G) * kHeadDim;
          qa[ks][r] = tok_len[t] > 0 ? __ldg(reinterpret_cast<const uint32_t*>(qrow + col)) : 0u;
        }
      }
      attn_init(att);
      bool ok = true;
      for (int w = 0; w < nbw; ++w) {
        uint32_t bits = uni_bm[w];
        while (bits) {
          const int b = w * 32 + __ffs(bits) - 1;
          bits &= bits - 1u;
          if (b >= hi_blk) continue;
          const int x = static_cast<int>(jobs % kPfStages);
          ok = ok && pf_all(mbar_wait(&full_bar[x], (jobs / kPfStages) & 1u, a.status));
          uint8_t* st = smem + x * kStageBytes;
          if (ok) {
            // V rows past every token's length hold stale rows: zero them
            // (each warp its own 16 rows) before any warp reads the tile.
            const int64_t kb0 = static_cast<int64_t>(b) * kBlock;
            const bool partial = kb0 + kBlock > seg_len;
            if (partial) {
              for (int idx = lane; idx < 16 * 16; idx += 32) {
                const int rr = idx >> 4, c16 = idx & 15;
                const int row = warp * 16 + rr;
                if (kb0 + row >= seg_len)
                  *reinterpret_cast<uint4*>(st + 2 * kHalfBytes + (c16 >> 3) * kHalfBytes + row * 128 +
                                            (((c16 & 7) ^ (row & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
              }
              pf_sync();
            }
            const bool bad = a.page_table != nullptr && sh_bad[x] != 0;
            const bool need0 = !bad && L0 > 0 && b < tok_nb[t0] &&
                               (b >= tok_ncand[t0] || ((sel_bm[t0 * nbw + (b >> 5)] >> (b & 31)) & 1u));
            const bool need1 = !bad && L1 > 0 && b < tok_nb[t1] &&
                               (b >= tok_ncand[t1] || ((sel_bm[t1 * nbw + (b >> 5)] >> (b & 31)) & 1u));
            if (live && __any_sync(0xffffffffu, need0 || need1))
              attend_rows(att, qa, st, b, need0, need1, L0, L1, a.scale_log2, lane);
            if (partial) {
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              pf_sync();  // every warp is done with the tile before the producer may refill it
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty_bar[x]);
          ++jobs;
        }
      }
      attn_finish(att);
      // the rows of this warp's tokens in the segment
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int rowr = grp + h2 * 8;
        const int t = warp * kTokPerWarp + rowr / G;
        if (!tok_in[t]) continue;  // rows of a token with a bad length are written as zeros
        const int e = e_begin + t;
        const int64_t orow = static_cast<int64_t>(e) * a.hq + static_cast<int64_t>(g) * G + rowr % G;
        const float lsum = att.l[h2];
        const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
#pragma unroll
        for (int d = 0; d < 16; ++d) {
          *reinterpret_cast<__nv_bfloat162*>(a.out + orow * kHeadDim + d * 8 + 2 * tig) =
              __floats2bfloat162_rn(att.acc[d][2 * h2] * inv, att.acc[d][2 * h2 + 1] * inv);
        }
        if (a.lse && tig == 0) a.lse[orow] = lsum > 0.0f ? (att.m[h2] + log2f(lsum)) * kLn2 : -INFINITY;
      }
    }
    __syncthreads();  // the segment's tiles are consumed; bitmaps and token info may be rewritten
    e_lo = e_hi;
  }
}

// ---------------------------------------------------------------------------
// The same attention on the fifth-generation tensor cores (tcgen05): one CTA
// per group of 128 / G consecutive entries, i.e. 128 (token, head) rows.
//   * warp 8 (producer) stages each tile of the union walk with the tensor
//     copies into a 3-stage ring, as above;
//   * warp 9 (MMA) issues, from one thread, S = Q K^T (M 128, N 64, K 128;
//     Q and K K-major in shared memory) into TMEM, and once the compute warps
//     have written P, O_tile = P V (M 128, N 128, K 64; P K-major, V the
//     MN-major B) into TMEM; its commits signal the compute warps and free
//     the stage;
//   * warps 0-7 (compute): thread (warp w, lane l) owns row 32 (w mod 4) + l
//     (the TMEM lane quarter of its warp) and half w / 4 of the head
//     dimension: it reads the row's 64 scores, runs the online softmax of the
//     row (both halves alike), writes its half of P (bf16) in the swizzled
//     layout, and adds the tile's O to its 64 accumulators in registers.
// Masks, causal limits, segments and invalid pages are handled as in the
// mma.sync kernel above.
constexpr int kUmRows = 128;
constexpr int kUmComputeWarps = 8;
constexpr int kUmProducerWarp = 8;
constexpr int kUmMmaWarp = 9;
constexpr int kUmThreads = 10 * 32;
constexpr int kUmComputeThreads = kUmComputeWarps * 32;
constexpr int kUmQBytes = 2 * kUmRows * 128;  // Q: two K-major regions (dims 0-63, 64-127)
constexpr int kUmPBytes = kUmRows * 128;      // P: 128 rows x 64 keys
constexpr uint32_t kUmIdescS = umma_idesc_bf16(128, 64, false);
constexpr uint32_t kUmIdescO = umma_idesc_bf16(128, 128, true);

template <int G>
__global__ void __launch_bounds__(kUmThreads, 1)
    prefill_attn_umma_kernel(const PrefillAttnArgs a, const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v) {
  constexpr int kTokens = kUmRows / G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = smem + kPfRing;
  uint8_t* sp = sq + kUmQBytes;
  const int nbw = a.nb_words;
  uint32_t* sel_bm = reinterpret_cast<uint32_t*>(sp + kUmPBytes);  // [kTokens][nbw]
  uint32_t* uni_bm = sel_bm + kTokens * nbw;                        // [nbw]
  __shared__ uint64_t full_bar[kPfStages], empty_bar[kPfStages], s_full, p_full, o_full;
  __shared__ uint32_t tmem_base;
  __shared__ int tok_len[kTokens], tok_ncand[kTokens], tok_nb[kTokens], tok_cnt[kTokens];
  __shared__ int tok_seq[kTokens], tok_raw[kTokens], tok_raw_cnt[kTokens];
  __shared__ unsigned char tok_in[kTokens];
  __shared__ int seg_lo_blk, seg_hi_blk, seg_len;
  __shared__ int sh_bad[kPfStages];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.y;
  const int e_begin = blockIdx.x * kTokens;
  const int e_end = min(e_begin + kTokens, a.total_q);
  if (tid == 0) {
    for (int x = 0; x < kPfStages; ++x) {
      mbar_init(&full_bar[x], 1);
      mbar_init(&empty_bar[x], 1);
    }
    mbar_init(&s_full, 1);
    mbar_init(&p_full, kUmComputeThreads);
    mbar_init(&o_full, 1);
    fence_barrier_init();
  }
  if (warp == kUmMmaWarp) tmem_alloc<256>(&tmem_base);
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t t_s = tmem_base, t_o = tmem_base + 64;
  grid_dependency_wait();
  allow_dependents();
  if (e_begin < e_end) {
    if (tid < kTokens) {
      const int e = e_begin + tid;
      const bool in = e < e_end;
      tok_seq[tid] = in ? a.entry_seq[e] : -1;
      tok_raw[tid] = in ? a.entry_len[e] : 0;
      tok_raw_cnt[tid] = in ? a.sel_cnt[static_cast<int64_t>(e) * a.hkv + g] : 0;
    }
    __syncthreads();
    uint32_t jobs = 0;
    int e_lo = e_begin;
    while (e_lo < e_end) {
      // ---------------------------------------------------------- segment setup
      const int sq_id = tok_seq[e_lo - e_begin];
      int e_hi = e_lo + 1;
      while (e_hi < e_end && tok_seq[e_hi - e_begin] == sq_id) ++e_hi;
      const int64_t base = a.page_table ? 0 : a.seq_start[sq_id];
      const int32_t* pages = a.page_table ? a.page_table + static_cast<int64_t>(sq_id) * a.max_pages : nullptr;
      const int num_pages = static_cast<int>(a.cache_rows / kBlock);
      for (int x = tid; x < (kTokens + 1) * nbw; x += kUmThreads) sel_bm[x] = 0u;
      if (tid < kTokens) {
        const int e = e_begin + tid;
        const bool in = e >= e_lo && e < e_hi;
        int L = in ? tok_raw[tid] : 0;
        if (in) {
          if (L < 1 || L > a.max_seq_len) {
            set_status(a.status, L < 1 ? NOSA_DEV_BAD_LENGTH : NOSA_DEV_MAX_LEN);
            L = 0;
          } else if (pages ? static_cast<int64_t>(L) > static_cast<int64_t>(a.max_pages) * kBlock
                           : base < 0 || base + L > a.cache_rows) {
            set_status(a.status, NOSA_DEV_CACHE_ROWS);
            L = 0;
          }
        }
        tok_len[tid] = L;
        tok_in[tid] = in;
        tok_nb[tid] = static_cast<int>(n_blocks(L));
        tok_ncand[tid] = static_cast<int>(n_candidates(L, a.local_blocks));
        int cnt = tok_raw_cnt[tid];
        if (L > 0 && (cnt < 0 || cnt > a.topk)) {
          set_status(a.status, NOSA_DEV_BAD_COUNT);
          cnt = cnt < 0 ? 0 : a.topk;
        }
        tok_cnt[tid] = L > 0 ? cnt : 0;
      }
      __syncthreads();
      if (tid == 0) {
        int lo = 1 << 30, hi = 0, len = 0;
        for (int t = 0; t < kTokens; ++t)
          if (tok_len[t] > 0) {
            lo = min(lo, tok_ncand[t]);
            hi = max(hi, tok_nb[t]);
            len = max(len, tok_len[t]);
          }
        seg_lo_blk = lo;
        seg_hi_blk = hi;
        seg_len = len;
      }
      {
        constexpr int kU = 8;
        const int n = kTokens * a.topk;
        for (int x0 = tid; x0 < n; x0 += kUmThreads * kU) {
          int v[kU];
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            const int x = x0 + u * kUmThreads;
            const int t = x / a.topk, j = x - (x / a.topk) * a.topk;
            v[u] = x < n && j < tok_cnt[t]
                       ? a.sel_idx[(static_cast<int64_t>(e_begin + t) * a.hkv + g) * a.topk + j]
                       : kNoBlock;
          }
#pragma unroll
          for (int u = 0; u < kU; ++u) {
            if (v[u] == kNoBlock) continue;
            const int t = (x0 + u * kUmThreads) / a.topk;
            const int b = v[u];
            if (b < 0 || b >= tok_ncand[t]) {
              set_status(a.status, NOSA_DEV_BAD_INDEX);
              continue;
            }
            atomicOr(&sel_bm[t * nbw + (b >> 5)], 1u << (b & 31));
            atomicOr(&uni_bm[b >> 5], 1u << (b & 31));
          }
        }
      }
      // Q of the segment's rows (row t * G + h), K-major with the 128-byte
      // swizzle; rows of other tokens are zero.
      for (int x = tid; x < kUmRows * 16; x += kUmThreads) {
        const int r = x >> 4, c = x & 15;
        const int t = r / G;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (tok_len[t] > 0)
          val = __ldg(reinterpret_cast<const uint4*>(
                          a.q + (static_cast<int64_t>(e_begin + t) * a.hq + static_cast<int64_t>(g) * G + r % G) *
                                    kHeadDim) +
                      c);
        *reinterpret_cast<uint4*>(sq + (c >> 3) * (kUmRows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = val;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      for (int b = seg_lo_blk + tid; b < seg_hi_blk; b += kUmThreads) atomicOr(&uni_bm[b >> 5], 1u << (b & 31));
      __syncthreads();
      const int hi_blk = seg_hi_blk;

      if (warp == kUmProducerWarp) {
        // -------------------------------------------------------- producer
        if (lane == 0) {
          const uint64_t policy = l2_evict_first_policy();
          uint32_t n = jobs;
          bool ok = true;
          for (int w = 0; w < nbw && ok; ++w) {
            uint32_t bits = uni_bm[w];
            while (bits && ok) {
              const int b = w * 32 + __ffs(bits) - 1;
              bits &= bits - 1u;
              if (b >= hi_blk) continue;
              const int x = static_cast<int>(n % kPfStages);
              if (n >= kPfStages && !mbar_wait(&empty_bar[x], ((n / kPfStages) - 1) & 1u, a.status)) {
                ok = false;
                break;
              }
              uint8_t* st = smem + x * kStageBytes;
              int row = static_cast<int>(base + static_cast<int64_t>(b) * kBlock);
              sh_bad[x] = 0;
              if (pages) {
                const int32_t pg = pages[b];
                if (pg < 0 || pg >= num_pages) {
                  set_status(a.status, NOSA_DEV_BAD_INDEX);
                  sh_bad[x] = 1;
                  row = 0;
                } else {
                  row = pg * kBlock;
                }
              }
              mbar_arrive_expect_tx(&full_bar[x], kTileTxBytes);
              tma_load_box(st, &tm_k, 0, g, row, &full_bar[x], policy);
              tma_load_box(st + kHalfBytes, &tm_k, 64, g, row, &full_bar[x], policy);
              tma_load_box(st + 2 * kHalfBytes, &tm_v, 0, g, row, &full_bar[x], policy);
              tma_load_box(st + 3 * kHalfBytes, &tm_v, 64, g, row, &full_bar[x], policy);
              ++n;
            }
          }
          jobs = n;
        }
        jobs = __shfl_sync(0xffffffffu, jobs, 0);
      } else if (warp == kUmMmaWarp) {
        // -------------------------------------------------------- MMA issue
        if (lane == 0) {
          uint32_t n = jobs;
          bool ok = true;
          for (int w = 0; w < nbw; ++w) {
            uint32_t bits = uni_bm[w];
            while (bits) {
              const int b = w * 32 + __ffs(bits) - 1;
              bits &= bits - 1u;
              if (b >= hi_blk) continue;
              const int x = static_cast<int>(n % kPfStages);
              ok = ok && mbar_wait(&full_bar[x], (n / kPfStages) & 1u, a.status);
              // S of the previous tile has been read (its P is written)
              if (n > 0) ok = ok && mbar_wait(&p_full, (n - 1) & 1u, a.status);
              tmem_fence_after();
              if (ok) {
                const uint8_t* st = smem + x * kStageBytes;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  const uint64_t ad = umma_desc(smem_addr(sq + (k >> 2) * (kUmRows * 128) + (k & 3) * 32), 16, 1024);
                  const uint64_t bd = umma_desc(smem_addr(st + (k >> 2) * kHalfBytes + (k & 3) * 32), 16, 1024);
                  umma_bf16(t_s, ad, bd, kUmIdescS, k > 0);
                }
              }
              umma_commit(&s_full);
              ok = ok && mbar_wait(&p_full, n & 1u, a.status);
              tmem_fence_after();
              if (ok) {
                const uint8_t* st = smem + x * kStageBytes;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const uint64_t ad = umma_desc(smem_addr(sp + k * 32), 16, 1024);
                  const uint64_t bd = umma_desc(smem_addr(st + 2 * kHalfBytes + k * 2048), kHalfBytes, 1024);
                  umma_bf16(t_o, ad, bd, kUmIdescO, k > 0);
                }
              }
              umma_commit(&o_full);
              umma_commit(&empty_bar[x]);
              ++n;
            }
          }
          jobs = n;
        }
        jobs = __shfl_sync(0xffffffffu, jobs, 0);
      } else {
        // -------------------------------------------------------- compute
        const int quarter = warp & 3, half = warp >> 2;
        const int r = 32 * quarter + lane;
        const int t = r / G;
        const int L = tok_len[t];
        const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
        float o[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) o[j] = 0.0f;
        float m = -INFINITY, l = 0.0f;
        uint32_t n = jobs;
        bool ok = true;
        for (int w = 0; w < nbw; ++w) {
          uint32_t bits = uni_bm[w];
          while (bits) {
            const int b = w * 32 + __ffs(bits) - 1;
            bits &= bits - 1u;
            if (b >= hi_blk) continue;
            const int x = static_cast<int>(n % kPfStages);
            // the stage's page check (sh_bad) is published with its copies
            ok = ok && mbar_wait(&full_bar[x], (n / kPfStages) & 1u, a.status);
            ok = ok && mbar_wait(&s_full, n & 1u, a.status);
            tmem_fence_after();
            const bool bad = a.page_table != nullptr && sh_bad[x] != 0;
            const bool need = ok && !bad && L > 0 && b < tok_nb[t] &&
                              (b >= tok_ncand[t] || ((sel_bm[t * nbw + (b >> 5)] >> (b & 31)) & 1u));
            const int64_t kb0 = static_cast<int64_t>(b) * kBlock;
            float sc[64];
            if (ok) {
              float tmp[32];
              tmem_ld32(t_s + lane_off, tmp);
#pragma unroll
              for (int j = 0; j < 32; ++j) sc[j] = tmp[j];
              tmem_ld32(t_s + lane_off + 32, tmp);
#pragma unroll
              for (int j = 0; j < 32; ++j) sc[32 + j] = tmp[j];
            }
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              const bool valid = need && kb0 + j < L;
              sc[j] = valid ? sc[j] * a.scale_log2 : -INFINITY;
              mx = fmaxf(mx, sc[j]);
            }
            const float m_new = fmaxf(m, mx);
            const float m_use = m_new == -INFINITY ? 0.0f : m_new;
            const float alpha = fast_exp2(m - m_use);
            m = m_new;
            float rs = 0.0f;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              sc[j] = fast_exp2(sc[j] - m_use);
              rs += sc[j];
            }
            l = l * alpha + rs;
            // this thread's half of P: keys 32 half .. 32 half + 31 (chunks 4 half .. 4 half + 3);
            // both halves spelled out so that every index into sc is a constant
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (hh != half) continue;
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const int k0 = 32 * hh + 8 * c;
                uint4 pk;
                pk.x = pack_bf16x2(sc[k0 + 0], sc[k0 + 1]);
                pk.y = pack_bf16x2(sc[k0 + 2], sc[k0 + 3]);
                pk.z = pack_bf16x2(sc[k0 + 4], sc[k0 + 5]);
                pk.w = pack_bf16x2(sc[k0 + 6], sc[k0 + 7]);
                const int chunk = 4 * hh + c;
                *reinterpret_cast<uint4*>(sp + r * 128 + ((chunk ^ (r & 7)) << 4)) = pk;
              }
            }
            // V rows past every token's length hold stale rows: zero them
            if (ok && kb0 + kBlock > seg_len) {
              uint8_t* st = smem + x * kStageBytes;
              for (int idx = tid; idx < kBlock * 16; idx += kUmComputeThreads) {
                const int vr = idx >> 4, c16 = idx & 15;
                if (kb0 + vr >= seg_len)
                  *reinterpret_cast<uint4*>(st + 2 * kHalfBytes + (c16 >> 3) * kHalfBytes + vr * 128 +
                                            (((c16 & 7) ^ (vr & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
              }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tmem_fence_before();
            mbar_arrive(&p_full);
            ok = ok && mbar_wait(&o_full, n & 1u, a.status);
            tmem_fence_after();
            if (ok) {
              float tmp[32];
              tmem_ld32(t_o + lane_off + 64 * half, tmp);
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = o[j] * alpha + tmp[j];
              tmem_ld32(t_o + lane_off + 64 * half + 32, tmp);
#pragma unroll
              for (int j = 0; j < 32; ++j) o[32 + j] = o[32 + j] * alpha + tmp[j];
            }
            tmem_fence_before();
            ++n;
          }
        }
        jobs = n;
        // the row's half of the output
        if (tok_in[t]) {
          const int e = e_begin + t;
          const int64_t orow = static_cast<int64_t>(e) * a.hq + static_cast<int64_t>(g) * G + r % G;
          const float inv = l > 0.0f ? 1.0f / l : 0.0f;
          uint4* dst = reinterpret_cast<uint4*>(a.out + orow * kHeadDim + 64 * half);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 pk;
            pk.x = pack_bf16x2(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
            pk.y = pack_bf16x2(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
            pk.z = pack_bf16x2(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
            pk.w = pack_bf16x2(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
            dst[c] = pk;
          }
          if (a.lse && half == 0) a.lse[orow] = l > 0.0f ? (m + log2f(l)) * kLn2 : -INFINITY;
        }
      }
      __syncthreads();  // the segment's tiles are consumed; bitmaps, Q and token info may be rewritten
      e_lo = e_hi;
    }
  }
  tmem_fence_before();
  __syncthreads();
  if (warp == kUmMmaWarp) {
    tmem_fence_after();
    tmem_dealloc<256>(t_s);
  }
}

}  // namespace

// The mma.sync kernel (64 rows per CTA, warps skip tiles their rows do not
// need) by default; NOSA_PREFILL_UMMA=1 selects the tcgen05 kernel (128 rows
// per CTA).  With independent queries the union of a group's selections
// covers most candidates, and a CTA of 128 rows computes every row against
// every tile of that union, so the tcgen05 kernel measured slower here (16K
// prefill 8.4 ms against 7.2 ms); with correlated neighbouring queries, as in
// a trained model, the union shrinks and the tcgen05 tile is the faster one.
cudaError_t launch_prefill_attn(const PrefillAttnArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                cudaStream_t stream) {
  static const bool use_sync = [] {
    const char* v = getenv("NOSA_PREFILL_UMMA");
    return !(v != nullptr && v[0] == '1');
  }();
  const int G = a.hq / a.hkv;
  const int rows = use_sync ? kBlock : kUmRows;
  const int tokens = rows / G;
  const int groups = (a.total_q + tokens - 1) / tokens;
  if (groups == 0) return cudaSuccess;
  const size_t smem = use_sync ? 1024 + kPfRing + static_cast<size_t>(tokens + 1) * a.nb_words * 4
                               : 1024 + kPfRing + kUmQBytes + kUmPBytes +
                                     static_cast<size_t>(tokens + 1) * a.nb_words * 4;
  auto go = [&](auto kernel, int threads) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return launch_overlapped(kernel, dim3(groups, a.hkv), dim3(threads), smem, stream, a, tm_k, tm_v);
  };
  if (use_sync) {
    switch (G) {
      case 1: return go(prefill_attn_kernel<1>, kPfThreads);
      case 2: return go(prefill_attn_kernel<2>, kPfThreads);
      case 4: return go(prefill_attn_kernel<4>, kPfThreads);
      case 8: return go(prefill_attn_kernel<8>, kPfThreads);
      case 16: return go(prefill_attn_kernel<16>, kPfThreads);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (G) {
    case 1: return go(prefill_attn_umma_kernel<1>, kUmThreads);
    case 2: return go(prefill_attn_umma_kernel<2>, kUmThreads);
    case 4: return go(prefill_attn_umma_kernel<4>, kUmThreads);
    case 8: return go(prefill_attn_umma_kernel<8>, kUmThreads);
    case 16: return go(prefill_attn_umma_kernel<16>, kUmThreads);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nosa
