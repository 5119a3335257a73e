// K3 -- exact attention over the selected blocks plus the local window,
// as a split-K flash-decode.
//
// "NOSA-1B 性能基准全解析" (wmrh.cn) §三.3: the TopK blocks chosen from the
// compressed scores get exact attention; §三.2: every query also attends to
// its fixed local window (1024 tokens = 16 blocks of 64).
//
// Work unit: one CTA per (sequence i, KV head g, split s).  The tile list of
// (i, g) is the local blocks [ncand, nb) followed by sel_idx[0..cnt); split s
// takes the balanced range [s*n/S, (s+1)*n/S) of it, resolved once into a
// shared-memory list.  Every tile is read once for all G query heads.
//
// Data movement: one producer thread issues, per 64-token tile, four 3-D
// tensor-TMA boxes {64 dims, 1 head, 64 tokens} (K low/high dims, V low/high
// dims; cp.async.bulk.tensor with the 128-byte swizzle) into a 3-stage
// shared-memory ring, completing on one mbarrier per stage (expect_tx), with
// empty barriers for reuse.  Rows past the end of the cache allocation are
// zero-filled by the TMA unit; rows past the sequence end are masked out of
// the softmax and their V rows zeroed in shared memory (then a proxy fence
// before the stage is reused), so stale or garbage rows cannot produce NaN.
//
// Math: four consumer warps each own 16 of the tile's 64 tokens.  With the
// group's queries as the A operand (16 rows, heads >= G zero) the warp runs
// S = Q K^T and O += P V on bf16 tensor cores (mma.sync m16n8k16, fp32
// accumulate); the S accumulator is re-packed in registers as the A operand
// of P V.  Each warp keeps its own online-softmax state (row max m, row sum
// l, O) in the exp2 domain.  At the end the four warps are merged in fixed
// order in shared memory; with more than one split the partial (O, m, l) goes
// to the workspace and the last CTA of (i, g) (atomic ticket, no spinning)
// merges the splits in split order, so results are bit-reproducible.
#include "nosa_common.cuh"
#include "nosa_kernels.h"

namespace nosa {

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 3;
constexpr int kHalfBytes = kBlock * 128;          // one 64-token x 64-dim box: 8 KB
constexpr int kStageBytes = 4 * kHalfBytes;        // K lo/hi, V lo/hi: 32 KB
constexpr int kRingBytes = kStages * kStageBytes;
constexpr uint32_t kTileTxBytes = kStageBytes;
constexpr int kCtasPerSm = 2;
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

// 3-D tiled TMA load of one {64 dims, 1 head, 64 tokens} box, completing on `bar`.
__device__ inline void tma_load_box(void* dst, const CUtensorMap* map, int dim0, int head, int row,
                                    uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(map), "r"(dim0), "r"(head), "r"(row), "r"(smem_addr(bar))
      : "memory");
}

// Address of 16-byte chunk `chunk` (0..7) of row `row` in a box written with
// the 128-byte swizzle: chunks are permuted by XOR with (row mod 8).
__device__ inline uint32_t swz(uint32_t box_base, int row, int chunk) {
  return box_base + row * 128 + ((chunk ^ (row & 7)) << 4);
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    sparse_decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ uint8_t smem_raw[];
  // 128-byte swizzled TMA boxes want 1024-byte aligned destinations.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ int blk_list[kMaxTilesPerSplit];
  __shared__ int sh_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int pair = blockIdx.y, split = blockIdx.x;
  const int i = pair / a.hkv, g = pair % a.hkv;
  const int G = a.group;
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kConsumerWarps);
    }
    fence_barrier_init();
  }
  if (warp == kConsumerWarps && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_k) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tm_v) : "memory");
  }
  grid_dependency_wait();
  allow_dependents();
  const int L = a.seq_len[i];
  const int64_t seq_base = a.seq_start[i];
  const int64_t out_row0 = static_cast<int64_t>(i) * a.hq + static_cast<int64_t>(g) * G;

  const bool bad_len = L < 1 || L > a.max_seq_len;
  const bool bad_rows = !bad_len && (seq_base < 0 || seq_base + L > a.cache_rows);
  if (bad_len || bad_rows) {
    if (split == 0) {
      if (tid == 0)
        set_status(a.status, bad_rows ? NOSA_DEV_CACHE_ROWS : (L < 1 ? NOSA_DEV_BAD_LENGTH : NOSA_DEV_MAX_LEN));
      for (int t = tid; t < G * kHeadDim; t += kThreads)
        a.out[out_row0 * kHeadDim + t] = __float2bfloat16_rn(0.0f);
      if (a.lse)
        for (int t = tid; t < G; t += kThreads) a.lse[out_row0 + t] = -INFINITY;
    }
    return;
  }
  const int nb = static_cast<int>(n_blocks(L));
  const int ncand = static_cast<int>(n_candidates(L, a.local_blocks));
  const int n_local = nb - ncand;
  int cnt = a.sel_cnt[pair];
  const int cnt_max = min(a.topk, ncand);
  if (cnt < 0 || cnt > cnt_max) {
    if (split == 0 && tid == 0) set_status(a.status, NOSA_DEV_BAD_COUNT);
    cnt = cnt < 0 ? 0 : cnt_max;
  }
  // Tiles of this pair: the local blocks first, then the selected ones;
  // split s takes the balanced range [s*n/S, (s+1)*n/S).
  const int ntiles = n_local + cnt;
  const int t_begin = static_cast<int>((static_cast<int64_t>(split) * ntiles) / a.nsplit);
  const int t_end = static_cast<int>((static_cast<int64_t>(split + 1) * ntiles) / a.nsplit);
  int my_n = t_end - t_begin;
  if (my_n > kMaxTilesPerSplit) {  // excluded by the host's split plan; reported, never overrun
    if (tid == 0) set_status(a.status, NOSA_DEV_BAD_COUNT);
    my_n = kMaxTilesPerSplit;
  }

  if (warp == kConsumerWarps) {
    const int32_t* sel = a.sel_idx + static_cast<int64_t>(pair) * a.topk;
    for (int n = lane; n < my_n; n += 32) {
      const int t = t_begin + n;
      int b;
      if (t < n_local) {
        b = ncand + t;
      } else {
        b = sel[t - n_local];
        if (b < 0 || b >= ncand) {
          set_status(a.status, NOSA_DEV_BAD_INDEX);
          b = -1;
        }
      }
      blk_list[n] = b;
    }
  }
  __syncthreads();

  float acc[16][4];
  float m_r[2] = {-INFINITY, -INFINITY};
  float l_r[2] = {0.0f, 0.0f};
#pragma unroll
  for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int issued = 0;
      for (int n = 0; n < my_n; ++n) {
        const int s = n % kStages;
        const uint32_t use = static_cast<uint32_t>(n / kStages);
        if (n >= kStages && !mbar_wait(&empty_bar[s], (use - 1) & 1u, a.status)) break;
        const int blk = blk_list[n];
        const int row = static_cast<int>(seq_base + (blk < 0 ? 0 : static_cast<int64_t>(blk) * kBlock));
        uint8_t* st = smem + s * kStageBytes;
        mbar_arrive_expect_tx(&full_bar[s], kTileTxBytes);
        tma_load_box(st, &tm_k, 0, g, row, &full_bar[s]);
        tma_load_box(st + kHalfBytes, &tm_k, 64, g, row, &full_bar[s]);
        tma_load_box(st + 2 * kHalfBytes, &tm_v, 0, g, row, &full_bar[s]);
        tma_load_box(st + 3 * kHalfBytes, &tm_v, 64, g, row, &full_bar[s]);
        issued = n + 1;
      }
      // Every copy this CTA issued has landed before shared memory is reused.
      for (int n = max(0, issued - kStages); n < issued; ++n)
        mbar_wait(&full_bar[n % kStages], static_cast<uint32_t>(n / kStages) & 1u, a.status);
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
      const int s = n % kStages;
      if (!mbar_wait(&full_bar[s], static_cast<uint32_t>(n / kStages) & 1u, a.status)) break;
      const int blk = blk_list[n];
      uint8_t* st = smem + s * kStageBytes;
      const uint32_t k_lo = smem_addr(st);
      const uint32_t v_lo = k_lo + 2 * kHalfBytes;
      const int64_t tok0 = static_cast<int64_t>(blk) * kBlock + wrow;
      // Rows of this warp past the sequence end (or a rejected tile) may hold
      // anything; zero their V rows so that P = 0 cannot meet a NaN.
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
      for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        const float m_new = fmaxf(m_r[r], mx[r]);
        m_use[r] = m_new == -INFINITY ? 0.0f : m_new;
        alpha[r] = exp2f(m_r[r] - m_use[r]);
        m_r[r] = m_new;
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
      if (lane == 0) mbar_arrive(&empty_bar[s]);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
      l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
    }
  }
  __syncthreads();  // ring drained: reuse it for the cross-warp merge

  float* mo = reinterpret_cast<float*>(smem);                    // [4][G][128]
  float* mm = mo + kConsumerWarps * G * kHeadDim;                // [4][G]
  float* ml = mm + kConsumerWarps * G;                           // [4][G]
  if (warp < kConsumerWarps) {
    const int grp = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int d = 0; d < 16; ++d) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = grp + (e >> 1) * 8;
        if (row < G) mo[(warp * G + row) * kHeadDim + d * 8 + 2 * tig + (e & 1)] = acc[d][e];
      }
    }
    if (tig == 0) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = grp + r * 8;
        if (row < G) {
          mm[warp * G + row] = m_r[r];
          ml[warp * G + row] = l_r[r];
        }
      }
    }
  }
  __syncthreads();

  const bool single = a.nsplit == 1;
  float* part = a.part + (static_cast<int64_t>(pair) * kMaxSplits + split) * part_stride(G);
  for (int t = tid; t < G * kHeadDim; t += kThreads) {
    const int row = t / kHeadDim, d = t % kHeadDim;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mm[w * G + row]);
    float lsum = 0.0f, o = 0.0f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = mm[w * G + row];
      if (mw == -INFINITY) continue;
      const float f = exp2f(mw - M);
      lsum += ml[w * G + row] * f;
      o += mo[(w * G + row) * kHeadDim + d] * f;
    }
    if (single) {
      a.out[(out_row0 + row) * kHeadDim + d] = __float2bfloat16_rn(lsum > 0.0f ? o / lsum : 0.0f);
      if (a.lse && d == 0) a.lse[out_row0 + row] = lsum > 0.0f ? (M + log2f(lsum)) * kLn2 : -INFINITY;
    } else {
      part[row * kHeadDim + d] = o;
      if (d == 0) {
        part[G * kHeadDim + row] = M;
        part[G * kHeadDim + G + row] = lsum;
      }
    }
  }
  if (single) return;

  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t t = atomicAdd(&a.tickets[pair], 1u);
    sh_last = (t == static_cast<uint32_t>(a.nsplit - 1));
  }
  __syncthreads();
  if (!sh_last) return;
  __threadfence();
  // Merge the splits in split order.  Their (m, l) go to shared memory first
  // (one parallel round trip), then every output float4 streams the splits'
  // partial O with independent loads.
  const float* pbase = a.part + static_cast<int64_t>(pair) * kMaxSplits * part_stride(G);
  const int stride = part_stride(G);
  float* sm_m = reinterpret_cast<float*>(smem);       // [nsplit][G], then weights in place
  float* sm_l = sm_m + kMaxSplits * kMaxGroup;        // [nsplit][G]
  float* sm_L = sm_l + kMaxSplits * kMaxGroup;        // [G]
  float* sm_M = sm_L + kMaxGroup;                     // [G]
  for (int t = tid; t < a.nsplit * G; t += kThreads) {
    const int s = t / G, row = t % G;
    sm_m[t] = __ldcg(pbase + s * stride + G * kHeadDim + row);
    sm_l[t] = __ldcg(pbase + s * stride + G * kHeadDim + G + row);
  }
  __syncthreads();
  for (int row = tid; row < G; row += kThreads) {
    float M = -INFINITY;
    for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, sm_m[s * G + row]);
    float lsum = 0.0f;
    for (int s = 0; s < a.nsplit; ++s) {
      const float ms = sm_m[s * G + row];
      const float w = ms == -INFINITY ? 0.0f : exp2f(ms - M);
      sm_m[s * G + row] = w;                          // becomes the split's weight
      lsum += sm_l[s * G + row] * w;
    }
    sm_L[row] = lsum;
    sm_M[row] = M;
  }
  __syncthreads();
  constexpr int kVec = kHeadDim / 4;
  for (int t = tid; t < G * kVec; t += kThreads) {
    const int row = t / kVec, d4 = t % kVec;
    const float4* src = reinterpret_cast<const float4*>(pbase + row * kHeadDim) + d4;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int s = 0; s < a.nsplit; ++s) {
      const float w = sm_m[s * G + row];
      const float4 x = __ldcg(src + s * (stride / 4));
      o.x = fmaf(w, x.x, o.x);
      o.y = fmaf(w, x.y, o.y);
      o.z = fmaf(w, x.z, o.z);
      o.w = fmaf(w, x.w, o.w);
    }
    const float lsum = sm_L[row];
    const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(a.out + (out_row0 + row) * kHeadDim + 4 * d4);
    dst[0] = __floats2bfloat162_rn(o.x * inv, o.y * inv);
    dst[1] = __floats2bfloat162_rn(o.z * inv, o.w * inv);
    if (a.lse && d4 == 0) a.lse[out_row0 + row] = lsum > 0.0f ? (sm_M[row] + log2f(lsum)) * kLn2 : -INFINITY;
  }
  if (tid == 0) a.tickets[pair] = 0u;
}

}  // namespace

void decode_split_plan(int pairs, int max_tiles, int num_sms, int* nsplit, int* tiles_per_split) {
  if (max_tiles < 1) max_tiles = 1;
  const int target = num_sms * kCtasPerSm;
  int ns = pairs > 0 ? target / pairs : 1;
  const int min_ns = (max_tiles + kMaxTilesPerSplit - 1) / kMaxTilesPerSplit;
  if (ns < min_ns) ns = min_ns;
  if (ns > max_tiles) ns = max_tiles;
  if (ns > kMaxSplits) ns = kMaxSplits;
  if (ns < 1) ns = 1;
  *nsplit = ns;
  *tiles_per_split = (max_tiles + ns - 1) / ns;
}

cudaError_t launch_sparse_decode(const DecodeArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                 cudaStream_t stream) {
  if (a.batch * a.hkv == 0) return cudaSuccess;
  const int smem = kRingBytes + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(sparse_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nsplit, a.batch * a.hkv);
  return launch_overlapped(sparse_decode_kernel, grid, dim3(kThreads), smem, stream, a, tm_k, tm_v);
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
  if (threadIdx.x == 0) mbar_wait(&bar, 0, status, max_iters);
}

cudaError_t launch_wait_selftest(uint32_t* status, uint32_t max_iters, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, max_iters);
  return cudaGetLastError();
}

}  // namespace nosa
