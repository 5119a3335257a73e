// K2 -- compressed scores, block scores and top-k block selection.
//
// "NOSA-1B 模型家族全景" (demingchina.com), 核心原理: compressed attention
// screens the history for the TopK blocks; "NOSA-1B 性能基准全解析" (wmrh.cn)
// §三.2 (block 64, local window of 16 blocks, TopK 64) and §三.3 (scores of
// the kernel-32 / stride-16 pooled keys, then TopK).
//
// Scoring pass: one CTA per (sequence, KV head, chunk of 16 blocks).  The
// chunk's pooled keys -- windows [4*b0-1, 4*b1) -- are one contiguous run of
// fp32 rows, fetched with a single bulk (TMA) copy into shared memory.  Each
// warp scores one window at a time: lane l holds dims 4l..4l+3 of the G
// queries of the group in registers, does 4*G FMAs against its float4 of the
// key, and a transposing butterfly leaves each lane with one head's full dot
// product after log2(G) halving exchanges plus 5 - log2(G) plain ones.  The
// block rule (max over the <= 5 overlapping windows, summed over the group's
// heads in ascending order) runs from shared memory.  The last CTA of each
// (sequence, KV head) -- found with an atomic ticket, no spinning -- selects
// the top-k with an exact 4 x 8-bit radix select on order-preserving keys and
// an index-ordered compaction, so ties go to the lowest block index and the
// output is ascending.  It then resets its ticket, leaving the workspace
// ready for the next call.
#include "nosa_common.cuh"
#include "nosa_kernels.h"

namespace nosa {

namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kChunkBlocks = 16;
constexpr int kChunkWindows = kChunkBlocks * kWindowsPerBlock + 1;  // 65
constexpr int kScoreStride = 68;                                    // floats per head row
constexpr int kKeyBytes = kHeadDim * 4;                             // 512

// Exchange half of `v` (n values) with lane ^ off; keep the half this lane's
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

// Sum of v[h] over the 32 lanes for the head h this lane ends up owning.
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
  uint32_t warp_eq[kSelWarps];
  uint32_t warp_take[kSelWarps];
  uint32_t prefix, need, run_eq, run_pos;
};

// Top-k of `ncand` scores (global, read with ld.global.cg when `coherent`),
// 256 threads.  Writes the pair's sel_idx row (ascending, -1 padded) and count.
__device__ void select_topk(const float* scores, bool coherent, int ncand, int topk,
                            int32_t* sel_row, int32_t* sel_cnt, uint32_t* ords, TopkShared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k_eff = ncand < topk ? ncand : topk;
  for (int b = tid; b < ncand; b += kSelThreads)
    ords[b] = order_key(coherent ? __ldcg(scores + b) : scores[b]);
  if (tid == 0) {
    sh.prefix = 0;
    sh.need = 0;
    sh.run_eq = 0;
    sh.run_pos = 0;
  }
  __syncthreads();
  uint32_t T = 0, need = 0;  // take all keys > 0, i.e. every candidate
  if (k_eff < ncand) {
    uint32_t prefix = 0;
    need = static_cast<uint32_t>(k_eff);
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
      for (int t = tid; t < 256; t += kSelThreads) sh.hist[t] = 0;
      __syncthreads();
      for (int b = tid; b < ncand; b += kSelThreads) {
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
  // Index-ordered compaction: every key > T, then the first `need` keys == T.
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < ncand; base += kSelThreads) {
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
      for (int w = 0; w < kSelWarps; ++w) {
        sh.run_eq += sh.warp_eq[w];
        sh.run_pos += sh.warp_take[w];
      }
    }
    __syncthreads();
  }
  for (int t = k_eff + tid; t < topk; t += kSelThreads) sel_row[t] = -1;
  if (tid == 0) *sel_cnt = k_eff;
}

// Marks a (sequence, KV head) as having no selection.
__device__ void write_empty_selection(const SelectArgs& a, int pair) {
  for (int t = threadIdx.x; t < a.topk; t += kSelThreads) a.sel_idx[static_cast<int64_t>(pair) * a.topk + t] = -1;
  if (threadIdx.x == 0) a.sel_cnt[pair] = 0;
}

template <int G>
__global__ void __launch_bounds__(kSelThreads) select_score_kernel(const SelectArgs a, int region_bytes) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ TopkShared sh;
  __shared__ int sh_last;
  float* keys = reinterpret_cast<float*>(smem);
  uint32_t* ords = reinterpret_cast<uint32_t*>(smem);
  float* ssm = reinterpret_cast<float*>(smem + region_bytes);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pair = blockIdx.y;
  const int i = pair / a.hkv, g = pair % a.hkv;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  grid_dependency_wait();
  allow_dependents();
  const int L = a.seq_len[i];
  if (L < 1 || L > a.max_seq_len) {
    if (blockIdx.x == 0) {
      if (tid == 0) set_status(a.status, L < 1 ? NOSA_DEV_BAD_LENGTH : NOSA_DEV_MAX_LEN);
      write_empty_selection(a, pair);
    }
    return;
  }
  int64_t nc = n_windows(L);
  if (nc > a.nc_cap) {
    if (blockIdx.x == 0 && tid == 0) set_status(a.status, NOSA_DEV_NC_CAP);
    nc = a.nc_cap;
  }
  const int nb = static_cast<int>(n_blocks(L));
  const int ncand = static_cast<int>(n_candidates(L, a.local_blocks));
  const int nbw = a.comp_out ? nb : ncand;
  const int nchunks = nbw > 0 ? (nbw + kChunkBlocks - 1) / kChunkBlocks : 1;
  if (static_cast<int>(blockIdx.x) >= nchunks) return;
  const int b0 = blockIdx.x * kChunkBlocks;
  const int b1 = min(b0 + kChunkBlocks, nbw);
  const int jlo = max(0, kWindowsPerBlock * b0 - 1);
  const int jhi = static_cast<int>(nc < static_cast<int64_t>(kWindowsPerBlock) * b1 ? nc : static_cast<int64_t>(kWindowsPerBlock) * b1);
  const int nwin = jhi - jlo;

  if (b1 > b0 && nwin > 0) {
    __syncthreads();  // barrier initialisation visible to every thread
    if (tid == 0) {
      const uint32_t bytes = static_cast<uint32_t>(nwin) * kKeyBytes;
      mbar_arrive_expect_tx(&bar, bytes);
      const float* src = a.pooled + ((static_cast<int64_t>(i) * a.hkv + g) * a.nc_cap + jlo) * kHeadDim;
      bulk_copy_g2s(keys, src, bytes, &bar);
    }
    // The group's queries, dims 4*lane .. 4*lane+3, widened to fp32.
    float4 qv[G];
    const __nv_bfloat16* qbase = a.q + (static_cast<int64_t>(i) * a.hq + g * G) * kHeadDim;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qbase + hh * kHeadDim) + lane);
      qv[hh] = make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                           __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u));
    }
    const bool ok = mbar_wait(&bar, 0, a.status);
    if (ok) {
      const int writer_mask = 32 / G - 1;
      for (int jj = warp; jj < nwin; jj += kSelWarps) {
        const float4 kv = reinterpret_cast<const float4*>(keys + jj * kHeadDim)[lane];
        float v[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          float d = qv[hh].x * kv.x;
          d = fmaf(qv[hh].y, kv.y, d);
          d = fmaf(qv[hh].z, kv.z, d);
          d = fmaf(qv[hh].w, kv.w, d);
          v[hh] = d;
        }
        int head;
        const float s = group_warp_sum<G>(v, lane, &head);
        if ((lane & writer_mask) == 0) ssm[head * kScoreStride + jj] = s * a.scale;
      }
    }
    __syncthreads();
    if (ok) {
      if (a.comp_out) {
        const int jo0 = kWindowsPerBlock * b0, jo1 = jhi;
        const int span = jo1 - jo0;
        for (int t = tid; t < G * span; t += kSelThreads) {
          const int hh = t / span, j = jo0 + t % span;
          a.comp_out[(static_cast<int64_t>(i) * a.hq + g * G + hh) * a.nc_cap + j] =
              ssm[hh * kScoreStride + (j - jlo)];
        }
      }
      const int bend = min(b1, ncand);
      for (int t = tid; t < bend - b0; t += kSelThreads) {
        const int b = b0 + t;
        const int j0 = max(0, kWindowsPerBlock * b - 1);
        const int j1 = static_cast<int>(nc < kWindowsPerBlock * b + 4 ? nc : kWindowsPerBlock * b + 4);
        float S = 0.0f;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          float m = -INFINITY;
          for (int j = j0; j < j1; ++j) m = fmaxf(m, ssm[hh * kScoreStride + (j - jlo)]);
          S += m;
        }
        a.bscratch[static_cast<int64_t>(pair) * a.nb_ws + b] = S;
        if (a.bs_out) a.bs_out[static_cast<int64_t>(pair) * a.nb_out + b] = S;
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t t = atomicAdd(&a.tickets[pair], 1u);
    sh_last = (t == static_cast<uint32_t>(nchunks - 1));
  }
  __syncthreads();
  if (!sh_last) return;
  __threadfence();
  select_topk(a.bscratch + static_cast<int64_t>(pair) * a.nb_ws, true, ncand, a.topk,
              a.sel_idx + static_cast<int64_t>(pair) * a.topk, a.sel_cnt + pair, ords, sh);
  if (tid == 0) a.tickets[pair] = 0u;
}

// Selection only, from caller-provided block scores: one CTA per pair.
__global__ void __launch_bounds__(kSelThreads) select_only_kernel(const SelectArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ TopkShared sh;
  const int pair = blockIdx.y;
  const int i = pair / a.hkv;
  grid_dependency_wait();
  allow_dependents();
  const int L = a.seq_len[i];
  if (L < 1 || L > a.max_seq_len) {
    if (threadIdx.x == 0) set_status(a.status, L < 1 ? NOSA_DEV_BAD_LENGTH : NOSA_DEV_MAX_LEN);
    write_empty_selection(a, pair);
    return;
  }
  const int ncand = static_cast<int>(n_candidates(L, a.local_blocks));
  select_topk(a.bs_in + static_cast<int64_t>(pair) * a.nb_in, false, ncand, a.topk,
              a.sel_idx + static_cast<int64_t>(pair) * a.topk, a.sel_cnt + pair,
              reinterpret_cast<uint32_t*>(smem), sh);
}

template <int G>
cudaError_t launch_scoring(const SelectArgs& a, cudaStream_t stream) {
  const int region = max(kChunkWindows * kKeyBytes, ((a.nb_ws * 4 + 127) / 128) * 128);
  const int smem = region + kMaxGroup * kScoreStride * 4;
  cudaError_t e = cudaFuncSetAttribute(select_score_kernel<G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int nb_max = static_cast<int>(n_blocks(a.max_seq_len));
  const int nbw = a.comp_out ? nb_max : static_cast<int>(n_candidates(a.max_seq_len, a.local_blocks));
  const int chunks = nbw > 0 ? (nbw + kChunkBlocks - 1) / kChunkBlocks : 1;
  dim3 grid(chunks, a.batch * a.hkv);
  return launch_overlapped(select_score_kernel<G>, grid, dim3(kSelThreads), smem, stream, a, region);
}

}  // namespace

cudaError_t launch_block_select(const SelectArgs& a, cudaStream_t stream) {
  if (a.batch * a.hkv == 0) return cudaSuccess;
  if (a.bs_in) {
    const int smem = ((a.nb_in * 4 + 127) / 128) * 128;
    cudaError_t e = cudaFuncSetAttribute(select_only_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_overlapped(select_only_kernel, dim3(1, a.batch * a.hkv), dim3(kSelThreads), smem, stream, a);
  }
  switch (a.group) {
    case 1: return launch_scoring<1>(a, stream);
    case 2: return launch_scoring<2>(a, stream);
    case 4: return launch_scoring<4>(a, stream);
    case 8: return launch_scoring<8>(a, stream);
    case 16: return launch_scoring<16>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nosa
