// Exact attention over the selected blocks plus the local window: the
// per-tile device routines of the decode-step kernel.
//
// "NOSA-1B 性能基准全解析" (wmrh.cn) §三.3: the TopK blocks chosen from the
// compressed scores get exact attention; §三.2: every query also attends to
// its fixed local window (1024 tokens = 16 blocks of 64).
//
//   T   = (U_{b in sel} [64b, 64b+64) U [64*ncand, L)) n [0, L)
//   out = sum_{t in T} softmax_t(scale * q . k_t) v_t
//
// A 64-token tile arrives in one 32 KB ring stage as four 3-D tensor-TMA
// boxes {64 dims, 1 head, 64 tokens} (K low/high dims, V low/high dims;
// cp.async.bulk.tensor with the 128-byte swizzle).  Rows past the cache
// allocation are zero-filled by the TMA unit; rows past the sequence end are
// masked out of the softmax and their V rows zeroed in shared memory (then a
// proxy fence before the stage is reused), so stale or garbage rows cannot
// produce NaN.
//
// Math: four consumer warps each own 16 of the tile's 64 tokens.  With the
// group's queries as the A operand (16 rows, heads >= G zero) a warp runs
// S = Q K^T and O += P V on bf16 tensor cores (mma.sync m16n8k16, fp32
// accumulate); the S accumulator is re-packed in registers as the A operand
// of P V.  Each warp keeps its own online softmax (row max m, row sum l, O)
// in the exp2 domain; the warps and then the CTAs of a cluster merge in
// fixed order, so results are bit-reproducible.
#pragma once

#include <cuda.h>

#include "nosa_common.cuh"
#include "nosa_kernels.h"

namespace nosa {

constexpr int kConsumerWarps = 4;                          // warps that own 16 tokens of a tile each
constexpr int kHalfBytes = kBlock * 128;                   // one 64-token x 64-dim box: 8 KB
constexpr int kStageBytes = 4 * kHalfBytes;                // K lo/hi, V lo/hi: 32 KB
constexpr int kMinStages = 3;                              // ring of 2 CTAs per SM
constexpr int kMaxStages = 6;                              // ring of 1 CTA per SM
constexpr int kRingBytes = kMinStages * kStageBytes;       // 96 KB: the smallest ring
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

// Per-warp online-softmax state of the attention over a CTA's tiles.
struct AttnState {
  float acc[16][4];  // O: 16 n-tiles of 8 dims; rows grp (e 0,1) and grp+8 (e 2,3)
  float m[2];        // running max (exp2 domain) of rows grp, grp+8
  float l[2];        // running sum (this lane's columns until attn_finish)
};

__device__ inline void attn_init(AttnState& st) {
#pragma unroll
  for (int n = 0; n < 16; ++n) st.acc[n][0] = st.acc[n][1] = st.acc[n][2] = st.acc[n][3] = 0.0f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.0f;
}

// The group's queries as the bf16 A operand of m16n8k16 (rows = heads,
// zero past G), 8 k-steps of 16 dimensions.
__device__ inline void load_attn_q(uint32_t (&qa)[8][4], const __nv_bfloat16* __restrict__ q_group, int G, int lane) {
  const int grp = lane >> 2, tig = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = grp + (r & 1) * 8;
      const int col = ks * 16 + 2 * tig + (r >> 1) * 8;
      qa[ks][r] = row < G ? __ldg(reinterpret_cast<const uint32_t*>(q_group + row * kHeadDim + col)) : 0u;
    }
  }
}

// One warp's share (tokens [16w, 16w+16)) of the tile of block `blk`
// (blk < 0: a rejected tile, all masked) staged at `st`, for a sequence of
// length L: S = Q K^T, online softmax update, O += P V.
__device__ inline void attend_tile(AttnState& s, const uint32_t (&qa)[8][4], uint8_t* st, int blk, int L,
                                   float scale_log2, int warp, int lane) {
  const int tig = lane & 3;
  const uint32_t k_lo = smem_addr(st);
  const uint32_t v_lo = k_lo + 2 * kHalfBytes;
  const int wrow = warp * 16;
  const int64_t tok0 = static_cast<int64_t>(blk) * kBlock + wrow;
  // Rows of this warp past the sequence end (or of a rejected tile) may hold
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
  // S = Q K^T over this warp's 16 tokens (two n-tiles of 8), even and odd
  // k-steps in separate accumulators (two short chains instead of one long).
  float sc[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    float s0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int row = wrow + nt * 8 + (lane & 7);
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
  // Scale into the exp2 domain and mask tokens outside [0, L) / rejected tiles.
  float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int64_t tok = tok0 + nt * 8 + 2 * tig + (e & 1);
      const bool valid = blk >= 0 && tok < L;
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
    alpha[rr] = exp2f(s.m[rr] - m_use[rr]);
    s.m[rr] = m_new;
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
  s.l[0] = s.l[0] * alpha[0] + rs[0];
  s.l[1] = s.l[1] * alpha[1] + rs[1];
#pragma unroll
  for (int d = 0; d < 16; ++d) {
    s.acc[d][0] *= alpha[0];
    s.acc[d][1] *= alpha[0];
    s.acc[d][2] *= alpha[1];
    s.acc[d][3] *= alpha[1];
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
    mma_bf16_16816(s.acc[2 * dp], pa, b0, b1);
    mma_bf16_16816(s.acc[2 * dp + 1], pa, b2, b3);
  }
  if (partial) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
}

// Completes the row sums (a row's columns are spread over a quad of lanes).
__device__ inline void attn_finish(AttnState& s) {
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    s.l[rr] += __shfl_xor_sync(0xffffffffu, s.l[rr], 1);
    s.l[rr] += __shfl_xor_sync(0xffffffffu, s.l[rr], 2);
  }
}

}  // namespace nosa
