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

#include "kv_int8.cuh"
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

// 2^x with the hardware approximation (ex2.approx.ftz: relative error about
// 2^-22, results below 2^-126 flushed to zero; 2^-inf = 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
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
  float vscale;      // INT8 caches: the V-scale factor U of acc (see attend_tile_int8)
};

__device__ inline void attn_init(AttnState& st) {
#pragma unroll
  for (int n = 0; n < 16; ++n) st.acc[n][0] = st.acc[n][1] = st.acc[n][2] = st.acc[n][3] = 0.0f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.0f;
  st.vscale = 0.0f;
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
    alpha[rr] = fast_exp2(s.m[rr] - m_use[rr]);
    s.m[rr] = m_new;
  }
  float rs[2] = {0.0f, 0.0f};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
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

// ------------------------------------------------------------ INT8 caches
// A ring stage holds two 64-token tiles: K and V of each are 64 x 128 int8
// codes (8 KB, one 3-D box {128 bytes, 1 head, 64 tokens} with the 128-byte
// swizzle) at stage offsets 0 / 8 KB (first tile) and 16 / 24 KB (second).
// Their scale rows (fp32, 68 values starting at the 16-byte aligned token at
// or below the tile's first row) sit in a separate slot area.
constexpr int kTileBytesInt8 = kBlock * kHeadDim;              // 8 KB
constexpr int kScaleBox = kBlock + 4;                           // scales per copy
constexpr int kScaleSlot = 384;                                 // 128-byte aligned slot for 272 bytes
constexpr int kScaleStageBytes = 4 * kScaleSlot;                // K0, V0, K1, V1
constexpr uint32_t kTileTxBytesInt8 = 2 * kTileBytesInt8 + 2 * kScaleBox * 4;

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ inline void mma_f16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Two codes as an exact f16x2 operand: `biased` holds codes XOR 0x80 (i.e.
// code + 128) in the bytes that `sel` places into the low byte of each half;
// the high bytes become 0x64, the f16 exponent of 1024, so each half is
// 1024 + code + 128, and subtracting 1152 leaves the code exactly.
__device__ __forceinline__ uint32_t biased_pair_to_f16x2(uint32_t biased, uint32_t sel) {
  uint32_t h = __byte_perm(biased, 0x64646464u, sel);
  asm("sub.rn.f16x2 %0, %0, %1;" : "+r"(h) : "r"(0x64806480u));
  return h;
}

// The group's queries as the f16 A operand for INT8 tiles, scaled by 2^-e
// (e >= 0, the smallest power that brings max |q| below 2^15, normally 0) so
// that every bf16 value converts exactly unless it is below f16's normal
// range (then to f16's subnormal grid).  The head dimension is permuted so
// that each lane's K operand is 32 contiguous bytes of a token row: k-step
// ks, quad position tig covers dims 32*tig + 4*ks + {0, 1} (slots 2tig,
// 2tig+1) and + {2, 3} (slots 2tig+8, 2tig+9); a dot product does not depend
// on the order of its terms.  Returns 2^e.
__device__ inline float load_attn_q_int8(uint32_t (&qa)[8][4], const __nv_bfloat16* __restrict__ q_group, int G,
                                         int lane) {
  const int grp = lane >> 2, tig = lane & 3;
  uint32_t raw[8][4];
  float m = 0.0f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = grp + (r & 1) * 8;
      const int col = 32 * tig + 4 * ks + 2 * (r >> 1);
      raw[ks][r] = row < G ? __ldg(reinterpret_cast<const uint32_t*>(q_group + row * kHeadDim + col)) : 0u;
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(raw[ks][r] << 16)), fabsf(__uint_as_float(raw[ks][r] & 0xFFFF0000u))));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int ilog = static_cast<int>((__float_as_uint(m) >> 23) & 0xFFu) - 127;
  const int e = ilog > 14 ? ilog - 14 : 0;
  const float down = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int r = 0; r < 4; ++r)
      qa[ks][r] = pack_f16x2(__uint_as_float(raw[ks][r] << 16) * down,
                             __uint_as_float(raw[ks][r] & 0xFFFF0000u) * down);
  }
  return __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
}

// One warp's share of an INT8 ring stage: tokens [16*warp, 16*warp + 16)
// of each of its NT tiles (NT = 1 or 2; tile x has codes at stage offsets
// 2x * 8 KB (K) and (2x + 1) * 8 KB (V), scales `ksc[x]` / `vsc[x]` indexed
// by the token's position in the tile, block `blk[x]`).  The codes become
// exact f16 operands in registers; the per-token scales are applied where
// they factor out of the tensor-core products:
//   score_t = scale * 2^e * ks_t * (q 2^-e . code_k,t)     (fp32 accumulate)
//   O       = U * sum_t (p_t * vs_t / U) code_v,t
// U is the warp's running maximum of vs over its tokens (`s.vscale`): P is
// rounded to f16 as p_t * vs_t / U <= 1, and when U grows the accumulator is
// rescaled together with the softmax correction.  The row sums are taken
// over p_t.  Masked tokens (past L, rejected tile) get p = 0 and never touch
// their scales, so stale rows cannot give NaN.  The O accumulator is
// permuted: acc[j][e] holds dim 32*tig + 16*(e & 1) + j (rows grp, grp + 8).
// Both tiles' scores come first (2 NT independent mma chains), then one
// softmax update and one rescale for the stage, then P V tile by tile.
template <int NT>
__device__ inline void attend_stage_int8(AttnState& s, const uint32_t (&qa)[8][4], float qpow, const uint8_t* st,
                                         const float* const (&ksc)[2], const float* const (&vsc)[2],
                                         const int (&blk)[2], int L, float scale_log2, int warp, int lane,
                                         uint64_t* stamps = nullptr) {
  const int grp = lane >> 2, tig = lane & 3;
  const int wrow = warp * 16;
  constexpr int kC = 2 * NT;  // score chains: (tile x, n-tile nt) = chain 2x + nt
  float sc[kC][4];
#pragma unroll
  for (int c = 0; c < kC; ++c) sc[c][0] = sc[c][1] = sc[c][2] = sc[c][3] = 0.0f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {  // k-steps 4 half .. 4 half + 3: chunk 2 tig + half of the row
    uint4 w[kC];
#pragma unroll
    for (int c = 0; c < kC; ++c)
      w[c] = lds128(swz(smem_addr(st + (c >> 1) * 2 * kTileBytesInt8), wrow + (c & 1) * 8 + grp, 2 * tig + half));
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        const uint32_t word = k4 == 0 ? w[c].x : k4 == 1 ? w[c].y : k4 == 2 ? w[c].z : w[c].w;
        const uint32_t u = word ^ 0x80808080u;
        mma_f16_16816(sc[c], qa[4 * half + k4], biased_pair_to_f16x2(u, 0x4140u), biased_pair_to_f16x2(u, 0x4342u));
      }
    }
  }
#ifdef NOSA_TRACE
  if (stamps) {
    asm volatile("" ::"f"(sc[0][0]), "f"(sc[kC - 1][3]));
    stamps[0] = global_timer_ns();
  }
#endif
  bool valid[kC][2];
  float vs[kC][2];
  float mx[2] = {-INFINITY, -INFINITY};
  float umax = 0.0f;
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    const int x = c >> 1, nt = c & 1;
    const int64_t tok0 = static_cast<int64_t>(blk[x]) * kBlock + wrow + nt * 8 + 2 * tig;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      const int tt = wrow + nt * 8 + 2 * tig + cc;  // position in the tile
      valid[c][cc] = blk[x] >= 0 && tok0 + cc < L;
      const float kmul = valid[c][cc] ? ksc[x][tt] * (scale_log2 * qpow) : 0.0f;
      vs[c][cc] = valid[c][cc] ? vsc[x][tt] : 0.0f;
      umax = fmaxf(umax, vs[c][cc]);
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        float& v = sc[c][2 * rr + cc];
        v = valid[c][cc] ? v * kmul : -INFINITY;
        mx[rr] = fmaxf(mx[rr], v);
      }
    }
  }
#ifdef NOSA_TRACE
  if (stamps) {
    asm volatile("" ::"f"(mx[0]), "f"(mx[1]), "f"(umax));
    stamps[1] = global_timer_ns();
  }
#endif
  umax = fmaxf(umax, __shfl_xor_sync(0xffffffffu, umax, 1));
  umax = fmaxf(umax, __shfl_xor_sync(0xffffffffu, umax, 2));
  const float u_new = fmaxf(s.vscale, umax);
  const float inv_u = u_new > 0.0f ? __frcp_rn(u_new) : 0.0f;
  const float uratio = u_new > 0.0f ? s.vscale * inv_u : 1.0f;  // 0 while nothing has been accumulated
  s.vscale = u_new;
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
#ifdef NOSA_TRACE
  if (stamps) {
    asm volatile("" ::"f"(alpha[0]), "f"(alpha[1]), "f"(inv_u), "f"(uratio));
    stamps[2] = global_timer_ns();
  }
#endif
  float rs[2] = {0.0f, 0.0f};
#pragma unroll
  for (int c = 0; c < kC; ++c) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float pe = fast_exp2(sc[c][e] - m_use[e >> 1]);
      rs[e >> 1] += pe;
      sc[c][e] = valid[c][e & 1] ? pe * (vs[c][e & 1] * inv_u) : 0.0f;
    }
  }
#ifdef NOSA_TRACE
  if (stamps) {
    asm volatile("" ::"f"(rs[0]), "f"(rs[1]), "f"(sc[kC - 1][3]));
    stamps[3] = global_timer_ns();
  }
#endif
  s.l[0] = s.l[0] * alpha[0] + rs[0];
  s.l[1] = s.l[1] * alpha[1] + rs[1];
  const float a0 = alpha[0] * uratio, a1 = alpha[1] * uratio;
#pragma unroll
  for (int d = 0; d < 16; ++d) {
    s.acc[d][0] *= a0;
    s.acc[d][1] *= a0;
    s.acc[d][2] *= a1;
    s.acc[d][3] *= a1;
  }
#ifdef NOSA_TRACE
  if (stamps) {
    asm volatile("" ::"f"(s.acc[15][3]), "f"(s.acc[0][0]));
    stamps[4] = global_timer_ns();
  }
#endif
#pragma unroll
  for (int x = 0; x < NT; ++x) {
    // P'' = p * vs / U of tile x as the A operand: slots 2tig, 2tig+1 are
    // tokens wrow + 2tig + {0, 1}, slots 2tig+8, 2tig+9 are wrow + 8 + 2tig + {0, 1}.
    const uint32_t pa[4] = {pack_f16x2(sc[2 * x][0], sc[2 * x][1]), pack_f16x2(sc[2 * x][2], sc[2 * x][3]),
                            pack_f16x2(sc[2 * x + 1][0], sc[2 * x + 1][1]),
                            pack_f16x2(sc[2 * x + 1][2], sc[2 * x + 1][3])};
    // V operand of n-tile j: dim 16*grp + j of those four tokens, i.e. byte
    // j of 16-byte chunk grp of their rows.  Bytes of two rows are
    // interleaved first, then each pair becomes one f16x2.
    const uint32_t v_base = smem_addr(st + (2 * x + 1) * kTileBytesInt8);
    const uint4 ra = lds128(swz(v_base, wrow + 2 * tig, grp)), rb = lds128(swz(v_base, wrow + 2 * tig + 1, grp));
    const uint4 rc = lds128(swz(v_base, wrow + 8 + 2 * tig, grp)), rd = lds128(swz(v_base, wrow + 9 + 2 * tig, grp));
    const uint32_t A[4] = {ra.x ^ 0x80808080u, ra.y ^ 0x80808080u, ra.z ^ 0x80808080u, ra.w ^ 0x80808080u};
    const uint32_t B[4] = {rb.x ^ 0x80808080u, rb.y ^ 0x80808080u, rb.z ^ 0x80808080u, rb.w ^ 0x80808080u};
    const uint32_t C[4] = {rc.x ^ 0x80808080u, rc.y ^ 0x80808080u, rc.z ^ 0x80808080u, rc.w ^ 0x80808080u};
    const uint32_t D[4] = {rd.x ^ 0x80808080u, rd.y ^ 0x80808080u, rd.z ^ 0x80808080u, rd.w ^ 0x80808080u};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      // bytes {0, 1} and {2, 3} of rows A/B and C/D, interleaved: [a0 b0 a1 b1], [a2 b2 a3 b3]
      const uint32_t ab01 = __byte_perm(A[wi], B[wi], 0x5140u), ab23 = __byte_perm(A[wi], B[wi], 0x7362u);
      const uint32_t cd01 = __byte_perm(C[wi], D[wi], 0x5140u), cd23 = __byte_perm(C[wi], D[wi], 0x7362u);
      mma_f16_16816(s.acc[4 * wi + 0], pa, biased_pair_to_f16x2(ab01, 0x4140u), biased_pair_to_f16x2(cd01, 0x4140u));
      mma_f16_16816(s.acc[4 * wi + 1], pa, biased_pair_to_f16x2(ab01, 0x4342u), biased_pair_to_f16x2(cd01, 0x4342u));
      mma_f16_16816(s.acc[4 * wi + 2], pa, biased_pair_to_f16x2(ab23, 0x4140u), biased_pair_to_f16x2(cd23, 0x4140u));
      mma_f16_16816(s.acc[4 * wi + 3], pa, biased_pair_to_f16x2(ab23, 0x4342u), biased_pair_to_f16x2(cd23, 0x4342u));
    }
  }
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
