// Per-window CIS mean pooling, shared by the pool-append kernel and the fused
// decode-step kernel.
//
// "从论文到代码：手把手教你理解NOSA-8B的高效注意力机制实现" (nzsm.cn),
// "NOSA-8B的核心实现模块" item 2; "NOSA-1B 性能基准全解析" (wmrh.cn) §三.3
// (kernel_size 32, stride 16):  pooled[j] = (1/32) * sum_{t=16j}^{16j+31} K[t].
#pragma once

#include "kv_int8.cuh"
#include "nosa_common.cuh"

namespace nosa {

__device__ inline float4 bf16x4_to_float4(uint2 raw) {
  float4 f;
  f.x = __uint_as_float(raw.x << 16);
  f.y = __uint_as_float(raw.x & 0xFFFF0000u);
  f.z = __uint_as_float(raw.y << 16);
  f.w = __uint_as_float(raw.y & 0xFFFF0000u);
  return f;
}

// The window sum `acc` (lane l: dims 4l..4l+3) x 1/32 (exact), stored as
// fp32 or rounded to bf16 (nearest, ties to even).
__device__ inline void store_pooled(float4 acc, void* __restrict__ dst, bool bf16, int lane) {
  constexpr float inv = 1.0f / kPoolKernel;
  const float4 m = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (bf16) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(m.x, m.y), hi = __floats2bfloat162_rn(m.z, m.w);
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t*>(&lo);
    packed.y = *reinterpret_cast<const uint32_t*>(&hi);
    reinterpret_cast<uint2*>(dst)[lane] = packed;
  } else {
    reinterpret_cast<float4*>(dst)[lane] = m;
  }
}

// One warp pools window j of one (sequence, KV head): lane l owns dims
// 4l..4l+3.  All 32 rows are loaded before any is summed (one memory round
// trip); the row of token `fresh_tok` (when >= 0) is taken from `fresh`
// instead of the cache -- the token being appended by the same launch.  The
// fp32 sum runs in ascending token order, then x 1/32 (exact), so appending
// and rebuilding give identical bits.  The window's tokens [16j, 16j+32) are
// found through `kv` (in a paged cache they span at most two pages); the
// caller checks that they lie inside the cache.  The mean is stored as fp32,
// or as bf16 (nearest, ties to even) when `bf16`.
__device__ inline void pool_window_warp(const __nv_bfloat16* __restrict__ k_cache, int hkv, const KvRows& kv,
                                        int h, int64_t j, int64_t fresh_tok, const uint2* __restrict__ fresh,
                                        void* __restrict__ dst, bool bf16, int lane) {
  const int64_t t0 = j * kPoolStride;
  // Tokens [t0, t0+split) are consecutive rows from row_a, the rest from row_b.
  const int split = kv.pages ? min(kPoolKernel, static_cast<int>(kPageTokens - t0 % kPageTokens)) : kPoolKernel;
  const int64_t row_a = kv.row(t0);
  const int64_t row_b = split < kPoolKernel ? kv.row(t0 + split) : 0;
  const uint2* src = reinterpret_cast<const uint2*>(k_cache) + static_cast<int64_t>(h) * (kHeadDim / 4) + lane;
  const int64_t row_stride = static_cast<int64_t>(hkv) * kHeadDim / 4;  // in uint2
  uint2 raw[kPoolKernel];
#pragma unroll
  for (int t = 0; t < kPoolKernel; ++t) {
    const int64_t row = t < split ? row_a + t : row_b + (t - split);
    raw[t] = __ldcg(src + row * row_stride);
  }
  const int64_t r = fresh_tok - t0;
  if (fresh != nullptr && r >= 0 && r < kPoolKernel) {
    const uint2 f = fresh[lane];
#pragma unroll
    for (int t = 0; t < kPoolKernel; ++t)
      if (t == r) raw[t] = f;
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int t = 0; t < kPoolKernel; ++t) {
    const float4 f = bf16x4_to_float4(raw[t]);
    acc.x += f.x;
    acc.y += f.y;
    acc.z += f.z;
    acc.w += f.w;
  }
  store_pooled(acc, dst, bf16, lane);
}

// The same window over an INT8 key cache: row t contributes s_t * code_t
// (one fp32 product per value), summed in ascending token order.  The fresh
// token's row is quantized here from `fresh` (bf16) exactly as the append
// stores it, so appending and rebuilding still give identical bits.
__device__ inline void pool_window_warp_int8(const Int8Cache& c, int hkv, const KvRows& kv, int h, int64_t j,
                                             int64_t fresh_tok, const uint2* __restrict__ fresh,
                                             void* __restrict__ dst, bool bf16, int lane) {
  const int64_t t0 = j * kPoolStride;
  const int split = kv.pages ? min(kPoolKernel, static_cast<int>(kPageTokens - t0 % kPageTokens)) : kPoolKernel;
  const int64_t row_a = kv.row(t0);
  const int64_t row_b = split < kPoolKernel ? kv.row(t0 + split) : 0;
  uint32_t codes[kPoolKernel];
  float sc[kPoolKernel];
#pragma unroll
  for (int t = 0; t < kPoolKernel; ++t) {
    const int64_t row = t < split ? row_a + t : row_b + (t - split);
    codes[t] = __ldcg(reinterpret_cast<const uint32_t*>(c.row(row, hkv, h)) + lane);
    sc[t] = __ldcg(c.scale(row, h));
  }
  const int64_t r = fresh_tok - t0;
  if (fresh != nullptr && r >= 0 && r < kPoolKernel) {
    float fs;
    const uint32_t fc = quantize_row_warp(fresh[lane], fs);
#pragma unroll
    for (int t = 0; t < kPoolKernel; ++t)
      if (t == r) {
        codes[t] = fc;
        sc[t] = fs;
      }
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int t = 0; t < kPoolKernel; ++t) {
    const float4 f = dequant4(codes[t], sc[t]);
    acc.x += f.x;
    acc.y += f.y;
    acc.z += f.z;
    acc.w += f.w;
  }
  store_pooled(acc, dst, bf16, lane);
}

}  // namespace nosa
