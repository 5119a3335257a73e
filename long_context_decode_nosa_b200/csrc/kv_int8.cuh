// INT8 K/V caches: quantization of a cache row and the conversions the
// kernels use to read one.
//
// "NOSA 技术架构解析" (devpress.csdn.net) §1.1 "双阶段稀疏注意力设计",
// "关键技巧": the decode stage may switch to 8-bit integers.  Reading taken
// here: every cache row (token, KV head) of 128 bf16 values x is kept as 128
// int8 codes and one fp32 scale, symmetric per row:
//     amax = max |x_d|,  s = amax / 127,  code_d = clamp(rint(x_d / s), -127, 127)
// with both divisions IEEE fp32 (round to nearest) and rint half to even; an
// all-zero row has s = 0 and zero codes.  Pooling and attention read the
// dequantized value s * code.
//
// Cache buffer (one for K, one for V): codes int8 [cache_rows, hkv, 128],
// then, at byte cache_rows * hkv * 128, scales fp32 [hkv, scale_stride] with
// scale_stride = cache_rows rounded up to a multiple of 4 (so a head's row of
// scales is 16-byte aligned for the tensor copies).
#pragma once

#include "nosa_common.cuh"

namespace nosa {

__host__ __device__ constexpr int64_t int8_scale_stride(int64_t cache_rows) { return (cache_rows + 3) & ~int64_t{3}; }
__host__ __device__ constexpr int64_t int8_scale_offset(int64_t cache_rows, int hkv) {
  return cache_rows * hkv * kHeadDim;
}

// Where a sequence's INT8 rows and scales are.
struct Int8Cache {
  int8_t* codes;   // [cache_rows, hkv, 128]
  float* scales;   // [hkv, stride]
  int64_t stride;

  __device__ int8_t* row(int64_t r, int hkv, int h) const { return codes + (r * hkv + h) * kHeadDim; }
  __device__ float* scale(int64_t r, int h) const { return scales + h * stride + r; }
};

// One warp quantizes a 128-value bf16 row (lane l holds values 4l..4l+3 as
// the 8-byte `raw`): returns the lane's four codes packed little-endian and
// the row's scale (the same in every lane).
__device__ inline uint32_t quantize_row_warp(uint2 raw, float& scale) {
  float x[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u), __uint_as_float(raw.y << 16),
                __uint_as_float(raw.y & 0xFFFF0000u)};
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 127.0f);
  uint32_t packed = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    int c = s > 0.0f ? __float2int_rn(__fdiv_rn(x[k], s)) : 0;
    c = c > 127 ? 127 : (c < -127 ? -127 : c);
    packed |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * k);
  }
  scale = s;
  return packed;
}

// Quantizes the bf16 row `src` (128 values) into row `r` of head `h` of an
// INT8 cache; lane 0 writes the scale.
__device__ inline void store_int8_row_warp(const Int8Cache& c, int hkv, int64_t r, int h, const uint2* __restrict__ src,
                                           int lane) {
  float s;
  const uint32_t codes = quantize_row_warp(src[lane], s);
  reinterpret_cast<uint32_t*>(c.row(r, hkv, h))[lane] = codes;
  if (lane == 0) *c.scale(r, h) = s;
}

// s * code for the four codes of a packed word (one fp32 product each).
__device__ inline float4 dequant4(uint32_t codes, float s) {
  return make_float4(s * static_cast<float>(static_cast<int8_t>(codes & 0xFFu)),
                     s * static_cast<float>(static_cast<int8_t>((codes >> 8) & 0xFFu)),
                     s * static_cast<float>(static_cast<int8_t>((codes >> 16) & 0xFFu)),
                     s * static_cast<float>(static_cast<int8_t>(codes >> 24)));
}

}  // namespace nosa
