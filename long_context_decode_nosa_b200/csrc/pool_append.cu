// K1 -- CIS mean pooling of the key cache, appended incrementally.
//
// "从论文到代码：手把手教你理解NOSA-8B的高效注意力机制实现" (nzsm.cn),
// "NOSA-8B的核心实现模块" item 2 (keys pooled with cis_pooling(k, cu_seqlens));
// "NOSA-1B 性能基准全解析" (wmrh.cn) §三.3 (kernel_size 32, stride 16).
//
// One warp per (sequence, KV head, new window).  Lane l owns dims 4l..4l+3:
// each of the 32 rows of the window is one coalesced 256-byte warp load
// (8 bytes per lane), summed in fp32 in ascending token order, then scaled by
// 1/32 (exact).  A fixed order makes an incremental append bit-identical to a
// rebuild.  With k_new/v_new given, warp 0 of chunk 0 also stores the new
// token's K/V rows into the caches; pooling reads that token from k_new, so
// no cross-warp ordering is needed.  Contiguous or paged caches (KvRows),
// bf16 or INT8 (the new rows are quantized on the way in; pooling reads
// s * code).
//
// Also the INT8 quantization of whole cache rows (kv_quantize_kernel), for
// caches filled outside the decode step.
#include "nosa_common.cuh"
#include "nosa_kernels.h"
#include "kv_int8.cuh"
#include "pool_device.cuh"

namespace nosa {

namespace {

constexpr int kWarpsPerCta = 4;

__global__ void __launch_bounds__(kWarpsPerCta * 32)
    pool_append_kernel(const PoolArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.y;
  const int i = pair / a.hkv, h = pair % a.hkv;
  grid_dependency_wait();
  allow_dependents();
  const int32_t len_new = a.len_new[i];
  const int32_t len_old = a.len_old ? a.len_old[i] : len_new - 1;
  KvRows kv;
  kv.pages = a.page_table ? a.page_table + static_cast<int64_t>(i) * a.max_pages : nullptr;
  kv.base = kv.pages ? 0 : a.seq_start[i];
  kv.num_pages = a.cache_rows / kPageTokens;
  if (len_old < 0 || len_new < len_old) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(a.status, NOSA_DEV_BAD_LENGTH);
    return;
  }
  const bool fits = kv.pages ? static_cast<int64_t>(len_new) <= static_cast<int64_t>(a.max_pages) * kPageTokens
                             : kv.base >= 0 && kv.base + len_new <= a.cache_rows;
  if (!fits) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(a.status, NOSA_DEV_CACHE_ROWS);
    return;
  }
  const bool append = a.k_new != nullptr;
  if (append && len_new != len_old + 1) {
    if (blockIdx.x == 0 && threadIdx.x == 0) set_status(a.status, NOSA_DEV_APPEND_ONE);
    return;
  }
  const uint2* knew_row =
      append ? reinterpret_cast<const uint2*>(a.k_new + (static_cast<int64_t>(i) * a.hkv + h) * kHeadDim)
             : nullptr;
  if (append && blockIdx.x == 0 && warp == 0) {
    if (!kv.page_ok(len_old)) {
      if (lane == 0) set_status(a.status, NOSA_DEV_BAD_INDEX);
      return;
    }
    const int64_t row = kv.row(len_old) * a.hkv + h;
    const uint2* vnew_row =
        reinterpret_cast<const uint2*>(a.v_new + (static_cast<int64_t>(i) * a.hkv + h) * kHeadDim);
    if (a.kv_int8) {
      const int64_t r = kv.row(len_old);
      store_int8_row_warp(Int8Cache{reinterpret_cast<int8_t*>(a.k_cache), a.k_scale, a.scale_stride}, a.hkv, r, h,
                          knew_row, lane);
      store_int8_row_warp(Int8Cache{reinterpret_cast<int8_t*>(a.v_cache), a.v_scale, a.scale_stride}, a.hkv, r, h,
                          vnew_row, lane);
    } else {
      reinterpret_cast<uint2*>(a.k_cache + row * kHeadDim)[lane] = knew_row[lane];
      reinterpret_cast<uint2*>(a.v_cache + row * kHeadDim)[lane] = vnew_row[lane];
    }
  }
  const int64_t j_first = n_windows(len_old), j_end = n_windows(len_new);
  if (j_end - j_first > a.max_new_keys && blockIdx.x == 0 && threadIdx.x == 0)
    set_status(a.status, NOSA_DEV_MAX_NEW_KEYS);
  const int64_t j = j_first + static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + warp;
  if (j >= j_end || j - j_first >= a.max_new_keys) return;
  if (j >= a.nc_cap) {
    if (lane == 0) set_status(a.status, NOSA_DEV_NC_CAP);
    return;
  }
  const int64_t at = ((static_cast<int64_t>(i) * a.hkv + h) * a.nc_cap + j) * kHeadDim;
  void* dst = a.pooled_bf16 ? static_cast<void*>(static_cast<__nv_bfloat16*>(a.pooled) + at)
                            : static_cast<void*>(static_cast<float*>(a.pooled) + at);
  if (!kv.page_ok(j * kPoolStride) || !kv.page_ok(j * kPoolStride + kPoolKernel - 1)) {
    if (lane == 0) set_status(a.status, NOSA_DEV_BAD_INDEX);
    return;
  }
  if (a.kv_int8)
    pool_window_warp_int8(Int8Cache{reinterpret_cast<int8_t*>(a.k_cache), a.k_scale, a.scale_stride}, a.hkv, kv, h, j,
                          append ? len_old : -1, knew_row, dst, a.pooled_bf16 != 0, lane);
  else
    pool_window_warp(a.k_cache, a.hkv, kv, h, j, append ? len_old : -1, knew_row, dst, a.pooled_bf16 != 0, lane);
}

// One warp per (row, KV head): src row r (bf16 [rows, hkv, 128]) into cache
// row row0 + r.
__global__ void __launch_bounds__(kWarpsPerCta * 32)
    kv_quantize_kernel(const __nv_bfloat16* __restrict__ src, int8_t* codes, float* scales, int64_t scale_stride,
                       int64_t row0, int64_t rows, int hkv) {
  const int lane = threadIdx.x & 31;
  const Int8Cache c{codes, scales, scale_stride};
  const int64_t units = rows * hkv;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5); u < units;
       u += static_cast<int64_t>(gridDim.x) * kWarpsPerCta) {
    const int64_t r = u / hkv;
    const int h = static_cast<int>(u % hkv);
    store_int8_row_warp(c, hkv, row0 + r, h, reinterpret_cast<const uint2*>(src + u * kHeadDim), lane);
  }
}

}  // namespace

cudaError_t launch_quantize_int8(const __nv_bfloat16* src, int8_t* codes, float* scales, int64_t scale_stride,
                                 int64_t row0, int64_t rows, int hkv, cudaStream_t stream) {
  const int64_t units = rows * hkv;
  if (units == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (units + kWarpsPerCta - 1) / kWarpsPerCta;
  const int blocks = static_cast<int>(want < static_cast<int64_t>(sms) * 16 ? want : static_cast<int64_t>(sms) * 16);
  kv_quantize_kernel<<<blocks, kWarpsPerCta * 32, 0, stream>>>(src, codes, scales, scale_stride, row0, rows, hkv);
  return cudaGetLastError();
}

cudaError_t launch_pool_append(const PoolArgs& a, cudaStream_t stream) {
  const int pairs = a.batch * a.hkv;
  if (pairs == 0) return cudaSuccess;
  const int chunks = (a.max_new_keys + kWarpsPerCta - 1) / kWarpsPerCta;
  dim3 grid(chunks > 0 ? chunks : 1, pairs);
  return launch_overlapped(pool_append_kernel, grid, dim3(kWarpsPerCta * 32), 0, stream, a);
}

}  // namespace nosa
