// The decode step for callers that cannot allocate device memory.
//
// nosa_decode_step_device needs a caller-provided workspace (device status
// word, block scores of very long sequences, staging).  Some callers have no way to provide one:
// a plugin loaded into an inference engine whose memory manager owns the
// whole device pool and exposes no workspace hook, or a serving loop that
// must not call cudaMalloc once the KV cache has claimed the free memory
// (and where an allocation would also synchronise the device).  For them,
// nosa_decode_step_device_noalloc runs the same fused step with its scratch
// in a fixed-size array that the library itself defines in device memory.
// The array belongs to this file's device code: CUDA creates it on a device
// when it loads that code there -- at the first call on the device under
// CUDA's default lazy loading -- and it stays until the process exits.
#include <cstdio>

#include "nosa.h"
#include "nosa_kernels.h"

namespace {

// The library's own scratch for nosa_decode_step_device_noalloc: 8 MiB per
// device (the NOSA-1B attention shape at batch 8 and 16K tokens needs 74 KB;
// sequences beyond 2048 candidates keep their block scores here too).
constexpr size_t kNoAllocScratchBytes = size_t{8} << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

}  // namespace

extern "C" {

int nosa_decode_step_device_noalloc(const nosa_params* p, const void* q, const void* k_new, const void* v_new,
                                    void* k_cache, void* v_cache, int64_t cache_rows, const int64_t* seq_start,
                                    const int32_t* seq_len, int batch, int max_seq_len, void* pooled, int nc_cap,
                                    int32_t* sel_idx, int32_t* sel_cnt, void* out, float* lse, void* stream) {
  // Every host check of the workspace entry point comes first: a rejected
  // call enqueues nothing.  An empty batch returns here, with no CUDA call.
  if (int rc = nosa::check_decode_step_device(p, q, k_new, v_new, k_cache, v_cache, cache_rows, seq_start, seq_len,
                                              batch, max_seq_len, pooled, nc_cap, sel_idx, sel_cnt, out))
    return rc;
  if (batch == 0) return NOSA_OK;
  const size_t need = nosa_workspace_size(p, batch, max_seq_len);
  if (need > kNoAllocScratchBytes) {
    char buf[256];
    snprintf(buf, sizeof buf,
             "this batch needs %zu bytes of scratch but the library's built-in scratch holds %zu; "
             "use nosa_decode_step_device with a workspace",
             need, kNoAllocScratchBytes);
    return nosa::record_error(NOSA_ERR_WORKSPACE, buf);
  }
  // In host code the array's name is a host-side stand-in, never a device
  // address: the device address is looked up on the current device at every
  // call (cheap once the code is loaded), so it is never stale -- not after
  // a device reset either.
  void* scratch = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
  if (e != cudaSuccess || scratch == nullptr) return nosa::record_error(NOSA_ERR_CUDA, cudaGetErrorString(e));
  // The array keeps whatever the previous call left; the status word starts
  // at zero.
  const size_t zero_bytes = nosa::workspace_counter_bytes(p, batch, max_seq_len);
  e = cudaMemsetAsync(scratch, 0, zero_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return nosa::record_error(NOSA_ERR_CUDA, cudaGetErrorString(e));
  return nosa_decode_step_device(p, q, k_new, v_new, k_cache, v_cache, cache_rows, seq_start, seq_len, batch,
                                 max_seq_len, pooled, nc_cap, sel_idx, sel_cnt, out, lse, scratch,
                                 kNoAllocScratchBytes, stream);
}

}  // extern "C"
