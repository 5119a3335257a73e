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
// Every GPU that loads the library holds that array until the process exits.
#include <cstdio>
#include <mutex>

#include "nosa.h"
#include "nosa_kernels.h"

namespace {

// The library's own scratch for nosa_decode_step_device_noalloc: 8 MiB per
// device (the NOSA-1B attention shape at batch 8 and 16K tokens needs 74 KB;
// sequences beyond 2048 candidates keep their block scores here too).
constexpr size_t kNoAllocScratchBytes = size_t{8} << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device.  In host code the array's
// name is only a host-side stand-in, never a device address, so the address
// is looked up once per device (with that device current) and cached.
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" {

int nosa_decode_step_device_noalloc(const nosa_params* p, const void* q, const void* k_new, const void* v_new,
                                    void* k_cache, void* v_cache, int64_t cache_rows, const int64_t* seq_start,
                                    const int32_t* seq_len, int batch, int max_seq_len, void* pooled, int nc_cap,
                                    int32_t* sel_idx, int32_t* sel_cnt, void* out, float* lse, void* stream) {
  const size_t need = nosa_workspace_size(p, batch, max_seq_len);
  if (need == 0)  // invalid parameters: let the regular entry point report them
    return nosa_decode_step_device(p, q, k_new, v_new, k_cache, v_cache, cache_rows, seq_start, seq_len, batch,
                                   max_seq_len, pooled, nc_cap, sel_idx, sel_cnt, out, lse, nullptr, 0, stream);
  if (need > kNoAllocScratchBytes) {
    char buf[256];
    snprintf(buf, sizeof buf,
             "this batch needs %zu bytes of scratch but the library's built-in scratch holds %zu; "
             "use nosa_decode_step_device with a workspace",
             need, kNoAllocScratchBytes);
    return nosa::record_error(NOSA_ERR_WORKSPACE, buf);
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nosa::record_error(NOSA_ERR_CUDA, "no current CUDA device (or device index above 63)");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
      void* addr = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
      if (e != cudaSuccess || addr == nullptr) return nosa::record_error(NOSA_ERR_CUDA, cudaGetErrorString(e));
      g_scratch_addr[dev] = addr;
    }
    scratch = g_scratch_addr[dev];
  }
  // The array keeps whatever the previous call left; the status word starts
  // at zero.
  const size_t zero_bytes = nosa::workspace_counter_bytes(p, batch, max_seq_len);
  const cudaError_t e = cudaMemsetAsync(scratch, 0, zero_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return nosa::record_error(NOSA_ERR_CUDA, cudaGetErrorString(e));
  return nosa_decode_step_device(p, q, k_new, v_new, k_cache, v_cache, cache_rows, seq_start, seq_len, batch,
                                 max_seq_len, pooled, nc_cap, sel_idx, sel_cnt, out, lse, scratch,
                                 kNoAllocScratchBytes, stream);
}

}  // extern "C"
