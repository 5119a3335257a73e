// Sparse prefill (the pages' NOSAS mode: sparse attention in prefill as well
// as in decode).
//
// "NOSA 技术架构解析" (devpress.csdn.net) §1.3 "混合稀疏模式支持": NOSAF runs a
// full prefill and sparse decode, NOSAS runs both stages sparse.  The pages
// give no separate prefill rule; the reading taken here applies the decode
// rule to every prefill token: the query at position t of a sequence sees the
// prefix [0, t] (L = t + 1), selects its own top-k blocks among the candidates
// of that prefix from the compressed scores, and attends exactly over them
// plus its local window (causal within the last block).
//
// Each query token is one entry of the step kernel (its own length, q,
// selection and output) that reads the cache and pooled keys of its sequence
// through StepArgs::seq_of.  This kernel writes the per-entry lengths and
// sequence indices.
#include "nosa_common.cuh"
#include "nosa_kernels.h"

namespace nosa {

namespace {

// One thread per entry: finds its sequence (last s with q_start[s] <= e) by
// binary search over the non-decreasing q_start.  An entry that falls
// outside its sequence's rows (a q_start that is not non-decreasing) gets
// length 0, which the step kernel reports (NOSA_DEV_BAD_LENGTH) and skips.
__global__ void prefill_entries_kernel(const int32_t* __restrict__ q_start, const int32_t* __restrict__ q_pos,
                                       int batch, int total_q, int32_t* __restrict__ seq_len,
                                       int32_t* __restrict__ seq_of) {
  grid_dependency_wait();
  allow_dependents();
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total_q; e += gridDim.x * blockDim.x) {
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (q_start[mid] <= e)
        lo = mid;
      else
        hi = mid - 1;
    }
    const int first = q_start[lo], end = q_start[lo + 1];
    const bool inside = first <= e && e < end;
    const int64_t len = static_cast<int64_t>(q_pos[lo]) + (e - first) + 1;
    seq_len[e] = inside && len > 0 && len < (int64_t{1} << 31) ? static_cast<int32_t>(len) : 0;
    seq_of[e] = lo;
  }
}

}  // namespace

cudaError_t launch_prefill_entries(const int32_t* q_start, const int32_t* q_pos, int batch, int total_q,
                                   int32_t* seq_len, int32_t* seq_of, cudaStream_t stream) {
  if (total_q == 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = (total_q + threads - 1) / threads < 1024 ? (total_q + threads - 1) / threads : 1024;
  return launch_overlapped(prefill_entries_kernel, dim3(blocks), dim3(threads), 0, stream, q_start, q_pos, batch,
                           total_q, seq_len, seq_of);
}

}  // namespace nosa
