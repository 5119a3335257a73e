// Launch interfaces of the three NOSA kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "nosa.h"

namespace nosa {

struct PoolArgs {
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  int64_t cache_rows;
  const int64_t* seq_start;
  const int32_t* len_old;  // nullable: len_new - 1
  const int32_t* len_new;
  float* pooled;
  const __nv_bfloat16* k_new;  // nullable
  const __nv_bfloat16* v_new;
  uint32_t* status;            // nullable
  int batch, hkv, nc_cap, max_new_keys;
};

struct SelectArgs {
  const __nv_bfloat16* q;
  const float* pooled;
  const int32_t* seq_len;
  const float* bs_in;      // nullable: selection only
  float* comp_out;         // nullable
  float* bs_out;           // nullable
  int32_t* sel_idx;
  int32_t* sel_cnt;
  float* bscratch;         // [pairs, nb_ws] block scores of the scoring pass
  uint32_t* tickets;       // [pairs]
  uint32_t* status;
  int batch, hq, hkv, group, local_blocks, topk, max_seq_len;
  int nc_cap, nb_in, nb_out, nb_ws;
  float scale;
};

struct DecodeArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_cache;
  const __nv_bfloat16* v_cache;
  int64_t cache_rows;
  const int64_t* seq_start;
  const int32_t* seq_len;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  __nv_bfloat16* out;
  float* lse;        // nullable
  float* part;       // [pairs, kMaxSplits, part_stride(group)] partial softmax state
  uint32_t* tickets; // [pairs]
  uint32_t* status;
  int batch, hq, hkv, group, local_blocks, topk, max_seq_len;
  int nsplit;
  float scale_log2;  // softmax scale * log2(e)
};

// Work mix of one launch of the persistent step kernel.
constexpr int kStepScore = 1;   // scoring items (+ top-k of each pair)
constexpr int kStepDecode = 2;  // decode items
constexpr int kStepAppend = 4;  // the first scoring item of a pair appends the new token and pools

struct StepArgs {
  SelectArgs sel;
  DecodeArgs dec;
  PoolArgs pool;
  uint32_t* work;   // [2]: queue position, CTAs finished (zero between launches)
  uint32_t* ready;  // [pairs]: selection published (zero between launches)
  int mode, pairs, n_score_items, n_items;
};

// Launches `kernel` with programmatic stream serialization, so that it can be
// scheduled while the previous kernel on `stream` finishes (the kernels wait
// on the dependency themselves before touching global memory).
template <typename... KArgs, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

cudaError_t launch_pool_append(const PoolArgs& a, cudaStream_t stream);
cudaError_t launch_step(const StepArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v, cudaStream_t stream);
cudaError_t launch_select_only(const SelectArgs& a, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint32_t* status, uint32_t max_iters, cudaStream_t stream);

// Bytes at the start of a workspace that must be zero before a call
// (status word, work queue, tickets, ready flags); 0 for invalid parameters.
size_t workspace_counter_bytes(const nosa_params* p, int batch, int max_seq_len);

// Records `msg` as the calling thread's last error and returns `code`.
int record_error(int code, const char* msg);

// CTAs of the step kernel that fit on the current device at once.
int step_resident_ctas(int group);

// Splits per (sequence, KV head) for the decode items: about one item per
// resident CTA, at most one per tile and kMaxSplits.
void decode_split_plan(int pairs, int max_tiles, int num_ctas, int* nsplit);

}  // namespace nosa
