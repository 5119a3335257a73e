// Launch interfaces of the three NOSA kernels (internal to the library).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nosa {

struct PoolArgs {
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
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
  const int64_t* seq_start;
  const int32_t* seq_len;
  const int32_t* sel_idx;
  const int32_t* sel_cnt;
  __nv_bfloat16* out;
  float* lse;        // nullable
  float* part;       // [pairs, kMaxSplits, group*(128+2)] partial softmax state
  uint32_t* tickets; // [pairs]
  uint32_t* status;
  int batch, hq, hkv, group, local_blocks, topk, max_seq_len;
  int nsplit, tiles_per_split;
  float scale_log2;  // softmax scale * log2(e)
};

cudaError_t launch_pool_append(const PoolArgs& a, cudaStream_t stream);
cudaError_t launch_block_select(const SelectArgs& a, cudaStream_t stream);
cudaError_t launch_sparse_decode(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint32_t* status, uint32_t max_iters, cudaStream_t stream);

// Number of splits and tiles per split that launch_sparse_decode will use.
void decode_split_plan(int pairs, int max_tiles, int num_sms, int* nsplit, int* tiles_per_split);

}  // namespace nosa
