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
  const int64_t* seq_start;    // contiguous caches (nullptr when paged)
  const int32_t* page_table;   // paged caches: [batch, max_pages] 64-token page indices (nullptr: contiguous)
  int max_pages;
  const int32_t* len_old;  // nullable: len_new - 1
  const int32_t* len_new;
  void* pooled;                // fp32, or bf16 when pooled_bf16
  const __nv_bfloat16* k_new;  // nullable
  const __nv_bfloat16* v_new;
  uint32_t* status;            // nullable
  int batch, hkv, nc_cap, max_new_keys;
  int pooled_bf16;
  int kv_int8;                 // INT8 caches: k_cache / v_cache hold int8 codes, scales below
  float* k_scale;              // [hkv, scale_stride] (INT8 caches)
  float* v_scale;
  int64_t scale_stride;
};

struct SelectArgs {  // selection from given block scores (select_only_kernel)
  const int32_t* seq_len;
  const float* bs_in;      // [pairs, nb_in]
  int32_t* sel_idx;
  int32_t* sel_cnt;
  uint32_t* status;
  int batch, hkv, local_blocks, topk, max_seq_len, nb_in;
};

// Work of one launch of the decode-step kernel (any of the three parts).
constexpr int kStepScore = 1;   // compressed scores, block scores and top-k of every pair
constexpr int kStepDecode = 2;  // attention over the local window and the selected blocks
constexpr int kStepAppend = 4;  // write the new token's K/V rows and pool the window it completes

struct StepArgs {
  const __nv_bfloat16* q;        // [batch, hq, 128]
  const int32_t* seq_len;        // [batch]
  const int32_t* seq_of;         // nullable: [batch] sequence of each entry (multi-query prefill); else entry i
                                 // is sequence i.  seq_start / page_table / pooled rows are per sequence.
  const int64_t* seq_start;      // [sequences] (decode / append, contiguous caches; nullptr when paged)
  const int32_t* page_table;     // [batch, max_pages] (paged caches; nullptr: contiguous)
  int max_pages;
  int64_t cache_rows;
  __nv_bfloat16* k_cache;        // [cache_rows, hkv, 128] (append writes; tiles come through tensor maps)
  __nv_bfloat16* v_cache;
  void* pooled;                  // [batch, hkv, nc_cap, 128] fp32 or bf16 (append writes; scoring reads
                                 // through a tensor map)
  const __nv_bfloat16* k_new;    // [batch, hkv, 128], nullable (append)
  const __nv_bfloat16* v_new;
  int32_t* sel_idx;              // [pairs, topk]: written when scoring, read otherwise
  int32_t* sel_cnt;              // [pairs]
  float* comp_out;               // nullable: [batch, hq, nc_cap] compressed scores
  float* bs_out;                 // nullable: [pairs, nb_out] block scores
  float* bs_spill;               // nullable: [pairs, nb_spill] block scores kept in global memory
  __nv_bfloat16* out;            // [batch, hq, 128] (decode)
  float* lse;                    // nullable: [batch, hq]
  uint32_t* status;
  int batch, hq, hkv, local_blocks, topk, max_seq_len, nc_cap, nb_out, nb_spill;
  int ncand_max;  // candidates of a sequence of max_seq_len tokens
  int pooled_bf16;
  int kv_int8;         // INT8 caches: k_cache / v_cache hold int8 codes [cache_rows, hkv, 128]
  float* k_scale;      // [hkv, scale_stride] per-row scales (INT8 caches)
  float* v_scale;
  int64_t scale_stride;
  int mode;
  float scale;       // softmax scale
  float scale_log2;  // softmax scale * log2(e)
};

// Attention of the sparse prefill over query groups (prefill_attn.cu).
struct PrefillAttnArgs {
  const __nv_bfloat16* q;     // [total_q, hq, 128]
  const int32_t* entry_len;   // [total_q] L of each entry (position + 1)
  const int32_t* entry_seq;   // [total_q] sequence of each entry
  const int64_t* seq_start;   // [sequences] first cache row (contiguous caches; nullptr when paged)
  const int32_t* page_table;  // [sequences, max_pages] 64-token pages (paged caches; nullptr: contiguous)
  int max_pages;
  int64_t cache_rows;
  const int32_t* sel_idx;     // [total_q, hkv, topk]
  const int32_t* sel_cnt;     // [total_q, hkv]
  __nv_bfloat16* out;         // [total_q, hq, 128]
  float* lse;                 // nullable: [total_q, hq]
  uint32_t* status;
  int total_q, hq, hkv, topk, local_blocks, max_seq_len;
  int nb_words;               // 32-bit words of a block bitmap: ceil(nb(max_seq_len) / 32)
  float scale_log2;
};

// Sequences up to this many blocks (256K tokens) use the grouped prefill
// attention; longer ones run every entry through the step kernel.
constexpr int kPrefillMaxBlocks = 4096;

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
// Tensor maps of one step launch: K and V tiles, pooled keys, and (INT8
// caches) the K and V scale rows.
struct StepMaps {
  CUtensorMap k, v, p, ks, vs;
};
cudaError_t launch_step(const StepArgs& a, const StepMaps& maps, cudaStream_t stream);
// Entries of a multi-query prefill: for sequence s with query rows
// [q_start[s], q_start[s+1]) at positions q_pos[s] + r, entry e = q_start[s]
// + r gets seq_len[e] = q_pos[s] + r + 1 and seq_of[e] = s.
cudaError_t launch_prefill_entries(const int32_t* q_start, const int32_t* q_pos, int batch, int total_q,
                                   int32_t* seq_len, int32_t* seq_of, cudaStream_t stream);
cudaError_t launch_prefill_attn(const PrefillAttnArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                cudaStream_t stream);
cudaError_t launch_quantize_int8(const __nv_bfloat16* src, int8_t* codes, float* scales, int64_t scale_stride,
                                 int64_t row0, int64_t rows, int hkv, cudaStream_t stream);
cudaError_t launch_select_only(const SelectArgs& a, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint32_t* status, uint32_t max_iters, cudaStream_t stream);

// Block scores of a pair stay in shared memory up to this many candidates
// (64 * 2048 tokens before the local window); beyond, they live in a
// workspace region of pairs x candidates floats.
constexpr int kSmemBlockScores = 2048;

// Bytes at the start of a workspace that must be zero before a call (the
// device status word); 0 for invalid parameters.
size_t workspace_counter_bytes(const nosa_params* p, int batch, int max_seq_len);

// Records `msg` as the calling thread's last error and returns `code`.
int record_error(int code, const char* msg);

// The host checks of nosa_decode_step_device except the workspace's (a
// status code, recorded as the last error; nothing is enqueued).
int check_decode_step_device(const nosa_params* p, const void* q, const void* k_new, const void* v_new,
                             const void* k_cache, const void* v_cache, int64_t cache_rows, const int64_t* seq_start,
                             const int32_t* seq_len, int batch, int max_seq_len, const void* pooled, int nc_cap,
                             const int32_t* sel_idx, const int32_t* sel_cnt, const void* out);

}  // namespace nosa
