// Host side of the C ABI declared in include/nosa.h: argument checks,
// workspace layout, launch planning and the host-buffer decode step.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include <cudaTypedefs.h>

#include "nosa.h"
#include "nosa_common.cuh"
#include "nosa_kernels.h"
#include "decode_device.cuh"
#include "kv_int8.cuh"
#include "select_device.cuh"

namespace {

thread_local std::string g_last_error;
thread_local uint32_t g_last_bits = 0;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return NOSA_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(NOSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_params(const nosa_params* p) {
  if (!p) return fail(NOSA_ERR_INVALID_ARG, "params is NULL");
  if (p->num_kv_heads < 1 || p->num_q_heads < 1 || p->num_q_heads % p->num_kv_heads != 0)
    return fail(NOSA_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                p->num_q_heads, p->num_kv_heads);
  const int G = p->num_q_heads / p->num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
    return fail(NOSA_ERR_UNSUPPORTED, "GQA group size %d not supported (1, 2, 4, 8 or 16)", G);
  if (p->head_dim != nosa::kHeadDim)
    return fail(NOSA_ERR_UNSUPPORTED, "head_dim %d not supported (128)", p->head_dim);
  if (p->pool_kernel != nosa::kPoolKernel || p->pool_stride != nosa::kPoolStride)
    return fail(NOSA_ERR_UNSUPPORTED, "pooling kernel/stride %d/%d not supported (32/16)",
                p->pool_kernel, p->pool_stride);
  if (p->block_size != nosa::kBlock)
    return fail(NOSA_ERR_UNSUPPORTED, "block_size %d not supported (64)", p->block_size);
  if (p->local_blocks < 0) return fail(NOSA_ERR_INVALID_ARG, "local_blocks < 0");
  if (p->local_blocks > nosa::kMaxLocalBlocks)
    return fail(NOSA_ERR_UNSUPPORTED, "local_blocks %d above %d", p->local_blocks, nosa::kMaxLocalBlocks);
  if (p->topk < 1 || p->topk > 1024) return fail(NOSA_ERR_UNSUPPORTED, "topk %d outside 1..1024", p->topk);
  if (!(p->softmax_scale >= 0.0f) || std::isinf(p->softmax_scale))
    return fail(NOSA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  if (p->pooled_bf16 != 0 && p->pooled_bf16 != 1) return fail(NOSA_ERR_INVALID_ARG, "pooled_bf16 must be 0 or 1");
  if (p->kv_int8 != 0 && p->kv_int8 != 1) return fail(NOSA_ERR_INVALID_ARG, "kv_int8 must be 0 or 1");
  return NOSA_OK;
}

// The scale rows of an INT8 cache buffer (codes first, then scales).
float* int8_scales(const void* cache, int64_t cache_rows, int hkv) {
  return reinterpret_cast<float*>(static_cast<uint8_t*>(const_cast<void*>(cache)) +
                                  nosa::int8_scale_offset(cache_rows, hkv));
}

float scale_of(const nosa_params* p) {
  return p->softmax_scale > 0.0f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(p->head_dim));
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout (all offsets 256-byte aligned): the device status word;
// block scores that do not fit in shared memory (pairs x candidates, only
// when a sequence may have more than kSmemBlockScores candidates); staging
// buffers of the host-buffer step (q, new K/V rows, out).
struct Layout {
  size_t status, spill, stage_q, stage_k, stage_v, stage_out, total;
  size_t entry_len, entry_seq;  // sparse prefill: per-entry lengths and sequence indices (int32)
  int nb_spill;  // candidates per pair in `spill` (0: block scores stay in shared memory)
};

Layout layout_of(const nosa_params* p, int batch, int max_seq_len) {
  Layout l{};
  const size_t pairs = static_cast<size_t>(batch) * p->num_kv_heads;
  const int64_t ncand_max = nosa::n_candidates(max_seq_len, p->local_blocks);
  l.nb_spill = ncand_max > nosa::kSmemBlockScores ? static_cast<int>(ncand_max) : 0;
  size_t off = 0;
  l.status = off;  // uint32 device status word
  off += 256;
  l.spill = off;
  off = round_up(off + pairs * static_cast<size_t>(l.nb_spill) * 4, 256);
  const size_t qbytes = static_cast<size_t>(batch) * p->num_q_heads * nosa::kHeadDim * 2;
  const size_t kvbytes = pairs * nosa::kHeadDim * 2;
  l.stage_q = off;
  off = round_up(off + qbytes, 256);
  l.stage_k = off;
  off = round_up(off + kvbytes, 256);
  l.stage_v = off;
  off = round_up(off + kvbytes, 256);
  l.stage_out = off;
  off = round_up(off + qbytes, 256);
  l.total = off;
  return l;
}

// Workspace of a sparse prefill over `total_q` query entries: the status
// word, spilled block scores per entry, the entries' lengths and sequences
// (no host-buffer staging).
Layout prefill_layout_of(const nosa_params* p, int total_q, int max_seq_len) {
  Layout l{};
  const size_t pairs = static_cast<size_t>(total_q) * p->num_kv_heads;
  const int64_t ncand_max = nosa::n_candidates(max_seq_len, p->local_blocks);
  l.nb_spill = ncand_max > nosa::kSmemBlockScores ? static_cast<int>(ncand_max) : 0;
  size_t off = 0;
  l.status = off;
  off += 256;
  l.spill = off;
  off = round_up(off + pairs * static_cast<size_t>(l.nb_spill) * 4, 256);
  l.entry_len = off;
  off = round_up(off + static_cast<size_t>(total_q) * 4, 256);
  l.entry_seq = off;
  off = round_up(off + static_cast<size_t>(total_q) * 4, 256);
  l.total = off;
  return l;
}

int check_ws(void* ws, size_t ws_bytes, const Layout& l) {
  if (!ws) return fail(NOSA_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned(ws, 256)) return fail(NOSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < l.total)
    return fail(NOSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, l.total);
  return NOSA_OK;
}


// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

// Recently encoded tensor maps of this host thread: a step re-encodes the
// same K, V and pooled maps every call, and encoding costs microseconds of
// host time per map.  Keyed by everything the encoding depends on.
struct MapKey {
  const void* base;
  int64_t a, b;
  int kind;
  bool operator==(const MapKey& o) const { return base == o.base && a == o.a && b == o.b && kind == o.kind; }
};
struct MapCache {
  static constexpr int kSlots = 16;
  MapKey key[kSlots] = {};
  CUtensorMap map[kSlots];
  int next = 0;
  const CUtensorMap* find(const MapKey& k) const {
    for (int x = 0; x < kSlots; ++x)
      if (key[x].base && key[x] == k) return &map[x];
    return nullptr;
  }
  void put(const MapKey& k, const CUtensorMap& m) {
    key[next] = k;
    map[next] = m;
    next = (next + 1) % kSlots;
  }
};
thread_local MapCache g_maps;

// 3-D map over a [rows, hkv, 128] cache: bf16 boxes of {64 dims, 1 head,
// 64 tokens}, or INT8 boxes of {128 codes, 1 head, 64 tokens}; 128-byte rows
// with the 128-byte swizzle, zero fill past `rows`.
int encode_kv_map(CUtensorMap* map, const void* base, int hkv, int64_t rows, bool int8) {
  const MapKey key{base, hkv, rows, int8 ? 1 : 0};
  if (const CUtensorMap* hit = g_maps.find(key)) {
    *map = *hit;
    return NOSA_OK;
  }
  auto enc = tensor_map_encoder();
  if (!enc) return fail(NOSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t esize = int8 ? 1 : 2;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(nosa::kHeadDim), static_cast<cuuint64_t>(hkv),
                              static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(nosa::kHeadDim) * esize,
                                 static_cast<cuuint64_t>(hkv) * nosa::kHeadDim * esize};
  const cuuint32_t box[3] = {int8 ? 128u : 64u, 1, static_cast<cuuint32_t>(nosa::kBlock)};
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = enc(map, int8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                   const_cast<void*>(base), dims, strides, box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NOSA_ERR_INVALID_ARG, "tensor map encode failed (code %d)", static_cast<int>(r));
  g_maps.put(key, *map);
  return NOSA_OK;
}

// 2-D map over the scale rows of an INT8 cache, fp32 [hkv, stride]: boxes of
// 68 consecutive tokens of one head (a tile's 64 scales from the 16-byte
// aligned token at or below its first row), no swizzle, zero fill past the
// row.
int encode_scale_map(CUtensorMap* map, const void* cache, int hkv, int64_t rows) {
  const MapKey key{cache, hkv, rows, 2};
  if (const CUtensorMap* hit = g_maps.find(key)) {
    *map = *hit;
    return NOSA_OK;
  }
  auto enc = tensor_map_encoder();
  if (!enc) return fail(NOSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const int64_t stride = nosa::int8_scale_stride(rows);
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(stride), static_cast<cuuint64_t>(hkv)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride) * 4};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(nosa::kScaleBox), 1};
  const cuuint32_t elem_strides[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, int8_scales(cache, rows, hkv), dims, strides, box,
                   elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NOSA_ERR_INVALID_ARG, "scale tensor map encode failed (code %d)", static_cast<int>(r));
  g_maps.put(key, *map);
  return NOSA_OK;
}

// The cache maps of a decode launch (K, V and, for INT8 caches, their
// scale rows).
int encode_cache_maps(nosa::StepMaps* m, const nosa_params* p, const void* k_cache, const void* v_cache,
                      int64_t rows) {
  const bool int8 = p->kv_int8 != 0;
  if (int rc = encode_kv_map(&m->k, k_cache, p->num_kv_heads, rows, int8)) return rc;
  if (int rc = encode_kv_map(&m->v, v_cache, p->num_kv_heads, rows, int8)) return rc;
  if (int8) {
    if (int rc = encode_scale_map(&m->ks, k_cache, p->num_kv_heads, rows)) return rc;
    if (int rc = encode_scale_map(&m->vs, v_cache, p->num_kv_heads, rows)) return rc;
  }
  return NOSA_OK;
}

// INT8 fields of the kernel arguments.
template <typename Args>
void set_int8(Args& a, const nosa_params* p, void* k_cache, const void* v_cache, int64_t rows) {
  a.kv_int8 = p->kv_int8;
  if (p->kv_int8) {
    a.k_scale = k_cache ? int8_scales(k_cache, rows, p->num_kv_heads) : nullptr;
    a.v_scale = v_cache ? int8_scales(v_cache, rows, p->num_kv_heads) : nullptr;
    a.scale_stride = nosa::int8_scale_stride(rows);
  }
}

// 2-D map over the pooled keys [batch * hkv * nc_cap rows, 128 fp32 or bf16]:
// boxes of 128-byte rows ({32 fp32 or 64 bf16 columns, 61 rows}: one slice of
// one scoring chunk), 128-byte swizzle, zero fill past the last row.
int encode_pooled_map(CUtensorMap* map, const void* pooled, int batch, int hkv, int nc_cap, bool bf16) {
  const MapKey key{pooled, static_cast<int64_t>(batch) * hkv, nc_cap, bf16 ? 4 : 3};
  if (const CUtensorMap* hit = g_maps.find(key)) {
    *map = *hit;
    return NOSA_OK;
  }
  auto enc = tensor_map_encoder();
  if (!enc) return fail(NOSA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t rows = static_cast<cuuint64_t>(batch) * hkv * nc_cap;
  // TMA row coordinates are signed 32-bit.
  if (rows >= (cuuint64_t{1} << 31)) return fail(NOSA_ERR_UNSUPPORTED, "batch * num_kv_heads * nc_cap must be below 2^31");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(nosa::kHeadDim), rows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(nosa::kHeadDim) * (bf16 ? 2 : 4)};
  // 128-byte box rows: 32 fp32 or 64 bf16 columns.
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(bf16 ? 64 : nosa::kBoxCols),
                             static_cast<cuuint32_t>(nosa::kBoxRows)};
  const cuuint32_t elem_strides[2] = {1, 1};
  CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                   const_cast<void*>(pooled), dims, strides, box,
                   elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NOSA_ERR_INVALID_ARG, "pooled tensor map encode failed (code %d)", static_cast<int>(r));
  g_maps.put(key, *map);
  return NOSA_OK;
}

// Where sequences live in the K/V caches: contiguous rows from seq_start[i],
// or 64-token pages through page_table[i * max_pages + block].
struct KvLayout {
  const int64_t* seq_start;
  const int32_t* page_table;
  int max_pages;
};

int check_layout(const KvLayout& kv, int64_t cache_rows) {
  if ((kv.seq_start == nullptr) == (kv.page_table == nullptr))
    return fail(NOSA_ERR_INVALID_ARG, "exactly one of seq_start and page_table must be given");
  if (kv.page_table) {
    if (kv.max_pages < 1) return fail(NOSA_ERR_INVALID_ARG, "max_pages must be >= 1");
    if (!aligned(kv.page_table, 4)) return fail(NOSA_ERR_INVALID_ARG, "page_table must be 4-byte aligned");
    if (cache_rows % nosa::kPageTokens != 0)
      return fail(NOSA_ERR_INVALID_ARG, "a paged cache holds whole 64-token pages");
  }
  return NOSA_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

int do_pool_append(const nosa_params* p, void* k_cache, void* v_cache, int64_t cache_rows, const KvLayout& kvl,
                   const int32_t* len_old, const int32_t* len_new, int batch, void* pooled, int nc_cap,
                   int max_new_keys, const void* k_new, const void* v_new, uint32_t* status,
                   cudaStream_t stream) {
  if (batch < 0 || nc_cap < 0 || max_new_keys < 0 || cache_rows < 0)
    return fail(NOSA_ERR_INVALID_ARG, "batch, nc_cap, max_new_keys and cache_rows must be >= 0");
  if (batch == 0) return ok();
  if (!k_cache || !len_new || !pooled)
    return fail(NOSA_ERR_INVALID_ARG, "k_cache, len_new and pooled must not be NULL");
  if (int rc = check_layout(kvl, cache_rows)) return rc;
  if ((k_new == nullptr) != (v_new == nullptr))
    return fail(NOSA_ERR_INVALID_ARG, "k_new and v_new must both be given or both be NULL");
  if (k_new && !v_cache) return fail(NOSA_ERR_INVALID_ARG, "v_cache must not be NULL when appending");
  if (!aligned(k_cache, 16) || !aligned(pooled, 16) || (v_cache && !aligned(v_cache, 16)) ||
      (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16))))
    return fail(NOSA_ERR_INVALID_ARG, "cache, pooled and new-row pointers must be 16-byte aligned");
  if (static_cast<int64_t>(batch) * p->num_kv_heads > 65535)
    return fail(NOSA_ERR_UNSUPPORTED, "batch * num_kv_heads above 65535");
  nosa::PoolArgs a{};
  a.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  a.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  a.cache_rows = cache_rows;
  a.seq_start = kvl.seq_start;
  a.page_table = kvl.page_table;
  a.max_pages = kvl.max_pages;
  a.len_old = len_old;
  a.len_new = len_new;
  a.pooled = pooled;
  a.pooled_bf16 = p->pooled_bf16;
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.status = status;
  a.batch = batch;
  a.hkv = p->num_kv_heads;
  a.nc_cap = nc_cap;
  a.max_new_keys = max_new_keys;
  set_int8(a, p, k_cache, v_cache, cache_rows);
  cudaError_t e = nosa::launch_pool_append(a, stream);
  if (e != cudaSuccess) return cuda_fail(e, "pool_append launch");
  return ok();
}

// Arguments of the step kernel common to its three uses.
nosa::StepArgs step_args(const nosa_params* p, const void* q, const int32_t* seq_len, int batch, int max_seq_len,
                         int32_t* sel_idx, int32_t* sel_cnt, void* ws, const Layout& l) {
  nosa::StepArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.seq_len = seq_len;
  a.sel_idx = sel_idx;
  a.sel_cnt = sel_cnt;
  a.bs_spill = l.nb_spill > 0 ? at<float>(ws, l.spill) : nullptr;
  a.nb_spill = l.nb_spill;
  a.status = at<uint32_t>(ws, l.status);
  a.batch = batch;
  a.hq = p->num_q_heads;
  a.hkv = p->num_kv_heads;
  a.local_blocks = p->local_blocks;
  a.topk = p->topk;
  a.max_seq_len = max_seq_len;
  a.ncand_max = static_cast<int>(nosa::n_candidates(max_seq_len, p->local_blocks));
  a.pooled_bf16 = p->pooled_bf16;
  a.nc_cap = 1;
  a.scale = scale_of(p);
  a.scale_log2 = a.scale * 1.4426950408889634f;
  return a;
}

int check_common(const nosa_params* p, int batch, int max_seq_len) {
  if (batch < 0 || max_seq_len < 1) return fail(NOSA_ERR_INVALID_ARG, "batch >= 0 and max_seq_len >= 1 required");
  if (static_cast<int64_t>(batch) * p->num_kv_heads > (1 << 20))
    return fail(NOSA_ERR_UNSUPPORTED, "batch * num_kv_heads above 2^20");
  if (max_seq_len > (1 << 30)) return fail(NOSA_ERR_UNSUPPORTED, "max_seq_len above 2^30");
  return NOSA_OK;
}

int do_block_select(const nosa_params* p, const void* q, const void* pooled, int nc_cap,
                    const int32_t* seq_len, int batch, int max_seq_len, const float* bs_in, int nb_in,
                    float* comp_out, float* bs_out, int nb_out, int32_t* sel_idx, int32_t* sel_cnt,
                    void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (int rc = check_common(p, batch, max_seq_len)) return rc;
  if (batch == 0) return ok();
  const Layout l = layout_of(p, batch, max_seq_len);
  if (int rc = check_ws(ws, ws_bytes, l)) return rc;
  if (!seq_len || !sel_idx || !sel_cnt) return fail(NOSA_ERR_INVALID_ARG, "seq_len, sel_idx and sel_cnt must not be NULL");
  const int ncand_max = static_cast<int>(nosa::n_candidates(max_seq_len, p->local_blocks));
  if (bs_in) {
    if (nb_in < ncand_max)
      return fail(NOSA_ERR_INVALID_ARG, "nb_cap_in %d below the %d candidates of max_seq_len", nb_in, ncand_max);
    if (static_cast<int64_t>(batch) * p->num_kv_heads > 65535)
      return fail(NOSA_ERR_UNSUPPORTED, "batch * num_kv_heads above 65535");
    if (static_cast<int64_t>(nb_in) * 4 > 200 * 1024)
      return fail(NOSA_ERR_UNSUPPORTED, "nb_cap_in %d above the selector's shared memory", nb_in);
    nosa::SelectArgs a{};
    a.seq_len = seq_len;
    a.bs_in = bs_in;
    a.sel_idx = sel_idx;
    a.sel_cnt = sel_cnt;
    a.status = at<uint32_t>(ws, l.status);
    a.batch = batch;
    a.hkv = p->num_kv_heads;
    a.local_blocks = p->local_blocks;
    a.topk = p->topk;
    a.max_seq_len = max_seq_len;
    a.nb_in = nb_in;
    cudaError_t e = nosa::launch_select_only(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "block_select launch");
    return ok();
  }
  if (!q || !pooled) return fail(NOSA_ERR_INVALID_ARG, "q and pooled must not be NULL when scoring");
  if (!aligned(pooled, 16) || !aligned(q, 8)) return fail(NOSA_ERR_INVALID_ARG, "pooled must be 16-byte and q 8-byte aligned");
  if (nc_cap < 1) return fail(NOSA_ERR_INVALID_ARG, "nc_cap must be >= 1");
  if (bs_out && nb_out < ncand_max)
    return fail(NOSA_ERR_INVALID_ARG, "nb_cap_out %d below the %d candidates of max_seq_len", nb_out, ncand_max);
  nosa::StepArgs s = step_args(p, q, seq_len, batch, max_seq_len, sel_idx, sel_cnt, ws, l);
  s.pooled = const_cast<void*>(pooled);
  s.nc_cap = nc_cap;
  s.comp_out = comp_out;
  s.bs_out = bs_out;
  s.nb_out = nb_out;
  s.mode = nosa::kStepScore;
  nosa::StepMaps maps;
  memset(&maps, 0, sizeof maps);
  if (int rc = encode_pooled_map(&maps.p, pooled, batch, p->num_kv_heads, nc_cap, p->pooled_bf16 != 0)) return rc;
  cudaError_t e = nosa::launch_step(s, maps, stream);
  if (e != cudaSuccess) return cuda_fail(e, "block_select launch");
  return ok();
}

int check_decode_ptrs(const void* q, const void* k_cache, const void* v_cache, int64_t cache_rows,
                      const KvLayout& kvl, const int32_t* seq_len, const int32_t* sel_idx,
                      const int32_t* sel_cnt, const void* out) {
  if (!q || !k_cache || !v_cache || !seq_len || !sel_idx || !sel_cnt || !out)
    return fail(NOSA_ERR_INVALID_ARG, "q, caches, seq_len, sel_idx, sel_cnt and out must not be NULL");
  if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 8))
    return fail(NOSA_ERR_INVALID_ARG, "caches must be 16-byte and q 8-byte aligned");
  if (cache_rows < 1 || cache_rows >= (int64_t{1} << 31))
    return fail(NOSA_ERR_UNSUPPORTED, "cache_rows must be in [1, 2^31)");
  return check_layout(kvl, cache_rows);
}

int do_sparse_decode(const nosa_params* p, const void* q, const void* k_cache, const void* v_cache,
                     int64_t cache_rows, const KvLayout& kvl, const int32_t* seq_len, int batch, int max_seq_len,
                     const int32_t* sel_idx, const int32_t* sel_cnt, void* out, float* lse, void* ws,
                     size_t ws_bytes, cudaStream_t stream) {
  if (int rc = check_common(p, batch, max_seq_len)) return rc;
  if (batch == 0) return ok();
  const Layout l = layout_of(p, batch, max_seq_len);
  if (int rc = check_ws(ws, ws_bytes, l)) return rc;
  if (int rc = check_decode_ptrs(q, k_cache, v_cache, cache_rows, kvl, seq_len, sel_idx, sel_cnt, out)) return rc;
  nosa::StepArgs s = step_args(p, q, seq_len, batch, max_seq_len, const_cast<int32_t*>(sel_idx),
                               const_cast<int32_t*>(sel_cnt), ws, l);
  s.seq_start = kvl.seq_start;
  s.page_table = kvl.page_table;
  s.max_pages = kvl.max_pages;
  s.cache_rows = cache_rows;
  s.out = static_cast<__nv_bfloat16*>(out);
  s.lse = lse;
  s.mode = nosa::kStepDecode;
  set_int8(s, p, const_cast<void*>(k_cache), v_cache, cache_rows);
  nosa::StepMaps maps;
  memset(&maps, 0, sizeof maps);
  if (int rc = encode_cache_maps(&maps, p, k_cache, v_cache, cache_rows)) return rc;
  cudaError_t e = nosa::launch_step(s, maps, stream);
  if (e != cudaSuccess) return cuda_fail(e, "sparse_decode launch");
  return ok();
}

// Buffer checks of the fused step (everything but the workspace).
int check_step_buffers(const void* q, const void* k_new, const void* v_new, const void* k_cache, const void* v_cache,
                       int64_t cache_rows, const KvLayout& kvl, const int32_t* seq_len, const void* pooled, int nc_cap,
                       const int32_t* sel_idx, const int32_t* sel_cnt, const void* out) {
  if (int rc = check_decode_ptrs(q, k_cache, v_cache, cache_rows, kvl, seq_len, sel_idx, sel_cnt, out)) return rc;
  if (!pooled || nc_cap < 1) return fail(NOSA_ERR_INVALID_ARG, "pooled must not be NULL and nc_cap >= 1");
  if (!aligned(pooled, 16)) return fail(NOSA_ERR_INVALID_ARG, "pooled must be 16-byte aligned");
  if ((k_new == nullptr) != (v_new == nullptr))
    return fail(NOSA_ERR_INVALID_ARG, "k_new and v_new must both be given or both be NULL");
  if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16)))
    return fail(NOSA_ERR_INVALID_ARG, "new-row pointers must be 16-byte aligned");
  return NOSA_OK;
}

// The fused step on device buffers: one launch appends, pools, selects and
// attends.  Needs at least two local blocks (then the window a new token
// completes is never read by the same step's selection); otherwise the three
// separate launches run.
int do_decode_step_device(const nosa_params* p, const void* q, const void* k_new, const void* v_new, void* k_cache,
                          void* v_cache, int64_t cache_rows, const KvLayout& kvl, const int32_t* seq_len,
                          int batch, int max_seq_len, void* pooled, int nc_cap, int32_t* sel_idx, int32_t* sel_cnt,
                          void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (int rc = check_common(p, batch, max_seq_len)) return rc;
  if (batch == 0) return ok();
  const Layout l = layout_of(p, batch, max_seq_len);
  if (int rc = check_ws(ws, ws_bytes, l)) return rc;
  if (int rc = check_step_buffers(q, k_new, v_new, k_cache, v_cache, cache_rows, kvl, seq_len, pooled, nc_cap,
                                  sel_idx, sel_cnt, out))
    return rc;
  if (p->local_blocks < 2) {
    int rc = do_pool_append(p, k_cache, v_cache, cache_rows, kvl, nullptr, seq_len, batch, pooled, nc_cap, 1,
                            k_new, v_new, at<uint32_t>(ws, l.status), stream);
    if (!rc) rc = do_block_select(p, q, pooled, nc_cap, seq_len, batch, max_seq_len, nullptr, 0, nullptr, nullptr, 0,
                                  sel_idx, sel_cnt, ws, ws_bytes, stream);
    if (!rc) rc = do_sparse_decode(p, q, k_cache, v_cache, cache_rows, kvl, seq_len, batch, max_seq_len,
                                   sel_idx, sel_cnt, out, lse, ws, ws_bytes, stream);
    return rc;
  }
  nosa::StepArgs s = step_args(p, q, seq_len, batch, max_seq_len, sel_idx, sel_cnt, ws, l);
  s.seq_start = kvl.seq_start;
  s.page_table = kvl.page_table;
  s.max_pages = kvl.max_pages;
  s.cache_rows = cache_rows;
  s.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  s.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  s.pooled = pooled;
  s.nc_cap = nc_cap;
  s.k_new = static_cast<const __nv_bfloat16*>(k_new);
  s.v_new = static_cast<const __nv_bfloat16*>(v_new);
  s.out = static_cast<__nv_bfloat16*>(out);
  s.lse = lse;
  s.mode = nosa::kStepScore | nosa::kStepDecode | nosa::kStepAppend;
  set_int8(s, p, k_cache, v_cache, cache_rows);
  nosa::StepMaps maps;
  memset(&maps, 0, sizeof maps);
  if (int rc = encode_cache_maps(&maps, p, k_cache, v_cache, cache_rows)) return rc;
  if (int rc = encode_pooled_map(&maps.p, pooled, batch, p->num_kv_heads, nc_cap, p->pooled_bf16 != 0)) return rc;
  cudaError_t e = nosa::launch_step(s, maps, stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode_step launch");
  return ok();
}

// Sparse prefill (NOSAS): every query row of every sequence is one entry of
// the step kernel (selection + attention, no append) with its own length
// (position + 1), reading its sequence's cache and pooled keys.
int do_sparse_prefill(const nosa_params* p, const void* q, const void* k_cache, const void* v_cache,
                      int64_t cache_rows, const KvLayout& kvl, const int32_t* q_start, const int32_t* q_pos,
                      int batch, int total_q, int max_seq_len, const void* pooled, int nc_cap, int32_t* sel_idx,
                      int32_t* sel_cnt, void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (int rc = check_common(p, total_q, max_seq_len)) return rc;
  if (batch < 1) return fail(NOSA_ERR_INVALID_ARG, "batch must be >= 1");
  if (total_q == 0) return ok();
  const Layout l = prefill_layout_of(p, total_q, max_seq_len);
  if (int rc = check_ws(ws, ws_bytes, l)) return rc;
  if (!q_start || !q_pos) return fail(NOSA_ERR_INVALID_ARG, "q_start and q_pos must not be NULL");
  if (!aligned(q_start, 4) || !aligned(q_pos, 4)) return fail(NOSA_ERR_INVALID_ARG, "q_start / q_pos must be 4-byte aligned");
  if (int rc = check_decode_ptrs(q, k_cache, v_cache, cache_rows, kvl, q_start, sel_idx, sel_cnt, out)) return rc;
  if (!pooled || nc_cap < 1) return fail(NOSA_ERR_INVALID_ARG, "pooled must not be NULL and nc_cap >= 1");
  if (!aligned(pooled, 16)) return fail(NOSA_ERR_INVALID_ARG, "pooled must be 16-byte aligned");
  int32_t* entry_len = at<int32_t>(ws, l.entry_len);
  int32_t* entry_seq = at<int32_t>(ws, l.entry_seq);
  cudaError_t e = nosa::launch_prefill_entries(q_start, q_pos, batch, total_q, entry_len, entry_seq, stream);
  if (e != cudaSuccess) return cuda_fail(e, "prefill entries launch");
  nosa::StepArgs s = step_args(p, q, entry_len, total_q, max_seq_len, sel_idx, sel_cnt, ws, l);
  s.seq_of = entry_seq;
  s.seq_start = kvl.seq_start;
  s.page_table = kvl.page_table;
  s.max_pages = kvl.max_pages;
  s.cache_rows = cache_rows;
  s.pooled = const_cast<void*>(pooled);
  s.nc_cap = nc_cap;
  s.out = static_cast<__nv_bfloat16*>(out);
  s.lse = lse;
  // bf16 caches of sequences up to kPrefillMaxBlocks blocks: selection per
  // entry in the step kernel, then the grouped attention kernel; otherwise
  // the step kernel attends per entry as well.
  const bool grouped = p->kv_int8 == 0 && nosa::n_blocks(max_seq_len) <= nosa::kPrefillMaxBlocks;
  s.mode = grouped ? nosa::kStepScore : nosa::kStepScore | nosa::kStepDecode;
  set_int8(s, p, const_cast<void*>(k_cache), v_cache, cache_rows);
  nosa::StepMaps maps;
  memset(&maps, 0, sizeof maps);
  if (int rc = encode_cache_maps(&maps, p, k_cache, v_cache, cache_rows)) return rc;
  if (int rc = encode_pooled_map(&maps.p, pooled, batch, p->num_kv_heads, nc_cap, p->pooled_bf16 != 0)) return rc;
  e = nosa::launch_step(s, maps, stream);
  if (e != cudaSuccess) return cuda_fail(e, "sparse_prefill launch");
  if (grouped) {
    nosa::PrefillAttnArgs pa{};
    pa.q = static_cast<const __nv_bfloat16*>(q);
    pa.entry_len = entry_len;
    pa.entry_seq = entry_seq;
    pa.seq_start = kvl.seq_start;
    pa.page_table = kvl.page_table;
    pa.max_pages = kvl.max_pages;
    pa.cache_rows = cache_rows;
    pa.sel_idx = sel_idx;
    pa.sel_cnt = sel_cnt;
    pa.out = static_cast<__nv_bfloat16*>(out);
    pa.lse = lse;
    pa.status = at<uint32_t>(ws, l.status);
    pa.total_q = total_q;
    pa.hq = p->num_q_heads;
    pa.hkv = p->num_kv_heads;
    pa.topk = p->topk;
    pa.local_blocks = p->local_blocks;
    pa.max_seq_len = max_seq_len;
    pa.nb_words = static_cast<int>((nosa::n_blocks(max_seq_len) + 31) / 32);
    pa.scale_log2 = s.scale_log2;
    e = nosa::launch_prefill_attn(pa, maps.k, maps.v, stream);
    if (e != cudaSuccess) return cuda_fail(e, "sparse_prefill attention launch");
  }
  return ok();
}

}  // namespace

namespace nosa {

size_t workspace_counter_bytes(const nosa_params* p, int batch, int max_seq_len) {
  if (check_params(p) != NOSA_OK || batch < 0 || max_seq_len < 1) return 0;
  return layout_of(p, batch, max_seq_len).spill;
}

int record_error(int code, const char* msg) { return fail(code, "%s", msg); }

int check_decode_step_device(const nosa_params* p, const void* q, const void* k_new, const void* v_new,
                             const void* k_cache, const void* v_cache, int64_t cache_rows, const int64_t* seq_start,
                             const int32_t* seq_len, int batch, int max_seq_len, const void* pooled, int nc_cap,
                             const int32_t* sel_idx, const int32_t* sel_cnt, const void* out) {
  if (int rc = check_params(p)) return rc;
  if (int rc = check_common(p, batch, max_seq_len)) return rc;
  if (batch == 0) return ok();
  return check_step_buffers(q, k_new, v_new, k_cache, v_cache, cache_rows, KvLayout{seq_start, nullptr, 0}, seq_len,
                            pooled, nc_cap, sel_idx, sel_cnt, out);
}

}  // namespace nosa

extern "C" {

void nosa_default_params(nosa_params* p) {
  if (!p) return;
  p->num_q_heads = 16;
  p->num_kv_heads = 2;
  p->head_dim = 128;
  p->pool_kernel = 32;
  p->pool_stride = 16;
  p->block_size = 64;
  p->local_blocks = 16;
  p->topk = 64;
  p->softmax_scale = 0.0f;
  p->pooled_bf16 = 0;
  p->kv_int8 = 0;
}

size_t nosa_kv_int8_bytes(int64_t cache_rows, int num_kv_heads) {
  if (cache_rows < 1 || cache_rows >= (int64_t{1} << 31) || num_kv_heads < 1) return 0;
  return static_cast<size_t>(nosa::int8_scale_offset(cache_rows, num_kv_heads)) +
         static_cast<size_t>(num_kv_heads) * nosa::int8_scale_stride(cache_rows) * 4;
}

int nosa_quantize_kv_int8(const nosa_params* p, const void* src, void* cache, int64_t cache_rows, int64_t row0,
                          int64_t rows, void* stream) {
  if (int rc = check_params(p)) return rc;
  if (!src || !cache) return fail(NOSA_ERR_INVALID_ARG, "src and cache must not be NULL");
  if (!aligned(src, 8) || !aligned(cache, 16))
    return fail(NOSA_ERR_INVALID_ARG, "src must be 8-byte and cache 16-byte aligned");
  if (cache_rows < 1 || cache_rows >= (int64_t{1} << 31))
    return fail(NOSA_ERR_UNSUPPORTED, "cache_rows must be in [1, 2^31)");
  if (row0 < 0 || rows < 0 || row0 + rows > cache_rows)
    return fail(NOSA_ERR_INVALID_ARG, "rows [%lld, %lld) outside the cache's %lld rows", static_cast<long long>(row0),
                static_cast<long long>(row0 + rows), static_cast<long long>(cache_rows));
  cudaError_t e = nosa::launch_quantize_int8(static_cast<const __nv_bfloat16*>(src), static_cast<int8_t*>(cache),
                                             int8_scales(cache, cache_rows, p->num_kv_heads),
                                             nosa::int8_scale_stride(cache_rows), row0, rows, p->num_kv_heads,
                                             static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return ok();
}

size_t nosa_workspace_size(const nosa_params* p, int batch, int max_seq_len) {
  if (check_params(p) != NOSA_OK || batch < 0 || max_seq_len < 1) return 0;
  return layout_of(p, batch, max_seq_len).total;
}

size_t nosa_prefill_workspace_size(const nosa_params* p, int total_q, int max_seq_len) {
  if (check_params(p) != NOSA_OK || total_q < 0 || max_seq_len < 1) return 0;
  return prefill_layout_of(p, total_q, max_seq_len).total;
}

int nosa_sparse_prefill(const nosa_params* p, const void* q, const void* k_cache, const void* v_cache,
                        int64_t cache_rows, const int64_t* seq_start, const int32_t* q_start, const int32_t* q_pos,
                        int batch, int total_q, int max_seq_len, const void* pooled, int nc_cap, int32_t* sel_idx,
                        int32_t* sel_cnt, void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_params(p)) return rc;
  return do_sparse_prefill(p, q, k_cache, v_cache, cache_rows, KvLayout{seq_start, nullptr, 0}, q_start, q_pos, batch,
                           total_q, max_seq_len, pooled, nc_cap, sel_idx, sel_cnt, out, lse, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream));
}

int nosa_sparse_prefill_paged(const nosa_params* p, const void* q, const void* k_cache, const void* v_cache,
                              int64_t num_pages, const int32_t* page_table, int max_pages, const int32_t* q_start,
                              const int32_t* q_pos, int batch, int total_q, int max_seq_len, const void* pooled,
                              int nc_cap, int32_t* sel_idx, int32_t* sel_cnt, void* out, float* lse, void* ws,
                              size_t ws_bytes, void* stream) {
  if (int rc = check_params(p)) return rc;
  if (!page_table) return fail(NOSA_ERR_INVALID_ARG, "page_table must not be NULL");
  if (num_pages < 1 || num_pages >= (int64_t{1} << 31) / nosa::kPageTokens)
    return fail(NOSA_ERR_UNSUPPORTED, "num_pages must be in [1, 2^31 / 64)");
  return do_sparse_prefill(p, q, k_cache, v_cache, num_pages * nosa::kPageTokens,
                           KvLayout{nullptr, page_table, max_pages}, q_start, q_pos, batch, total_q, max_seq_len,
                           pooled, nc_cap, sel_idx, sel_cnt, out, lse, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream));
}

int nosa_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256) return fail(NOSA_ERR_WORKSPACE, "workspace NULL or smaller than 256 bytes");
  if (!aligned(ws, 256)) return fail(NOSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "workspace memset");
  return ok();
}

int nosa_pool_append(const nosa_params* p, void* k_cache, void* v_cache, int64_t cache_rows, const int64_t* seq_start,
                     const int32_t* len_old, const int32_t* len_new, int batch, void* pooled, int nc_cap,
                     int max_new_keys, const void* k_new, const void* v_new, void* ws, size_t ws_bytes,
                     void* stream) {
  if (int rc = check_params(p)) return rc;
  uint32_t* status = nullptr;
  if (ws) {
    if (ws_bytes < 256 || !aligned(ws, 256)) return fail(NOSA_ERR_WORKSPACE, "workspace must be 256-byte aligned and >= 256 bytes");
    status = at<uint32_t>(ws, 0);
  }
  return do_pool_append(p, k_cache, v_cache, cache_rows, KvLayout{seq_start, nullptr, 0}, len_old, len_new, batch,
                        pooled, nc_cap, max_new_keys, k_new, v_new, status, static_cast<cudaStream_t>(stream));
}

int nosa_pool_append_paged(const nosa_params* p, void* k_cache, void* v_cache, int64_t num_pages,
                           const int32_t* page_table, int max_pages, const int32_t* len_old,
                           const int32_t* len_new, int batch, void* pooled, int nc_cap, int max_new_keys,
                           const void* k_new, const void* v_new, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_params(p)) return rc;
  if (!page_table) return fail(NOSA_ERR_INVALID_ARG, "page_table must not be NULL");
  if (num_pages < 1 || num_pages >= (int64_t{1} << 31) / nosa::kPageTokens)
    return fail(NOSA_ERR_UNSUPPORTED, "num_pages must be in [1, 2^31 / 64)");
  uint32_t* status = nullptr;
  if (ws) {
    if (ws_bytes < 256 || !aligned(ws, 256)) return fail(NOSA_ERR_WORKSPACE, "workspace must be 256-byte aligned and >= 256 bytes");
    status = at<uint32_t>(ws, 0);
  }
  return do_pool_append(p, k_cache, v_cache, num_pages * nosa::kPageTokens, KvLayout{nullptr, page_table, max_pages},
                        len_old, len_new, batch, pooled, nc_cap, max_new_keys, k_new, v_new, status,
                        static_cast<cudaStream_t>(stream));
}

int nosa_block_select(const nosa_params* p, const void* q, const void* pooled, int nc_cap,
                      const int32_t* seq_len, int batch, int max_seq_len, const float* block_scores_in,
                      int nb_cap_in, float* comp_scores_out, float* block_scores_out, int nb_cap_out,
                      int32_t* sel_idx, int32_t* sel_cnt, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_params(p)) return rc;
  return do_block_select(p, q, pooled, nc_cap, seq_len, batch, max_seq_len, block_scores_in, nb_cap_in,
                         comp_scores_out, block_scores_out, nb_cap_out, sel_idx, sel_cnt, ws, ws_bytes,
                         static_cast<cudaStream_t>(stream));
}

int nosa_sparse_decode(const nosa_params* p, const void* q, const void* k_cache, const void* v_cache,
                       int64_t cache_rows, const int64_t* seq_start, const int32_t* seq_len, int batch, int max_seq_len,
                       const int32_t* sel_idx, const int32_t* sel_cnt, void* out, float* lse, void* ws,
                       size_t ws_bytes, void* stream) {
  if (int rc = check_params(p)) return rc;
  return do_sparse_decode(p, q, k_cache, v_cache, cache_rows, KvLayout{seq_start, nullptr, 0}, seq_len, batch,
                          max_seq_len, sel_idx, sel_cnt, out, lse, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int nosa_sparse_decode_paged(const nosa_params* p, const void* q, const void* k_cache, const void* v_cache,
                             int64_t num_pages, const int32_t* page_table, int max_pages, const int32_t* seq_len,
                             int batch, int max_seq_len, const int32_t* sel_idx, const int32_t* sel_cnt, void* out,
                             float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (int rc = check_params(p)) return rc;
  if (!page_table) return fail(NOSA_ERR_INVALID_ARG, "page_table must not be NULL");
  if (num_pages < 1 || num_pages >= (int64_t{1} << 31) / nosa::kPageTokens)
    return fail(NOSA_ERR_UNSUPPORTED, "num_pages must be in [1, 2^31 / 64)");
  return do_sparse_decode(p, q, k_cache, v_cache, num_pages * nosa::kPageTokens,
                          KvLayout{nullptr, page_table, max_pages}, seq_len, batch, max_seq_len, sel_idx, sel_cnt, out,
                          lse, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int nosa_decode_step_device(const nosa_params* p, const void* q, const void* k_new, const void* v_new,
                            void* k_cache, void* v_cache, int64_t cache_rows, const int64_t* seq_start,
                            const int32_t* seq_len, int batch, int max_seq_len, void* pooled, int nc_cap,
                            int32_t* sel_idx, int32_t* sel_cnt, void* out, float* lse, void* ws, size_t ws_bytes,
                            void* stream) {
  if (int rc = check_params(p)) return rc;
  return do_decode_step_device(p, q, k_new, v_new, k_cache, v_cache, cache_rows, KvLayout{seq_start, nullptr, 0},
                               seq_len, batch, max_seq_len, pooled, nc_cap, sel_idx, sel_cnt, out, lse, ws, ws_bytes,
                               static_cast<cudaStream_t>(stream));
}

int nosa_decode_step_device_paged(const nosa_params* p, const void* q, const void* k_new, const void* v_new,
                                  void* k_cache, void* v_cache, int64_t num_pages, const int32_t* page_table,
                                  int max_pages, const int32_t* seq_len, int batch, int max_seq_len, void* pooled,
                                  int nc_cap, int32_t* sel_idx, int32_t* sel_cnt, void* out, float* lse, void* ws,
                                  size_t ws_bytes, void* stream) {
  if (int rc = check_params(p)) return rc;
  if (!page_table) return fail(NOSA_ERR_INVALID_ARG, "page_table must not be NULL");
  if (num_pages < 1 || num_pages >= (int64_t{1} << 31) / nosa::kPageTokens)
    return fail(NOSA_ERR_UNSUPPORTED, "num_pages must be in [1, 2^31 / 64)");
  return do_decode_step_device(p, q, k_new, v_new, k_cache, v_cache, num_pages * nosa::kPageTokens,
                               KvLayout{nullptr, page_table, max_pages}, seq_len, batch, max_seq_len, pooled, nc_cap,
                               sel_idx, sel_cnt, out, lse, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// The host-buffer step after the input copies: the fused step on the
// staging area, then the output copy back.
int step_from_staging(const nosa_params* p, const Layout& l, void* out_host, void* k_cache, void* v_cache,
                      int64_t cache_rows, const int64_t* seq_start, const int32_t* seq_len, int batch,
                      int max_seq_len, void* pooled, int nc_cap, int32_t* sel_idx, int32_t* sel_cnt, void* ws,
                      size_t ws_bytes, cudaStream_t s) {
  const size_t qbytes = static_cast<size_t>(batch) * p->num_q_heads * nosa::kHeadDim * 2;
  int rc = do_decode_step_device(p, at<void>(ws, l.stage_q), at<void>(ws, l.stage_k), at<void>(ws, l.stage_v), k_cache,
                                 v_cache, cache_rows, KvLayout{seq_start, nullptr, 0}, seq_len, batch, max_seq_len,
                                 pooled, nc_cap, sel_idx, sel_cnt, at<void>(ws, l.stage_out), nullptr, ws, ws_bytes, s);
  if (rc) return rc;
  cudaError_t e = cudaMemcpyAsync(out_host, at<void>(ws, l.stage_out), qbytes, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy out");
  return ok();
}

int check_host_step(const nosa_params* p, int batch, int max_seq_len, void* ws, size_t ws_bytes, Layout* l) {
  if (int rc = check_params(p)) return rc;
  if (int rc = check_common(p, batch, max_seq_len)) return rc;
  *l = layout_of(p, batch, max_seq_len);
  return batch == 0 ? NOSA_OK : check_ws(ws, ws_bytes, *l);
}

}  // namespace

extern "C" {

int nosa_decode_step(const nosa_params* p, const void* q_host, const void* k_new_host,
                     const void* v_new_host, void* out_host, void* k_cache, void* v_cache,
                     int64_t cache_rows, const int64_t* seq_start, const int32_t* seq_len, int batch, int max_seq_len,
                     void* pooled, int nc_cap, int32_t* sel_idx, int32_t* sel_cnt, void* ws,
                     size_t ws_bytes, void* stream) {
  Layout l;
  if (int rc = check_host_step(p, batch, max_seq_len, ws, ws_bytes, &l)) return rc;
  if (batch == 0) return ok();
  if (!q_host || !k_new_host || !v_new_host || !out_host)
    return fail(NOSA_ERR_INVALID_ARG, "host buffers must not be NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t qbytes = static_cast<size_t>(batch) * p->num_q_heads * nosa::kHeadDim * 2;
  const size_t kvbytes = static_cast<size_t>(batch) * p->num_kv_heads * nosa::kHeadDim * 2;
  cudaError_t e;
  if ((e = cudaMemcpyAsync(at<void>(ws, l.stage_q), q_host, qbytes, cudaMemcpyHostToDevice, s)) != cudaSuccess)
    return cuda_fail(e, "copy q");
  if ((e = cudaMemcpyAsync(at<void>(ws, l.stage_k), k_new_host, kvbytes, cudaMemcpyHostToDevice, s)) != cudaSuccess)
    return cuda_fail(e, "copy k_new");
  if ((e = cudaMemcpyAsync(at<void>(ws, l.stage_v), v_new_host, kvbytes, cudaMemcpyHostToDevice, s)) != cudaSuccess)
    return cuda_fail(e, "copy v_new");
  return step_from_staging(p, l, out_host, k_cache, v_cache, cache_rows, seq_start, seq_len, batch, max_seq_len,
                           pooled, nc_cap, sel_idx, sel_cnt, ws, ws_bytes, s);
}

int nosa_decode_step_packed(const nosa_params* p, const void* qkv_host, void* out_host, void* k_cache, void* v_cache,
                            int64_t cache_rows, const int64_t* seq_start, const int32_t* seq_len, int batch,
                            int max_seq_len, void* pooled, int nc_cap, int32_t* sel_idx, int32_t* sel_cnt, void* ws,
                            size_t ws_bytes, void* stream) {
  Layout l;
  if (int rc = check_host_step(p, batch, max_seq_len, ws, ws_bytes, &l)) return rc;
  if (batch == 0) return ok();
  if (!qkv_host || !out_host) return fail(NOSA_ERR_INVALID_ARG, "host buffers must not be NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t qbytes = static_cast<size_t>(batch) * p->num_q_heads * nosa::kHeadDim * 2;
  const size_t kvbytes = static_cast<size_t>(batch) * p->num_kv_heads * nosa::kHeadDim * 2;
  // q, k_new and v_new are whole 256-byte rows, so the staging area holds
  // them back to back too: the packed buffer goes in one copy.
  cudaError_t e = cudaMemcpyAsync(at<void>(ws, l.stage_q), qkv_host, qbytes + 2 * kvbytes, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy q, k_new, v_new");
  return step_from_staging(p, l, out_host, k_cache, v_cache, cache_rows, seq_start, seq_len, batch, max_seq_len,
                           pooled, nc_cap, sel_idx, sel_cnt, ws, ws_bytes, s);
}

int nosa_read_device_status(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256 || !aligned(ws, 256)) return fail(NOSA_ERR_WORKSPACE, "workspace NULL, small or misaligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t bits = 0;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&bits, ws, sizeof bits, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof bits, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "read device status");
  g_last_bits = bits;
  if (bits & NOSA_DEV_TIMEOUT) return fail(NOSA_ERR_TIMEOUT, "device status 0x%08x: a bounded wait gave up", bits);
  if (bits) return fail(NOSA_ERR_DEVICE_CHECK, "device status 0x%08x", bits);
  return ok();
}

uint32_t nosa_last_device_bits(void) { return g_last_bits; }

int nosa_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t max_iters, void* stream) {
  if (!ws || ws_bytes < 256 || !aligned(ws, 256)) return fail(NOSA_ERR_WORKSPACE, "workspace NULL, small or misaligned");
  if (max_iters < 1 || max_iters > (1u << 20)) return fail(NOSA_ERR_INVALID_ARG, "max_iters must be 1..2^20");
  cudaError_t e = nosa::launch_wait_selftest(at<uint32_t>(ws, 0), max_iters, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "wait selftest launch");
  return ok();
}

const char* nosa_status_string(int status) {
  switch (status) {
    case NOSA_OK: return "ok";
    case NOSA_ERR_INVALID_ARG: return "invalid argument";
    case NOSA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case NOSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case NOSA_ERR_CUDA: return "CUDA error";
    case NOSA_ERR_DEVICE_CHECK: return "device data check failed";
    case NOSA_ERR_TIMEOUT: return "bounded device wait timed out";
    default: return "unknown status";
  }
}

const char* nosa_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
