/*
 * nosa.h -- C ABI of the B200 (sm_100a) NOSA sparse decode attention library.
 *
 * NOSA (Native and Offloadable Sparse Attention) answers one decode query per
 * sequence by (1) mean-pooling the key cache into compressed keys, (2) scoring
 * the compressed keys against every query head and reducing them to 64-token
 * block scores shared by each GQA group, (3) choosing the top-k blocks plus a
 * forced local window, and (4) running exact attention over only those blocks.
 *
 * Pages that define the operations (cited by title and section):
 *   "从论文到代码：手把手教你理解NOSA-8B的高效注意力机制实现" (nzsm.cn),
 *       "NOSA-8B的核心实现模块" item 2: forward pools the keys with
 *       cis_pooling(k, cu_seqlens) before attention.
 *   "NOSA-1B 模型家族全景：从 1B 到 8B，三款稀疏注意力模型怎么选"
 *       (demingchina.com), "核心原理": local window of 1024 tokens; two-level
 *       retrieval -- compressed attention screens the history for the TopK
 *       blocks, which are then read exactly.
 *   "NOSA-1B 性能基准全解析：5.04× 解码吞吐提升是怎么测出来的" (wmrh.cn),
 *       §三.2 (window 1024, block 64, about 16 local blocks, TopK 64 blocks),
 *       §三.3 (pooling kernel_size 32 / stride 16, coarse scores, top-k,
 *       exact attention), §四 config table (16 q / 2 KV heads, bfloat16).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  * All tensor arguments are DEVICE pointers to caller-owned memory, except
 *    where an argument is documented as a host pointer.  The library keeps no
 *    global state besides a per-thread last-error string, and allocates no
 *    device memory: scratch space is the caller's workspace `ws`.  The one
 *    exception is nosa_decode_step_device_noalloc, whose scratch is a fixed
 *    array that the library defines in device memory (see there).
 *  * `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.  Every call only enqueues work on it (no host synchronisation),
 *    except nosa_read_device_status.
 *  * Layouts (row-major, innermost last):
 *      q            bf16 [batch, num_q_heads, head_dim]
 *      k_cache/v_cache bf16 [cache_rows, num_kv_heads, head_dim], cache_rows
 *                   < 2^31; sequence i occupies rows seq_start[i] ..
 *                   seq_start[i] + len - 1 (varlen packing as with
 *                   cu_seqlens: seq_start[i] = cu_seqlens[i]).  With
 *                   p->kv_int8: INT8 buffers (see nosa_kv_int8_bytes).
 *      pooled       fp32 (or bf16 when p->pooled_bf16) [batch, num_kv_heads, nc_cap,
 *                   head_dim]
 *      sel_idx      int32 [batch, num_kv_heads, topk] (ascending, -1 padded)
 *      sel_cnt      int32 [batch, num_kv_heads]
 *      out          bf16 [batch, num_q_heads, head_dim]
 *      lse          fp32 [batch, num_q_heads]  (natural log of the softmax
 *                   denominator of scale*q.k over the attended tokens)
 *    Query head h belongs to KV head h / (num_q_heads / num_kv_heads).
 *  * Lengths: seq_len[i] counts the tokens of sequence i INCLUDING the token
 *    being decoded (its K/V row is in the cache before the attention call).
 *  * Geometry: window j covers tokens [16j, 16j+32); nc(L) = L >= 32 ?
 *    (L-32)/16 + 1 : 0.  Block b covers tokens [64b, 64b+64); nb(L) =
 *    ceil(L/64).  The local window is the last local_blocks blocks; the
 *    candidates for top-k are blocks [0, ncand), ncand = max(0, nb-local_blocks).
 *  * Errors: problems visible on the host (null pointers, unsupported shapes,
 *    small workspace) return a status code at once and enqueue nothing.  A
 *    failed launch returns NOSA_ERR_CUDA.  Problems that depend on device
 *    data (a length < 1, a window past nc_cap, an index out of range, a
 *    bounded wait that gave up) never trap: the kernel skips that unit,
 *    writes zeros where it owns output, and sets a bit in the workspace's
 *    device status word, which nosa_read_device_status returns and clears.
 *  * An empty batch (batch 0, or total_q 0 for the prefill calls) returns
 *    NOSA_OK at once, before the other buffers are checked and without any
 *    CUDA call; the paged calls still check the page pool's geometry (a
 *    page table pointer and num_pages >= 1).
 *  * Calls that share one workspace must not overlap on the GPU (order them
 *    on one stream): the workspace holds the status word, block scores of
 *    very long sequences and the host-buffer step's staging.
 */
#ifndef NOSA_B200_H
#define NOSA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(NOSA_BUILD) && defined(__GNUC__)
#define NOSA_API __attribute__((visibility("default")))
#else
#define NOSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NOSA_OK = 0,
  NOSA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad enum */
  NOSA_ERR_UNSUPPORTED = 2,  /* a shape/parameter this build does not handle */
  NOSA_ERR_WORKSPACE = 3,    /* workspace null, misaligned or too small */
  NOSA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  NOSA_ERR_DEVICE_CHECK = 5, /* device status word had a data-check bit set */
  NOSA_ERR_TIMEOUT = 6       /* device status word had the bounded-wait bit set */
} nosa_status;

/* Device status bits (returned by nosa_read_device_status in
 * nosa_last_device_bits()). */
#define NOSA_DEV_BAD_LENGTH 0x1u     /* seq_len < 1, or len_old > len_new */
#define NOSA_DEV_NC_CAP 0x2u         /* nc(L) exceeds nc_cap */
#define NOSA_DEV_BAD_INDEX 0x4u      /* sel_idx entry outside [0, ncand) */
#define NOSA_DEV_BAD_COUNT 0x8u      /* sel_cnt outside [0, topk] */
#define NOSA_DEV_MAX_NEW_KEYS 0x10u  /* more new windows than max_new_keys */
#define NOSA_DEV_APPEND_ONE 0x20u    /* k_new given but len_new != len_old + 1 */
#define NOSA_DEV_MAX_LEN 0x40u       /* seq_len above the call's max_seq_len */
#define NOSA_DEV_CACHE_ROWS 0x80u    /* a sequence's rows reach past cache_rows */
#define NOSA_DEV_TIMEOUT 0x80000000u /* an mbarrier wait hit its iteration limit */

typedef struct {
  int num_q_heads;     /* Hq; multiple of num_kv_heads */
  int num_kv_heads;    /* Hkv; G = Hq/Hkv must be 1..16 */
  int head_dim;        /* must be 128 */
  int pool_kernel;     /* must be 32 */
  int pool_stride;     /* must be 16 */
  int block_size;      /* must be 64 */
  int local_blocks;    /* forced local window in blocks (16 = 1024 tokens); 0..256 */
  int topk;            /* selected blocks per (sequence, KV head); 1..1024 */
  float softmax_scale; /* 0 => 1/sqrt(head_dim); used for scores and attention */
  int pooled_bf16;     /* 0: pooled keys fp32 (default); 1: pooled keys bf16, each the
                          round-to-nearest-even of the fp32 mean (half the selection bytes) */
  int kv_int8;         /* 0: K/V caches bf16 (default); 1: INT8 caches (codes + per-row
                          scales, see nosa_kv_int8_bytes): half the attention bytes */
} nosa_params;

/* Fills `p` with the NOSA-1B attention defaults: 16 q / 2 KV heads, head_dim
 * 128, kernel 32 / stride 16, block 64, 16 local blocks, topk 64, scale 0,
 * fp32 pooled keys, bf16 caches. */
NOSA_API void nosa_default_params(nosa_params* p);

/* INT8 K/V caches (p->kv_int8 = 1; reading of "NOSA 技术架构解析"
 * (devpress.csdn.net) §1.1 "关键技巧": the decode stage may switch to 8-bit
 * integers).  Each cache row (token, KV head) of 128 bf16 values x is stored
 * as 128 int8 codes and one fp32 scale, symmetric per row:
 *     s = max|x| / 127,  code = clamp(rint(x / s), -127, 127)
 * (IEEE fp32 divisions, rint half to even; s = 0 for an all-zero row), and
 * read back as s * code.  With kv_int8 set, every k_cache / v_cache argument
 * of the calls below is one such buffer (K and V separately):
 *     codes  int8 [cache_rows, Hkv, 128]                at byte 0
 *     scales fp32 [Hkv, scale_stride]                   at byte cache_rows * Hkv * 128
 * with scale_stride = cache_rows rounded up to a multiple of 4 (for paged
 * caches cache_rows = num_pages * 64).  The new token's k_new / v_new stay
 * bf16: the calls quantize them on append.  Pooling reads s * code (the
 * pooled keys are as in the bf16 case), attention uses s * code for K and V.
 * nosa_kv_int8_bytes returns the buffer size (0 if the arguments are
 * invalid); nosa_quantize_kv_int8 quantizes bf16 rows src [rows, Hkv, 128]
 * into rows row0 .. row0 + rows - 1 of such a buffer (e.g. after a prefill). */
NOSA_API size_t nosa_kv_int8_bytes(int64_t cache_rows, int num_kv_heads);
NOSA_API int nosa_quantize_kv_int8(const nosa_params* p, const void* src, void* cache, int64_t cache_rows,
                                   int64_t row0, int64_t rows, void* stream);

/* Bytes of device workspace that nosa_block_select / nosa_sparse_decode /
 * nosa_decode_step need for `batch` sequences of at most `max_seq_len`
 * tokens: the device status word; block scores [batch * Hkv, ncand] fp32
 * when a sequence of max_seq_len tokens has more than 2048 candidates (fewer
 * stay in shared memory); the staging buffers of nosa_decode_step (q, new
 * K/V rows, out).  Returns 0 if the parameters are invalid.  The workspace
 * must be 256-byte aligned and zeroed once with nosa_workspace_init before
 * first use. */
NOSA_API size_t nosa_workspace_size(const nosa_params* p, int batch, int max_seq_len);

/* Zeroes the workspace (device status word included) on `stream`. */
NOSA_API int nosa_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Step 1 -- CIS mean pooling of keys, appended incrementally
 * ("从论文到代码…" item 2; "NOSA-1B 性能基准全解析" §三.3 kernel 32 / stride 16).
 * For every sequence i and KV head h, and every window j with
 * nc(len_old[i]) <= j < nc(len_new[i]):
 *     pooled[i][h][j][:] = (1/32) * sum_{t=16j}^{16j+31} K[seq_start[i]+t][h][:]
 * summed in fp32 in ascending t (so rebuilding and appending give identical
 * bits), then stored as fp32, or rounded to bf16 (nearest, ties to even) when
 * p->pooled_bf16.  Windows outside that range are not touched.
 * Optional fused append: when k_new/v_new (bf16 [batch, Hkv, head_dim]) are
 * non-NULL, len_new[i] must equal len_old[i] + 1 and the row is first written
 * to k_cache/v_cache at seq_start[i] + len_old[i] (the new token's K is read
 * from k_new for pooling, so no ordering hazard exists).
 * len_old may be NULL, meaning len_new[i] - 1 for every i.
 * At most max_new_keys windows per (sequence, KV head) are produced; more sets
 * NOSA_DEV_MAX_NEW_KEYS.  A window past nc_cap sets NOSA_DEV_NC_CAP.
 * Uses only the workspace's status word; `ws` may be NULL (then device data
 * errors are not reported). */
NOSA_API int nosa_pool_append(const nosa_params* p, void* k_cache, void* v_cache,
                     int64_t cache_rows, const int64_t* seq_start, const int32_t* len_old,
                     const int32_t* len_new, int batch, void* pooled,
                     int nc_cap, int max_new_keys, const void* k_new,
                     const void* v_new, void* ws, size_t ws_bytes, void* stream);

/* Steps 2-3 -- compressed scores, block scores and top-k selection
 * ("NOSA-1B 模型家族全景" 核心原理; "NOSA-1B 性能基准全解析" §三.2/§三.3):
 *   s[i][h][j]  = scale * q[i][h] . pooled[i][h/G][j]          (j < nc(L_i))
 *   S[i][g][b]  = sum_{h in group g, ascending} max_{j in J(b)} s[i][h][j],
 *                 J(b) = {4b-1, ..., 4b+3} n [0, nc(L_i)), for b < ncand(L_i)
 *   sel[i][g]   = the min(topk, ncand) candidates with the largest S, ties to
 *                 the lower block index (-0.0 == +0.0, NaN ranks as -inf),
 *                 written in ascending order and padded with -1.
 * If block_scores_in (fp32 [batch, Hkv, nb_cap_in]) is non-NULL, scoring is
 * skipped and the selection runs on those scores (q/pooled may then be NULL).
 * comp_scores_out (fp32 [batch, Hq, nc_cap], nullable) receives s for every
 * j < nc(L_i); block_scores_out (fp32 [batch, Hkv, nb_cap_out], nullable)
 * receives S for every candidate block.  Other entries are not written.
 * seq_len[i] must not exceed max_seq_len (else NOSA_DEV_MAX_LEN, the pair is
 * skipped with sel_cnt = 0). */
NOSA_API int nosa_block_select(const nosa_params* p, const void* q, const void* pooled,
                      int nc_cap, const int32_t* seq_len, int batch,
                      int max_seq_len, const float* block_scores_in,
                      int nb_cap_in, float* comp_scores_out,
                      float* block_scores_out, int nb_cap_out,
                      int32_t* sel_idx, int32_t* sel_cnt, void* ws,
                      size_t ws_bytes, void* stream);

/* Step 4 -- exact sparse attention ("NOSA-1B 性能基准全解析" §三.3, exact
 * attention on the TopK blocks, plus the §三.2 local window):
 *   T_i,g = (U_{t < sel_cnt} [64*sel_idx[t], 64*sel_idx[t]+64) U [64*ncand, L_i)) n [0, L_i)
 *   out[i][h] = sum_{t in T} softmax_t(scale * q[i][h] . k_t) v_t
 * computed as a split-K flash-decode over 64-token KV tiles with fp32
 * accumulation and a fixed-order fp32 merge of the partial softmaxes (bit-
 * reproducible run to run).  Selected indices must be distinct; the order of
 * sel_idx does not matter.  lse (fp32 [batch, Hq]) is nullable. */
NOSA_API int nosa_sparse_decode(const nosa_params* p, const void* q, const void* k_cache,
                       const void* v_cache, int64_t cache_rows, const int64_t* seq_start,
                       const int32_t* seq_len, int batch, int max_seq_len,
                       const int32_t* sel_idx, const int32_t* sel_cnt,
                       void* out, float* lse, void* ws, size_t ws_bytes,
                       void* stream);

/* One whole decode step on DEVICE buffers, fused into a single launch
 * (steps 1-4 above, in the pages' order): appends the new
 * token's K/V rows (k_new / v_new, bf16 [batch, Hkv, D], nullable: then the
 * rows must already be in the caches) at seq_start[i] + seq_len[i] - 1, pools
 * the window it completes, scores and selects blocks (sel_idx / sel_cnt
 * receive the selection) and attends, writing out (bf16 [batch, Hq, D]) and
 * lse (nullable).  Results are bit-identical to nosa_pool_append +
 * nosa_block_select + nosa_sparse_decode on the same inputs.  Each
 * (sequence, KV head) is one thread-block cluster: its CTAs score the
 * pooled keys, exchange block scores through distributed shared memory,
 * select, attend over their share of the tiles and merge in the cluster;
 * every wait is bounded (NOSA_DEV_TIMEOUT on expiry).  With fewer than two
 * local blocks the three separate launches run instead. */
NOSA_API int nosa_decode_step_device(const nosa_params* p, const void* q, const void* k_new,
                                     const void* v_new, void* k_cache, void* v_cache,
                                     int64_t cache_rows, const int64_t* seq_start,
                                     const int32_t* seq_len, int batch, int max_seq_len,
                                     void* pooled, int nc_cap, int32_t* sel_idx,
                                     int32_t* sel_cnt, void* out, float* lse, void* ws,
                                     size_t ws_bytes, void* stream);

/* The fused decode step for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a deployment variant of
 * nosa_decode_step_device.  Some callers cannot provide a workspace -- a
 * plugin inside an inference engine whose memory manager owns the whole
 * device pool and offers no workspace hook, or a serving loop that must not
 * call cudaMalloc once the KV cache has taken the free memory.  This entry
 * point takes the same arguments without `ws` and keeps its scratch in an
 * 8 MiB array that the library defines in device memory.  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *  * Host checks are those of nosa_decode_step_device and come first: a
 *    rejected call returns its status code and enqueues nothing.  An empty
 *    batch returns NOSA_OK with no CUDA call.
 *  * A batch whose nosa_workspace_size exceeds 8 MiB is rejected with
 *    NOSA_ERR_WORKSPACE (nothing is enqueued); use nosa_decode_step_device.
 *  * The array is part of the library's device code: CUDA creates it on a
 *    device when it loads that code there, and it stays until the process
 *    exits.  Under CUDA's default lazy loading that happens at the first
 *    call on the device (with batch >= 1), so that first call -- like any
 *    first kernel launch -- needs the 8 MiB of free device memory and may
 *    synchronise: make it before the KV cache claims the free memory and
 *    before any stream capture.  (CUDA_MODULE_LOADING=EAGER creates it when
 *    the context is created instead.)  Every call looks the array's device
 *    address up on the current device, so calls stay valid across devices
 *    and after a device reset.
 *  * Every call on a device shares the one array, which keeps what the last
 *    call left: the call clears its status word first (asynchronously, on
 *    `stream`), but calls that overlap on the GPU race.  Order them on one
 *    stream.
 *  * Device-side data checks land in the array's status word, which no entry
 *    point reads back; callers that need those reports use the workspace
 *    variant and nosa_read_device_status. */
NOSA_API int nosa_decode_step_device_noalloc(const nosa_params* p, const void* q,
                                             const void* k_new, const void* v_new,
                                             void* k_cache, void* v_cache, int64_t cache_rows,
                                             const int64_t* seq_start, const int32_t* seq_len,
                                             int batch, int max_seq_len, void* pooled,
                                             int nc_cap, int32_t* sel_idx, int32_t* sel_cnt,
                                             void* out, float* lse, void* stream);

/* Paged KV cache.  "NOSA 技术架构解析" (devpress.csdn.net) §2.1
 * (内核级优化技术, 内存池化管理) gives NOSI's memory pool a
 * PagedAttention-style page layout, and §4.2 (典型问题排查, 问题3) lists the paged-cache switch
 * `--use_paged_kv 1`; neither fixes a page size or table format, so the
 * layout below is this library's.  The caches are a pool of 64-token pages, k_cache / v_cache bf16
 * [num_pages * 64, Hkv, head_dim]; token t of sequence i lives in row
 *     page_table[i * max_pages + t / 64] * 64 + t % 64,
 * page_table int32 [batch, max_pages].  The page size equals the block size,
 * so a selected block is exactly one page.  These three calls are
 * nosa_pool_append, nosa_sparse_decode and nosa_decode_step_device with
 * (num_pages, page_table, max_pages) in place of (cache_rows, seq_start);
 * the results are bit-identical to the contiguous calls on the same tokens.
 * A sequence longer than max_pages * 64 sets NOSA_DEV_CACHE_ROWS; a page
 * index outside [0, num_pages) sets NOSA_DEV_BAD_INDEX (that tile, window or
 * row is skipped; nothing traps).  num_pages must be below 2^31 / 64. */
NOSA_API int nosa_pool_append_paged(const nosa_params* p, void* k_cache, void* v_cache, int64_t num_pages,
                                    const int32_t* page_table, int max_pages, const int32_t* len_old,
                                    const int32_t* len_new, int batch, void* pooled, int nc_cap,
                                    int max_new_keys, const void* k_new, const void* v_new, void* ws,
                                    size_t ws_bytes, void* stream);
NOSA_API int nosa_sparse_decode_paged(const nosa_params* p, const void* q, const void* k_cache,
                                      const void* v_cache, int64_t num_pages, const int32_t* page_table,
                                      int max_pages, const int32_t* seq_len, int batch, int max_seq_len,
                                      const int32_t* sel_idx, const int32_t* sel_cnt, void* out, float* lse,
                                      void* ws, size_t ws_bytes, void* stream);
NOSA_API int nosa_decode_step_device_paged(const nosa_params* p, const void* q, const void* k_new,
                                           const void* v_new, void* k_cache, void* v_cache, int64_t num_pages,
                                           const int32_t* page_table, int max_pages, const int32_t* seq_len,
                                           int batch, int max_seq_len, void* pooled, int nc_cap,
                                           int32_t* sel_idx, int32_t* sel_cnt, void* out, float* lse, void* ws,
                                           size_t ws_bytes, void* stream);

/* Sparse prefill (the pages' NOSAS mode, "NOSA 技术架构解析" §1.3: sparse
 * attention in prefill as well as decode; the pages give no separate prefill
 * rule, so each prefill token follows the decode rule on its own prefix).
 * For every sequence s and query row r of q_start[s] <= e < q_start[s+1]
 * (e = q_start[s] + r), the token at position t = q_pos[s] + r:
 *   L_e     = t + 1 (the prefix the token sees, itself included)
 *   sel[e]  = steps 2-3 above for q[e] against sequence s's pooled keys, L_e
 *   out[e]  = step 4 above over sequence s's cache with L_e and sel[e]
 * i.e. causal, each token selecting its own top-k blocks among the
 * candidates of its prefix plus its local window.
 *   q        bf16 [total_q, Hq, head_dim] (rows of all sequences, packed)
 *   q_start  int32 [batch + 1] (device) non-decreasing row offsets into q,
 *            q_start[0] = 0, q_start[batch] = total_q
 *   q_pos    int32 [batch] (device) position of each sequence's first row
 *   k/v_cache, seq_start: as for nosa_sparse_decode (one start per
 *            sequence); the caches must already hold tokens [0, q_pos[s] +
 *            rows) of each sequence
 *   pooled   [batch, Hkv, nc_cap, head_dim] per sequence, holding every
 *            window complete within each sequence's prefix (append the new
 *            rows' windows first with nosa_pool_append, len_old = q_pos,
 *            len_new = q_pos + rows, max_new_keys >= rows / 16 + 1)
 *   sel_idx  int32 [total_q, Hkv, topk], sel_cnt int32 [total_q, Hkv]
 *   out      bf16 [total_q, Hq, head_dim]; lse fp32 [total_q, Hq] nullable
 * Each entry runs as one decode query of the step kernel (scoring, top-k and
 * attention, no append): the selection is the one nosa_block_select gives
 * for that token with L_e, and the output equals nosa_sparse_decode's up to
 * rounding (the cluster size, and so the split of the tiles and the bf16
 * rounding of the softmax weights, depends on how many entries one launch
 * holds).  The
 * workspace (nosa_prefill_workspace_size bytes, 256-byte aligned, zeroed once
 * with nosa_workspace_init) holds the status word, spilled block scores and
 * the entries' lengths.  A position past max_seq_len sets NOSA_DEV_MAX_LEN;
 * a row outside its sequence's q_start range (q_start not non-decreasing)
 * sets NOSA_DEV_BAD_LENGTH; those entries are skipped. */
NOSA_API size_t nosa_prefill_workspace_size(const nosa_params* p, int total_q, int max_seq_len);
NOSA_API int nosa_sparse_prefill(const nosa_params* p, const void* q, const void* k_cache, const void* v_cache,
                                 int64_t cache_rows, const int64_t* seq_start, const int32_t* q_start,
                                 const int32_t* q_pos, int batch, int total_q, int max_seq_len, const void* pooled,
                                 int nc_cap, int32_t* sel_idx, int32_t* sel_cnt, void* out, float* lse, void* ws,
                                 size_t ws_bytes, void* stream);
/* The same over a paged cache (see the paged calls above): (num_pages,
 * page_table, max_pages) in place of (cache_rows, seq_start); results are
 * bit-identical to the contiguous call on the same tokens. */
NOSA_API int nosa_sparse_prefill_paged(const nosa_params* p, const void* q, const void* k_cache, const void* v_cache,
                                       int64_t num_pages, const int32_t* page_table, int max_pages,
                                       const int32_t* q_start, const int32_t* q_pos, int batch, int total_q,
                                       int max_seq_len, const void* pooled, int nc_cap, int32_t* sel_idx,
                                       int32_t* sel_cnt, void* out, float* lse, void* ws, size_t ws_bytes,
                                       void* stream);

/* One whole decode step from HOST buffers (the pages' per-token decode,
 * steps 1-4 above in order): copies q_host (bf16 [batch, Hq, D]) and the new
 * token's k_new_host / v_new_host (bf16 [batch, Hkv, D]) to the device,
 * appends the new rows to the caches at seq_start[i] + seq_len[i] - 1, pools
 * any window that the new token completes, selects blocks, attends, and
 * copies the bf16 output back to out_host.  seq_len (device) already counts
 * the new token.  All copies and kernels are enqueued on `stream`; the call
 * returns without waiting, so out_host is valid after the stream synchronises.
 * Host buffers should be pinned for the copies to be asynchronous.  The
 * three inputs travel in three copies (nosa_decode_step_packed below takes
 * them as one buffer and one copy).  The device staging area comes from
 * `ws` (nosa_workspace_size covers it).  The kernels run as in
 * nosa_decode_step_device.  sel_idx / sel_cnt (device) receive the
 * selection. */
NOSA_API int nosa_decode_step(const nosa_params* p, const void* q_host,
                     const void* k_new_host, const void* v_new_host,
                     void* out_host, void* k_cache, void* v_cache,
                     int64_t cache_rows, const int64_t* seq_start, const int32_t* seq_len,
                     int batch, int max_seq_len, void* pooled, int nc_cap,
                     int32_t* sel_idx, int32_t* sel_cnt, void* ws,
                     size_t ws_bytes, void* stream);

/* nosa_decode_step with the three inputs in ONE host buffer: qkv_host holds
 * q (bf16 [batch, Hq, D]), then k_new (bf16 [batch, Hkv, D]), then v_new
 * (bf16 [batch, Hkv, D]), back to back, batch * (Hq + 2 Hkv) * D * 2 bytes
 * in all, within one host allocation (pinned, for the copy to be
 * asynchronous).  It travels to the device in a single copy; everything else
 * is as in nosa_decode_step, and the results are bit-identical to it.  The
 * caller owns both host buffers; out_host is valid after `stream`
 * synchronises.  Errors as in nosa_decode_step (NULL host buffer:
 * NOSA_ERR_INVALID_ARG; a copy the runtime refuses: NOSA_ERR_CUDA). */
NOSA_API int nosa_decode_step_packed(const nosa_params* p, const void* qkv_host, void* out_host,
                                     void* k_cache, void* v_cache, int64_t cache_rows,
                                     const int64_t* seq_start, const int32_t* seq_len, int batch,
                                     int max_seq_len, void* pooled, int nc_cap, int32_t* sel_idx,
                                     int32_t* sel_cnt, void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream`, reads and clears the workspace's device status word.
 * Returns NOSA_OK, NOSA_ERR_TIMEOUT (timeout bit set), NOSA_ERR_DEVICE_CHECK
 * (any other bit) or NOSA_ERR_CUDA.  The raw bits of the last read are
 * available from nosa_last_device_bits(). */
NOSA_API int nosa_read_device_status(void* ws, size_t ws_bytes, void* stream);
NOSA_API uint32_t nosa_last_device_bits(void);

/* Diagnostic for the failure-reporting path (no counterpart on the pages):
 * launches one CTA whose thread waits on an mbarrier that nothing arrives on,
 * bounded by max_iters polls (1..2^20).  The wait gives up, sets
 * NOSA_DEV_TIMEOUT in the workspace status word and the kernel returns, so a
 * following nosa_read_device_status returns NOSA_ERR_TIMEOUT. */
NOSA_API int nosa_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t max_iters, void* stream);

/* Static description of a status code. */
NOSA_API const char* nosa_status_string(int status);

/* Detail of the last error returned on the calling host thread ("" if none). */
NOSA_API const char* nosa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* NOSA_B200_H */
