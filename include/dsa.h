/*
 * dsa.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * Three steps, each one call, plus a fused forward:
 *   dsa_indexer_scores   lightning-indexer scores of every query against every
 *                        causally preceding index key
 *   dsa_topk             per-query top-k token selection over those scores
 *   dsa_sparse_mla_attn  MLA attention (absorbed MQA form) over the selected rows
 *   dsa_forward          the three in sequence, chunked over query rows
 *
 * Conventions shared by every entry point
 *  - Every tensor pointer is DEVICE memory owned by the caller; the library
 *    never allocates, frees or keeps a pointer after the call returns (its
 *    one device array, the scratch of dsa_forward_static_scratch, is static
 *    and comes with the library's device code).
 *  - Calls are asynchronous on `stream`.  Argument errors are detected on the
 *    host and returned before anything is launched; nothing is written then.
 *  - The decode indexer (at most one query row per sequence), the top-k and
 *    the sparse attention are launched with programmatic stream serialisation:
 *    they may start while the kernel before them on `stream` finishes, and
 *    wait for it to complete before they read or write any memory it may use,
 *    so the results are those of plain stream order.  (Only this library's
 *    kernels release their successor early; after any other kernel the
 *    launch waits for it as usual.)
 *  - Sequences are packed ("varlen"): sequence b owns query rows
 *    [cu_q[b], cu_q[b+1]) and key/cache rows [cu_k[b], cu_k[b+1]).  The new
 *    queries are the last q_len_b tokens of the sequence, so local query i sits
 *    at absolute position pos = kv_len_b - q_len_b + i and may attend to keys
 *    0..pos (its own position included: the causal mask is -inf strictly above
 *    the diagonal -- "DeepSeek-V3.2-Exp" token-ids page, "Position IDs").
 *    Key indices in scores and idx are sequence-local (0 = first key of the
 *    sequence).  The caller appends the new tokens to the index-key cache and to
 *    the latent cache before the call ("DeepSeek-V3.2", transformers doc: besides
 *    the main cache, the indexer stores one single-head key per token in a
 *    cache of its own, refreshed before scoring).
 *  - A query range [q_begin, q_end) of global query rows selects the rows a
 *    call processes.  Tensors indexed by query row (q_idx, w, q, out, lse) are
 *    addressed by GLOBAL row; the scores and idx buffers of the stage calls are
 *    CHUNK-relative: their row r belongs to global row q_begin + r.
 *  - Supported shapes: the released layer (index heads 64, index dim 128,
 *    attention heads 128, q/k dim 576 = 512 latent + 64 RoPE, v dim 512) and a
 *    tiny test shape (4, 32 | 4, 80, 64).  Others return DSA_ERR_UNSUPPORTED.
 *  - Device-side waits are bounded.  If one gives up, the kernel records a code
 *    in a library-global device word, skips its remaining work and returns;
 *    dsa_device_error() reads and clears it.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* null pointer, bad length, misaligned buffer, ... */
  DSA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set */
  DSA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  DSA_ERR_DEVICE_TIMEOUT = 4,/* a bounded device-side wait gave up (see dsa_device_error) */
  DSA_ERR_WORKSPACE = 5      /* workspace missing or smaller than dsa_forward_workspace_size */
} dsa_status;

typedef enum {
  DSA_KIDX_BF16 = 0,        /* index keys stored as bf16 [sum kv, idx_dim] */
  DSA_KIDX_FP8_E4M3 = 1     /* index keys stored as e4m3 bytes [sum kv, idx_dim] plus one fp32
                               scale per key: k = e4m3(byte) * k_scale[key] */
} dsa_kidx_dtype;

/* Sequence layout.  The device and host copies must hold the same values:
 * cu_q[0] = cu_k[0] = 0, non-decreasing, q_len_b <= kv_len_b.  kv_len_b =
 * cu_k[b+1] - cu_k[b] is the number of cache entries of sequence b (its new
 * tokens included).
 *
 * Caches ("DeepSeek-V3.2", transformers doc, DSA: the indexer's per-token key
 * cache is kept beside the main cache, in a growing or a preallocated cache
 * layer).  The index-key cache (with its scales) and the latent cache share
 * one row layout:
 *  - packed (block_table NULL; the page fields are then ignored): entry s of
 *    sequence b is cache row cu_k[b] + s, and the caches hold cu_k[B] rows;
 *  - paged: a pool of n_pages pages of page_size rows; entry s of sequence b
 *    is row s % page_size of page block_table[b * pages_per_seq + s / page_size].
 *    page_size is a power of two >= 64, pages_per_seq * page_size >= every kv_len,
 *    n_pages * page_size <= 2^31 - 1, block_table 4-byte aligned (else
 *    DSA_ERR_INVALID_ARG).  The table lives on the device and is not read by
 *    the host: a page entry outside [0, n_pages) reads as zeros in the
 *    indexer, makes the attention skip that entry and records device error
 *    code 2 (see dsa_device_error); it never causes an access outside the
 *    caches. */
typedef struct {
  int32_t batch;              /* B >= 1 */
  const int32_t* cu_q;        /* device, [B+1]: query-row offsets */
  const int32_t* cu_k;        /* device, [B+1]: cache-entry offsets */
  const int32_t* cu_q_host;   /* host,   [B+1]: same values as cu_q */
  const int32_t* cu_k_host;   /* host,   [B+1]: same values as cu_k */
  const int32_t* block_table; /* device, [B, pages_per_seq] page ids, or NULL (packed caches) */
  int32_t page_size;          /* rows per page (paged): a power of two >= 64 */
  int32_t pages_per_seq;      /* row stride of block_table (paged) */
  int64_t n_pages;            /* pages in the pool (paged) */
} dsa_varlen;

/*
 * Step 1: lightning-indexer scores.
 * Source: "DeepSeek-V3.2" (transformers model doc), section "DeepSeek Sparse
 * Attention (DSA)", item 1 -- a cheap module with few heads scores every key
 * at or before each query's position; the released config has index_n_heads 64 and
 * index_head_dim 128 ("DeepSeek-V3.2-Exp" token-ids page).  Score:
 *     I[t,s] = sum_j w[t,j] * max(0, q_idx[t,j,:] . k[s,:]),   0 <= s <= pos(t)
 * q_idx     bf16 [T, n_idx_heads, idx_dim], row-major, global rows; or, for
 *           the FP8 indexer (q_scale not NULL), e4m3 bytes of the same shape
 *           from dsa_hadamard_quantize_fp8
 * q_scale   NULL (bf16 queries), or fp32 [T, n_idx_heads]: the scale of each
 *           query head vector from dsa_hadamard_quantize_fp8.  The keys must
 *           then be e4m3 prepared the same way (k_dtype DSA_KIDX_FP8_E4M3);
 *           the MMAs take both e4m3 operands as they are and the score is
 *           sum_j w[t,j] q_scale[t,j] 2^-7 max(0, qq[t,j,:] . kq[s,:]) k_scale[s]
 *           (2^-7 undoes the factor 128 of the unnormalised rotation).
 *           Released shape only.
 * w         fp32 [T, n_idx_heads]
 * k_idx     bf16 or e4m3 bytes [sum kv, idx_dim] (see dsa_kidx_dtype);
 *           k_scale fp32 [sum kv] for e4m3, NULL for bf16
 * scores    fp32 [q_end - q_begin, ld_scores], chunk-relative rows.  Row r
 *           receives columns 0..pos(q_begin+r); columns past the diagonal in
 *           the same 128-key tile are set to -inf; later columns are not
 *           written.  ld_scores >= the longest kv_len among the rows.
 * part_max  fp32 [q_end - q_begin, ld_part_max] or NULL: the first step of
 *           the top-k, done in the same epilogue.  Element (r, p) is the
 *           largest score of keys 8p .. 8p+7 of row r that are <= pos (keys
 *           past pos count as -inf); written for every part whose first key
 *           is inside the sequence.  ld_part_max >= ceil(longest kv_len / 8),
 *           a multiple of 4.  dsa_topk given these maxima reads only the
 *           parts of the row that can hold a selected key.
 * Accumulation is fp32 (bf16 x bf16 products are exact); for e4m3 keys the
 * per-key scale multiplies the head-reduced score (scale > 0 commutes with ReLU).
 * With e4m3 keys and at most one query row per sequence (the decode kernel),
 * the tensor cores multiply f16 operands: the keys widen exactly, and each
 * query tile (all heads of the row) is multiplied by the power of two 2^sq
 * that puts its largest magnitude 2^E(1+f) below 2^15 and rounded to f16 --
 * exact for every element of magnitude >= 2^(E-31), smaller ones move by at
 * most 2^(E-39) -- and the score by 2^-sq.
 * Alignment: all tensors 16-byte aligned; ld_scores a multiple of 4.
 */
dsa_status dsa_indexer_scores(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                              const float* k_scale, dsa_kidx_dtype k_dtype, dsa_varlen v,
                              int32_t n_idx_heads, int32_t idx_dim, int64_t q_begin,
                              int64_t q_end, float* scores, int64_t ld_scores, float* part_max,
                              int64_t ld_part_max, cudaStream_t stream);

/*
 * Step 2: fine-grained token selection.
 * Source: "DeepSeek-V3.2" (transformers model doc), section "DeepSeek Sparse
 * Attention (DSA)", item 2 -- every query retains the index_topk (default
 * 2048) keys with the highest scores.  Ties are broken toward the lower key
 * index; -0.0 ties +0.0.
 * scores    fp32 [q_end - q_begin, ld_scores] chunk-relative, as written by
 *           dsa_indexer_scores (only columns 0..pos(t) are read)
 * part_max  NULL, or the part maxima dsa_indexer_scores wrote beside these
 *           scores (same rows, layout as described there).  With them, a row
 *           with at least 1.25 topk parts and at most 262,144 keys is selected
 *           from the maxima and the parts whose maximum reaches the topk-th
 *           largest maximum; the result is the same set.  Maxima that do not
 *           belong to the scores give a wrong selection (never an access
 *           outside the row).
 * idx       int32 [q_end - q_begin, topk] chunk-relative.  Row r holds the
 *           min(topk, pos+1) selected sequence-local key indices followed by
 *           -1.  With pos+1 <= topk that is 0..pos.  The SET is the
 *           definition; the order within a row is unspecified but
 *           deterministic, so repeated runs are bit-identical.
 * topk in [1, 2048].  Scores must not be NaN.  Rows longer than 1,040,384
 * keys return DSA_ERR_UNSUPPORTED (nothing launched).
 */
dsa_status dsa_topk(const float* scores, int64_t ld_scores, const float* part_max, int64_t ld_part_max,
                    dsa_varlen v, int64_t q_begin, int64_t q_end, int32_t topk, int32_t* idx,
                    cudaStream_t stream);

/*
 * Step 3: MLA attention in absorbed MQA form over the selected rows.
 * Sources: "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse
 * Attention (DSA)", item 2 -- main MLA attention is computed only over the
 * selected tokens; "DeepSeek-V3.2 - Experimental Exp Version" (altools),
 * "Technical Principles" -- MLA with MQA, key entries shared by all query
 * heads; "DeepSeek-V3.2 / Exp" (visual-learn explainer) -- the cached entries
 * are MLA's compressed vectors.  For query row t, head h, selected row s:
 *     z_s = scale * q[t,h,:d_qk] . latent[s,:d_qk]
 *     out[t,h,:] = sum_s softmax(z)_s * latent[s, :d_v],   lse[t,h] = log sum_s exp(z_s)
 * q         bf16 [T, n_heads, d_qk] global rows: per head the d_v-wide absorbed
 *           query then the (d_qk - d_v)-wide RoPE part
 * latent    bf16 [sum kv, d_qk]: per token the 512-d latent then the 64-d RoPE key
 *           (already rotated at its own position)
 * rope_cs   NULL: q's RoPE part is used as given (already rotated).  Otherwise
 *           fp32 [rope_max_pos, (d_qk - d_v) / 2, 2], 8-byte aligned: the
 *           (cos, sin) of each position and rotation pair ("DeepSeek-V3.2-Exp"
 *           token-ids page, released config: qk_rope_head_dim 64).  The
 *           kernel rotates the RoPE part of every query row at its position
 *           pos(t) while loading it: element pair (2i, 2i+1) of that part,
 *           read as the complex number x_2i + i x_2i+1, is multiplied by
 *           cos + i sin of entry [pos(t)][i] (fp32, rounded back to bf16).
 *           rope_max_pos must be at least the longest kv length of the range.
 * idx       int32 [q_end - q_begin, topk] chunk-relative, sequence-local rows.
 *           Entries outside 0..pos(t) (including the -1 padding) are ignored.
 * out       bf16 [T, n_heads, d_v] global rows; lse fp32 [T, n_heads] (nullable).
 *           A row with no valid entry gets out = 0 and lse = -inf.
 * QK and PV run on the tensor cores (bf16 in, fp32 accumulate); the softmax
 * probabilities are rounded to bf16 for PV.  topk in [1, 2048]; any value in
 * that range (the rows are processed in tiles of 32 and the tail of the last
 * tile is skipped).
 */
dsa_status dsa_sparse_mla_attn(const void* q, const void* latent, const int32_t* idx,
                               dsa_varlen v, int64_t q_begin, int64_t q_end, int32_t topk,
                               int32_t n_heads, int32_t d_qk, int32_t d_v, float scale,
                               const float* rope_cs, int64_t rope_max_pos,
                               void* out, float* lse, cudaStream_t stream);

/*
 * Inputs of the FP8 indexer.
 * Source: "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse
 * Attention (DSA)", item 1 -- DeepSeek's own indexer scores in e4m3 after a
 * Hadamard rotation of both operands (rotate_activation); "DeepSeek-V3.2-Exp" token-ids page,
 * released config: scale_fmt ue8m0 (power-of-two scales).
 * Each of the n vectors of 128 values is rotated by the Sylvester-Hadamard
 * matrix H (entries +-1, H[i][j] = (-1)^popcount(i & j), not normalised) and
 * quantized: scale[v] = 2^e with e the smallest integer such that
 * max|Hx| <= 448 * 2^e (scale 1 for a zero vector), q[v, i] = the e4m3 byte
 * nearest to (Hx)_i / scale[v] (ties to even).  Index queries ([T * 64]
 * vectors) and index keys ([sum kv] vectors) prepared this way are the FP8
 * indexer's operands (dsa_indexer_scores with q_scale); since
 * (Hq).(Hk) = 128 (q.k), that score divides the factor 128 back out.
 * x  bf16 [n, 128];  q  e4m3 bytes [n, 128];  scale  fp32 [n].
 * x and q 16-byte aligned.
 */
dsa_status dsa_hadamard_quantize_fp8(const void* x, int64_t n, void* q, float* scale, cudaStream_t stream);

/* How dsa_cache_append stores an index key. */
typedef enum {
  DSA_KQ_BF16 = 0,           /* bf16 copy (a DSA_KIDX_BF16 cache) */
  DSA_KQ_E4M3_AMAX = 1,      /* e4m3, scale = amax / 448 in fp32 (1 for a zero key), byte = nearest e4m3
                                (ties to even) to the fp32 quotient x / scale (a DSA_KIDX_FP8_E4M3 cache) */
  DSA_KQ_E4M3_HADAMARD = 2   /* the Hadamard rotation and power-of-two scale of dsa_hadamard_quantize_fp8:
                                the keys of the FP8 indexer (dsa_indexer_scores with q_scale) */
} dsa_kidx_quant;

/*
 * Appends a step's new tokens to the caches (the update before scoring).
 * Source: "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse
 * Attention (DSA)": besides the main cache, the indexer stores one
 * single-head key per token in a cache of its own, refreshed each step
 * (update_indexer), in a growing or a preallocated cache layer; "DeepSeek-V3.2-Exp" token-ids page, released
 * config: kv_lora_rank 512, qk_rope_head_dim 64, index_head_dim 128.
 * The new tokens are the step's query rows: global row t is entry pos(t) of
 * its sequence (v's kv lengths already count the new tokens), stored at that
 * entry's cache row (packed or paged, see dsa_varlen).
 * latent_new   bf16 [T, d_qk] or NULL: the new latent rows; latent_cache bf16
 *              [cache rows, d_qk] (NULL with latent_new NULL).  (d_qk, d_v) is
 *              (576, 512) or (80, 64).
 * rope_cs      NULL (latents stored as given), or fp32 [rope_max_pos,
 *              (d_qk - d_v) / 2, 2] (cos, sin), 8-byte aligned: columns from
 *              d_v on are rotated at pos(t) as dsa_sparse_mla_attn rotates
 *              queries (fp32, rounded to bf16).  rope_max_pos >= longest kv.
 * kidx_new     bf16 [T, idx_dim] or NULL: the new index keys; k_cache [cache
 *              rows, idx_dim] bf16 (DSA_KQ_BF16, idx_dim 128 or 32) or e4m3
 *              bytes (the two e4m3 forms, idx_dim 128) with k_scale fp32
 *              [cache rows].
 * Buffers 16-byte aligned (k_scale 4).  Entries whose page is missing are not
 * written and record device error code 2.  Other cache rows are untouched.
 */
dsa_status dsa_cache_append(const void* latent_new, const void* kidx_new, dsa_varlen v, int32_t d_qk, int32_t d_v,
                            int32_t idx_dim, const float* rope_cs, int64_t rope_max_pos, dsa_kidx_quant k_quant,
                            void* latent_cache, void* k_cache, float* k_scale, cudaStream_t stream);

/*
 * Per-head value up-projection of the attention output (the end of step 3).
 * Source: "DeepSeek-V3.2" (transformers model doc), "DeepSeek Sparse
 * Attention (DSA)": MLA, whose cached entries (the compressed latents) are
 * shared by all heads, so the absorbed attention of dsa_sparse_mla_attn leaves
 * each head's output in the 512-wide latent space; "DeepSeek-V3.2-Exp"
 * token-ids page, released config: kv_lora_rank 512, v_head_dim 128,
 * n_heads 128.  Each head h has its own W_UV[h] of [d_c, d_v]:
 *     y[r, h, e] = sum_c o[r, h, c] * W_UV[h, c, e]
 * o     bf16 [n_rows, n_heads, d_c] (the out of dsa_sparse_mla_attn)
 * w_uv  bf16 [n_heads, d_c, d_v], row-major; y  bf16 [n_rows, n_heads, d_v]
 * All three 16-byte aligned.  Released shape only (128, 512, 128), else
 * DSA_ERR_UNSUPPORTED; n_rows <= 8,388,480.  Tensor cores, bf16 in, fp32
 * accumulate, y rounded to bf16 (nearest even).  n_rows = 0 is a no-op.
 */
dsa_status dsa_mla_up_proj(const void* o, const void* w_uv, int64_t n_rows, int32_t n_heads, int32_t d_c,
                           int32_t d_v, void* y, cudaStream_t stream);

/*
 * Bytes of device workspace dsa_forward needs for this layout when it runs at
 * most q_chunk query rows per pass (q_chunk <= 0: all rows in one pass).  The
 * workspace holds one pass's fp32 scores, their part maxima (one per 8 keys)
 * and the int32 selections.  Returns 0 for invalid arguments.
 */
size_t dsa_forward_workspace_size(dsa_varlen v, int32_t topk, int64_t q_chunk);

/*
 * The whole hot path for every query row: dsa_indexer_scores -> dsa_topk ->
 * dsa_sparse_mla_attn, in passes of at most q_chunk rows so that the score
 * buffer stays bounded; all launches go to `stream` in order.  Arguments as
 * for the three steps (q_scale not NULL: the FP8 indexer).  idx_out
 * (nullable) receives the selections of every row, [T, topk] int32, global
 * rows.  workspace: device, at least
 * dsa_forward_workspace_size(v, topk, q_chunk) bytes, 256-byte aligned.
 * Prefill, chunked prefill and decode are the same call: they differ only in
 * the lengths held by v.  Every pass's argument and launch-limit checks run
 * before the first launch, so an error status means nothing was launched.
 */
dsa_status dsa_forward(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                       const float* k_scale, dsa_kidx_dtype k_dtype, const void* q,
                       const void* latent, dsa_varlen v, int32_t n_idx_heads,
                       int32_t idx_dim, int32_t topk, int32_t n_heads, int32_t d_qk,
                       int32_t d_v, float scale, int64_t q_chunk, void* out, float* lse,
                       int32_t* idx_out, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/*
 * dsa_forward without a caller-provided workspace, for callers that cannot
 * allocate device memory: code whose device memory belongs to a host
 * framework or a preallocated pool that forbids cudaMalloc once serving has
 * started, or a latency-critical loop that cannot afford the device-wide
 * synchronisation cudaMalloc/cudaFree imply.  The pages describe no such
 * entry point; it exists only for those callers.
 *
 * Scratch (the fp32 scores and int32 selections of one pass) lives in one
 * file-scope device array of DSA_STATIC_SCRATCH_BYTES, which every GPU that
 * loads the library keeps until the process exits.  Inputs and outputs are
 * still the caller's, exactly as for dsa_forward; the query rows are processed
 * in the largest passes whose scratch fits the array.  The array holds one
 * query row of any layout the top-k supports (rows up to 1,040,384 keys;
 * longer rows return DSA_ERR_UNSUPPORTED as for dsa_forward); were a row's
 * scores and selections ever larger than the array, the call would return
 * DSA_ERR_WORKSPACE.  Either way nothing is launched.  Calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 * Device memory for the array: the CUDA runtime loads this library's device
 * code on a device lazily, at the first call into the library there (of any
 * entry point), and that load allocates the array and may synchronise the
 * device.  The first call of this entry point on a device also looks up the
 * array's device address (cudaGetSymbolAddress, with that device current).
 * So make one warm-up call per device before serving starts and before any
 * stream capture.  All calls on a device share the array and it
 * keeps the last call's contents; nothing in it needs to start at zero (every
 * score and selection is written before it is read).  Calls whose kernels
 * overlap on the GPU (other streams, other host threads) race on the array:
 * serialise them.
 */
#define DSA_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
dsa_status dsa_forward_static_scratch(const void* q_idx, const float* q_scale, const float* w, const void* k_idx,
                                      const float* k_scale, dsa_kidx_dtype k_dtype,
                                      const void* q, const void* latent, dsa_varlen v,
                                      int32_t n_idx_heads, int32_t idx_dim, int32_t topk,
                                      int32_t n_heads, int32_t d_qk, int32_t d_v, float scale,
                                      void* out, float* lse, int32_t* idx_out,
                                      cudaStream_t stream);

/* Reads and clears the device error word of the current device (synchronises
 * `stream` first).  *code = 0 when nothing was recorded.  Otherwise the low 8
 * bits give the kind and bits 8.. the site: kind 1, a bounded device-side
 * wait gave up (the kernel skipped its remaining work); kind 2, a paged cache
 * entry that was needed had no valid page (that entry was skipped). */
dsa_status dsa_device_error(int32_t* code, cudaStream_t stream);

/* Diagnostics for profiling builds (compiled with -DDSA_PROFILE_WAITS): for
 * each bounded-wait site (index = the site code recorded on a timeout), the
 * device cycles lane 0 of the waiting warps spent in completed waits and how
 * many such waits there were.  Synchronises the device; copies min(n, 64)
 * entries into the host arrays; reset != 0 clears the counters.  Regular
 * builds return DSA_ERR_UNSUPPORTED and touch nothing.  No counterpart on the
 * pages: it exists to attribute kernel time to pipeline stages. */
dsa_status dsa_debug_wait_profile(uint64_t* cycles, uint64_t* counts, int32_t n, int32_t reset);

/* Diagnostics: exercises the bounded-wait timeout path on the GPU without
 * faulting or hanging it.  Launches one CTA (one warp) on `stream` whose only
 * work is one bounded wait on an mbarrier that nothing ever arrives on; after
 * limit_cycles device cycles (1 .. 2e9; about 1 ms per 2e6 cycles at the
 * boost clock) the wait gives up the way every wait of the DSA kernels does:
 * it records 1 | (99 << 8) (timeout, wait site 99) in the device error word
 * and the kernel returns.  Read and clear the word with dsa_device_error()
 * before the next real call: kernels that start while it is set skip their
 * work.  No counterpart on the pages: it exists to test failure detection. */
dsa_status dsa_debug_wait_selftest(int64_t limit_cycles, cudaStream_t stream);

/* Static description of a status code. */
const char* dsa_status_string(dsa_status status);

/* Library version, "major.minor.patch". */
const char* dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
