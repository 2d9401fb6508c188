/*
 * li.h -- lightning-indexer scan for NVIDIA B200 (sm_100a): the C ABI.
 *
 * The lightning indexer of DeepSeek Sparse Attention gives every visible cache
 * position s of a query token t one score and keeps the k highest-scoring
 * positions for that layer's sparse attention (Multi-layer Indexer abstract:
 * a scan over the whole cache, then the k = 2048 best tokens; IndexCache
 * explainer, Symbol Map: each visible position gets one score, and top-k
 * follows).  The score computed here is
 *
 *     I[t,s] = sum_j w[t,j] * ReLU(q[t,j,:] . k[s,:])        (j < H heads)
 *
 * LatentIndex (LatentIndex abstract and Figure 1) replaces the per-layer key
 * cache of a G-layer group by one shared latent cache c, defines layer keys
 * through per-layer decoders k_j[s] = W_dec[j] c[s], and absorbs the decoder
 * into the query (q~_j = W_dec[j]^T q_j) so that the shared cache is scored
 * directly.  In hierarchical selection (HS) the anchor's full scan proposes a
 * candidate set that every follower re-scores and re-selects.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory and keeps no pointer after the call returns.
 *   - Tensors are dense, row-major, in the layouts stated per argument.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  No call synchronises the host, except li_get_last_error.
 *   - Arguments are validated on the host before anything is launched; a
 *     rejected call returns LI_ERR_INVALID_ARG or LI_ERR_UNSUPPORTED and has no
 *     effect.  LI_ERR_CUDA means a CUDA runtime call failed (no device, launch
 *     failure); the CUDA error is then cleared.  No exception or exit crosses
 *     this boundary.
 *   - Kernels never trap: a bounded wait that runs out or an index out of range
 *     sets a device-side error word, the kernel returns, and the next
 *     li_get_last_error reports it.
 */
#ifndef LI_H_
#define LI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* li_stream_t; /* same type as cudaStream_t */

typedef enum {
    LI_OK = 0,
    LI_ERR_INVALID_ARG = 1, /* a size, pointer, stride or alignment the call does not accept */
    LI_ERR_UNSUPPORTED = 2, /* a valid combination this build does not implement */
    LI_ERR_CUDA = 3,        /* a CUDA runtime call failed */
    LI_ERR_TIMEOUT = 4,     /* (device) a bounded wait inside a kernel ran out */
    LI_ERR_BOUNDS = 5       /* (device) a kernel met an index outside its tensor */
} li_status;

typedef enum {
    LI_DTYPE_F32 = 0,
    LI_DTYPE_BF16 = 1,
    LI_DTYPE_E4M3 = 2 /* OCP FP8 e4m3 ("fn": no infinities, max 448) */
} li_dtype;

/* Longest score row li_topk accepts, and the largest k. */
#define LI_TOPK_MAX_LEN 262144

/* Human-readable name of a status code (static storage). */
const char* li_status_string(li_status s);

/* Reads and clears the device error word of the current device after a
 * cudaDeviceSynchronize.  Returns LI_OK, LI_ERR_TIMEOUT, LI_ERR_BOUNDS, or
 * LI_ERR_CUDA when the synchronisation itself fails.  This is the only call
 * that blocks the host. */
li_status li_get_last_error(void);

/* ------------------------------------------------------------------------ */
/* Query quantisation (FP8 scoring needs an e4m3 query as well as e4m3 keys) */
/* ------------------------------------------------------------------------ */
/* The pages fix no query precision; the FP8 tensor-core score needs both
 * operands in e4m3.  Per (row, head), in fp32:
 *     sq     = absmax(q[r,j,:]) / 448        (1 when the head is all zero)
 *     q8     = e4m3(q[r,j,:] / sq)           (IEEE division, nearest-even, saturating at +-448)
 *     w_eff  = w[r,j] * sq
 * li_index_score performs this internally; this call exposes its bytes.
 *   q_bf16  [rows, heads, dim] bf16          w      [rows, heads] fp32
 *   q_e4m3  [rows, heads, dim] bytes (out)   q_scale[rows, heads] fp32 (out)
 *   w_eff   [rows, heads] fp32 (out; may be NULL together with w)
 * dim must be a multiple of 4 and at most 1024. */
li_status li_quantize_query(const void* q_bf16, const float* w, int rows, int heads, int dim,
                            uint8_t* q_e4m3, float* q_scale, float* w_eff, li_stream_t stream);

/* ------------------------------------------------------------------------ */
/* DSA lightning-indexer score (decode and causal prefill)                   */
/* ------------------------------------------------------------------------ */
typedef struct {
    int rows;          /* R: decode -> requests B (one query token each); prefill -> query tokens T */
    int heads;         /* H indexer heads */
    int dim;           /* d, the indexer key/query width */
    int max_len;       /* L: positions per request cache (decode) or of the shared cache (prefill) */
    int causal;        /* 0: row r sees positions s < len[r] (len NULL: s < L).
                          1: row t sees positions s <= t + causal_offset (and s < L) */
    int causal_offset; /* prefill: cache position of query row 0 */
    li_dtype q_dtype;  /* LI_DTYPE_BF16: quantised per (row, head) as li_quantize_query, FP8 tensor cores.
                          LI_DTYPE_F32 : exact fp32 scalar path (k_dtype must be LI_DTYPE_F32). */
    li_dtype k_dtype;  /* LI_DTYPE_E4M3 (k_scale required) or LI_DTYPE_F32 (k_scale NULL) */
    int tokens_per_request; /* decode with T query tokens per request (multi-token prediction), 0 or 1 = one.
                          Rows = requests * T; row r is token r % T of request r / T, reads that
                          request's cache (cache_batch_rows, len[] and the histogram's row count are
                          per request) and sees positions s < len[r / T] - (T - 1 - r % T): the
                          request's newest T tokens are its last T cache positions.  FP8 decode only. */
} li_score_desc;

/* Scores every visible cache position of every row:
 *     scores[r * scores_ld + s] = sk[s] * sum_j w_eff[r,j] * ReLU(q8[r,j,:] . k8[s,:])
 * which is I[r,s] of the header comment with q = q8*sq and k = k8*sk.
 * Each row's scan covers its entire cache (Multi-layer Indexer abstract).  In
 * prefill each token sees its prefix, its own position included (IndexCache
 * explainer, Why This Exists: the indexer runs over the prefix).
 *   q        [rows, heads, dim] (q_dtype)     w [rows, heads] fp32
 *   k        key rows of `dim` elements (k_dtype); request r's cache begins at row
 *            r * cache_batch_rows (0 = every row reads the same cache)
 *   k_scale  one fp32 per key row, same row numbering as k (E4M3 only)
 *   len      [rows] int32 visible lengths (decode; NULL = max_len; each must lie in [0, max_len])
 *   scores   fp32, row r at scores + r * scores_ld; only visible positions are written
 * Tensor-core path: dim == 128, k base 16-byte aligned, k_dtype E4M3; heads == 64
 * (DeepSeek-V3.2's indexer) or, for decode (causal == 0), heads == 32 (GLM-5's;
 * Multi-layer Indexer, Appendix settings table).
 * workspace: li_index_score_workspace(desc) bytes (0 for decode; may be NULL then). */
li_status li_index_score(const void* q, const float* w, const void* k, const float* k_scale,
                         int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                         const li_score_desc* desc, void* workspace, size_t workspace_bytes,
                         li_stream_t stream);

/* Bytes of device workspace li_index_score needs for this descriptor. */
size_t li_index_score_workspace(const li_score_desc* desc);

/* Workspace sizes by operation, in the one-call form (op, rows, max_len, k).
 * Each call's own *_workspace function gives the exact size for its full
 * argument set; this one returns a size that is enough for every call of the
 * operation with these sizes (a workspace larger than needed is accepted):
 *   LI_OP_SCORE          li_index_score over `rows` query rows of 64 heads x 128
 *                        (the causal prefill form; the decode forms need none)
 *   LI_OP_TOPK           li_topk: 0 (it takes no workspace)
 *   LI_OP_HS             li_hs_refine / li_hs_refine_fp8 with batch = rows,
 *                        n_cand = max_len and any follower count up to 4
 *   LI_OP_DECODE_SELECT  li_decode_select over `rows` rows (zero it once)
 * k is accepted for the form's sake and changes no size.  An unknown op or a
 * negative size returns 0. */
typedef enum { LI_OP_SCORE = 0, LI_OP_TOPK = 1, LI_OP_HS = 2, LI_OP_DECODE_SELECT = 3 } li_op;
size_t li_workspace_size(int op, int rows, int max_len, int k);

/* ------------------------------------------------------------------------ */
/* Top-k selection                                                           */
/* ------------------------------------------------------------------------ */
/* Keeps the k highest scores of each row (IndexCache explainer, Symbol Map:
 * the selected set holds k positions; k = 2,048 in the pages' models).
 * Order: larger score first, equal scores to the lower position, NaN below
 * every number, -0.0 equal to +0.0.  Row r holds n_r valid scores:
 * min(max_len, r + 1 + causal_offset) when causal, else len[r] (len NULL:
 * max_len).  The min(k, n_r) selected positions are written in ascending
 * position order, then -1 up to k.
 *   scores [rows] x scores_ld fp32 (scores_ld a multiple of 4, base 16-byte aligned)
 *   idx    [rows, k] int32 (out)      vals [rows, k] fp32 (out, nullable; pads -inf)
 * 1 <= k <= LI_TOPK_MAX_LEN, max_len <= LI_TOPK_MAX_LEN. */
li_status li_topk(const float* scores, int64_t scores_ld, const int32_t* len, int rows, int max_len, int causal,
                  int causal_offset, int k, int32_t* idx, float* vals, li_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Decode indexer step: score, then select                                   */
/* ------------------------------------------------------------------------ */
/* One decode step of the indexer: li_index_score in its decode form (causal
 * 0) followed by li_topk(k_top) on the same scores, with identical results.
 * The difference is internal.  The pages run the indexer as a full scan that
 * scores every visible position, with top-k after it (IndexCache explainer,
 * Symbol Map), and this call keeps that order.  While writing each score, the
 * scorer also counts it by the top 11 bits of the selection's order key.  The
 * top-k takes its first radix digit from those counts instead of sweeping the
 * row for it.
 *   q, w, k, k_scale, cache_batch_rows, len, scores, scores_ld, desc
 *           as li_index_score (desc->causal must be 0; tensor-core path only:
 *           BF16 query, E4M3 keys, heads 64 or 32, dim 128).  scores_ld must be a
 *           multiple of 4 and scores 16-byte aligned, as li_topk requires.
 *   k_top, idx, vals   as li_topk's k, idx, vals.
 *   workspace  li_decode_select_workspace(desc) bytes of device memory,
 *           256-byte aligned, holding one 2048-bin histogram per row.  It must
 *           be all zero before the first call (a cudaMemset after allocating
 *           it).  Each call leaves it all zero again when its kernels
 *           complete.  Calls that overlap in time must not share one.
 * If the workspace was not zero, the result is still exact, but slower:
 * the top-k checks the counts against the keys and runs its plain passes.
 * The next li_get_last_error then reports LI_ERR_BOUNDS.  The histogram is
 * zero again afterwards. */
li_status li_decode_select(const void* q, const float* w, const void* k, const float* k_scale, int64_t cache_batch_rows,
                           const int32_t* len, float* scores, int64_t scores_ld, const li_score_desc* desc, int k_top,
                           int32_t* idx, float* vals, void* workspace, size_t workspace_bytes, li_stream_t stream);

/* Bytes of zeroed device workspace li_decode_select needs: desc->rows * 8 KB,
 * rounded up to 256 (0 when desc->rows <= 0); the other fields do not change
 * it.  It is also the histogram buffer li_decode_score_hist and li_topk_hist
 * take. */
size_t li_decode_select_workspace(const li_score_desc* desc);

/* li_decode_select as its two kernels, for callers that place or time them
 * separately; li_decode_select is exactly this pair on one stream, with the
 * same arguments and workspace.
 * li_decode_select_score: the scan (li_decode_score_hist into the workspace).
 * li_decode_select_finish: the top-k from the scores and the workspace's
 *   counts (li_topk_hist); leaves the workspace zero.  Its result equals
 *   li_topk's (causal 0) on the same scores. */
li_status li_decode_select_score(const void* q, const float* w, const void* k, const float* k_scale,
                                 int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                                 const li_score_desc* desc, void* workspace, size_t workspace_bytes,
                                 li_stream_t stream);
li_status li_decode_select_finish(const float* scores, int64_t scores_ld, const int32_t* len,
                                  const li_score_desc* desc, int k_top, int32_t* idx, float* vals, void* workspace,
                                  size_t workspace_bytes, li_stream_t stream);

/* The same pair with the histogram as a plain argument (the form the latent
 * scan, the HS followers and the shard merge use as well).
 * li_decode_score_hist: li_index_score in its decode form (same arguments and
 *   restrictions as li_decode_select).  For every score it writes, it also
 *   adds 1 to hist[r * 2048 + (key >> 21)], where key is the score's order key
 *   (fp32 bits made monotonic: larger score, larger key; NaN lowest; -0.0
 *   as +0.0).  hist: [rows, 2048] uint32, 16-byte aligned, zero before the
 *   call; it is added to, not overwritten.
 * li_topk_hist: li_topk (causal 0) that takes its first digit from hist and
 *   leaves hist all zero.  tokens_per_request as in li_score_desc (len per
 *   request, rows = requests * T).  The result equals li_topk's for any hist.  When hist
 *   does not count exactly the row's scores, the call reports LI_ERR_BOUNDS
 *   through li_get_last_error and selects without it. */
li_status li_decode_score_hist(const void* q, const float* w, const void* k, const float* k_scale,
                               int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                               const li_score_desc* desc, uint32_t* hist, li_stream_t stream);
li_status li_topk_hist(const float* scores, int64_t scores_ld, const int32_t* len, int rows, int max_len, int k,
                       int32_t* idx, float* vals, uint32_t* hist, int tokens_per_request, li_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Page-locked host buffers used directly by the kernels                    */
/* ------------------------------------------------------------------------ */
/* A decode step's inputs and outputs are small (the query and weights in, k
 * positions per request out).  DMA copies of them cost more in a step than
 * their size suggests, so a caller may hand the kernels page-locked host
 * memory instead.
 * li_host_device_pointer: the device-side address of page-locked host memory
 *   (cudaHostGetDevicePointer); LI_ERR_INVALID_ARG when host_ptr is not
 *   page-locked memory mapped for the current device.  The address can be
 *   given to li_decode_select / li_topk as idx or vals: the kernels then write
 *   the selections straight into host memory (visible to the host once the
 *   stream has been synchronised).
 * li_copy_from_host: copies `bytes` from such a device-side address of host
 *   memory into device memory with a kernel (both 16-byte aligned), ordered on
 *   `stream` like any launch. */
li_status li_host_device_pointer(const void* host_ptr, void** dev_ptr);
li_status li_copy_from_host(void* dst, const void* src_mapped, size_t bytes, li_stream_t stream);

/* ------------------------------------------------------------------------ */
/* One long context split along L over several shards (GPUs)                */
/* ------------------------------------------------------------------------ */
/* Merges per-shard selections into the global top-k.  Each request's cache
 * is cut into `shards` consecutive slices of shard_len positions; shard p
 * selected the k best of its slice (li_decode_select or li_topk with values,
 * positions local to the slice).  The global top-k is the top-k of the union
 * of those candidates: a position among the k best of the whole cache is
 * among the k best of its own slice.  Order and ties are those of li_topk over
 * global positions (p * shard_len + local).
 *   vals [shards, rows, k] fp32 and idx [shards, rows, k] int32: the shards'
 *        outputs stacked in shard order (as an all-gather delivers them)
 *   out_idx [rows, k_out] int32 (global positions, ascending, -1 pads),
 *   out_vals [rows, k_out] fp32 (nullable)
 *   workspace  li_merge_shards_workspace(shards, rows, k) bytes, 256-byte aligned.
 *              Its last rows * 8 KB hold the candidates' first-digit histograms for
 *              the row top-k: zero the workspace once after allocating it; each call
 *              leaves them zero again.  If they were not zero, the result is the same,
 *              only slower, and LI_ERR_BOUNDS is reported.
 * shards * k <= LI_TOPK_MAX_LEN and shards * shard_len < 2^31.  Each shard's
 * list must hold its valid positions first; a request whose lists leave a
 * valid candidate after a pad (only possible if a shard other than the last
 * one the request reaches had fewer than k positions) is reported through
 * li_get_last_error as LI_ERR_BOUNDS. */
li_status li_merge_shards(const float* vals, const int32_t* idx, int shards, int rows, int k, int64_t shard_len,
                          int k_out, int32_t* out_idx, float* out_vals, void* workspace, size_t workspace_bytes,
                          li_stream_t stream);
size_t li_merge_shards_workspace(int shards, int rows, int k);

/* ------------------------------------------------------------------------ */
/* LatentIndex: decoder absorption and latent-cache scoring                  */
/* ------------------------------------------------------------------------ */
/* Absorbs one layer's key decoder into its queries (LatentIndex abstract,
 * Figure 1):  q~[b,j,:] = W_dec[j]^T q[b,j,:], accumulated in fp32 and rounded
 * once to bf16.
 *   q_bf16      [batch, heads, dim] bf16
 *   w_dec_bf16  [heads, dim, latent_dim] bf16 (maps a latent row to head j's key)
 *   q_tilde     [batch, heads, latent_dim] bf16 (out)
 * dim <= 256, latent_dim a multiple of 64, w_dec 16-byte aligned. */
li_status li_absorb_query(const void* q_bf16, const void* w_dec_bf16, void* q_tilde_bf16, int batch, int heads,
                          int dim, int latent_dim, li_stream_t stream);

/* li_absorb_query for `layers` layers of a group in one launch: layer l's query
 * is at q_bf16 + l*batch*heads*dim, its decoder at w_dec_bf16 +
 * l*heads*dim*latent_dim and its output at q_tilde_bf16 + l*batch*heads*latent_dim
 * (elements).  Same arithmetic per layer; 0 <= layers <= 65535. */
li_status li_absorb_query_layers(const void* q_bf16, const void* w_dec_bf16, void* q_tilde_bf16, int layers,
                                 int batch, int heads, int dim, int latent_dim, li_stream_t stream);

/* Scores the shared latent cache with absorbed queries:
 *     scores[b * scores_ld + s] = sum_j w[b,j] * ReLU(q~[b,j,:] . c[b,s,:])   for s < len[b]
 *   q_tilde [batch, heads, latent_dim] bf16     w [batch, heads] fp32
 *   c       latent rows of latent_dim bf16; request b's rows begin at row b * cache_batch_rows
 *   len     [batch] int32 or NULL (= max_len)
 * Tensor-core path (bf16): heads == 64 or 32, latent_dim == 256, c base 16-byte
 * aligned. */
li_status li_latent_score(const void* q_tilde_bf16, const float* w, const void* c_bf16, int64_t cache_batch_rows,
                          const int32_t* len, float* scores, int64_t scores_ld, int batch, int heads, int latent_dim,
                          int max_len, li_stream_t stream);

/* li_latent_score that also counts every score it writes into
 * hist[b * 2048 + (key >> 21)], key being the score's order key as for
 * li_decode_score_hist.  hist: [batch, 2048] uint32, 16-byte aligned and zero
 * before the call.  li_topk_hist then selects from the same scores, for
 * example the anchor's candidate set of hierarchical selection. */
li_status li_latent_score_hist(const void* q_tilde_bf16, const float* w, const void* c_bf16,
                               int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                               int batch, int heads, int latent_dim, int max_len, uint32_t* hist, li_stream_t stream);

/* The LatentIndex scan over an FP8 latent cache: latent rows stored in e4m3
 * with one fp32 scale per row, c = c8 * cs (per-row absmax / 448, as the DSA
 * key cache).  The latent width is 192, DeepSeek-V3.2's shared latent of 64
 * RoPE and 128 NoPE dimensions (LatentIndex appendix, Table 5).  The absorbed
 * bf16 query is quantised per (request, head) inside the call exactly as
 * li_quantize_query does, and the score is
 *     scores[b * scores_ld + s] = cs[s] * sum_j w_eff[b,j] * ReLU(q8[b,j,:] . c8[s,:])
 * for s < len[b], with w_eff = w * sq.
 *   q_tilde [batch, 64, 192] bf16 (16-byte aligned)   w [batch, 64] fp32
 *   c_e4m3  latent rows of 192 bytes (16-byte aligned); request b's rows begin
 *           at row b * cache_batch_rows (0 = one cache shared by all requests)
 *   c_scale one fp32 per latent row, same numbering
 *   hist    NULL, or [batch, 2048] uint32 first-digit counts added to as
 *           li_latent_score_hist does (zero before the call), for li_topk_hist
 * heads must be 64 and latent_dim 192 (LI_ERR_UNSUPPORTED otherwise). */
li_status li_latent_score_fp8(const void* q_tilde_bf16, const float* w, const void* c_e4m3, const float* c_scale,
                              int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                              int batch, int heads, int latent_dim, int max_len, uint32_t* hist, li_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Hierarchical selection: followers refine the anchor's candidates         */
/* ------------------------------------------------------------------------ */
/* LatentIndex abstract: the anchor proposes one candidate set, shared by its
 * followers, and each follower refines it on its own.  For every follower f and request b, each
 * candidate latent row c[b, cand[b,i]] is gathered once and scored against all
 * followers' absorbed queries,
 *     I_f[b,i] = sum_j w[f,b,j] * ReLU(q~[f,b,j,:] . c[b, cand[b,i], :]),
 * then the k best candidates by (score desc, cache position asc) are kept and
 * written as cache positions in ascending order, padded with -1.  Negative
 * candidates are padding and are never selected.  Candidates must be listed in
 * ascending cache position (li_topk's output order), padding last.
 *   c       latent rows as in li_latent_score     cand [batch, n_cand] int32
 *   q_tilde [followers, batch, heads, latent_dim] bf16   w [followers, batch, heads] fp32
 *   out_idx [followers, batch, k] int32 (out)
 * Candidates outside [0, rows of c) are reported as LI_ERR_BOUNDS by
 * li_get_last_error and are not read.  heads == 64 or 32, latent_dim == 256,
 * 1 <= followers <= 4, n_cand <= LI_TOPK_MAX_LEN.
 * workspace: workspace_bytes >= li_hs_refine_workspace(...) bytes of device
 *   memory, 16-byte aligned.  Its first part holds the candidate scores; its
 *   last followers * batch * 8 KB (from workspace_bytes back, rounded down to
 *   16 bytes) hold the rescoring kernel's first-digit histograms for the
 *   follower top-k, as li_topk_hist uses them.  Zero the workspace once after
 *   allocating it; each call leaves those histograms zero again when its
 *   kernels finish.  If they were not zero, the result is the same, only
 *   slower: the top-k checks each histogram against its keys, falls back to
 *   its plain passes and reports LI_ERR_BOUNDS through li_get_last_error. */
li_status li_hs_refine(const void* c_bf16, int64_t cache_batch_rows, int64_t cache_rows, const int32_t* cand,
                       int batch, int n_cand, const void* q_tilde_bf16, const float* w, int followers, int heads,
                       int latent_dim, int k, int32_t* out_idx, void* workspace, size_t workspace_bytes,
                       li_stream_t stream);

size_t li_hs_refine_workspace(int batch, int n_cand, int followers);

/* li_hs_refine over DeepSeek-V3.2's FP8 latent (LatentIndex appendix, Table 5:
 * 64 RoPE + 128 NoPE dimensions), the cache li_latent_score_fp8 scans: e4m3 rows
 * of 192 bytes with one fp32 scale per row.  Each follower's absorbed query is
 * quantised per (follower, request, head) as li_quantize_query does, so
 *     I_f[b,i] = cs[r] * sum_j w_eff[f,b,j] * ReLU(q8[f,b,j,:] . c8[b,r,:]),  r = cand[b,i].
 *   c_e4m3 / c_scale  rows and scales as in li_latent_score_fp8 (c_e4m3 16-byte aligned)
 *   q_tilde [followers, batch, 64, 192] bf16   w [followers, batch, 64] fp32
 * Everything else (candidates, ties, padding, output, errors, workspace) as
 * li_hs_refine.  heads == 64, latent_dim == 192, 1 <= followers <= 4
 * (LI_ERR_UNSUPPORTED otherwise). */
li_status li_hs_refine_fp8(const void* c_e4m3, const float* c_scale, int64_t cache_batch_rows, int64_t cache_rows,
                           const int32_t* cand, int batch, int n_cand, const void* q_tilde_bf16, const float* w,
                           int followers, int heads, int latent_dim, int k, int32_t* out_idx, void* workspace,
                           size_t workspace_bytes, li_stream_t stream);

/* Capacity, in floats (4 MiB), of the fixed scratch behind li_hs_refine_noalloc. */
#define LI_HS_NOALLOC_MAX_SCRATCH_FLOATS 1048576

/* li_hs_refine without a workspace argument, for callers that cannot
 * allocate device memory: for example code inside an engine that owns and
 * budgets all device memory and forbids allocation while serving, or a
 * plugin that receives only its inputs and outputs.  The pages have no
 * counterpart to this call; it exists only for such callers.
 *
 * Same arguments, results and errors as li_hs_refine.  The workspace
 * li_hs_refine would take -- the followers' candidate scores and the follower
 * top-k's histograms -- is a file-scope device array of
 * LI_HS_NOALLOC_MAX_SCRATCH_FLOATS floats that every GPU loading the library
 * holds until the process exits; the call allocates nothing.
 *   - Limit: li_hs_refine_workspace(batch, n_cand, followers) must not exceed
 *     4 * LI_HS_NOALLOC_MAX_SCRATCH_FLOATS bytes (4 MiB); a larger call returns
 *     LI_ERR_INVALID_ARG before anything is launched.  For example one
 *     follower and 4 requests take at most 260,096 candidates, three followers
 *     and 16 requests at most 19,796.
 *   - The array is shared by all calls on a device and keeps the last call's
 *     contents.  Each call clears its own histograms (the array's last
 *     followers * batch * 8 KB) with one cudaMemsetAsync on `stream` before its
 *     kernels, so what an earlier call of other sizes left there changes
 *     neither the result nor the status.  Calls that overlap on the GPU
 *     (unordered streams) race on the array: serialise them.
 *   - The first call on a device looks up the array's device address and
 *     caches it for the process; make that first call before any stream
 *     capture begins.  After cudaDeviceReset the cached address is stale. */
li_status li_hs_refine_noalloc(const void* c_bf16, int64_t cache_batch_rows, int64_t cache_rows, const int32_t* cand,
                               int batch, int n_cand, const void* q_tilde_bf16, const float* w, int followers,
                               int heads, int latent_dim, int k, int32_t* out_idx, li_stream_t stream);


/* ------------------------------------------------------------------------ */
/* The consumer: sparse attention over a selection                           */
/* ------------------------------------------------------------------------ */
/* Each new token of a DSA layer attends only the positions its indexer
 * selected (Multi-layer Indexer, long-version transcript: 2048 tokens per
 * layer, and the selection is the only link between indexer and attention).
 * This call is that attention in DeepSeek-V3.2's absorbed-MLA decode form: a
 * cache row is one 576-element bf16 vector (512 latent + 64 RoPE) shared by
 * every query head, the key is the whole row and the value its first 512
 * elements:
 *     out[b,h,:] = sum_i p_i * kv[b, sel[b,i], 0:512],
 *     p = softmax over the valid i of scale * (q[b,h,:] . kv[b, sel[b,i], :])
 * A selection is valid when 0 <= sel < cache_rows; -1 (a top-k pad) is skipped
 * and any other value outside that range is skipped and reported as
 * LI_ERR_BOUNDS by li_get_last_error.  A request with no valid selection gets
 * out = 0.
 *   q_bf16   [batch, heads, 576] bf16, 16-byte aligned; heads a multiple of 64
 *   kv_bf16  rows of 576 bf16 (1152 bytes); request b's rows begin at row
 *            b * cache_batch_rows (0 = one cache shared by every request)
 *   cache_rows  rows a selection may address (<= cache_batch_rows when that is > 0)
 *   sel      [batch, k] int32 cache rows (li_topk's output, any order)
 *   scale    softmax scale, finite and > 0
 *   out      [batch, heads, 512] fp32 (out), 16-byte aligned
 *   workspace  li_sparse_attention_workspace(batch, heads, k) bytes of device
 *            memory, 256-byte aligned (per 256 selections and head: 512 + 2 fp32)
 * Nothing is allocated and the host is not synchronised. */
size_t li_sparse_attention_workspace(int batch, int heads, int k);
li_status li_sparse_attention(const void* q_bf16, const void* kv_bf16, int64_t cache_batch_rows, int64_t cache_rows,
                              const int32_t* sel, int batch, int heads, int k, float scale, float* out,
                              void* workspace, size_t workspace_bytes, li_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Graphs whose kernels keep their streams' priorities                       */
/* ------------------------------------------------------------------------ */
/* Multi-layer Indexer (long-version transcript): the indexer runs on a second
 * stream beside attention and the rest of the layer, and the whole pattern is
 * captured once into the decode graph.  Kernels captured from a stream carry
 * that stream's priority, but a graph uses it only when it is instantiated
 * with node priorities; without them a side-stream indexer competes for SMs
 * on equal terms with the main stream's critical path.
 *   li_graph_instantiate: `graph` is a captured cudaGraph_t (e.g. torch's
 *     CUDAGraph(keep_graph=True).raw_cuda_graph()); with use_node_priority != 0
 *     the executable honours each kernel node's priority.  *exec receives a
 *     cudaGraphExec_t owned by the caller (li_graph_destroy); the graph itself
 *     stays the caller's.  LI_ERR_CUDA if the runtime rejects it.
 *   li_graph_launch: one replay of `exec` on `stream` (asynchronous).
 *   li_graph_destroy: frees `exec` (NULL is a no-op). */
li_status li_graph_instantiate(void* graph, int use_node_priority, void** exec);
li_status li_graph_launch(void* exec, li_stream_t stream);
li_status li_graph_destroy(void* exec);

/* ------------------------------------------------------------------------ */
/* Diagnostics                                                               */
/* ------------------------------------------------------------------------ */
/* Launches one block whose only work is the library's bounded wait on an
 * mbarrier that nothing ever arrives on, with the given limit in nanoseconds.
 * The wait runs out, the kernel records LI_ERR_TIMEOUT and returns; the next
 * li_get_last_error reports it.  Exercises the failure path of every
 * pipeline wait without faulting or hanging the device. */
li_status li_selftest_wait_timeout(uint64_t limit_ns, li_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LI_H_ */
