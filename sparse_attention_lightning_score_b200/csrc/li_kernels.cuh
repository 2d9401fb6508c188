// Kernel launchers of the li library (host-callable, internal).  Arguments are
// validated by the C-ABI layer (li_abi.cu) before any of these is reached.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "li.h"
#include "li_common.cuh"

namespace li {

// ---------------------------------------------------------------- streaming scorer
struct StreamArgs {
    const void* q;          // FP8 kind: bf16 [B,H,128]; BF16 kind: bf16 [B,H,256]
    const float* w;         // [B,H]
    int heads;              // H: 64 or 32
    const float* kscale;    // FP8 kind: one per cache row
    const int32_t* len;     // [B] or nullptr
    float* scores;
    long long scores_ld;
    long long batch_rows;   // cache rows between requests (0 = shared cache)
    int max_len;
    int tiles_per_cta;      // set by the launcher
    uint32_t* hist;         // optional: [B, LI_HIST_BINS] counts of order_key(score) >> LI_HIST_SHIFT are
                            // added to it (the caller provides it zeroed)
    int w_bulk;             // FP8: w is 16-byte aligned, so its rows can come in by bulk copy
    int tokens;             // query rows per request (multi-token decode; >= 1): row r belongs to request
                            // r / tokens and sees len - (tokens - 1 - r % tokens) positions of its cache
    DevErr err;
};
li_status launch_stream_score_fp8(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max,
                                  cudaStream_t st);
li_status launch_stream_score_fp8_hist(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max,
                                       cudaStream_t st);
li_status launch_stream_score_bf16(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max,
                                   cudaStream_t st);
li_status launch_stream_score_bf16_hist(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max,
                                        cudaStream_t st);

// ---------------------------------------------------------------- FP8 latent scorer (d_c = 192)
struct Latent8Args {
    const void* q;          // absorbed query q~, bf16 [B,64,192]
    const float* w;         // [B,64]
    const float* cscale;    // one fp32 per latent row
    const int32_t* len;     // [B] or nullptr
    float* scores;
    long long scores_ld;
    long long batch_rows;   // latent rows between requests (0 = shared cache)
    int max_len;
    int tiles_per_cta;      // set by the launcher
    uint32_t* hist;         // optional [B, LI_HIST_BINS] first-digit counts, added to
    DevErr err;
};
li_status launch_latent8_score(const CUtensorMap& map, const Latent8Args& args, int batch, int ntiles_max,
                               cudaStream_t st);

// ---------------------------------------------------------------- causal prefill scorer
struct PrefillArgs {
    const float* w_eff;     // [T,64] (w * per-(token, head) query scale)
    const float* kscale;    // [L]
    float* scores;
    long long scores_ld;
    int T, L;
    int causal_offset;
    DevErr err;
};
li_status launch_prefill_score(const CUtensorMap& qmap, const CUtensorMap& kmap, const PrefillArgs& args,
                               cudaStream_t st);

// ---------------------------------------------------------------- copy from mapped host memory
li_status launch_host_copy(void* dst, const void* src, size_t bytes, cudaStream_t st);

// ---------------------------------------------------------------- query quantiser
li_status launch_quantize_query(const void* q, const float* w, int rows, int heads, int dim, uint8_t* q8, float* sq,
                                float* w_eff, cudaStream_t st);

// ---------------------------------------------------------------- exact fp32 scorer
struct SimtArgs {
    const float* q;         // [R,H,d]
    const float* w;         // [R,H]
    const float* k;         // rows of d
    const int32_t* len;
    float* scores;
    long long scores_ld;
    long long batch_rows;
    int R, H, d, L;
    int causal, causal_offset;
    DevErr err;
};
li_status launch_simt_score(const SimtArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- top-k
struct TopkArgs {
    const float* scores;
    long long ld;
    const int32_t* len;
    int rows, max_len, causal, causal_offset, k;
    int32_t* idx;
    float* vals;
    // optional position map (hierarchical selection): row r's slot i reports
    // map[(r % map_rows) * map_ld + i] instead of i
    const int32_t* map;
    long long map_ld;
    int map_rows;
    // optional [rows, LI_HIST_BINS] histogram of the rows' keys by their top
    // LI_HIST_BITS bits (counted by the decode scorer); the top-k takes its first
    // digit from it and leaves it all zero
    uint32_t* hist;
    int cand_cap;           // set by the launcher: candidate keys one CTA can hold
    int tokens;             // query rows per request, as for the scorer (0 or 1: one row per len entry)
    DevErr err;
    // optional (shard merge): row r's length from nparts lists of part_k slots each,
    // len_parts[r * nparts + p] = valid slots at the head of list p | 0x80000000 if list p has a
    // valid slot after a pad.  The row is the valid prefix of the lists side by side; a valid slot
    // after it is reported as a bounds error and left out.
    const int32_t* len_parts;
    int nparts, part_k;
};
li_status launch_topk(const TopkArgs& a, cudaStream_t st);

// ---------------------------------------------------------------- L-sharded selection merge
// parts: [rows, shards] valid-prefix counts per list (the top-k's len_parts); hist (optional):
// [rows, LI_HIST_BINS], zero on entry, receives the valid candidates' first digits
li_status launch_merge_prep(const float* vals, const int32_t* idx, int shards, int rows, int k, long long shard_len,
                            float* mvals, int32_t* mpos, int32_t* parts, long long ld, uint32_t* hist,
                            const DevErr& err, cudaStream_t st);

// ---------------------------------------------------------------- absorption
li_status launch_absorb(const void* q, const void* wdec, void* qt, int G, int B, int H, int d, int dc,
                        cudaStream_t st);

// ---------------------------------------------------------------- HS gather + rescore
struct HsArgs {
    const void* c;          // bf16 latent rows of 256
    long long batch_rows;
    long long cache_rows;   // rows addressable from c
    const int32_t* cand;    // [B, C]
    int B, C, F;
    int H;                  // heads per follower: 64 or 32
    const void* qt;         // bf16 [F,B,H,256]
    const float* w;         // [F,B,H]
    float* out;             // [F,B,C] candidate scores (workspace)
    uint32_t* hist;         // optional [F*B, LI_HIST_BINS]: out's first-digit counts are added here
    DevErr err;
};
// qmap: q~ as [F * B * H, 256] bf16, box 64 x H, 128-byte swizzle
li_status launch_hs_rescore(const CUtensorMap& qmap, const HsArgs& a, cudaStream_t st);

// HS over DeepSeek-V3.2's FP8 latent: e4m3 rows of 192 with one fp32 scale per row, 64 heads per follower
struct Hs8Args {
    const void* c8;         // e4m3 latent rows of 192 bytes
    const float* cscale;    // one fp32 per latent row, same numbering
    long long batch_rows;
    long long cache_rows;   // rows addressable from c8
    const int32_t* cand;    // [B, C]
    int B, C, F;
    const void* qt;         // bf16 [F,B,64,192]
    const float* w;         // [F,B,64]
    float* out;             // [F,B,round4(C)] candidate scores (workspace)
    uint32_t* hist;         // optional [F*B, LI_HIST_BINS]: out's first-digit counts are added here
    DevErr err;
};
li_status launch_hs_rescore8(const Hs8Args& a, cudaStream_t st);

// ---------------------------------------------------------------- sparse attention over a selection
struct SparseAttnArgs {
    const void* q;          // bf16 [batch, heads, 576]
    const void* kv;         // bf16 rows of 576; request b's rows begin at row b * batch_rows
    long long batch_rows;   // 0 = one cache shared by every request
    long long rows_visible; // rows a selection may address
    const int32_t* sel;     // [batch, k] cache rows, -1 = none
    int batch, heads, k;
    int splits;             // set by the launcher: ceil(k / 256)
    float scale;            // softmax scale applied to q . kv
    float* opart;           // [batch, splits, heads, 512] unnormalised split outputs (workspace)
    float* mpart;           // [batch, splits, heads] split maxima, log2 domain (workspace)
    float* lpart;           // [batch, splits, heads] split sums of exponentials (workspace)
    float* out;             // fp32 [batch, heads, 512]
    DevErr err;
};
size_t sparse_attn_workspace_bytes(int batch, int heads, int k);
int sparse_attn_splits(int k);
// qmap: q as [batch * heads, 576] bf16, box 64 x 64, 128-byte swizzle
li_status launch_sparse_attn(const CUtensorMap& qmap, SparseAttnArgs a, cudaStream_t st);

// ---------------------------------------------------------------- diagnostics
li_status launch_selftest_wait(unsigned long long limit_ns, cudaStream_t st);

}  // namespace li
