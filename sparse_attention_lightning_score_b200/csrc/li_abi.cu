// The exported C ABI of the li library (declared in include/li.h): argument
// validation, TMA tensor-map encoding, workspace carving and dispatch to the
// kernel launchers.  Nothing here allocates device memory or blocks the host
// (except li_get_last_error).
#include <cudaTypedefs.h>

#include <cstring>

#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

__device__ unsigned g_li_error_word;

namespace {

constexpr int kMaxDev = 64;

int current_device() {
    int d = 0;
    cudaGetDevice(&d);
    return d;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    }
    return fn;
}

// 2-D tensor map over `rows` rows of `row_elems` elements (row pitch
// `row_bytes`), box = [box_inner elements, box_rows rows], 128-byte swizzle.
bool encode_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t row_elems, uint64_t rows,
                   uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                   CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {row_elems, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The followers' first-digit histograms sit at the END of the workspace the caller gives (so
// that a fixed scratch shared by calls of different sizes keeps them in one place).
size_t hs_hist_bytes(int batch, int followers) { return (size_t)followers * batch * LI_HIST_BINS * sizeof(uint32_t); }
uint32_t* hs_hist_of(void* workspace, size_t workspace_bytes, int batch, int followers) {
    return reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) +
                                       ((workspace_bytes - hs_hist_bytes(batch, followers)) & ~(size_t)15));
}

}  // namespace

DevErr host_dev_err() {
    static unsigned* addr[kMaxDev] = {};
    const int d = current_device();
    if (d < kMaxDev && !addr[d]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_li_error_word) == cudaSuccess) addr[d] = static_cast<unsigned*>(p);
        else cudaGetLastError();
    }
    return DevErr{d < kMaxDev ? addr[d] : nullptr, kDefaultWaitLimitNs};
}

int host_num_sms() {
    static int n[kMaxDev] = {};
    const int d = current_device();
    if (d < kMaxDev && n[d] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) {
            cudaGetLastError();
            v = 148;
        }
        n[d] = v;
    }
    return d < kMaxDev ? n[d] : 148;
}

li_status host_check_launch() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LI_OK : LI_ERR_CUDA;
}

// The device must answer before any launch: an absent device or a missing
// error word becomes LI_ERR_CUDA instead of a fault.
static li_status ready(DevErr* e) {
    *e = host_dev_err();
    if (!e->word) return LI_ERR_CUDA;
    return LI_OK;
}

}  // namespace li

using namespace li;

extern "C" {

const char* li_status_string(li_status s) {
    switch (s) {
    case LI_OK: return "LI_OK";
    case LI_ERR_INVALID_ARG: return "LI_ERR_INVALID_ARG";
    case LI_ERR_UNSUPPORTED: return "LI_ERR_UNSUPPORTED";
    case LI_ERR_CUDA: return "LI_ERR_CUDA";
    case LI_ERR_TIMEOUT: return "LI_ERR_TIMEOUT";
    case LI_ERR_BOUNDS: return "LI_ERR_BOUNDS";
    }
    return "LI_ERR_UNKNOWN";
}

li_status li_get_last_error(void) {
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        return LI_ERR_CUDA;
    }
    unsigned v = 0;
    if (cudaMemcpy(&v, e.word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return LI_ERR_CUDA;
    }
    const unsigned zero = 0;
    if (v && cudaMemcpy(e.word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaGetLastError();
        return LI_ERR_CUDA;
    }
    if (v & ERRBIT_TIMEOUT) return LI_ERR_TIMEOUT;
    if (v & ERRBIT_BOUNDS) return LI_ERR_BOUNDS;
    return LI_OK;
}

li_status li_quantize_query(const void* q_bf16, const float* w, int rows, int heads, int dim, uint8_t* q_e4m3,
                            float* q_scale, float* w_eff, li_stream_t stream) {
    if (rows < 0 || heads <= 0 || dim <= 0 || dim > 1024 || (dim % 4) != 0) return LI_ERR_INVALID_ARG;
    if (rows == 0) return LI_OK;
    if (!q_bf16 || !q_e4m3 || !q_scale || (w_eff && !w)) return LI_ERR_INVALID_ARG;
    if (dim == 128 && !aligned(q_bf16, 8)) return LI_ERR_INVALID_ARG;
    if (!aligned(q_bf16, 2) || (dim == 128 && !aligned(q_e4m3, 4))) return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    return launch_quantize_query(q_bf16, w, rows, heads, dim, q_e4m3, q_scale, w_eff, stream);
}

size_t li_index_score_workspace(const li_score_desc* d) {
    if (!d || !d->causal || d->q_dtype != LI_DTYPE_BF16 || d->k_dtype != LI_DTYPE_E4M3 || d->rows <= 0) return 0;
    const size_t nh = (size_t)d->rows * d->heads;
    return align_up(nh * d->dim, 256) + 2 * align_up(nh * sizeof(float), 256);
}

li_status li_index_score(const void* q, const float* w, const void* k, const float* k_scale,
                         int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                         const li_score_desc* desc, void* workspace, size_t workspace_bytes, li_stream_t stream) {
    if (!desc) return LI_ERR_INVALID_ARG;
    const li_score_desc d = *desc;
    if (d.rows < 0 || d.heads <= 0 || d.dim <= 0 || d.max_len < 0 || cache_batch_rows < 0) return LI_ERR_INVALID_ARG;
    if (d.rows == 0 || d.max_len == 0) return LI_OK;
    if (!q || !w || !k || !scores || scores_ld < d.max_len) return LI_ERR_INVALID_ARG;
    if (d.causal && (cache_batch_rows != 0 || len)) return LI_ERR_INVALID_ARG;
    if (d.causal && (d.causal_offset < 0)) return LI_ERR_INVALID_ARG;
    const int T = d.tokens_per_request > 1 ? d.tokens_per_request : 1;
    if (d.rows % T != 0) return LI_ERR_INVALID_ARG;
    if (T > 1 && (d.causal || d.q_dtype != LI_DTYPE_BF16)) return LI_ERR_UNSUPPORTED;  // multi-token: FP8 decode
    const bool f32 = d.q_dtype == LI_DTYPE_F32 && d.k_dtype == LI_DTYPE_F32;
    if (!f32) {
        if (d.q_dtype != LI_DTYPE_BF16 || d.k_dtype != LI_DTYPE_E4M3) return LI_ERR_UNSUPPORTED;
        if ((d.heads != 64 && (d.heads != 32 || d.causal)) || d.dim != 128) return LI_ERR_UNSUPPORTED;
    }
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;

    if (f32) {
        if (k_scale || (size_t)d.heads * d.dim > 12000) return LI_ERR_UNSUPPORTED;
        SimtArgs a{static_cast<const float*>(q), w, static_cast<const float*>(k), len, scores, scores_ld,
                   cache_batch_rows, d.rows, d.heads, d.dim, d.max_len, d.causal, d.causal_offset, e};
        return launch_simt_score(a, stream);
    }
    if (!k_scale) return LI_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(q, 16)) return LI_ERR_INVALID_ARG;
    const uint64_t total_rows = cache_batch_rows > 0 ? (uint64_t)(d.rows / T - 1) * cache_batch_rows + d.max_len
                                                     : (uint64_t)d.max_len;
    if (total_rows >= (1ull << 31)) return LI_ERR_UNSUPPORTED;
    CUtensorMap kmap;
    if (!encode_map_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, k, 128, total_rows, 128, 128, 128)) return LI_ERR_CUDA;

    if (!d.causal) {
        StreamArgs a{};
        a.q = q;
        a.w = w;
        a.kscale = k_scale;
        a.len = len;
        a.scores = scores;
        a.scores_ld = scores_ld;
        a.batch_rows = cache_batch_rows;
        a.max_len = d.max_len;
        a.w_bulk = aligned(w, 16) ? 1 : 0;
        a.tokens = T;
        a.heads = d.heads;
        a.err = e;
        const int ntiles = (d.max_len + 127) / 128;
        return launch_stream_score_fp8(kmap, a, d.rows, ntiles, stream);
    }
    // causal prefill: quantise all query rows into the workspace, then score
    const size_t need = li_index_score_workspace(&d);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return LI_ERR_INVALID_ARG;
    const size_t nh = (size_t)d.rows * d.heads;
    uint8_t* q8 = static_cast<uint8_t*>(workspace);
    float* sq = reinterpret_cast<float*>(q8 + align_up(nh * d.dim, 256));
    float* weff = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sq) + align_up(nh * sizeof(float), 256));
    li_status s = launch_quantize_query(q, w, d.rows, d.heads, d.dim, q8, sq, weff, stream);
    if (s != LI_OK) return s;
    CUtensorMap qmap;
    if (!encode_map_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, q8, 128, nh, 128, 128, 256)) return LI_ERR_CUDA;
    PrefillArgs pa{weff, k_scale, scores, scores_ld, d.rows, d.max_len, d.causal_offset, e};
    return launch_prefill_score(qmap, kmap, pa, stream);
}

li_status li_topk(const float* scores, int64_t scores_ld, const int32_t* len, int rows, int max_len, int causal,
                  int causal_offset, int k, int32_t* idx, float* vals, li_stream_t stream) {
    if (rows < 0 || max_len < 0 || k < 1 || k > LI_TOPK_MAX_LEN || max_len > LI_TOPK_MAX_LEN) return LI_ERR_INVALID_ARG;
    if (rows == 0) return LI_OK;
    if (!idx || (!scores && max_len > 0) || scores_ld < max_len || (scores_ld % 4) != 0) return LI_ERR_INVALID_ARG;
    if (scores && !aligned(scores, 16)) return LI_ERR_INVALID_ARG;
    if (causal && len) return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    TopkArgs a{scores, scores_ld, len, rows, max_len, causal ? 1 : 0, causal_offset, k, idx, vals, nullptr, 0, 1,
                nullptr, 0, 1, e};
    return launch_topk(a, stream);
}

size_t li_decode_select_workspace(const li_score_desc* d) {
    if (!d || d->rows <= 0) return 0;
    return align_up((size_t)d->rows * LI_HIST_BINS * sizeof(uint32_t), 256);
}

li_status li_decode_score_hist(const void* q, const float* w, const void* k, const float* k_scale,
                               int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                               const li_score_desc* desc, uint32_t* hist, li_stream_t stream) {
    if (!desc) return LI_ERR_INVALID_ARG;
    const li_score_desc d = *desc;
    if (d.rows < 0 || d.heads <= 0 || d.dim <= 0 || d.max_len < 0 || cache_batch_rows < 0 || d.causal)
        return LI_ERR_INVALID_ARG;
    if (d.rows == 0 || d.max_len == 0) return LI_OK;
    if (d.q_dtype != LI_DTYPE_BF16 || d.k_dtype != LI_DTYPE_E4M3) return LI_ERR_UNSUPPORTED;
    if ((d.heads != 64 && d.heads != 32) || d.dim != 128) return LI_ERR_UNSUPPORTED;
    if (!q || !w || !k || !k_scale || !scores || !hist || scores_ld < d.max_len) return LI_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(q, 16) || !aligned(hist, 16)) return LI_ERR_INVALID_ARG;
    const int T = d.tokens_per_request > 1 ? d.tokens_per_request : 1;
    if (d.rows % T != 0) return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    const uint64_t total_rows = cache_batch_rows > 0 ? (uint64_t)(d.rows / T - 1) * cache_batch_rows + d.max_len
                                                     : (uint64_t)d.max_len;
    if (total_rows >= (1ull << 31)) return LI_ERR_UNSUPPORTED;
    CUtensorMap kmap;
    if (!encode_map_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, k, 128, total_rows, 128, 128, 128)) return LI_ERR_CUDA;
    StreamArgs a{};
    a.q = q;
    a.w = w;
    a.kscale = k_scale;
    a.len = len;
    a.scores = scores;
    a.scores_ld = scores_ld;
    a.batch_rows = cache_batch_rows;
    a.max_len = d.max_len;
    a.hist = hist;
    a.w_bulk = aligned(w, 16) ? 1 : 0;
    a.tokens = T;
    a.heads = d.heads;
    a.err = e;
    return launch_stream_score_fp8_hist(kmap, a, d.rows, (d.max_len + 127) / 128, stream);
}

li_status li_topk_hist(const float* scores, int64_t scores_ld, const int32_t* len, int rows, int max_len, int k,
                       int32_t* idx, float* vals, uint32_t* hist, int tokens_per_request, li_stream_t stream) {
    const int T = tokens_per_request > 1 ? tokens_per_request : 1;
    if (rows % T != 0) return LI_ERR_INVALID_ARG;
    if (rows < 0 || max_len < 0 || k < 1 || k > LI_TOPK_MAX_LEN || max_len > LI_TOPK_MAX_LEN) return LI_ERR_INVALID_ARG;
    if (rows == 0) return LI_OK;
    if (!idx || !hist || (!scores && max_len > 0) || scores_ld < max_len || (scores_ld % 4) != 0)
        return LI_ERR_INVALID_ARG;
    if ((scores && !aligned(scores, 16)) || !aligned(hist, 16)) return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    TopkArgs a{scores, scores_ld, len, rows, max_len, 0, 0, k, idx, vals, nullptr, 0, 1, hist, 0, T, e};
    return launch_topk(a, stream);
}

}  // extern "C"

namespace li {
namespace {

// The checks li_decode_select and its two halves share.
li_status check_decode_select(const void* q, const float* w, const void* k, const float* k_scale,
                              int64_t cache_batch_rows, const float* scores, int64_t scores_ld,
                              const li_score_desc* desc, int k_top, bool need_idx, const int32_t* idx,
                              const void* workspace, size_t workspace_bytes) {
    if (!desc) return LI_ERR_INVALID_ARG;
    const li_score_desc d = *desc;
    if (d.rows < 0 || d.heads <= 0 || d.dim <= 0 || d.max_len < 0 || cache_batch_rows < 0 || d.causal)
        return LI_ERR_INVALID_ARG;
    if (need_idx && (k_top < 1 || k_top > LI_TOPK_MAX_LEN)) return LI_ERR_INVALID_ARG;
    if (d.max_len > LI_TOPK_MAX_LEN) return LI_ERR_INVALID_ARG;
    if (d.rows == 0) return LI_OK;
    if (d.q_dtype != LI_DTYPE_BF16 || d.k_dtype != LI_DTYPE_E4M3) return LI_ERR_UNSUPPORTED;
    if ((d.heads != 64 && d.heads != 32) || d.dim != 128) return LI_ERR_UNSUPPORTED;
    if ((need_idx && !idx) || !workspace || workspace_bytes < li_decode_select_workspace(&d) ||
        !aligned(workspace, 256))
        return LI_ERR_INVALID_ARG;
    if (d.tokens_per_request > 1 && d.rows % d.tokens_per_request != 0) return LI_ERR_INVALID_ARG;
    if (d.max_len > 0) {
        if (!scores || scores_ld < d.max_len || (scores_ld % 4) != 0) return LI_ERR_INVALID_ARG;
        if (!aligned(scores, 16)) return LI_ERR_INVALID_ARG;
        if (!need_idx) {
            if (!q || !w || !k || !k_scale) return LI_ERR_INVALID_ARG;
            if (!aligned(k, 16) || !aligned(q, 16)) return LI_ERR_INVALID_ARG;
        }
    }
    return LI_OK;
}

}  // namespace
}  // namespace li

extern "C" {

li_status li_decode_select_score(const void* q, const float* w, const void* k, const float* k_scale,
                                 int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                                 const li_score_desc* desc, void* workspace, size_t workspace_bytes,
                                 li_stream_t stream) {
    li_status s = check_decode_select(q, w, k, k_scale, cache_batch_rows, scores, scores_ld, desc, 1, false, nullptr,
                                      workspace, workspace_bytes);
    if (s != LI_OK || desc->rows == 0 || desc->max_len == 0) return s;
    return li_decode_score_hist(q, w, k, k_scale, cache_batch_rows, len, scores, scores_ld, desc,
                                static_cast<uint32_t*>(workspace), stream);
}

li_status li_decode_select_finish(const float* scores, int64_t scores_ld, const int32_t* len,
                                  const li_score_desc* desc, int k_top, int32_t* idx, float* vals, void* workspace,
                                  size_t workspace_bytes, li_stream_t stream) {
    li_status s = check_decode_select(nullptr, nullptr, nullptr, nullptr, 0, scores, scores_ld, desc, k_top, true,
                                      idx, workspace, workspace_bytes);
    if (s != LI_OK || desc->rows == 0) return s;
    const li_score_desc d = *desc;
    return li_topk_hist(scores, d.max_len > 0 ? scores_ld : 4, len, d.rows, d.max_len, k_top, idx, vals,
                        static_cast<uint32_t*>(workspace), d.tokens_per_request, stream);
}

li_status li_decode_select(const void* q, const float* w, const void* k, const float* k_scale, int64_t cache_batch_rows,
                           const int32_t* len, float* scores, int64_t scores_ld, const li_score_desc* desc, int k_top,
                           int32_t* idx, float* vals, void* workspace, size_t workspace_bytes, li_stream_t stream) {
    li_status s = check_decode_select(q, w, k, k_scale, cache_batch_rows, scores, scores_ld, desc, k_top, true, idx,
                                      workspace, workspace_bytes);
    if (s != LI_OK || desc->rows == 0) return s;
    s = li_decode_select_score(q, w, k, k_scale, cache_batch_rows, len, scores, scores_ld, desc, workspace,
                               workspace_bytes, stream);
    if (s != LI_OK) return s;
    return li_decode_select_finish(scores, desc->max_len > 0 ? scores_ld : 4, len, desc, k_top, idx, vals, workspace,
                                   workspace_bytes, stream);
}

li_status li_host_device_pointer(const void* host_ptr, void** dev_ptr) {
    if (!host_ptr || !dev_ptr) return LI_ERR_INVALID_ARG;
    *dev_ptr = nullptr;
    void* p = nullptr;
    if (cudaHostGetDevicePointer(&p, const_cast<void*>(host_ptr), 0) != cudaSuccess || !p) {
        cudaGetLastError();
        return LI_ERR_INVALID_ARG;  // not page-locked memory mapped for this device
    }
    *dev_ptr = p;
    return LI_OK;
}

li_status li_copy_from_host(void* dst, const void* src_mapped, size_t bytes, li_stream_t stream) {
    if (bytes == 0) return LI_OK;
    if (!dst || !src_mapped || !aligned(dst, 16) || !aligned(src_mapped, 16)) return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    return launch_host_copy(dst, src_mapped, bytes, stream);
}

size_t li_merge_shards_workspace(int shards, int rows, int k) {
    if (shards <= 0 || rows <= 0 || k <= 0) return 0;
    const size_t ld = align_up((size_t)shards * k, 4);
    return align_up((size_t)rows * ld * 4, 256) * 2 + align_up((size_t)rows * shards * 4, 256) +
           (size_t)rows * LI_HIST_BINS * sizeof(uint32_t);
}

li_status li_merge_shards(const float* vals, const int32_t* idx, int shards, int rows, int k, int64_t shard_len,
                          int k_out, int32_t* out_idx, float* out_vals, void* workspace, size_t workspace_bytes,
                          li_stream_t stream) {
    if (shards <= 0 || rows < 0 || k <= 0 || k_out < 1 || k_out > LI_TOPK_MAX_LEN || shard_len <= 0)
        return LI_ERR_INVALID_ARG;
    if ((long long)shards * k > LI_TOPK_MAX_LEN || (long long)shards * shard_len >= (1ll << 31))
        return LI_ERR_INVALID_ARG;
    if (rows == 0) return LI_OK;
    if (!vals || !idx || !out_idx || !workspace || !aligned(workspace, 256) ||
        workspace_bytes < li_merge_shards_workspace(shards, rows, k))
        return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    const size_t ld = align_up((size_t)shards * k, 4);
    float* mvals = static_cast<float*>(workspace);
    int32_t* mpos = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + align_up((size_t)rows * ld * 4, 256));
    int32_t* parts = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(mpos) + align_up((size_t)rows * ld * 4, 256));
    // the rows' first-digit histograms close the workspace (zero before the first call, left zero)
    uint32_t* hist =
        reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(parts) + align_up((size_t)rows * shards * 4, 256));
    li_status s = launch_merge_prep(vals, idx, shards, rows, k, shard_len, mvals, mpos, parts, (long long)ld, hist, e,
                                    stream);
    if (s != LI_OK) return s;
    TopkArgs t{mvals, (long long)ld, nullptr, rows, shards * k, 0, 0, k_out, out_idx, out_vals, mpos, (long long)ld,
               rows, hist, 0, 1, e, parts, shards, k};
    return launch_topk(t, stream);
}

li_status li_absorb_query_layers(const void* q_bf16, const void* w_dec_bf16, void* q_tilde_bf16, int layers,
                                 int batch, int heads, int dim, int latent_dim, li_stream_t stream) {
    if (layers < 0 || layers > 65535 || batch < 0 || heads <= 0 || dim <= 0 || dim > 256 || latent_dim <= 0 ||
        (latent_dim % 64) != 0 || heads > 65535)
        return LI_ERR_INVALID_ARG;
    if (batch == 0 || layers == 0) return LI_OK;
    if (!q_bf16 || !w_dec_bf16 || !q_tilde_bf16 || !aligned(w_dec_bf16, 16) || !aligned(q_tilde_bf16, 2))
        return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    return launch_absorb(q_bf16, w_dec_bf16, q_tilde_bf16, layers, batch, heads, dim, latent_dim, stream);
}

li_status li_absorb_query(const void* q_bf16, const void* w_dec_bf16, void* q_tilde_bf16, int batch, int heads,
                          int dim, int latent_dim, li_stream_t stream) {
    return li_absorb_query_layers(q_bf16, w_dec_bf16, q_tilde_bf16, 1, batch, heads, dim, latent_dim, stream);
}

static li_status latent_score_impl(const void* q_tilde_bf16, const float* w, const void* c_bf16,
                                   int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                                   int batch, int heads, int latent_dim, int max_len, uint32_t* hist,
                                   li_stream_t stream) {
    if (batch < 0 || heads <= 0 || latent_dim <= 0 || max_len < 0 || cache_batch_rows < 0) return LI_ERR_INVALID_ARG;
    if (batch == 0 || max_len == 0) return LI_OK;
    if (!q_tilde_bf16 || !w || !c_bf16 || !scores || scores_ld < max_len) return LI_ERR_INVALID_ARG;
    if ((heads != 64 && heads != 32) || latent_dim != 256) return LI_ERR_UNSUPPORTED;
    if (!aligned(c_bf16, 16) || !aligned(q_tilde_bf16, 16) || (hist && !aligned(hist, 16))) return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    const uint64_t total_rows = cache_batch_rows > 0 ? (uint64_t)(batch - 1) * cache_batch_rows + max_len
                                                     : (uint64_t)max_len;
    if (total_rows >= (1ull << 31)) return LI_ERR_UNSUPPORTED;
    CUtensorMap cmap;
    if (!encode_map_2d(&cmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c_bf16, 256, total_rows, 512, 64, 128))
        return LI_ERR_CUDA;
    StreamArgs a{};
    a.q = q_tilde_bf16;
    a.w = w;
    a.kscale = nullptr;
    a.len = len;
    a.scores = scores;
    a.scores_ld = scores_ld;
    a.batch_rows = cache_batch_rows;
    a.max_len = max_len;
    a.hist = hist;
    a.heads = heads;
    a.err = e;
    const int ntiles = (max_len + 127) / 128;
    return hist ? launch_stream_score_bf16_hist(cmap, a, batch, ntiles, stream)
                : launch_stream_score_bf16(cmap, a, batch, ntiles, stream);
}

li_status li_latent_score(const void* q_tilde_bf16, const float* w, const void* c_bf16, int64_t cache_batch_rows,
                          const int32_t* len, float* scores, int64_t scores_ld, int batch, int heads, int latent_dim,
                          int max_len, li_stream_t stream) {
    return latent_score_impl(q_tilde_bf16, w, c_bf16, cache_batch_rows, len, scores, scores_ld, batch, heads,
                             latent_dim, max_len, nullptr, stream);
}

li_status li_latent_score_hist(const void* q_tilde_bf16, const float* w, const void* c_bf16,
                               int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                               int batch, int heads, int latent_dim, int max_len, uint32_t* hist, li_stream_t stream) {
    if (!hist && batch > 0 && max_len > 0) return LI_ERR_INVALID_ARG;
    return latent_score_impl(q_tilde_bf16, w, c_bf16, cache_batch_rows, len, scores, scores_ld, batch, heads,
                             latent_dim, max_len, hist, stream);
}

li_status li_latent_score_fp8(const void* q_tilde_bf16, const float* w, const void* c_e4m3, const float* c_scale,
                              int64_t cache_batch_rows, const int32_t* len, float* scores, int64_t scores_ld,
                              int batch, int heads, int latent_dim, int max_len, uint32_t* hist, li_stream_t stream) {
    if (batch < 0 || heads <= 0 || latent_dim <= 0 || max_len < 0 || cache_batch_rows < 0) return LI_ERR_INVALID_ARG;
    if (batch == 0 || max_len == 0) return LI_OK;
    if (!q_tilde_bf16 || !w || !c_e4m3 || !c_scale || !scores || scores_ld < max_len) return LI_ERR_INVALID_ARG;
    if (heads != 64 || latent_dim != 192) return LI_ERR_UNSUPPORTED;
    if (!aligned(c_e4m3, 16) || !aligned(q_tilde_bf16, 16) || (hist && !aligned(hist, 16))) return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    const uint64_t total_rows = cache_batch_rows > 0 ? (uint64_t)(batch - 1) * cache_batch_rows + max_len
                                                     : (uint64_t)max_len;
    if (total_rows >= (1ull << 31)) return LI_ERR_UNSUPPORTED;
    CUtensorMap cmap;  // 192-byte rows, boxes of 64 bytes x 128 rows, 64-byte swizzle
    if (!encode_map_2d(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, c_e4m3, 192, total_rows, 192, 64, 128,
                       CU_TENSOR_MAP_SWIZZLE_64B))
        return LI_ERR_CUDA;
    Latent8Args a{};
    a.q = q_tilde_bf16;
    a.w = w;
    a.cscale = c_scale;
    a.len = len;
    a.scores = scores;
    a.scores_ld = scores_ld;
    a.batch_rows = cache_batch_rows;
    a.max_len = max_len;
    a.hist = hist;
    a.err = e;
    return launch_latent8_score(cmap, a, batch, (max_len + 127) / 128, stream);
}

size_t li_hs_refine_workspace(int batch, int n_cand, int followers) {
    if (batch <= 0 || n_cand <= 0 || followers <= 0) return 0;
    return align_up((size_t)followers * batch * align_up((size_t)n_cand, 4) * sizeof(float), 16) +
           hs_hist_bytes(batch, followers);
}

size_t li_workspace_size(int op, int rows, int max_len, int k) {
    (void)k;
    if (rows < 0 || max_len < 0) return 0;
    switch (op) {
    case LI_OP_SCORE: {
        li_score_desc d{};
        d.rows = rows;
        d.heads = 64;
        d.dim = 128;
        d.max_len = max_len;
        d.causal = 1;
        d.q_dtype = LI_DTYPE_BF16;
        d.k_dtype = LI_DTYPE_E4M3;
        return li_index_score_workspace(&d);
    }
    case LI_OP_TOPK: return 0;
    case LI_OP_HS: return li_hs_refine_workspace(rows, max_len, 4);
    case LI_OP_DECODE_SELECT: {
        li_score_desc d{};
        d.rows = rows;
        d.max_len = max_len;
        return li_decode_select_workspace(&d);
    }
    }
    return 0;
}

li_status li_hs_refine(const void* c_bf16, int64_t cache_batch_rows, int64_t cache_rows, const int32_t* cand,
                       int batch, int n_cand, const void* q_tilde_bf16, const float* w, int followers, int heads,
                       int latent_dim, int k, int32_t* out_idx, void* workspace, size_t workspace_bytes,
                       li_stream_t stream) {
    if (batch < 0 || n_cand < 0 || followers <= 0 || heads <= 0 || latent_dim <= 0 || k < 1 ||
        k > LI_TOPK_MAX_LEN || n_cand > LI_TOPK_MAX_LEN || cache_batch_rows < 0 || cache_rows < 0)
        return LI_ERR_INVALID_ARG;
    if (batch == 0) return LI_OK;
    if (!out_idx) return LI_ERR_INVALID_ARG;
    if ((heads != 64 && heads != 32) || latent_dim != 256 || followers > 4) return LI_ERR_UNSUPPORTED;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    if (n_cand == 0) {
        TopkArgs t{nullptr, 4, nullptr, followers * batch, 0, 0, 0, k, out_idx, nullptr, nullptr, 0, 1, nullptr, 0, 1,
                   e};
        return launch_topk(t, stream);
    }
    if (!c_bf16 || !cand || !q_tilde_bf16 || !w || !aligned(c_bf16, 16) || !aligned(q_tilde_bf16, 16))
        return LI_ERR_INVALID_ARG;
    const size_t need = li_hs_refine_workspace(batch, n_cand, followers);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return LI_ERR_INVALID_ARG;
    const int ldw = (int)align_up((size_t)n_cand, 4);
    float* sc = static_cast<float*>(workspace);
    uint32_t* hist = hs_hist_of(workspace, workspace_bytes, batch, followers);
    HsArgs h{c_bf16, cache_batch_rows, cache_rows, cand, batch, n_cand, followers, heads, q_tilde_bf16, w, sc, hist, e};
    if ((uint64_t)followers * batch * heads >= (1ull << 31)) return LI_ERR_UNSUPPORTED;
    CUtensorMap qmap;
    if (!encode_map_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q_tilde_bf16, 256, (uint64_t)followers * batch * heads,
                       512, 64, (uint32_t)heads))
        return LI_ERR_CUDA;
    li_status s = launch_hs_rescore(qmap, h, stream);
    if (s != LI_OK) return s;
    TopkArgs t{sc, ldw, nullptr, followers * batch, n_cand, 0, 0, k, out_idx, nullptr, cand, n_cand, batch,
               hist, 0, 1, e};
    return launch_topk(t, stream);
}

li_status li_hs_refine_fp8(const void* c_e4m3, const float* c_scale, int64_t cache_batch_rows, int64_t cache_rows,
                           const int32_t* cand, int batch, int n_cand, const void* q_tilde_bf16, const float* w,
                           int followers, int heads, int latent_dim, int k, int32_t* out_idx, void* workspace,
                           size_t workspace_bytes, li_stream_t stream) {
    if (batch < 0 || n_cand < 0 || followers <= 0 || heads <= 0 || latent_dim <= 0 || k < 1 ||
        k > LI_TOPK_MAX_LEN || n_cand > LI_TOPK_MAX_LEN || cache_batch_rows < 0 || cache_rows < 0)
        return LI_ERR_INVALID_ARG;
    if (heads != 64 || latent_dim != 192 || followers > 4) return LI_ERR_UNSUPPORTED;
    if (batch == 0) return LI_OK;
    if (!out_idx) return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    if (n_cand == 0) {
        TopkArgs t{nullptr, 4, nullptr, followers * batch, 0, 0, 0, k, out_idx, nullptr, nullptr, 0, 1, nullptr, 0, 1,
                   e};
        return launch_topk(t, stream);
    }
    if (!c_e4m3 || !c_scale || !cand || !q_tilde_bf16 || !w || !aligned(c_e4m3, 16) || !aligned(q_tilde_bf16, 16))
        return LI_ERR_INVALID_ARG;
    const size_t need = li_hs_refine_workspace(batch, n_cand, followers);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return LI_ERR_INVALID_ARG;
    const int ldw = (int)align_up((size_t)n_cand, 4);
    float* sc = static_cast<float*>(workspace);
    uint32_t* hist = hs_hist_of(workspace, workspace_bytes, batch, followers);
    Hs8Args h{c_e4m3, c_scale, cache_batch_rows, cache_rows, cand, batch, n_cand, followers, q_tilde_bf16, w, sc, hist, e};
    li_status s = launch_hs_rescore8(h, stream);
    if (s != LI_OK) return s;
    TopkArgs t{sc, ldw, nullptr, followers * batch, n_cand, 0, 0, k, out_idx, nullptr, cand, n_cand, batch,
               hist, 0, 1, e};
    return launch_topk(t, stream);
}

size_t li_sparse_attention_workspace(int batch, int heads, int k) {
    if (batch <= 0 || heads <= 0 || k <= 0) return 0;
    return sparse_attn_workspace_bytes(batch, heads, k);
}

li_status li_sparse_attention(const void* q_bf16, const void* kv_bf16, int64_t cache_batch_rows, int64_t cache_rows,
                              const int32_t* sel, int batch, int heads, int k, float scale, float* out,
                              void* workspace, size_t workspace_bytes, li_stream_t stream) {
    if (batch < 0 || heads <= 0 || k < 0 || cache_batch_rows < 0 || cache_rows < 0) return LI_ERR_INVALID_ARG;
    if (cache_batch_rows > 0 && cache_rows > cache_batch_rows) return LI_ERR_INVALID_ARG;
    if (!(scale > 0.f) || !(scale < 3.0e38f)) return LI_ERR_INVALID_ARG;
    if (heads % 64 != 0 || heads > 65535 || batch > 65535) return LI_ERR_UNSUPPORTED;
    if (batch == 0) return LI_OK;
    if (!q_bf16 || !kv_bf16 || !out || (k > 0 && !sel)) return LI_ERR_INVALID_ARG;
    if (!aligned(q_bf16, 16) || !aligned(kv_bf16, 16) || !aligned(out, 16)) return LI_ERR_INVALID_ARG;
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    if (k == 0) {  // nothing selected: every output is 0
        if (cudaMemsetAsync(out, 0, (size_t)batch * heads * 512 * sizeof(float), stream) != cudaSuccess)
            return LI_ERR_CUDA;
        return LI_OK;
    }
    const size_t need = sparse_attn_workspace_bytes(batch, heads, k);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return LI_ERR_INVALID_ARG;
    const uint64_t total_rows = cache_batch_rows > 0 ? (uint64_t)(batch - 1) * cache_batch_rows + cache_rows
                                                     : (uint64_t)cache_rows;
    if (total_rows >= (1ull << 31) - 1 || (uint64_t)batch * heads >= (1ull << 31)) return LI_ERR_UNSUPPORTED;
    CUtensorMap qmap;
    if (!encode_map_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q_bf16, 576, (uint64_t)batch * heads, 1152, 64, 64))
        return LI_ERR_CUDA;
    const size_t parts = (size_t)batch * sparse_attn_splits(k) * heads;
    SparseAttnArgs a{};
    a.q = q_bf16;
    a.kv = kv_bf16;
    a.batch_rows = cache_batch_rows;
    a.rows_visible = cache_rows;
    a.sel = sel;
    a.batch = batch;
    a.heads = heads;
    a.k = k;
    a.scale = scale;
    a.opart = static_cast<float*>(workspace);
    a.mpart = a.opart + parts * 512;
    a.lpart = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.mpart) + align_up(parts * 4, 256));
    a.out = out;
    a.err = e;
    return launch_sparse_attn(qmap, a, stream);
}

li_status li_graph_instantiate(void* graph, int use_node_priority, void** exec) {
    if (!graph || !exec) return LI_ERR_INVALID_ARG;
    *exec = nullptr;
    cudaGraphExec_t ge = nullptr;
    const unsigned long long flags = use_node_priority ? cudaGraphInstantiateFlagUseNodePriority : 0ull;
    if (cudaGraphInstantiateWithFlags(&ge, static_cast<cudaGraph_t>(graph), flags) != cudaSuccess) {
        cudaGetLastError();
        return LI_ERR_CUDA;
    }
    *exec = ge;
    return LI_OK;
}

li_status li_graph_launch(void* exec, li_stream_t stream) {
    if (!exec) return LI_ERR_INVALID_ARG;
    if (cudaGraphLaunch(static_cast<cudaGraphExec_t>(exec), stream) != cudaSuccess) {
        cudaGetLastError();
        return LI_ERR_CUDA;
    }
    return LI_OK;
}

li_status li_graph_destroy(void* exec) {
    if (!exec) return LI_OK;
    return cudaGraphExecDestroy(static_cast<cudaGraphExec_t>(exec)) == cudaSuccess ? LI_OK : LI_ERR_CUDA;
}

li_status li_selftest_wait_timeout(uint64_t limit_ns, li_stream_t stream) {
    DevErr e;
    if (ready(&e) != LI_OK) return LI_ERR_CUDA;
    return launch_selftest_wait(limit_ns, stream);
}

}  // extern "C"
