// li_hs_refine_noalloc: hierarchical-selection refinement for callers that
// cannot allocate device memory.
//
// li_hs_refine needs a caller-provided workspace for the followers' candidate
// scores.  Some callers cannot provide one: code embedded in an engine that
// owns and budgets every byte of device memory (and forbids allocation once
// serving has started), or a plugin that is handed only its inputs and
// outputs.  This entry point keeps that scratch in a fixed file-scope device
// array instead, so it allocates nothing.
//
// Limits and sharing:
//   - The array holds LI_HS_NOALLOC_MAX_SCRATCH_FLOATS floats (4 MiB).  Every
//     GPU that loads the library reserves it until the process exits.
//   - A call is accepted when li_hs_refine_workspace(batch, n_cand, followers)
//     -- the candidate scores plus the follower top-k's histograms -- fits in
//     those 4 MiB; a larger one returns LI_ERR_INVALID_ARG before anything is
//     launched.
//   - All calls on a device share the one array and it keeps the previous
//     call's contents.  Every score slot the selection reads is written first
//     by the same call.  The histograms sit at the array's end, where an
//     earlier call with other sizes may have left scores, so every call
//     clears its own histograms on its stream (cudaMemsetAsync, no
//     allocation) before its kernels run.  Calls that overlap on the GPU
//     (different streams, no ordering between them) race on the array and
//     must be serialised by the caller.
//   - The first call on a device looks up the array's device address (set-up);
//     make that first call before any stream capture begins.  The address is
//     cached per device for the life of the process: after cudaDeviceReset
//     the array is a new allocation and this cache no longer names it.
#include <cuda_runtime.h>

#include <atomic>

#include "li.h"

namespace {

// The scratch lives here, in device memory of every GPU that loads the library.
static __device__ __align__(256) float g_hs_noalloc_scratch[LI_HS_NOALLOC_MAX_SCRATCH_FLOATS];

constexpr int kMaxDevices = 64;

// one follower row's first-digit histogram in li_hs_refine's workspace: 2048 bins of uint32
constexpr size_t kHistBytesPerRow = 8192;

// Host code cannot use g_hs_noalloc_scratch's name as a device address (on the
// host it names a stand-in object); the address is fetched per device, with
// that device current, and cached (atomically: several host threads may make
// their first call at once; each then stores the same address).
std::atomic<float*> g_scratch_addr[kMaxDevices];

li_status scratch_for_current_device(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LI_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return LI_ERR_UNSUPPORTED;
    float* a = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!a) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_hs_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return LI_ERR_CUDA;
        }
        a = static_cast<float*>(p);
        g_scratch_addr[dev].store(a, std::memory_order_release);
    }
    *out = a;
    return LI_OK;
}

}  // namespace

extern "C" li_status li_hs_refine_noalloc(const void* c_bf16, int64_t cache_batch_rows, int64_t cache_rows,
                                          const int32_t* cand, int batch, int n_cand, const void* q_tilde_bf16,
                                          const float* w, int followers, int heads, int latent_dim, int k,
                                          int32_t* out_idx, li_stream_t stream) {
    if (batch < 0 || n_cand < 0 || followers <= 0) return LI_ERR_INVALID_ARG;
    const size_t need = li_hs_refine_workspace(batch, n_cand, followers);
    if (need > sizeof(g_hs_noalloc_scratch)) return LI_ERR_INVALID_ARG;
    float* scratch = nullptr;
    const li_status s = scratch_for_current_device(&scratch);
    if (s != LI_OK) return s;
    // this call's histograms are the last followers * batch * 8 KB of the workspace it is given (the
    // layout li_hs_refine documents); an earlier call with other sizes may have left scores there
    const size_t hist_bytes = (size_t)followers * batch * kHistBytesPerRow;
    if (hist_bytes == 0 || n_cand == 0)
        return li_hs_refine(c_bf16, cache_batch_rows, cache_rows, cand, batch, n_cand, q_tilde_bf16, w, followers,
                            heads, latent_dim, k, out_idx, scratch, sizeof(g_hs_noalloc_scratch), stream);
    uint8_t* hist = reinterpret_cast<uint8_t*>(scratch) + (sizeof(g_hs_noalloc_scratch) - hist_bytes);
    if (cudaMemsetAsync(hist, 0, hist_bytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return LI_ERR_CUDA;
    }
    return li_hs_refine(c_bf16, cache_batch_rows, cache_rows, cand, batch, n_cand, q_tilde_bf16, w, followers, heads,
                        latent_dim, k, out_idx, scratch, sizeof(g_hs_noalloc_scratch), stream);
}
