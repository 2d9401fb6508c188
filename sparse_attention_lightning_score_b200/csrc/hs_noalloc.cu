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
//   - Calls with followers * batch * round_up(n_cand, 4) floats beyond that
//     are rejected with LI_ERR_INVALID_ARG before anything is launched.
//   - All calls on a device share the one array and it keeps the previous
//     call's contents.  Every score slot the selection reads is written first
//     by the same call.  The follower top-k's histograms sit at the array's
//     end: zero at load, left zero by every call, and only a speed-up (a
//     histogram that disagrees with the keys sends the top-k to its plain
//     passes).  Calls that overlap on the GPU (different streams, no ordering
//     between them) race on the array and must be serialised by the caller.
//   - The first call on a device looks up the array's device address (set-up);
//     make that first call before any stream capture begins.
#include <cuda_runtime.h>

#include "li.h"

namespace {

// The scratch lives here, in device memory of every GPU that loads the library.
static __device__ __align__(256) float g_hs_noalloc_scratch[LI_HS_NOALLOC_MAX_SCRATCH_FLOATS];

constexpr int kMaxDevices = 64;

// Host code cannot use g_hs_noalloc_scratch's name as a device address (on the
// host it names a stand-in object); the address is fetched per device, with
// that device current, and cached.
float* g_scratch_addr[kMaxDevices] = {};

li_status scratch_for_current_device(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LI_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return LI_ERR_UNSUPPORTED;
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_hs_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return LI_ERR_CUDA;
        }
        g_scratch_addr[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_addr[dev];
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
    return li_hs_refine(c_bf16, cache_batch_rows, cache_rows, cand, batch, n_cand, q_tilde_bf16, w, followers, heads,
                        latent_dim, k, out_idx, scratch, sizeof(g_hs_noalloc_scratch), stream);
}
