// Merge of per-shard selections for one long context split along L (the
// cache of every request is cut into `shards` slices of `shard_len` positions;
// shard p holds positions p * shard_len .. (p + 1) * shard_len - 1).  Every
// shard selects its k best positions with their scores; the global top-k is
// the top-k of the union of those candidates, since any position among the
// global k best is among its own shard's k best.
//
// Shard p's list is its selected positions in ascending order followed by -1
// pads, and shard p's positions all precede shard p+1's, so the shard lists
// laid side by side are in ascending global position order with every valid
// candidate before every pad (a shard holds fewer than k valid candidates only
// when it is the last one the request reaches).  This kernel lays the lists of
// each request side by side (one CTA per list), turns local positions into
// global ones and counts each list's valid candidates (and their first radix
// digits); the row top-k then takes the row's length from those counts and
// selects over them from that histogram with the global positions as its
// position map, so ties still go to the lower position.
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

constexpr int MP_THREADS = 256;
constexpr int MP_PER = 8;  // candidates per thread per round, loads all in flight

// grid: (shards, rows), one CTA per shard list of a request row; vals / idx are [shards, rows, k].
// parts[r * shards + p] receives list p's count of valid slots before its first pad, with the top
// bit set when a valid slot follows a pad.  With hist, every valid candidate's score is also
// counted by its first radix digit into the row's histogram, one atomic per distinct digit per
// warp, so that the row top-k starts from it.
__global__ void __launch_bounds__(MP_THREADS) merge_prep_kernel(const float* __restrict__ vals,
                                                                const int32_t* __restrict__ idx, int shards, int rows,
                                                                int k, long long shard_len, float* __restrict__ mvals,
                                                                int32_t* __restrict__ mpos, int32_t* __restrict__ parts,
                                                                long long ld, uint32_t* __restrict__ hist, DevErr err) {
    pdl_trigger();
    pdl_wait();  // the lists may come from the previous kernel of the stream
    const int p = blockIdx.x, r = blockIdx.y;
    __shared__ int first_pad;  // lowest slot of the list holding a pad
    __shared__ int last_valid;  // highest slot of the list holding a candidate
    if (threadIdx.x == 0) {
        first_pad = k;
        last_valid = -1;
    }
    __syncthreads();
    uint32_t* gh = hist ? hist + (size_t)r * LI_HIST_BINS : nullptr;
    const size_t src0 = ((size_t)p * rows + r) * k;
    const size_t dst0 = (size_t)r * ld + (size_t)p * k;
    int fp = k, lv = -1;
    // the same number of rounds in every thread: the histogram's warp votes need whole warps
    for (int base = 0; base < k; base += MP_THREADS * MP_PER) {
        int32_t x[MP_PER];
        float v[MP_PER];
#pragma unroll
        for (int u = 0; u < MP_PER; ++u) {
            const int i = base + u * MP_THREADS + (int)threadIdx.x;
            x[u] = -1;
            v[u] = 0.f;
            if (i < k) {
                x[u] = __ldg(idx + src0 + i);
                v[u] = __ldg(vals + src0 + i);
            }
        }
#pragma unroll
        for (int u = 0; u < MP_PER; ++u) {
            const int i = base + u * MP_THREADS + (int)threadIdx.x;
            const bool valid = i < k && x[u] >= 0 && (long long)x[u] < shard_len;
            if (i < k) {
                mvals[dst0 + i] = v[u];
                mpos[dst0 + i] = valid ? (int32_t)(x[u] + (long long)p * shard_len) : -1;
                if (valid) lv = max(lv, i);
                else fp = min(fp, i);
                if (x[u] >= shard_len) record_error(err, ERRBIT_BOUNDS);
            }
            if (gh) warp_hist_add(gh, v[u], valid);
        }
    }
    atomicMin(&first_pad, fp);
    atomicMax(&last_valid, lv);
    __syncthreads();
    if (threadIdx.x == 0)
        parts[(size_t)r * shards + p] = first_pad | (last_valid > first_pad ? (int32_t)0x80000000 : 0);
}

}  // namespace

li_status launch_merge_prep(const float* vals, const int32_t* idx, int shards, int rows, int k, long long shard_len,
                            float* mvals, int32_t* mpos, int32_t* parts, long long ld, uint32_t* hist,
                            const DevErr& err, cudaStream_t st) {
    if (rows <= 0) return LI_OK;
    if (launch_pdl(merge_prep_kernel, dim3(shards, rows), dim3(MP_THREADS), 0, st, 1, vals, idx, shards, rows, k,
                   shard_len, mvals, mpos, parts, ld, hist, err) != cudaSuccess)
        return host_check_launch();
    return host_check_launch();
}

}  // namespace li
