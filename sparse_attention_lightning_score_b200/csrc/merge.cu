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
// each request side by side, turns local positions into global ones and counts
// the valid candidates; the row top-k then selects over them with the global
// positions as its position map, so ties still go to the lower position.
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

// grid: one CTA per request row; vals / idx are [shards, rows, k]
__global__ void __launch_bounds__(256) merge_prep_kernel(const float* __restrict__ vals, const int32_t* __restrict__ idx,
                                                         int shards, int rows, int k, long long shard_len,
                                                         float* __restrict__ mvals, int32_t* __restrict__ mpos,
                                                         int32_t* __restrict__ mlen, long long ld, DevErr err) {
    const int r = blockIdx.x;
    const int n = shards * k;
    __shared__ int first_pad;  // lowest slot holding a pad
    __shared__ int last_valid;  // highest slot holding a candidate
    if (threadIdx.x == 0) {
        first_pad = n;
        last_valid = -1;
    }
    __syncthreads();
    int fp = n, lv = -1;
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const int p = j / k, i = j - p * k;
        const size_t src = ((size_t)p * rows + r) * k + i;
        const int32_t x = __ldg(idx + src);
        const bool valid = x >= 0 && (long long)x < shard_len;
        mvals[(size_t)r * ld + j] = __ldg(vals + src);
        mpos[(size_t)r * ld + j] = valid ? (int32_t)(x + (long long)p * shard_len) : -1;
        if (valid) lv = max(lv, j);
        else fp = min(fp, j);
        if (x >= shard_len) record_error(err, ERRBIT_BOUNDS);
    }
    atomicMin(&first_pad, fp);
    atomicMax(&last_valid, lv);
    __syncthreads();
    if (threadIdx.x == 0) {
        // the valid candidates must form a prefix of the row (see above); otherwise report it and
        // keep only the prefix
        if (last_valid >= first_pad) record_error(err, ERRBIT_BOUNDS);
        mlen[r] = first_pad;
    }
}

}  // namespace

li_status launch_merge_prep(const float* vals, const int32_t* idx, int shards, int rows, int k, long long shard_len,
                            float* mvals, int32_t* mpos, int32_t* mlen, long long ld, const DevErr& err,
                            cudaStream_t st) {
    if (rows <= 0) return LI_OK;
    merge_prep_kernel<<<rows, 256, 0, st>>>(vals, idx, shards, rows, k, shard_len, mvals, mpos, mlen, ld, err);
    return host_check_launch();
}

}  // namespace li
