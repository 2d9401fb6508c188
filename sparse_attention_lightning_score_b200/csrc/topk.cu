// Per-row top-k select over fp32 scores (IndexCache explainer, Symbol Map: the
// indexer's scores are followed by top-k, k = 2,048 token positions).
//
// Order: larger score first; equal scores go to the lower position; NaN ranks
// below every number; -0.0 equals +0.0.  The selected positions are written in
// ascending order (then -1 pads when a row holds fewer than k scores).
//
// Method: MSB-first radix select (8-bit digits) on an order-preserving
// uint32 image of the fp32 bits, as in Alabi et al., "Fast k-Selection
// Algorithms for Graphics Processing Units" (2012).  A row is split over a
// thread-block cluster of CS CTAs; each CTA keeps its slice of the row in
// shared memory, so HBM is read once.  Per digit, each CTA builds a 256-bin
// histogram of the still-undecided keys with warp-aggregated shared-memory
// atomics (__match_any_sync groups lanes holding the same digit, one atomic
// per group), the histograms are summed across the cluster through
// distributed shared memory, and every CTA takes the same decision.  The
// final compaction is an ordered scan (CTA prefix over the cluster, block
// prefix inside the CTA), so the output does not depend on atomic order.
#include <cooperative_groups.h>

#include "li_common.cuh"
#include "li_kernels.cuh"

namespace cg = cooperative_groups;

namespace li {

namespace {

constexpr int TK_THREADS = 512;
constexpr int TK_WARPS = TK_THREADS / 32;
constexpr int TK_IPT = 4;                     // keys per thread per compaction tile
constexpr int TK_TILE = TK_THREADS * TK_IPT;  // 2048
constexpr int TK_MAX_SMEM = 160 * 1024;       // key slice budget per CTA

__device__ __forceinline__ uint32_t order_key(float f) {
    if (f != f) return 0u;  // NaN: the only key mapped to 0, below -inf (0x007FFFFF)
    uint32_t u = __float_as_uint(f);
    if (f == 0.f) u = 0u;   // fold -0.0 onto +0.0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive prefix sum over the 512 threads of the block; *total receives the
// block sum.  Contains __syncthreads; call from all threads.
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t* wsum, uint32_t* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t x = lane < TK_WARPS ? wsum[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += t;
        }
        if (lane < TK_WARPS) wsum[lane] = x;
    }
    __syncthreads();
    const uint32_t add = warp > 0 ? wsum[warp - 1] : 0u;
    *total = wsum[TK_WARPS - 1];
    __syncthreads();
    return v + add;
}

template <bool CLUSTER>
__device__ __forceinline__ void cl_sync() {
    if constexpr (CLUSTER) cg::this_cluster().sync();
    else __syncthreads();
}

template <bool CLUSTER>
__device__ __forceinline__ const uint32_t* cl_peer(uint32_t* p, int rank) {
    if constexpr (CLUSTER) return cg::this_cluster().map_shared_rank(p, rank);
    else return p;
}

template <bool CLUSTER>
__global__ void __launch_bounds__(TK_THREADS) topk_kernel(const TopkArgs a, int row0, int chunk) {
    extern __shared__ uint4 tk_dyn[];
    uint32_t* keys = reinterpret_cast<uint32_t*>(tk_dyn);
    __shared__ uint32_t hist[2][256];
    __shared__ uint32_t tot[256];
    __shared__ uint32_t wsum[TK_WARPS];
    __shared__ uint32_t bc[4];
    __shared__ uint32_t xch[2];

    const int r = row0 + blockIdx.y;
    const int CS = gridDim.x;
    const int c = blockIdx.x;  // == cluster rank: the cluster spans gridDim.x
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    long long nl = a.causal ? (long long)r + 1 + a.causal_offset : (a.len ? (long long)__ldg(a.len + r) : a.max_len);
    if (!a.causal && a.len && (nl < 0 || nl > a.max_len) && c == 0 && threadIdx.x == 0) record_error(a.err, ERRBIT_BOUNDS);
    nl = nl < 0 ? 0 : (nl > a.max_len ? a.max_len : nl);
    const int n = (int)nl;
    const int k = a.k;
    const int base = c * chunk;
    const int cnt = max(0, min(n - base, chunk));
    int32_t* oidx = a.idx + (size_t)r * k;
    float* oval = a.vals ? a.vals + (size_t)r * k : nullptr;
    const float* srow = a.scores + (size_t)r * a.ld;
    const int32_t* mrow = a.map ? a.map + (size_t)(r % a.map_rows) * a.map_ld : nullptr;

    if (n <= k) {  // every score is selected; the branch is uniform over the cluster
        for (int i = threadIdx.x; i < cnt; i += TK_THREADS) {
            const int p = base + i;
            oidx[p] = mrow ? __ldg(mrow + p) : p;
            if (oval) oval[p] = __ldg(srow + p);
        }
        for (int p = n + c * TK_THREADS + threadIdx.x; p < k; p += CS * TK_THREADS) {
            oidx[p] = -1;
            if (oval) oval[p] = -INFINITY;
        }
        return;
    }

    // ---- load this CTA's slice (row start and slice start are 16-byte aligned)
    const float4* s4 = reinterpret_cast<const float4*>(srow + base);
    const int nvec = (cnt + 3) >> 2;
    for (int i = threadIdx.x; i < nvec; i += TK_THREADS) {
        const float4 v = __ldg(s4 + i);
        tk_dyn[i] = make_uint4(order_key(v.x), order_key(v.y), order_key(v.z), order_key(v.w));
    }
    for (int i = threadIdx.x; i < 512; i += TK_THREADS) (&hist[0][0])[i] = 0u;
    __syncthreads();

    // ---- radix select, most significant digit first
    uint32_t prefix = 0u, mask = 0u;
    int krem = k;
    bool ties = true;
    const int cnt32 = (cnt + 31) & ~31;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        uint32_t* h = hist[pass & 1];
        for (int i0 = warp * 32; i0 < cnt32; i0 += TK_THREADS) {
            const int i = i0 + lane;
            bool act = false;
            uint32_t dig = 0u;
            if (i < cnt) {
                const uint32_t kk = keys[i];
                act = (kk & mask) == prefix;
                dig = (kk >> shift) & 255u;
            }
            const uint32_t am = __ballot_sync(0xffffffffu, act);
            if (act) {
                const uint32_t peers = __match_any_sync(am, dig);
                if (lane == __ffs(peers) - 1) atomicAdd(&h[dig], (uint32_t)__popc(peers));
            }
        }
        cl_sync<CLUSTER>();
        if (threadIdx.x < 256) {
            uint32_t t = 0u;
            for (int q = 0; q < CS; ++q) t += cl_peer<CLUSTER>(h, q)[threadIdx.x];
            tot[threadIdx.x] = t;
            hist[(pass + 1) & 1][threadIdx.x] = 0u;  // read by peers one pass ago: free again
        }
        __syncthreads();
        const uint32_t v = threadIdx.x < 256 ? tot[255 - threadIdx.x] : 0u;
        uint32_t total;
        const uint32_t incl = block_incl_scan(v, wsum, &total);
        if (threadIdx.x < 256 && v > 0u && incl >= (uint32_t)krem && incl - v < (uint32_t)krem) {
            bc[0] = 255u - threadIdx.x;  // the digit holding the k-th largest key
            bc[1] = incl - v;            // keys above that digit
            bc[2] = v;                   // keys in that digit
        }
        __syncthreads();
        const uint32_t digit = bc[0], above = bc[1], inbin = bc[2];
        prefix |= digit << shift;
        mask |= 255u << shift;
        krem -= (int)above;
        __syncthreads();
        if ((int)inbin == krem) {  // the whole bin is taken: no tie to break
            ties = false;
            break;
        }
    }
    const uint32_t T = prefix;

    // ---- counts of this slice, exchanged over the cluster
    uint32_t my = 0u;
    for (int i = threadIdx.x; i < cnt; i += TK_THREADS) {
        const uint32_t kk = keys[i];
        if (ties ? kk > T : kk >= T) my += 1u << 16;
        else if (ties && kk == T) my += 1u;
    }
    // per-thread counts fit 16 bits (cnt <= 32768 per slice, 64 per thread here)
    uint32_t ctot;
    (void)block_incl_scan(my, wsum, &ctot);
    if (threadIdx.x == 0) {
        xch[0] = ctot >> 16;
        xch[1] = ctot & 0xffffu;
    }
    cl_sync<CLUSTER>();
    uint32_t gt_before = 0u, eq_before = 0u;
    for (int q = 0; q < c; ++q) {
        const uint32_t* px = cl_peer<CLUSTER>(xch, q);
        gt_before += px[0];
        eq_before += px[1];
    }
    const int quota = ties ? max(0, krem - (int)eq_before) : 0;
    const int out_base = (int)gt_before + (ties ? min((int)eq_before, krem) : 0);

    // ---- ordered compaction of this slice
    int carry_gt = 0, carry_eq = 0;
    for (int tb = 0; tb < cnt; tb += TK_TILE) {
        const int i0 = tb + threadIdx.x * TK_IPT;
        uint4 kv = make_uint4(0u, 0u, 0u, 0u);
        if (i0 < cnt) kv = tk_dyn[i0 >> 2];
        const uint32_t kk[4] = {kv.x, kv.y, kv.z, kv.w};
        uint32_t gm = 0u, em = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool valid = i0 + e < cnt;
            if (valid && (ties ? kk[e] > T : kk[e] >= T)) gm |= 1u << e;
            else if (valid && ties && kk[e] == T) em |= 1u << e;
        }
        const uint32_t packed = ((uint32_t)__popc(gm) << 16) | (uint32_t)__popc(em);
        uint32_t ttot;
        const uint32_t excl = block_incl_scan(packed, wsum, &ttot) - packed;
        int gb = carry_gt + (int)(excl >> 16);
        int eb = carry_eq + (int)(excl & 0xffffu);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int pos = -1;
            if (gm & (1u << e)) {
                pos = out_base + gb + min(eb, quota);
                ++gb;
            } else if (em & (1u << e)) {
                if (eb < quota) pos = out_base + gb + eb;
                ++eb;
            }
            if (pos >= k) {  // cannot happen when the counts agree; never write past the row
                record_error(a.err, ERRBIT_BOUNDS);
                pos = -1;
            }
            if (pos >= 0) {
                const int p = base + i0 + e;
                oidx[pos] = mrow ? __ldg(mrow + p) : p;
                if (oval) oval[pos] = __ldg(srow + p);
            }
        }
        carry_gt += (int)(ttot >> 16);
        carry_eq += (int)(ttot & 0xffffu);
    }
    cl_sync<CLUSTER>();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace

li_status launch_topk(const TopkArgs& a, cudaStream_t st) {
    if (a.rows <= 0) return LI_OK;
    const int sms = host_num_sms();
    const int maxl = max(a.max_len, 1);
    int cs = 1;
    if (a.rows < sms) cs = min(8, (2 * sms + a.rows - 1) / a.rows);
    auto chunk_of = [&](int csz) { return (((maxl + csz - 1) / csz) + 3) & ~3; };
    while (cs < 8 && chunk_of(cs) * 4 > TK_MAX_SMEM) ++cs;
    // keep small rows on few CTAs: a slice below one compaction tile wastes the cluster
    while (cs > 1 && chunk_of(cs) < TK_TILE / 2 && chunk_of(cs / 2) * 4 <= TK_MAX_SMEM) cs /= 2;
    const int chunk = chunk_of(cs);
    if (chunk * 4 > TK_MAX_SMEM || chunk > 32768) return LI_ERR_UNSUPPORTED;
    const size_t smem = (size_t)chunk * 4;

    static bool attr_done[64][2] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev][cs > 1]) {
        if (cs > 1) cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, TK_MAX_SMEM);
        else cudaFuncSetAttribute(topk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, TK_MAX_SMEM);
        attr_done[dev][cs > 1] = true;
    }
    for (int row0 = 0; row0 < a.rows; row0 += 65535) {
        const int nr = min(65535, a.rows - row0);
        if (cs == 1) {
            topk_kernel<false><<<dim3(1, nr), TK_THREADS, smem, st>>>(a, row0, chunk);
        } else {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(cs, nr);
            cfg.blockDim = dim3(TK_THREADS);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = st;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = cs;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaLaunchKernelEx(&cfg, topk_kernel<true>, a, row0, chunk) != cudaSuccess) return host_check_launch();
        }
        const li_status s = host_check_launch();
        if (s != LI_OK) return s;
    }
    return LI_OK;
}

}  // namespace li
