// Per-row top-k select over fp32 scores (IndexCache explainer, Symbol Map: the
// indexer's scores are followed by top-k, k = 2,048 token positions).
//
// Order: larger score first; equal scores go to the lower position; NaN ranks
// below every number; -0.0 equals +0.0.  The selected positions are written in
// ascending order (then -1 pads when a row holds fewer than k scores).
//
// Method: MSB-first radix select on an order-preserving uint32 image of the
// fp32 bits, as in Alabi et al., "Fast k-Selection Algorithms for Graphics
// Processing Units" (2012).  A pass stops the select early when the bin that
// holds the k-th key is taken whole (no tie to break), which for real scores
// happens after 22-24 bits.
//
// Each CTA keeps its slice of the row in shared memory, so the scores are read
// from HBM (or L2) once.  Many rows (causal prefill): one CTA per row, 11-bit
// digits (three passes at most), every pass a shared-memory histogram plus
// block barriers.  Few rows (decode): each row is split over a thread-block
// cluster so that about 4K keys land on each CTA and every sweep runs on many
// SMs; the CTAs' histograms are summed through distributed shared memory after
// one cluster barrier per pass, with 8-bit digits so that a merge moves 256
// bins (measured: merging 2048-bin histograms cost more than the extra pass).
//
// Histograms: warp w adds into private copy w % NCOPY with plain shared-memory
// atomics, which spreads the few hot bins a pass of real scores concentrates
// on (aggregating lanes by digit with __match_any_sync was measured 6x slower
// on B200); a warp ballot skips warps with no undecided key.  Each owner
// thread folds the copies of its bins, merges them over the cluster and feeds
// a block-wide scan (warp shuffles) that finds the digit of the k-th key.
//
// Compaction: the slice's counts above / at the threshold are exchanged over
// the cluster once, then the slice is written in order, 4 or 8 consecutive
// keys per thread per sweep, positions from a block-wide scan.  No output
// depends on the order of any atomic operation.
//
// With a histogram from the decode scorer (HIST): its LI_HIST_BITS-bit digit
// is the first pass, found by one block-wide scan in every CTA with no cluster
// merge.  The keys in the k-th key's bin (the candidates, about 3-5% of a row
// of real scores) are appended to a list per CTA; one cluster exchange gives
// every CTA the whole row's list, and the remaining 21 bits are selected from
// it locally (two passes, no cluster barrier).  The exchange also checks the
// histogram against the keys (the counts above and in the bin must agree);
// if they do not, or the bin holds more candidates than a CTA can keep, the
// plain passes run instead, so the result never depends on the histogram.
// The histogram is left all zero for the next step.
#include <algorithm>
#include <cooperative_groups.h>

#include "block_scan.cuh"
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace cg = cooperative_groups;

namespace li {

namespace {

constexpr int TK_SMEM_ROW = 40960;  // longest slice held by one CTA (160 KB of keys)
constexpr int TK_MAX_CS = 16;       // largest cluster (above 8: non-portable, checked at launch)
constexpr int TK_SLICE = 4096;      // target slice of a row per cluster CTA

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

// Kernel shape: NT threads, DBITS-bit digits (11 for a row held by one CTA:
// three passes, no merge; 8 for a row split over a cluster: up to four
// passes, but each cluster merge moves 256 bins instead of 2048).
template <int NT, bool CLUSTER>
struct TopkShape {
    static constexpr int WARPS = NT / 32;
    static constexpr int DBITS = CLUSTER ? 8 : 11;
    static constexpr int BINS = 1 << DBITS;
    static constexpr int PASSES = (32 + DBITS - 1) / DBITS;
    static constexpr int OWNERS = BINS < NT ? BINS : NT;  // threads that own bins
    static constexpr int BPT = BINS / OWNERS;              // bins per owner
    static constexpr int NCOPY = CLUSTER ? 8 : (NT >= 1024 ? 4 : 2);  // private histogram copies
    // dynamic shared memory: keys, NCOPY histogram copies, then (cluster) the
    // double-buffered merged histogram the peers read
    static size_t smem(int chunk) {
        return (size_t)((chunk + 3) & ~3) * 4 + (size_t)NCOPY * BINS * 4 + (CLUSTER ? 2 * BINS * 4 : 0);
    }
    // with a histogram: this CTA's candidate list and (cluster) the row's gathered list
    static size_t smem_hist(int chunk, int cap) { return smem(chunk) + (size_t)cap * 4 * (CLUSTER ? 2 : 1); }
    static_assert(NCOPY * BINS >= LI_HIST_BINS, "the histogram copies hold the scorer's histogram");
    __device__ static int shift(int p) { return 32 - DBITS * (p + 1) > 0 ? 32 - DBITS * (p + 1) : 0; }
    __device__ static uint32_t digits(int p) {
        const int lo = shift(p), hi = 32 - DBITS * p;  // bits [lo, hi)
        return (hi - lo >= 32) ? 0xffffffffu : ((1u << (hi - lo)) - 1u);
    }
};

// KPT consecutive keys of the slice from shared memory (keys at or past cnt read as 0); i0 % 4 == 0.
template <int KPT>
__device__ __forceinline__ void load_keys(const uint4* t, int i0, int cnt, uint32_t (&kk)[KPT]) {
#pragma unroll
    for (int q = 0; q < KPT / 4; ++q) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (i0 + 4 * q < cnt) v = t[(i0 >> 2) + q];
        kk[4 * q] = v.x;
        kk[4 * q + 1] = v.y;
        kk[4 * q + 2] = v.z;
        kk[4 * q + 3] = v.w;
    }
}

// Thread t < OWNERS owns the BPT contiguous bins BINS-BPT(t+1) .. BINS-BPT*t-1
// (descending positions BPT*t .. BPT*t+BPT-1).
template <int NT, bool CLUSTER, bool HIST>
__global__ void __launch_bounds__(NT) topk_kernel(const TopkArgs a, int row0, int chunk) {
    using S = TopkShape<NT, CLUSTER>;
    constexpr int BPT = S::BPT, NW = S::WARPS, NCOPY = S::NCOPY, BINS = S::BINS;
    // keys per thread in the candidate and compaction sweeps: 4 for the 1024-thread cluster CTAs
    // (slices of at most 4096 keys, so every thread has keys and one block-wide scan covers the
    // slice), 8 otherwise
    constexpr int KPT = (CLUSTER && NT == 1024) ? 4 : 8;
    static_assert(BPT == 1 || BPT == 2 || BPT == 4 || BPT == 8, "bins per owner");
    extern __shared__ uint4 tk_dyn[];
    uint32_t* keys = reinterpret_cast<uint32_t*>(tk_dyn);
    uint32_t* hcopy = keys + ((chunk + 3) & ~3);     // [NCOPY][BINS]
    uint32_t* pub = hcopy + NCOPY * BINS;            // [2][BINS], cluster only
    uint32_t* cand = pub + (CLUSTER ? 2 * BINS : 0); // HIST: this CTA's candidate keys [cand_cap]
    uint32_t* gath = CLUSTER ? cand + a.cand_cap : cand;  // HIST: the row's candidate keys [cand_cap]
    __shared__ uint32_t wsum[2][32];
    __shared__ uint32_t bc[4];
    __shared__ uint32_t xch[2];
    __shared__ uint32_t xcand[2];                    // HIST: candidates and keys above the bin, this CTA
    __shared__ uint32_t coff[TK_MAX_CS + 1];         // HIST: candidate list offsets by cluster rank

    pdl_trigger();
    pdl_wait();  // the scores come from the previous kernel of the stream
    // causal rows grow with the row index: the longest are dealt first, so that the short ones fill
    // the SMs at the end of the launch
    const int r = row0 + (a.causal ? (int)(gridDim.y - 1 - blockIdx.y) : (int)blockIdx.y);
    const int CS = gridDim.x;
    const int c = blockIdx.x;  // == cluster rank: the cluster spans gridDim.x
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    const int tokens = a.tokens > 1 ? a.tokens : 1;  // multi-token decode: rows per len entry
    long long nl = a.causal ? (long long)r + 1 + a.causal_offset
                            : (a.len ? (long long)__ldg(a.len + r / tokens) : a.max_len);
    if (!a.causal && a.len && (nl < 0 || nl > a.max_len) && c == 0 && threadIdx.x == 0) record_error(a.err, ERRBIT_BOUNDS);
    nl = nl < 0 ? 0 : (nl > a.max_len ? a.max_len : nl);
    if (!a.causal) nl = nl - (tokens - 1 - r % tokens) < 0 ? 0 : nl - (tokens - 1 - r % tokens);
    if (a.len_parts) {
        // shard merge: the valid prefix of the lists side by side
        const int32_t* pr = a.len_parts + (size_t)r * a.nparts;
        const long long full = (long long)a.nparts * a.part_k;
        long long fpad = full;
        bool gap = false;
        for (int p = 0; p < a.nparts; ++p) {
            const uint32_t v = (uint32_t)__ldg(pr + p);
            const int cnt = (int)(v & 0x7fffffffu);
            gap |= (v >> 31) != 0u;
            if (fpad == full) {
                if (cnt < a.part_k) fpad = (long long)p * a.part_k + cnt;
            } else if (cnt > 0) {
                gap = true;
            }
        }
        if (gap && c == 0 && threadIdx.x == 0) record_error(a.err, ERRBIT_BOUNDS);
        nl = fpad < nl ? fpad : nl;
    }
    const int n = (int)nl;
    const int k = a.k;
    const int base = c * chunk;
    const int cnt = max(0, min(n - base, chunk));
    int32_t* oidx = a.idx + (size_t)r * k;
    float* oval = a.vals ? a.vals + (size_t)r * k : nullptr;
    const float* srow = a.scores + (size_t)r * a.ld;
    const int32_t* mrow = a.map ? a.map + (size_t)(r % a.map_rows) * a.map_ld : nullptr;
    uint32_t* hrow = HIST ? a.hist + (size_t)r * LI_HIST_BINS : nullptr;

    if (n <= k) {  // every score is selected; the branch is uniform over the cluster
        if constexpr (HIST) {
            if (c == 0)
                for (int i = threadIdx.x; i < LI_HIST_BINS; i += NT) hrow[i] = 0u;
        }
        for (int i = threadIdx.x; i < cnt; i += NT) {
            const int p = base + i;
            oidx[p] = mrow ? __ldg(mrow + p) : p;
            if (oval) oval[p] = __ldg(srow + p);
        }
        for (int p = n + c * NT + threadIdx.x; p < k; p += CS * NT) {
            oidx[p] = -1;
            if (oval) oval[p] = -INFINITY;
        }
        return;
    }

    // ---- load this CTA's slice (row start and slice start are 16-byte aligned), LU loads in
    // flight per thread; the histogram's loads go out first
    if constexpr (HIST) {
        const uint4* h4 = reinterpret_cast<const uint4*>(hrow);
        for (int i = threadIdx.x; i < LI_HIST_BINS / 4; i += NT) reinterpret_cast<uint4*>(hcopy)[i] = __ldcg(h4 + i);
    } else {
        for (int i = threadIdx.x; i < NCOPY * BINS; i += NT) hcopy[i] = 0u;
    }
    {
        constexpr int LU = 4;
        const float4* s4 = reinterpret_cast<const float4*>(srow + base);
        const int nvec = (cnt + 3) >> 2;
        for (int i0 = threadIdx.x; i0 < nvec; i0 += NT * LU) {
            float4 v[LU];
#pragma unroll
            for (int u = 0; u < LU; ++u) {
                const int i = i0 + u * NT;
                v[u] = i < nvec ? __ldg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < LU; ++u) {
                const int i = i0 + u * NT;
                if (i < nvec)
                    tk_dyn[i] = make_uint4(order_key(v[u].x), order_key(v[u].y), order_key(v[u].z), order_key(v[u].w));
            }
        }
    }
    __syncthreads();

    uint32_t prefix = 0u, mask = 0u;
    int krem = k;
    bool ties = true;
    bool selected = false;
    uint32_t gt_before = 0u, eq_before = 0u;  // selected keys in lower-ranked CTAs: above T, at T
    bool have_offsets = false;
    if constexpr (HIST) {
        // ---- first digit from the scorer's histogram (the same in every CTA of the cluster)
        find_digit<NT, LI_HIST_BINS>(hcopy, krem, wsum[0], bc);
        const uint32_t b1 = bc[0], above_h = bc[1], inbin_h = bc[2], total_h = bc[3];
        if (total_h != (uint32_t)n && c == 0 && threadIdx.x == 0) record_error(a.err, ERRBIT_BOUNDS);
        if (total_h == (uint32_t)n && inbin_h <= (uint32_t)a.cand_cap) {
            // ---- this slice's candidates (keys in bin b1, in position order) and its count of keys
            // above the bin: KPT consecutive keys per thread, offsets from one block-wide scan
            uint32_t ncand = 0u, nabove = 0u;
            for (int tb = 0, flip = 0; tb < cnt; tb += NT * KPT, flip ^= 1) {
                const int i0 = tb + threadIdx.x * KPT;
                uint32_t kk[KPT];
                load_keys<KPT>(tk_dyn, i0, cnt, kk);
                uint32_t cm = 0u, na = 0u;
#pragma unroll
                for (int e = 0; e < KPT; ++e) {
                    const uint32_t d = kk[e] >> LI_HIST_SHIFT;
                    const bool valid = i0 + e < cnt;
                    cm |= (valid && d == b1) ? 1u << e : 0u;
                    na += (valid && d > b1) ? 1u : 0u;
                }
                const uint32_t packed = (na << 16) | (uint32_t)__popc(cm);
                uint32_t tot;
                const uint32_t excl = block_scan1<NW>(packed, wsum[flip], &tot) - packed;
                uint32_t slot = ncand + (excl & 0xffffu);
#pragma unroll
                for (int e = 0; e < KPT; ++e)
                    if (cm & (1u << e)) {
                        if (slot < (uint32_t)a.cand_cap) cand[slot] = kk[e];
                        ++slot;
                    }
                ncand += tot & 0xffffu;
                nabove += tot >> 16;
            }
            if (threadIdx.x == 0) {
                xcand[0] = ncand;
                xcand[1] = nabove;
            }
            uint32_t ntot, above_sum, above_before = 0u, cand_before = 0u;
            if constexpr (CLUSTER) {
                cl_sync<true>();
                // gather every CTA's candidates, in rank order, into gath
                if (warp == 0) {
                    uint32_t cq = 0u, aq = 0u;
                    if (lane < CS) {
                        const uint32_t* px = cl_peer<true>(xcand, lane);
                        cq = px[0];
                        aq = px[1];
                    }
                    const bool over = __ballot_sync(0xffffffffu, cq > (uint32_t)a.cand_cap) != 0u;
                    cq = min(cq, (uint32_t)a.cand_cap);
                    const uint32_t incl = warp_incl_scan(cq, lane);
                    const uint32_t sum = __shfl_sync(0xffffffffu, incl, 31);
                    uint32_t as = aq;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) as += __shfl_xor_sync(0xffffffffu, as, o);
                    uint32_t ab = lane < c ? aq : 0u;  // keys above the bin in lower-ranked CTAs
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) ab += __shfl_xor_sync(0xffffffffu, ab, o);
                    if (lane < CS) coff[lane + 1] = incl;
                    if (lane == 0) {
                        coff[0] = 0u;
                        bc[0] = over ? (uint32_t)a.cand_cap + 1u : sum;  // bc is free again: broadcast through it
                        bc[1] = as;
                        bc[2] = ab;
                    }
                }
                __syncthreads();
                ntot = bc[0];
                above_sum = bc[1];
                above_before = bc[2];
                cand_before = coff[c];
                if (ntot <= (uint32_t)a.cand_cap) {
#pragma unroll 4
                    for (int j = threadIdx.x; j < (int)ntot; j += NT) {
                        int q = 0;
#pragma unroll
                        for (int t = 1; t < TK_MAX_CS; ++t) q += (t < CS && (uint32_t)j >= coff[t]) ? 1 : 0;
                        gath[j] = cl_peer<true>(cand, q)[j - (int)coff[q]];
                    }
                }
                __syncthreads();
                // this CTA reads no peer's shared memory from here on; peers may leave after the final wait
                asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
            } else {
                __syncthreads();
                ntot = xcand[0];
                above_sum = xcand[1];
            }
            __syncthreads();
            if (ntot == inbin_h && above_sum == above_h) {
                // ---- the remaining 21 bits, from the candidates alone: 11 then 10 bits
                krem -= (int)above_h;
                prefix = b1 << LI_HIST_SHIFT;
                mask = ~0u << LI_HIST_SHIFT;
                ties = (int)inbin_h != krem;
                for (int lp = 0; ties && lp < 2; ++lp) {
                    const int sh = lp == 0 ? 10 : 0;
                    const uint32_t dm = lp == 0 ? 0x7ffu : 0x3ffu;
                    for (int i = threadIdx.x; i < LI_HIST_BINS; i += NT) hcopy[i] = 0u;
                    __syncthreads();
                    for (int i = threadIdx.x; i < (int)ntot; i += NT) {
                        const uint32_t kk = gath[i];
                        if ((kk & mask) == prefix) atomicAdd(&hcopy[(kk >> sh) & dm], 1u);
                    }
                    __syncthreads();
                    find_digit<NT, LI_HIST_BINS>(hcopy, krem, wsum[lp & 1], bc);
                    krem -= (int)bc[1];
                    prefix |= bc[0] << sh;
                    mask |= dm << sh;
                    if ((int)bc[2] == krem) ties = false;
                }
                selected = true;
                // output offset: keys above the bin in lower ranks, plus their candidates above / at T
                uint32_t my = 0u;
                for (int j = threadIdx.x; j < (int)cand_before; j += NT) {
                    const uint32_t kk = gath[j];
                    if (ties ? kk > prefix : kk >= prefix) my += 1u << 16;
                    else if (ties && kk == prefix) my += 1u;
                }
                uint32_t tot;
                (void)block_scan1<NW>(my, wsum[0], &tot);
                gt_before = above_before + (tot >> 16);
                eq_before = tot & 0xffffu;
                have_offsets = true;
            } else {
                if (c == 0 && threadIdx.x == 0) record_error(a.err, ERRBIT_BOUNDS);  // the histogram does not
                                                                                       // describe these keys
                // close the phase opened by the arrive above before the plain passes' own cluster barriers
                if constexpr (CLUSTER) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
            }
        }
        if (!selected) {
            for (int i = threadIdx.x; i < NCOPY * BINS; i += NT) hcopy[i] = 0u;
            __syncthreads();
        }
    }

    // ---- radix select, most significant digit first
    const bool owner = threadIdx.x < S::OWNERS;
    const int b0 = BINS - BPT * (threadIdx.x + 1);  // an owner's bins b0 .. b0+BPT-1
    uint32_t* hmine = hcopy + (warp % NCOPY) * BINS;
    for (int pass = 0; !selected && pass < S::PASSES; ++pass) {
        const int shift = S::shift(pass);
        const uint32_t dm = S::digits(pass);
        for (int i = threadIdx.x; i < ((cnt + 31) & ~31); i += NT) {
            const uint32_t kk = i < cnt ? keys[i] : 0u;
            const bool act = i < cnt && (kk & mask) == prefix;
            if (__ballot_sync(0xffffffffu, act) == 0u) continue;  // nothing undecided in this warp
            if (act) atomicAdd(&hmine[(kk >> shift) & dm], 1u);
        }
        __syncthreads();
        // fold the private copies of an owner's bins (and clear them for the next pass);
        // tot[i]: bin b0+BPT-1-i (descending position BPT*t + i) summed over the cluster
        uint32_t tot[BPT];
#pragma unroll
        for (int i = 0; i < BPT; ++i) tot[i] = 0u;
        if (owner) {
            uint32_t mine[BPT];
#pragma unroll
            for (int v = 0; v < BPT; ++v) mine[v] = 0u;
#pragma unroll
            for (int cp = 0; cp < NCOPY; ++cp) {
#pragma unroll
                for (int v = 0; v < BPT; ++v) {
                    mine[v] += hcopy[cp * BINS + b0 + v];
                    hcopy[cp * BINS + b0 + v] = 0u;
                }
            }
            if constexpr (!CLUSTER) {
#pragma unroll
                for (int i = 0; i < BPT; ++i) tot[i] = mine[BPT - 1 - i];
            } else {
                uint32_t* pb = pub + (pass & 1) * BINS;  // read by the peers one pass ago: free again
#pragma unroll
                for (int v = 0; v < BPT; ++v) pb[b0 + v] = mine[v];
            }
        }
        if constexpr (CLUSTER) {
            cl_sync<true>();
            if (owner) {
                const uint32_t* pb = pub + (pass & 1) * BINS;
                uint32_t pv[TK_MAX_CS][BPT];
#pragma unroll
                for (int q = 0; q < TK_MAX_CS; ++q)
                    if (q < CS) {
                        const uint32_t* src = cl_peer<true>(const_cast<uint32_t*>(pb), q) + b0;
#pragma unroll
                        for (int v = 0; v < BPT; ++v) pv[q][v] = src[v];
                    }
#pragma unroll
                for (int q = 0; q < TK_MAX_CS; ++q)
                    if (q < CS) {
#pragma unroll
                        for (int i = 0; i < BPT; ++i) tot[i] += pv[q][BPT - 1 - i];
                    }
            }
        }
        uint32_t s = 0u;
#pragma unroll
        for (int i = 0; i < BPT; ++i) s += tot[i];
        uint32_t total;
        const uint32_t incl = block_scan1<NW>(s, wsum[pass & 1], &total);
        const uint32_t excl = incl - s;
        if (owner && excl < (uint32_t)krem && incl >= (uint32_t)krem) {
            uint32_t run = excl;
#pragma unroll
            for (int i = 0; i < BPT; ++i) {
                if (run < (uint32_t)krem && run + tot[i] >= (uint32_t)krem) {
                    bc[0] = (uint32_t)(BINS - 1 - (BPT * threadIdx.x + i));  // digit of the k-th key
                    bc[1] = run;                                             // keys above that digit
                    bc[2] = tot[i];                                          // keys in that digit
                }
                run += tot[i];
            }
        }
        __syncthreads();
        const uint32_t digit = bc[0], above = bc[1], inbin = bc[2];
        krem -= (int)above;
        prefix |= digit << shift;
        mask |= dm << shift;
        if ((int)inbin == krem) {  // the k-th key's bin is taken entirely: no tie
            ties = false;
            break;
        }
    }
    const uint32_t T = prefix;

    // ---- counts of this slice; with a cluster, exchanged for the CTA's output offset
    // (the histogram path has its offsets already)
    if (!have_offsets) {
        uint32_t my = 0u;
        for (int i = threadIdx.x; i < cnt; i += NT) {
            const uint32_t kk = keys[i];
            if (ties ? kk > T : kk >= T) my += 1u << 16;
            else if (ties && kk == T) my += 1u;
        }
        uint32_t ctot;
        (void)block_scan1<NW>(my, wsum[0], &ctot);  // per-thread counts < 2^16: slices <= 40960 keys
        if constexpr (CLUSTER) {
            if (threadIdx.x == 0) {
                xch[0] = ctot >> 16;
                xch[1] = ctot & 0xffffu;
            }
            cl_sync<true>();
            if (warp == 0) {  // lane q < c reads CTA q's counts; all peers at once
                uint32_t g = 0u, q = 0u;
                if (lane < c) {
                    const uint32_t* px = cl_peer<true>(xch, lane);
                    g = px[0];
                    q = px[1];
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    g += __shfl_xor_sync(0xffffffffu, g, o);
                    q += __shfl_xor_sync(0xffffffffu, q, o);
                }
                if (lane == 0) {
                    bc[0] = g;
                    bc[1] = q;
                }
            }
            __syncthreads();
            gt_before = bc[0];
            eq_before = bc[1];
            // peers read this CTA's shared memory no more; they may leave after the wait below
            asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
        }
    }
    const int quota = ties ? max(0, krem - (int)eq_before) : 0;
    const int out_base = (int)gt_before + (ties ? min((int)eq_before, krem) : 0);

    // ---- ordered compaction of the slice: KPT consecutive keys per thread, positions from a
    // block-wide scan per NT * KPT keys
    int carry_gt = 0, carry_eq = 0;
    for (int tb = 0, flip = 1; tb < cnt; tb += NT * KPT, flip ^= 1) {
        const int i0 = tb + threadIdx.x * KPT;
        uint32_t kk[KPT];
        load_keys<KPT>(tk_dyn, i0, cnt, kk);
        uint32_t gm = 0u, em = 0u;
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
            const bool valid = i0 + e < cnt;
            if (valid && (ties ? kk[e] > T : kk[e] >= T)) gm |= 1u << e;
            else if (valid && ties && kk[e] == T) em |= 1u << e;
        }
        const uint32_t packed = ((uint32_t)__popc(gm) << 16) | (uint32_t)__popc(em);
        uint32_t ttot;
        const uint32_t excl = block_scan1<NW>(packed, wsum[flip], &ttot) - packed;
        int gb = carry_gt + (int)(excl >> 16);
        int eb = carry_eq + (int)(excl & 0xffffu);
        if (gm | em) {
#pragma unroll
            for (int e = 0; e < KPT; ++e) {
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
        }
        carry_gt += (int)(ttot >> 16);
        carry_eq += (int)(ttot & 0xffffu);
    }
    if constexpr (CLUSTER) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if constexpr (HIST) {
        // every CTA of the cluster has read the histogram (before the first cluster barrier)
        if (c == 0) {
            uint4* h4 = reinterpret_cast<uint4*>(hrow);
            for (int i = threadIdx.x; i < LI_HIST_BINS / 4; i += NT) h4[i] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

constexpr int TK_SMEM_BUDGET = 220 * 1024;  // dynamic shared memory a top-k CTA may take
constexpr int TK_CAND_MAX = 8192;            // candidate keys per list (HIST)

template <int NT, bool CLUSTER, bool HIST>
cudaError_t launch_one(const TopkArgs& a, int row0, int nr, int cs, int chunk, cudaStream_t st) {
    using S = TopkShape<NT, CLUSTER>;
    auto kern = topk_kernel<NT, CLUSTER, HIST>;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TK_SMEM_BUDGET);
        if (CLUSTER) cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        attr_done[dev] = true;
    }
    TopkArgs b = a;
    size_t smem = S::smem(chunk);
    if constexpr (HIST) {
        // candidate lists take what the slice leaves; below 256 keys the plain passes always run
        const long long room = ((long long)TK_SMEM_BUDGET - (long long)smem) / (CLUSTER ? 8 : 4);
        int cap = (int)std::min<long long>(TK_CAND_MAX, std::max<long long>(room, 0)) & ~3;
        if (cap < 256) cap = 0;
        b.cand_cap = cap;
        smem = S::smem_hist(chunk, cap);
    }
    return launch_pdl(kern, dim3(CLUSTER ? cs : 1, nr), dim3(NT), smem, st, CLUSTER ? cs : 1, b, row0, chunk);
}

// Whether a cluster of 16 top-k CTAs, each with the whole shared-memory budget, can be resident at
// once on this device (a non-portable size: it needs 16 free SMs of one GPC); otherwise 8 is the cap.
int cluster_cap() {
    static int cap[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && cap[dev]) return cap[dev];
    int c = 8;
    auto kern = topk_kernel<512, true, true>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TK_SMEM_BUDGET) == cudaSuccess &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(16, 1, 1);
        cfg.blockDim = dim3(512, 1, 1);
        cfg.dynamicSmemBytes = TK_SMEM_BUDGET;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 16;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= 1) c = 16;
    }
    cudaGetLastError();
    if (dev < 64) cap[dev] = c;
    return c;
}

}  // namespace

li_status launch_topk(const TopkArgs& a, cudaStream_t st) {
    if (a.rows <= 0) return LI_OK;
    const int maxl = max(a.max_len, 1);
    const int sms = host_num_sms();
    auto chunk_of = [&](int csz) { return (((maxl + csz - 1) / csz) + 3) & ~3; };
    // few rows: split each row over a cluster so that about 4K keys land on each CTA
    // (the load and every sweep run on many SMs); many rows: one CTA per row
    // (a cluster larger than 8 only while every row's cluster still fits beside the others in one wave)
    const int cap = cluster_cap();
    int cs = 1;
    if (a.rows < sms)
        while (cs < cap && chunk_of(cs) > TK_SLICE && (cs < 8 || (long long)(2 * cs) * a.rows <= sms)) cs *= 2;
    while (cs < cap && chunk_of(cs) > TK_SMEM_ROW) cs *= 2;
    const int chunk = chunk_of(cs);
    if (chunk > TK_SMEM_ROW) return LI_ERR_UNSUPPORTED;
    const bool small = chunk <= 8192;
    for (int row0 = 0; row0 < a.rows; row0 += 65535) {
        const int nr = min(65535, a.rows - row0);
        cudaError_t e;
        if (a.hist) {
            if (cs == 1) e = small ? launch_one<512, false, true>(a, row0, nr, cs, chunk, st)
                                   : launch_one<1024, false, true>(a, row0, nr, cs, chunk, st);
            // slices of up to 4096 keys in clusters of 2 to 8: 1024 threads, four keys each in the
            // sweeps (measured faster in the decode step at B = 8, L = 8K-32K, and no slower for the
            // HS followers' 2-CTA rows); longer slices keep 512 (1024 was much slower on 8K-key slices)
            else if (chunk <= TK_SLICE && cs >= 2 && cs <= 8)
                e = launch_one<1024, true, true>(a, row0, nr, cs, chunk, st);
            else e = launch_one<512, true, true>(a, row0, nr, cs, chunk, st);
        } else {
            if (cs == 1) e = small ? launch_one<512, false, false>(a, row0, nr, cs, chunk, st)
                                   : launch_one<1024, false, false>(a, row0, nr, cs, chunk, st);
            else e = launch_one<512, true, false>(a, row0, nr, cs, chunk, st);
        }
        if (e != cudaSuccess) return host_check_launch();
        const li_status s = host_check_launch();
        if (s != LI_OK) return s;
    }
    return LI_OK;
}

}  // namespace li
