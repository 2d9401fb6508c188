// Causal prefill scorer: every query token t scans its own prefix, positions
// s <= t + causal_offset (IndexCache explainer, Why This Exists: in prefill the
// indexer runs over each token's prefix), I[t,s] = sk[s] * sum_j w_eff[t,j] * ReLU(q8[t,j,:] . k8[s,:]).
//
// This is the compute-bound form of the indexer (the indexer is 81% of prefill
// at 200K context on the IndexCache explainer's 30B model).  One MMA tile is
// 128 keys (M, TMEM lanes) x 4 query tokens * 64 heads (N = 256) x d = 128,
// four tcgen05.mma.kind::f8f6f4 instructions with K = 32 each; the accumulator
// (256 fp32 columns) is double-buffered in TMEM (512 columns).
//
// Persistent CTAs, one per SM.  Work units are query blocks of 4 tokens; a
// block of tokens t0..t0+3 needs key tiles 0..(t0+3+offset)/128 (causal
// block skipping).  Blocks are dealt to CTAs largest-first in zigzag order
// so that every CTA gets about the same number of key tiles.  The query block
// (32 KB e4m3) stays in shared memory while its key tiles stream past it
// through a ring of TMA stages; keys of the shared cache are re-read from L2.
//
// Warps: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2..17 epilogue (four
// warps per TMEM lane quarter, one per token).  The epilogue is exact fp32:
// ReLU as FMNMX and the head-weighted sum as packed fp32x2 FMAs, 1.5
// instructions per logit; sixteen warps keep enough of them in flight to
// overlap the next tile's MMA.  A warp holds its token's 64 head weights in
// registers for the whole block: read from shared memory per tile, the
// broadcast loads alone kept the load/store pipe busier than the tensor pipe.
// The next block's weights are fetched from global memory while the current
// block's tiles are processed.
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

constexpr int PF_NT = 4;                       // query tokens per block
constexpr int PF_H = 64;
constexpr int PF_N = PF_NT * PF_H;             // 256
constexpr int PF_M = 128;
constexpr int PF_STAGES = 8;
constexpr int PF_KSTAGE = PF_M * 128;          // 16 KB
constexpr int PF_QBYTES = PF_N * 128;          // 32 KB
constexpr int PF_OFF_Q = PF_STAGES * PF_KSTAGE;
constexpr int PF_OFF_W = PF_OFF_Q + 2 * PF_QBYTES;
constexpr int PF_OFF_BAR = PF_OFF_W + 2 * PF_N * 4;
constexpr int PF_NBAR = 2 * PF_STAGES + 2 + 2 + 2 + 2;
constexpr int PF_OFF_TMEM = PF_OFF_BAR + PF_NBAR * 8;
constexpr int PF_SMEM = PF_OFF_TMEM + 16 + 1024;
constexpr int PF_THREADS = 576;
constexpr int PF_EPI_THREADS = 512;

// 16 consecutive TMEM columns of this thread's lane (32x32b shape, 16 repeats).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// a0/a1 += w[j] * max(v[j - j0], 0) for the 16 heads j0 .. j0+15 (packed fp32x2 FMAs).
template <int J0>
__device__ __forceinline__ void relu_acc16(const uint32_t (&v)[16], const float (&w)[PF_H], float2& a0, float2& a1) {
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        ffma2(a0, fmaxf(__uint_as_float(v[j]), 0.f), fmaxf(__uint_as_float(v[j + 1]), 0.f), w[J0 + j], w[J0 + j + 1]);
        ffma2(a1, fmaxf(__uint_as_float(v[j + 2]), 0.f), fmaxf(__uint_as_float(v[j + 3]), 0.f), w[J0 + j + 2],
              w[J0 + j + 3]);
    }
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Block list of CTA c: positions c, 2G-1-c, 2G+c, 4G-1-c, ... of the blocks
// sorted by decreasing work (block nqb-1 first).
__device__ __forceinline__ int pf_block_at(int i, int c, int G, int nqb) {
    const int pair = i >> 1;
    const int pos = (i & 1) ? (2 * G * pair + 2 * G - 1 - c) : (2 * G * pair + c);
    return pos < nqb ? nqb - 1 - pos : -1;
}

__device__ __forceinline__ int pf_ntiles(int qb, const PrefillArgs& a) {
    long long last = (long long)qb * PF_NT + PF_NT - 1 + a.causal_offset;  // last visible position of the block
    if (last > a.L - 1) last = a.L - 1;
    return last < 0 ? 0 : (int)(last / PF_M) + 1;
}

__global__ void __launch_bounds__(PF_THREADS, 1) prefill_score_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                      const __grid_constant__ CUtensorMap kmap,
                                                                      const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const int nqb = (a.T + PF_NT - 1) / PF_NT;

    uint64_t* kfull = reinterpret_cast<uint64_t*>(smem + PF_OFF_BAR);
    uint64_t* kempty = kfull + PF_STAGES;
    uint64_t* qfull = kempty + PF_STAGES;
    uint64_t* qempty = qfull + 2;
    uint64_t* accf = qempty + 2;
    uint64_t* acce = accf + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + PF_OFF_TMEM);
    float* wbuf = reinterpret_cast<float*>(smem + PF_OFF_W);

    if (pf_block_at(0, c, G, nqb) < 0) return;  // no work for this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < PF_STAGES; ++s) {
            mbar_init(&kfull[s], 1);
            mbar_init(&kempty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], 1);
            mbar_init(&accf[i], 1);
            mbar_init(&acce[i], PF_EPI_THREADS);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&qmap);
            tma_prefetch_desc(&kmap);
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_k = l2_policy_evict_last();
            int stage = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int bi = 0; ok; ++bi) {
                const int qb = pf_block_at(bi, c, G, nqb);
                if (qb < 0) break;
                const int qbuf = bi & 1;
                if (!mbar_wait(&qempty[qbuf], ((bi >> 1) & 1) ^ 1u, a.err)) break;
                mbar_arrive_expect_tx(&qfull[qbuf], PF_QBYTES);
                tma_load_2d(smem + PF_OFF_Q + qbuf * PF_QBYTES, &qmap, 0, qb * PF_NT * PF_H, &qfull[qbuf], pol_q);
                const int nt = pf_ntiles(qb, a);
                for (int kt = 0; kt < nt; ++kt) {
                    if (!mbar_wait(&kempty[stage], ph ^ 1u, a.err)) { ok = false; break; }
                    mbar_arrive_expect_tx(&kfull[stage], PF_KSTAGE);
                    tma_load_2d(smem + stage * PF_KSTAGE, &kmap, 0, kt * PF_M, &kfull[stage], pol_k);
                    if (++stage == PF_STAGES) { stage = 0; ph ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_f32acc(PF_M, PF_N, kFmtE4M3);
            int stage = 0;
            uint32_t ph = 0;
            uint32_t tc = 0;
            bool ok = true;
            for (int bi = 0; ok; ++bi) {
                const int qb = pf_block_at(bi, c, G, nqb);
                if (qb < 0) break;
                const int qbuf = bi & 1;
                if (!mbar_wait(&qfull[qbuf], (bi >> 1) & 1, a.err)) break;
                tc_fence_after();
                const uint32_t baddr = smem_u32(smem + PF_OFF_Q + qbuf * PF_QBYTES);
                const int nt = pf_ntiles(qb, a);
                for (int kt = 0; kt < nt; ++kt, ++tc) {
                    const uint32_t acc = tc & 1u;
                    if (!mbar_wait(&acce[acc], ((tc >> 1) & 1u) ^ 1u, a.err)) { ok = false; break; }
                    if (!mbar_wait(&kfull[stage], ph, a.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t aaddr = smem_u32(smem + stage * PF_KSTAGE);
                    const uint32_t dt = tmem_base + acc * PF_N;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_e4m3(dt, sw128_kmajor_desc(aaddr + kk * 32), sw128_kmajor_desc(baddr + kk * 32), IDESC,
                                 kk != 0);
                    tc_commit(&kempty[stage]);
                    tc_commit(&accf[acc]);
                    if (++stage == PF_STAGES) { stage = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&qempty[qbuf]);
            }
        }
    } else {
        const int e = warp - 2;         // 0..15
        const int g = warp & 3;         // TMEM lane quarter
        const int u = e >> 2;           // this warp's token within the block
        const int et = threadIdx.x - 64;
        // w_eff of block bi is staged in wbuf[bi & 1]; thread et < PF_N owns entry et
        auto w_of = [&](int qb) {
            const int t = qb * PF_NT + et / PF_H;
            return (qb >= 0 && et < PF_N && t < a.T) ? __ldg(a.w_eff + (size_t)qb * PF_N + et) : 0.f;
        };
        float wnext = w_of(pf_block_at(0, c, G, nqb));
        uint32_t tc = 0;
        bool ok = true;
        for (int bi = 0; ok; ++bi) {
            const int qb = pf_block_at(bi, c, G, nqb);
            if (qb < 0) break;
            const int t0 = qb * PF_NT;
            float* wb = wbuf + (bi & 1) * PF_N;
            if (et < PF_N) wb[et] = wnext;
            asm volatile("bar.sync 1, 512;" ::: "memory");
            wnext = w_of(pf_block_at(bi + 1, c, G, nqb));  // consumed at the next block
            float wr[PF_H];
#pragma unroll
            for (int j = 0; j < PF_H; j += 4) {
                const float4 w4 = *reinterpret_cast<const float4*>(wb + u * PF_H + j);
                wr[j] = w4.x;
                wr[j + 1] = w4.y;
                wr[j + 2] = w4.z;
                wr[j + 3] = w4.w;
            }
            const int t = t0 + u;
            float* orow = a.scores + (size_t)t * a.scores_ld;
            const int nt = pf_ntiles(qb, a);
            for (int kt = 0; kt < nt; ++kt, ++tc) {
                const uint32_t acc = tc & 1u;
                const int s = kt * PF_M + g * 32 + lane;
                const float sk = s < a.L ? __ldg(a.kscale + s) : 0.f;
                if (!mbar_wait(&accf[acc], (tc >> 1) & 1u, a.err)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tb = tmem_base + ((uint32_t)(g * 32) << 16) + acc * PF_N + u * PF_H;
                uint32_t v[16];
                float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
                tmem_ld16(tb, v);
                tmem_ld_wait();
                relu_acc16<0>(v, wr, a0, a1);
                tmem_ld16(tb + 16, v);
                tmem_ld_wait();
                relu_acc16<16>(v, wr, a0, a1);
                tmem_ld16(tb + 32, v);
                tmem_ld_wait();
                relu_acc16<32>(v, wr, a0, a1);
                tmem_ld16(tb + 48, v);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&acce[acc]);
                relu_acc16<48>(v, wr, a0, a1);
                const float sum = (a0.x + a0.y) + (a1.x + a1.y);
                if (t < a.T && s <= t + a.causal_offset && s < a.L) orow[s] = sum * sk;
            }
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace

li_status launch_prefill_score(const CUtensorMap& qmap, const CUtensorMap& kmap, const PrefillArgs& a,
                               cudaStream_t st) {
    if (a.T <= 0 || a.L <= 0) return LI_OK;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(prefill_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM) !=
            cudaSuccess)
            return host_check_launch();
        attr_done[dev] = true;
    }
    const int nqb = (a.T + PF_NT - 1) / PF_NT;
    const int grid = min(host_num_sms(), nqb);
    prefill_score_kernel<<<grid, PF_THREADS, PF_SMEM, st>>>(qmap, kmap, a);
    return host_check_launch();
}

}  // namespace li
