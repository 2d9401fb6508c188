// Hierarchical selection (LatentIndex abstract): followers independently
// refine the candidate set proposed by the anchor.  This kernel gathers each
// candidate latent row c[b, cand[b,i]] ONCE and scores it against the
// absorbed queries of all F followers in one tensor-core pass:
//
//     I_f[b,i] = sum_j w[f,b,j] * ReLU(q~[f,b,j,:] . c[b, cand[b,i], :])
//
// MMA tile: 128 gathered candidates (M) x F*H follower-heads (N <= 256; H = 64
// for DeepSeek-V3.2's indexer, 32 for GLM-5's) x 256
// latent dims (four 128-byte K blocks, 16 tcgen05.mma.kind::f16 with K = 16).
// Rows are gathered with 16-byte cp.async into the 128-byte-swizzled K-major
// layout the MMA reads; padding (negative) candidates are zero-filled and
// scored -inf so the following top-k never prefers them; candidates outside
// the cache are reported (LI_ERR_BOUNDS) and zero-filled, never read.
//
// The followers' query blocks (F x 4 K blocks of H rows) come by TMA from a
// tensor map over q~, straight into the same layout.
//
// Warps: 0..3 gather producers, 4 TMEM allocator + MMA issuer, 5..8 follower
// weights (one thread issues the query TMA) and epilogue.  Output: scores [F*B, round4(C)] fp32, and
// (optionally) each row's first-digit histogram for the follower top-k, counted
// by the epilogue warps with one global atomic per distinct digit per warp.
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

constexpr int HS_M = 128;
constexpr int HS_DC = 256;
constexpr int HS_KBLK = 4;
constexpr int HS_STAGES = 6;
constexpr int HS_STAGE_BYTES = HS_M * 128;
constexpr int HS_DEPTH = 3;  // cp.async groups in flight per producer thread
constexpr int HS_THREADS = 288;

template <int F, int H>
struct HsCfg {
    static_assert(H == 64 || H == 32, "head count");
    static constexpr int N = F * H;
    static constexpr int Q_BYTES = HS_KBLK * N * 128;
    static constexpr int OFF_Q = HS_STAGES * HS_STAGE_BYTES;
    static constexpr int OFF_W = OFF_Q + Q_BYTES;
    static constexpr int OFF_BAR = OFF_W + N * 4;
    static constexpr int NBAR = 2 * HS_STAGES + 2 + 2 + 1;  // full, empty, accf, acce, qtma
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_TMEM + 16 + 1024;
    static constexpr int TMEM_COLS = (2 * N <= 128) ? 128 : ((2 * N <= 256) ? 256 : 512);
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int F, int H>
__global__ void __launch_bounds__(HS_THREADS, 1) hs_rescore_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                    const HsArgs a, int tiles_per_cta) {
    using C = HsCfg<F, H>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = (a.C + HS_M - 1) / HS_M;
    const int t0 = blockIdx.x * tiles_per_cta;
    const int nt = min(t0 + tiles_per_cta, ntiles) - t0;
    if (nt <= 0) return;
    const int ldw = (a.C + 3) & ~3;

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + HS_STAGES;
    uint64_t* accf = empty + HS_STAGES;
    uint64_t* acce = accf + 2;
    uint64_t* qtma = acce + 2;  // the followers' query blocks, by TMA
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
    float* wsm = reinterpret_cast<float*>(smem + C::OFF_W);
    uint8_t* qsm = smem + C::OFF_Q;

    if (threadIdx.x == 0) {
        for (int s = 0; s < HS_STAGES; ++s) {
            mbar_init(&full[s], 128);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&accf[i], 1);
            mbar_init(&acce[i], 128);
        }
        mbar_init(qtma, 1);
        fence_mbar_init();
    }
    if (warp == 4) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int32_t* cand = a.cand + (size_t)b * a.C;
    const long long rowbase = (long long)b * a.batch_rows;

    if (warp < 4) {
        // ------------------------------------------------------------ gather producers
        // Thread p handles row (p) of every stage: 8 chunks of 16 bytes of one
        // 128-byte K block, written at their swizzled positions.
        const int p = threadIdx.x;  // 0..127 = row within the tile
        int stage = 0;
        uint32_t ph = 0;
        int pending = 0;
        int pend_stage[HS_DEPTH + 1];
        bool ok = true;
        for (int it = 0; ok && it < nt; ++it) {
            const int i = (t0 + it) * HS_M + p;
            int s = i < a.C ? __ldg(cand + i) : -1;
            uint32_t nbytes = 16;
            const long long lim = a.batch_rows > 0 ? min((long long)a.batch_rows, a.cache_rows - rowbase)
                                                   : a.cache_rows;
            if (s < 0) nbytes = 0;
            else if (s >= lim) {
                record_error(a.err, ERRBIT_BOUNDS);
                nbytes = 0;
            }
            const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.c) +
                                       (nbytes ? (size_t)(rowbase + s) * HS_DC : 0);
            for (int kb = 0; kb < HS_KBLK; ++kb) {
                if (!mbar_wait(&empty[stage], ph ^ 1u, a.err)) { ok = false; break; }
                const uint32_t dst = smem_u32(smem + stage * HS_STAGE_BYTES);
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    cp_async16(dst + sw128_offset(p, ch), src + kb * 64 + ch * 8, nbytes);
                cp_async_commit();
                pend_stage[pending++] = stage;
                if (pending > HS_DEPTH) {
                    cp_async_wait<HS_DEPTH>();
                    fence_proxy_async_smem();
                    mbar_arrive(&full[pend_stage[0]]);
#pragma unroll
                    for (int q = 0; q < HS_DEPTH; ++q) pend_stage[q] = pend_stage[q + 1];
                    --pending;
                }
                if (++stage == HS_STAGES) { stage = 0; ph ^= 1u; }
            }
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        for (int q = 0; q < pending; ++q) mbar_arrive(&full[pend_stage[q]]);
    } else if (warp == 4) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_f32acc(HS_M, C::N, kFmtBF16);
            bool ok = mbar_wait(qtma, 0, a.err);
            tc_fence_after();
            const uint32_t qaddr = smem_u32(qsm);
            int stage = 0;
            uint32_t ph = 0;
            for (int it = 0; ok && it < nt; ++it) {
                const int acc = it & 1;
                if (!mbar_wait(&acce[acc], ((it >> 1) & 1) ^ 1u, a.err)) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + (uint32_t)(acc * C::N);
                for (int kb = 0; kb < HS_KBLK; ++kb) {
                    if (!mbar_wait(&full[stage], ph, a.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t aaddr = smem_u32(smem + stage * HS_STAGE_BYTES);
                    const uint32_t baddr = qaddr + (uint32_t)(kb * C::N * 128);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(dt, sw128_kmajor_desc(aaddr + kk * 32), sw128_kmajor_desc(baddr + kk * 32), IDESC,
                                 (kb | kk) != 0);
                    tc_commit(&empty[stage]);
                    if (++stage == HS_STAGES) { stage = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&accf[acc]);
            }
        }
    } else {
        // ------------------------------------------------------------ follower queries
        const int et = threadIdx.x - 160;  // 0..127
        constexpr int CH = HS_KBLK * 8;    // 16-byte chunks per query row
        constexpr int PER = C::N * CH / 128;  // 16 chunks per thread per follower
        // the F query blocks come by TMA, one 64-element K block of H rows per load, straight into
        // the 128-byte-swizzled K-major layout the MMA reads (register-staged, then per-thread
        // cp.async copies of the same 96 KB took 4.9, then 3.8 us of a CTA's time at one request)
        if (et == 0) {
            mbar_arrive_expect_tx(qtma, (uint32_t)(F * HS_KBLK * H * 128));
#pragma unroll
            for (int f = 0; f < F; ++f)
#pragma unroll
                for (int kb = 0; kb < HS_KBLK; ++kb)
                    tma_load_2d(qsm + kb * (C::N * 128) + f * H * 128, &qmap, kb * 64, (f * a.B + b) * H, qtma,
                                l2_policy_evict_last());
        }
        for (int r = et; r < C::N; r += 128) {
            const int f = r / H, j = r % H;
            wsm[r] = __ldg(a.w + ((size_t)f * a.B + b) * H + j);
        }
        // the head weights, visible to every epilogue thread
        asm volatile("bar.sync 1, 128;" ::: "memory");

        // ------------------------------------------------------------ epilogue
        const int g = warp & 3;
        for (int it = 0; it < nt; ++it) {
            const int acc = it & 1;
            const int i = (t0 + it) * HS_M + g * 32 + lane;
            const int s = i < a.C ? __ldg(cand + i) : -1;
            // warp-uniform exit: the histogram below needs every lane of the warp
            if (!__all_sync(0xffffffffu, mbar_wait(&accf[acc], (it >> 1) & 1, a.err))) break;
            tc_fence_after();
            float res[F];
#pragma unroll
            for (int f = 0; f < F; ++f) {
                const uint32_t tb = tmem_base + ((uint32_t)(g * 32) << 16) + (uint32_t)(acc * C::N + f * H);
                if constexpr (H == 64) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(tb, v0);
                    tmem_ld32(tb + 32, v1);
                    tmem_ld_wait();
                    res[f] = relu_dot32(v0, wsm + f * H) + relu_dot32(v1, wsm + f * H + 32);
                } else {
                    uint32_t v0[32];
                    tmem_ld32(tb, v0);
                    tmem_ld_wait();
                    res[f] = relu_dot32(v0, wsm + f * H);
                }
            }
            tc_fence_before();
            mbar_arrive(&acce[acc]);
#pragma unroll
            for (int f = 0; f < F; ++f) {
                const float v = s >= 0 ? res[f] : -INFINITY;
                if (i < a.C) a.out[((size_t)f * a.B + b) * ldw + i] = v;
                if (a.hist) warp_hist_add(a.hist + ((size_t)f * a.B + b) * LI_HIST_BINS, v, i < a.C);
            }
        }
    }
    // the query blocks' TMA must have landed before the CTA may leave (the MMA issuer waited for
    // them unless it gave up)
    if (threadIdx.x == 160) (void)mbar_wait(qtma, 0, a.err);
    __syncwarp();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <int F, int H>
li_status launch_f(const CUtensorMap& qmap, const HsArgs& a, cudaStream_t st) {
    using C = HsCfg<F, H>;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(hs_rescore_kernel<F, H>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
            cudaSuccess)
            return host_check_launch();
        attr_done[dev] = true;
    }
    const int ntiles = (a.C + HS_M - 1) / HS_M;
    const int sms = host_num_sms();
    int cpr = max(1, sms / max(1, a.B));
    int tpc = max(1, (ntiles + cpr - 1) / cpr);
    cpr = (ntiles + tpc - 1) / tpc;
    hs_rescore_kernel<F, H><<<dim3(cpr, a.B), HS_THREADS, C::SMEM, st>>>(qmap, a, tpc);
    return host_check_launch();
}

}  // namespace

li_status launch_hs_rescore(const CUtensorMap& qmap, const HsArgs& a, cudaStream_t st) {
    if (a.B <= 0 || a.C <= 0) return LI_OK;
    if (a.H == 64) {
        switch (a.F) {
        case 1: return launch_f<1, 64>(qmap, a, st);
        case 2: return launch_f<2, 64>(qmap, a, st);
        case 3: return launch_f<3, 64>(qmap, a, st);
        case 4: return launch_f<4, 64>(qmap, a, st);
        default: return LI_ERR_UNSUPPORTED;
        }
    }
    if (a.H == 32) {
        switch (a.F) {
        case 1: return launch_f<1, 32>(qmap, a, st);
        case 2: return launch_f<2, 32>(qmap, a, st);
        case 3: return launch_f<3, 32>(qmap, a, st);
        case 4: return launch_f<4, 32>(qmap, a, st);
        default: return LI_ERR_UNSUPPORTED;
        }
    }
    return LI_ERR_UNSUPPORTED;
}

}  // namespace li
