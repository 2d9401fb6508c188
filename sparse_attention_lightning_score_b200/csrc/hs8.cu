// Hierarchical selection over DeepSeek-V3.2's FP8 latent (LatentIndex
// abstract: followers refine the anchor's candidate set on their own): the
// shared latent is d_c = 192 e4m3 bytes per cached token (64 RoPE + 128 NoPE,
// LatentIndex appendix, Table 5) with one fp32 scale per token, as the FP8
// latent scan reads it.  Each candidate row is gathered ONCE and scored
// against every follower's absorbed query in one tensor-core pass:
//
//     I_f[b,i] = cs[r] * sum_j w_eff[f,b,j] * ReLU(q8[f,b,j,:] . c8[b, r, :]),   r = cand[b,i]
//
// with q8 / w_eff the absorbed bf16 query q~ quantised per (follower, request,
// head) exactly as li_quantize_query does (absmax / 448 scale).
//
// MMA tile: 128 gathered candidates (M) x F*64 follower-heads (N <= 256) x
// 192 bytes: three 64-byte K blocks (64-byte swizzle), two
// tcgen05.mma.kind::f8f6f4 steps of K = 32 each.  Rows come in by coalesced
// 16-byte cp.async (four threads per 64-byte row segment); padding (negative)
// candidates are zero-filled and scored -inf; candidates outside the cache are
// reported (LI_ERR_BOUNDS) and zero-filled, never read.
//
// Warps: 0..3 gather producers, 4 TMEM allocator + MMA issuer, 5..8 follower
// query quantisation, then the epilogue.  Output: scores [F*B, round4(C)] and
// (optionally) each row's first-digit histogram, as the bf16 kernel counts it.
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

constexpr int H8_M = 128;                       // candidates per tile = MMA M
constexpr int H8_H = 64;                        // heads per follower
constexpr int H8_DC = 192;                      // bytes per e4m3 latent row
constexpr int H8_KB = 64;                       // bytes per K block
constexpr int H8_KBLK = H8_DC / H8_KB;          // 3
constexpr int H8_STAGES = 9;                    // K blocks in flight: three tiles
constexpr int H8_STAGE_BYTES = H8_M * H8_KB;    // 8 KB
constexpr int H8_DEPTH = 4;                     // cp.async groups a producer thread keeps in flight
constexpr int H8_THREADS = 288;
// a producer arrives on a stage only once H8_DEPTH newer stages are issued, and waits for the stage
// H8_STAGES back to be released first: that stage must already have been arrived on
static_assert(H8_STAGES >= H8_DEPTH + 1, "stages for the copies held back");

template <int F>
struct H8Cfg {
    static constexpr int N = F * H8_H;                  // follower-heads = MMA N
    static constexpr int QBLK = N * H8_KB;              // bytes of one query K block
    static constexpr int OFF_Q = H8_STAGES * H8_STAGE_BYTES;
    static constexpr int OFF_W = OFF_Q + H8_KBLK * QBLK;
    static constexpr int OFF_BAR = OFF_W + N * 4;
    static constexpr int NBAR = 2 * H8_STAGES + 2 + 2 + 1;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_TMEM + 16 + 1024;   // + slack to align the base to 1024
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

template <int F>
__global__ void __launch_bounds__(H8_THREADS, 1) hs_rescore8_kernel(const Hs8Args a, int tiles_per_cta) {
    using C = H8Cfg<F>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = (a.C + H8_M - 1) / H8_M;
    const int t0 = blockIdx.x * tiles_per_cta;
    const int nt = min(t0 + tiles_per_cta, ntiles) - t0;
    if (nt <= 0) return;
    const int ldw = (a.C + 3) & ~3;

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + H8_STAGES;
    uint64_t* accf = empty + H8_STAGES;
    uint64_t* acce = accf + 2;
    uint64_t* qready = acce + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
    float* wsm = reinterpret_cast<float*>(smem + C::OFF_W);
    uint8_t* qsm = smem + C::OFF_Q;

    if (threadIdx.x == 0) {
        for (int s = 0; s < H8_STAGES; ++s) {
            mbar_init(&full[s], 128);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&accf[i], 1);
            mbar_init(&acce[i], 128);
        }
        mbar_init(qready, 128);
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
    const long long lim = a.batch_rows > 0 ? min((long long)a.batch_rows, a.cache_rows - rowbase) : a.cache_rows;

    if (warp < 4) {
        // ------------------------------------------------------------ gather producers
        // Thread p copies 16-byte unit p % 4 of tile rows p / 4 + 32 j (j < 4) of every 64-byte K
        // block: each warp instruction reads eight whole row segments.
        const int p = threadIdx.x;
        const int u = p & 3;
        int stage = 0;
        uint32_t ph = 0;
        int pending = 0;
        int pend_stage[H8_DEPTH + 1];
        bool ok = true;
        for (int it = 0; ok && it < nt; ++it) {
            const uint8_t* src[4];
            uint32_t nbytes[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = (t0 + it) * H8_M + (p >> 2) + 32 * j;
                const int s = i < a.C ? __ldg(cand + i) : -1;
                bool use = s >= 0;
                if (use && s >= lim) {
                    record_error(a.err, ERRBIT_BOUNDS);
                    use = false;
                }
                nbytes[j] = use ? 16u : 0u;
                src[j] = static_cast<const uint8_t*>(a.c8) + (use ? (size_t)(rowbase + s) * H8_DC : 0) + u * 16;
            }
            for (int kb = 0; kb < H8_KBLK; ++kb) {
                if (!mbar_wait(&empty[stage], ph ^ 1u, a.err)) { ok = false; break; }
                const uint32_t dst = smem_u32(smem + stage * H8_STAGE_BYTES);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    cp_async16(dst + sw64_offset((p >> 2) + 32 * j, u), src[j] + kb * H8_KB, nbytes[j]);
                cp_async_commit();
                pend_stage[pending++] = stage;
                if (pending > H8_DEPTH) {
                    cp_async_wait<H8_DEPTH>();
                    fence_proxy_async_smem();
                    mbar_arrive(&full[pend_stage[0]]);
#pragma unroll
                    for (int q = 0; q < H8_DEPTH; ++q) pend_stage[q] = pend_stage[q + 1];
                    --pending;
                }
                if (++stage == H8_STAGES) { stage = 0; ph ^= 1u; }
            }
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        for (int q = 0; q < pending; ++q) mbar_arrive(&full[pend_stage[q]]);
    } else if (warp == 4) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_f32acc(H8_M, C::N, kFmtE4M3);
            bool ok = mbar_wait(qready, 0, a.err);
            tc_fence_after();
            const uint32_t qaddr = smem_u32(qsm);
            int stage = 0;
            uint32_t ph = 0;
            for (int it = 0; ok && it < nt; ++it) {
                const int acc = it & 1;
                if (!mbar_wait(&acce[acc], ((it >> 1) & 1) ^ 1u, a.err)) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + (uint32_t)(acc * C::N);
                for (int kb = 0; kb < H8_KBLK; ++kb) {
                    if (!mbar_wait(&full[stage], ph, a.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t aaddr = smem_u32(smem + stage * H8_STAGE_BYTES);
                    const uint32_t baddr = qaddr + (uint32_t)(kb * C::QBLK);
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)  // 32-byte K slices of the 64-byte block
                        mma_e4m3(dt, sw64_kmajor_desc(aaddr + kk * 32), sw64_kmajor_desc(baddr + kk * 32), IDESC,
                                 (kb | kk) != 0);
                    tc_commit(&empty[stage]);
                    if (++stage == H8_STAGES) { stage = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&accf[acc]);
            }
        }
    } else {
        // ------------------------------------------------------------ follower queries
        // Row r = f * 64 + j of the B operand: follower f's head j, four lanes per row, 48
        // bf16 elements per lane, quantised per (follower, request, head) into the three
        // 64-byte-swizzled query K blocks; 32 rows per pass of the four warps.
        const int et = threadIdx.x - 160;  // 0..127
        const int l4 = et & 3;
        // the next pass's rows are loaded while this pass is quantised
        auto load_rows = [&](int r0, uint4 (&raw)[6]) {
            const int r = r0 + (et >> 2);
            const size_t qrow = ((size_t)(r / H8_H) * a.B + b) * H8_H + r % H8_H;
            const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.qt) +
                                                              qrow * H8_DC) +
                               6 * l4;
#pragma unroll
            for (int v = 0; v < 6; ++v) raw[v] = __ldg(src + v);
        };
        uint4 raw[6], nxt[6];
        load_rows(0, raw);
        for (int r0 = 0; r0 < C::N; r0 += 32) {
            if (r0 + 32 < C::N) load_rows(r0 + 32, nxt);
            const int r = r0 + (et >> 2);
            const size_t qrow = ((size_t)(r / H8_H) * a.B + b) * H8_H + r % H8_H;
            const float wq = l4 == 0 ? __ldg(a.w + qrow) : 0.f;
            float m = 0.f;
#pragma unroll
            for (int v = 0; v < 6; ++v) {
                const uint32_t wv[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
#pragma unroll
                for (int x = 0; x < 4; ++x)
                    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[x] << 16)), fabsf(__uint_as_float(wv[x] & 0xffff0000u))));
            }
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            const float sq = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
            const float rc = __frcp_rn(sq);
#pragma unroll
            for (int v = 0; v < 3; ++v) {  // 16 elements (two raw vectors) -> one 16-byte chunk of e4m3
                const uint32_t wv[8] = {raw[2 * v].x, raw[2 * v].y, raw[2 * v].z, raw[2 * v].w,
                                        raw[2 * v + 1].x, raw[2 * v + 1].y, raw[2 * v + 1].z, raw[2 * v + 1].w};
                float xe[16], ye[16];
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    xe[2 * x] = __uint_as_float(wv[x] << 16);
                    xe[2 * x + 1] = __uint_as_float(wv[x] & 0xffff0000u);
                }
                quotients_for_e4m3<16>(xe, sq, rc, ye);
                uint32_t pk[4];
#pragma unroll
                for (int x = 0; x < 4; ++x)
                    pk[x] = e4m3x2(ye[4 * x], ye[4 * x + 1]) | (e4m3x2(ye[4 * x + 2], ye[4 * x + 3]) << 16);
                const int gch = 3 * l4 + v;  // 16-byte chunk of the 192-byte row
                *reinterpret_cast<uint4*>(qsm + (gch >> 2) * C::QBLK + sw64_offset(r, gch & 3)) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            if (l4 == 0) wsm[r] = wq * sq;
#pragma unroll
            for (int v = 0; v < 6; ++v) raw[v] = nxt[v];
        }
        fence_proxy_async_smem();
        mbar_arrive(qready);
        asm volatile("bar.sync 1, 128;" ::: "memory");

        // ------------------------------------------------------------ epilogue
        const int g = warp & 3;
        for (int it = 0; it < nt; ++it) {
            const int acc = it & 1;
            const int i = (t0 + it) * H8_M + g * 32 + lane;
            const int s = i < a.C ? __ldg(cand + i) : -1;
            const float scale = (s >= 0 && s < lim) ? __ldg(a.cscale + rowbase + s) : 0.f;
            // warp-uniform exit: the histogram below needs every lane of the warp
            if (!__all_sync(0xffffffffu, mbar_wait(&accf[acc], (it >> 1) & 1, a.err))) break;
            tc_fence_after();
            float res[F];
#pragma unroll
            for (int f = 0; f < F; ++f) {
                const uint32_t tb = tmem_base + ((uint32_t)(g * 32) << 16) + (uint32_t)(acc * C::N + f * H8_H);
                uint32_t v0[32], v1[32];
                tmem_ld32(tb, v0);
                tmem_ld32(tb + 32, v1);
                tmem_ld_wait();
                res[f] = relu_dot32(v0, wsm + f * H8_H) + relu_dot32(v1, wsm + f * H8_H + 32);
            }
            tc_fence_before();
            mbar_arrive(&acce[acc]);
#pragma unroll
            for (int f = 0; f < F; ++f) {
                const float v = s >= 0 ? res[f] * scale : -INFINITY;
                if (i < a.C) a.out[((size_t)f * a.B + b) * ldw + i] = v;
                if (a.hist) warp_hist_add(a.hist + ((size_t)f * a.B + b) * LI_HIST_BINS, v, i < a.C);
            }
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

template <int F>
li_status launch_f(const Hs8Args& a, cudaStream_t st) {
    using C = H8Cfg<F>;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(hs_rescore8_kernel<F>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
            cudaSuccess)
            return host_check_launch();
        attr_done[dev] = true;
    }
    const int ntiles = (a.C + H8_M - 1) / H8_M;
    const int sms = host_num_sms();
    int cpr = max(1, sms / max(1, a.B));
    int tpc = max(1, (ntiles + cpr - 1) / cpr);
    cpr = (ntiles + tpc - 1) / tpc;
    hs_rescore8_kernel<F><<<dim3(cpr, a.B), H8_THREADS, C::SMEM, st>>>(a, tpc);
    return host_check_launch();
}

}  // namespace

li_status launch_hs_rescore8(const Hs8Args& a, cudaStream_t st) {
    if (a.B <= 0 || a.C <= 0) return LI_OK;
    switch (a.F) {
    case 1: return launch_f<1>(a, st);
    case 2: return launch_f<2>(a, st);
    case 3: return launch_f<3>(a, st);
    case 4: return launch_f<4>(a, st);
    default: return LI_ERR_UNSUPPORTED;
    }
}

}  // namespace li
