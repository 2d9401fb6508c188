// FP8 latent-cache scorer: the LatentIndex scan over a shared latent cache
// stored in e4m3 with one fp32 scale per cached token,
//
//   I[b,s] = cs[s] * sum_j w_eff[b,j] * ReLU(q8[b,j,:] . c8[s,:]),
//
// where q8 / w_eff come from the absorbed bf16 query q~ quantised per
// (request, head) exactly as li_quantize_query does (absmax / 448 scale), so
// that q = q8 * sq and c = c8 * cs.  The latent width is d_c = 192: the
// DeepSeek-V3.2 layout of LatentIndex's shared latent, 64 RoPE + 128 NoPE
// dimensions (LatentIndex appendix, Table 5).
//
// A 192-byte latent row is loaded as three 64-byte K blocks (TMA boxes of
// 128 rows x 64 bytes with the 64-byte swizzle); each block is two
// tcgen05.mma.kind::f8f6f4 steps of K = 32.  Keys are the M = 128 operand (one
// TMEM lane per key), heads the N = 64 operand, as in the FP8 decode scorer;
// the head reduction, ReLU and the key scale happen in the epilogue's
// registers and only one fp32 score per key is written.
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 TMEM allocator and
// MMA issuer, warps 2..9 quantise the query, warps 2..5 then run the
// epilogue.  Grid: (CTAs per request, requests); two CTAs per SM.
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

constexpr int L8_H = 64;                    // heads = MMA N
constexpr int L8_M = 128;                   // keys per tile = MMA M
constexpr int L8_DC = 192;                  // latent width (bytes per e4m3 row)
constexpr int L8_KB = 64;                   // bytes per K block
constexpr int L8_KBLK = L8_DC / L8_KB;      // 3
constexpr int L8_STAGES = 9;                // K blocks in flight: three tiles
constexpr int L8_NACC = 4;                  // TMEM accumulators of 64 columns
constexpr int L8_STAGE_BYTES = L8_M * L8_KB;                  // 8 KB
constexpr int L8_QBLK_BYTES = L8_H * L8_KB;                   // 4 KB per query K block
constexpr int L8_OFF_Q = L8_STAGES * L8_STAGE_BYTES;
constexpr int L8_OFF_W = L8_OFF_Q + L8_KBLK * L8_QBLK_BYTES;
constexpr int L8_OFF_BAR = L8_OFF_W + L8_H * 4;
constexpr int L8_NBAR = 2 * L8_STAGES + 2 * L8_NACC + 1;
constexpr int L8_OFF_TMEM = L8_OFF_BAR + L8_NBAR * 8;
constexpr int L8_OFF_HIST = (L8_OFF_TMEM + 16 + 15) & ~15;
constexpr int L8_PRO_WARPS = 8;
constexpr int L8_THREADS = 64 + 32 * L8_PRO_WARPS;

__host__ __device__ constexpr int l8_smem(bool hist) { return L8_OFF_HIST + (hist ? LI_HIST_BINS * 4 : 0) + 1024; }

__device__ __forceinline__ uint8_t* l8_align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <bool HIST>
__global__ void __launch_bounds__(L8_THREADS, 2) latent8_score_kernel(const __grid_constant__ CUtensorMap cmap,
                                                                     const Latent8Args a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = l8_align1024(smem_raw);
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();
    if ((int)blockIdx.x >= (a.max_len + L8_M - 1) / L8_M) return;  // no tile for any length

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L8_OFF_BAR);
    uint64_t* empty = full + L8_STAGES;
    uint64_t* accf = empty + L8_STAGES;
    uint64_t* acce = accf + L8_NACC;
    uint64_t* qready = acce + L8_NACC;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L8_OFF_TMEM);
    float* wsm = reinterpret_cast<float*>(smem + L8_OFF_W);
    uint8_t* qsm = smem + L8_OFF_Q;
    uint32_t* hs = reinterpret_cast<uint32_t*>(smem + L8_OFF_HIST);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L8_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < L8_NACC; ++i) {
            mbar_init(&accf[i], 1);
            mbar_init(&acce[i], 128);
        }
        mbar_init(qready, 32 * L8_PRO_WARPS);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, L8_NACC * L8_H);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    pdl_wait();
    int len_b = a.len ? __ldg(a.len + b) : a.max_len;
    if (len_b < 0 || len_b > a.max_len) {
        if (threadIdx.x == 0 && blockIdx.x == 0) record_error(a.err, ERRBIT_BOUNDS);
        len_b = len_b < 0 ? 0 : a.max_len;
    }
    const int ntiles = (len_b + L8_M - 1) / L8_M;
    // tiles are dealt round robin: CTA c takes tiles c, c + G, c + 2G, ... (G = CTAs per request), so
    // that every CTA reads from the whole of its request's cache
    const int t0 = blockIdx.x;
    const int tstride = gridDim.x;
    const int nt = t0 < ntiles ? (ntiles - t0 + tstride - 1) / tstride : 0;
    if (nt <= 0) goto done;  // uniform over the CTA

    if (warp == 0) {
        // ------------------------------------------------------------ producer: 3 K blocks per tile
        if (lane == 0) {
            tma_prefetch_desc(&cmap);
            const uint64_t pol = l2_policy_evict_first();
            const long long rowbase = (long long)b * a.batch_rows;
            int stage = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int it = 0; ok && it < nt; ++it) {
                const int y = (int)(rowbase + (long long)(t0 + it * tstride) * L8_M);
                for (int kb = 0; kb < L8_KBLK; ++kb) {
                    if (!mbar_wait(&empty[stage], ph ^ 1u, a.err)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], L8_STAGE_BYTES);
                    tma_load_2d(smem + stage * L8_STAGE_BYTES, &cmap, kb * L8_KB, y, &full[stage], pol);
                    if (++stage == L8_STAGES) { stage = 0; ph ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_f32acc(L8_M, L8_H, kFmtE4M3);
            bool ok = mbar_wait(qready, 0, a.err);
            tc_fence_after();
            const uint32_t qaddr = smem_u32(qsm);
            int stage = 0;
            uint32_t ph = 0;
            for (int it = 0; ok && it < nt; ++it) {
                const int acc = it % L8_NACC;
                const uint32_t aph = (uint32_t)(it / L8_NACC) & 1u;
                if (!mbar_wait(&acce[acc], aph ^ 1u, a.err)) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + (uint32_t)(acc * L8_H);
                for (int kb = 0; kb < L8_KBLK; ++kb) {
                    if (!mbar_wait(&full[stage], ph, a.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t aaddr = smem_u32(smem + stage * L8_STAGE_BYTES);
                    const uint32_t baddr = qaddr + (uint32_t)(kb * L8_QBLK_BYTES);
#pragma unroll
                    for (int kk = 0; kk < L8_KB / 32; ++kk)  // 32-byte K slices of the 64-byte block
                        mma_e4m3(dt, sw64_kmajor_desc(aaddr + kk * 32), sw64_kmajor_desc(baddr + kk * 32), IDESC,
                                 (kb | kk) != 0);
                    tc_commit(&empty[stage]);
                    if (++stage == L8_STAGES) { stage = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&accf[acc]);
            }
        }
    } else {
        // ------------------------------------------------------------ query prep (warps 2..9)
        // Eight heads per warp, four lanes per head, 48 latent elements per lane: the
        // per-(request, head) e4m3 quantisation of li_quantize_query, written in the
        // 64-byte-swizzled K blocks of the MMA's B operand.
        const int et = threadIdx.x - 64;
        const int ew = et >> 5;
        const int h = lane >> 2, l4 = lane & 3;
        const int j = 8 * ew + h;
        const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.q) +
                                                          ((size_t)b * L8_H + j) * L8_DC) +
                           6 * l4;
        uint4 raw[6];
#pragma unroll
        for (int u = 0; u < 6; ++u) raw[u] = __ldg(src + u);
        const float wj = __ldg(a.w + (size_t)b * L8_H + j);
        if constexpr (HIST) {
            for (int i = et; i < LI_HIST_BINS; i += 32 * L8_PRO_WARPS) hs[i] = 0u;
        }
        float m = 0.f;
#pragma unroll
        for (int u = 0; u < 6; ++u) {
            const uint32_t wv[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
            for (int x = 0; x < 4; ++x)
                m = fmaxf(m, fmaxf(fabsf(__uint_as_float(wv[x] << 16)), fabsf(__uint_as_float(wv[x] & 0xffff0000u))));
        }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        const float sq = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
        const float r = __frcp_rn(sq);
#pragma unroll
        for (int u = 0; u < 3; ++u) {  // 16 elements (two raw vectors) -> one 16-byte chunk of e4m3
            const uint32_t wv[8] = {raw[2 * u].x, raw[2 * u].y, raw[2 * u].z, raw[2 * u].w,
                                    raw[2 * u + 1].x, raw[2 * u + 1].y, raw[2 * u + 1].z, raw[2 * u + 1].w};
            float xe[16], ye[16];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                xe[2 * x] = __uint_as_float(wv[x] << 16);
                xe[2 * x + 1] = __uint_as_float(wv[x] & 0xffff0000u);
            }
            quotients_for_e4m3<16>(xe, sq, r, ye);
            uint32_t pk[4];
#pragma unroll
            for (int x = 0; x < 4; ++x)
                pk[x] = e4m3x2(ye[4 * x], ye[4 * x + 1]) | (e4m3x2(ye[4 * x + 2], ye[4 * x + 3]) << 16);
            const int gch = 3 * l4 + u;  // 16-byte chunk of the 192-byte row
            *reinterpret_cast<uint4*>(qsm + (gch >> 2) * L8_QBLK_BYTES + sw64_offset(j, gch & 3)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        if (l4 == 0) wsm[j] = wj * sq;
        fence_proxy_async_smem();
        mbar_arrive(qready);
        asm volatile("bar.sync 1, %0;" ::"n"(32 * L8_PRO_WARPS) : "memory");
        if (warp >= 6) goto done;

        // ------------------------------------------------------------ epilogue (warps 2..5)
        const int g = warp & 3;  // TMEM lane quarter this warp may access
        const long long srow = (long long)b * a.batch_rows;
        float* out = a.scores + (size_t)b * a.scores_ld;
        for (int it = 0; it < nt; ++it) {
            const int acc = it % L8_NACC;
            const uint32_t aph = (uint32_t)(it / L8_NACC) & 1u;
            const int s = (t0 + it * tstride) * L8_M + g * 32 + lane;
            const float sk = s < len_b ? __ldg(a.cscale + srow + s) : 1.f;
            if (!mbar_wait(&accf[acc], aph, a.err)) break;
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(g * 32) << 16) + (uint32_t)(acc * L8_H);
            uint32_t v0[32], v1[32];
            tmem_ld32(tb, v0);
            tmem_ld32(tb + 32, v1);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&acce[acc]);
            const float sum = relu_dot32(v0, wsm) + relu_dot32(v1, wsm + 32);
            if (s < len_b) {
                const float sc = sum * sk;
                out[s] = sc;
                if constexpr (HIST) atomicAdd(&hs[order_key(sc) >> LI_HIST_SHIFT], 1u);
            }
        }
    }
done:
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, L8_NACC * L8_H);
    }
    if constexpr (HIST) {
        // every epilogue count is in (the barrier above): all warps add the non-empty bins to the
        // request's histogram, four bins per shared-memory load
        if (nt > 0) {
            uint32_t* gh = a.hist + (size_t)b * LI_HIST_BINS;
            const uint4* h4 = reinterpret_cast<const uint4*>(hs);
            for (int i = threadIdx.x; i < LI_HIST_BINS / 4; i += L8_THREADS) {
                const uint4 v = h4[i];
                if (v.x) atomicAdd(gh + 4 * i, v.x);
                if (v.y) atomicAdd(gh + 4 * i + 1, v.y);
                if (v.z) atomicAdd(gh + 4 * i + 2, v.z);
                if (v.w) atomicAdd(gh + 4 * i + 3, v.w);
            }
        }
    }
}

template <bool HIST>
li_status launch_impl(const CUtensorMap& map, const Latent8Args& args, int batch, int ntiles_max, cudaStream_t st) {
    auto kern = latent8_score_kernel<HIST>;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, l8_smem(HIST)) != cudaSuccess)
            return host_check_launch();
        attr_done[dev] = true;
    }
    const int sms = host_num_sms();
    // two CTAs per SM in total, spread over the requests, each with about the same number of tiles
    int cpr = max(1, (2 * sms) / max(1, batch));
    int tpc = max(1, (ntiles_max + cpr - 1) / cpr);
    cpr = (ntiles_max + tpc - 1) / tpc;
    Latent8Args a = args;
    a.tiles_per_cta = tpc;
    if (launch_pdl(kern, dim3(max(cpr, 1), batch), dim3(L8_THREADS), l8_smem(HIST), st, 1, map, a) != cudaSuccess)
        return host_check_launch();
    return host_check_launch();
}

}  // namespace

li_status launch_latent8_score(const CUtensorMap& map, const Latent8Args& args, int batch, int ntiles_max,
                               cudaStream_t st) {
    return args.hist ? launch_impl<true>(map, args, batch, ntiles_max, st)
                     : launch_impl<false>(map, args, batch, ntiles_max, st);
}

}  // namespace li
