// Streaming indexer scorer for decode: one query token per request scans its
// entire cache (Multi-layer Indexer abstract: the indexer scores every cached
// token).
//
//   FP8 kind (DSA decode):   I[b,s] = sk[s] * sum_j w_eff[b,j] * ReLU(q8[b,j,:] . k8[s,:])
//                            q8/w_eff come from the bf16 query, quantised per
//                            (request, head) inside the prologue.
//   BF16 kind (LatentIndex): I[b,s] = sum_j w[b,j] * ReLU(q~[b,j,:] . c[s,:])
//                            scoring the shared latent cache with the absorbed
//                            query (LatentIndex abstract and Figure 1).
//
// The logits q.k form a [128 keys x H heads] tile per step: a dense
// contraction, so it runs on the tcgen05 tensor cores with the keys as the
// M=128 operand (one TMEM lane per key) and the heads as N = H (64 for
// DeepSeek-V3.2's indexer, 32 for GLM-5's).  The head
// reduction, ReLU and key scale happen in registers after one tcgen05.ld per
// 32 columns, so the [H, L] logits never reach HBM; only one fp32 score per
// key is written.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: 128-key x 128-byte tiles of the cache, 128-byte
//               swizzle, into a STAGES-deep ring of shared-memory stages.
//   warp 1      TMEM allocator and MMA issuer (one thread): per key tile, the
//               K/32 (FP8) or K/16 (bf16) MMAs into one of NACC accumulators.
//   warps 2..5  query preparation, then the epilogue: TMEM -> registers ->
//               weighted ReLU sum -> one score per key.
// Grid: (CTAs per request, requests).  Each CTA streams every G-th key tile of
// one request (G = CTAs per request); sized for two CTAs per SM.
//
// HIST variants (score + top-k): every written score's order key is also
// counted by its top LI_HIST_BITS bits in a shared-memory histogram, which the
// whole CTA adds to the request's global histogram at the end; the top-k then
// starts from that digit instead of sweeping the row for it.
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

template <int NH, bool FP8, int KBLK, int STAGES, int NACC, bool HIST>
struct StreamCfg {
    static constexpr int H = NH;                       // heads = MMA N (64: DeepSeek-V3.2, 32: GLM-5)
    static_assert(NH == 32 || NH == 64, "head count");
    static constexpr int M = 128;                      // keys per tile = MMA M = TMEM lanes
    static constexpr int STAGE_BYTES = M * 128;        // one 128-byte K block of 128 keys
    static constexpr int Q_BYTES = KBLK * H * 128;     // query operand, same K blocks
    static constexpr int OFF_Q = STAGES * STAGE_BYTES;
    static constexpr int OFF_W = OFF_Q + Q_BYTES;
    static constexpr int OFF_BAR = OFF_W + H * 4;
    static constexpr int NBAR = 2 * STAGES + 2 * NACC + 2;  // ... qready, qload
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int OFF_HIST = OFF_TMEM + 16;
    static constexpr int SMEM = OFF_HIST + (HIST ? LI_HIST_BINS * 4 : 0) + 1024;  // + slack to align the base to 1024
    static_assert(OFF_HIST % 16 == 0, "the histogram is swept 16 bytes at a time");
    static constexpr int TMEM_COLS = NACC * H;
    // FP8: warps 6..9 only help quantise the query in the prologue
    static constexpr int PRO_WARPS = FP8 ? 8 : 4;
    static constexpr int THREADS = 64 + 32 * PRO_WARPS;
    static constexpr int ELEMS_PER_KBLOCK = FP8 ? 128 : 64;
    static_assert(TMEM_COLS == 128 || TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM columns");
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int NH, bool FP8, int KBLK, int STAGES, int NACC, bool HIST>
__global__ void __launch_bounds__(StreamCfg<NH, FP8, KBLK, STAGES, NACC, HIST>::THREADS, 2)
    stream_score_kernel(const __grid_constant__ CUtensorMap kmap, const StreamArgs a) {
    using C = StreamCfg<NH, FP8, KBLK, STAGES, NACC, HIST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);

    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();  // the next kernel of the stream may be scheduled; it waits for this one itself
    if ((int)blockIdx.x >= (a.max_len + C::M - 1) / C::M) return;  // no tile for any length

    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* accf = empty + STAGES;
    uint64_t* acce = accf + NACC;
    uint64_t* qready = acce + NACC;
    uint64_t* qload = qready + 1;  // FP8: the query row's bulk copy into the last stage's buffer
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
    float* wsm = reinterpret_cast<float*>(smem + C::OFF_W);
    uint8_t* qsm = smem + C::OFF_Q;
    uint32_t* hs = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&accf[i], 1);
            mbar_init(&acce[i], 128);
        }
        mbar_init(qready, 32 * C::PRO_WARPS);
        mbar_init(qload, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // everything above overlaps the previous kernel; inputs are read only after it completed
    pdl_wait();
    // FP8: the request's bf16 query row (16 KB) comes in by one bulk copy into the last stage's
    // buffer, issued before any key tile so that it is not queued behind them; the head weights
    // are loaded by the prologue warps.  Both are issued before the length is known.
    constexpr int QHPW = C::H / C::PRO_WARPS;  // heads per prologue warp
    constexpr int QIT = QHPW / 4;              // four heads at a time, eight lanes per head
    constexpr uint32_t QROW_BYTES = C::H * 128 * 2;
    static_assert(!FP8 || QROW_BYTES <= C::STAGE_BYTES, "the query row fits one stage buffer");
    uint8_t* qstage = smem + (STAGES - 1) * C::STAGE_BYTES;
    float qw[FP8 ? QIT : 1];
    if constexpr (FP8) {
        if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(qload, QROW_BYTES + (a.w_bulk ? C::H * 4 : 0));
            bulk_load(qstage, reinterpret_cast<const uint8_t*>(a.q) + (size_t)b * QROW_BYTES, QROW_BYTES, qload);
            if (a.w_bulk) bulk_load(wsm, a.w + (size_t)b * C::H, C::H * 4, qload);  // head weights into wsm
        }
        if (warp >= 2 && !a.w_bulk) {
            const int ew = (threadIdx.x - 64) >> 5;
            const int g8 = lane >> 3;
#pragma unroll
            for (int i = 0; i < QIT; ++i) qw[i] = __ldg(a.w + (size_t)b * C::H + QHPW * ew + 4 * i + g8);
        }
    }
    // multi-token decode: row b is token b % tokens of request b / tokens, which sees its request's
    // cache up to len - (tokens - 1 - b % tokens)
    const int tokens = a.tokens > 1 ? a.tokens : 1;
    const int req = b / tokens;
    int len_b = a.len ? __ldg(a.len + req) : a.max_len;
    if (len_b < 0 || len_b > a.max_len) {
        if (threadIdx.x == 0 && blockIdx.x == 0) record_error(a.err, ERRBIT_BOUNDS);
        len_b = len_b < 0 ? 0 : a.max_len;
    }
    len_b = max(0, len_b - (tokens - 1 - b % tokens));
    const int ntiles = (len_b + C::M - 1) / C::M;
    // tiles are dealt round robin: CTA c takes tiles c, c + G, c + 2G, ... (G = CTAs per request), so
    // that every CTA reads from the whole of its request's cache
    const int t0 = blockIdx.x;
    const int tstride = gridDim.x;
    const int nt = t0 < ntiles ? (ntiles - t0 + tstride - 1) / tstride : 0;
    if (nt <= 0) goto done;  // uniform over the CTA

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&kmap);
            const uint64_t pol = l2_policy_evict_first();
            const long long rowbase = (long long)req * a.batch_rows;
            int stage = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int it = 0; ok && it < nt; ++it) {
                const int y = (int)(rowbase + (long long)(t0 + it * tstride) * C::M);
                for (int kb = 0; kb < KBLK; ++kb) {
                    // FP8: the last stage's buffer first holds the query row, until it is quantised
                    if (FP8 && stage == STAGES - 1 && ph == 0u && !mbar_wait(qready, 0, a.err)) { ok = false; break; }
                    // FP8: one key tile goes out ahead of the query row, the rest once it has landed, so
                    // that the row does not queue behind every CTA's whole first wave of key loads
                    if (FP8 && it * KBLK + kb == 1 && !mbar_wait(qload, 0, a.err)) { ok = false; break; }
                    if (!mbar_wait(&empty[stage], ph ^ 1u, a.err)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
                    tma_load_2d(smem + stage * C::STAGE_BYTES, &kmap, kb * C::ELEMS_PER_KBLOCK, y, &full[stage],
                                pol);
                    if (++stage == STAGES) { stage = 0; ph ^= 1u; }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_f32acc(C::M, C::H, FP8 ? kFmtE4M3 : kFmtBF16);
            bool ok = mbar_wait(qready, 0, a.err);
            tc_fence_after();
            const uint32_t qaddr = smem_u32(qsm);
            int stage = 0;
            uint32_t ph = 0;
            for (int it = 0; ok && it < nt; ++it) {
                const int acc = it % NACC;
                const uint32_t aph = (uint32_t)(it / NACC) & 1u;
                if (!mbar_wait(&acce[acc], aph ^ 1u, a.err)) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + (uint32_t)(acc * C::H);
                for (int kb = 0; kb < KBLK; ++kb) {
                    if (!mbar_wait(&full[stage], ph, a.err)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t aaddr = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t baddr = qaddr + (uint32_t)(kb * C::H * 128);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {  // 32-byte K slices of the 128-byte row
                        const uint64_t ad = sw128_kmajor_desc(aaddr + kk * 32);
                        const uint64_t bd = sw128_kmajor_desc(baddr + kk * 32);
                        if constexpr (FP8) mma_e4m3(dt, ad, bd, IDESC, (kb | kk) != 0);
                        else mma_bf16(dt, ad, bd, IDESC, (kb | kk) != 0);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&accf[acc]);
            }
        }
    } else {
        // ------------------------------------------------------------ query prep
        const int et = threadIdx.x - 64;  // 0 .. 32*PRO_WARPS-1
        const int ew = et >> 5;
        if constexpr (FP8) {
            // 8 heads per warp, four at a time (8 lanes per head, 16 elements per
            // lane), from the query row in shared memory
            const int g8 = lane >> 3, l8 = lane & 7;
            const bool qin = mbar_wait(qload, 0, a.err);
            uint4 qraw[QIT][2];
#pragma unroll
            for (int i = 0; i < QIT; ++i) {
                const int j = QHPW * ew + 4 * i + g8;
                const uint4* src = reinterpret_cast<const uint4*>(qstage + j * 256) + 2 * l8;
                qraw[i][0] = qin ? src[0] : make_uint4(0u, 0u, 0u, 0u);
                qraw[i][1] = qin ? src[1] : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < QIT; ++i) {
                const int j = QHPW * ew + 4 * i + g8;
                float sq;
                const uint4 packed = quantize_head128_g8(qraw[i][0], qraw[i][1], &sq);
                *reinterpret_cast<uint4*>(qsm + sw128_offset(j, l8)) = packed;
                if (l8 == 0) wsm[j] = (a.w_bulk ? wsm[j] : qw[i]) * sq;
            }
        } else {
            constexpr int CH = KBLK * 8;                // 16-byte chunks per query row
            constexpr int PER = C::H * CH / 128;        // chunks per thread
            // every 16-byte chunk straight to its swizzled place by cp.async, all in flight at once
            const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.q) + (size_t)b * C::H * KBLK * 64;
#pragma unroll 4
            for (int g = 0; g < PER; ++g) {
                const int ci = et + 128 * g;
                const int r = ci / CH, cc = ci % CH;
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                                 smem_u32(qsm + (cc >> 3) * (C::H * 128) + sw128_offset(r, cc & 7))),
                             "l"(src + (size_t)ci * 8)
                             : "memory");
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
            if (et < C::H) wsm[et] = __ldg(a.w + (size_t)b * C::H + et);
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        if constexpr (HIST) {
            for (int i = et; i < LI_HIST_BINS; i += 32 * C::PRO_WARPS) hs[i] = 0u;
        }
        fence_proxy_async_smem();
        mbar_arrive(qready);
        // w_eff visible to every epilogue thread
        asm volatile("bar.sync 1, %0;" ::"n"(32 * C::PRO_WARPS) : "memory");
        if (warp >= 6) goto done;  // prologue helpers: nothing more to do

        // ------------------------------------------------------------ epilogue
        const int g = warp & 3;  // TMEM lane quarter this warp may access
        const long long srow = (long long)req * a.batch_rows;
        float* out = a.scores + (size_t)b * a.scores_ld;
        for (int it = 0; it < nt; ++it) {
            const int acc = it % NACC;
            const uint32_t aph = (uint32_t)(it / NACC) & 1u;
            const int s = (t0 + it * tstride) * C::M + g * 32 + lane;
            float sk = 1.f;
            if (FP8 && s < len_b) sk = __ldg(a.kscale + srow + s);
            if (!mbar_wait(&accf[acc], aph, a.err)) break;
            tc_fence_after();
            const uint32_t tb = tmem_base + ((uint32_t)(g * 32) << 16) + (uint32_t)(acc * C::H);
            float sum;
            if constexpr (C::H == 64) {
                uint32_t v0[32], v1[32];
                tmem_ld32(tb, v0);
                tmem_ld32(tb + 32, v1);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&acce[acc]);
                sum = relu_dot32(v0, wsm) + relu_dot32(v1, wsm + 32);
            } else {
                uint32_t v0[32];
                tmem_ld32(tb, v0);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&acce[acc]);
                sum = relu_dot32(v0, wsm);
            }
            if (s < len_b) {
                const float sc = FP8 ? sum * sk : sum;
                out[s] = sc;
                if constexpr (HIST) atomicAdd(&hs[order_key(sc) >> LI_HIST_SHIFT], 1u);
            }
        }
    }
done:
    // the query row's bulk copy must have landed before the CTA may leave (a CTA without a
    // tile never waited for it)
    if (FP8 && threadIdx.x == 0) (void)mbar_wait(qload, 0, a.err);
    __syncwarp();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
    if constexpr (HIST) {
        // every epilogue count is in (the barrier above): add the non-empty bins to the request's
        // histogram.  All warps share the sweep, four bins per shared-memory load; over the four
        // epilogue warps alone, one bin at a time, it took about 1.2 us of the CTA's tail.
        if (nt > 0) {
            uint32_t* gh = a.hist + (size_t)b * LI_HIST_BINS;
            const uint4* h4 = reinterpret_cast<const uint4*>(hs);
            for (int i = threadIdx.x; i < LI_HIST_BINS / 4; i += C::THREADS) {
                const uint4 v = h4[i];
                if (v.x) atomicAdd(gh + 4 * i, v.x);
                if (v.y) atomicAdd(gh + 4 * i + 1, v.y);
                if (v.z) atomicAdd(gh + 4 * i + 2, v.z);
                if (v.w) atomicAdd(gh + 4 * i + 3, v.w);
            }
        }
    }
}

template <int NH, bool FP8, int KBLK, int STAGES, int NACC, bool HIST = false>
li_status launch_one(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max, cudaStream_t st) {
    using C = StreamCfg<NH, FP8, KBLK, STAGES, NACC, HIST>;
    auto kern = stream_score_kernel<NH, FP8, KBLK, STAGES, NACC, HIST>;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
            return host_check_launch();
        attr_done[dev] = true;
    }
    const int sms = host_num_sms();
    // two CTAs per SM in total, spread over the requests, each with about the same number of tiles
    int cpr = max(1, (2 * sms) / max(1, batch));
    int tpc = (ntiles_max + cpr - 1) / cpr;
    tpc = max(tpc, 1);
    cpr = (ntiles_max + tpc - 1) / tpc;
    StreamArgs a = args;
    a.tiles_per_cta = tpc;
    dim3 grid(max(cpr, 1), batch);
    if (launch_pdl(kern, grid, dim3(C::THREADS), C::SMEM, st, 1, map, a) != cudaSuccess) return host_check_launch();
    return host_check_launch();
}

template <bool FP8, int KBLK, int STAGES, int NACC, bool HIST = false>
li_status launch_impl(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max, cudaStream_t st) {
    if (args.heads == 64) return launch_one<64, FP8, KBLK, STAGES, NACC, HIST>(map, args, batch, ntiles_max, st);
    if (args.heads == 32) return launch_one<32, FP8, KBLK, STAGES, NACC, HIST>(map, args, batch, ntiles_max, st);
    return LI_ERR_UNSUPPORTED;
}

}  // namespace

li_status launch_stream_score_fp8(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max,
                                  cudaStream_t st) {
    return launch_impl<true, 1, 6, 4>(map, args, batch, ntiles_max, st);
}

li_status launch_stream_score_fp8_hist(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max,
                                       cudaStream_t st) {
    // five stages instead of six leave room for the histogram at two CTAs per SM
    return launch_impl<true, 1, 5, 4, true>(map, args, batch, ntiles_max, st);
}

li_status launch_stream_score_bf16(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max,
                                   cudaStream_t st) {
    return launch_impl<false, 4, 4, 4>(map, args, batch, ntiles_max, st);
}

li_status launch_stream_score_bf16_hist(const CUtensorMap& map, const StreamArgs& args, int batch, int ntiles_max,
                                        cudaStream_t st) {
    return launch_impl<false, 4, 4, 4, true>(map, args, batch, ntiles_max, st);
}

}  // namespace li
