// Sparse attention over the indexer's selection: the consumer of the top-k.
// Every layer of a DSA model attends, for each new token, only the 2048 cache
// positions its indexer selected (Multi-layer Indexer, long-version transcript:
// the selection is the only thing that ties the indexer to attention).  The
// attention here has DeepSeek-V3.2's absorbed-MLA decode shape: each cache row
// is one 576-element bf16 vector (512 latent + 64 RoPE) shared by all query
// heads, used whole as the key and through its first 512 elements as the value:
//
//   o[b,h,:] = sum_i softmax_i(scale * q[b,h,:] . kv[b, sel[b,i], :]) * kv[b, sel[b,i], :512]
//
// over the valid selections (sel >= 0).  A request with none gets o = 0.
//
// One CTA takes one request, 64 query heads and 256 selected positions (two
// tiles of 128; a split); a second kernel merges the splits (flash-decoding).
// Inside a CTA:
//   - warps 0-3 stream 16 KB chunks of 64 elements x 128 positions into a ring
//     of shared-memory slots with 16-byte cp.async (eight threads per 128-byte
//     row segment, 128-byte swizzle; pads and rejected selections read as
//     zeros), keeping several chunks in flight per thread;
//   - thread 0 loads the 64 query rows of the CTA's heads by TMA at the start;
//     warp 4 issues S^T_t = K_t Q^T for both tiles (M = 128 positions, N = 64 heads, K = 576)
//     into TMEM and, once P^T_t is ready, O^T += V_t^T P^T_t (M = 128 value
//     elements per block, N = 64 heads, K = 128 positions) with V^T and P^T
//     read MN-major, so nothing is transposed in shared memory;
//   - warps 5-8 (one position per TMEM lane) take each head's maximum over the
//     CTA's 256 positions with warp butterflies, then write P^T_t in bf16 and
//     sum the exponentials, and finally write the split's unnormalised O,
//     maxima and sums.
// The value chunks come through the ring a second time (from L2): the two
// phases keep the softmax exact without rescaling O.
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

constexpr int SA_D = 576;                 // key elements per row
constexpr int SA_DV = 512;                // value elements (the latent part)
constexpr int SA_NH = 64;                 // query heads per CTA (MMA N)
constexpr int SA_M = 128;                 // positions per tile (MMA M of S^T, K of O^T)
constexpr int SA_NT = 2;                  // tiles per CTA
constexpr int SA_POS = SA_NT * SA_M;      // positions per CTA (one split)
constexpr int SA_CH = SA_D / 64;          // 9 chunks of 64 elements per row
constexpr int SA_VCH = SA_DV / 64;        // 8 of them hold the value
constexpr int SA_RS = 6;                  // ring slots
constexpr int SA_CHUNK = SA_M * 128;      // 16 KB: 128 rows x 128 bytes
constexpr int SA_QCHUNK = SA_NH * 128;    // 8 KB: 64 rows x 128 bytes
constexpr int SA_THREADS = 288;           // warps 0-3: gather, warp 4: TMEM + TMA + MMA, warps 5-8: softmax
constexpr int SA_DEPTH = 4;               // chunks in flight per gather thread (< SA_RS)
constexpr int SA_TMEM_COLS = 512;         // S^T: 2 x 64 columns, O^T: 4 blocks x 64 columns
constexpr int SA_O_COL = SA_NT * SA_NH;   // first O^T column
// a value block (M = 128) spans two chunks that must sit in adjacent slots: the
// key phase fills an even number of slots and value chunks come in pairs
static_assert(SA_RS % 2 == 0 && (SA_CH * SA_NT) % 2 == 0 && SA_VCH % 2 == 0, "value chunk pairs");
// a gather thread arrives on a chunk's barrier only once SA_DEPTH newer chunks are issued, and waits
// for the slot of the chunk SA_RS back: that chunk must have been released already
static_assert(SA_RS >= SA_DEPTH + 1, "ring deep enough for the chunks held back");

constexpr int OFF_Q = 0;
constexpr int OFF_RING = OFF_Q + SA_CH * SA_QCHUNK;
constexpr int OFF_P = OFF_RING + SA_RS * SA_CHUNK;
constexpr int OFF_RED = OFF_P + SA_NT * SA_CHUNK;       // [4 warps][64] fp32
constexpr int OFF_M = OFF_RED + 4 * SA_NH * 4;          // [64] per-head maxima
constexpr int OFF_SEL = OFF_M + SA_NH * 4;              // [256] tensor-map rows (-1: none)
constexpr int OFF_BAR = OFF_SEL + SA_POS * 4;           // full[RS], empty[RS], qfull, sdone, pready[NT], odone
constexpr int NBAR = 2 * SA_RS + 3 + SA_NT;
constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr int SA_SMEM = OFF_TMEM + 16 + 1024;           // + slack to align the base to 1024
static_assert(SA_SMEM <= 232448, "shared memory per CTA");

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// 2^x by the SFU's approximation (a couple of ulp; the weights are rounded to bf16 right after).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Shared-memory descriptor for an MN-major operand with the 128-byte swizzle:
// each 128-byte row holds 64 consecutive M (or N) elements of one K index, 8
// rows form a 1024-byte swizzle atom, atoms follow each other along K every
// `sbo` bytes and blocks of 64 M elements every `lbo` bytes.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= uint64_t((smem_addr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1u) << 46;
    d |= uint64_t(2u) << 61;
    return d;
}

// Reduce-scatter of 64 values over the warp: afterwards lane l holds, in v[0]
// and v[1], the reduction over all 32 lanes of heads 2l and 2l+1.  Each step
// keeps the half of the array selected by one lane bit and adds the partner's
// copy of that half: 32 + 16 + 8 + 4 + 2 shuffles.
template <bool MAX>
__device__ __forceinline__ void warp_reduce_scatter64(float (&v)[64], int lane) {
#pragma unroll
    for (int step = 0; step < 5; ++step) {
        const int o = 16 >> step;
        const int half = 32 >> step;
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = MAX ? fmaxf(keep, recv) : keep + recv;
        }
    }
}

__global__ void __launch_bounds__(SA_THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap qmap, const SparseAttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const int split = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    uint8_t* qs = smem + OFF_Q;
    uint8_t* ring = smem + OFF_RING;
    uint8_t* pbuf = smem + OFF_P;
    float* red = reinterpret_cast<float*>(smem + OFF_RED);
    float* msm = reinterpret_cast<float*>(smem + OFF_M);
    int32_t* srow = reinterpret_cast<int32_t*>(smem + OFF_SEL);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint64_t* empty = full + SA_RS;
    uint64_t* qfull = empty + SA_RS;
    uint64_t* sdone = qfull + 1;
    uint64_t* pready = sdone + 1;
    uint64_t* odone = pready + SA_NT;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_TMEM);

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&qmap);
        for (int i = 0; i < SA_RS; ++i) {
            mbar_init(&full[i], 128);
            mbar_init(&empty[i], 1);
        }
        mbar_init(qfull, 1);
        mbar_init(sdone, 1);
        for (int t = 0; t < SA_NT; ++t) mbar_init(&pready[t], 128);
        mbar_init(odone, 1);
        fence_mbar_init();
    }
    if (warp == 4) {
        tmem_alloc(tmem_slot, SA_TMEM_COLS);
        tmem_relinquish();
    }
    pdl_wait();  // the selections may come from the previous kernel of the stream
    if (threadIdx.x == 0) {
        // the 64 query rows of the CTA's heads, first of all (nothing can be consumed before them)
        mbar_arrive_expect_tx(qfull, SA_CH * SA_QCHUNK);
        for (int c = 0; c < SA_CH; ++c)
            tma_load_2d(qs + c * SA_QCHUNK, &qmap, c * 64, b * a.heads + hg * SA_NH, qfull, l2_policy_evict_last());
    }
    if (warp == 0) {
        // the CTA's selections as rows of kv; pads and rejected ones become -1
        for (int i = lane; i < SA_POS; i += 32) {
            const int pos = split * SA_POS + i;
            long long r = -1;
            if (pos < a.k) {
                r = __ldg(a.sel + (size_t)b * a.k + pos);
                if (r >= a.rows_visible) {
                    record_error(a.err, ERRBIT_BOUNDS);
                    r = -1;
                }
                r = r < 0 ? -1 : r + (long long)b * a.batch_rows;
            }
            srow[i] = (int32_t)r;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < 4) {
        // ---------------------------------------------------------------- gather
        // eight threads per 128-byte row segment: thread p copies 16-byte unit p % 8 of positions
        // p / 8 + 16 j (j < 8) of every chunk, so each warp instruction reads four whole segments
        const int p = threadIdx.x;
        const int w16 = p & 7;
        const uint32_t ring_s = smem_u32(ring);
        int pend_slot[SA_DEPTH + 1];
        int pending = 0;
        bool ok = true;
        int n = 0;
        for (int ph2 = 0; ok && ph2 < 2; ++ph2) {  // key phase: chunks 0..8 of each tile; value phase: 0..7
            const int nch = ph2 == 0 ? SA_CH : SA_VCH;
            for (int t = 0; ok && t < SA_NT; ++t) {
                const uint8_t* src[8];
                uint32_t nbytes[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int r = srow[t * SA_M + (p >> 3) + 16 * j];
                    src[j] = static_cast<const uint8_t*>(a.kv) + (r >= 0 ? (size_t)r * (SA_D * 2) : 0) + w16 * 16;
                    nbytes[j] = r >= 0 ? 16u : 0u;
                }
                for (int c = 0; c < nch; ++c, ++n) {
                    const int slot = n % SA_RS;
                    if (!mbar_wait(&empty[slot], ((n / SA_RS) & 1) ^ 1, a.err)) { ok = false; break; }
                    const uint32_t dst = ring_s + slot * SA_CHUNK;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        cp_async16(dst + sw128_offset((p >> 3) + 16 * j, w16), src[j] + c * 128, nbytes[j]);
                    cp_async_commit();
                    pend_slot[pending++] = slot;
                    if (pending > SA_DEPTH) {
                        cp_async_wait<SA_DEPTH>();
                        fence_proxy_async_smem();
                        mbar_arrive(&full[pend_slot[0]]);
#pragma unroll
                        for (int i = 0; i < SA_DEPTH; ++i) pend_slot[i] = pend_slot[i + 1];
                        --pending;
                    }
                }
            }
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        for (int i = 0; i < pending; ++i) mbar_arrive(&full[pend_slot[i]]);
    } else if (warp == 4) {
        // ---------------------------------------------------------------- query load and MMA issuer
        if (lane == 0) {
            const uint32_t ring_s = smem_u32(ring), q_s = smem_u32(qs), p_s = smem_u32(pbuf);
            bool ok = mbar_wait(qfull, 0, a.err);
            tc_fence_after();
            int n = 0;
            constexpr uint32_t IDESC_S = idesc_f32acc(SA_M, SA_NH, kFmtBF16);
            for (int t = 0; ok && t < SA_NT; ++t) {
                for (int c = 0; c < SA_CH; ++c, ++n) {
                    const int slot = n % SA_RS;
                    if (!mbar_wait(&full[slot], (n / SA_RS) & 1, a.err)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)  // 16-element K slices of the 64-element chunk
                        mma_bf16(tmem_base + (uint32_t)(t * SA_NH),
                                 sw128_kmajor_desc(ring_s + slot * SA_CHUNK + kk * 32),
                                 sw128_kmajor_desc(q_s + c * SA_QCHUNK + kk * 32), IDESC_S, (c | kk) != 0);
                    tc_commit(&empty[slot]);
                }
            }
            if (ok) tc_commit(sdone);
            // V^T (M = value elements, K = positions) and P^T (N = heads, K = positions), both MN-major
            constexpr uint32_t IDESC_O = idesc_f32acc(128, SA_NH, kFmtBF16) | (1u << 15) | (1u << 16);
            for (int t = 0; ok && t < SA_NT; ++t) {
                if (!mbar_wait(&pready[t], 0, a.err)) { ok = false; break; }
                tc_fence_after();
                for (int blk = 0; blk < SA_VCH / 2; ++blk, n += 2) {
                    const int slot = n % SA_RS;  // even: its pair is slot + 1
                    if (!mbar_wait(&full[slot], (n / SA_RS) & 1, a.err) ||
                        !mbar_wait(&full[slot + 1], (n / SA_RS) & 1, a.err)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < SA_M / 16; ++ks)  // 16 positions = two 8-row swizzle atoms
                        mma_bf16(tmem_base + (uint32_t)(SA_O_COL + blk * SA_NH),
                                 sw128_mnmajor_desc(ring_s + slot * SA_CHUNK + ks * 2048, SA_CHUNK, 1024),
                                 sw128_mnmajor_desc(p_s + t * SA_CHUNK + ks * 2048, SA_CHUNK, 1024), IDESC_O,
                                 (t | ks) != 0);
                    tc_commit(&empty[slot]);
                    tc_commit(&empty[slot + 1]);
                }
            }
            if (ok) tc_commit(odone);
        }
    } else {
        // ---------------------------------------------------------------- softmax and output
        const int q4 = warp & 3;            // TMEM lane quarter of this warp
        const int row = q4 * 32 + lane;     // position within a tile
        const int te = threadIdx.x - 160;   // 0..127
        const float c2 = a.scale * 1.4426950408889634f;  // exp(x) = exp2(x log2 e)
        const bool sok = mbar_wait(sdone, 0, a.err);
        if (sok) tc_fence_after();
        float v[64];
#pragma unroll
        for (int h = 0; h < 64; ++h) v[h] = -INFINITY;
        if (sok) {
#pragma unroll 1
            for (int t = 0; t < SA_NT; ++t) {
                const uint32_t tb = tmem_base + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(t * SA_NH);
                uint32_t r0[32], r1[32];
                tmem_ld32(tb, r0);
                tmem_ld32(tb + 32, r1);
                tmem_ld_wait();
                if (srow[t * SA_M + row] >= 0) {
#pragma unroll
                    for (int h = 0; h < 32; ++h) {
                        v[h] = fmaxf(v[h], __uint_as_float(r0[h]) * c2);
                        v[h + 32] = fmaxf(v[h + 32], __uint_as_float(r1[h]) * c2);
                    }
                }
            }
        }
        warp_reduce_scatter64<true>(v, lane);
        *reinterpret_cast<float2*>(red + q4 * SA_NH + 2 * lane) = make_float2(v[0], v[1]);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (te < SA_NH) msm[te] = fmaxf(fmaxf(red[te], red[SA_NH + te]), fmaxf(red[2 * SA_NH + te], red[3 * SA_NH + te]));
        asm volatile("bar.sync 1, 128;" ::: "memory");
        float l[64];
#pragma unroll
        for (int h = 0; h < 64; ++h) l[h] = 0.f;
#pragma unroll 1
        for (int t = 0; t < SA_NT; ++t) {
            const bool valid = sok && srow[t * SA_M + row] >= 0;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {  // 32 heads at a time
                uint32_t r[32];
                if (sok) {
                    tmem_ld32(tmem_base + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(t * SA_NH + hh * 32), r);
                    tmem_ld_wait();
                }
                uint32_t pk[16];
#pragma unroll
                for (int h = 0; h < 32; h += 2) {
                    const float2 m2 = *reinterpret_cast<const float2*>(msm + hh * 32 + h);
                    const float p0 = valid ? ex2_approx(__fmaf_rn(__uint_as_float(r[h]), c2, -m2.x)) : 0.f;
                    const float p1 = valid ? ex2_approx(__fmaf_rn(__uint_as_float(r[h + 1]), c2, -m2.y)) : 0.f;
                    l[hh * 32 + h] += p0;
                    l[hh * 32 + h + 1] += p1;
                    __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
                    pk[h >> 1] = *reinterpret_cast<uint32_t*>(&pp);
                }
                // P^T_t row: heads 32hh..32hh+31 in bf16, 128-byte swizzle
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    *reinterpret_cast<uint4*>(pbuf + t * SA_CHUNK + sw128_offset(row, hh * 4 + w)) =
                        make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&pready[t]);
        }
        warp_reduce_scatter64<false>(l, lane);  // the maxima in red were read before the last barrier
        *reinterpret_cast<float2*>(red + q4 * SA_NH + 2 * lane) = make_float2(l[0], l[1]);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const size_t part = ((size_t)b * a.splits + split) * a.heads + (size_t)hg * SA_NH;
        if (te < SA_NH) {
            a.mpart[part + te] = msm[te];
            a.lpart[part + te] = (red[te] + red[SA_NH + te]) + (red[2 * SA_NH + te] + red[3 * SA_NH + te]);
        }
        if (mbar_wait(odone, 0, a.err)) {
            tc_fence_after();
            float* op = a.opart + part * SA_DV;
#pragma unroll 1
            for (int blk = 0; blk < SA_DV / 128; ++blk) {
                const uint32_t tb = tmem_base + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(SA_O_COL + blk * SA_NH);
                uint32_t r0[32], r1[32];
                tmem_ld32(tb, r0);
                tmem_ld32(tb + 32, r1);
                tmem_ld_wait();
                const int d = blk * 128 + row;
#pragma unroll
                for (int h = 0; h < 32; ++h) {
                    op[(size_t)h * SA_DV + d] = __uint_as_float(r0[h]);
                    op[(size_t)(h + 32) * SA_DV + d] = __uint_as_float(r1[h]);
                }
            }
        }
    }
    __syncwarp();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem_base, SA_TMEM_COLS);
    }
}

// Merge of the splits: o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s with M
// the largest m_s (maxima are in the log2 domain).  One CTA per (head, request),
// four value elements per thread.
__global__ void __launch_bounds__(128) sparse_attn_merge_kernel(const SparseAttnArgs a) {
    const int h = blockIdx.x, b = blockIdx.y;
    const int d = threadIdx.x * 4;
    float M = -INFINITY;
    for (int s = 0; s < a.splits; ++s) M = fmaxf(M, a.mpart[((size_t)b * a.splits + s) * a.heads + h]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < a.splits; ++s) {
            const size_t part = ((size_t)b * a.splits + s) * a.heads + h;
            const float m = a.mpart[part];
            if (m == -INFINITY) continue;
            const float f = exp2f(m - M);
            L += f * a.lpart[part];
            const float4 o = *reinterpret_cast<const float4*>(a.opart + part * SA_DV + d);
            acc.x += f * o.x;
            acc.y += f * o.y;
            acc.z += f * o.z;
            acc.w += f * o.w;
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    *reinterpret_cast<float4*>(a.out + ((size_t)b * a.heads + h) * SA_DV + d) =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

}  // namespace

size_t sparse_attn_workspace_bytes(int batch, int heads, int k) {
    const size_t splits = (size_t)(k + SA_POS - 1) / SA_POS;
    const size_t parts = (size_t)batch * splits * heads;
    return parts * SA_DV * 4 + 2 * ((parts * 4 + 255) / 256 * 256);
}

int sparse_attn_splits(int k) { return (k + SA_POS - 1) / SA_POS; }

li_status launch_sparse_attn(const CUtensorMap& qmap, SparseAttnArgs a, cudaStream_t st) {
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SA_SMEM) !=
            cudaSuccess)
            return host_check_launch();
        attr_done[dev] = true;
    }
    a.splits = sparse_attn_splits(a.k);
    dim3 grid(a.splits, a.heads / SA_NH, a.batch);
    if (launch_pdl(sparse_attn_kernel, grid, dim3(SA_THREADS), SA_SMEM, st, 1, qmap, a) != cudaSuccess)
        return host_check_launch();
    const li_status s = host_check_launch();
    if (s != LI_OK) return s;
    sparse_attn_merge_kernel<<<dim3(a.heads, a.batch), 128, 0, st>>>(a);
    return host_check_launch();
}

}  // namespace li
