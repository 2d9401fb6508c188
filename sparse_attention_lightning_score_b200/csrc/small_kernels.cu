// Small kernels of the li library: the standalone query quantiser, the exact
// fp32 scorer, LatentIndex decoder absorption, and the wait self-test.
#include <algorithm>

#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

// ---------------------------------------------------------------------------
// Query quantisation.  Same per-(row, head) recipe as the prologue of the FP8
// scorer (absmax / 448 scale, the quotient rounded as IEEE division rounds it,
// nearest-even saturating e4m3 conversion).  For d = 128 a warp takes four
// heads at a time (8 lanes per head) and walks a grid-stride list of such
// groups with the next two groups' loads in flight while it converts one: the
// conversion is long enough that, without them, too few bytes are in flight to
// keep HBM busy.  Other d: one warp per (row, head).
// ---------------------------------------------------------------------------
constexpr int QZ_BLOCKS_PER_SM = 4;  // 64 registers a thread

// the group's query elements of this lane and, on a head's first lane, its weight
struct QzIn {
    uint4 lo, hi;
    float w;
};

__device__ __forceinline__ QzIn qz_load(const __nv_bfloat16* __restrict__ q, const float* __restrict__ w,
                                        long long nheads, long long grp, int lane) {
    const long long head = grp * 4 + (lane >> 3);
    QzIn in{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u), 0.f};
    if (head < nheads) {
        const uint4* src = reinterpret_cast<const uint4*>(q + head * 128) + 2 * (lane & 7);
        in.lo = __ldg(src);
        in.hi = __ldg(src + 1);
        if (w && (lane & 7) == 0) in.w = __ldg(w + head);
    }
    return in;
}

// all 32 lanes call it together (the absmax shuffles span the warp's 8-lane groups)
__device__ __forceinline__ void qz_convert(long long nheads, long long grp, int lane, const QzIn& in,
                                           uint8_t* __restrict__ q8, float* __restrict__ sq,
                                           float* __restrict__ w_eff) {
    const long long head = grp * 4 + (lane >> 3);
    float s;
    const uint4 packed = quantize_head128_g8(in.lo, in.hi, &s);
    if (head < nheads) {
        reinterpret_cast<uint4*>(q8 + head * 128)[lane & 7] = packed;
        if ((lane & 7) == 0) {
            sq[head] = s;
            if (w_eff) w_eff[head] = in.w * s;
        }
    }
}

__global__ void __launch_bounds__(256, QZ_BLOCKS_PER_SM) quantize_query_kernel(const __nv_bfloat16* __restrict__ q,
                                                             const float* __restrict__ w, long long nheads, int dim,
                                                             uint8_t* __restrict__ q8, float* __restrict__ sq,
                                                             float* __restrict__ w_eff) {
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (dim == 128) {
        const long long ngroups = (nheads + 3) / 4;
        const long long stride = (long long)gridDim.x * (blockDim.x >> 5);
        const float* wq = w_eff ? w : nullptr;
        QzIn in_a = qz_load(q, wq, nheads, gw, lane);           // group g
        QzIn in_b = qz_load(q, wq, nheads, gw + stride, lane);  // group g + stride
        for (long long g = gw; g < ngroups; g += 2 * stride) {  // g is warp-uniform
            const QzIn in_c = qz_load(q, wq, nheads, g + 2 * stride, lane);
            qz_convert(nheads, g, lane, in_a, q8, sq, w_eff);
            if (g + stride < ngroups) {
                const QzIn in_d = qz_load(q, wq, nheads, g + 3 * stride, lane);
                qz_convert(nheads, g + stride, lane, in_b, q8, sq, w_eff);
                in_b = in_d;
            }
            in_a = in_c;
        }
        return;
    }
    if (gw >= nheads) return;  // whole warp
    const __nv_bfloat16* src = q + gw * dim;
    float s;
    {
        float m = 0.f;
        for (int e = lane; e < dim; e += 32) m = fmaxf(m, fabsf(__bfloat162float(src[e])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        s = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
        const float r = __frcp_rn(s);
        for (int e0 = 0; e0 < dim; e0 += 32) {  // uniform trip count: the quotient votes across the warp
            const int e = e0 + lane;
            const uint32_t b = e4m3_quotient(e < dim ? __bfloat162float(src[e]) : 0.f, s, r);
            if (e < dim) q8[gw * dim + e] = (uint8_t)b;
        }
    }
    if (lane == 0) {
        sq[gw] = s;
        if (w_eff) w_eff[gw] = w[gw] * s;
    }
}

// ---------------------------------------------------------------------------
// Exact fp32 scorer (no tensor cores): one thread per cache position, the
// query row and weights of the block's row in shared memory.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) simt_score_kernel(const SimtArgs a) {
    extern __shared__ float sh[];
    float* qs = sh;
    float* ws = sh + a.H * a.d;
    const int r = blockIdx.y;
    for (int i = threadIdx.x; i < a.H * a.d; i += blockDim.x) qs[i] = a.q[(size_t)r * a.H * a.d + i];
    for (int i = threadIdx.x; i < a.H; i += blockDim.x) ws[i] = a.w[(size_t)r * a.H + i];
    __syncthreads();
    long long n = a.causal ? (long long)r + 1 + a.causal_offset : (a.len ? (long long)a.len[r] : a.L);
    if (!a.causal && a.len && (n < 0 || n > a.L) && threadIdx.x == 0 && blockIdx.x == 0) record_error(a.err, ERRBIT_BOUNDS);
    n = n < 0 ? 0 : (n > a.L ? a.L : n);
    for (long long s = (long long)blockIdx.x * blockDim.x + threadIdx.x; s < n; s += (long long)gridDim.x * blockDim.x) {
        const float* kr = a.k + ((long long)r * a.batch_rows + s) * a.d;
        float I = 0.f;
        for (int j = 0; j < a.H; ++j) {
            float x = 0.f;
            for (int e = 0; e < a.d; ++e) x = fmaf(qs[j * a.d + e], kr[e], x);
            I = fmaf(ws[j], fmaxf(x, 0.f), I);
        }
        a.scores[(size_t)r * a.scores_ld + s] = I;
    }
}

// ---------------------------------------------------------------------------
// Decoder absorption: q~[b,j,c] = sum_e q[b,j,e] * W[j,e,c], fp32 accumulate,
// one rounding to bf16.  Grid (heads, dc/64): a block owns head j and 64
// columns of W[j] (d rows x 128 bytes), read once for all requests.  Thread t
// holds 8 columns (one 16-byte load) of rows e = t/8 + 32*i; every load of W is
// issued before any arithmetic, so the block's slice of W is in flight at
// once.  Partial sums over the 32 row groups are reduced with warp shuffles,
// then across the 8 warps through shared memory.
// ---------------------------------------------------------------------------
constexpr int AB_COLS = 64;   // output columns per CTA
constexpr int AB_BMAX = 32;   // requests staged per pass

__host__ __device__ constexpr size_t ab_smem(int d) {
    return (size_t)d * AB_COLS * 2 + (size_t)AB_BMAX * (d + 1) * 4;
}

// One CTA per (head j, 64 output columns, layer): the W slice [d x 64] and up to 32 requests'
// query rows are staged in shared memory with one round trip; thread t owns column t % 64 for the
// requests t / 64, t / 64 + 4, ... and sums over d in its registers (fp32, in order of e), then
// rounds once to bf16.
__global__ void __launch_bounds__(256) absorb_kernel(const __nv_bfloat16* __restrict__ q,
                                                     const __nv_bfloat16* __restrict__ W,
                                                     __nv_bfloat16* __restrict__ qt, int B, int H, int d, int dc) {
    extern __shared__ __align__(16) uint8_t ab_smem_raw[];
    __nv_bfloat16* wsh = reinterpret_cast<__nv_bfloat16*>(ab_smem_raw);                 // [d][64]
    float* qsh = reinterpret_cast<float*>(ab_smem_raw + (size_t)d * AB_COLS * 2);       // [32][d + 1]
    const int j = blockIdx.x;
    const int c0 = blockIdx.y * AB_COLS;
    // layer blockIdx.z: its queries, decoder and output follow the previous layer's
    q += (size_t)blockIdx.z * B * H * d;
    W += (size_t)blockIdx.z * H * d * dc;
    qt += (size_t)blockIdx.z * B * H * dc;
    const int t = threadIdx.x;
    // W slice: d rows x 128 bytes, eight 16-byte units per row, by cp.async with every unit in
    // flight at once (a load-then-store loop waited out one round trip per unit)
    for (int u = t; u < d * 8; u += 256) {
        const int e = u >> 3, v = u & 7;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(wsh + e * AB_COLS + 8 * v)),
                     "l"(W + ((size_t)j * d + e) * dc + c0 + 8 * v)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    const int c = t & (AB_COLS - 1);
    for (int b0 = 0; b0 < B; b0 += AB_BMAX) {
        const int nb = min(AB_BMAX, B - b0);
        for (int i = t; i < nb * d; i += 256) {
            const int bb = i / d, e = i - bb * d;
            qsh[bb * (d + 1) + e] = __bfloat162float(q[((size_t)(b0 + bb) * H + j) * d + e]);
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        for (int bb = t >> 6; bb < nb; bb += 4) {
            const float* qr = qsh + bb * (d + 1);
            float acc = 0.f;
#pragma unroll 8
            for (int e = 0; e < d; ++e) acc = fmaf(qr[e], __bfloat162float(wsh[e * AB_COLS + c]), acc);
            qt[((size_t)(b0 + bb) * H + j) * dc + c0 + c] = __float2bfloat16_rn(acc);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Self-test of the bounded wait: nothing ever arrives on the barrier.
// ---------------------------------------------------------------------------
__global__ void selftest_wait_kernel(const DevErr e) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, e);
}

// ---------------------------------------------------------------------------
// Copy from page-locked host memory mapped into the device's address space
// (a decode step's query and weights): PCIe reads issued by many threads, so
// that the copy is one kernel of the step instead of a separate DMA transfer.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) host_copy_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                                        size_t n16, uint8_t* __restrict__ dst_tail,
                                                        const uint8_t* __restrict__ src_tail, int tail) {
    pdl_trigger();
    pdl_wait();  // the destination may still be read by the previous kernel of the stream
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += stride) dst[i] = src[i];
    if (blockIdx.x == 0 && (int)threadIdx.x < tail) dst_tail[threadIdx.x] = src_tail[threadIdx.x];
}

}  // namespace

li_status launch_host_copy(void* dst, const void* src, size_t bytes, cudaStream_t st) {
    if (bytes == 0) return LI_OK;
    const size_t n16 = bytes / 16;
    const int tail = (int)(bytes % 16);
    const int blocks = (int)std::min<size_t>((n16 + 255) / 256 + 1, 2 * (size_t)host_num_sms());
    if (launch_pdl(host_copy_kernel, dim3(std::max(blocks, 1)), dim3(256), 0, st, 1, static_cast<uint4*>(dst),
                   static_cast<const uint4*>(src), n16, static_cast<uint8_t*>(dst) + n16 * 16,
                   static_cast<const uint8_t*>(src) + n16 * 16, tail) != cudaSuccess)
        return host_check_launch();
    return host_check_launch();
}

li_status launch_quantize_query(const void* q, const float* w, int rows, int heads, int dim, uint8_t* q8, float* sq,
                                float* w_eff, cudaStream_t st) {
    const long long nh = (long long)rows * heads;
    if (nh == 0) return LI_OK;
    const long long warps = dim == 128 ? (nh + 3) / 4 : nh;
    long long blocks = (warps * 32 + 255) / 256;
    if (dim == 128) blocks = std::min<long long>(blocks, (long long)host_num_sms() * QZ_BLOCKS_PER_SM);
    quantize_query_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(q), w, nh, dim, q8,
                                                            sq, w_eff);
    return host_check_launch();
}

li_status launch_simt_score(const SimtArgs& a, cudaStream_t st) {
    if (a.R == 0 || a.L == 0) return LI_OK;
    const size_t smem = (size_t)(a.H * a.d + a.H) * sizeof(float);
    if (smem > 48 * 1024) cudaFuncSetAttribute(simt_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int bx = min((a.L + 127) / 128, 1024);
    for (int r0 = 0; r0 < a.R; r0 += 65535) {
        SimtArgs s = a;
        const int nr = min(65535, a.R - r0);
        s.q = a.q + (size_t)r0 * a.H * a.d;
        s.w = a.w + (size_t)r0 * a.H;
        s.len = a.len ? a.len + r0 : nullptr;
        s.scores = a.scores + (size_t)r0 * a.scores_ld;
        s.k = a.k + (size_t)r0 * a.batch_rows * a.d;
        s.causal_offset = a.causal_offset + r0;
        simt_score_kernel<<<dim3(bx, nr), 128, smem, st>>>(s);
        const li_status e = host_check_launch();
        if (e != LI_OK) return e;
    }
    return LI_OK;
}

li_status launch_absorb(const void* q, const void* wdec, void* qt, int G, int B, int H, int d, int dc,
                        cudaStream_t st) {
    if (B == 0 || G == 0) return LI_OK;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
        if (cudaFuncSetAttribute(absorb_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ab_smem(256)) !=
            cudaSuccess)
            return host_check_launch();
        attr_done[dev] = true;
    }
    absorb_kernel<<<dim3(H, dc / 64, G), 256, ab_smem(d), st>>>(reinterpret_cast<const __nv_bfloat16*>(q),
                                                     reinterpret_cast<const __nv_bfloat16*>(wdec),
                                                     reinterpret_cast<__nv_bfloat16*>(qt), B, H, d, dc);
    return host_check_launch();
}

li_status launch_selftest_wait(unsigned long long limit_ns, cudaStream_t st) {
    DevErr e = host_dev_err();
    e.limit_ns = limit_ns;
    selftest_wait_kernel<<<1, 32, 0, st>>>(e);
    return host_check_launch();
}

}  // namespace li
