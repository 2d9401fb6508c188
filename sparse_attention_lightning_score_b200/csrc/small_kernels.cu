// Small kernels of the li library: the standalone query quantiser, the exact
// fp32 scorer, LatentIndex decoder absorption, and the wait self-test.
#include "li_common.cuh"
#include "li_kernels.cuh"

namespace li {

namespace {

// ---------------------------------------------------------------------------
// Query quantisation: one warp per (row, head).  Same per-(row, head) recipe
// as the prologue of the FP8 scorer (absmax / 448 scale, IEEE division,
// nearest-even saturating e4m3 conversion).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_query_kernel(const __nv_bfloat16* __restrict__ q,
                                                             const float* __restrict__ w, long long nheads, int dim,
                                                             uint8_t* __restrict__ q8, float* __restrict__ sq,
                                                             float* __restrict__ w_eff) {
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (dim == 128) {  // four heads per warp, 8 lanes per head
        const long long head = gw * 4 + (lane >> 3);
        if (gw * 4 >= nheads) return;  // whole warp
        const bool live = head < nheads;
        const int l8 = lane & 7;
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
        if (live) {
            const uint4* src = reinterpret_cast<const uint4*>(q + head * 128) + 2 * l8;
            lo = __ldg(src);
            hi = __ldg(src + 1);
        }
        float s;
        const uint4 packed = quantize_head128_g8(lo, hi, &s);  // all lanes take part in the shuffles
        if (live) {
            reinterpret_cast<uint4*>(q8 + head * 128)[l8] = packed;
            if (l8 == 0) {
                sq[head] = s;
                if (w_eff) w_eff[head] = w[head] * s;
            }
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
        for (int e = lane; e < dim; e += 32)
            q8[gw * dim + e] = __nv_cvt_float_to_fp8(__fdiv_rn(__bfloat162float(src[e]), s), __NV_SATFINITE, __NV_E4M3);
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
// one rounding to bf16.  Grid (heads, dc/64); the block's 256 threads cover
// 64 columns as 32 bf16 pairs x 8 groups of e; W[j] is read once per block.
// ---------------------------------------------------------------------------
constexpr int AB_BCH = 16;  // requests per pass over W

__global__ void __launch_bounds__(256) absorb_kernel(const __nv_bfloat16* __restrict__ q,
                                                     const __nv_bfloat16* __restrict__ W,
                                                     __nv_bfloat16* __restrict__ qt, int B, int H, int d, int dc) {
    __shared__ __nv_bfloat16 qsh[AB_BCH][256];
    __shared__ float2 red[8][AB_BCH][32];
    const int j = blockIdx.x;
    const int c0 = blockIdx.y * 64;
    const int cp = threadIdx.x & 31;   // column pair
    const int eg = threadIdx.x >> 5;   // e group
    for (int b0 = 0; b0 < B; b0 += AB_BCH) {
        const int nb = min(AB_BCH, B - b0);
        __syncthreads();
        for (int i = threadIdx.x; i < nb * d; i += blockDim.x) {
            const int bb = i / d, e = i % d;
            qsh[bb][e] = q[((size_t)(b0 + bb) * H + j) * d + e];
        }
        __syncthreads();
        float2 acc[AB_BCH];
#pragma unroll
        for (int bb = 0; bb < AB_BCH; ++bb) acc[bb] = make_float2(0.f, 0.f);
        for (int e = eg; e < d; e += 8) {
            const __nv_bfloat162 wv =
                *reinterpret_cast<const __nv_bfloat162*>(W + ((size_t)j * d + e) * dc + c0 + 2 * cp);
            const float w0 = __low2float(wv), w1 = __high2float(wv);
#pragma unroll
            for (int bb = 0; bb < AB_BCH; ++bb) {
                if (bb < nb) {
                    const float qv = __bfloat162float(qsh[bb][e]);
                    acc[bb].x = fmaf(qv, w0, acc[bb].x);
                    acc[bb].y = fmaf(qv, w1, acc[bb].y);
                }
            }
        }
#pragma unroll
        for (int bb = 0; bb < AB_BCH; ++bb) red[eg][bb][cp] = acc[bb];
        __syncthreads();
        for (int i = threadIdx.x; i < nb * 32; i += blockDim.x) {
            const int bb = i / 32, p = i % 32;
            float2 s = red[0][bb][p];
#pragma unroll
            for (int g = 1; g < 8; ++g) {
                s.x += red[g][bb][p].x;
                s.y += red[g][bb][p].y;
            }
            *reinterpret_cast<__nv_bfloat162*>(qt + ((size_t)(b0 + bb) * H + j) * dc + c0 + 2 * p) =
                __floats2bfloat162_rn(s.x, s.y);
        }
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

}  // namespace

li_status launch_quantize_query(const void* q, const float* w, int rows, int heads, int dim, uint8_t* q8, float* sq,
                                float* w_eff, cudaStream_t st) {
    const long long nh = (long long)rows * heads;
    if (nh == 0) return LI_OK;
    const long long warps = dim == 128 ? (nh + 3) / 4 : nh;
    const long long blocks = (warps * 32 + 255) / 256;
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

li_status launch_absorb(const void* q, const void* wdec, void* qt, int B, int H, int d, int dc, cudaStream_t st) {
    if (B == 0) return LI_OK;
    absorb_kernel<<<dim3(H, dc / 64), 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(q),
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
