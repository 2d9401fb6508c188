// Device-side building blocks shared by the li kernels (sm_100a only):
// mbarrier pipelines with bounded waits, TMA tile loads, tcgen05 (5th-gen
// tensor core) MMA issue, TMEM allocation and loads, shared-memory matrix
// descriptors, and the device error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "li.h"

namespace li {

// ---------------------------------------------------------------------------
// Error reporting: kernels never trap.  A bounded wait that runs out or an
// out-of-range index sets a bit in a per-device word; the host reads it with
// li_get_last_error().
// ---------------------------------------------------------------------------
enum : unsigned { ERRBIT_TIMEOUT = 1u, ERRBIT_BOUNDS = 2u };

struct DevErr {
    unsigned* word;                 // device address of the error word
    unsigned long long limit_ns;    // wait budget for every bounded wait of the launch
};

// Host side (li_abi.cu): per-device error word and the default wait budget.
DevErr host_dev_err();
li_status host_check_launch();      // maps cudaGetLastError() to li_status
int host_num_sms();

constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull; // 2 s

// Launch with programmatic stream serialisation (and an optional cluster shape).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (cluster_x > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = cluster_x;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

#if defined(__CUDACC__)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_error(const DevErr& e, unsigned bit) {
    atomicOr(e.word, bit);
}

// ---------------------------------------------------------------------------
// mbarrier (shared::cta)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed.  Gives up after
// e.limit_ns of wall time, records ERRBIT_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const DevErr& e) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0u && globaltimer_ns() - t0 > e.limit_ns) {
            record_error(e, ERRBIT_TIMEOUT);
            return false;
        }
    }
}

// Programmatic dependent launch.  A kernel launched with the programmatic
// stream-serialisation attribute may start while the previous kernel of the
// stream is still running; pdl_wait() blocks the calling thread until that
// kernel has completed and its memory is visible (a no-op without the
// attribute).  pdl_trigger() lets the next kernel of the stream be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Make generic-proxy writes to shared memory visible to the async proxy
// (TMA, tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 2-D tiled load global -> this CTA's shared memory; completion is signalled
// as transaction bytes on `bar`.  x is the innermost (contiguous) coordinate.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Contiguous global -> shared copy by the TMA engine, completing on `bar`.
// dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA issue, completion, loads
// ---------------------------------------------------------------------------
// Executed by one full warp.  Writes the TMEM base address to *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive (once) on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, both operands K-major.
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor (32 bit): D format F32 at bits [4,6), A/B formats at
// [7,10) and [10,13) (e4m3 = 0 for kind::f8f6f4, bf16 = 1 for kind::f16),
// both operands K-major (bits 15, 16 clear), N/8 at [17,23), M/16 at [24,29).
__host__ __device__ constexpr uint32_t idesc_f32acc(int M, int N, uint32_t ab_format) {
    return (1u << 4) | (ab_format << 7) | (ab_format << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}
constexpr uint32_t kFmtE4M3 = 0u;
constexpr uint32_t kFmtBF16 = 1u;

// Shared-memory matrix descriptor for a K-major operand stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row (1024-byte) swizzle atoms placed
// 1024 bytes apart (stride byte offset), leading byte offset unused (1),
// descriptor version 1, layout type SWIZZLE_128B (2) in bits [61,64).  The
// start address may be advanced by the byte offset of a K slice inside the
// 128-byte row.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= uint64_t((smem_addr >> 4) & 0x3FFFu);
    d |= uint64_t(1u) << 16;
    d |= uint64_t(1024u >> 4) << 32;
    d |= uint64_t(1u) << 46;
    d |= uint64_t(2u) << 61;
    return d;
}

// The same for a K-major operand stored with the 64-byte swizzle: rows of 64
// bytes, 8-row (512-byte) swizzle atoms 512 bytes apart, layout type
// SWIZZLE_64B (4).
__device__ __forceinline__ uint64_t sw64_kmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= uint64_t((smem_addr >> 4) & 0x3FFFu);
    d |= uint64_t(1u) << 16;
    d |= uint64_t(512u >> 4) << 32;
    d |= uint64_t(1u) << 46;
    d |= uint64_t(4u) << 61;
    return d;
}

// Byte offset of 16-byte chunk `chunk` (0..3) of row `row` inside a
// 64-byte-swizzled tile whose base is 512-byte aligned: the chunk index is
// XORed with address bits 7-8, i.e. (row / 2) mod 4.
__device__ __forceinline__ uint32_t sw64_offset(uint32_t row, uint32_t chunk) {
    return row * 64u + (((chunk ^ (row >> 1)) & 3u) << 4);
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a
// 128-byte-swizzled tile whose base is 1024-byte aligned.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
    return row * 128u + (((chunk ^ (row & 7u)) & 7u) << 4);
}

// 32 lanes x 32 columns of 32-bit TMEM cells: thread t of the warp receives
// lane (taddr.lane + t), columns taddr.col .. +31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Weighted ReLU reduction over 32 head values: sum_j wj * max(v_j, 0).
__device__ __forceinline__ float relu_dot32(const uint32_t (&v)[32], const float* __restrict__ wsm) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(wsm + j);
        a0 = fmaf(w4.x, fmaxf(__uint_as_float(v[j + 0]), 0.f), a0);
        a1 = fmaf(w4.y, fmaxf(__uint_as_float(v[j + 1]), 0.f), a1);
        a2 = fmaf(w4.z, fmaxf(__uint_as_float(v[j + 2]), 0.f), a2);
        a3 = fmaf(w4.w, fmaxf(__uint_as_float(v[j + 3]), 0.f), a3);
    }
    return (a0 + a1) + (a2 + a3);
}

// Order-preserving uint32 image of an fp32 score for the top-k: larger score,
// larger key; NaN maps to 0 (below -inf), -0.0 to the key of +0.0.
__device__ __forceinline__ uint32_t order_key(float f) {
    if (f != f) return 0u;
    uint32_t u = __float_as_uint(f);
    if (f == 0.f) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The decode scorer counts the top LI_HIST_BITS bits of every score's key
// into a per-row histogram that the top-k then uses as its first radix digit.
constexpr int LI_HIST_BITS = 11;
constexpr int LI_HIST_BINS = 1 << LI_HIST_BITS;
constexpr int LI_HIST_SHIFT = 32 - LI_HIST_BITS;

// Adds each valid lane's score to the global first-digit histogram gh with one
// atomic per distinct digit in the warp (lanes are grouped by digit).  Every
// lane of the warp must make the call together.
__device__ __forceinline__ void warp_hist_add(uint32_t* gh, float v, bool valid) {
    const uint32_t bin = valid ? (order_key(v) >> LI_HIST_SHIFT) : 0xffffffffu;
    const uint32_t peers = __match_any_sync(0xffffffffu, bin);
    if (valid && (int)(threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(gh + bin, (uint32_t)__popc(peers));
}

// acc.{x,y} += a.{0,1} * b.{0,1} with one packed fp32x2 FMA (same rounding as two fmaf).
__device__ __forceinline__ void ffma2(float2& acc, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(acc.x), "+f"(acc.y)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Weighted ReLU reduction over 32 head values with packed FMAs:
// sum_j wj * max(v_j, 0), 1.5 instructions per value (FMNMX + half an FFMA2).
__device__ __forceinline__ float relu_dot32_x2(const uint32_t (&v)[32], const float* __restrict__ wsm) {
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(wsm + j);
        ffma2(a0, fmaxf(__uint_as_float(v[j + 0]), 0.f), fmaxf(__uint_as_float(v[j + 1]), 0.f), w4.x, w4.y);
        ffma2(a1, fmaxf(__uint_as_float(v[j + 2]), 0.f), fmaxf(__uint_as_float(v[j + 3]), 0.f), w4.z, w4.w);
    }
    return (a0.x + a0.y) + (a1.x + a1.y);
}

// y[i] = x[i] / sq rounded as IEEE fp32 division rounds it (nearest even), for
// the e4m3 conversion that follows, without a division in the common case.
// Method: Markstein's FMA correction of an approximate quotient (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000 processor",
// IBM J. Res. Dev. 34(1), 1990; Muller et al., Handbook of Floating-Point
// Arithmetic, the FMA-based division chapter).  With r the correctly rounded
// reciprocal of sq:
//   y0 = RN(x r)                      within about 2.5 ulp of x / sq
//   y1 = RN(y0 + RN(x - y0 sq) r)     faithful (within 1 ulp)
//   y  = RN(y1 + RN(x - y1 sq) r)     correctly rounded: the residual of a
//                                     faithful quotient is exact with an FMA,
//                                     and r is within half an ulp of 1/sq.
// The residuals stay clear of underflow while sq >= 2^-90 and |x / sq| >= 2^-11;
// smaller quotients can be off by an ulp, but every value below 2^-10 converts
// to an e4m3 zero of the same sign either way.  A zero x keeps its sign (the
// FMA steps would turn -0 into +0).  Scales outside [2^-90, 2^127] (tiny, or
// inf / NaN from a non-finite head) make the whole warp divide instead.
// (Before this, a product x r was taken and the warp divided whenever one of
// its quotients fell within 8 ulp of an e4m3 rounding midpoint; bf16 inputs hit
// exact midpoints so often that most warps divided.)
// All 32 lanes must call this together.
template <int N>
__device__ __forceinline__ void quotients_for_e4m3(const float (&x)[N], float sq, float r, float (&y)[N]) {
    const bool sq_ok = sq >= 0x1p-90f && sq <= 0x1p127f;
    if (__all_sync(0xffffffffu, sq_ok)) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const float y0 = __fmul_rn(x[i], r);
            const float y1 = __fmaf_rn(__fmaf_rn(-y0, sq, x[i]), r, y0);
            const float y2 = __fmaf_rn(__fmaf_rn(-y1, sq, x[i]), r, y1);
            y[i] = __uint_as_float((__float_as_uint(y2) & 0x7fffffffu) | (__float_as_uint(x[i]) & 0x80000000u));
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) y[i] = __fdiv_rn(x[i], sq);
    }
}

// Two fp32 values to e4m3 (nearest even, saturating to +-448): lo in the low byte, hi in the high byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return d;
}

// One element (all 32 lanes call together).
__device__ __forceinline__ uint32_t e4m3_quotient(float x, float sq, float r) {
    const float xs[1] = {x};
    float y[1];
    quotients_for_e4m3<1>(xs, sq, r, y);
    return e4m3x2(y[0], 0.f) & 0xffu;
}

// Per-(row, head) e4m3 quantisation of one 128-element bf16 head vector held
// as 4 consecutive elements per lane of a warp.  Returns the packed 4 bytes
// of this lane and writes the head scale to *sq (all lanes).
__device__ __forceinline__ uint32_t quantize_head128(uint2 raw, float* sq_out) {
    __nv_bfloat162 p0 = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
    __nv_bfloat162 p1 = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
    float x0 = __low2float(p0), x1 = __high2float(p0), x2 = __low2float(p1), x3 = __high2float(p1);
    float m = fmaxf(fmaxf(fabsf(x0), fabsf(x1)), fmaxf(fabsf(x2), fabsf(x3)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float sq = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
    *sq_out = sq;
    const float r = __frcp_rn(sq);
    const float xs[4] = {x0, x1, x2, x3};
    float y[4];
    quotients_for_e4m3<4>(xs, sq, r, y);
    return e4m3x2(y[0], y[1]) | (e4m3x2(y[2], y[3]) << 16);
}

// Same quantisation with 8 lanes per head: the lane holds 16 consecutive bf16
// elements (16*l8 .. 16*l8+15 of the head, `lo` then `hi`) and returns their 16
// e4m3 bytes; *sq_out receives the head scale.  All 32 lanes of the warp must
// call it (the absmax reduction shuffles within aligned groups of 8 lanes).
__device__ __forceinline__ uint4 quantize_head128_g8(uint4 lo, uint4 hi, float* sq_out) {
    float x[16];
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(x[i]));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float sq = m > 0.f ? __fdiv_rn(m, 448.f) : 1.f;
    *sq_out = sq;
    const float r = __frcp_rn(sq);
    float y[16];
    quotients_for_e4m3<16>(x, sq, r, y);
    uint32_t b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) b[i] = e4m3x2(y[4 * i], y[4 * i + 1]) | (e4m3x2(y[4 * i + 2], y[4 * i + 3]) << 16);
    return make_uint4(b[0], b[1], b[2], b[3]);
}

#endif  // __CUDACC__

}  // namespace li
