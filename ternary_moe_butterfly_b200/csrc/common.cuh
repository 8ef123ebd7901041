// common.cuh -- shared device helpers for the sm_100a kernels: status word,
// bounded mbarrier waits, bulk copies and the tcgen05 (5th-generation tensor
// core / tensor memory) instructions, written as inline PTX.
#pragma once

#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/bfmoe.h"

namespace bfmoe {

// Every bounded device-side wait gives up after this many nanoseconds of
// %globaltimer, records BFMOE_ERR_TIMEOUT in the status word and unwinds.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

// Record the first device-side error; later errors do not overwrite it.
__device__ __forceinline__ void set_status(uint32_t *status, uint32_t code)
{
    if (status) atomicCAS(status, 0u, code);
}

__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------- phase trace --
// Built with -DBFMOE_TRACE_PHASES, kernels record %globaltimer at phase
// boundaries: g_bfmoe_trace[kernel][block][slot] (read back with
// bfmoe_trace_read).  Without the flag the macro compiles to nothing.
#ifdef BFMOE_TRACE_PHASES
constexpr int kTraceKernels = 5, kTraceBlocks = 1024, kTraceSlots = 16;
__device__ unsigned long long g_bfmoe_trace[kTraceKernels][kTraceBlocks][kTraceSlots];
#define BFMOE_TRACE(kernel, cond, slot)                                                     \
    do {                                                                                    \
        if ((cond) && blockIdx.x < kTraceBlocks)                                            \
            ::bfmoe::g_bfmoe_trace[(kernel)][blockIdx.x][(slot)] = ::bfmoe::globaltimer_ns(); \
    } while (0)
#else
#define BFMOE_TRACE(kernel, cond, slot) \
    do {                                \
    } while (0)
#endif

// ------------------------------------------------------------- mbarrier --

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar_addr), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase of `bar` with the given parity has completed, for at
// most kWaitLimitNs.  Returns false on timeout (the caller unwinds).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_addr(bar);
    if (mbar_try_wait(a, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(a, parity)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// ------------------------------------------------------------ bulk copy --

// 1-D bulk copy global -> shared, completing `bytes` of transaction count on
// `bar`.  Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// -------------------------------------------------------------- tcgen05 --

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor (tcgen05), no swizzle, K-major canonical
// layout: 8-row x 16-byte core matrices; `lbo` = byte stride between core
// matrices along K, `sbo` = byte stride between 8-row groups along M/N.
__device__ __forceinline__ uint64_t sdesc_noswizzle(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;  // descriptor version for sm_100
    return d;                 // base offset 0, layout type 0 (no swizzle)
}

// Instruction descriptor, kind::f16: A = B = fp16, D = fp32, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N)
{
    return (1u << 4)                              // D format fp32
           | (0u << 7) | (0u << 10)               // A, B fp16
           | ((uint32_t)(N >> 3) << 17)           // N / 8
           | ((uint32_t)(M >> 4) << 24);          // M / 16
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// columns [col, col+32) of TMEM lane (warp's lane base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Issue a 32-column TMEM load without waiting; the registers are valid only
// after tmem_ld_wait_regs on the same array.
__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Wait for every TMEM load of this thread; the array is an in/out operand so
// that no use of its values can be scheduled before the wait.
template <int NV>
__device__ __forceinline__ void tmem_ld_wait_regs(float (&v)[NV])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < NV; ++i) asm volatile("" : "+f"(v[i]));
}

// 32 lanes x 32 consecutive 32-bit columns, registers -> TMEM.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 4 consecutive 32-bit columns (no wait; call tmem_ld_wait()).
__device__ __forceinline__ void tmem_ld4_nowait(uint32_t taddr, float &a, float &b, float &c, float &d)
{
    uint32_t r0, r1, r2, r3;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(taddr));
    a = __uint_as_float(r0);
    b = __uint_as_float(r1);
    c = __uint_as_float(r2);
    d = __uint_as_float(r3);
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------ fp32 pairs --
// sm_100 two-lane fp32 arithmetic (.x and .y independently, round to
// nearest): one instruction does the work of two.
__device__ __forceinline__ unsigned long long f2_bits(float2 v)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
    return r;
}
__device__ __forceinline__ float2 f2_val(unsigned long long r)
{
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b)
{
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return f2_val(r);
}
__device__ __forceinline__ float2 f2_sub(float2 a, float2 b)
{
    unsigned long long r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)));
    return f2_val(r);
}
__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c)
{
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(f2_bits(a)), "l"(f2_bits(b)), "l"(f2_bits(c)));
    return f2_val(r);
}

// Cos/sin tables store their rotations in consumption order, each aligned
// pair of rotations (2q, 2q+1) as the four floats
// (cos_2q, cos_2q+1, sin_2q, sin_2q+1), so that one 16-byte load gives two
// rotations in the lane layout of the pair arithmetic.  A table of n
// rotations (n even) takes n float2 slots.
//
// Two Givens rotations at once, lane-wise: (a, b) <- (c a - s b, s a + c b).
__device__ __forceinline__ void rot2(float2 &a, float2 &b, float2 c, float2 s)
{
    const float2 sa = f2_mul(s, a);
    const float2 na = f2_sub(f2_mul(c, a), f2_mul(s, b));
    b = f2_fma(c, b, sa);
    a = na;
}
// One rotation: (a, b) <- (c a - s b, s a + c b).
__device__ __forceinline__ void rot1(float &a, float &b, float c, float s)
{
    const float x = a, y = b;
    a = fmaf(c, x, -(s * y));
    b = fmaf(s, x, c * y);
}

// ------------------------------------------------ explicit shared memory --
// Typed accesses through 32-bit shared-window addresses, so that the loads and
// stores are shared-memory instructions whatever the compiler can prove
// about a pointer's origin.
__device__ __forceinline__ float lds_f32(uint32_t a)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) { asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory"); }
__device__ __forceinline__ float2 lds_f32x2(uint32_t a)
{
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ float4 lds_f32x4(uint32_t a)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}

// A cos/sin table that lives in shared memory (address) or global memory.
// ld4(i), i even: rotations i, i+1 as (cos_i, cos_i+1, sin_i, sin_i+1);
// cs(i): rotation i alone as (cos, sin).
struct SmemTab {
    uint32_t base;  // shared-window byte address of slot 0
    __device__ __forceinline__ float4 ld4(int i) const { return lds_f32x4(base + 8u * (uint32_t)i); }
    __device__ __forceinline__ float2 cs(int i) const
    {
        const uint32_t a = base + 8u * (uint32_t)(i & ~1) + 4u * (uint32_t)(i & 1);
        return make_float2(lds_f32(a), lds_f32(a + 8u));
    }
    __device__ __forceinline__ SmemTab operator+(int i) const { return SmemTab{base + 8u * (uint32_t)i}; }
};
struct GmemTab {
    const float2 *p;
    __device__ __forceinline__ float4 ld4(int i) const { return __ldg(reinterpret_cast<const float4 *>(p + i)); }
    __device__ __forceinline__ float2 cs(int i) const
    {
        const float *f = reinterpret_cast<const float *>(p + (i & ~1)) + (i & 1);
        return make_float2(__ldg(f), __ldg(f + 2));
    }
    __device__ __forceinline__ GmemTab operator+(int i) const { return GmemTab{p + i}; }
};

// Copy n elements global -> shared by the threads tid = 0..nthr-1: each
// thread issues a batch of 8 loads into registers before storing any of
// them, so the loads overlap (a copy loop that interleaves loads and stores
// through possibly aliasing pointers would wait out every load).
template <typename T>
__device__ __forceinline__ void copy_g2s(const T *__restrict__ src, T *dst, int n, int tid, int nthr)
{
    for (int q0 = tid; q0 < n; q0 += 8 * nthr) {
        T v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * nthr;
            if (q < n) v[u] = __ldcg(src + q);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * nthr;
            if (q < n) dst[q] = v[u];
        }
    }
}

// ------------------------------------------------ programmatic dependent launch --

// Wait until the grids this grid depends on have completed and their memory
// is visible (no-op when launched without a programmatic dependency).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Allow the dependent grid to start launching (its CTAs still wait in pdl_wait).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------- numerics --

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

// Unpack 8 bf16 held in a uint4 into fp32.
__device__ __forceinline__ void unpack_bf16x8(const uint4 &u, float *f)
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float *f)
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 pack_f16x8(const float *f)
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace bfmoe
