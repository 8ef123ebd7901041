// prep.cuh -- per-call preparation of the layer's weights, the first
// kernel of a forward: the butterfly angles become {cos, sin} tables in the
// order the kernels consume them, and the 2-bit packed base becomes the
// tensor-core operand layout.
//
// It is launched with a programmatic dependency on the previous call's last
// kernel (the combine, which reads no table), so it runs while that kernel
// finishes: nothing it writes is read by the previous call's combine, and it
// waits for that call to complete only at its end, before it clears the
// status word.  The routing kernel depends on it in turn.
#pragma once

#include "butterfly.cuh"
#include "common.cuh"
#include "contract.cuh"
#include "route.cuh"

namespace bfmoe {

struct PrepParams {
    const float *theta, *phi;  // [N][L][d/2]
    float2 *coef_t;            // [N][L*d/2] input engine table (B^T order, see engine_entry)
    float2 *coef_p;            // [N][L*d/2] output table (see out_table_entry)
    int ncoef;                 // N * L * d/2
    int d, L;
    const uint32_t *packed;    // packed base (header + words)
    __half *wdec;              // decoded base, GEMM B-operand blocks
    uint32_t *status;
    const void *x;             // layer input, prefetched into L2 ([x_bytes], 16-byte multiple)
    size_t x_bytes;
    const void *logits;        // router logits, prefetched into L2 ([logit_bytes])
    size_t logit_bytes;
};

// Bring block `blk` of `nblk`'s share of [base, base + bytes) into L2 (one
// thread; shares rounded to 16 bytes, the prefetch unit; `bytes` a multiple
// of 16; nothing for a base that is not 16-byte aligned).
__device__ __forceinline__ void l2_prefetch_share(const void *base, size_t bytes, int blk, int nblk)
{
    const size_t share = ((bytes + nblk - 1) / nblk + 15) & ~size_t(15);
    const size_t lo = (size_t)blk * share;
    if (!base || (reinterpret_cast<uintptr_t>(base) & 15) || lo >= bytes) return;  // 16-byte rule
    const size_t n = bytes - lo < share ? bytes - lo : share;
    for (size_t o = 0; o < n; o += (1u << 20)) {
        const uint32_t c = (uint32_t)(n - o < (1u << 20) ? n - o : (1u << 20));
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<const char *>(base) + lo + o),
                     "r"(c)
                     : "memory");
    }
}

// {cos, sin} tables of every expert in consumption order: theta -> the
// input engine's B^T table (engine_entry order, sign of B^T folded in), phi
// -> the output table (out_table_entry order).  Threads walk the tables in
// position order, so each table line is written whole by one warp, and
// gather their angles (the kernels that read the tables right after run
// faster from lines that were not assembled from many SMs' partial writes).
// Instantiated per L = log2 d, so that the index decoding divides by
// compile-time constants.
template <int LL>
__global__ void __launch_bounds__(256) k_prep(PrepParams p)
{
    // the routing kernel may become resident now; it waits for this grid
    // to complete before it touches the workspace
    BFMOE_TRACE(4, threadIdx.x == 0, 0);
    pdl_trigger();
    if (threadIdx.x == 0) {
        // the routing reads the logits and the input kernel gathers x right
        // after this kernel: bring this block's shares into L2 now (a
        // prefetch reads nothing into the program, so it may run before the
        // wait for the previous kernel)
        l2_prefetch_share(p.logits, p.logit_bytes, blockIdx.x, gridDim.x);
        l2_prefetch_share(p.x, p.x_bytes, blockIdx.x, gridDim.x);
    }
    constexpr int L = LL, d = 1 << LL, half = d >> 1;
    constexpr int tab = L * half;
    const int gtid = blockIdx.x * blockDim.x + threadIdx.x;
    const int gthreads = gridDim.x * blockDim.x;
    // rotation pairs: the input table, then the output table's slice part
    // (its combine part is not written: the combine reads phi itself)
    constexpr int used = slice_stages(gemm_bn(d)) * half;  // output rotations per expert
    const int nexp = p.ncoef / tab;
    const int npair_in = p.ncoef / 2, npair = npair_in + nexp * (used / 2);
    for (int j0 = gtid; j0 < npair; j0 += 2 * gthreads) {
        float a[2][2];
        int dst[2];
        bool outt[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = j0 + u * gthreads;
            dst[u] = -1;
            outt[u] = false;
            a[u][0] = a[u][1] = 0.0f;
            if (j < npair) {
                const bool out = j >= npair_in;
                const int jj = out ? j - npair_in : j;
                const int per = out ? used : tab;
                const int e = (2 * jj) / per, r = (2 * jj) % per;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    int st, pp;
                    if (out)
                        out_table_entry(d, L, r + h, st, pp);
                    else
                        engine_entry(d, L, true, r + h, st, pp);
                    a[u][h] = __ldg((out ? p.phi : p.theta) + (size_t)e * tab + st * half + pp);
                }
                dst[u] = (e * tab + r) / 2;  // float4 index of the pair
                outt[u] = out;
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (dst[u] < 0) continue;
            float s0, c0, s1, c1;
            __sincosf(a[u][0], &s0, &c0);
            __sincosf(a[u][1], &s1, &c1);
            if (outt[u])
                reinterpret_cast<float4 *>(p.coef_p)[dst[u]] = make_float4(c0, c1, s0, s1);
            else
                reinterpret_cast<float4 *>(p.coef_t)[dst[u]] = make_float4(c0, c1, -s0, -s1);
        }
    }
    BFMOE_TRACE(4, threadIdx.x == 0, 1);
    const bool bad_header = gtid == 0 && (p.packed[0] != kPackMagic || p.packed[1] != (uint32_t)d);
    constexpr int nq = d * d / 8;
    for (int q = gtid; q < nq; q += gthreads) decode_chunk(p.packed, d, p.wdec, q);
    BFMOE_TRACE(4, threadIdx.x == 0, 2);
    // complete only after the previous call on this stream has (its last
    // kernels may still read the routing results this call overwrites);
    // then this call's status starts clear
    pdl_wait();
    if (gtid == 0) *reinterpret_cast<volatile uint32_t *>(p.status) = bad_header ? (uint32_t)BFMOE_ERR_INVALID_ARG : 0u;
    BFMOE_TRACE(4, threadIdx.x == 0, 3);
}

}  // namespace bfmoe
