// prep.cuh -- per-call preparation of the layer's weights, run beside the
// routing: the butterfly angles become {cos, sin} tables in the order the
// kernels consume them, and the 2-bit packed base becomes the tensor-core
// operand layout.
//
// The prep kernel is launched with a programmatic dependency on the
// cooperative routing kernel, which lets it start at once: it uses the SM
// resources the routing leaves free, and ends by waiting for the routing to
// complete, so that the kernels after it see both results.
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
};

// {cos, sin} tables of every expert in consumption order: theta -> the
// input engine's B^T table (engine_entry order, sign of B^T folded in), phi
// -> the output table (out_table_entry order).  Threads walk the tables in
// position order, so each table line is written whole by one warp, and
// gather their angles (the kernels that read the tables right after run
// faster from lines that were not assembled from many SMs' partial writes).
__global__ void __launch_bounds__(256) k_prep(PrepParams p)
{
    const int d = p.d, L = p.L, half = d >> 1;
    const int tab = L * half;
    const int gtid = blockIdx.x * blockDim.x + threadIdx.x;
    const int gthreads = gridDim.x * blockDim.x;
    const int total = 2 * p.ncoef;
    for (int i0 = gtid; i0 < total; i0 += 4 * gthreads) {
        float a[4];
        int dst[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * gthreads;
            dst[u] = -1;
            a[u] = 0.0f;
            if (i < total) {
                const bool out = i >= p.ncoef;
                const int j = out ? i - p.ncoef : i;
                const int e = j / tab, r = j - e * tab;
                int st, pp;
                if (out)
                    out_table_entry(d, L, r, st, pp);
                else
                    engine_entry(d, L, true, r, st, pp);
                a[u] = __ldg((out ? p.phi : p.theta) + (size_t)e * tab + st * half + pp);
                dst[u] = i;
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (dst[u] < 0) continue;
            float sn, cs;
            __sincosf(a[u], &sn, &cs);
            if (dst[u] >= p.ncoef)
                p.coef_p[dst[u] - p.ncoef] = make_float2(cs, sn);
            else
                p.coef_t[dst[u]] = make_float2(cs, -sn);
        }
    }
    if (gtid == 0 && (p.packed[0] != kPackMagic || p.packed[1] != (uint32_t)d)) set_status(p.status, BFMOE_ERR_INVALID_ARG);
    const int nq = d * d / 8;
    for (int q = gtid; q < nq; q += gthreads) decode_chunk(p.packed, d, p.wdec, q);
    pdl_wait();  // complete only after the routing has
}

}  // namespace bfmoe
