// butterfly.cuh -- butterfly rotations on a shared-memory tile of rows.
//
// A butterfly B(a) is a product of L = log2 d layers of Givens rotations
// (ButterflyMoE summaries, section 2 / 2.2; ButterflyViT summary, section 2:
// block-diagonal Givens factors).  Convention: stage s rotates the pairs
// (j, j + 2^s) with bit s of j clear, pair index
// p = (j >> (s+1)) * 2^s + (j & (2^s - 1)),
//     y_j = c x_j - s x_{j+2^s},   y_{j+2^s} = s x_j + c x_{j+2^s};
// B applies stages 0..L-1, B^T applies L-1..0 with negated angles.
//
// Engine: the tile holds `rows` rows of d fp32 values, row stride d+1 floats
// (the +1 makes same-column accesses of consecutive rows hit distinct
// banks).  The L stages are split into passes of at most 5 stages; in a pass
// a thread loads the 2^g values of one row that the pass's g stages mix (a
// "subset": indices that differ only in bits s0..s1-1), rotates them in
// registers, and stores them back.  Threads are laid out rows-fastest, so a
// warp works on up to 32 rows of the same subset and its cos/sin loads are
// broadcasts whenever those rows share an expert.
#pragma once

#include "common.cuh"

namespace bfmoe {

// cos/sin table: float2 {cos a, sin a} per angle, [N][L][d/2].
template <int G, bool TRANSPOSE>
__device__ __forceinline__ void bfly_subset(float *row, int base, int s0, const float2 *__restrict__ cf, int half)
{
    constexpr int M = 1 << G;
    float v[M];
#pragma unroll
    for (int m = 0; m < M; ++m) v[m] = row[base + (m << s0)];
#pragma unroll
    for (int q = 0; q < G; ++q) {
        const int ls = TRANSPOSE ? (G - 1 - q) : q;  // local stage
        const int s = s0 + ls;
        const int h = 1 << s;
        const float2 *cs = cf + (size_t)s * half;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            if (m & (1 << ls)) continue;
            const int j = base + (m << s0);
            const int p = ((j >> (s + 1)) << s) | (j & (h - 1));
            const float2 c = cs[p];
            const float sn = TRANSPOSE ? -c.y : c.y;
            const float a = v[m], b = v[m + (1 << ls)];
            v[m] = fmaf(c.x, a, -(sn * b));
            v[m + (1 << ls)] = fmaf(sn, a, c.x * b);
        }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) row[base + (m << s0)] = v[m];
}

// Row r uses the table  coef + sexp[r] * estride  (sexp == nullptr: every
// row uses `coef`, e.g. one expert's table staged in shared memory).
template <int G, bool TRANSPOSE>
__device__ void bfly_pass(float *tile, int ld, int rows, int d, int s0, const int *sexp,
                          const float2 *__restrict__ coef, size_t estride, int nthreads)
{
    const int half = d >> 1;
    const int nsub = d >> G;
    const int s1 = s0 + G;
    const int items = rows * nsub;
    for (int it = threadIdx.x; it < items; it += nthreads) {
        const int r = it % rows;
        const int sub = it / rows;
        const int base = ((sub >> s0) << s1) | (sub & ((1 << s0) - 1));
        const float2 *cf = sexp ? coef + (size_t)sexp[r] * estride : coef;
        bfly_subset<G, TRANSPOSE>(tile + (size_t)r * ld, base, s0, cf, half);
    }
}

template <bool TRANSPOSE>
__device__ __forceinline__ void bfly_pass_g(int g, float *tile, int ld, int rows, int d, int s0, const int *sexp,
                                            const float2 *coef, size_t estride, int nthreads)
{
    switch (g) {
    case 1: bfly_pass<1, TRANSPOSE>(tile, ld, rows, d, s0, sexp, coef, estride, nthreads); break;
    case 2: bfly_pass<2, TRANSPOSE>(tile, ld, rows, d, s0, sexp, coef, estride, nthreads); break;
    case 3: bfly_pass<3, TRANSPOSE>(tile, ld, rows, d, s0, sexp, coef, estride, nthreads); break;
    case 4: bfly_pass<4, TRANSPOSE>(tile, ld, rows, d, s0, sexp, coef, estride, nthreads); break;
    default: bfly_pass<5, TRANSPOSE>(tile, ld, rows, d, s0, sexp, coef, estride, nthreads); break;
    }
}

// Apply B (transpose == false) or B^T (transpose == true) to every row r <
// rows of the tile; row r uses the table of expert sexp[r] (tables of
// L*d/2 entries, back to back) or, with sexp == nullptr, the single table
// `coef`.  Must be called by all threads of the block (has __syncthreads).
__device__ void bfly_tile(float *tile, int ld, int rows, int d, int L, const int *sexp, const float2 *coef,
                          bool transpose)
{
    const size_t estride = (size_t)L * (d >> 1);
    const int npass = (L + 4) / 5;
    for (int q = 0; q < npass; ++q) {
        const int pi = transpose ? (npass - 1 - q) : q;
        const int s0 = pi * L / npass;
        const int s1 = (pi + 1) * L / npass;
        if (transpose)
            bfly_pass_g<true>(s1 - s0, tile, ld, rows, d, s0, sexp, coef, estride, blockDim.x);
        else
            bfly_pass_g<false>(s1 - s0, tile, ld, rows, d, s0, sexp, coef, estride, blockDim.x);
        __syncthreads();
    }
}

// Rows per shared-memory tile: up to 32, at most 16384 floats of data.
__host__ __device__ constexpr int tile_rows_for(int d) { return (16384 / d) < 32 ? (16384 / d) : 32; }

}  // namespace bfmoe
