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

// Pair index of the pair (j, j + 2^s) in stage s: j with bit s deleted.
__host__ __device__ constexpr int pair_of(int j, int s) { return ((j >> (s + 1)) << s) | (j & ((1 << s) - 1)); }

// One "subset" of a row: the 2^G values whose indices differ only in bits
// S0..S0+G-1, index base | (m << S0).  Deleting bit s is additive over the
// disjoint bit sets of base and m << S0, so a rotation's table entry is
// pair_of(base, s) + pair_of(m << S0, s): one runtime term per stage and a
// compile-time offset per rotation.  cos/sin table: float2 {cos a, sin a},
// [L][d/2] for one expert.
template <int G, int S0, bool TRANSPOSE>
__device__ __forceinline__ void bfly_subset(float *row, int base, const float2 *__restrict__ cf, int half)
{
    constexpr int M = 1 << G;
    float v[M];
#pragma unroll
    for (int m = 0; m < M; ++m) v[m] = row[base + (m << S0)];
#pragma unroll
    for (int q = 0; q < G; ++q) {
        const int ls = TRANSPOSE ? (G - 1 - q) : q;  // local stage
        const int s = S0 + ls;
        const float2 *cs = cf + (size_t)s * half + pair_of(base, s);
#pragma unroll
        for (int m = 0; m < M; ++m) {
            if (m & (1 << ls)) continue;
            const float2 c = cs[pair_of(m << S0, s)];
            const float sn = TRANSPOSE ? -c.y : c.y;
            const float a = v[m], b = v[m + (1 << ls)];
            v[m] = fmaf(c.x, a, -(sn * b));
            v[m + (1 << ls)] = fmaf(sn, a, c.x * b);
        }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) row[base + (m << S0)] = v[m];
}

// Row r uses the table  coef + sexp[r] * estride  (sexp == nullptr: every
// row uses `coef`, e.g. one expert's table staged in shared memory).
template <int G, int S0, bool TRANSPOSE>
__device__ void bfly_pass(float *tile, int ld, int rows, int d, const int *sexp, const float2 *__restrict__ coef,
                          size_t estride, int nthreads)
{
    const int half = d >> 1;
    const int nsub = d >> G;
    constexpr int S1 = S0 + G;
    const int items = rows * nsub;
    for (int it = threadIdx.x; it < items; it += nthreads) {
        const int r = it % rows;
        const int sub = it / rows;
        const int base = ((sub >> S0) << S1) | (sub & ((1 << S0) - 1));
        const float2 *cf = sexp ? coef + (size_t)sexp[r] * estride : coef;
        bfly_subset<G, S0, TRANSPOSE>(tile + (size_t)r * ld, base, cf, half);
    }
}

// Stage split of a butterfly of L stages into passes of at most 5 stages:
// pass q covers stages [q*L/np, (q+1)*L/np), np = ceil(L/5).
template <bool TRANSPOSE>
__device__ __forceinline__ void bfly_pass_dispatch(int L, int pass, float *tile, int ld, int rows, int d,
                                                   const int *sexp, const float2 *coef, size_t estride)
{
    const int nt = blockDim.x;
#define BFLY_CASE(LL, PP, GG, SS)                                                                     \
    if (L == LL && pass == PP) {                                                                      \
        bfly_pass<GG, SS, TRANSPOSE>(tile, ld, rows, d, sexp, coef, estride, nt);                     \
        return;                                                                                       \
    }
    BFLY_CASE(6, 0, 3, 0) BFLY_CASE(6, 1, 3, 3)
    BFLY_CASE(7, 0, 3, 0) BFLY_CASE(7, 1, 4, 3)
    BFLY_CASE(8, 0, 4, 0) BFLY_CASE(8, 1, 4, 4)
    BFLY_CASE(9, 0, 4, 0) BFLY_CASE(9, 1, 5, 4)
    BFLY_CASE(10, 0, 5, 0) BFLY_CASE(10, 1, 5, 5)
    BFLY_CASE(11, 0, 3, 0) BFLY_CASE(11, 1, 4, 3) BFLY_CASE(11, 2, 4, 7)
    BFLY_CASE(12, 0, 4, 0) BFLY_CASE(12, 1, 4, 4) BFLY_CASE(12, 2, 4, 8)
#undef BFLY_CASE
}

// Apply B (transpose == false) or B^T (transpose == true) to every row r <
// rows of the tile; row r uses the table of expert sexp[r] (tables of
// L*d/2 entries, back to back) or, with sexp == nullptr, the single table
// `coef`.  6 <= L <= 12.  Must be called by all threads of the block (has
// __syncthreads).
__device__ void bfly_tile(float *tile, int ld, int rows, int d, int L, const int *sexp, const float2 *coef,
                          bool transpose)
{
    const size_t estride = (size_t)L * (d >> 1);
    const int npass = (L + 4) / 5;
    for (int q = 0; q < npass; ++q) {
        const int pi = transpose ? (npass - 1 - q) : q;
        if (transpose)
            bfly_pass_dispatch<true>(L, pi, tile, ld, rows, d, sexp, coef, estride);
        else
            bfly_pass_dispatch<false>(L, pi, tile, ld, rows, d, sexp, coef, estride);
        __syncthreads();
    }
}

// Rows per shared-memory tile: up to 32, at most 16384 floats of data.
__host__ __device__ constexpr int tile_rows_for(int d) { return (16384 / d) < 32 ? (16384 / d) : 32; }

}  // namespace bfmoe
