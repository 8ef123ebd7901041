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
// warp works on up to 32 rows of the same subset; the cos/sin table is laid
// out in consumption order, so a warp reads it with 16-byte loads that are
// broadcasts whenever its rows share an expert.
#pragma once

#include "common.cuh"

namespace bfmoe {

// Pair index of the pair (j, j + 2^s) in stage s: j with bit s deleted.
__host__ __device__ constexpr int pair_of(int j, int s) { return ((j >> (s + 1)) << s) | (j & ((1 << s) - 1)); }

// The ri-th integer whose bit b is clear.
__host__ __device__ constexpr int insert_zero_bit(int ri, int b) { return ((ri >> b) << (b + 1)) | (ri & ((1 << b) - 1)); }

// Stage split of a butterfly of L stages (6 <= L <= 12) into passes of at
// most 5 stages: pass pi covers stages [pi*L/np, (pi+1)*L/np), np = ceil(L/5).
__host__ __device__ inline int npass_of(int L) { return (L + 4) / 5; }
__host__ __device__ inline void pass_bounds(int L, int pi, int &s0, int &g)
{
    const int np = npass_of(L);
    s0 = pi * L / np;
    g = (pi + 1) * L / np - s0;
}

// Engine tables hold each expert's {cos a, +-sin a} in the order the
// row engine consumes them: passes in execution order, then subsets, then
// stages in execution order, then the subset's rotations (m ascending among
// the indices whose local-stage bit is clear), stored in the paired layout
// (see rot2).  The sign of B^T is folded in.  engine_entry gives the (stage,
// pair) of rotation r of one expert's table.
__host__ __device__ inline void engine_entry(int d, int L, bool transpose, int r, int &s, int &p)
{
    const int np = npass_of(L), half = d >> 1;
    int q = 0, off = 0, s0 = 0, g = 1;
    for (; q < np; ++q) {
        pass_bounds(L, transpose ? np - 1 - q : q, s0, g);
        if (r < off + g * half) break;
        off += g * half;
    }
    const int w = r - off;
    const int per = g << (g - 1);  // entries per subset
    const int sub = w / per, rr = w % per;
    const int ql = rr >> (g - 1), ri = rr & ((1 << (g - 1)) - 1);
    const int ls = transpose ? g - 1 - ql : ql;
    const int base = ((sub >> s0) << (s0 + g)) | (sub & ((1 << s0) - 1));
    s = s0 + ls;
    p = pair_of(base | (insert_zero_bit(ri, ls) << s0), s);
}

// Delete bit b of x (the inverse of insert_zero_bit).
__host__ __device__ constexpr int delete_bit(int x, int b) { return ((x >> (b + 1)) << b) | (x & ((1 << b) - 1)); }

// Inverse of engine_entry: the table position of the (stage s, pair p) entry.
__host__ __device__ inline int engine_pos(int d, int L, bool transpose, int s, int p)
{
    const int np = npass_of(L), half = d >> 1;
    int poff = 0, s0 = 0, g = 1;
    for (int q = 0; q < np; ++q) {
        pass_bounds(L, transpose ? np - 1 - q : q, s0, g);
        if (s >= s0 && s < s0 + g) break;
        poff += g * half;
    }
    const int j = insert_zero_bit(p, s);                // lower element of the pair
    const int m = (j >> s0) & ((1 << g) - 1);           // position inside the subset
    const int sub = ((j >> (s0 + g)) << s0) | (j & ((1 << s0) - 1));
    const int ls = s - s0;
    const int ql = transpose ? g - 1 - ls : ls;
    return poff + sub * (g << (g - 1)) + (ql << (g - 1)) + delete_bit(m, ls);
}

// One "subset" of a row: the 2^G values whose indices differ only in bits
// S0..S0+G-1, index base | (m << S0).  `row` is the shared-window address of
// the row; `tab` the subset's G * 2^(G-1) table rotations.  Rotations ri and
// ri+1 (ri even) of a stage above the subset's lowest bit act on the
// adjacent pairs (m, m+1), (m+h, m+1+h): one pair instruction each.
template <int G, int S0, bool TRANSPOSE, typename Tab>
__device__ __forceinline__ void bfly_subset(uint32_t row, int base, Tab tab)
{
    constexpr int M = 1 << G;
    constexpr int H = M / 2;  // rotations per stage
    float v[M];
#pragma unroll
    for (int m = 0; m < M; ++m) v[m] = lds_f32(row + 4u * (uint32_t)(base + (m << S0)));
#pragma unroll
    for (int ql = 0; ql < G; ++ql) {
        const int ls = TRANSPOSE ? (G - 1 - ql) : ql;
        const int h = 1 << ls;
#pragma unroll
        for (int i = 0; i < H / 2; ++i) {
            const float4 w = tab.ld4(ql * H + 2 * i);
            const int m0 = insert_zero_bit(2 * i, ls), m1 = insert_zero_bit(2 * i + 1, ls);
            if (ls > 0) {
                float2 a = make_float2(v[m0], v[m1]), b = make_float2(v[m0 + h], v[m1 + h]);
                rot2(a, b, make_float2(w.x, w.y), make_float2(w.z, w.w));
                v[m0] = a.x;
                v[m1] = a.y;
                v[m0 + h] = b.x;
                v[m1 + h] = b.y;
            } else {
                rot1(v[m0], v[m0 + h], w.x, w.z);
                rot1(v[m1], v[m1 + h], w.y, w.w);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) sts_f32(row + 4u * (uint32_t)(base + (m << S0)), v[m]);
}

// One pass over the 2^lrows rows of the tile (shared address `tile`, row
// stride `ld` floats).  Row r uses the table  tab0 + sexp[r] * estride  (sexp
// == nullptr: every row uses tab0); `poff` is the pass's offset in a table.
// Consecutive threads take consecutive rows of one subset, so a warp's
// table loads are broadcasts when its rows share a table.
template <int G, int S0, bool TRANSPOSE, typename Tab>
__device__ __forceinline__ void bfly_pass(uint32_t tile, int ld, int lrows, int d, const int *sexp, Tab tab0,
                                          int estride, int poff, int nthreads)
{
    const int nsub = d >> G;
    constexpr int S1 = S0 + G;
    constexpr int PER = G << (G - 1);
    const int items = nsub << lrows;
    const int rmask = (1 << lrows) - 1;
    for (int it = threadIdx.x; it < items; it += nthreads) {
        const int r = it & rmask;
        const int sub = it >> lrows;
        const int base = ((sub >> S0) << S1) | (sub & ((1 << S0) - 1));
        const Tab tab = tab0 + ((sexp ? sexp[r] * estride : 0) + poff + sub * PER);
        bfly_subset<G, S0, TRANSPOSE>(tile + 4u * (uint32_t)(r * ld), base, tab);
    }
}

template <bool TRANSPOSE, typename Tab>
__device__ __forceinline__ void bfly_pass_dispatch(int L, int pass, uint32_t tile, int ld, int lrows, int d,
                                                   const int *sexp, Tab tab0, int estride, int poff)
{
    const int nt = blockDim.x;
#define BFLY_CASE(LL, PP, GG, SS)                                                                     \
    if (L == LL && pass == PP) {                                                                      \
        bfly_pass<GG, SS, TRANSPOSE>(tile, ld, lrows, d, sexp, tab0, estride, poff, nt);              \
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
// 2^lrows of the shared-memory tile `tile`; row r uses the engine table (for
// that direction) at tab0 + sexp[r] * estride (estride >= L*d/2 slots, even)
// or, with sexp == nullptr, the single table tab0.  6 <= L <= 12.  Must be
// called by all threads of the block (has __syncthreads).
template <typename Tab>
__device__ __forceinline__ void bfly_tile(float *tile, int ld, int lrows, int d, int L, const int *sexp, Tab tab0,
                                          int estride, bool transpose)
{
    const uint32_t ts = smem_addr(tile);
    const int np = npass_of(L);
    int poff = 0;
    for (int q = 0; q < np; ++q) {
        const int pi = transpose ? (np - 1 - q) : q;
        int s0, g;
        pass_bounds(L, pi, s0, g);
        if (transpose)
            bfly_pass_dispatch<true>(L, pi, ts, ld, lrows, d, sexp, tab0, estride, poff);
        else
            bfly_pass_dispatch<false>(L, pi, ts, ld, lrows, d, sexp, tab0, estride, poff);
        poff += g * (d >> 1);
        __syncthreads();
    }
}

// log2 of a power of two.
__host__ __device__ constexpr int ilog2_pow2(int x) { return x <= 1 ? 0 : 1 + ilog2_pow2(x >> 1); }

// Rows per shared-memory tile: up to 32 (a warp's lanes), at most 16384
// floats of data.
__host__ __device__ constexpr int tile_rows_for(int d) { return (16384 / d) < 32 ? (16384 / d) : 32; }

}  // namespace bfmoe
