// layer.cuh -- the expert-layer kernels around the contraction:
//   k_pack_base    int8 ternary W_base -> 2-bit packed words
//   k_expert_in    gather each single-expert tile of bucketed rows, input
//                  rotation B(theta_e)^T, fp16 operand blocks for the GEMM
//   k_combine      output stages the GEMM epilogue could not reach (those
//                  that mix columns 256 or more apart), alpha * gate, and
//                  the per-token sum over the k routed rows
//   k_bfly_apply   standalone row butterfly (B or B^T)
//
// The method: expert i is W_i = alpha B(phi_i) W_base B(theta_i)^T with a
// single shared ternary W_base and per-expert butterflies; W_i is never
// formed -- input rotation, ternary product, output rotation in sequence
// (ButterflyMoE summaries, section 2 / 2.1; ButterflyViT summary, section 2).
#pragma once

#include "butterfly.cuh"
#include "common.cuh"
#include "route.cuh"

namespace bfmoe {

constexpr int kBM = 128;  // GEMM rows per tile (tcgen05 M)

// GEMM operand layout ("blocks"): a matrix with rows m and contraction index
// k is stored as blocks of 64 k-columns; block (mt, kc) holds rows
// [mt*BR, mt*BR + BR) x k in [64 kc, 64 kc + 64) as 8x8 core matrices of
// fp16, element (m, k) at ((m/8)*8 + (k%64)/8)*64 + (m%8)*8 + k%8 inside the
// block, and blocks are ordered (mt, kc) row-major.  One block is one
// contiguous bulk copy into shared memory, already in the tensor core's
// canonical K-major no-swizzle layout (core matrices 128 B apart along K,
// 1024 B apart along M).
__device__ __forceinline__ size_t block_elem_offset(int m, int k, int BR, int KC)
{
    const int mt = m / BR, mi = m % BR, kc = k / kBK, ki = k % kBK;
    return ((size_t)mt * KC + kc) * ((size_t)BR * kBK) + (size_t)(((mi >> 3) << 3) + (ki >> 3)) * 64 +
           (size_t)((mi & 7) << 3) + (ki & 7);
}

// ------------------------------------------------------------- packing --

// One thread per output word (the host writes the 16-byte header).  Any
// value outside {-1, 0, +1} sets *bad.
__global__ void k_pack_base(const int8_t *__restrict__ w, int d, uint32_t *__restrict__ words, uint32_t *bad)
{
    const size_t nwords = (size_t)d * d / 16;
    const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (q >= nwords) return;
    const int4 raw = *reinterpret_cast<const int4 *>(w + q * 16);
    const int8_t *v = reinterpret_cast<const int8_t *>(&raw);
    uint32_t word = 0;
    bool ok = true;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int x = v[i];
        ok &= (x >= -1 && x <= 1);
        const uint32_t code = x == 1 ? 1u : (x == -1 ? 3u : 0u);
        word |= code << (2 * i);
    }
    words[q] = word;
    if (!ok) atomicOr(bad, 1u);
}

// Engine table (see engine_entry) of every expert for one direction, from
// angles [N][L][d/2].
__global__ void k_engine_table(const float *__restrict__ angles, int N, int d, int L, bool transpose,
                               float2 *__restrict__ out)
{
    const int tab = L * (d / 2);
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= N * tab) return;
    const int e = i / tab, r = i % tab;
    int s, p;
    engine_entry(d, L, transpose, r, s, p);
    float sn, cs;
    sincosf(angles[((size_t)e * L + s) * (d / 2) + p], &sn, &cs);
    out[i] = make_float2(cs, transpose ? -sn : sn);
}

// ------------------------------------------------------- tile row I/O --

// Load one row of d values of type T into a tile row (fp32), cooperatively
// by one warp with 16-byte loads.
template <typename T>
__device__ __forceinline__ void warp_load_row(const T *__restrict__ src, float *dst, int d, int lane);

template <>
__device__ __forceinline__ void warp_load_row<float>(const float *__restrict__ src, float *dst, int d, int lane)
{
    for (int c = lane * 4; c < d; c += 128) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(src + c));
        dst[c] = v.x;
        dst[c + 1] = v.y;
        dst[c + 2] = v.z;
        dst[c + 3] = v.w;
    }
}

template <>
__device__ __forceinline__ void warp_load_row<__nv_bfloat16>(const __nv_bfloat16 *__restrict__ src, float *dst,
                                                             int d, int lane)
{
    for (int c = lane * 8; c < d; c += 256) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(src + c));
        float f[8];
        unpack_bf16x8(u, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[c + i] = f[i];
    }
}

template <typename T>
__device__ __forceinline__ void store8(T *dst, const float *f);
template <>
__device__ __forceinline__ void store8<float>(float *dst, const float *f)
{
    reinterpret_cast<float4 *>(dst)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4 *>(dst)[1] = make_float4(f[4], f[5], f[6], f[7]);
}
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16 *dst, const float *f)
{
    *reinterpret_cast<uint4 *>(dst) = pack_bf16x8(f);
}

__device__ __forceinline__ void store1(float *dst, float v) { *dst = v; }
__device__ __forceinline__ void store1(__nv_bfloat16 *dst, float v) { *dst = __float2bfloat16_rn(v); }

// ---------------------------------------------------------- input side --

struct ExpertInParams {
    const void *x;
    int d, L, k, N, R;
    const int32_t *perm;
    const int4 *tiles;       // single-expert row tiles {expert, row0, nrows, -}
    const int32_t *n_tiles;
    int max_tiles;           // capacity of `tiles`
    const float2 *coef_t;    // [N][L*d/2] engine table of theta (B^T order)
    __half *a_blocks;        // fp16 operand blocks, rows in bucket order
    uint32_t *status;
};

// Persistent over the tile list: gather the rows of one expert's tile, rotate
// by B(theta_e)^T (the expert's cos/sin table is staged in shared memory when
// it fits, so every coefficient load is a broadcast), write fp16 A blocks.
constexpr int kInThreads = 128;  // four CTAs per SM

template <typename T, bool SMEM_COEF>
__global__ void __launch_bounds__(kInThreads, 4) k_expert_in(ExpertInParams p)
{
    extern __shared__ __align__(16) float smem_f[];
    const int d = p.d, L = p.L;
    const int RT = tile_rows_for(d);
    const int ld = d + 1;
    const size_t tab = (size_t)L * (d >> 1);
    float2 *sc = reinterpret_cast<float2 *>(smem_f);  // [tab] when SMEM_COEF
    float *tile = smem_f + (SMEM_COEF ? 2 * tab : 0);
    int *stok = reinterpret_cast<int *>(tile + (size_t)RT * ld);
    BFMOE_TRACE(1, threadIdx.x == 0, 0);
    pdl_wait();
    pdl_trigger();
    BFMOE_TRACE(1, threadIdx.x == 0, 1);
    // a routing that gave up (timeout) leaves the list unspecified: clamp it
    const int ntiles = min(max(*p.n_tiles, 0), p.max_tiles);
    const T *x = reinterpret_cast<const T *>(p.x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int KC = d / kBK;
    for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x) {
        const int4 tl = p.tiles[ti];
        const int e = min(max(tl.x, 0), p.N - 1);
        const int r0 = tl.y;
        int nr = min(max(tl.z, 0), RT);
        if (r0 < 0 || r0 > p.R - nr) nr = 0;
        if (nr == 0) continue;  // uniform across the block
        const float2 *gtab = p.coef_t + (size_t)e * tab;
        BFMOE_TRACE(1, threadIdx.x == 0 && ti == (int)blockIdx.x, 5);
        if ((int)threadIdx.x < RT) {
            int t = -1;
            const int r = r0 + (int)threadIdx.x;
            if ((int)threadIdx.x < nr && r >= 0 && r < p.R) {
                const int i = p.perm[r];
                if (i >= 0 && i < p.R) t = i / p.k;
            }
            stok[threadIdx.x] = t;
        }
        __syncthreads();
        // gather: lane = tile row, warp = 16-byte column chunk, so the scalar
        // shared-memory stores of a warp hit 32 distinct banks; the first
        // batch of loads is issued before the expert's table is built, so
        // the two overlap
        BFMOE_TRACE(1, threadIdx.x == 0 && ti == (int)blockIdx.x, 6);
        const int t_lane = lane < nr ? stok[lane] : -1;
        constexpr int VPC = 16 / sizeof(T);  // values per 16-byte chunk
        const int nchunk = d / VPC;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)(t_lane >= 0 ? t_lane : 0) * d);
        float *dst = tile + (size_t)lane * ld;
        for (int c0 = warp; c0 < nchunk; c0 += 8 * nw) {
            uint4 u[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int c = c0 + q * nw;
                u[q] = (t_lane >= 0 && c < nchunk) ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            }
            if (SMEM_COEF && c0 == warp) {
                // stage the expert's table (contiguous) while the row loads fly
                copy_g2s(reinterpret_cast<const float4 *>(gtab), reinterpret_cast<float4 *>(sc), (int)tab / 2,
                         threadIdx.x, blockDim.x);
                BFMOE_TRACE(1, threadIdx.x == 0 && ti == (int)blockIdx.x, 7);
            }
            if (lane < nr) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int c = c0 + q * nw;
                    if (c >= nchunk) break;
                    float f[8];
                    if (VPC == 8) {
                        unpack_bf16x8(u[q], f);
                    } else {
                        f[0] = __uint_as_float(u[q].x);
                        f[1] = __uint_as_float(u[q].y);
                        f[2] = __uint_as_float(u[q].z);
                        f[3] = __uint_as_float(u[q].w);
                    }
#pragma unroll
                    for (int i = 0; i < VPC; ++i) dst[c * VPC + i] = f[i];
                }
            }
        }
        __syncthreads();
        BFMOE_TRACE(1, threadIdx.x == 0 && ti == (int)blockIdx.x, 3);
        if (SMEM_COEF)
            bfly_tile(tile, ld, nr, d, L, nullptr, SmemTab{smem_addr(sc)}, /*transpose=*/true);
        else
            bfly_tile(tile, ld, nr, d, L, nullptr, GmemTab{gtab}, /*transpose=*/true);
        BFMOE_TRACE(1, threadIdx.x == 0 && ti == (int)blockIdx.x, 4);
        bool overflow = false;
        const int nch = nr * (d / 8);
        for (int q = threadIdx.x; q < nch; q += blockDim.x) {
            const int rq = q % nr, c8 = q / nr;
            const float *src = tile + (size_t)rq * ld + c8 * 8;
            float f[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                f[i] = src[i];
                overflow |= !(fabsf(f[i]) <= 65504.0f);
            }
            const size_t off = block_elem_offset(r0 + rq, c8 * 8, kBM, KC);
            *reinterpret_cast<uint4 *>(p.a_blocks + off) = pack_f16x8(f);
        }
        if (overflow) set_status(p.status, BFMOE_ERR_NONFINITE);
        __syncthreads();
    }
    BFMOE_TRACE(1, threadIdx.x == 0, 2);
}

__host__ inline size_t expert_in_smem_bytes(int d, int L, bool smem_coef)
{
    const int RT = tile_rows_for(d);
    return (smem_coef ? (size_t)L * (d / 2) * 8 : 0) + (size_t)RT * (d + 1) * 4 + (size_t)RT * 4;
}

__host__ inline bool expert_in_smem_coef(int d, int L) { return (size_t)L * (d / 2) * 8 <= 40 * 1024; }

// ------------------------------------------------------------ combine --

// Slot layout.  The contraction epilogue leaves each routed row i = t*k + j
// as alpha * g_{t,j} * (output butterfly stages 0 .. SIN-1 applied), fp16,
// d values.  Inside the row, BN-column slice nh holds its columns
// nh*BN + 8*grp + q + 32*m (grp < 4, q < 8, m < BN/32) at position
// nh*BN + (grp * (BN/32) + m) * 8 + q: each epilogue thread's 8 x BN/32 values
// form one contiguous run, and every run of 8 holds 8 consecutive columns.
struct CombineParams {
    const __half *slot;       // [T*k][d] fp16, rows in token order (i = t*k + j), slot layout
    int T, d, L, k, N;
    int s_lo;                 // first output stage left to apply (log2 of the GEMM's N tile)
    const int32_t *topk_idx;
    const float2 *coef_p;     // [N][L*d/2] output table (see out_table_entry)
    void *y;
    uint32_t *status;
};

template <typename T>
__device__ __forceinline__ void store_cols(T *dst, const float *f, int n);
template <>
__device__ __forceinline__ void store_cols<float>(float *dst, const float *f, int n)
{
    for (int i = 0; i < n; i += 4) *reinterpret_cast<float4 *>(dst + i) = make_float4(f[i], f[i + 1], f[i + 2], f[i + 3]);
}
template <>
__device__ __forceinline__ void store_cols<__nv_bfloat16>(__nv_bfloat16 *dst, const float *f, int n)
{
    if (n == 8) {
        *reinterpret_cast<uint4 *>(dst) = pack_bf16x8(f);
    } else {
        for (int i = 0; i < n; i += 2) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[i], f[i + 1]);
            *reinterpret_cast<__nv_bfloat162 *>(dst + i) = h;
        }
    }
}

// n consecutive fp16 values (n = 2, 4 or 8, aligned to 2n bytes) as one load
template <int n>
__device__ __forceinline__ void load_halves(const __half *src, float *f)
{
    uint32_t w[n / 2];
    if constexpr (n == 8) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(src));
        w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
    } else if constexpr (n == 4) {
        const uint2 u = __ldcs(reinterpret_cast<const uint2 *>(src));
        w[0] = u.x, w[1] = u.y;
    } else {
        w[0] = __ldcs(reinterpret_cast<const unsigned int *>(src));
    }
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
        __half2 h;
        *reinterpret_cast<uint32_t *>(&h) = w[i];
        const float2 x = __half22float2(h);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}

// y_t = sum_j (stages s_lo..L-1 of B(phi_e)) slot_{t,j}: the rows arrive
// already scaled by alpha * g.  HS = L - s_lo stages mix the NH = 2^HS slices
// (pairs of slices nh, nh + 2^ls at the same in-slice column).  One thread per
// (token, 8-column group, m) handles QW of the group's 8 columns per round in
// all NH slices; the k rows are summed in j order.
template <typename T, int HS, int BN, int QW>
__global__ void __launch_bounds__(256) k_combine(CombineParams p)
{
    BFMOE_TRACE(3, threadIdx.x == 0, 0);
    pdl_wait();
    BFMOE_TRACE(3, threadIdx.x == 0, 1);
    pdl_trigger();
    constexpr int NH = 1 << HS;
    constexpr int M2 = BN / 32;
    constexpr int TPT = 4 * M2;  // threads per token
    constexpr int PC = HS > 0 ? (HS << (HS - 1)) : 1;  // table entries per column
    const int tid = blockIdx.x * blockDim.x + threadIdx.x;
    const int t = tid / TPT;
    if (t >= p.T) return;
    const int g = (tid % TPT) / M2, m = tid % M2;
    const int d = p.d, half = d >> 1;
    const int col0 = 8 * g + 32 * m;           // first of the thread's 8 in-slice columns
    const int pos0 = (g * M2 + m) * 8;         // their slot position inside a slice
    bool bad = false;
#pragma unroll 1
    for (int q0 = 0; q0 < 8; q0 += QW) {
        float acc[NH][QW];
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int q = 0; q < QW; ++q) acc[h][q] = 0.0f;
#pragma unroll 1
        for (int j = 0; j < p.k; ++j) {
            const int i = t * p.k + j;
            const __half *row = p.slot + (size_t)i * d + pos0 + q0;
            float v[NH][QW];
#pragma unroll
            for (int h = 0; h < NH; ++h) load_halves<QW>(row + h * BN, v[h]);
            if (HS > 0) {
                const int e = min(max(p.topk_idx[i], 0), p.N - 1);
                // combine part of the output table: [column][ls][pair over slices]
                const float2 *cf = p.coef_p + (size_t)e * p.L * half + (size_t)p.s_lo * half;
#pragma unroll
                for (int q = 0; q < QW; ++q) {
                    const float2 *cq = cf + (size_t)(col0 + q0 + q) * PC;
#pragma unroll
                    for (int ls = 0; ls < HS; ++ls)
#pragma unroll
                        for (int ri = 0; ri < NH / 2; ++ri) {
                            const int h = insert_zero_bit(ri, ls);
                            const float2 w = __ldg(cq + (ls << (HS > 0 ? HS - 1 : 0)) + ri);
                            const float a = v[h][q], b = v[h + (1 << ls)][q];
                            v[h][q] = fmaf(w.x, a, -(w.y * b));
                            v[h + (1 << ls)][q] = fmaf(w.y, a, w.x * b);
                        }
                }
            }
#pragma unroll
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int q = 0; q < QW; ++q) acc[h][q] += v[h][q];
        }
        T *y = reinterpret_cast<T *>(p.y) + (size_t)t * d + col0 + q0;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
#pragma unroll
            for (int q = 0; q < QW; ++q) bad |= !isfinite(acc[h][q]);
            store_cols<T>(y + h * BN, acc[h], QW);
        }
    }
    if (bad) set_status(p.status, BFMOE_ERR_NONFINITE);
}

// ------------------------------------------------------ standalone rows --

template <typename T>
__global__ void __launch_bounds__(256) k_bfly_apply(const T *__restrict__ x, int rows, int d, int L,
                                                    const int32_t *__restrict__ expert_of_row,
                                                    const float2 *__restrict__ coef, int transpose,
                                                    T *__restrict__ y, int N, uint32_t *status)
{
    extern __shared__ float tile[];
    const int RT = tile_rows_for(d);
    const int ld = d + 1;
    int *sexp = reinterpret_cast<int *>(tile + (size_t)RT * ld);
    const int r0 = blockIdx.x * RT;
    const int nr = min(RT, rows - r0);
    if (threadIdx.x < RT) {
        int e = 0;
        if ((int)threadIdx.x < nr && expert_of_row) {
            e = expert_of_row[r0 + threadIdx.x];
            if (e < 0 || e >= N) {
                set_status(status, BFMOE_ERR_INVALID_ARG);
                e = 0;
            }
        }
        sexp[threadIdx.x] = e;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int q = warp; q < RT; q += nw) {
        float *dst = tile + (size_t)q * ld;
        if (q < nr)
            warp_load_row<T>(x + (size_t)(r0 + q) * d, dst, d, lane);
        else
            for (int c = lane; c < d; c += 32) dst[c] = 0.0f;
    }
    __syncthreads();
    bfly_tile(tile, ld, RT, d, L, sexp, GmemTab{coef}, transpose != 0);
    const int nch = nr * (d / 8);
    for (int q = threadIdx.x; q < nch; q += blockDim.x) {
        const int rq = q / (d / 8), c8 = q % (d / 8);
        const float *src = tile + (size_t)rq * ld + c8 * 8;
        float f[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = src[i];
        store8<T>(y + (size_t)(r0 + rq) * d + c8 * 8, f);
    }
}

__host__ inline size_t rows_smem_bytes(int d, int extra_ints_per_row)
{
    const int RT = tile_rows_for(d);
    return (size_t)RT * (d + 1) * 4 + (size_t)RT * 4 * extra_ints_per_row;
}

}  // namespace bfmoe
