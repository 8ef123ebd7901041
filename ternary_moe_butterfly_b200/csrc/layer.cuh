// layer.cuh -- the expert-layer kernels around the contraction:
//   k_pack_base    int8 ternary W_base -> 2-bit packed words
//   k_expert_in    gather each 32-row tile of bucketed rows (one or two
//                  experts' tables staged, else read from global memory),
//                  input rotation B(theta_e)^T, fp16 operand blocks for the
//                  GEMM
//   k_combine      output stages the GEMM epilogue could not reach (those
//                  that mix columns 256 or more apart, angles read from phi)
//                  and the per-token sum over the k routed rows, which the
//                  epilogue already scaled by alpha * gate
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
    const int i = blockIdx.x * blockDim.x + threadIdx.x;  // rotation pair
    if (i >= N * tab / 2) return;
    const int e = (2 * i) / tab, r = (2 * i) % tab;
    float c[2], sn[2];
    for (int h = 0; h < 2; ++h) {
        int s, p;
        engine_entry(d, L, transpose, r + h, s, p);
        sincosf(angles[((size_t)e * L + s) * (d / 2) + p], &sn[h], &c[h]);
        if (transpose) sn[h] = -sn[h];
    }
    reinterpret_cast<float4 *>(out)[i] = make_float4(c[0], c[1], sn[0], sn[1]);
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
    const int32_t *row_tok;  // [R] token of each bucket row
    const int32_t *row_exp;  // [R] expert of each bucket row
    const float2 *coef_t;    // [N][L*d/2] engine table of theta (B^T order)
    __half *a_blocks;        // fp16 operand blocks, rows in bucket order
    uint32_t *status;
};

// Persistent over tiles of tile_rows_for(d) consecutive bucket rows (one
// lane per row at d <= 512): gather the rows, rotate each by B(theta_e)^T of
// its own expert, write fp16 A blocks.  A tile holds the ends of at most a
// few buckets: when its rows have at most two experts, both experts'
// cos/sin tables are staged in shared memory (16 bytes apart in bank terms,
// so the two addresses of a warp's table load fall in distinct banks), else
// the rows read their tables from global memory.  Rows and tables arrive by
// bulk copies on one mbarrier (one memory latency per tile); the raw rows
// land in the fp32 tile's own bytes and are widened in place, in row groups
// whose order never overwrites raw data that is still to be read.
constexpr int kInThreads = 256;  // two CTAs per SM

// Byte stride of a raw staged row: 16 bytes of padding put the rows' 16-byte
// chunks in distinct bank groups for the lanes-are-rows widening loads.
__host__ __device__ constexpr uint32_t raw_row_stride(int d, int esize) { return (uint32_t)(d * esize + 16); }
// Shared-memory stride between the two staged tables, in entries.
__host__ __device__ constexpr int staged_table_stride(int d, int L) { return L * (d >> 1) + 2; }

template <typename T, bool SMEM_COEF>
__global__ void __launch_bounds__(kInThreads, 2) k_expert_in(ExpertInParams p)
{
    extern __shared__ __align__(16) uint8_t smem_in[];
    const int d = p.d, L = p.L;
    const int RT = tile_rows_for(d);
    const int ld = d + 1;
    const int tab = L * (d >> 1);
    const int tstride = staged_table_stride(d, L);
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem_in);
    int *mode = reinterpret_cast<int *>(smem_in + 8);    // 1: this tile's tables are staged
    int *stok = reinterpret_cast<int *>(smem_in + 16);   // [32] token of each tile row, -1: none
    int *sexp = reinterpret_cast<int *>(smem_in + 144);  // [32] table index of each tile row
    float2 *sc = reinterpret_cast<float2 *>(smem_in + 272);  // [2][tstride] when SMEM_COEF
    uint8_t *region = smem_in + 272 + (SMEM_COEF ? (size_t)2 * tstride * 8 : 0);
    float *tile = reinterpret_cast<float *>(region);  // [RT][ld] fp32, raw rows land here first
    constexpr int VPC = 16 / sizeof(T);                 // values per 16-byte chunk
    const uint32_t rs = raw_row_stride(d, sizeof(T));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    BFMOE_TRACE(1, threadIdx.x == 0, 0);
    pdl_wait();
    pdl_trigger();
    BFMOE_TRACE(1, threadIdx.x == 0, 1);
    const T *x = reinterpret_cast<const T *>(p.x);
    const int KC = d / kBK;
    const int nchunk = d / VPC;  // 16-byte chunks per row
    const int ntiles = (p.R + RT - 1) / RT;
    const int T_ = p.R / p.k;
    // rows widened per group: at most 8 chunks in flight per thread
    const int grows = max(1, min(RT, 8 * kInThreads / nchunk));
    uint32_t phase = 0;
    for (int ti = blockIdx.x; ti < ntiles; ti += gridDim.x) {
        const int r0 = ti * RT;
        const int nr = min(RT, p.R - r0);
        BFMOE_TRACE(1, threadIdx.x == 0 && ti == (int)blockIdx.x, 5);
        if (warp == 0) {
            // the rows' tokens and experts: one memory latency
            int t = -1, e = 0;
            if (lane < nr) {
                t = p.row_tok[r0 + lane];
                e = p.row_exp[r0 + lane];
                if (t < 0 || t >= T_) t = -1;
                if (e < 0 || e >= p.N) {
                    e = 0;
                    t = -1;
                }
            }
            const int ea = __shfl_sync(0xffffffffu, e, 0), eb = __shfl_sync(0xffffffffu, e, nr - 1);
            const bool two = SMEM_COEF && __all_sync(0xffffffffu, lane >= nr || e == ea || e == eb);
            if (lane < RT) {
                stok[lane] = t;
                sexp[lane] = two ? (e == ea ? 0 : 1) : e;
            }
            const unsigned have = __ballot_sync(0xffffffffu, t >= 0);
            if (lane == 0) {
                // the previous tile's reads of this memory (generic proxy)
                // come before the bulk copies' writes (async proxy)
                fence_proxy_async_smem();
                const uint32_t tb = (uint32_t)tab * 8;
                const uint32_t bytes = (uint32_t)__popc(have) * (uint32_t)(d * sizeof(T)) +
                                       (two ? (ea == eb ? tb : 2 * tb) : 0u);
                mbar_arrive_expect_tx(bar, bytes);
                if (two) {
                    bulk_g2s(sc, p.coef_t + (size_t)ea * tab, tb, bar);
                    if (eb != ea) bulk_g2s(sc + tstride, p.coef_t + (size_t)eb * tab, tb, bar);
                }
            }
            __syncwarp();
            if (t >= 0) {
                fence_proxy_async_smem();
                bulk_g2s(region + (size_t)lane * rs, x + (size_t)t * d, (uint32_t)(d * sizeof(T)), bar);
            }
            if (lane == 0) *mode = two ? 1 : 0;
        }
        const uint32_t cur = phase;
        const bool ok = __syncthreads_and(mbar_wait(bar, cur));
        phase ^= 1;
        if (!ok) {
            if (threadIdx.x == 0) {
                set_status(p.status, BFMOE_ERR_TIMEOUT);
                // the copies of this tile must land before the block's
                // shared memory is released: one more bounded wait
                mbar_wait(bar, cur);
            }
            __syncthreads();
            break;
        }
        const bool two = *mode != 0;
        BFMOE_TRACE(1, threadIdx.x == 0 && ti == (int)blockIdx.x, 6);
        // widen raw -> fp32 rows in place: 2-byte types from the last group
        // down (an fp32 row starts at or beyond twice its raw row's offset),
        // 4-byte types from the first group up (a raw row is the longer one)
        const int ngr = (nr + grows - 1) / grows;
        for (int gi = 0; gi < ngr; ++gi) {
            const int g = sizeof(T) == 2 ? ngr - 1 - gi : gi;
            const int ra = g * grows, rn = min(grows, nr - ra);
            uint4 u[8];
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const int q = (int)threadIdx.x + w * kInThreads;
                const int rr = q % rn, c = q / rn;
                u[w] = make_uint4(0, 0, 0, 0);
                if (c < nchunk && stok[ra + rr] >= 0)
                    u[w] = *reinterpret_cast<const uint4 *>(region + (size_t)(ra + rr) * rs + (size_t)c * 16);
            }
            __syncthreads();
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const int q = (int)threadIdx.x + w * kInThreads;
                const int rr = q % rn, c = q / rn;
                if (c >= nchunk) break;
                float f[VPC];
                if constexpr (VPC == 8) {
                    unpack_bf16x8(u[w], f);
                } else {
                    f[0] = __uint_as_float(u[w].x);
                    f[1] = __uint_as_float(u[w].y);
                    f[2] = __uint_as_float(u[w].z);
                    f[3] = __uint_as_float(u[w].w);
                }
                float *dst = tile + (size_t)(ra + rr) * ld + c * VPC;
#pragma unroll
                for (int i = 0; i < VPC; ++i) dst[i] = f[i];
            }
        }
        __syncthreads();
        BFMOE_TRACE(1, threadIdx.x == 0 && ti == (int)blockIdx.x, 3);
        // all RT rows go through the engine (rows past nr hold stale values
        // and are never stored): a power-of-two row count maps threads to
        // rows with masks
        if (two)
            bfly_tile(tile, ld, ilog2_pow2(RT), d, L, sexp, SmemTab{smem_addr(sc)}, tstride, /*transpose=*/true);
        else
            bfly_tile(tile, ld, ilog2_pow2(RT), d, L, sexp, GmemTab{p.coef_t}, tab, /*transpose=*/true);
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

__host__ inline size_t expert_in_smem_bytes(int d, int L, bool smem_coef, int esize)
{
    const size_t RT = tile_rows_for(d);
    const size_t raw = RT * raw_row_stride(d, esize), wide = RT * (size_t)(d + 1) * 4;
    return 272 + (smem_coef ? (size_t)2 * staged_table_stride(d, L) * 8 : 0) + (raw > wide ? raw : wide);
}

// Whether tiles may stage their experts' tables in shared memory: two
// tables of up to 20 KB.
__host__ inline bool expert_in_smem_coef(int d, int L) { return (size_t)L * (d / 2) * 8 <= 20 * 1024; }

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
    const float *phi;         // [N][L][d/2] output-butterfly angles
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
// all NH slices; the k rows are summed in j order.  KC > 0 fixes k = KC at
// compile time and issues the loads of all k rows together (expert indices,
// then rows and tables: two memory latencies per token); KC = 0 takes k from
// the parameters, one row at a time.
template <typename T, int HS, int BN, int QW, int KC>
__global__ void __launch_bounds__(256) k_combine(CombineParams p)
{
    BFMOE_TRACE(3, threadIdx.x == 0, 0);
    constexpr int NH = 1 << HS;
    constexpr int M2 = BN / 32;
    constexpr int TPT = 4 * M2;  // threads per token
    constexpr int KB = KC > 0 ? KC : 1;                 // rows loaded together
    const int tid = blockIdx.x * blockDim.x + threadIdx.x;
    const int t = tid / TPT;
    // with k fixed, the rows' expert indices are read before the wait (the
    // routing finished before the kernel this grid depends on started), so
    // that after it the products and the angles load together
    int ev_pre[KB];
#pragma unroll
    for (int b = 0; b < KB; ++b)
        ev_pre[b] = (KC > 0 && HS > 0 && t < p.T) ? min(max(__ldg(p.topk_idx + t * KB + b), 0), p.N - 1) : 0;
    pdl_wait();
    BFMOE_TRACE(3, threadIdx.x == 0, 1);
    pdl_trigger();
    if (t >= p.T) return;
    const int k = KC > 0 ? KC : p.k;
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
        for (int j0 = 0; j0 < k; j0 += KB) {
            float v[KB][NH][QW];
            int ev[KB];
#pragma unroll
            for (int b = 0; b < KB; ++b) {
                const int i = t * k + j0 + b;
                ev[b] = HS == 0 ? 0 : (KC > 0 ? ev_pre[b] : min(max(__ldg(p.topk_idx + i), 0), p.N - 1));
                const __half *row = p.slot + (size_t)i * d + pos0 + q0;
#pragma unroll
                for (int h = 0; h < NH; ++h) load_halves<QW>(row + h * BN, v[b][h]);
            }
#pragma unroll
            for (int b = 0; b < KB; ++b) {
                if (HS > 0) {
                    // stages s_lo + ls pair slices h, h + 2^ls at the same
                    // in-slice column c: pair index c + BN * ri, with ri the
                    // lower slice's index with bit ls deleted.  The angles come
                    // straight from phi (no table: the next call's preparation
                    // may already be rewriting the tables)
                    const float *ph = p.phi + (size_t)ev[b] * p.L * half + (size_t)p.s_lo * half + col0 + q0;
#pragma unroll
                    for (int ls = 0; ls < HS; ++ls)
#pragma unroll
                        for (int ri = 0; ri < NH / 2; ++ri) {
                            const int h = insert_zero_bit(ri, ls);
                            float a[QW];
#pragma unroll
                            for (int q = 0; q < QW; ++q) a[q] = __ldg(ph + (size_t)ls * half + BN * ri + q);
#pragma unroll
                            for (int q = 0; q < QW; ++q) {
                                float sn, cs;
                                __sincosf(a[q], &sn, &cs);
                                rot1(v[b][h][q], v[b][h + (1 << ls)][q], cs, sn);
                            }
                        }
                }
#pragma unroll
                for (int h = 0; h < NH; ++h)
#pragma unroll
                    for (int q = 0; q < QW; ++q) acc[h][q] += v[b][h][q];
            }
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
    BFMOE_TRACE(3, (threadIdx.x & 31) == 0, 2);
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
    bfly_tile(tile, ld, ilog2_pow2(RT), d, L, sexp, GmemTab{coef}, L * (d >> 1), transpose != 0);
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
