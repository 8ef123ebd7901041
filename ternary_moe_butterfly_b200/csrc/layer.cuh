// layer.cuh -- the expert-layer kernels other than routing:
//   k_pack_base      int8 ternary W_base -> 2-bit packed base (+ header)
//   k_decode_base    packed base -> fp16 B-operand blocks for the GEMM
//   k_coef           angles -> {cos, sin} tables
//   k_expert_in      gather routed rows by bucket, input rotation B(theta)^T,
//                    fp16 A-operand blocks
//   k_contract       ONE tcgen05 GEMM of all routed rows against W_base
//   k_expert_out     output rotation B(phi), alpha * gate, combine per token
//   k_bfly_apply     standalone row butterfly (B or B^T)
//
// The method: expert i is W_i = alpha B(phi_i) W_base B(theta_i)^T with a
// single shared ternary W_base and per-expert butterflies; W_i is never
// formed -- input rotation, ternary product, output rotation in sequence
// (ButterflyMoE summaries, section 2 / 2.1; ButterflyViT summary, section 2).
//
// GEMM operand layout ("blocks"): a matrix with rows m and contraction index
// k is stored as blocks of 64 k-columns; block (mt, kc) holds rows
// [mt*BR, mt*BR + BR) x k in [64 kc, 64 kc + 64) as 8x8 core matrices of
// fp16, element (m, k) at ((m/8)*8 + (k%64)/8)*64 + (m%8)*8 + k%8 inside the
// block, and blocks are ordered (mt, kc) row-major.  One block is one
// contiguous bulk copy into shared memory, already in the tensor core's
// canonical K-major no-swizzle layout (core matrices 128 B apart along K,
// 1024 B apart along M).
#pragma once

#include "butterfly.cuh"
#include "common.cuh"

namespace bfmoe {

constexpr int kBM = 128;          // GEMM rows per tile (tcgen05 M)
constexpr int kBK = 64;           // contraction columns per pipeline stage
constexpr int kGemmStages = 4;
constexpr uint32_t kPackMagic = 0x32574642u;  // "BFW2"

__host__ __device__ constexpr int gemm_bn(int d) { return d < 256 ? d : 256; }

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

// Packed base -> fp16 B blocks (rows = output index n, contraction = k).
// One thread per 16-byte chunk (8 consecutive k of one row).
__global__ void k_decode_base(const uint32_t *__restrict__ packed, int d, __half *__restrict__ wb,
                              uint32_t *status)
{
    const int BN = gemm_bn(d);
    const int KC = d / kBK;
    const size_t nchunks = (size_t)d * d / 8;
    const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (q == 0 && (packed[0] != kPackMagic || packed[1] != (uint32_t)d)) set_status(status, BFMOE_ERR_INVALID_ARG);
    if (q >= nchunks) return;
    // q enumerates chunks in memory order of the block layout
    const size_t blk = q / ((size_t)BN * 8);
    const int within = (int)(q % ((size_t)BN * 8));
    const int core = within >> 3, rr = within & 7;
    const int nt = (int)(blk / KC), kc = (int)(blk % KC);
    const int n = nt * BN + ((core >> 3) << 3) + rr;
    const int k0 = kc * kBK + ((core & 7) << 3);
    const uint32_t word = packed[4 + (size_t)n * (d / 16) + (k0 >> 4)];
    const uint32_t bits = word >> (2 * (k0 & 15));
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t c0 = (bits >> (4 * i)) & 3u, c1 = (bits >> (4 * i + 2)) & 3u;
        // 01 -> +1 (0x3C00), 11 -> -1 (0xBC00), 00 / 10 -> 0
        const uint32_t lo = c0 == 1u ? 0x3C00u : (c0 == 3u ? 0xBC00u : 0u);
        const uint32_t hi = c1 == 1u ? 0x3C00u : (c1 == 3u ? 0xBC00u : 0u);
        h[i] = lo | (hi << 16);
    }
    reinterpret_cast<uint4 *>(wb)[q] = make_uint4(h[0], h[1], h[2], h[3]);
}

// --------------------------------------------------------------- angles --

__global__ void k_coef(const float *__restrict__ a0, const float *__restrict__ a1, int count,
                       float2 *__restrict__ c0, float2 *__restrict__ c1)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < count) {
        float s, c;
        sincosf(a0[i], &s, &c);
        c0[i] = make_float2(c, s);
    } else if (a1 && i < 2 * count) {
        float s, c;
        sincosf(a1[i - count], &s, &c);
        c1[i - count] = make_float2(c, s);
    }
}

// ------------------------------------------------------- tile row loads --

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

// ---------------------------------------------------------- input side --

// Rows r in [blockIdx.x*RT, +RT) of the bucket-sorted row list: gather x of
// the row's token, rotate by B(theta_e)^T, write fp16 A blocks.  Rows >= R
// (tile padding) are written as zeros.
template <typename T>
__global__ void __launch_bounds__(256) k_expert_in(const T *__restrict__ x, int d, int L, int k, int R,
                                                   const int32_t *__restrict__ perm,
                                                   const int32_t *__restrict__ topk_idx,
                                                   const float2 *__restrict__ coef_theta, __half *__restrict__ a_blocks,
                                                   uint32_t *status)
{
    extern __shared__ float tile[];
    const int RT = tile_rows_for(d);
    const int ld = d + 1;
    int *sexp = reinterpret_cast<int *>(tile + (size_t)RT * ld);
    int *stok = sexp + RT;
    const int r0 = blockIdx.x * RT;
    if (threadIdx.x < RT) {
        const int r = r0 + threadIdx.x;
        int e = 0, t = -1;
        if (r < R) {
            const int i = perm[r];
            t = i / k;
            e = topk_idx[i];
        }
        sexp[threadIdx.x] = e;
        stok[threadIdx.x] = t;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int q = warp; q < RT; q += nw) {
        const int t = stok[q];
        float *dst = tile + (size_t)q * ld;
        if (t >= 0)
            warp_load_row<T>(x + (size_t)t * d, dst, d, lane);
        else
            for (int c = lane; c < d; c += 32) dst[c] = 0.0f;
    }
    __syncthreads();
    bfly_tile(tile, ld, RT, d, L, sexp, coef_theta, /*transpose=*/true);
    // fp16 A blocks: one thread per (row, 8-column chunk), rows fastest.
    const int KC = d / kBK;
    const int nch = RT * (d / 8);
    bool overflow = false;
    for (int q = threadIdx.x; q < nch; q += blockDim.x) {
        const int rq = q % RT, c8 = q / RT;
        const float *src = tile + (size_t)rq * ld + c8 * 8;
        float f[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            f[i] = src[i];
            overflow |= !(fabsf(f[i]) <= 65504.0f);
        }
        const size_t off = block_elem_offset(r0 + rq, c8 * 8, kBM, KC);
        *reinterpret_cast<uint4 *>(a_blocks + off) = pack_f16x8(f);
    }
    if (overflow) set_status(status, BFMOE_ERR_NONFINITE);
}

// ----------------------------------------------------------- contraction --

// Z[m][n] = sum_k A[m][k] * W[n][k] for one 128 x BN tile, fp16 operands,
// fp32 accumulation in tensor memory.  Thread 0 streams the A and W blocks
// with bulk copies through a kGemmStages-deep ring; thread 32 issues the
// tcgen05.mma instructions; all four warps drain the accumulator (warp w
// owns TMEM lanes 32w..32w+31 = tile rows 32w..32w+31) to fp32 Z.
__global__ void __launch_bounds__(128, 1) k_contract(const __half *__restrict__ a_blocks,
                                                     const __half *__restrict__ w_blocks, float *__restrict__ z,
                                                     int d, uint32_t *status)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int BN = gemm_bn(d);
    const int KC = d / kBK;
    const int S = KC < kGemmStages ? KC : kGemmStages;
    const uint32_t a_bytes = kBM * kBK * 2, b_bytes = (uint32_t)BN * kBK * 2;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + (size_t)S * a_bytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sB + (size_t)S * b_bytes);
    uint64_t *full = bars, *empty = bars + kGemmStages, *done = bars + 2 * kGemmStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kGemmStages + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int mt = blockIdx.x, nt = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, (uint32_t)BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (threadIdx.x == 0) {
        // producer
        const __half *a_src = a_blocks + (size_t)mt * KC * (kBM * kBK);
        const __half *b_src = w_blocks + (size_t)nt * KC * ((size_t)BN * kBK);
        int issued = 0;
        for (int kc = 0; kc < KC; ++kc) {
            const int s = kc % S;
            const uint32_t ph = (uint32_t)(kc / S) & 1u;
            if (!mbar_wait(&empty[s], ph ^ 1u)) {
                set_status(status, BFMOE_ERR_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            if (*abort_flag) break;
            mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
            bulk_g2s(sA + (size_t)s * a_bytes, a_src + (size_t)kc * (kBM * kBK), a_bytes, &full[s]);
            bulk_g2s(sB + (size_t)s * b_bytes, b_src + (size_t)kc * ((size_t)BN * kBK), b_bytes, &full[s]);
            issued = kc + 1;
        }
        // before leaving, every copy issued must have landed
        for (int kc = issued - S > 0 ? issued - S : 0; kc < issued; ++kc)
            if (!mbar_wait(&full[kc % S], (uint32_t)(kc / S) & 1u)) set_status(status, BFMOE_ERR_TIMEOUT);
    } else if (threadIdx.x == 32) {
        // MMA issuer
        const uint32_t idesc = idesc_f16_f32(kBM, BN);
        for (int kc = 0; kc < KC; ++kc) {
            const int s = kc % S;
            if (!mbar_wait(&full[s], (uint32_t)(kc / S) & 1u)) {
                set_status(status, BFMOE_ERR_TIMEOUT);
                *abort_flag = 1;
                break;
            }
            if (*abort_flag) break;
            tc_fence_after();
            const uint32_t a0 = smem_addr(sA + (size_t)s * a_bytes), b0 = smem_addr(sB + (size_t)s * b_bytes);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
                const uint64_t ad = sdesc_noswizzle(a0 + kk * 256, 128, 1024);
                const uint64_t bd = sdesc_noswizzle(b0 + kk * 256, 128, 1024);
                mma_f16(tmem, ad, bd, idesc, (kc | kk) != 0);
            }
            mma_commit(&empty[s]);
        }
        mma_commit(done);  // arrives once every MMA issued above has completed
    }
    __syncwarp();
    // epilogue: all 128 threads; every branch below is warp-uniform so the
    // .sync.aligned TMEM loads see converged warps
    bool ok = mbar_wait(done, 0);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) set_status(status, BFMOE_ERR_TIMEOUT);
    tc_fence_after();
    const bool aborted = __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;
    if (ok && !aborted) {
        const int row = mt * kBM + warp * 32 + lane;
        float *zrow = z + (size_t)row * d + (size_t)nt * BN;
        for (int c = 0; c < BN; c += 32) {
            float v[32];
            tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4 *>(zrow + c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, (uint32_t)BN);
}

__host__ inline size_t contract_smem_bytes(int d)
{
    const int BN = gemm_bn(d);
    const int KC = d / kBK;
    const int S = KC < kGemmStages ? KC : kGemmStages;
    return 1024 + (size_t)S * (kBM * kBK * 2 + (size_t)BN * kBK * 2) + (2 * kGemmStages + 1) * 8 + 16;
}

// ---------------------------------------------------------- output side --

// Tokens [blockIdx.x*TT, +TT): for each routed row (t, j) read Z at its
// bucket position, rotate by B(phi_e), then y_t = alpha sum_j g_j u_j.
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

template <typename T>
__global__ void __launch_bounds__(256) k_expert_out(const float *__restrict__ z, int d, int L, int T_, int k,
                                                    const int32_t *__restrict__ row_pos,
                                                    const int32_t *__restrict__ topk_idx,
                                                    const float *__restrict__ gates,
                                                    const float2 *__restrict__ coef_phi,
                                                    const uint32_t *__restrict__ packed, T *__restrict__ y)
{
    extern __shared__ float tile[];
    const int RT0 = tile_rows_for(d);
    const int TT = RT0 / k > 0 ? RT0 / k : 1;
    const int RT = TT * k;
    const int ld = d + 1;
    int *sexp = reinterpret_cast<int *>(tile + (size_t)RT * ld);
    int *spos = sexp + RT;
    float *sg = reinterpret_cast<float *>(spos + RT);
    const int t0 = blockIdx.x * TT;
    if (threadIdx.x < RT) {
        const int t = t0 + threadIdx.x / k;
        int e = 0, pos = -1;
        float g = 0.0f;
        if (t < T_) {
            const int i = t * k + threadIdx.x % k;
            pos = row_pos[i];
            e = topk_idx[i];
            g = gates[i];
        }
        sexp[threadIdx.x] = e;
        spos[threadIdx.x] = pos;
        sg[threadIdx.x] = g;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int q = warp; q < RT; q += nw) {
        const int pos = spos[q];
        float *dst = tile + (size_t)q * ld;
        if (pos >= 0)
            warp_load_row<float>(z + (size_t)pos * d, dst, d, lane);
        else
            for (int c = lane; c < d; c += 32) dst[c] = 0.0f;
    }
    __syncthreads();
    bfly_tile(tile, ld, RT, d, L, sexp, coef_phi, /*transpose=*/false);
    const float alpha = __uint_as_float(packed[2]);
    const int nch = TT * (d / 8);
    for (int q = threadIdx.x; q < nch; q += blockDim.x) {
        const int tt = q / (d / 8), c8 = q % (d / 8);
        const int t = t0 + tt;
        if (t >= T_) continue;
        float f[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] = 0.0f;
        for (int j = 0; j < k; ++j) {
            const float *src = tile + (size_t)(tt * k + j) * ld + c8 * 8;
            const float g = sg[tt * k + j];
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = fmaf(g, src[i], f[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] *= alpha;
        store8<T>(y + (size_t)t * d + c8 * 8, f);
    }
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
    bfly_tile(tile, ld, RT, d, L, sexp, coef, transpose != 0);
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
