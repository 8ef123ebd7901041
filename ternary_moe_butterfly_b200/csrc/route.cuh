// route.cuh -- top-k gate over given router logits and deterministic
// bucketing of the routed rows by expert, in ONE cooperative kernel.
//
// A standard top-k gate selects each token's active experts (ButterflyMoE
// summary, Dutch page, section 2 "Three phases", gated routing).  Order:
// larger logit first, ties to the lower expert index; gate = softmax over
// the k selected logits.  Bucketing is a stable counting sort of the rows
// i = t*k + j by expert, so each bucket lists its rows in token order.
//
// Phases, separated by one or two bounded grid barriers (all blocks are
// co-resident: the kernel is launched cooperatively):
//   A  each block takes a contiguous token range; batches of its tokens'
//      logits are staged in shared memory and one thread (one warp beyond
//      256 experts) per token selects the top-k; the block counts its rows
//      per expert (hist[block][e]).
//   B  up to 512 experts, every block reads the (expert-major) histogram
//      and forms the expert totals and its own prefix over the blocks before
//      it; beyond, one warp per expert scans the column over the blocks and a
//      second grid barrier publishes the prefixes.
//   C  every block scans the expert totals into bucket offsets, then ranks
//      the rows of its tokens inside their buckets (warp match + popcount)
//      and scatters perm / row_pos; the blocks also write the list of
//      single-expert row tiles that the input-butterfly kernel walks.
#pragma once

#include "butterfly.cuh"
#include "common.cuh"

namespace bfmoe {

__host__ __device__ inline void out_table_entry(int d, int L, int r, int &s, int &p);
__host__ __device__ inline int out_pos(int d, int L, int s, int p);
// log2 of the contraction's output slice width BN: the output-butterfly
// stages its epilogue applies (the rest go to the combine).
__host__ __device__ constexpr int slice_stages(int BN) { return BN == 256 ? 8 : (BN == 128 ? 7 : 6); }

constexpr int kRouteThreads = 256;
constexpr int kMaxK = 8;
constexpr int kMaxRouteBlocks = 512;  // capacity of the per-block histogram
constexpr int kOneBarrierMaxN = 512;  // up to this many experts the routing needs one grid barrier
constexpr int kHistStageInts = 8192;  // histogram ints staged per chunk (32 KB)
constexpr uint32_t kPackMagic = 0x32574642u;  // "BFW2"

__host__ __device__ constexpr int gemm_bn(int d) { return d < 256 ? d : 256; }
constexpr int kBK = 64;  // contraction columns per GEMM operand block

struct RouteParams {
    const float *logits;
    int T, N, k;
    int32_t *topk_idx;   // [T][k]
    float *gates;        // [T][k]
    int32_t *perm;       // [T*k]
    int32_t *row_pos;    // [T*k] or null
    int32_t *offsets;    // [N+1]
    int32_t *hist;       // [gridDim][N] -> per-block bucket bases
    int32_t *total;      // [N]
    uint32_t *sync;      // grid barrier counter, zero at launch
    uint32_t *status;
    int skip_arrive_block;  // test hook: this block never reaches barrier 1 (-1: none)
    int d;
    // forward only: single-expert row tiles for the input butterfly
    int4 *in_tiles;
    int32_t *n_in_tiles;
    int tile_rows;
};

// Up to this many experts one thread selects a token's top-k.
constexpr int kThreadTopkMaxN = 256;

// Tokens staged per batch: one per thread (at most 256), at most ~40 KB of
// logits.
__host__ __device__ inline int route_batch_tokens(int N)
{
    const int b = (40 * 1024 / 4) / (N + 1);
    return b < 1 ? 1 : (b > 256 ? 256 : b);
}

// (va, a) ranks before (vb, b)?  NaN has been mapped to -inf by the caller.
__device__ __forceinline__ bool ranks_before(float va, int a, float vb, int b)
{
    return va > vb || (va == vb && a < b);
}

// Split-phase grid-wide barrier on a monotonically increasing counter:
// arrive publishes the block's earlier writes; wait (bounded) returns false,
// block-uniformly, if the other blocks did not arrive in time.
__device__ __forceinline__ void grid_arrive(uint32_t *ctr)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1u);
    }
}

__device__ bool grid_wait(uint32_t *ctr, uint32_t target, uint32_t *status)
{
    __shared__ int ok;
    if (threadIdx.x == 0) {
        ok = 1;
        const unsigned long long t0 = globaltimer_ns();
        while (true) {
            const uint32_t v = *reinterpret_cast<volatile uint32_t *>(ctr);
            if (v >= target) break;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                set_status(status, BFMOE_ERR_TIMEOUT);
                ok = 0;
                break;
            }
        }
        __threadfence();
    }
    __syncthreads();
    return ok != 0;
}

// Gates of one token from its k selected logits (best first): softmax over
// the k, or its limit when a selected logit is infinite.
__device__ __forceinline__ void gates_of(const float *val, int k, float *g)
{
    const float m = val[0];
    if (m == INFINITY) {
        int cnt = 0;
        for (int j = 0; j < k; ++j) cnt += (val[j] == INFINITY);
        for (int j = 0; j < k; ++j) g[j] = (val[j] == INFINITY) ? 1.0f / (float)cnt : 0.0f;
    } else if (m == -INFINITY) {
        for (int j = 0; j < k; ++j) g[j] = 1.0f / (float)k;
    } else {
        float z = 0.0f;
        for (int j = 0; j < k; ++j) {
            g[j] = expf(val[j] - m);
            z += g[j];
        }
        const float rz = 1.0f / z;
        for (int j = 0; j < k; ++j) g[j] *= rz;
    }
}

// Top-k of one token by one thread: a sorted list of the K best (value,
// index) pairs in registers, one pass over the N logits at stride `stride`.
template <int K>
__device__ __forceinline__ void topk_thread(const RouteParams &p, int t, const float *l, int *sh_hist)
{
    float val[K];
    int sel[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
        val[j] = -INFINITY;
        sel[j] = 0x7fffffff;  // ranks after every real candidate
    }
    for (int e = 0; e < p.N; ++e) {
        const float v = l[e];
        bool b[K];
#pragma unroll
        for (int j = 0; j < K; ++j) b[j] = ranks_before(v, e, val[j], sel[j]);
#pragma unroll
        for (int j = K - 1; j > 0; --j) {
            if (b[j]) {
                val[j] = b[j - 1] ? val[j - 1] : v;
                sel[j] = b[j - 1] ? sel[j - 1] : e;
            }
        }
        if (b[0]) {
            val[0] = v;
            sel[0] = e;
        }
    }
    float g[K];
    gates_of(val, K, g);
#pragma unroll
    for (int j = 0; j < K; ++j) {
        p.topk_idx[(size_t)t * K + j] = sel[j];
        p.gates[(size_t)t * K + j] = g[j];
        atomicAdd(&sh_hist[sel[j]], 1);
    }
}

// Top-k and gates of one token whose N logits are in shared memory (NaN
// already replaced by -inf); one warp.  Lane 0 writes the results and counts
// the token's rows in the block histogram.
__device__ __forceinline__ void topk_token(const RouteParams &p, int t, const float *l, int *sh_hist)
{
    const int N = p.N, k = p.k;
    const int lane = threadIdx.x & 31;
    int sel[kMaxK];
    float val[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        if (j >= k) break;
        float bv = -INFINITY;
        int be = 0x7fffffff;
        for (int e = lane; e < N; e += 32) {
            bool taken = false;
#pragma unroll
            for (int jj = 0; jj < kMaxK; ++jj)
                if (jj < j) taken |= (sel[jj] == e);
            if (taken) continue;
            const float v = l[e];
            if (be == 0x7fffffff || ranks_before(v, e, bv, be)) {
                bv = v;
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (oe != 0x7fffffff && (be == 0x7fffffff || ranks_before(ov, oe, bv, be))) {
                bv = ov;
                be = oe;
            }
        }
        sel[j] = be;
        val[j] = bv;
    }
    if (lane == 0) {
        float g[kMaxK];
        gates_of(val, k, g);
        for (int j = 0; j < k; ++j) {
            p.topk_idx[(size_t)t * k + j] = sel[j];
            p.gates[(size_t)t * k + j] = g[j];
            atomicAdd(&sh_hist[sel[j]], 1);
        }
    }
}

// Top-k, gates and the histogram of the block's token range [t0, t1).
// Batches of tokens are staged in shared memory with coalesced 16-byte loads
// (one memory latency per batch; NaN becomes -inf and is reported).  Up to
// kThreadTopkMaxN experts one thread selects for one token (rows padded to
// N+1 floats so the threads' column reads hit distinct banks); beyond, one
// warp per token.
__device__ void topk_range(const RouteParams &p, int t0, int t1, int *sh_hist, float *sh_logits, bool &saw_nan)
{
    const int N = p.N;
    const bool per_thread = N <= kThreadTopkMaxN;
    const int ldl = per_thread ? N + 1 : N;
    const int batch = route_batch_tokens(N);
    for (int e = threadIdx.x; e < N; e += blockDim.x) sh_hist[e] = 0;
    const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int b0 = t0; b0 < t1; b0 += batch) {
        const int nb = min(batch, t1 - b0);
        const size_t nval = (size_t)nb * N;
        const float *src = p.logits + (size_t)b0 * N;
        __syncthreads();
        if ((N & 3) == 0 && (reinterpret_cast<uintptr_t>(p.logits) & 15) == 0) {
            const float4 *s4 = reinterpret_cast<const float4 *>(src);
            const int n4 = (int)(nval / 4);
            for (int q0 = threadIdx.x; q0 < n4; q0 += 8 * blockDim.x) {
                float4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int q = q0 + u * blockDim.x;
                    if (q < n4) v[u] = __ldg(s4 + q);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int q = q0 + u * blockDim.x;
                    if (q >= n4) break;
                    const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    const int tok = (4 * q) / N, e0 = (4 * q) % N;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float xv = f[i];
                        if (xv != xv) {
                            saw_nan = true;
                            xv = -INFINITY;
                        }
                        sh_logits[(size_t)tok * ldl + e0 + i] = xv;
                    }
                }
            }
        } else {
            for (size_t q = threadIdx.x; q < nval; q += blockDim.x) {
                float xv = __ldg(src + q);
                if (xv != xv) {
                    saw_nan = true;
                    xv = -INFINITY;
                }
                sh_logits[(q / N) * ldl + q % N] = xv;
            }
        }
        __syncthreads();
        if (per_thread) {
            const int q = threadIdx.x;
            if (q < nb) {
                const float *l = sh_logits + (size_t)q * ldl;
                switch (p.k) {
                case 1: topk_thread<1>(p, b0 + q, l, sh_hist); break;
                case 2: topk_thread<2>(p, b0 + q, l, sh_hist); break;
                case 3: topk_thread<3>(p, b0 + q, l, sh_hist); break;
                case 4: topk_thread<4>(p, b0 + q, l, sh_hist); break;
                case 5: topk_thread<5>(p, b0 + q, l, sh_hist); break;
                case 6: topk_thread<6>(p, b0 + q, l, sh_hist); break;
                case 7: topk_thread<7>(p, b0 + q, l, sh_hist); break;
                default: topk_thread<8>(p, b0 + q, l, sh_hist); break;
                }
            }
        } else {
            for (int q = warp; q < nb; q += nw) topk_token(p, b0 + q, sh_logits + (size_t)q * ldl, sh_hist);
        }
    }
    __syncthreads();
}

// Packed base -> fp16 B blocks for the contraction (rows = output index n,
// contraction = k; see the operand layout in contract.cuh).  One call per
// 16-byte output chunk q (8 consecutive k of one row).
__device__ __forceinline__ void decode_chunk(const uint32_t *__restrict__ packed, int d, __half *__restrict__ wb,
                                             size_t q)
{
    const int BN = gemm_bn(d);
    const int KC = d / kBK;
    const size_t blk = q / ((size_t)BN * 8);
    const int within = (int)(q % ((size_t)BN * 8));
    const int core = within >> 3, rr = within & 7;
    const int nt = (int)(blk / KC), kc = (int)(blk % KC);
    const int n = nt * BN + ((core >> 3) << 3) + rr;
    const int k0 = kc * kBK + ((core & 7) << 3);
    const uint32_t word = __ldg(packed + 4 + (size_t)n * (d / 16) + (k0 >> 4));
    const uint32_t bits = word >> (2 * (k0 & 15));
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t c0 = (bits >> (4 * i)) & 3u, c1 = (bits >> (4 * i + 2)) & 3u;
        // 01 -> +1 (fp16 0x3C00), 11 -> -1 (0xBC00), 00 / 10 -> 0
        const uint32_t lo = c0 == 1u ? 0x3C00u : (c0 == 3u ? 0xBC00u : 0u);
        const uint32_t hi = c1 == 1u ? 0x3C00u : (c1 == 3u ? 0xBC00u : 0u);
        h[i] = lo | (hi << 16);
    }
    reinterpret_cast<uint4 *>(wb)[q] = make_uint4(h[0], h[1], h[2], h[3]);
}

// Exclusive scan of src[0..n) into dst[0..n) by the whole block (warp
// shuffles; `scratch` holds 72 ints); returns the sum.  src and dst may alias.
__device__ int block_exclusive_scan(const int *src, int *dst, int n, int *scratch)
{
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    int s = 0;
    for (int e = lo; e < hi; ++e) s += src[e];
    int incl = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < nw ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += o;
        }
        if (lane < nw) scratch[32 + lane] = wi - w;  // exclusive prefix of the warp totals
        if (lane == nw - 1) scratch[64] = wi;         // block total
    }
    __syncthreads();
    int run = scratch[32 + warp] + incl - s;
    const int total = scratch[64];
    for (int e = lo; e < hi; ++e) {
        const int v = src[e];
        dst[e] = run;
        run += v;
    }
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(kRouteThreads) k_route(RouteParams p)
{
    extern __shared__ int sh[];  // phase A: hist[N] + staged logits; phase C: off, tstart, cnt, scratch
    const int N = p.N, k = p.k;
    const int nblk = gridDim.x;  // one histogram row per block

    BFMOE_TRACE(0, threadIdx.x == 0, 0);
    pdl_trigger();  // the prep kernel may start now and run beside the routing
    // ---- phase A: top-k over this block's token range
    float *sh_logits = reinterpret_cast<float *>(sh + ((N + 3) & ~3));
    bool saw_nan = false;
    const int tpb = (p.T + nblk - 1) / nblk;  // tokens per block
    const int t0 = min(p.T, (int)blockIdx.x * tpb), t1 = min(p.T, t0 + tpb);
    topk_range(p, t0, t1, sh, sh_logits, saw_nan);
    const bool one_barrier = N <= kOneBarrierMaxN;  // one grid barrier
    const int np4 = (N + 3) & ~3;                    // histogram row stride, 16-byte multiple
    for (int e = threadIdx.x; e < N; e += blockDim.x) p.hist[(size_t)blockIdx.x * (one_barrier ? np4 : N) + e] = sh[e];
    if (__any_sync(0xffffffffu, saw_nan) && (threadIdx.x & 31) == 0) set_status(p.status, BFMOE_ERR_NONFINITE);
    BFMOE_TRACE(0, threadIdx.x == 0, 1);
    const bool arrive = (int)blockIdx.x != p.skip_arrive_block;  // test hook: one block never arrives
    if (arrive) grid_arrive(p.sync);

    const size_t gtid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t gthreads = (size_t)gridDim.x * blockDim.x;
    BFMOE_TRACE(0, threadIdx.x == 0, 2);
    if (!arrive) return;
    if (!grid_wait(p.sync, nblk, p.status)) return;
    BFMOE_TRACE(0, threadIdx.x == 0, 3);

    int *off = sh;              // [N+1]
    int *tstart = off + N + 1;  // [N+1]
    int *cnt = tstart + N + 1;  // [N]
    int *scratch = cnt + N;     // [72]
    if (one_barrier) {
        // ---- every block: expert totals and its own prefix over the blocks
        // before it, from the expert-major histogram, staged in shared memory
        // in chunks of experts with coalesced 16-byte loads
        int *stage = sh + ((3 * N + 82 + 3) & ~3);  // [rb * np4], 16-byte aligned
        const int rb = max(1, kHistStageInts / np4);  // histogram rows per chunk
        for (int e = threadIdx.x; e < N; e += blockDim.x) {
            off[e] = 0;
            cnt[e] = 0;
        }
        for (int b0 = 0; b0 < nblk; b0 += rb) {
            const int nb = min(rb, nblk - b0);
            copy_g2s(reinterpret_cast<const int4 *>(p.hist + (size_t)b0 * np4), reinterpret_cast<int4 *>(stage),
                     nb * np4 / 4, threadIdx.x, blockDim.x);
            __syncthreads();
            for (int e = threadIdx.x; e < N; e += blockDim.x) {
                int tot = 0, pre = 0;
                for (int b = 0; b < nb; ++b) {
                    const int v = stage[b * np4 + e];
                    tot += v;
                    pre += (b0 + b < (int)blockIdx.x) ? v : 0;
                }
                off[e] += tot;
                cnt[e] += pre;  // becomes the block's bucket base below
            }
            __syncthreads();
        }
    } else {
        // ---- phase B: one warp per expert, exclusive prefix over the blocks
        const int warp = (int)(gtid >> 5), lane = threadIdx.x & 31;
        const int nwarps = (int)(gthreads >> 5);
        constexpr int kPerLane = kMaxRouteBlocks / 32;
        for (int e = warp; e < N; e += nwarps) {
            int v[kPerLane];
#pragma unroll
            for (int q = 0; q < kPerLane; ++q) {
                const int c = q * 32 + lane;
                v[q] = c < nblk ? p.hist[(size_t)c * N + e] : 0;
            }
            int running = 0;
#pragma unroll
            for (int q = 0; q < kPerLane; ++q) {
                if (q * 32 >= nblk) break;
                int incl = v[q];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int x = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += x;
                }
                const int c = q * 32 + lane;
                if (c < nblk) p.hist[(size_t)c * N + e] = running + incl - v[q];
                running += __shfl_sync(0xffffffffu, incl, 31);
            }
            if (lane == 0) p.total[e] = running;
        }
        grid_arrive(p.sync);
        if (!grid_wait(p.sync, 2 * nblk, p.status)) return;
        for (int e = threadIdx.x; e < N; e += blockDim.x) {
            off[e] = p.total[e];
            cnt[e] = p.hist[(size_t)blockIdx.x * N + e];
        }
        __syncthreads();
    }
    BFMOE_TRACE(0, threadIdx.x == 0, 4);

    // ---- phase C: bucket offsets, tile list, ranks and scatter
    for (int e = threadIdx.x; e < N; e += blockDim.x)
        tstart[e] = p.tile_rows > 0 ? (off[e] + p.tile_rows - 1) / p.tile_rows : 0;
    __syncthreads();
    const int rsum = block_exclusive_scan(off, off, N, scratch);
    const int ntiles = p.in_tiles ? block_exclusive_scan(tstart, tstart, N, scratch) : 0;
    if (threadIdx.x == 0) {
        off[N] = rsum;
        tstart[N] = ntiles;
    }
    for (int e = threadIdx.x; e < N; e += blockDim.x) cnt[e] += off[e];
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= N; e += blockDim.x) p.offsets[e] = off[e];
        if (threadIdx.x == 0 && p.n_in_tiles) *p.n_in_tiles = ntiles;
    }
    if (p.in_tiles) {
        for (int e = (int)gtid; e < N; e += (int)gthreads) {
            const int n_e = off[e + 1] - off[e];
            int q = tstart[e];
            for (int r = 0; r < n_e; r += p.tile_rows, ++q)
                p.in_tiles[q] = make_int4(e, off[e] + r, min(p.tile_rows, n_e - r), 0);
        }
    }
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const unsigned lt = (1u << lane) - 1u;
        const int i0 = t0 * k, i1 = t1 * k;
        for (int c0 = i0; c0 < i1; c0 += 32) {
            const int i = c0 + lane;
            const bool valid = i < i1;
            const int e = valid ? p.topk_idx[i] : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int pos = valid ? cnt[e] + __popc(peers & lt) : 0;
            __syncwarp();
            if (valid && (__ffs(peers) - 1) == lane) cnt[e] += __popc(peers);
            __syncwarp();
            if (valid) {
                p.perm[pos] = i;
                if (p.row_pos) p.row_pos[i] = pos;
            }
        }
    }
    BFMOE_TRACE(0, threadIdx.x == 0, 5);
}

__host__ inline size_t route_smem_bytes(int N)
{
    const size_t ldl = N <= kThreadTopkMaxN ? N + 1 : N;
    const size_t a = (size_t)((N + 3) & ~3) * 4 + (size_t)route_batch_tokens(N) * ldl * 4;  // phase A
    const size_t c = (size_t)(((3 * N + 82 + 3) & ~3) + kHistStageInts) * 4;               // phase B/C
    return a > c ? a : c;
}

}  // namespace bfmoe
