// route.cuh -- top-k gate over given router logits and deterministic
// bucketing of the routed rows by expert.
//
// A standard top-k gate selects each token's active experts (ButterflyMoE
// summary, Dutch page, section 2 "Three phases", gated routing).  Order:
// larger logit first, ties to the lower expert index; gate = softmax over
// the k selected logits.  Bucketing is a stable counting sort of the rows
// i = t*k + j by expert, so each bucket lists its rows in token order.
//
// Three launches: (1) one warp per token selects the top-k and counts the
// block's rows per expert; (2) one block turns the per-block counts into
// bucket offsets and per-block bases; (3) per block, one warp ranks the
// block's rows inside their buckets (warp match + popcount) and scatters.
#pragma once

#include "common.cuh"

namespace bfmoe {

constexpr int kRouteThreads = 256;
constexpr int kRouteTokensPerBlock = 64;  // 8 warps x 8 tokens
constexpr int kMaxK = 8;

// (va, a) ranks before (vb, b)?  NaN has been mapped to -inf by the caller.
__device__ __forceinline__ bool ranks_before(float va, int a, float vb, int b)
{
    return va > vb || (va == vb && a < b);
}

__global__ void __launch_bounds__(kRouteThreads) k_topk(const float *__restrict__ logits, int T, int N, int k,
                                                        int32_t *__restrict__ topk_idx,
                                                        float *__restrict__ gates, int32_t *__restrict__ hist,
                                                        uint32_t *status)
{
    extern __shared__ int sh_hist[];  // [N]
    for (int e = threadIdx.x; e < N; e += blockDim.x) sh_hist[e] = 0;
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tok0 = blockIdx.x * kRouteTokensPerBlock + warp * (kRouteTokensPerBlock / 8);
    bool saw_nan = false;
    for (int q = 0; q < kRouteTokensPerBlock / 8; ++q) {
        const int t = tok0 + q;
        if (t >= T) break;
        const float *l = logits + (size_t)t * N;
        int sel[kMaxK];
        float val[kMaxK];
        for (int j = 0; j < k; ++j) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
            for (int e = lane; e < N; e += 32) {
                bool taken = false;
                for (int jj = 0; jj < j; ++jj) taken |= (sel[jj] == e);
                if (taken) continue;
                float v = __ldg(l + e);
                if (v != v) {
                    saw_nan = true;
                    v = -INFINITY;
                }
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
            const float m = val[0];
            if (m == INFINITY) {
                int c = 0;
                for (int j = 0; j < k; ++j) c += (val[j] == INFINITY);
                for (int j = 0; j < k; ++j) g[j] = (val[j] == INFINITY) ? 1.0f / (float)c : 0.0f;
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
            for (int j = 0; j < k; ++j) {
                topk_idx[(size_t)t * k + j] = sel[j];
                gates[(size_t)t * k + j] = g[j];
                atomicAdd(&sh_hist[sel[j]], 1);
            }
        }
    }
    if (__any_sync(0xffffffffu, saw_nan) && lane == 0) set_status(status, BFMOE_ERR_NONFINITE);
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += blockDim.x) hist[(size_t)blockIdx.x * N + e] = sh_hist[e];
}

// One block: base[b][e] = offsets[e] + sum_{b' < b} hist[b'][e] (in place),
// offsets[e] = sum_{e' < e} total[e'], offsets[N] = R.
__global__ void __launch_bounds__(1024) k_bucket_scan(int32_t *__restrict__ hist_base, int nblk, int N,
                                                      int32_t *__restrict__ offsets)
{
    extern __shared__ int sh[];  // total[N] then scratch[1024]
    int *total = sh;
    int *part = sh + N;
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        int run = 0;
        for (int b = 0; b < nblk; ++b) {
            const int h = hist_base[(size_t)b * N + e];
            hist_base[(size_t)b * N + e] = run;
            run += h;
        }
        total[e] = run;
    }
    __syncthreads();
    // exclusive scan of total[0..N) with 1024 threads, ceil(N/1024) items each
    const int per = (N + blockDim.x - 1) / blockDim.x;
    const int lo = threadIdx.x * per, hi = min(N, lo + per);
    int s = 0;
    for (int e = lo; e < hi; ++e) s += total[e];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int off = 1; off < (int)blockDim.x; off <<= 1) {
        const int v = (threadIdx.x >= (unsigned)off) ? part[threadIdx.x - off] : 0;
        __syncthreads();
        part[threadIdx.x] += v;
        __syncthreads();
    }
    int run = part[threadIdx.x] - s;  // exclusive prefix of this thread's range
    for (int e = lo; e < hi; ++e) {
        const int t = total[e];
        total[e] = run;
        run += t;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += blockDim.x) offsets[e] = total[e];
    if (threadIdx.x == blockDim.x - 1) offsets[N] = part[blockDim.x - 1];
    for (int e = threadIdx.x; e < N; e += blockDim.x) {
        const int o = total[e];
        for (int b = 0; b < nblk; ++b) hist_base[(size_t)b * N + e] += o;
    }
}

// Per block (same token partition as k_topk): rank the block's rows inside
// their buckets in row order and scatter perm / row_pos.
__global__ void __launch_bounds__(kRouteThreads) k_bucket_scatter(const int32_t *__restrict__ topk_idx,
                                                                  const int32_t *__restrict__ base, int T, int N,
                                                                  int k, int32_t *__restrict__ perm,
                                                                  int32_t *__restrict__ row_pos)
{
    extern __shared__ int cnt[];  // [N]
    for (int e = threadIdx.x; e < N; e += blockDim.x) cnt[e] = base[(size_t)blockIdx.x * N + e];
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    const int t0 = blockIdx.x * kRouteTokensPerBlock;
    const int t1 = min(T, t0 + kRouteTokensPerBlock);
    const int i0 = t0 * k, i1 = t1 * k;
    const unsigned lt = (1u << lane) - 1u;
    for (int c0 = i0; c0 < i1; c0 += 32) {
        const int i = c0 + lane;
        const bool valid = i < i1;
        const int e = valid ? topk_idx[i] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int pos = valid ? cnt[e] + __popc(peers & lt) : 0;
        __syncwarp();
        if (valid && (__ffs(peers) - 1) == lane) cnt[e] += __popc(peers);
        __syncwarp();
        if (valid) {
            perm[pos] = i;
            if (row_pos) row_pos[i] = pos;
        }
    }
}

}  // namespace bfmoe
