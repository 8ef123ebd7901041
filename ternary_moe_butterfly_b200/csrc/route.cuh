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
//      logits are staged in shared memory and a group of lanes per token
//      selects the top-k; the block counts its rows per expert
//      (hist[block][e]) and keeps its rows' experts in shared memory.
//   B  up to 512 experts, every block reads the block-major histogram and
//      forms the expert totals and its own prefix over the blocks before it;
//      beyond, one warp per expert scans the column over the blocks and a
//      second grid barrier publishes the prefixes.
//   C  one warp per block scans the expert totals into bucket offsets, then
//      ranks the rows of the block's tokens inside their buckets (warp match
//      + popcount) and scatters perm / row_pos, and for the forward the
//      token and expert of every bucket row.
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
    uint32_t *sync;      // grid barrier counter (returned to zero by the last block to leave)
    uint32_t *departed;  // blocks done with the barrier counter
    unsigned long long *epoch;  // launch token of the last reset of the counters
    unsigned long long token;   // this launch's token
    uint32_t *status;
    int skip_arrive_block;  // test hook: this block never reaches barrier 1 (-1: none)
    int d;
    // forward only: the bucket rows' tokens and experts for the input butterfly
    int32_t *row_tok;    // [T*k] token of each bucket row, or null
    int32_t *row_exp;    // [T*k] expert of each bucket row, or null
    int clear_status;    // the routing starts the call: it clears the status word
};

// Histogram budget of the route kernel's shared memory, and the number of
// selected experts of its own rows a block keeps for the scatter.
constexpr int kSelCap = 2048;

// Staged logits per batch: 40 KB, or 120 KB above 128 experts (a block's
// token range then still fits in one batch at the usual sizes, so its
// loads take two rounds rather than two per batch).
__host__ __device__ constexpr int route_stage_ints(int N) { return N > 128 ? 30720 : 10240; }

// Padded shared-memory row of one token's logits when `grp` lanes share
// the token: rows G floats apart on top of a 32-float multiple put the group's
// reads on distinct banks.
__host__ __device__ inline int logit_row_stride(int N, int grp) { return grp < 32 ? ((N + 31) & ~31) + grp : N; }

// Tokens staged per batch: at most 256 and what the staging area holds at
// the widest row stride (16 lanes per token).
__host__ __device__ inline int route_batch_tokens(int N)
{
    const int b = route_stage_ints(N) / logit_row_stride(N, 16);
    return b < 1 ? 1 : (b > 256 ? 256 : b);
}

// (va, a) ranks before (vb, b)?  NaN has been mapped to -inf by the caller.
__device__ __forceinline__ bool ranks_before(float va, int a, float vb, int b)
{
    return va > vb || (va == vb && a < b);
}

// The barrier counters live in the caller's workspace and need no clearing
// between calls: the last block to leave a launch returns them to zero, and a
// launch whose token differs from the stored epoch (a fresh workspace, whose
// words may hold anything) has block 0 clear them and publish the token
// before any block arrives.
__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Block 0, thread 0, first thing: clear the counters if this launch's token
// is new to the workspace.
__device__ __forceinline__ void grid_epoch_open(uint32_t *ctr, uint32_t *departed, unsigned long long *epoch,
                                                unsigned long long token)
{
    if (ld_acquire_u64(epoch) != token) {
        atomicExch(ctr, 0u);
        atomicExch(departed, 0u);
        __threadfence();
        st_release_u64(epoch, token);
    }
}

// Thread 0 of every block, before arriving: wait (bounded) until the
// counters are known clear for this launch.
__device__ __forceinline__ bool grid_epoch_wait(const unsigned long long *epoch, unsigned long long token)
{
    if (ld_acquire_u64(epoch) == token) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (ld_acquire_u64(epoch) != token)
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    return true;
}

// Every block, once, after its last use of the counter (also on a timeout):
// the last one returns the counters to zero for the next launch.
__device__ __forceinline__ void grid_depart(uint32_t *ctr, uint32_t *departed, int nblk)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(departed, 1u) == (uint32_t)nblk - 1u) {
            atomicExch(ctr, 0u);
            atomicExch(departed, 0u);
        }
    }
}

// Split-phase grid-wide barrier on a monotonically increasing counter:
// arrive publishes the block's earlier writes; wait (bounded) returns false,
// block-uniformly, if the other blocks did not arrive in time.
__device__ __forceinline__ void grid_arrive(uint32_t *ctr)
{
    __syncthreads();
    // a release add: the block's earlier writes (ordered before this thread
    // by the barrier) become visible before the count does
    if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}

__device__ bool grid_wait(uint32_t *ctr, uint32_t target, uint32_t *status)
{
    __shared__ int ok;
    if (threadIdx.x == 0) {
        ok = 1;
        const unsigned long long t0 = globaltimer_ns();
        while (true) {
            uint32_t v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
            if (v >= target) break;  // the acquire orders the other blocks' writes before ours
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                set_status(status, BFMOE_ERR_TIMEOUT);
                ok = 0;
                break;
            }
        }
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

// Insert (v, e) into the sorted list of the K best (value, index) pairs.
template <int K>
__device__ __forceinline__ void topk_insert(float (&val)[K], int (&sel)[K], float v, int e)
{
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

// Top-K of one token by a group of `grp` lanes (a power of two <= 32,
// aligned inside the warp): lane s of the group keeps the sorted K best of
// experts s, s + grp, ...; the lists are merged across the group with xor
// shuffles (every lane of the warp takes part; `active` only gates the scan
// and the writes).  The order is total (value, then index), so the merged
// list is the exact top-K whatever the scan order.  Lane 0 of the group
// writes the indices and gates, counts the rows in the block histogram and
// keeps the indices in `keep` (when non-null).
template <int K>
__device__ __forceinline__ void topk_group(const RouteParams &p, int t, const float *l, int s, int grp, bool active,
                                           int *sh_hist, int *keep)
{
    float val[K];
    int sel[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
        val[j] = -INFINITY;
        sel[j] = 0x7fffffff;  // ranks after every real candidate
    }
    if (active)
        for (int e = s; e < p.N; e += grp) topk_insert<K>(val, sel, l[e], e);
    for (int off = 1; off < grp; off <<= 1) {
        float ov[K];
        int oe[K];
#pragma unroll
        for (int j = 0; j < K; ++j) {
            ov[j] = __shfl_xor_sync(0xffffffffu, val[j], off);
            oe[j] = __shfl_xor_sync(0xffffffffu, sel[j], off);
        }
#pragma unroll
        for (int j = 0; j < K; ++j) topk_insert<K>(val, sel, ov[j], oe[j]);
    }
    if (active && s == 0) {
        float g[K];
        gates_of(val, K, g);
#pragma unroll
        for (int j = 0; j < K; ++j) {
            p.topk_idx[(size_t)t * K + j] = sel[j];
            p.gates[(size_t)t * K + j] = g[j];
            atomicAdd(&sh_hist[sel[j]], 1);
            if (keep) keep[j] = sel[j];
        }
    }
}

// Top-k, gates and the histogram of the block's token range [t0, t1).
// Batches of tokens are staged in shared memory with coalesced 16-byte loads
// (one memory latency per batch; NaN becomes -inf and is reported); a group
// of lanes (as many as 256 threads allow per staged token, up to a warp)
// selects each token's experts.  `keep` (or null) receives the selected
// experts of the range's rows in row order.
__device__ void topk_range(const RouteParams &p, int t0, int t1, int *sh_hist, float *sh_logits, int *keep,
                           bool &saw_nan)
{
    const int N = p.N;
    const int want = max(1, min(t1 - t0, route_batch_tokens(N)));
    int grp = 1;
    while (grp < 32 && 2 * grp * want <= (int)blockDim.x) grp <<= 1;
    const int batch = min(want, (int)blockDim.x / grp);
    const int ldl = logit_row_stride(N, grp);
    for (int e = threadIdx.x; e < N; e += blockDim.x) sh_hist[e] = 0;
    const int q = threadIdx.x / grp, s = threadIdx.x % grp;
    for (int b0 = t0; b0 < t1; b0 += batch) {
        const int nb = min(batch, t1 - b0);
        const size_t nval = (size_t)nb * N;
        const float *src = p.logits + (size_t)b0 * N;
        __syncthreads();
        if ((N & 3) == 0 && (reinterpret_cast<uintptr_t>(p.logits) & 15) == 0) {
            const float4 *s4 = reinterpret_cast<const float4 *>(src);
            const int n4 = (int)(nval / 4);
            constexpr int kRound = 16;  // 16-byte loads in flight per thread
            for (int q0 = threadIdx.x; q0 < n4; q0 += kRound * blockDim.x) {
                float4 v[kRound];
#pragma unroll
                for (int u = 0; u < kRound; ++u) {
                    const int qq = q0 + u * blockDim.x;
                    if (qq < n4) v[u] = __ldg(s4 + qq);
                }
#pragma unroll
                for (int u = 0; u < kRound; ++u) {
                    const int qq = q0 + u * blockDim.x;
                    if (qq >= n4) break;
                    const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    const int tok = (4 * qq) / N, e0 = (4 * qq) % N;
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
            for (size_t qq = threadIdx.x; qq < nval; qq += blockDim.x) {
                float xv = __ldg(src + qq);
                if (xv != xv) {
                    saw_nan = true;
                    xv = -INFINITY;
                }
                sh_logits[(qq / N) * ldl + qq % N] = xv;
            }
        }
        __syncthreads();
        // threads beyond batch * grp (blockDim not a multiple) sit out whole warps
        if ((int)(threadIdx.x & ~31u) < batch * grp) {
            const bool active = q < nb;
            const int t = b0 + q;
            const float *l = sh_logits + (size_t)(active ? q : 0) * ldl;
            int *kp = (keep && active) ? keep + (size_t)(t - t0) * p.k : nullptr;
            switch (p.k) {
            case 1: topk_group<1>(p, t, l, s, grp, active, sh_hist, kp); break;
            case 2: topk_group<2>(p, t, l, s, grp, active, sh_hist, kp); break;
            case 3: topk_group<3>(p, t, l, s, grp, active, sh_hist, kp); break;
            case 4: topk_group<4>(p, t, l, s, grp, active, sh_hist, kp); break;
            case 5: topk_group<5>(p, t, l, s, grp, active, sh_hist, kp); break;
            case 6: topk_group<6>(p, t, l, s, grp, active, sh_hist, kp); break;
            case 7: topk_group<7>(p, t, l, s, grp, active, sh_hist, kp); break;
            default: topk_group<8>(p, t, l, s, grp, active, sh_hist, kp); break;
            }
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

// Partial sums of the histogram read, per half: parts * N <= 4 * threads
// (see the one-barrier read in k_route).
constexpr int kRouteRedInts = 4 * kRouteThreads;

// Shared-memory plan of the route kernel, in ints: the kept experts of the
// block's rows, then either phase A (histogram + staged logits, the latter
// 16-byte aligned) or phases B/C (offsets, bucket bases, partial sums).
struct RouteSmem {
    int keep, a_hist, a_logits, off, cnt, red, total;
    __host__ __device__ explicit RouteSmem(int N)
    {
        const int np4 = (N + 3) & ~3;
        keep = 0;
        a_hist = kSelCap;
        a_logits = a_hist + np4;
        const int a_end = a_logits + route_stage_ints(N);
        off = kSelCap;
        cnt = off + N + 1;
        red = cnt + N;
        const int c_end = red + 2 * kRouteRedInts;
        total = a_end > c_end ? a_end : c_end;
    }
};

__global__ void __launch_bounds__(kRouteThreads) k_route(RouteParams p)
{
    extern __shared__ __align__(16) int sh[];
    const int N = p.N, k = p.k;
    const int nblk = gridDim.x;  // one histogram row per block
    const RouteSmem lay(N);

    BFMOE_TRACE(0, threadIdx.x == 0, 0);
    pdl_wait();     // (launched after the previous call's kernels: they read this workspace)
    BFMOE_TRACE(0, threadIdx.x == 0, 11);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        // a new call's status; every other status write of this launch comes
        // after the grid barrier, which block 0 reaches after this store
        if (p.clear_status) *reinterpret_cast<volatile uint32_t *>(p.status) = 0u;
        grid_epoch_open(p.sync, p.departed, p.epoch, p.token);
    }
    // ---- phase A: top-k over this block's token range
    bool saw_nan = false;
    const int tpb = (p.T + nblk - 1) / nblk;  // tokens per block
    const int t0 = min(p.T, (int)blockIdx.x * tpb), t1 = min(p.T, t0 + tpb);
    const bool kept = (t1 - t0) * k <= kSelCap;  // the scatter reads the experts from shared memory
    int *keep = kept ? sh + lay.keep : nullptr;
    int *hist_a = sh + lay.a_hist;
    topk_range(p, t0, t1, hist_a, reinterpret_cast<float *>(sh + lay.a_logits), keep, saw_nan);
    const bool one_barrier = N <= kOneBarrierMaxN;  // one grid barrier
    const int np4 = (N + 3) & ~3;                    // histogram row stride, 16-byte multiple
    for (int e = threadIdx.x; e < N; e += blockDim.x)
        p.hist[(size_t)blockIdx.x * (one_barrier ? np4 : N) + e] = hist_a[e];
    const bool nan_here = __syncthreads_or(saw_nan);
    BFMOE_TRACE(0, threadIdx.x == 0, 1);
    const bool arrive = (int)blockIdx.x != p.skip_arrive_block;  // test hook: one block never arrives
    {
        __shared__ int epoch_ok;
        if (threadIdx.x == 0) epoch_ok = grid_epoch_wait(p.epoch, p.token) ? 1 : 0;
        __syncthreads();
        if (!epoch_ok) {
            if (threadIdx.x == 0) set_status(p.status, BFMOE_ERR_TIMEOUT);
            grid_depart(p.sync, p.departed, nblk);
            return;
        }
    }
    if (arrive) grid_arrive(p.sync);

    const size_t gtid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t gthreads = (size_t)gridDim.x * blockDim.x;
    BFMOE_TRACE(0, threadIdx.x == 0, 2);
    if (!arrive) {
        grid_depart(p.sync, p.departed, nblk);
        return;
    }
    const bool one_ok = grid_wait(p.sync, nblk, p.status);
    if (one_ok && one_barrier) grid_depart(p.sync, p.departed, nblk);  // the only barrier is behind us
    if (!one_ok) {
        grid_depart(p.sync, p.departed, nblk);
        return;
    }
    // the input-butterfly kernel may become resident now (earlier, its
    // blocks would crowd the routing's)
    pdl_trigger();
    if (nan_here && threadIdx.x == 0) set_status(p.status, BFMOE_ERR_NONFINITE);
    BFMOE_TRACE(0, threadIdx.x == 0, 3);

    int *off = sh + lay.off;        // [N+1]
    int *cnt = sh + lay.cnt;        // [N]
    if (one_barrier) {
        // ---- every block: expert totals and its own prefix over the blocks
        // before it, straight from the block-major histogram: `parts`
        // threads per expert (or per 4 experts, with 16-byte loads when N is
        // a multiple of 4: the rows are then 16-byte aligned and unpadded)
        // take every parts-th row, many loads in flight per thread.
        // parts * N <= 4 * blockDim.x either way.
        int *red = sh + lay.red;  // [2][parts * N]
        const bool by4 = (N & 3) == 0 && (reinterpret_cast<uintptr_t>(p.hist) & 15) == 0;
        const int cols = by4 ? N >> 2 : N;
        const int parts = max(1, (int)blockDim.x / cols);
        if (by4) {
            const int4 *h4 = reinterpret_cast<const int4 *>(p.hist);
            for (int idx = threadIdx.x; idx < parts * cols; idx += blockDim.x) {
                const int c = idx % cols, part = idx / cols;
                int4 tot = make_int4(0, 0, 0, 0), pre = make_int4(0, 0, 0, 0);
                for (int b0 = part; b0 < nblk; b0 += 16 * parts) {
                    int4 v[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int b = b0 + u * parts;
                        v[u] = b < nblk ? __ldcg(h4 + (size_t)b * cols + c) : make_int4(0, 0, 0, 0);
                    }
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        tot.x += v[u].x, tot.y += v[u].y, tot.z += v[u].z, tot.w += v[u].w;
                        if (b0 + u * parts < (int)blockIdx.x)
                            pre.x += v[u].x, pre.y += v[u].y, pre.z += v[u].z, pre.w += v[u].w;
                    }
                }
                int *rt = red + part * N + 4 * c, *rp = rt + parts * N;
                rt[0] = tot.x, rt[1] = tot.y, rt[2] = tot.z, rt[3] = tot.w;
                rp[0] = pre.x, rp[1] = pre.y, rp[2] = pre.z, rp[3] = pre.w;
            }
        } else {
            for (int idx = threadIdx.x; idx < parts * N; idx += blockDim.x) {
                const int e = idx % N, part = idx / N;
                int tot = 0, pre = 0;
                for (int b0 = part; b0 < nblk; b0 += 32 * parts) {
                    int v[32];
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const int b = b0 + u * parts;
                        v[u] = b < nblk ? __ldcg(p.hist + (size_t)b * np4 + e) : 0;
                    }
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        tot += v[u];
                        pre += (b0 + u * parts < (int)blockIdx.x) ? v[u] : 0;
                    }
                }
                red[idx] = tot;
                red[parts * N + idx] = pre;
            }
        }
        __syncthreads();
        BFMOE_TRACE(0, threadIdx.x == 0, 6);
        for (int e = threadIdx.x; e < N; e += blockDim.x) {
            int tot = 0, pre = 0;
            for (int q = 0; q < parts; ++q) {
                tot += red[q * N + e];
                pre += red[parts * N + q * N + e];
            }
            off[e] = tot;  // scanned into bucket offsets below
            cnt[e] = pre;  // becomes the block's bucket base below
        }
        __syncthreads();
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
        const bool two_ok = grid_wait(p.sync, 2 * nblk, p.status);
        grid_depart(p.sync, p.departed, nblk);
        if (!two_ok) return;
        for (int e = threadIdx.x; e < N; e += blockDim.x) {
            off[e] = p.total[e];
            cnt[e] = p.hist[(size_t)blockIdx.x * N + e];
        }
        __syncthreads();
    }
    BFMOE_TRACE(0, threadIdx.x == 0, 4);

    // ---- phase C: bucket offsets and bucket bases by one warp (lane-serial
    // chunks + a shuffle scan), then ranks and scatter
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int per = (N + 31) / 32;
        const int lo = min(N, lane * per), hi = min(N, lo + per);
        int srow = 0;
        for (int e = lo; e < hi; ++e) srow += off[e];
        int irow = srow;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int a = __shfl_up_sync(0xffffffffu, irow, o);
            if (lane >= o) irow += a;
        }
        int run = irow - srow;
        for (int e = lo; e < hi; ++e) {
            const int n = off[e];
            off[e] = run;
            cnt[e] += run;
            run += n;
        }
        if (lane == 31) off[N] = irow;
    }
    __syncthreads();
    BFMOE_TRACE(0, threadIdx.x == 0, 8);
    if (blockIdx.x == 0)
        for (int e = threadIdx.x; e <= N; e += blockDim.x) p.offsets[e] = off[e];
    if (threadIdx.x < 32) {
        // one warp ranks the block's rows in row order: stable inside buckets
        const int lane = threadIdx.x;
        const unsigned lt = (1u << lane) - 1u;
        const int i0 = t0 * k, i1 = t1 * k;
        for (int c0 = i0; c0 < i1; c0 += 32) {
            const int i = c0 + lane;
            const bool valid = i < i1;
            const int e = valid ? (kept ? keep[i - i0] : p.topk_idx[i]) : -1;
            const unsigned peers = __match_any_sync(0xffffffffu, e);
            const int pos = valid ? cnt[e] + __popc(peers & lt) : 0;
            __syncwarp();
            if (valid && (__ffs(peers) - 1) == lane) cnt[e] += __popc(peers);
            __syncwarp();
            if (valid) {
                p.perm[pos] = i;
                if (p.row_pos) p.row_pos[i] = pos;
                if (p.row_tok) {
                    p.row_tok[pos] = i / k;
                    p.row_exp[pos] = e;
                }
            }
        }
    }
    BFMOE_TRACE(0, threadIdx.x == 0, 5);
}

__host__ inline size_t route_smem_bytes(int N) { return (size_t)RouteSmem(N).total * 4; }

}  // namespace bfmoe
