// bfmoe.cu -- the C ABI: argument checks, workspace layout and kernel
// launches on the caller's stream.  The declarations and the contract of
// every entry point are in include/bfmoe.h.
#include <cuda_runtime.h>

#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "layer.cuh"
#include "route.cuh"

using namespace bfmoe;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool is_pow2(int d) { return d > 0 && (d & (d - 1)) == 0; }

int ilog2(int d)
{
    int L = 0;
    while ((1 << L) < d) ++L;
    return L;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// Width, expert and top-k limits shared by every entry point.
bfmoe_status check_d(int d)
{
    if (d <= 0) return BFMOE_ERR_INVALID_ARG;
    if (!is_pow2(d)) return BFMOE_ERR_INVALID_ARG;
    if (d < 64 || d > 4096) return BFMOE_ERR_UNSUPPORTED;
    return BFMOE_OK;
}

bfmoe_status check_route_shape(int T, int N, int k)
{
    if (T <= 0 || N <= 0 || k <= 0 || k > N) return BFMOE_ERR_INVALID_ARG;
    if (N > 4096 || k > kMaxK) return BFMOE_ERR_UNSUPPORTED;
    if ((long long)T * k > (1ll << 24)) return BFMOE_ERR_UNSUPPORTED;
    return BFMOE_OK;
}

int route_blocks(int T) { return (T + kRouteTokensPerBlock - 1) / kRouteTokensPerBlock; }

struct RouteLayout {
    size_t status, hist, total;
};

RouteLayout route_layout(int T, int N)
{
    RouteLayout l{};
    size_t o = 0;
    l.status = o;
    o += kAlign;
    l.hist = o;
    o += align_up((size_t)route_blocks(T) * N * 4);
    l.total = o;
    return l;
}

struct FwdLayout {
    size_t status, topk_idx, gates, perm, row_pos, offsets, hist, coef_t, coef_p, wdec, a_blocks, z, total;
};

int padded_rows(int T, int k) { return (T * k + kBM - 1) / kBM * kBM; }

FwdLayout fwd_layout(int T, int d, int N, int k)
{
    FwdLayout l{};
    const size_t R = (size_t)T * k, Rp = (size_t)padded_rows(T, k);
    const size_t ncoef = (size_t)N * ilog2(d) * (d / 2);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += align_up(bytes);
        return at;
    };
    l.status = take(16);
    l.topk_idx = take(R * 4);
    l.gates = take(R * 4);
    l.perm = take(R * 4);
    l.row_pos = take(R * 4);
    l.offsets = take(((size_t)N + 1) * 4);
    l.hist = take((size_t)route_blocks(T) * N * 4);
    l.coef_t = take(ncoef * 8);
    l.coef_p = take(ncoef * 8);
    l.wdec = take((size_t)d * d * 2);
    l.a_blocks = take(Rp * d * 2);
    l.z = take(Rp * d * 4);
    l.total = o;
    return l;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per
// (device, kernel, size).
std::mutex g_attr_mu;
std::map<std::pair<int, const void *>, size_t> g_attr;

bool ensure_smem(const void *fn, size_t bytes)
{
    if (bytes <= 48 * 1024) return true;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> g(g_attr_mu);
    auto key = std::make_pair(dev, fn);
    auto it = g_attr.find(key);
    if (it != g_attr.end() && it->second >= bytes) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    g_attr[key] = bytes;
    return true;
}

bfmoe_status launched()
{
    return cudaGetLastError() == cudaSuccess ? BFMOE_OK : BFMOE_ERR_CUDA;
}

// Routing launches shared by bfmoe_route and bfmoe_forward.
struct StageRec;
void mark(StageRec *r, cudaStream_t st);

bfmoe_status launch_route(const float *logits, int T, int N, int k, int32_t *idx, float *gates, int32_t *perm,
                          int32_t *offsets, int32_t *row_pos, int32_t *hist, uint32_t *status, cudaStream_t st,
                          StageRec *rec = nullptr)
{
    const int nblk = route_blocks(T);
    if (!ensure_smem((const void *)k_bucket_scan, (size_t)(N + 1024) * 4)) return BFMOE_ERR_CUDA;
    k_topk<<<nblk, kRouteThreads, (size_t)N * 4, st>>>(logits, T, N, k, idx, gates, hist, status);
    mark(rec, st);
    k_bucket_scan<<<1, 1024, (size_t)(N + 1024) * 4, st>>>(hist, nblk, N, offsets);
    mark(rec, st);
    k_bucket_scatter<<<nblk, kRouteThreads, (size_t)N * 4, st>>>(idx, hist, T, N, k, perm, row_pos);
    mark(rec, st);
    return launched();
}

// Optional per-kernel event recorder used by bfmoe_forward_profile.
struct StageRec {
    cudaEvent_t ev[BFMOE_MAX_STAGES + 1];
    int n = 0;
    bool on = false;
};

const char *const kStageNames[] = {"coef", "decode_base", "route_topk", "route_scan", "route_scatter",
                                   "expert_in", "contract", "expert_out"};
constexpr int kNumStages = 8;

void mark(StageRec *r, cudaStream_t st)
{
    if (r && r->on && r->n <= BFMOE_MAX_STAGES) cudaEventRecord(r->ev[r->n++], st);
}

template <typename T>
bfmoe_status launch_layer(const void *x, int T_, int d, int N, int k, const void *packed, const float *theta,
                          const float *phi, void *y, uint8_t *ws, const FwdLayout &l, const float *logits,
                          cudaStream_t st, StageRec *rec = nullptr)
{
    const int L = ilog2(d);
    const int R = T_ * k, Rp = padded_rows(T_, k);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws + l.status);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + l.topk_idx);
    float *gates = reinterpret_cast<float *>(ws + l.gates);
    int32_t *perm = reinterpret_cast<int32_t *>(ws + l.perm);
    int32_t *row_pos = reinterpret_cast<int32_t *>(ws + l.row_pos);
    int32_t *offsets = reinterpret_cast<int32_t *>(ws + l.offsets);
    int32_t *hist = reinterpret_cast<int32_t *>(ws + l.hist);
    float2 *ct = reinterpret_cast<float2 *>(ws + l.coef_t);
    float2 *cp = reinterpret_cast<float2 *>(ws + l.coef_p);
    __half *wdec = reinterpret_cast<__half *>(ws + l.wdec);
    __half *ablk = reinterpret_cast<__half *>(ws + l.a_blocks);
    float *z = reinterpret_cast<float *>(ws + l.z);

    if (cudaMemsetAsync(status, 0, 4, st) != cudaSuccess) return BFMOE_ERR_CUDA;
    mark(rec, st);
    const int ncoef = N * L * (d / 2);
    k_coef<<<(2 * ncoef + 255) / 256, 256, 0, st>>>(theta, phi, ncoef, ct, cp);
    mark(rec, st);
    const size_t nchunks = (size_t)d * d / 8;
    k_decode_base<<<(unsigned)((nchunks + 255) / 256), 256, 0, st>>>(reinterpret_cast<const uint32_t *>(packed), d,
                                                                       wdec, status);
    mark(rec, st);
    bfmoe_status s = launch_route(logits, T_, N, k, idx, gates, perm, offsets, row_pos, hist, status, st, rec);
    if (s != BFMOE_OK) return s;

    const int RT = tile_rows_for(d);
    const size_t in_smem = rows_smem_bytes(d, 2);
    if (!ensure_smem((const void *)k_expert_in<T>, in_smem)) return BFMOE_ERR_CUDA;
    k_expert_in<T><<<Rp / RT, 256, in_smem, st>>>(reinterpret_cast<const T *>(x), d, L, k, R, perm, idx, ct, ablk,
                                                  status);
    mark(rec, st);

    const size_t c_smem = contract_smem_bytes(d);
    if (!ensure_smem((const void *)k_contract, c_smem)) return BFMOE_ERR_CUDA;
    dim3 cgrid(Rp / kBM, d / gemm_bn(d));
    k_contract<<<cgrid, 128, c_smem, st>>>(ablk, wdec, z, d, status);
    mark(rec, st);

    const int TT = RT / k > 0 ? RT / k : 1;
    const size_t out_smem = (size_t)TT * k * (d + 1) * 4 + (size_t)TT * k * 12;
    if (!ensure_smem((const void *)k_expert_out<T>, out_smem)) return BFMOE_ERR_CUDA;
    k_expert_out<T><<<(T_ + TT - 1) / TT, 256, out_smem, st>>>(z, d, L, T_, k, row_pos, idx, gates, cp,
                                                              reinterpret_cast<const uint32_t *>(packed),
                                                              reinterpret_cast<T *>(y));
    mark(rec, st);
    return launched();
}

}  // namespace

extern "C" {

const char *bfmoe_status_string(bfmoe_status s)
{
    switch (s) {
    case BFMOE_OK: return "ok";
    case BFMOE_ERR_INVALID_ARG: return "invalid argument";
    case BFMOE_ERR_UNSUPPORTED: return "unsupported size";
    case BFMOE_ERR_WORKSPACE: return "workspace too small";
    case BFMOE_ERR_NONFINITE: return "non-finite value";
    case BFMOE_ERR_TIMEOUT: return "device wait timed out";
    case BFMOE_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

int bfmoe_version(void) { return 100; }

size_t bfmoe_packed_base_bytes(int d)
{
    if (check_d(d) != BFMOE_OK) return 0;
    return 16 + (size_t)d * d / 4;
}

bfmoe_status bfmoe_pack_base(const int8_t *w, int d, float alpha, void *packed, void *stream)
{
    bfmoe_status s = check_d(d);
    if (s != BFMOE_OK) return s;
    if (!w || !packed || !aligned(w, 16) || !aligned(packed, 16)) return BFMOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    uint32_t *hdr = reinterpret_cast<uint32_t *>(packed);
    if (cudaMemsetAsync(hdr, 0, 16, st) != cudaSuccess) return BFMOE_ERR_CUDA;
    const size_t nwords = (size_t)d * d / 16;
    k_pack_base<<<(unsigned)((nwords + 255) / 256), 256, 0, st>>>(w, d, hdr + 4, hdr + 3);
    if (launched() != BFMOE_OK) return BFMOE_ERR_CUDA;
    uint32_t bad = 0;
    if (cudaMemcpyAsync(&bad, hdr + 3, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return BFMOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BFMOE_ERR_CUDA;
    if (bad) return BFMOE_ERR_INVALID_ARG;
    uint32_t h[4];
    h[0] = kPackMagic;
    h[1] = (uint32_t)d;
    memcpy(&h[2], &alpha, 4);
    h[3] = 1u;
    if (cudaMemcpyAsync(hdr, h, 16, cudaMemcpyHostToDevice, st) != cudaSuccess) return BFMOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BFMOE_ERR_CUDA;
    return BFMOE_OK;
}

size_t bfmoe_route_workspace_bytes(int T, int N, int k)
{
    if (check_route_shape(T, N, k) != BFMOE_OK) return 0;
    return route_layout(T, N).total;
}

bfmoe_status bfmoe_route(const float *logits, int T, int N, int k, int32_t *topk_idx, float *gates, int32_t *perm,
                         int32_t *offsets, void *ws, size_t ws_bytes, void *stream)
{
    bfmoe_status s = check_route_shape(T, N, k);
    if (s != BFMOE_OK) return s;
    if (!logits || !topk_idx || !gates || !perm || !offsets || !ws) return BFMOE_ERR_INVALID_ARG;
    if (!aligned(ws, kAlign) || !aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(gates, 4) ||
        !aligned(perm, 4) || !aligned(offsets, 4))
        return BFMOE_ERR_INVALID_ARG;
    const RouteLayout l = route_layout(T, N);
    if (ws_bytes < l.total) return BFMOE_ERR_WORKSPACE;
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    cudaStream_t st = as_stream(stream);
    uint32_t *status = reinterpret_cast<uint32_t *>(w + l.status);
    if (cudaMemsetAsync(status, 0, 4, st) != cudaSuccess) return BFMOE_ERR_CUDA;
    return launch_route(logits, T, N, k, topk_idx, gates, perm, offsets, nullptr,
                        reinterpret_cast<int32_t *>(w + l.hist), status, st);
}

size_t bfmoe_butterfly_workspace_bytes(int d, int N)
{
    if (check_d(d) != BFMOE_OK || N <= 0 || N > 4096) return 0;
    return kAlign + align_up((size_t)N * ilog2(d) * (d / 2) * 8);
}

bfmoe_status bfmoe_butterfly_apply(const void *x, bfmoe_dtype dt, int rows, int d, int N, const float *angles,
                                   const int32_t *expert_of_row, int transpose, void *y, void *ws, size_t ws_bytes,
                                   void *stream)
{
    bfmoe_status s = check_d(d);
    if (s != BFMOE_OK) return s;
    if (rows < 0 || N <= 0) return BFMOE_ERR_INVALID_ARG;
    if (N > 4096) return BFMOE_ERR_UNSUPPORTED;
    if (dt != BFMOE_F32 && dt != BFMOE_BF16) return BFMOE_ERR_INVALID_ARG;
    if (!angles || !ws || (rows > 0 && (!x || !y))) return BFMOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ws, kAlign) || !aligned(angles, 4) ||
        !aligned(expert_of_row, 4))
        return BFMOE_ERR_INVALID_ARG;
    if (x == y && rows > 0) return BFMOE_ERR_INVALID_ARG;
    if (ws_bytes < bfmoe_butterfly_workspace_bytes(d, N)) return BFMOE_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    uint32_t *status = reinterpret_cast<uint32_t *>(w);
    float2 *coef = reinterpret_cast<float2 *>(w + kAlign);
    if (cudaMemsetAsync(status, 0, 4, st) != cudaSuccess) return BFMOE_ERR_CUDA;
    if (rows == 0) return BFMOE_OK;
    const int L = ilog2(d);
    const int ncoef = N * L * (d / 2);
    k_coef<<<(ncoef + 255) / 256, 256, 0, st>>>(angles, nullptr, ncoef, coef, nullptr);
    const int RT = tile_rows_for(d);
    const size_t smem = rows_smem_bytes(d, 1);
    const unsigned grid = (unsigned)((rows + RT - 1) / RT);
    if (dt == BFMOE_F32) {
        if (!ensure_smem((const void *)k_bfly_apply<float>, smem)) return BFMOE_ERR_CUDA;
        k_bfly_apply<float><<<grid, 256, smem, st>>>(reinterpret_cast<const float *>(x), rows, d, L, expert_of_row,
                                                     coef, transpose, reinterpret_cast<float *>(y), N, status);
    } else {
        if (!ensure_smem((const void *)k_bfly_apply<__nv_bfloat16>, smem)) return BFMOE_ERR_CUDA;
        k_bfly_apply<__nv_bfloat16><<<grid, 256, smem, st>>>(reinterpret_cast<const __nv_bfloat16 *>(x), rows, d,
                                                             L, expert_of_row, coef, transpose,
                                                             reinterpret_cast<__nv_bfloat16 *>(y), N, status);
    }
    return launched();
}

size_t bfmoe_forward_workspace_bytes(int T, int d, int N, int k)
{
    if (check_d(d) != BFMOE_OK || check_route_shape(T, N, k) != BFMOE_OK) return 0;
    return fwd_layout(T, d, N, k).total;
}

bfmoe_status bfmoe_forward_ws_layout(int T, int d, int N, int k, bfmoe_ws_layout *out)
{
    bfmoe_status s = check_d(d);
    if (s != BFMOE_OK) return s;
    s = check_route_shape(T, N, k);
    if (s != BFMOE_OK) return s;
    if (!out) return BFMOE_ERR_INVALID_ARG;
    const FwdLayout l = fwd_layout(T, d, N, k);
    out->status = l.status;
    out->topk_idx = l.topk_idx;
    out->gates = l.gates;
    out->perm = l.perm;
    out->offsets = l.offsets;
    out->total = l.total;
    return BFMOE_OK;
}

static bfmoe_status forward_impl(const void *x, bfmoe_dtype dt, int T, int d, const float *logits, int N, int k,
                                 const void *packed_base, const float *theta, const float *phi, void *y, void *ws,
                                 size_t ws_bytes, void *stream, StageRec *rec)
{
    bfmoe_status s = check_d(d);
    if (s != BFMOE_OK) return s;
    s = check_route_shape(T, N, k);
    if (s != BFMOE_OK) return s;
    if (dt != BFMOE_F32 && dt != BFMOE_BF16) return BFMOE_ERR_INVALID_ARG;
    if (!x || !logits || !packed_base || !theta || !phi || !y || !ws) return BFMOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ws, kAlign) || !aligned(packed_base, 16) ||
        !aligned(logits, 4) || !aligned(theta, 4) || !aligned(phi, 4))
        return BFMOE_ERR_INVALID_ARG;
    if (x == y) return BFMOE_ERR_INVALID_ARG;
    const FwdLayout l = fwd_layout(T, d, N, k);
    if (ws_bytes < l.total) return BFMOE_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    if (dt == BFMOE_F32) return launch_layer<float>(x, T, d, N, k, packed_base, theta, phi, y, w, l, logits, st, rec);
    return launch_layer<__nv_bfloat16>(x, T, d, N, k, packed_base, theta, phi, y, w, l, logits, st, rec);
}

bfmoe_status bfmoe_forward(const void *x, bfmoe_dtype dt, int T, int d, const float *logits, int N, int k,
                           const void *packed_base, const float *theta, const float *phi, void *y, void *ws,
                           size_t ws_bytes, void *stream)
{
    return forward_impl(x, dt, T, d, logits, N, k, packed_base, theta, phi, y, ws, ws_bytes, stream, nullptr);
}

bfmoe_status bfmoe_forward_profile(const void *x, bfmoe_dtype dt, int T, int d, const float *logits, int N, int k,
                                   const void *packed_base, const float *theta, const float *phi, void *y, void *ws,
                                   size_t ws_bytes, void *stream, float *stage_ms, int *n_stages)
{
    if (!stage_ms || !n_stages) return BFMOE_ERR_INVALID_ARG;
    StageRec rec;
    for (int i = 0; i <= BFMOE_MAX_STAGES; ++i)
        if (cudaEventCreate(&rec.ev[i]) != cudaSuccess) {
            for (int j = 0; j < i; ++j) cudaEventDestroy(rec.ev[j]);
            return BFMOE_ERR_CUDA;
        }
    rec.on = true;
    bfmoe_status s = forward_impl(x, dt, T, d, logits, N, k, packed_base, theta, phi, y, ws, ws_bytes, stream, &rec);
    if (s == BFMOE_OK && cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) s = BFMOE_ERR_CUDA;
    *n_stages = 0;
    if (s == BFMOE_OK) {
        for (int i = 0; i + 1 < rec.n; ++i) {
            float ms = 0.0f;
            cudaEventElapsedTime(&ms, rec.ev[i], rec.ev[i + 1]);
            stage_ms[i] = ms;
        }
        *n_stages = rec.n > 0 ? rec.n - 1 : 0;
    }
    for (int i = 0; i <= BFMOE_MAX_STAGES; ++i) cudaEventDestroy(rec.ev[i]);
    return s;
}

const char *bfmoe_stage_name(int i) { return (i >= 0 && i < kNumStages) ? kStageNames[i] : nullptr; }

bfmoe_status bfmoe_sync_status(void *ws, void *stream)
{
    if (!ws) return BFMOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return BFMOE_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return BFMOE_ERR_CUDA;
    if (v != 0 && cudaMemset(ws, 0, 4) != cudaSuccess) return BFMOE_ERR_CUDA;
    if (v > (uint32_t)BFMOE_ERR_CUDA) return BFMOE_ERR_CUDA;
    return (bfmoe_status)v;
}

}  // extern "C"
