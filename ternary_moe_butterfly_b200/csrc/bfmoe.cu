// bfmoe.cu -- the C ABI: argument checks, workspace layout and kernel
// launches on the caller's stream.  The declarations and the contract of
// every entry point are in include/bfmoe.h.
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <map>
#include <random>
#include <mutex>
#include <utility>

#include <algorithm>

#include "contract.cuh"
#include "layer.cuh"
#include "prep.cuh"
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

// Rows of the per-block histogram (the routing grid never exceeds it).
int route_chunks(int) { return kMaxRouteBlocks; }

// Every workspace opens with the 32-byte header (status word, grid-barrier
// and departure counters, launch epoch) in its first aligned slot; the
// barrier words clear themselves, so no call issues a memset.
struct RouteLayout {
    size_t status, hist, total, total_bytes;
};

RouteLayout route_layout(int T, int N)
{
    RouteLayout l{};
    size_t o = 0;
    l.status = o;
    o += kAlign;
    l.hist = o;
    o += align_up((size_t)route_chunks(T) * N * 4);
    l.total = o;
    o += align_up((size_t)N * 4);
    l.total_bytes = o;
    return l;
}

struct FwdLayout {
    size_t status, topk_idx, gates, perm, offsets, hist, total, row_tok, row_exp, coef_t, coef_p, wdec, a_blocks,
        slot, total_bytes;
};

int padded_rows(int T, int k) { return (T * k + kBM - 1) / kBM * kBM; }
int in_tiles(int T, int d, int k) { return (T * k + tile_rows_for(d) - 1) / tile_rows_for(d); }

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
    l.status = take(32);
    l.topk_idx = take(R * 4);
    l.gates = take(R * 4);
    l.perm = take(R * 4);
    l.offsets = take(((size_t)N + 1) * 4);
    l.hist = take((size_t)route_chunks(T) * N * 4);
    l.total = take((size_t)N * 4);
    l.row_tok = take(R * 4);
    l.row_exp = take(R * 4);
    l.coef_t = take(ncoef * 8);
    l.coef_p = take(ncoef * 8);
    l.wdec = take((size_t)d * d * 2);
    l.a_blocks = take(Rp * d * 2);
    l.slot = take(R * d * 2);
    l.total_bytes = o;
    return l;
}

// Per-device facts and per-(device, kernel, smem) attributes, cached.
std::mutex g_mu;
std::map<std::pair<int, const void *>, size_t> g_smem_attr;
std::map<std::pair<std::pair<int, const void *>, size_t>, int> g_occ;
std::map<int, int> g_sms;

int device_sms()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> g(g_mu);
    auto it = g_sms.find(dev);
    if (it != g_sms.end()) return it->second;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_sms[dev] = n;
    return n;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per
// (device, kernel, size).
bool ensure_smem(const void *fn, size_t bytes)
{
    if (bytes <= 48 * 1024) return true;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> g(g_mu);
    auto key = std::make_pair(dev, fn);
    auto it = g_smem_attr.find(key);
    if (it != g_smem_attr.end() && it->second >= bytes) return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    g_smem_attr[key] = bytes;
    return true;
}

// Resident blocks per SM of `fn` at `threads` x `smem` (0 on failure).
int occupancy(const void *fn, int threads, size_t smem)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    {
        std::lock_guard<std::mutex> g(g_mu);
        auto it = g_occ.find(std::make_pair(std::make_pair(dev, fn), smem));
        if (it != g_occ.end()) return it->second;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> g(g_mu);
    g_occ[std::make_pair(std::make_pair(dev, fn), smem)] = n;
    return n;
}

bfmoe_status launched() { return cudaGetLastError() == cudaSuccess ? BFMOE_OK : BFMOE_ERR_CUDA; }

// Scratch of bfmoe_route_static, for callers that cannot allocate: one
// array per device that loads the library, held until the process exits.
constexpr size_t kStaticScratchBytes = 1u << 20;
static __device__ __align__(256) unsigned char g_route_scratch[kStaticScratchBytes];
std::map<int, void *> g_static_scratch;  // device -> device address of g_route_scratch

// The device address of g_route_scratch on the current device (host code
// cannot use the symbol itself), looked up once per device.
void *static_scratch()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> g(g_mu);
    auto it = g_static_scratch.find(dev);
    if (it != g_static_scratch.end()) return it->second;
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess || !ptr) return nullptr;
    g_static_scratch[dev] = ptr;
    return ptr;
}

// Process-wide test hook (bfmoe_debug_set): the routing block that skips the
// first grid barrier, or -1.
int g_skip_arrive_block = -1;

// Launch tokens of the routing barrier: unique per launch within the process,
// from a random 64-bit start (a fresh workspace's epoch word matches one only
// by a 2^-64 chance).
std::atomic<unsigned long long> g_token{0};
unsigned long long next_token()
{
    static const unsigned long long base = [] {
        std::random_device rd;
        return ((unsigned long long)rd() << 32) ^ (unsigned long long)rd() ^ 0x9e3779b97f4a7c15ull;
    }();
    return base + 2ull * g_token.fetch_add(1, std::memory_order_relaxed) + 1ull;
}

// The status / barrier header at the start of every workspace (32 bytes):
// status word, barrier counter, departed counter, pad, 64-bit epoch.
void set_header(RouteParams &rp, uint8_t *hdr)
{
    uint32_t *w = reinterpret_cast<uint32_t *>(hdr);
    rp.status = w;
    rp.sync = w + 1;
    rp.departed = w + 2;
    rp.epoch = reinterpret_cast<unsigned long long *>(hdr + 16);
    rp.token = next_token();
}

// Optional per-kernel event recorder used by bfmoe_forward_profile.
struct StageRec {
    cudaEvent_t ev[BFMOE_MAX_STAGES + 1];
    int n = 0;
    bool on = false;
};

const char *const kStageNames[] = {"prep", "route", "expert_in", "contract", "combine"};
constexpr int kNumStages = 5;

void mark(StageRec *r, cudaStream_t st)
{
    if (r && r->on && r->n <= BFMOE_MAX_STAGES) cudaEventRecord(r->ev[r->n++], st);
}

template <typename K, typename... Args>
cudaError_t launch(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl, bool coop,
                   Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (coop) {
        attr[na].id = cudaLaunchAttributeCooperative;
        attr[na].val.cooperative = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The routing kernel, launched cooperatively on as many blocks as fit, with a
// programmatic dependency on whatever precedes it on the stream: it becomes
// resident while the previous call's last kernel runs and waits for it
// before touching memory.
bfmoe_status launch_route(RouteParams rp, cudaStream_t st)
{
    const size_t smem = route_smem_bytes(rp.N);
    if (!ensure_smem((const void *)k_route, smem)) return BFMOE_ERR_CUDA;
    const int sms = device_sms();
    const int occ = occupancy((const void *)k_route, kRouteThreads, smem);
    if (sms <= 0 || occ <= 0) return BFMOE_ERR_CUDA;
    // one block per SM at most (cheaper grid barriers), never more than the
    // histogram holds, and at least 32 tokens per block (a smaller histogram
    // to scan; the top-k of a block's tokens runs on lane groups in parallel)
    const int by_tokens = (int)std::min<long long>(kMaxRouteBlocks, ((long long)rp.T + 31) / 32);
    const int grid = std::max(1, std::min(std::min(std::min(sms, occ * sms), kMaxRouteBlocks), by_tokens));
    rp.skip_arrive_block = g_skip_arrive_block;
    if (launch(k_route, dim3(grid), dim3(kRouteThreads), smem, st, true, true, rp) != cudaSuccess)
        return BFMOE_ERR_CUDA;
    return BFMOE_OK;
}

template <typename T>
bfmoe_status launch_layer(const void *x, int T_, int d, int N, int k, const void *packed, const float *theta,
                          const float *phi, void *y, uint8_t *ws, const FwdLayout &l, const float *logits,
                          cudaStream_t st, StageRec *rec)
{
    const int L = ilog2(d);
    const int R = T_ * k, Rp = padded_rows(T_, k);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws + l.status);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + l.topk_idx);
    float *gates = reinterpret_cast<float *>(ws + l.gates);
    int32_t *perm = reinterpret_cast<int32_t *>(ws + l.perm);
    float2 *ct = reinterpret_cast<float2 *>(ws + l.coef_t);
    float2 *cp = reinterpret_cast<float2 *>(ws + l.coef_p);
    __half *wdec = reinterpret_cast<__half *>(ws + l.wdec);
    __half *ablk = reinterpret_cast<__half *>(ws + l.a_blocks);
    __half *slot = reinterpret_cast<__half *>(ws + l.slot);
    int32_t *row_tok = reinterpret_cast<int32_t *>(ws + l.row_tok);
    int32_t *row_exp = reinterpret_cast<int32_t *>(ws + l.row_exp);
    const int sms = device_sms();
    if (sms <= 0) return BFMOE_ERR_CUDA;

    mark(rec, st);

    PrepParams pp{};
    pp.theta = theta;
    pp.phi = phi;
    pp.coef_t = ct;
    pp.coef_p = cp;
    pp.ncoef = N * L * (d / 2);
    pp.d = d;
    pp.L = L;
    pp.packed = reinterpret_cast<const uint32_t *>(packed);
    pp.wdec = wdec;
    pp.status = status;
    pp.x = x;
    pp.x_bytes = (size_t)T_ * d * sizeof(T);
    pp.logits = logits;
    pp.logit_bytes = ((size_t)T_ * N * 4) & ~size_t(15);
    // two blocks per SM, beside the previous call's combine
    const int prep_grid = std::max(1, std::min((2 * pp.ncoef + 255) / 256, 2 * sms));
    void (*kp)(PrepParams) = nullptr;
    switch (L) {
    case 6: kp = k_prep<6>; break;
    case 7: kp = k_prep<7>; break;
    case 8: kp = k_prep<8>; break;
    case 9: kp = k_prep<9>; break;
    case 10: kp = k_prep<10>; break;
    case 11: kp = k_prep<11>; break;
    default: kp = k_prep<12>; break;
    }
    if (launch(kp, dim3(prep_grid), dim3(256), 0, st, rec == nullptr, false, pp) != cudaSuccess)
        return BFMOE_ERR_CUDA;
    mark(rec, st);

    RouteParams rp{};
    rp.logits = logits;
    rp.T = T_;
    rp.N = N;
    rp.k = k;
    rp.topk_idx = idx;
    rp.gates = gates;
    rp.perm = perm;
    rp.row_pos = nullptr;
    rp.offsets = reinterpret_cast<int32_t *>(ws + l.offsets);
    rp.hist = reinterpret_cast<int32_t *>(ws + l.hist);
    rp.total = reinterpret_cast<int32_t *>(ws + l.total);
    set_header(rp, ws + l.status);
    rp.row_tok = row_tok;
    rp.row_exp = row_exp;
    rp.d = d;
    rp.clear_status = 0;  // the prep kernel, first in the call, clears it
    bfmoe_status s = launch_route(rp, st);
    if (s != BFMOE_OK) return s;
    mark(rec, st);

    ExpertInParams ep{};
    ep.x = x;
    ep.d = d;
    ep.L = L;
    ep.k = k;
    ep.N = N;
    ep.R = R;
    ep.row_tok = row_tok;
    ep.row_exp = row_exp;
    ep.coef_t = ct;
    ep.a_blocks = ablk;
    ep.status = status;
    const bool smc = expert_in_smem_coef(d, L);
    const size_t in_smem = expert_in_smem_bytes(d, L, smc, (int)sizeof(T));
    auto kin = smc ? k_expert_in<T, true> : k_expert_in<T, false>;
    if (!ensure_smem((const void *)kin, in_smem)) return BFMOE_ERR_CUDA;
    const int in_occ = occupancy((const void *)kin, kInThreads, in_smem);
    const int in_grid = std::max(1, std::min(in_tiles(T_, d, k), std::max(1, in_occ) * sms));
    if (launch(kin, dim3(in_grid), dim3(kInThreads), in_smem, st, true, false, ep) != cudaSuccess)
        return BFMOE_ERR_CUDA;
    mark(rec, st);

    ContractParams cpar{};
    cpar.a_blocks = ablk;
    cpar.w_blocks = wdec;
    cpar.slot = slot;
    cpar.perm = perm;
    cpar.topk_idx = idx;
    cpar.coef_p = cp;
    cpar.gates = gates;
    cpar.packed = reinterpret_cast<const uint32_t *>(packed);
    cpar.d = d;
    cpar.L = L;
    cpar.N = N;
    cpar.R = R;
    cpar.Rp = Rp;
    cpar.status = status;
    const int BN = gemm_bn(d);
    const int nunits = (Rp / kBM) * (d / BN);
    const size_t c_smem = contract_smem_bytes(d);
    auto kc = BN == 256 ? k_contract<256> : (BN == 128 ? k_contract<128> : k_contract<64>);
    if (!ensure_smem((const void *)kc, c_smem)) return BFMOE_ERR_CUDA;
    if (launch(kc, dim3(std::min(nunits, sms)), dim3(contract_threads(BN)), c_smem, st, true, false, cpar) !=
        cudaSuccess)
        return BFMOE_ERR_CUDA;
    mark(rec, st);

    CombineParams cb{};
    cb.slot = slot;
    cb.T = T_;
    cb.d = d;
    cb.L = L;
    cb.k = k;
    cb.N = N;
    cb.s_lo = ilog2(BN);
    cb.topk_idx = idx;
    cb.phi = phi;
    cb.y = y;
    cb.status = status;
    const int HS = L - cb.s_lo;
    const unsigned cthreads = (unsigned)T_ * (unsigned)(BN / 8);  // BN/8 threads per token
    const dim3 cgrid2((cthreads + 255) / 256);
    cudaError_t e = cudaSuccess;
    const bool pdl = rec == nullptr;
    const bool k2 = k == 2;
    switch (HS) {
    case 0:
        if (BN == 256)
            e = k2 ? launch(k_combine<T, 0, 256, 8, 2>, cgrid2, dim3(256), 0, st, pdl, false, cb)
                   : launch(k_combine<T, 0, 256, 8, 0>, cgrid2, dim3(256), 0, st, pdl, false, cb);
        else if (BN == 128)
            e = k2 ? launch(k_combine<T, 0, 128, 8, 2>, cgrid2, dim3(256), 0, st, pdl, false, cb)
                   : launch(k_combine<T, 0, 128, 8, 0>, cgrid2, dim3(256), 0, st, pdl, false, cb);
        else
            e = k2 ? launch(k_combine<T, 0, 64, 8, 2>, cgrid2, dim3(256), 0, st, pdl, false, cb)
                   : launch(k_combine<T, 0, 64, 8, 0>, cgrid2, dim3(256), 0, st, pdl, false, cb);
        break;
    case 1:
        e = k2 ? launch(k_combine<T, 1, 256, 8, 2>, cgrid2, dim3(256), 0, st, pdl, false, cb)
               : launch(k_combine<T, 1, 256, 8, 0>, cgrid2, dim3(256), 0, st, pdl, false, cb);
        break;
    case 2:
        e = k2 ? launch(k_combine<T, 2, 256, 8, 2>, cgrid2, dim3(256), 0, st, pdl, false, cb)
               : launch(k_combine<T, 2, 256, 8, 0>, cgrid2, dim3(256), 0, st, pdl, false, cb);
        break;
    case 3: e = launch(k_combine<T, 3, 256, 4, 0>, cgrid2, dim3(256), 0, st, pdl, false, cb); break;
    default: e = launch(k_combine<T, 4, 256, 2, 0>, cgrid2, dim3(256), 0, st, pdl, false, cb); break;
    }
    if (e != cudaSuccess) return BFMOE_ERR_CUDA;
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
    return route_layout(T, N).total_bytes;
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
    if (ws_bytes < l.total_bytes) return BFMOE_ERR_WORKSPACE;
    uint8_t *w = reinterpret_cast<uint8_t *>(ws);
    cudaStream_t st = as_stream(stream);
    RouteParams rp{};
    rp.logits = logits;
    rp.T = T;
    rp.N = N;
    rp.k = k;
    rp.topk_idx = topk_idx;
    rp.gates = gates;
    rp.perm = perm;
    rp.offsets = offsets;
    rp.hist = reinterpret_cast<int32_t *>(w + l.hist);
    rp.total = reinterpret_cast<int32_t *>(w + l.total);
    set_header(rp, w + l.status);
    rp.clear_status = 1;
    s = launch_route(rp, st);
    if (s != BFMOE_OK) return s;
    return launched();
}

bfmoe_status bfmoe_route_static(const float *logits, int T, int N, int k, int32_t *topk_idx, float *gates,
                                int32_t *perm, int32_t *offsets, void *stream)
{
    bfmoe_status s = check_route_shape(T, N, k);
    if (s != BFMOE_OK) return s;
    if (!logits || !topk_idx || !gates || !perm || !offsets) return BFMOE_ERR_INVALID_ARG;
    if (!aligned(logits, 4) || !aligned(topk_idx, 4) || !aligned(gates, 4) || !aligned(perm, 4) ||
        !aligned(offsets, 4))
        return BFMOE_ERR_INVALID_ARG;
    const RouteLayout l = route_layout(T, N);
    if (l.total_bytes > kStaticScratchBytes) return BFMOE_ERR_UNSUPPORTED;
    uint8_t *w = reinterpret_cast<uint8_t *>(static_scratch());
    if (!w) return BFMOE_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    RouteParams rp{};
    rp.logits = logits;
    rp.T = T;
    rp.N = N;
    rp.k = k;
    rp.topk_idx = topk_idx;
    rp.gates = gates;
    rp.perm = perm;
    rp.offsets = offsets;
    rp.hist = reinterpret_cast<int32_t *>(w + l.hist);
    rp.total = reinterpret_cast<int32_t *>(w + l.total);
    set_header(rp, w + l.status);
    rp.clear_status = 1;
    s = launch_route(rp, st);
    if (s != BFMOE_OK) return s;
    return launched();
}

void bfmoe_debug_set(int key, int value)
{
    if (key == BFMOE_DEBUG_SKIP_ARRIVE_BLOCK) g_skip_arrive_block = value;
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
    k_engine_table<<<(ncoef + 255) / 256, 256, 0, st>>>(angles, N, d, L, transpose != 0, coef);
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
    return fwd_layout(T, d, N, k).total_bytes;
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
    out->total = l.total_bytes;
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
    if (ws_bytes < l.total_bytes) return BFMOE_ERR_WORKSPACE;
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

#ifdef BFMOE_TRACE_PHASES
// Copy the phase trace (4 kernels x 1024 blocks x 16 slots of u64) to host.
BFMOE_API int bfmoe_trace_read(unsigned long long *host, int clear)
{
    if (cudaDeviceSynchronize() != cudaSuccess) return BFMOE_ERR_CUDA;
    if (cudaMemcpyFromSymbol(host, g_bfmoe_trace, sizeof(g_bfmoe_trace)) != cudaSuccess) return BFMOE_ERR_CUDA;
    if (clear) {
        static unsigned long long zeros[kTraceKernels][kTraceBlocks][kTraceSlots];
        if (cudaMemcpyToSymbol(g_bfmoe_trace, zeros, sizeof(zeros)) != cudaSuccess) return BFMOE_ERR_CUDA;
    }
    return BFMOE_OK;
}
#endif

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
