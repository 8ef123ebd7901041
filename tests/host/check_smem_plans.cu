// Host check of the kernels' shared-memory plans (no GPU): for every expert
// count the routing kernel's staged logits, kept experts, partial sums,
// offsets and bucket bases stay inside its plan; every kernel's dynamic
// shared memory fits one CTA.  Built with nvcc as host code and run by
// tests/test_smem_plans.py; prints "ok".
#include <cstdio>

#include "contract.cuh"
#include "layer.cuh"

using namespace bfmoe;

static constexpr size_t kMaxDynSmem = 227 * 1024;  // per CTA, opt-in maximum
static constexpr size_t kStaticMargin = 1024;      // the kernels' own __shared__ words

static int fail(const char *what, int a, long long b)
{
    std::printf("FAIL %s (%d, %lld)\n", what, a, b);
    return 1;
}

int main()
{
    int bad = 0;
    for (int N = 1; N <= 4096; ++N) {
        const RouteSmem lay(N);
        const int stage = route_stage_ints(N);
        const int bt = route_batch_tokens(N);
        if (bt < 1 || bt > 256) bad |= fail("batch tokens", N, bt);
        // a batch never holds more tokens than route_batch_tokens, whatever
        // the group width the kernel picks for it
        for (int grp = 1; grp <= 32; grp <<= 1)
            if ((long long)bt * logit_row_stride(N, grp) > stage) bad |= fail("staged batch", N, grp);
        if (lay.a_logits % 4 != 0) bad |= fail("staging alignment", N, lay.a_logits);
        if (lay.a_hist < lay.keep + kSelCap) bad |= fail("kept experts overlap", N, lay.a_hist);
        if (lay.a_logits < lay.a_hist + N) bad |= fail("block histogram overlap", N, lay.a_logits);
        if (lay.a_logits + stage > lay.total) bad |= fail("staging end", N, lay.a_logits + stage);
        if (lay.off < lay.keep + kSelCap) bad |= fail("offsets overlap", N, lay.off);
        if (lay.cnt < lay.off + N + 1 || lay.red < lay.cnt + N) bad |= fail("bases overlap", N, lay.cnt);
        if (lay.red + 2 * kRouteRedInts > lay.total) bad |= fail("partial sums end", N, lay.red);
        if (N <= kOneBarrierMaxN) {
            // the one-barrier histogram read: `parts` threads per column of
            // 4 experts (16-byte loads) or of one expert
            for (int by4 = 0; by4 < 2; ++by4) {
                if (by4 && (N & 3)) continue;
                const int cols = by4 ? N / 4 : N;
                const int parts = (kRouteThreads / cols) > 1 ? kRouteThreads / cols : 1;
                if (parts * N > kRouteRedInts) bad |= fail("partial sums", N, (long long)parts * N);
            }
        }
        if (route_smem_bytes(N) + kStaticMargin > kMaxDynSmem) bad |= fail("routing smem", N, route_smem_bytes(N));
    }
    for (int L = 6; L <= 12; ++L) {
        const int d = 1 << L;
        for (int esize : {2, 4}) {
            const size_t b = expert_in_smem_bytes(d, L, expert_in_smem_coef(d, L), esize);
            if (b + kStaticMargin > kMaxDynSmem) bad |= fail("input kernel smem", d, (long long)b);
        }
        if (contract_smem_bytes(d) + kStaticMargin > kMaxDynSmem) bad |= fail("contraction smem", d, (long long)contract_smem_bytes(d));
    }
    if (bad) return 1;
    std::printf("ok\n");
    return 0;
}
