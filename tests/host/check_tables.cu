// Host check of the table layouts the kernels share: every generator
// (engine_entry, out_table_entry, slot_col) against its inverse, and the
// engine order against a direct walk of the butterfly's stages.  Built with
// nvcc as host code and run by tests/test_table_layout.py; prints "ok".
#include <cstdio>
#include <vector>

#include "butterfly.cuh"
#include "contract.cuh"

using namespace bfmoe;

static int fail(const char *what, int d, int r)
{
    std::printf("FAIL %s d=%d r=%d\n", what, d, r);
    return 1;
}

int main()
{
    int bad = 0;
    for (int BN : {64, 128, 256})
        for (int sp = 0; sp < BN; ++sp)
            if (slot_pos(BN, slot_col(BN, sp)) != sp) bad |= fail("slot order", BN, sp);
    for (int L = 6; L <= 12; ++L) {
        const int d = 1 << L, half = d / 2, n = L * half;
        for (int transpose = 0; transpose < 2; ++transpose) {
            // every (stage, pair) exactly once, and the inverse agrees
            std::vector<int> seen((size_t)n, 0);
            for (int r = 0; r < n; ++r) {
                int s, p;
                engine_entry(d, L, transpose != 0, r, s, p);
                if (s < 0 || s >= L || p < 0 || p >= half) return fail("engine range", d, r);
                if (seen[(size_t)s * half + p]++) bad |= fail("engine duplicate", d, r);
                if (engine_pos(d, L, transpose != 0, s, p) != r) bad |= fail("engine inverse", d, r);
            }
            // passes come in execution order: B runs pass 0 (stage 0 up)
            // first, B^T the last pass (top stages) first
            const int np = npass_of(L);
            int prev_rank = 0;
            for (int r = 0; r < n; ++r) {
                int s, p;
                engine_entry(d, L, transpose != 0, r, s, p);
                int pass = 0;
                for (int q = 0; q < np; ++q) {
                    int s0, g;
                    pass_bounds(L, q, s0, g);
                    if (s >= s0 && s < s0 + g) pass = q;
                }
                const int rank = transpose ? np - 1 - pass : pass;
                if (rank < prev_rank) bad |= fail("engine pass order", d, r);
                prev_rank = rank;
            }
        }
        std::vector<int> seen((size_t)n, 0);
        const int BN = gemm_bn(d), SIN = slice_stages(BN);
        for (int r = 0; r < n; ++r) {
            int s, p;
            out_table_entry(d, L, r, s, p);
            if (s < 0 || s >= L || p < 0 || p >= half) return fail("out range", d, r);
            if (seen[(size_t)s * half + p]++) bad |= fail("out duplicate", d, r);
            if (out_pos(d, L, s, p) != r) bad |= fail("out inverse", d, r);
            // the slice part holds exactly the stages below SIN, the rest after
            if ((r < SIN * half) != (s < SIN)) bad |= fail("out slice split", d, r);
        }
    }
    std::printf(bad ? "FAILED\n" : "ok\n");
    return bad;
}
