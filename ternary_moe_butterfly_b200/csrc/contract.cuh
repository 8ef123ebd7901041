// contract.cuh -- the ternary contraction of all routed rows against the one
// shared W_base on the 5th-generation tensor cores, with the expert output
// rotation fused into the epilogue.
//
// Z = X' W_base^T for every routed row at once (M = rows in bucket order,
// N = K = d): W_base is shared by all experts, so the experts differ only in
// the rotations around this single GEMM (ButterflyMoE summaries, section 2 /
// 2.1: experts are never materialised; the ternary product "needs only
// additions", section 3 -- on a tensor core the {-1, 0, +1} operand is exact
// in fp16).
//
// Work unit = (128-row tile, BN-column slice of the output), BN = min(d, 256).
// Persistent CTAs walk the units.  Warp roles:
//   warp 0   one thread streams the A and W operand blocks with bulk copies
//            through a kStages-deep shared-memory ring;
//   warp 1   one thread issues tcgen05.mma (M=128, N=BN, K=16) into one of
//            two TMEM accumulators (double buffered: 2 x BN columns);
//   warps 2-9  the epilogue: TMEM lane = tile row = thread, so each thread
//            (two warps per row, each on half of the columns) applies the
//            output-butterfly stages that stay inside the slice
//            (stages 0 .. log2 BN - 1) to its own row, with the row's expert
//            table, scales by alpha * gate and stores fp16 to the row's
//            token-order slot (the slot layout described with CombineParams).
//            Stages 0-4 act inside 32-column blocks (one 32-column TMEM load,
//            rotate, store back); stages 5.. act on columns 32 apart (4-column
//            TMEM loads).  The remaining stages, which mix slices, are
//            applied by the combine kernel.
#pragma once

#include "common.cuh"
#include "layer.cuh"

namespace bfmoe {

// Epilogue warps per TMEM lane quadrant (each takes 1/parts of a row's
// columns), and the CTA size: a producer warp, an MMA warp, 4 * parts
// epilogue warps.
__host__ __device__ constexpr int epi_parts(int) { return 2; }
__host__ __device__ constexpr int contract_threads(int BN) { return 64 + 128 * epi_parts(BN); }
constexpr int kStages = 3;


// Shared-memory cos/sin tables staged per TMEM lane quadrant: two experts x
// slice_stages(BN) stages x BN/2 pairs, the second table 16 bytes further on
// so that a warp whose rows use both tables reads them from distinct banks.
__host__ __device__ constexpr int staged_slice_stride(int BN) { return slice_stages(BN) * (BN / 2) + 2; }
__host__ __device__ constexpr int pair_table_floats2(int BN) { return 2 * staged_slice_stride(BN); }

// Output tables hold each expert's {cos a, sin a} of phi in the order the
// epilogue and the combine consume them.  For each BN-column slice nh:
//   pass 1: 32-column blocks blk, stages 0..4, rotations m (bit s clear)
//           ascending: 80 entries per block;
//   pass 2: 8-column groups g, stages 5..SIN-1, columns q = 0..7, rotations
//           over m (columns 8g + q + 32 m) with the stage's bit clear.
// Then, for the combine, the in-slice columns c < BN in slot order (column
// 8g + 32m + q at slot position (g * BN/32 + m) * 8 + q, the order in which
// the combine's threads read them): stages SIN..L-1, rotations over the
// slices h (columns c + BN h).  out_table_entry gives the (stage, pair) of
// entry r; out_pos is its inverse.
__host__ __device__ constexpr int slot_col(int BN, int sp)
{
    return 8 * (sp / (BN / 4)) + 32 * ((sp >> 3) % (BN / 32)) + (sp & 7);
}
__host__ __device__ constexpr int slot_pos(int BN, int c) { return ((c >> 3) & 3) * (BN / 4) + (c >> 5) * 8 + (c & 7); }
__host__ __device__ inline void out_table_entry(int d, int L, int r, int &s, int &p)
{
    const int BN = gemm_bn(d), SIN = slice_stages(BN);
    const int slice = SIN * (BN / 2), NH = d / BN;
    if (r < NH * slice) {
        const int nh = r / slice;
        int w = r % slice;
        const int p1 = (BN / 32) * 80;
        int jj;
        if (w < p1) {
            const int blk = w / 80, rr = w % 80;
            s = rr / 16;
            jj = blk * 32 + insert_zero_bit(rr % 16, s);
        } else {
            w -= p1;
            const int G2 = SIN - 5, M2h = 1 << (G2 - 1);
            const int per = G2 * 8 * M2h;
            const int grp = w / per, rr = w % per;
            const int ls = rr / (8 * M2h), rem = rr % (8 * M2h);
            s = 5 + ls;
            jj = grp * 8 + rem / M2h + 32 * insert_zero_bit(rem % M2h, ls);
        }
        p = nh * (BN / 2) + pair_of(jj, s);
    } else {
        const int w = r - NH * slice;
        const int HS = L - SIN, per = HS << (HS - 1);
        const int c = slot_col(BN, w / per), rr = w % per;
        const int ls = rr >> (HS - 1);
        s = SIN + ls;
        p = pair_of(c + BN * insert_zero_bit(rr & ((1 << (HS - 1)) - 1), ls), s);
    }
}

struct ContractParams {
    const __half *a_blocks;   // [Rp/128][d/64] blocks of 128 x 64
    const __half *w_blocks;   // [d/BN][d/64] blocks of BN x 64
    __half *slot;             // [R][d] fp16 alpha*gate*u, token order (row i = t*k + j), slot layout
    const float *gates;       // [R] gate of row i
    const uint32_t *packed;   // alpha in word 2
    const int32_t *perm;      // bucket position -> i
    const int32_t *topk_idx;  // i -> expert
    const float2 *coef_p;     // [N][L*d/2] output table (see out_table_entry)
    int d, L, N, R, Rp;
    uint32_t *status;
};

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}


// Inverse of out_table_entry: the output-table position of (stage s, pair p).
__host__ __device__ inline int out_pos(int d, int L, int s, int p)
{
    const int BN = gemm_bn(d), SIN = slice_stages(BN);
    const int slice = SIN * (BN / 2), NH = d / BN, NB = BN / 32;
    if (s < SIN) {
        const int nh = p / (BN / 2);
        const int jj = insert_zero_bit(p % (BN / 2), s);  // column inside the slice
        if (s < 5) return nh * slice + (jj >> 5) * 80 + s * 16 + delete_bit(jj & 31, s);
        const int G2 = SIN - 5, M2h = 1 << (G2 - 1), PER2 = G2 * 8 * M2h;
        const int ls = s - 5, c = jj & 31, m = jj >> 5;
        return nh * slice + NB * 80 + (c >> 3) * PER2 + (ls * 8 + (c & 7)) * M2h + delete_bit(m, ls);
    }
    const int HS = L - SIN, pc = HS << (HS - 1);
    const int jj = insert_zero_bit(p, s);
    const int c = jj % BN, m = jj / BN, ls = s - SIN;
    return NH * slice + slot_pos(BN, c) * pc + (ls << (HS - 1)) + delete_bit(m, ls);
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// AND of `pred` over the `nthreads` threads of named barrier `id` (a
// barrier itself): every participant gets the same answer.
__device__ __forceinline__ bool bar_red_and(int id, int nthreads, bool pred)
{
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((int)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Output-butterfly stages 0 .. log2(BN)-1 of one row held in TMEM columns
// [tbase, tbase + BN) of this warp's lanes, then store to `out` (if
// non-null).  `tab` is the row's expert's slice table in the output-table
// order (shared or global memory, as the caller's pointer type says).
// epi_parts(BN) warps share the row's lanes: `part` selects this warp's share
// of the 32-column blocks (pass 1) and of the 8-column groups (pass 2);
// `bar_id` is the named barrier of those warps.
template <int BN, typename Tab>
__device__ __forceinline__ void epilogue_row(uint32_t tbase, Tab tab, __half *__restrict__ out, float scale,
                                             int part, int bar_id)
{
    constexpr int SIN = slice_stages(BN);
    constexpr int G2 = SIN - 5;  // stages at stride >= 32
    constexpr int M2 = 1 << G2;
    constexpr int NB = BN / 32;
    constexpr int PER2 = G2 * 8 * (M2 / 2);
    constexpr int PARTS = epi_parts(BN);
    // pass 1: stages 0..4 inside each 32-column block; the next block's TMEM
    // load is in flight while this one rotates
    auto pass1_block = [&](int blk, float (&v)[32]) {
        const Tab t4 = tab + blk * 80;
#pragma unroll
        for (int s = 0; s < 5; ++s) {
            const int h = 1 << s;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 w = t4.ld4(s * 16 + 2 * i);
                const int m0 = insert_zero_bit(2 * i, s), m1 = insert_zero_bit(2 * i + 1, s);
                if (s > 0) {  // m1 = m0 + 1: one pair instruction per rotation pair
                    float2 a = make_float2(v[m0], v[m1]), b = make_float2(v[m0 + h], v[m1 + h]);
                    rot2(a, b, make_float2(w.x, w.y), make_float2(w.z, w.w));
                    v[m0] = a.x;
                    v[m1] = a.y;
                    v[m0 + h] = b.x;
                    v[m1 + h] = b.y;
                } else {
                    rot1(v[m0], v[m0 + h], w.x, w.z);
                    rot1(v[m1], v[m1 + h], w.y, w.w);
                }
            }
        }
        tmem_st32(tbase + (uint32_t)(blk * 32), v);
    };
    {
        constexpr int NBH = NB / PARTS;  // blocks per warp
        const int b0 = part * NBH;
        float va[32], vb[32];
        tmem_ld32_async(tbase + (uint32_t)(b0 * 32), va);
        tmem_ld_wait_regs(va);
#pragma unroll
        for (int i = 0; i < NBH; i += 2) {
            if (i + 1 < NBH) tmem_ld32_async(tbase + (uint32_t)((b0 + i + 1) * 32), vb);
            pass1_block(b0 + i, va);
            if (i + 1 < NBH) {
                tmem_ld_wait_regs(vb);
                if (i + 2 < NBH) tmem_ld32_async(tbase + (uint32_t)((b0 + i + 2) * 32), va);
                pass1_block(b0 + i + 1, vb);
                if (i + 2 < NBH) tmem_ld_wait_regs(va);
            }
        }
    }
    tmem_st_wait();
    BFMOE_TRACE(2, threadIdx.x == 64, 9);
    named_bar_sync(bar_id, 32 * PARTS);
    BFMOE_TRACE(2, threadIdx.x == 64, 10);
    // pass 2: stages 5..SIN-1 on columns c0 + q + 32 m, 8-column groups
    constexpr int GPP = 4 / PARTS;  // groups per warp
#pragma unroll 1
    for (int grp = part * GPP; grp < (part + 1) * GPP; ++grp) {
        const int c0 = grp * 8;
        const Tab t2 = tab + (NB * 80 + grp * PER2);
        // the group's 8 columns in two halves of 4 (fewer live registers);
        // the fp16 results of both halves meet in h for the 32-byte stores
        uint32_t h[M2 * 4];
#pragma unroll
        for (int qh = 0; qh < 8; qh += 4) {
            float v[4][M2];
#pragma unroll
            for (int m = 0; m < M2; ++m)
                tmem_ld4_nowait(tbase + (uint32_t)(c0 + qh + 32 * m), v[0][m], v[1][m], v[2][m], v[3][m]);
            tmem_ld_wait();
#pragma unroll
            for (int ls = 0; ls < G2; ++ls) {
                const int hs = 1 << ls;
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    const int q = qh + qq;
                    if constexpr (M2 >= 4) {
                        // rotations ri, ri+1 of column q: one paired table load
#pragma unroll
                        for (int ri = 0; ri < M2 / 2; ri += 2) {
                            const float4 w = t2.ld4((ls * 8 + q) * (M2 / 2) + ri);
                            const int m0 = insert_zero_bit(ri, ls), m1 = insert_zero_bit(ri + 1, ls);
                            if (ls > 0) {
                                float2 a = make_float2(v[qq][m0], v[qq][m1]);
                                float2 b = make_float2(v[qq][m0 + hs], v[qq][m1 + hs]);
                                rot2(a, b, make_float2(w.x, w.y), make_float2(w.z, w.w));
                                v[qq][m0] = a.x;
                                v[qq][m1] = a.y;
                                v[qq][m0 + hs] = b.x;
                                v[qq][m1 + hs] = b.y;
                            } else {
                                rot1(v[qq][m0], v[qq][m0 + hs], w.x, w.z);
                                rot1(v[qq][m1], v[qq][m1 + hs], w.y, w.w);
                            }
                        }
                    } else {
                        // one rotation per column and stage: the pair partner
                        // is the next column's
                        const float2 cs = t2.cs((ls * 8 + q) * (M2 / 2));
                        rot1(v[qq][0], v[qq][hs], cs.x, cs.y);
                    }
                }
            }
            // alpha * gate, fp16, packed in [m][q] order
#pragma unroll
            for (int m = 0; m < M2; ++m)
#pragma unroll
                for (int qq = 0; qq < 4; qq += 2) {
                    __half2 hv = __floats2half2_rn(scale * v[qq][m], scale * v[qq + 1][m]);
                    h[m * 4 + (qh + qq) / 2] = *reinterpret_cast<uint32_t *>(&hv);
                }
        }
        if (out) {
            // the group's M2 x 8 values as one contiguous run (slot row
            // layout [group][m][q], described with CombineParams)
            __half *dst = out + grp * (8 * M2);
#pragma unroll
            for (int w = 0; w < M2 / 2; ++w)
                asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst + 16 * w), "r"(h[8 * w]),
                             "r"(h[8 * w + 1]), "r"(h[8 * w + 2]), "r"(h[8 * w + 3]), "r"(h[8 * w + 4]),
                             "r"(h[8 * w + 5]), "r"(h[8 * w + 6]), "r"(h[8 * w + 7])
                             : "memory");
        }
    }
}

template <int BN>
__global__ void __launch_bounds__(contract_threads(BN), 1) k_contract(ContractParams p)
{
    constexpr int PARTS = epi_parts(BN);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const int d = p.d;
    const int KC = d / kBK;
    const int NH = d / BN;
    const int MT = p.Rp / kBM;
    const int nunits = MT * NH;
    const int half = d >> 1;
    constexpr uint32_t a_bytes = kBM * kBK * 2, b_bytes = (uint32_t)BN * kBK * 2;
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + (size_t)kStages * a_bytes;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sB + (size_t)kStages * b_bytes);
    uint64_t *full = bars, *empty = bars + kStages;
    uint64_t *tfull = bars + 2 * kStages, *tempty = tfull + 2, *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    float2 *tables = reinterpret_cast<float2 *>(reinterpret_cast<uint8_t *>(bars) + 256);  // [4 pairs][...]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    BFMOE_TRACE(2, threadIdx.x == 0, 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4 * PARTS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 2 * BN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    BFMOE_TRACE(2, threadIdx.x == 0, 1);
    // The W operand blocks were decoded by the prep kernel, which completed
    // before the input-butterfly kernel (this grid's predecessor) could
    // start: the producer streams the first stages' W blocks before it
    // waits.  Everything else waits for the input kernel (the A blocks).
    const bool early_w = warp == 0 && lane == 0 && (int)blockIdx.x < nunits;
    const int npre = early_w ? (KC < kStages ? KC : kStages) : 0;
    if (early_w) {
        const __half *b_src = p.w_blocks + (size_t)(blockIdx.x % NH) * KC * ((size_t)BN * kBK);
        for (int kc = 0; kc < npre; ++kc) {
            mbar_arrive_expect_tx(&full[kc], a_bytes + b_bytes);
            bulk_g2s(sB + (size_t)kc * b_bytes, b_src + (size_t)kc * ((size_t)BN * kBK), b_bytes, &full[kc]);
        }
    }
    pdl_wait();  // the A blocks come from the input-butterfly kernel
    pdl_trigger();
    BFMOE_TRACE(2, threadIdx.x == 0, 2);

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            for (int u = blockIdx.x; u < nunits && !*abort_flag; u += gridDim.x) {
                const int mt = u / NH, nh = u % NH;
                const __half *a_src = p.a_blocks + (size_t)mt * KC * (kBM * kBK);
                const __half *b_src = p.w_blocks + (size_t)nh * KC * ((size_t)BN * kBK);
                for (int kc = 0; kc < KC; ++kc, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (uint32_t)(it / kStages) & 1u;
                    if (it < npre) {  // its W block is already on the way
                        BFMOE_TRACE(2, it == 0, 3);
                        bulk_g2s(sA + (size_t)s * a_bytes, a_src + (size_t)kc * (kBM * kBK), a_bytes, &full[s]);
                        continue;
                    }
                    if (!mbar_wait(&empty[s], ph ^ 1u)) {
                        set_status(p.status, BFMOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                        break;
                    }
                    BFMOE_TRACE(2, it == 0, 3);
                    mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
                    bulk_g2s(sA + (size_t)s * a_bytes, a_src + (size_t)kc * (kBM * kBK), a_bytes, &full[s]);
                    bulk_g2s(sB + (size_t)s * b_bytes, b_src + (size_t)kc * ((size_t)BN * kBK), b_bytes, &full[s]);
                }
            }
            // every copy issued must have landed before the CTA exits
            for (int q = it - kStages > 0 ? it - kStages : 0; q < it; ++q)
                if (!mbar_wait(&full[q % kStages], (uint32_t)(q / kStages) & 1u)) set_status(p.status, BFMOE_ERR_TIMEOUT);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_f32(kBM, BN);
            int it = 0, li = 0;
            for (int u = blockIdx.x; u < nunits && !*abort_flag; u += gridDim.x, ++li) {
                const int b = li & 1;
                if (!mbar_wait(&tempty[b], ((uint32_t)(li >> 1) & 1u) ^ 1u)) {
                    set_status(p.status, BFMOE_ERR_TIMEOUT);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t dcol = tmem + (uint32_t)(b * BN);
                bool ok = true;
                for (int kc = 0; kc < KC; ++kc, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait(&full[s], (uint32_t)(it / kStages) & 1u)) {
                        set_status(p.status, BFMOE_ERR_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    BFMOE_TRACE(2, it == 0, 4);
                    BFMOE_TRACE(2, it == KC - 1, 5);
                    const uint32_t a0 = smem_addr(sA + (size_t)s * a_bytes), b0 = smem_addr(sB + (size_t)s * b_bytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t ad = sdesc_noswizzle(a0 + kk * 256, 128, 1024);
                        const uint64_t bd = sdesc_noswizzle(b0 + kk * 256, 128, 1024);
                        mma_f16(dcol, ad, bd, idesc, (kc | kk) != 0);
                    }
                    mma_commit(&empty[s]);
                }
                if (!ok) break;
                mma_commit(&tfull[b]);
            }
            // drain: wait until every MMA issued above has completed
            mma_commit(drain);
            if (!mbar_wait(drain, 0)) set_status(p.status, BFMOE_ERR_TIMEOUT);
        }
    } else {
        // epilogue warps 2..: warp w owns TMEM lanes 32*(w % 4) .. +31 and
        // 1/PARTS of the row's columns (part = (w - 2) / 4)
        const int lane_base = (warp & 3) * 32;
        const int part = (warp - 2) >> 2;
        const int bar_id = 1 + (warp & 3);
        constexpr int SIN = slice_stages(BN);
        constexpr int HB = BN / 2;  // pairs per stage inside the slice
        float2 *ptab = tables + (size_t)(warp & 3) * pair_table_floats2(BN);
        const int pt = (part << 5) | lane;  // thread index inside the warp pair
        int li = 0;
        for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++li) {
            const int b = li & 1;
            const int mt = u / NH, nh = u % NH;
            const int r = mt * kBM + lane_base + lane;
            int i = -1, e = 0;
            if (r < p.R) {
                i = p.perm[r];
                if (i < 0 || i >= p.R) i = -1;
                else e = min(max(p.topk_idx[i], 0), p.N - 1);
            }
            // the rows are in bucket order: stage the slice tables of the
            // first and last row's experts while the MMA runs
            const int ea = __shfl_sync(0xffffffffu, e, 0), eb = __shfl_sync(0xffffffffu, e, 31);
            named_bar_sync(bar_id, 32 * PARTS);  // the quadrant's warps are done with the previous tables
            {
                // the two experts' slice tables: contiguous copies
                constexpr int SL4 = SIN * HB / 2;  // float4 per slice table
#pragma unroll
                for (int t = 0; t < 2; ++t)
                    copy_g2s(reinterpret_cast<const float4 *>(p.coef_p + (size_t)(t ? eb : ea) * p.L * half +
                                                              (size_t)nh * SIN * HB),
                             reinterpret_cast<float4 *>(ptab + (size_t)t * staged_slice_stride(BN)), SL4, pt,
                             32 * PARTS);
            }
            BFMOE_TRACE(2, threadIdx.x == 64 && li == 0, 13);
            bool ok = mbar_wait(&tfull[b], (uint32_t)(li >> 1) & 1u);
            // both warps sharing these lanes take the same branch (they meet
            // at named barriers inside epilogue_row); the barrier also makes
            // the staged tables visible to the pair
            ok = bar_red_and(bar_id, 32 * PARTS, ok);
            if (!ok) {
                if (lane == 0) set_status(p.status, BFMOE_ERR_TIMEOUT);
                break;
            }
            tc_fence_after();
            BFMOE_TRACE(2, threadIdx.x == 64 && li == 0, 6);
            BFMOE_TRACE(2, threadIdx.x == 192 && li == 0, 11);
            __half *out = i >= 0 ? p.slot + (size_t)i * d + (size_t)nh * BN : nullptr;
            const float scale = i >= 0 ? __uint_as_float(__ldg(p.packed + 2)) * p.gates[i] : 0.0f;
            const uint32_t tb = tmem + (uint32_t)(b * BN) + ((uint32_t)lane_base << 16);
            if (__all_sync(0xffffffffu, e == ea || e == eb)) {
                const SmemTab st{smem_addr(ptab + (e == ea ? 0 : staged_slice_stride(BN)))};
                epilogue_row<BN>(tb, st, out, scale, part, bar_id);
            } else {  // a third expert inside these 32 rows (a bucket of fewer than 32
                // rows): every lane reads its own expert's table from global memory
                epilogue_row<BN>(tb, GmemTab{p.coef_p + (size_t)e * p.L * half + (size_t)nh * SIN * HB}, out, scale,
                                 part, bar_id);
            }
            BFMOE_TRACE(2, threadIdx.x == 64 && li == 0, 7);
            BFMOE_TRACE(2, threadIdx.x == 192 && li == 0, 12);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[b]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem, 2 * BN);
    BFMOE_TRACE(2, threadIdx.x == 0, 8);
}

__host__ inline size_t contract_smem_bytes(int d)
{
    const int BN = gemm_bn(d);
    return 1024 + (size_t)kStages * (kBM * kBK * 2 + (size_t)BN * kBK * 2) + 256 +
           (size_t)4 * pair_table_floats2(BN) * 8;
}

}  // namespace bfmoe
