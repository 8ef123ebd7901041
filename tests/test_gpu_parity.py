"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Bars: routing (top-k indices, perm, offsets) and packing bit-exact; gates
within 1e-6 relative; y within relative Frobenius error 5e-3 and
max |y - y*| <= 1e-2 * max |y*| (bf16 I/O, fp32 rotations and accumulation,
fp16 tensor-core operand for the rotated rows).
"""
import math

import numpy as np
import pytest

import oracle
from ternary_moe_butterfly_b200 import workloads as wl

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

REL_FRO = 5e-3
REL_MAX = 1e-2


@pytest.fixture(scope="module")
def bf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import ternary_moe_butterfly_b200 as m
    from ternary_moe_butterfly_b200 import build
    build.build()
    return m


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def to_x(inp):
    return dev(inp.x, torch.bfloat16 if inp.wl.dtype == "bf16" else torch.float32)


def check_close(y, ref, what=""):
    y = np.asarray(y, dtype=np.float64)
    fro = np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300)
    mx = np.abs(y - ref).max() / max(np.abs(ref).max(), 1e-300)
    assert fro <= REL_FRO and mx <= REL_MAX, f"{what}: rel fro {fro:.3e}, rel max {mx:.3e}"
    return fro, mx


# ------------------------------------------------------------------ pack

@pytest.mark.parametrize("d", [64, 512, 4096])
def test_pack_bit_exact(bf, d):
    rng = np.random.default_rng(d)
    w = wl.random_ternary(rng, d, p_zero=0.4)
    packed = bf.pack_base(dev(w), 0.0353)
    np.testing.assert_array_equal(packed.cpu().numpy(), oracle.pack_base(w, 0.0353))


def test_pack_rejects_values_outside_ternary(bf):
    w = np.zeros((64, 64), np.int8)
    w[5, 7] = 3
    with pytest.raises(bf.BfmoeError) as e:
        bf.pack_base(dev(w), 1.0)
    assert e.value.code == bf.ERR_INVALID_ARG


# ----------------------------------------------------------------- route

def check_route(bf, logits, k):
    idx, gates, perm, offsets, ws = bf.route(dev(logits), k)
    assert bf.sync_status(ws) == bf.OK
    ridx, rg, rperm, roff = oracle.route(logits, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(perm.cpu().numpy(), rperm)
    np.testing.assert_array_equal(offsets.cpu().numpy(), roff)
    np.testing.assert_allclose(gates.cpu().numpy().astype(np.float64), rg, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("name", ["tiny", "headline", "many_experts", "llm_width", "vit"])
def test_route_full_size_bit_exact(bf, name):
    w = wl.WORKLOADS[name]
    rng = np.random.default_rng(w.seed)
    logits = (rng.standard_normal((w.T, w.N)) * w.logit_std).astype(np.float32)
    check_route(bf, logits, w.k)


@pytest.mark.parametrize("T,N,k", [(1, 1, 1), (7, 3, 3), (65, 8, 2), (130, 300, 8), (1000, 4096, 2), (64, 64, 8)])
def test_route_shapes_ties_and_signed_zero(bf, T, N, k):
    rng = np.random.default_rng(T + N + k)
    lg = np.round(rng.standard_normal((T, N)) * 2).astype(np.float32) / 2  # many exact ties
    lg[:: 3] *= -0.0  # signed zeros
    check_route(bf, lg, k)


def test_route_infinities_and_crowded_expert(bf):
    rng = np.random.default_rng(3)
    T, N, k = 300, 16, 2
    lg = rng.standard_normal((T, N)).astype(np.float32)
    lg[:, 5] += 100.0            # every token picks expert 5 first: one bucket holds T rows
    lg[10, :] = -np.inf
    lg[11, 2] = np.inf
    lg[12, 3] = lg[12, 9] = np.inf
    check_route(bf, lg, k)


def test_route_nan_sets_status_and_stays_valid(bf):
    T, N, k = 100, 8, 2
    lg = np.random.default_rng(4).standard_normal((T, N)).astype(np.float32)
    lg[17, 3] = np.nan
    idx, gates, perm, offsets, ws = bf.route(dev(lg), k)
    assert bf.sync_status(ws) == bf.ERR_NONFINITE
    p = perm.cpu().numpy()
    assert sorted(p.tolist()) == list(range(T * k))
    assert bf.sync_status(ws) == bf.OK  # the word was cleared


# ------------------------------------------------------------- butterfly

@pytest.mark.parametrize("d", [64, 128, 256, 512, 1024, 2048, 4096])
@pytest.mark.parametrize("transpose", [False, True])
def test_butterfly_apply_fp32(bf, d, transpose):
    rng = np.random.default_rng(d + transpose)
    N, rows = 5, 37  # ragged: not a multiple of any tile height
    ang = wl.random_angles(rng, N, d)
    x = rng.standard_normal((rows, d)).astype(np.float32)
    e = rng.integers(0, N, rows).astype(np.int32)
    y, ws = bf.butterfly_apply(dev(x), dev(ang), dev(e), transpose=transpose)
    assert bf.sync_status(ws) == bf.OK
    ref = oracle.butterfly(x.astype(np.float64), ang, transpose=transpose, expert_of_row=e)
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref).max()
    assert err <= 2e-5 * np.abs(ref).max(), err


@pytest.mark.parametrize("d", [64, 512, 4096])
def test_butterfly_apply_bf16_and_default_expert(bf, d):
    rng = np.random.default_rng(7 * d)
    ang = wl.random_angles(rng, 1, d)
    x = wl.round_to_bf16(rng.standard_normal((9, d)).astype(np.float32))
    y, ws = bf.butterfly_apply(dev(x, torch.bfloat16), dev(ang), None, transpose=False)
    assert bf.sync_status(ws) == bf.OK
    ref = oracle.butterfly(x.astype(np.float64), ang[0])
    check_close(y.float().cpu().numpy(), ref, "bf16 butterfly")


def test_butterfly_apply_zero_rows(bf):
    ang = dev(np.zeros((1, 6, 32), np.float32))
    x = torch.zeros((0, 64), dtype=torch.float32, device="cuda")
    y, ws = bf.butterfly_apply(x, ang)
    assert y.shape == (0, 64) and bf.sync_status(ws) == bf.OK


# --------------------------------------------------------------- forward

def run_forward(bf, inp, k=None):
    k = inp.wl.k if k is None else k
    x = to_x(inp)
    packed = bf.pack_base(dev(inp.w_base), inp.alpha)
    y, ws = bf.forward(x, dev(inp.logits), k, packed, dev(inp.theta), dev(inp.phi))
    st = bf.sync_status(ws)
    return y, ws, st


def oracle_forward(inp, rows=None, k=None):
    k = inp.wl.k if k is None else k
    x, lg = inp.x, inp.logits
    if rows is not None:
        x, lg = x[rows], lg[rows]
    return oracle.forward(x, lg, k, inp.w_base, inp.alpha, inp.theta, inp.phi)


# reduced token counts the oracle finishes in seconds; all span several
# 128-row tiles and end in a ragged tile
REDUCED = {"tiny": 128, "headline": 300, "many_experts": 333, "llm_width": 70, "vit": 201}


@pytest.mark.parametrize("name", list(REDUCED))
def test_forward_matches_oracle(bf, name):
    inp = wl.make_inputs(name, T=REDUCED[name])
    y, ws, st = run_forward(bf, inp)
    assert st == bf.OK
    ref = oracle_forward(inp)
    check_close(y.float().cpu().numpy(), ref, name)
    # routing left in the workspace is bit-exact too
    w = inp.wl
    idx, gates, perm, offsets = bf.forward_routing(ws, w.T, w.d, w.N, w.k)
    ridx, rg, rperm, roff = oracle.route(inp.logits, w.k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(perm.cpu().numpy(), rperm)
    np.testing.assert_array_equal(offsets.cpu().numpy(), roff)


@pytest.mark.parametrize("name", ["headline", "many_experts", "llm_width", "vit"])
def test_forward_full_size_sampled_tokens(bf, name):
    """Full-size workload in the benchmark's launch configuration; the oracle
    checks a sample of tokens (the layer is token-wise, so a token's output
    depends only on its own x and logits)."""
    inp = wl.make_inputs(name)
    y, ws, st = run_forward(bf, inp)
    assert st == bf.OK
    T = inp.wl.T
    rng = np.random.default_rng(99)
    n = 24 if name == "llm_width" else 64
    rows = np.unique(np.concatenate([[0, 1, T - 1, T // 2], rng.choice(T, n, replace=False)]))
    ref = oracle_forward(inp, rows=rows)
    check_close(y.float().cpu().numpy()[rows], ref, name)
    yf = y.float()
    assert torch.isfinite(yf).all()


@pytest.mark.parametrize("d,N,k,T", [(64, 1, 1, 1), (64, 4, 4, 5), (128, 16, 8, 40), (256, 3, 1, 129),
                                     (2048, 8, 2, 33), (4096, 2, 1, 3)])
def test_forward_edge_shapes(bf, d, N, k, T):
    rng = np.random.default_rng(d + N + k + T)
    x = wl.round_to_bf16(rng.standard_normal((T, d)).astype(np.float32))
    w = wl.random_ternary(rng, d)
    th, ph = wl.random_angles(rng, N, d), wl.random_angles(rng, N, d)
    lg = rng.standard_normal((T, N)).astype(np.float32)
    packed = bf.pack_base(dev(w), 0.05)
    y, ws = bf.forward(dev(x, torch.bfloat16), dev(lg), k, packed, dev(th), dev(ph))
    assert bf.sync_status(ws) == bf.OK
    ref = oracle.forward(x, lg, k, w, 0.05, th, ph)
    check_close(y.float().cpu().numpy(), ref, f"d={d} N={N} k={k} T={T}")


def test_forward_all_tokens_one_expert_and_zero_angles(bf):
    """Zero angles reduce every expert to alpha W_base; one crowded bucket."""
    rng = np.random.default_rng(12)
    T, d, N, k = 260, 512, 8, 1
    x = wl.round_to_bf16(rng.standard_normal((T, d)).astype(np.float32))
    w = wl.random_ternary(rng, d)
    zero = np.zeros((N, 9, d // 2), np.float32)
    lg = rng.standard_normal((T, N)).astype(np.float32)
    lg[:, 6] = 50.0
    packed = bf.pack_base(dev(w), 0.5)
    y, ws = bf.forward(dev(x, torch.bfloat16), dev(lg), k, packed, dev(zero), dev(zero))
    assert bf.sync_status(ws) == bf.OK
    ref = 0.5 * (x.astype(np.float64) @ w.T.astype(np.float64))
    check_close(y.float().cpu().numpy(), ref, "zero angles")
    _, _, _, offsets = bf.forward_routing(ws, T, d, N, k)
    off = offsets.cpu().numpy()
    assert off[6] == 0 and off[7] == T


def test_forward_nan_logit_reports_nonfinite(bf):
    inp = wl.make_inputs("tiny", T=50)
    inp.logits[3, 2] = np.nan
    _, _, st = run_forward(bf, inp)
    assert st == bf.ERR_NONFINITE


def test_forward_twice_same_workspace_is_deterministic(bf):
    inp = wl.make_inputs("headline", T=200)
    x = to_x(inp)
    packed = bf.pack_base(dev(inp.w_base), inp.alpha)
    lg, th, ph = dev(inp.logits), dev(inp.theta), dev(inp.phi)
    y1, ws = bf.forward(x, lg, 2, packed, th, ph)
    y2, _ = bf.forward(x, lg, 2, packed, th, ph, ws=ws)
    assert bf.sync_status(ws) == bf.OK
    assert torch.equal(y1, y2)


def test_forward_workspace_header_garbage_and_graph_replay(bf):
    # the status / barrier words of a fresh workspace may hold anything, and
    # a graph replays the same launch (same barrier token) back to back
    inp = wl.make_inputs("headline", T=300)
    x = to_x(inp)
    packed = bf.pack_base(dev(inp.w_base), inp.alpha)
    lg, th, ph = dev(inp.logits), dev(inp.theta), dev(inp.phi)
    ref, ws0 = bf.forward(x, lg, 2, packed, th, ph)
    assert bf.sync_status(ws0) == bf.OK
    ws = torch.full_like(ws0, 0xA5)
    y, _ = bf.forward(x, lg, 2, packed, th, ph, ws=ws)
    assert bf.sync_status(ws) == bf.OK
    assert torch.equal(y, ref)
    stream = torch.cuda.Stream()
    out = torch.empty_like(ref)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        bf.forward(x, lg, 2, packed, th, ph, ws=ws, out=out, stream=stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            bf.forward(x, lg, 2, packed, th, ph, ws=ws, out=out, stream=stream)
        for _ in range(3):
            out.zero_()
            g.replay()
            stream.synchronize()
            assert torch.equal(out, ref)
    assert bf.sync_status(ws) == bf.OK
    del g


# ------------------------------------------------------ failure detection
# A routing block that never reaches the grid barrier (host-side test hook)
# makes the others' bounded waits run out: the call must report
# BFMOE_ERR_TIMEOUT through the status word, not hang or fault, and the
# context must stay usable.

def test_route_barrier_timeout_reports_status(bf):
    T, N, k = 2000, 16, 2
    lg = np.random.default_rng(21).standard_normal((T, N)).astype(np.float32)
    bf.bfmoe_debug_set(bf.DEBUG_SKIP_ARRIVE_BLOCK, 0)
    try:
        _, _, _, _, ws = bf.route(dev(lg), k)
        st = bf.sync_status(ws)
    finally:
        bf.bfmoe_debug_set(bf.DEBUG_SKIP_ARRIVE_BLOCK, -1)
    assert st == bf.ERR_TIMEOUT
    check_route(bf, lg, k)
    # the barrier words left by the timed-out call are usable again
    idx, gates, perm, offsets, _ = bf.route(dev(lg), k, ws=ws)
    assert bf.sync_status(ws) == bf.OK
    ref = oracle.route(lg, k)
    assert np.array_equal(idx.cpu().numpy(), ref[0])
    assert np.array_equal(perm.cpu().numpy(), ref[2])


def test_forward_barrier_timeout_reports_status(bf):
    inp = wl.make_inputs("headline", T=300)
    bf.bfmoe_debug_set(bf.DEBUG_SKIP_ARRIVE_BLOCK, 1)
    try:
        _, ws_timed_out, st = run_forward(bf, inp)
    finally:
        bf.bfmoe_debug_set(bf.DEBUG_SKIP_ARRIVE_BLOCK, -1)
    assert st == bf.ERR_TIMEOUT
    y, ws, st = run_forward(bf, inp)
    assert st == bf.OK
    ref = oracle_forward(inp)
    check_close(y.float().cpu().numpy(), ref, "after timeout")
    # the same workspace, whose barrier words the timed-out call left behind
    y2, _ = bf.forward(to_x(inp), dev(inp.logits), inp.wl.k, bf.pack_base(dev(inp.w_base), inp.alpha),
                       dev(inp.theta), dev(inp.phi), ws=ws_timed_out)
    assert bf.sync_status(ws_timed_out) == bf.OK
    check_close(y2.float().cpu().numpy(), ref, "same workspace after timeout")
