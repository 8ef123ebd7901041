"""Pins of the fp64 oracle against what the pages and mathematics fix.

None of these tests re-types the oracle's own loops: each checks a closed
form (Kronecker / Hadamard / single Givens structure), an invariant
(orthogonality, norm), a brute-force definition (full sort for top-k, dense
materialised experts) or a hand-worked fixture.  Citations name the page
title and section of the ButterflyMoE / ButterflyViT summaries.
"""
import math
import os

import numpy as np
import pytest

import oracle
from ternary_moe_butterfly_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rot(a):
    c, s = math.cos(a), math.sin(a)
    return np.array([[c, -s], [s, c]])


def dense_B(angles, transpose=False):
    """Dense matrix of the oracle's butterfly: its action on the identity."""
    d = angles.shape[-1] * 2
    cols = oracle.butterfly(np.eye(d), angles, transpose=transpose)  # rows are B e_i
    return cols.T


# --------------------------------------------------------------- butterfly
# The butterfly matrices are orthogonal products of layered Givens rotations
# with O(d log d) angles (ButterflyMoE summaries, section 2 / 2.2).

@pytest.mark.parametrize("d", [2, 4, 8, 16, 64, 256])
def test_butterfly_is_orthogonal(d):
    rng = np.random.default_rng(d)
    ang = wl.random_angles(rng, 1, d)[0]
    B = dense_B(ang)
    np.testing.assert_allclose(B.T @ B, np.eye(d), atol=1e-12, rtol=0)
    np.testing.assert_allclose(B @ B.T, np.eye(d), atol=1e-12, rtol=0)
    x = rng.standard_normal(d)
    y = oracle.butterfly(x, ang)
    assert abs(np.linalg.norm(y) - np.linalg.norm(x)) <= 1e-12 * np.linalg.norm(x)


@pytest.mark.parametrize("d", [4, 64, 512])
def test_transpose_mode_is_matrix_transpose_and_inverse(d):
    rng = np.random.default_rng(100 + d)
    ang = wl.random_angles(rng, 1, d)[0]
    x = rng.standard_normal((3, d))
    y = oracle.butterfly(x, ang)
    back = oracle.butterfly(y, ang, transpose=True)
    np.testing.assert_allclose(back, x, atol=1e-12 * np.abs(x).max(), rtol=0)
    if d <= 64:
        np.testing.assert_allclose(dense_B(ang, transpose=True), dense_B(ang).T, atol=1e-13, rtol=0)


@pytest.mark.parametrize("d", [2, 8, 64])
def test_constant_angle_per_stage_is_kronecker(d):
    """Stage s rotates along bit s; with one angle a_s per stage the
    butterfly is kron(R(a_{L-1}), ..., R(a_0)) (bit L-1 is the leading
    Kronecker factor)."""
    L = int(math.log2(d))
    rng = np.random.default_rng(7 * d)
    a = rng.uniform(-math.pi, math.pi, L)
    ang = np.repeat(a[:, None], d // 2, axis=1).astype(np.float32)
    expect = np.array([[1.0]])
    for s in reversed(range(L)):
        expect = np.kron(expect, rot(float(ang[s, 0])))
    np.testing.assert_allclose(dense_B(ang), expect, atol=1e-13, rtol=0)


def givens(d, j, h, a):
    G = np.eye(d)
    c, s = math.cos(a), math.sin(a)
    G[j, j], G[j, j + h], G[j + h, j], G[j + h, j + h] = c, -s, s, c
    return G


@pytest.mark.parametrize("d", [8, 64])
def test_single_angle_is_one_givens_rotation(d):
    """A single non-zero angle at (stage s, pair p) gives one Givens rotation
    in the plane (j, j + 2^s), where j is the p-th index with bit s clear.
    This pins the pair numbering and the rotation's sign."""
    L = int(math.log2(d))
    rng = np.random.default_rng(3 + d)
    cases = [(s, p) for s in range(L) for p in range(d // 2)]
    if d > 8:
        cases = [cases[i] for i in rng.choice(len(cases), 40, replace=False)]
    for s, p in cases:
        ang = np.zeros((L, d // 2), np.float32)
        ang[s, p] = np.float32(rng.uniform(-3, 3))
        h = 1 << s
        js = [j for j in range(d) if not (j & h)]
        j = js[p]
        np.testing.assert_allclose(dense_B(ang), givens(d, j, h, float(ang[s, p])), atol=1e-15, rtol=0)


def test_stage_order_stage0_acts_first():
    """B = stage_{L-1} ... stage_0: with a rotation of the plane (0,1) in
    stage 0 and one of (0,2) in stage 1, B = G_{02}(b) G_{01}(a)."""
    d = 4
    ang = np.zeros((2, 2), np.float32)
    ang[0, 0] = np.float32(0.7)   # stage 0, pair 0 -> plane (0, 1)
    ang[1, 0] = np.float32(-1.3)  # stage 1, pair 0 -> plane (0, 2)
    expect = givens(d, 0, 2, float(ang[1, 0])) @ givens(d, 0, 1, float(ang[0, 0]))
    np.testing.assert_allclose(dense_B(ang), expect, atol=1e-15, rtol=0)
    # and B^T is the reverse product with negated angles
    np.testing.assert_allclose(dense_B(ang, transpose=True), expect.T, atol=1e-15, rtol=0)


@pytest.mark.parametrize("d", [2, 16, 128])
def test_all_quarter_pi_is_hadamard(d):
    """All angles pi/4 turn the butterfly into the normalised Sylvester
    Hadamard transform (the static global Hadamard rotation that the
    ButterflyMoE summary, Chinese page, section 1, names as prior art)."""
    L = int(math.log2(d))
    ang = np.full((L, d // 2), math.pi / 4, np.float32)
    H = np.array([[1.0]])
    for _ in range(L):
        H = np.kron(H, np.array([[1.0, -1.0], [1.0, 1.0]]))
    H *= 2.0 ** (-L / 2)
    # angles are fp32(pi/4): compare with the Kronecker form at that angle
    exact = np.array([[1.0]])
    for _ in range(L):
        exact = np.kron(exact, rot(float(np.float32(math.pi / 4))))
    np.testing.assert_allclose(dense_B(ang), exact, atol=1e-13, rtol=0)
    np.testing.assert_allclose(dense_B(ang), H, atol=1e-7, rtol=0)


def test_rows_use_their_own_expert():
    rng = np.random.default_rng(11)
    d, N = 16, 3
    ang = wl.random_angles(rng, N, d)
    x = rng.standard_normal((5, d))
    e = np.array([2, 0, 1, 2, 0], np.int32)
    y = oracle.butterfly(x, ang, transpose=True, expert_of_row=e)
    for r in range(5):
        np.testing.assert_allclose(y[r], dense_B(ang[e[r]]).T @ x[r], atol=1e-13, rtol=0)


# ----------------------------------------------------------------- routing
# A standard top-k gate selects the active experts (ButterflyMoE summary,
# Dutch page, section 2 "Three phases").  Tie and softmax rules are the
# library's (lower index first; softmax over the selected k).

def brute_topk(lrow, k):
    order = sorted(range(len(lrow)), key=lambda e: (-float(lrow[e]), e))
    return order[:k]


@pytest.mark.parametrize("T,N,k", [(50, 8, 1), (50, 8, 2), (40, 64, 4), (30, 5, 5), (20, 300, 8)])
def test_topk_matches_full_sort(T, N, k):
    rng = np.random.default_rng(T * N + k)
    lg = rng.standard_normal((T, N)).astype(np.float32)
    lg[: T // 2] = np.round(lg[: T // 2] * 2) / 2  # many exact ties
    lg[0, :] = 0.0
    lg[1, ::2] = -0.0
    idx, gates, perm, offsets = oracle.route(lg, k)
    for t in range(T):
        assert list(idx[t]) == brute_topk(lg[t], k)


def test_topk_handles_infinities_and_signed_zero():
    lg = np.array([
        [0.0, -0.0, 0.0, -1.0],
        [-np.inf, -np.inf, -np.inf, -np.inf],
        [1.0, np.inf, np.inf, 3.0],
        [-np.inf, 2.0, -np.inf, 2.0],
    ], np.float32)
    idx, gates, _, _ = oracle.route(lg, 2)
    assert idx.tolist() == [[0, 1], [0, 1], [1, 2], [1, 3]]
    np.testing.assert_allclose(gates[0], [0.5, 0.5], rtol=0, atol=1e-15)
    np.testing.assert_allclose(gates[1], [0.5, 0.5], rtol=0, atol=1e-15)  # all -inf: 1/k
    np.testing.assert_allclose(gates[2], [0.5, 0.5], rtol=0, atol=1e-15)  # two +inf share
    np.testing.assert_allclose(gates[3], [0.5, 0.5], rtol=0, atol=1e-15)
    lg2 = np.array([[np.inf, 1.0, 0.0]], np.float32)
    _, g2, _, _ = oracle.route(lg2, 3)
    np.testing.assert_allclose(g2[0], [1.0, 0.0, 0.0], rtol=0, atol=0)


def test_nan_logit_is_rejected():
    lg = np.zeros((3, 4), np.float32)
    lg[2, 1] = np.nan
    with pytest.raises(oracle.OracleError) as e:
        oracle.route(lg, 2)
    assert e.value.code == oracle.ERR_NONFINITE


def test_gates_closed_forms():
    rng = np.random.default_rng(5)
    lg = rng.standard_normal((64, 16)).astype(np.float32) * 3
    _, g1, _, _ = oracle.route(lg, 1)
    assert np.all(g1 == 1.0)
    idx, g2, _, _ = oracle.route(lg, 2)
    for t in range(64):
        l0, l1 = float(lg[t, idx[t, 0]]), float(lg[t, idx[t, 1]])
        sig = 1.0 / (1.0 + math.exp(l1 - l0))  # 2-way softmax is a logistic
        assert abs(g2[t, 0] - sig) < 1e-15 and abs(g2[t, 1] - (1 - sig)) < 1e-15
    idx4, g4, _, _ = oracle.route(lg, 4)
    np.testing.assert_allclose(g4.sum(1), 1.0, atol=1e-15, rtol=0)
    for t in range(64):
        for j in range(1, 4):
            ratio = g4[t, j] / g4[t, 0]
            assert abs(ratio - math.exp(float(lg[t, idx4[t, j]]) - float(lg[t, idx4[t, 0]]))) < 1e-14


@pytest.mark.parametrize("T,N,k", [(100, 8, 2), (257, 64, 2), (64, 16, 1), (33, 256, 8), (0, 4, 2)])
def test_bucketing_invariants(T, N, k):
    rng = np.random.default_rng(T + 17 * N)
    lg = rng.standard_normal((T, N)).astype(np.float32)
    lg[:, 0] += 3.0  # one crowded expert, several empty ones
    idx, _, perm, offsets = oracle.route(lg, k)
    R = T * k
    assert sorted(perm.tolist()) == list(range(R))
    hist = np.bincount(idx.reshape(-1), minlength=N)
    assert offsets[0] == 0 and offsets[N] == R
    np.testing.assert_array_equal(np.diff(offsets), hist)
    keys = [(int(idx.reshape(-1)[i]), i // k) for i in perm]
    assert keys == sorted(keys)
    for e in range(N):
        for pos in range(offsets[e], offsets[e + 1]):
            assert idx.reshape(-1)[perm[pos]] == e


# ----------------------------------------------------------------- packing

def read_pack_golden():
    rows, header = {}, None
    with open(os.path.join(GOLDEN, "pack_d16.txt")) as f:
        for line in f:
            if line.startswith("header"):
                header = bytes(int(b, 16) for b in line.split()[1:])
            elif line.startswith("row"):
                parts = line.split()
                rows[int(parts[1])] = int(parts[-1], 16)
    return header, rows


def test_pack_matches_hand_worked_example():
    header, rows = read_pack_golden()
    d = 16
    w = np.zeros((d, d), np.int8)
    w[0, 0], w[0, 2] = 1, -1
    w[1, :] = 1
    w[2, :] = -1
    w[3, 15] = -1
    w[4, 0::2], w[4, 1::2] = 1, -1
    packed = oracle.pack_base(w, 1.0)
    assert packed.size == 16 + d * d // 4
    assert bytes(packed[:16]) == header
    words = packed[16:].view("<u4")
    for r in range(d):
        assert words[r] == rows.get(r, 0), r


def test_pack_roundtrip_and_rejects_bad_values():
    rng = np.random.default_rng(1)
    w = wl.random_ternary(rng, 64)
    packed = oracle.pack_base(w, 0.125)
    w2, a2 = oracle.unpack_base(packed)
    np.testing.assert_array_equal(w, w2)
    assert a2 == 0.125
    bad = w.copy()
    bad[3, 5] = 2
    with pytest.raises(oracle.OracleError):
        oracle.pack_base(bad, 1.0)


# ----------------------------------------------------------------- forward

def test_zero_angles_reduce_to_scaled_ternary_product():
    """All angles 0: B = I, so each expert is alpha * W_base and the layer is
    sum_j g_j alpha W_base x (the substrate alone)."""
    rng = np.random.default_rng(2)
    T, d, N, k = 20, 64, 6, 2
    x = rng.standard_normal((T, d)).astype(np.float32)
    w = wl.random_ternary(rng, d)
    lg = rng.standard_normal((T, N)).astype(np.float32)
    zero = np.zeros((N, 6, d // 2), np.float32)
    alpha = 0.37
    y = oracle.forward(x, lg, k, w, alpha, zero, zero)
    _, g, _, _ = oracle.route(lg, k)
    expect = (g.sum(1)[:, None] * np.float64(np.float32(alpha))) * (x.astype(np.float64) @ w.T.astype(np.float64))
    np.testing.assert_allclose(y, expect, atol=1e-12 * np.abs(expect).max(), rtol=0)


def dense_B_by_stages(ang):
    """Butterfly as an explicit product of dense per-stage matrices."""
    L, half = ang.shape
    d = 2 * half
    B = np.eye(d)
    for s in range(L):
        h = 1 << s
        S = np.eye(d)
        p = 0
        for j in range(d):
            if j & h:
                continue
            a = float(ang[s, p])
            S[j, j], S[j, j + h], S[j + h, j], S[j + h, j + h] = math.cos(a), -math.sin(a), math.sin(a), math.cos(a)
            p += 1
        B = S @ B
    return B


def test_sequential_equals_materialised_expert():
    """The layer never materialises W_i = B(phi) W_base B(theta)^T (ButterflyMoE
    summaries, section 2 / 2.1); the sequential rotate -> ternary -> rotate
    result must equal the dense materialised expert."""
    inp = wl.make_inputs("tiny")
    x, w, a, th, ph, lg = inp.x[:16], inp.w_base, inp.alpha, inp.theta, inp.phi, inp.logits[:16]
    k = inp.wl.k
    y = oracle.forward(x, lg, k, w, a, th, ph)
    idx, g, _, _ = oracle.route(lg, k)
    Wd = w.astype(np.float64)
    for t in range(x.shape[0]):
        acc = np.zeros(inp.wl.d)
        for j in range(k):
            e = idx[t, j]
            Wi = dense_B_by_stages(ph[e]) @ Wd @ dense_B_by_stages(th[e]).T
            acc += g[t, j] * np.float64(np.float32(a)) * (Wi @ x[t].astype(np.float64))
        np.testing.assert_allclose(y[t], acc, atol=1e-12 * np.abs(acc).max(), rtol=0)


def test_hadamard_rotations_around_identity_base_are_identity():
    """theta = phi = pi/4 everywhere gives B = H (orthogonal Hadamard); with
    W_base = I the expert is H I H^T = I, so y = alpha x for k = 1."""
    d, T, N = 64, 8, 4
    rng = np.random.default_rng(9)
    x = rng.standard_normal((T, d)).astype(np.float32)
    ang = np.full((N, 6, d // 2), np.float32(math.pi / 4), np.float32)
    w = np.eye(d, dtype=np.int8)
    lg = rng.standard_normal((T, N)).astype(np.float32)
    y = oracle.forward(x, lg, 1, w, 2.0, ang, ang)
    np.testing.assert_allclose(y, 2.0 * x.astype(np.float64), atol=1e-12, rtol=0)


def test_memory_model_matches_closed_form_fixture():
    """(d/2) log2 d angles per butterfly, two per expert, plus d^2/4 bytes of
    2-bit base: the O(d^2 + N d log d) memory of the ButterflyMoE summaries,
    section 2."""
    with open(os.path.join(GOLDEN, "memory_model.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for d, N, apb, lb, dense in (map(int, r) for r in rows):
        assert oracle.angles_per_butterfly(d) == apb
        assert oracle.layer_bytes(d, N) == lb
        assert N * d * d * 4 == dense
        # the stored arrays have exactly that size
        th = np.zeros((N, int(math.log2(d)), d // 2), np.float32)
        assert oracle.packed_base_bytes(d) + 2 * th.nbytes == lb
    # d = 512, N = 64: about 1.19 MiB against 64 MiB of dense fp32 experts
    assert abs(oracle.layer_bytes(512, 64) / 2**20 - 1.1875) < 1e-3
