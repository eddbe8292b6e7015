"""Pins of the CPU oracle against facts fixed outside it.

Each test names what it pins and the mistake it is there to catch. Nothing here calls the
CUDA library.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle as O


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------- generator

def test_splitmix64_published_vector(golden_dir):
    """Published SplitMix64 sequence for seed 1234567 (catches a wrong constant or shift)."""
    kat = _load(golden_dir, "splitmix64_kat.json")
    got = [int(O.splitmix64_draws(np.uint64(kat["seed"]), t)) for t in range(5)]
    assert got == [int(v) for v in kat["outputs"]]


def test_draws_are_counter_based():
    """draw(key, t) equals the t-th output of the sequential generator for every t."""
    key = np.uint64(0xDEADBEEFCAFEF00D)
    state = int(key)
    for t in range(50):
        state = (state + O.GAMMA) % (1 << 64)
        assert int(O.splitmix64_draws(key, t)) == int(O.mix64(np.uint64(state)))


def test_fisher_yates_is_uniform():
    """All 24 permutations of 4 items appear equally often over many independent blocks.

    A Sattolo-style off-by-one (j in [0, i)) yields only the 6 cyclic permutations, and a
    naive 'swap with any position' shuffle is biased; both fail the chi-square bound.
    """
    n = 48000
    keys = O.block_key(12345, np.arange(n))
    perm = O.block_permutation(keys, 4)
    counts = {}
    for p in map(tuple, perm):
        counts[p] = counts.get(p, 0) + 1
    assert len(counts) == 24
    exp = n / 24
    chi2 = sum((v - exp) ** 2 / exp for v in counts.values())
    assert chi2 < 60.0  # 23 dof: P(chi2 > 60) ~ 4e-5


def test_fisher_yates_positions_uniform_bk128():
    """Each value lands in each position with probability 1/BK (BK = 128)."""
    BK, n = 128, 4000
    perm = O.block_permutation(O.block_key(7, np.arange(n)), BK)
    for row in perm[:50]:
        assert sorted(row.tolist()) == list(range(BK))
    # position of value 0 and of value BK-1: uniform over [0, BK)
    for v in (0, BK - 1):
        pos = np.argmax(perm == v, axis=1)
        hist = np.bincount(pos // 16, minlength=8)
        exp = n / 8
        chi2 = float(((hist - exp) ** 2 / exp).sum())
        assert chi2 < 30.0  # 7 dof


def test_signs_balanced():
    g = O.block_signs(O.block_key(99, np.arange(2000)), 64).astype(np.int64)
    frac = (g == 1).mean()
    assert abs(frac - 0.5) < 0.01
    assert set(np.unique(g).tolist()) == {-1, 1}


def test_signs_independent_of_permutation():
    """A block's signs are drawn apart from its shuffle. With BK = 4 the first shuffle step
    puts its pick j (in [0, 3]) at position 3 and no later step moves it, so perm[3] is that
    draw's result; (perm[3], g[0]) must be uniform over its 8 cells. Signs that reuse the
    shuffle's draws (g from draw k instead of draw BK - 1 + k) tie g[0] to j and fail."""
    n = 40000
    keys = O.block_key(31, np.arange(n))
    perm = O.block_permutation(keys, 4)
    g = O.block_signs(keys, 4)
    cell = perm[:, 3] * 2 + (g[:, 0] > 0)
    hist = np.bincount(cell, minlength=8)
    exp = n / 8
    chi2 = float(((hist - exp) ** 2 / exp).sum())
    assert chi2 < 30.0  # 7 dof: P(chi2 > 30) ~ 1e-4


# ---------------------------------------------------------------------------- tables

@pytest.mark.parametrize("K,N,c,BK,BN,seed", [
    (768, 768, 2, 64, 64, 0),
    (1280, 512, 4, 128, 128, 2),
    (1024, 256, 8, 256, 128, 3),
    (512, 256, 8, 128, 128, 4),
    (512, 256, 1, 128, 128, 4),
])
def test_table_invariants(K, N, c, BK, BN, seed):
    """Every chunk maps onto its own S columns, exactly c inputs per column, signs +-1."""
    h, g = O.ss1_tables(K, N, c, BK, BN, seed)
    NB, KC, S = N // BN, K // BK, BK // c
    assert h.shape == (NB, K) and g.shape == (NB, K)
    assert set(np.unique(g).tolist()) <= {-1, 1}
    for nb in range(NB):
        for kc in range(KC):
            hh = h[nb, kc * BK:(kc + 1) * BK]
            assert hh.min() >= kc * S and hh.max() < (kc + 1) * S
            assert np.all(np.bincount(hh - kc * S, minlength=S) == c)
    if c == 1:
        assert np.array_equal(h, np.broadcast_to(np.arange(K), (NB, K)))
        assert np.all(g == 1)


def test_tables_independent_per_block_and_seed():
    h, g = O.ss1_tables(1024, 512, 2, 128, 128, 5)
    blocks = [(h[nb, kc * 128:(kc + 1) * 128] - kc * 64).tobytes() for nb in range(4) for kc in range(8)]
    assert len(set(blocks)) == len(blocks)
    h2, _ = O.ss1_tables(1024, 512, 2, 128, 128, 6)
    assert not np.array_equal(h, h2)
    h3, g3 = O.ss1_tables(1024, 512, 2, 128, 128, 5)
    assert np.array_equal(h, h3) and np.array_equal(g, g3)


def test_fold_is_mod_S():
    """hl(k) = perm[k] mod S: recomputed from the permutation of one block."""
    K, N, c, BK, BN, seed = 256, 128, 4, 128, 128, 11
    h, _ = O.ss1_tables(K, N, c, BK, BN, seed)
    S = BK // c
    perm = O.block_permutation(O.block_key(seed, [1]), BK)[0]   # block id 1 = (nb 0, kc 1)
    assert np.array_equal(h[0, BK:2 * BK] - S, perm % S)


def test_tables_regression(golden_dir):
    ref = _load(golden_dir, "tables_regression.json")
    for case in ref["cases"]:
        K, N, c, BK, BN, seed = (case[k] for k in ("K", "N", "c", "BK", "BN", "seed"))
        h, g = O.ss1_tables(K, N, c, BK, BN, seed)
        assert h[0, :BK].tolist() == case["h_nb0_kc0"]
        assert g[0, :BK].tolist() == case["g_nb0_kc0"]
        assert h[-1, K - BK:K - BK + 16].tolist() == case["h_last16"]
        assert g[-1, K - BK:K - BK + 16].tolist() == case["g_last16"]


@pytest.mark.parametrize("c", [1, 2, 4, 8])
def test_sketch_gram_identity(c):
    """S^T S = c I for every block's sketch operator (count-sketch with balanced buckets)."""
    K, N, BK, BN = 512, 256, 128, 128
    h, g = O.ss1_tables(K, N, c, BK, BN, 3)
    for nb in range(N // BN):
        Sk = O.sketch_matrix(h, g, nb, K, K // c)
        assert np.array_equal(Sk.T @ Sk, c * np.eye(K // c))


# ---------------------------------------------------------------------------- forward

def test_handworked_examples(golden_dir):
    ref = _load(golden_dir, "handworked_forward.json")
    for case in ref["cases"]:
        h = np.array(case["h"], dtype=np.int32)
        g = np.array(case["g"], dtype=np.int8)
        X = np.array(case["X"], dtype=np.float64)
        Wc = np.array(case["Wc"], dtype=np.float64)
        want = np.array(case["Y"], dtype=np.float64)
        assert np.array_equal(O.ss1_forward(X, Wc, h, g, case["BN"]), want), case["name"]
        assert np.array_equal(O.ss1_forward_sketch(X, Wc, h, g, case["BN"]), want), case["name"]


def test_c1_is_dense_gemm():
    """With c = 1 (identity hash) the layer is X Wc^T (catches a transposed operand)."""
    rng = np.random.default_rng(0)
    M, K, N = 7, 256, 384
    X = rng.standard_normal((M, K))
    Wc = rng.standard_normal((N, K))
    h, g = O.ss1_tables(K, N, 1, 128, 128, 4)
    np.testing.assert_allclose(O.ss1_forward(X, Wc, h, g, 128), X @ Wc.T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("K,N,c,BK,BN", [(64, 32, 2, 16, 8), (256, 256, 4, 64, 64), (512, 256, 8, 256, 128),
                                         (768, 768, 2, 64, 64)])
def test_two_routes_agree(K, N, c, BK, BN):
    """Definition (expanded tied weight) and sketch-then-multiply agree to fp64 rounding."""
    rng = np.random.default_rng(K + N + c)
    X = rng.standard_normal((9, K))
    Wc = rng.standard_normal((N, K // c))
    h, g = O.ss1_tables(K, N, c, BK, BN, 1)
    a = O.ss1_forward(X, Wc, h, g, BN)
    b = O.ss1_forward_sketch(X, Wc, h, g, BN)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-11 * np.abs(a).max())


@pytest.mark.parametrize("c", [1, 2, 4, 8])
def test_frobenius_identity(c):
    """Each row of the tied weight holds every Wc entry of its row exactly c times, +-1:
    ||W_full[n,:]||^2 = c ||Wc[n,:]||^2 (catches a dropped or duplicated term)."""
    K, N, BK, BN = 512, 256, 128, 128
    rng = np.random.default_rng(c)
    Wc = rng.standard_normal((N, K // c))
    h, g = O.ss1_tables(K, N, c, BK, BN, 8)
    W = np.concatenate([O.expand_weight(Wc, h, g, BN, nb) for nb in range(N // BN)])
    np.testing.assert_allclose((W ** 2).sum(1), c * (Wc ** 2).sum(1), rtol=1e-12)


def test_one_hot_probe_structure():
    """Probing the forward with the identity (X = I_K) returns the tied weight. With all Wc
    entries distinct, each probed value decodes to one (n, j): j must lie in the chunk's
    column range, every j of a chunk must appear exactly c times per neuron, the map must be
    the same for the neurons of one block and differ between blocks."""
    K, N, c, BK, BN = 256, 64, 4, 64, 16
    Kc = K // c
    Wc = (np.arange(N)[:, None] * 1000 + np.arange(Kc)[None, :] + 1).astype(np.float64)
    h, g = O.ss1_tables(K, N, c, BK, BN, 21)
    Wt = O.ss1_forward(np.eye(K), Wc, h, g, BN)            # [K, N] = W_full^T
    mag = np.abs(Wt)
    nrow = (mag // 1000).astype(np.int64)
    j = (mag - nrow * 1000 - 1).astype(np.int64)
    assert np.all(nrow == np.arange(N)[None, :])
    S = BK // c
    maps = []
    for n in range(N):
        col = j[:, n]
        for kc in range(K // BK):
            seg = col[kc * BK:(kc + 1) * BK]
            assert seg.min() >= kc * S and seg.max() < (kc + 1) * S
            assert np.all(np.bincount(seg - kc * S, minlength=S) == c)
        maps.append((col.tobytes(), np.sign(Wt[:, n]).tobytes()))
    for nb in range(N // BN):
        assert len(set(maps[nb * BN:(nb + 1) * BN])) == 1
    assert len(set(maps[::BN])) == N // BN


def test_linearity_and_sign_symmetry():
    rng = np.random.default_rng(5)
    K, N, c, BK, BN = 256, 128, 2, 128, 64
    h, g = O.ss1_tables(K, N, c, BK, BN, 2)
    Wc = rng.standard_normal((N, K // c))
    X1, X2 = rng.standard_normal((4, K)), rng.standard_normal((4, K))
    f = lambda X: O.ss1_forward(X, Wc, h, g, BN)  # noqa: E731
    np.testing.assert_allclose(f(2.5 * X1 - 1.5 * X2), 2.5 * f(X1) - 1.5 * f(X2), rtol=1e-10, atol=1e-10)
    assert np.array_equal(f(np.zeros((3, K))), np.zeros((3, N)))
    assert np.array_equal(f(-X1), -f(X1))


def test_rows_sample_matches_full():
    rng = np.random.default_rng(6)
    K, N, c, BK, BN = 256, 256, 4, 128, 128
    h, g = O.ss1_tables(K, N, c, BK, BN, 2)
    X = rng.standard_normal((33, K))
    Wc = rng.standard_normal((N, K // c))
    full = O.ss1_forward(X, Wc, h, g, BN)
    rows = [0, 5, 32]
    assert np.array_equal(O.ss1_forward_rows(X, Wc, h, g, BN, rows), full[rows])


# ---------------------------------------------------------------------------- projection

def test_projection_at_c1_is_identity():
    """c = 1: every slot holds one input with sign +1, so projecting W returns W itself."""
    rng = np.random.default_rng(8)
    K, N, BK, BN = 256, 64, 64, 32
    h, g = O.ss1_tables(K, N, 1, BK, BN, 4)
    W = rng.standard_normal((N, K))
    assert np.array_equal(O.project_dense(W, h, g, BN, 1), W)


def test_projection_recovers_tied_weights():
    """Projecting an SS1 tied weight returns its Wc; the residual of a dense W is
    orthogonal to the SS1 subspace (least squares, from S^T S = c I)."""
    rng = np.random.default_rng(7)
    K, N, c, BK, BN = 256, 128, 4, 64, 32
    h, g = O.ss1_tables(K, N, c, BK, BN, 9)
    Wc = rng.standard_normal((N, K // c))
    Wfull = np.concatenate([O.expand_weight(Wc, h, g, BN, nb) for nb in range(N // BN)])
    np.testing.assert_allclose(O.project_dense(Wfull, h, g, BN, c), Wc, rtol=1e-12, atol=1e-12)
    W = rng.standard_normal((N, K))
    P = O.project_dense(W, h, g, BN, c)
    Wp = np.concatenate([O.expand_weight(P, h, g, BN, nb) for nb in range(N // BN)])
    R = W - Wp
    # residual is orthogonal to every tied direction: projecting it gives zero
    np.testing.assert_allclose(O.project_dense(R, h, g, BN, c), 0.0, atol=1e-12)
    assert math.isclose((W * W).sum(), (Wp * Wp).sum() + (R * R).sum(), rel_tol=1e-12)


# ---------------------------------------------------------------------------- backward

def _loss_pieces(seed, M=3, K=16, N=8, c=2, BK=8, BN=4):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    Wc = rng.standard_normal((N, K // c))
    R = rng.standard_normal((M, N))          # loss L = sum(R * Y), so dL/dY = R
    h, g = O.ss1_tables(K, N, c, BK, BN, seed)
    return X, Wc, R, h, g


@pytest.mark.parametrize("c,BK,BN", [(2, 8, 4), (4, 8, 8), (1, 4, 4), (8, 16, 4)])
def test_backward_input_finite_differences(c, BK, BN):
    """dX from the oracle against central differences of L(X) = sum(R * Y(X)) in float64. L is
    linear in X, so the central difference is exact up to rounding; a transposed operand, a
    missing sign or the wrong N-block's tables all change dX by O(1)."""
    X, Wc, R, h, g = _loss_pieces(7 + c, c=c, BK=BK, BN=BN)
    dX = O.ss1_backward_input(R, Wc, h, g, BN)
    eps = 0.5
    num = np.empty_like(X)
    for m in range(X.shape[0]):
        for k in range(X.shape[1]):
            E = np.zeros_like(X)
            E[m, k] = eps
            num[m, k] = (np.sum(R * O.ss1_forward(X + E, Wc, h, g, BN)) -
                         np.sum(R * O.ss1_forward(X - E, Wc, h, g, BN))) / (2 * eps)
    assert np.allclose(dX, num, rtol=0, atol=1e-12)


@pytest.mark.parametrize("c,BK,BN", [(2, 8, 4), (4, 8, 8), (1, 4, 4), (8, 16, 4)])
def test_backward_weight_finite_differences(c, BK, BN):
    """dWc against central differences of L(Wc) = sum(R * Y(Wc)): the chain rule through the
    tying must collect every input k of a slot with its sign, in the slot's own N-block."""
    X, Wc, R, h, g = _loss_pieces(11 + c, c=c, BK=BK, BN=BN)
    dWc = O.ss1_backward_weight(X, R, h, g, BN, Wc.shape[1])
    eps = 0.5
    num = np.empty_like(Wc)
    for n in range(Wc.shape[0]):
        for j in range(Wc.shape[1]):
            E = np.zeros_like(Wc)
            E[n, j] = eps
            num[n, j] = (np.sum(R * O.ss1_forward(X, Wc + E, h, g, BN)) -
                         np.sum(R * O.ss1_forward(X, Wc - E, h, g, BN))) / (2 * eps)
    assert np.allclose(dWc, num, rtol=0, atol=1e-12)


def test_backward_c1_is_plain_matrix_calculus():
    """With the identity hash the layer is Y = X Wc^T, so dX = dY Wc and dWc = dY^T X."""
    rng = np.random.default_rng(3)
    M, K, N = 5, 12, 8
    X, Wc, dY = rng.standard_normal((M, K)), rng.standard_normal((N, K)), rng.standard_normal((M, N))
    h, g = O.ss1_tables(K, N, 1, 4, 4, 9)
    assert np.allclose(O.ss1_backward_input(dY, Wc, h, g, 4), dY @ Wc, atol=1e-12)
    assert np.allclose(O.ss1_backward_weight(X, dY, h, g, 4, K), dY.T @ X, atol=1e-12)


def test_backward_weight_is_c_times_projection_of_dense_gradient():
    """The tied-sum of the dense gradient equals c times the least-squares projection of it
    (the projection divides the same signed sum by c): ties the two oracle functions together."""
    X, Wc, R, h, g = _loss_pieces(5, M=6, K=32, N=8, c=4, BK=16, BN=4)
    dWc = O.ss1_backward_weight(X, R, h, g, 4, Wc.shape[1])
    assert np.allclose(dWc, 4 * O.project_dense(R.T @ X, h, g, 4, 4), atol=1e-12)


# ---------------------------------------------------------------------------- FP8 (E4M3)

def test_e4m3_decode_matches_library_and_closed_forms():
    """All 256 codes against torch's float8_e4m3fn (an independent implementation of the OCP
    E4M3 format), plus closed forms: 2^-9 (smallest subnormal), 7 * 2^-9, 2^-6 (smallest
    normal), 1.0 = 0x38, 448 = 0x7E (largest), NaN at 0x7F and 0xFF, sign symmetry."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(ours[ok], lib[ok])
    assert ours[0x01] == 2.0 ** -9 and ours[0x07] == 7 * 2.0 ** -9 and ours[0x08] == 2.0 ** -6
    assert ours[0x38] == 1.0 and ours[0x7E] == 448.0 and ours[0xFE] == -448.0
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF]) and np.sum(np.isnan(ours)) == 2
    assert np.array_equal(ours[0x80:0xFF], -ours[0x00:0x7F])


def test_e4m3_encode_round_trip_ties_and_saturation():
    """encode(decode(c)) == c for every finite code; halfway values go to the even mantissa;
    magnitudes past 448 saturate; random values agree with torch's round-to-nearest-even cast."""
    import torch
    codes = np.arange(256)
    v = O.e4m3_decode(codes)
    ok = ~np.isnan(v)
    assert np.array_equal(O.e4m3_encode(v[ok]), codes[ok].astype(np.uint8))
    # 1.0 (0x38) and 1.125 (0x39): the midpoint 1.0625 goes to 0x38; 1.1875 (between 0x39 and
    # 0x3A) goes to 0x3A; 2^-10 (between 0 and the smallest subnormal) goes to 0
    assert O.e4m3_encode(1.0625) == 0x38 and O.e4m3_encode(1.1875) == 0x3A and O.e4m3_encode(2.0 ** -10) == 0
    assert O.e4m3_encode(1000.0) == 0x7E and O.e4m3_encode(-449.0) == 0xFE
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(20000) * np.exp2(rng.uniform(-12, 8, 20000))).clip(-448, 448).astype(np.float32)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x), lib)


def test_quantize_rows_and_fp8_forward():
    """Each row's largest |Wc| maps to +-448 (code 0x7E / 0xFE); the dequantised weight is within
    half an E4M3 step (2^-4 relative) of Wc; the FP8 forward with scale 1 on codes of exactly
    representable weights is the plain forward."""
    rng = np.random.default_rng(1)
    Wc = rng.standard_normal((16, 24)).astype(np.float32) * 0.02
    Wq, scale = O.quantize_rows_e4m3(Wc)
    assert scale.dtype == np.float32 and Wq.dtype == np.uint8
    big = np.argmax(np.abs(Wc), axis=1)
    assert all((Wq[n, big[n]] & 0x7F) == 0x7E for n in range(16))
    deq = O.e4m3_decode(Wq) * scale[:, None].astype(np.float64)
    assert (np.abs(deq - Wc) <= 2.0 ** -4 * np.abs(Wc) + 2.0 ** -10 * scale[:, None]).all()
    h, g = O.ss1_tables(48, 16, 2, 16, 8, 4)
    X = rng.standard_normal((3, 48))
    W_exact = O.e4m3_decode(rng.integers(0, 0x7E, size=(16, 24)))
    Y8 = O.ss1_forward_fp8(X, O.e4m3_encode(W_exact), np.ones(16, np.float32), h, g, 8)
    assert np.array_equal(Y8, O.ss1_forward(X, W_exact, h, g, 8))
    # the scale of neuron n multiplies output column n alone, linearly
    one_hot = np.zeros(16, np.float32)
    one_hot[5] = 4.0
    Ys = O.ss1_forward_fp8(X, O.e4m3_encode(W_exact), one_hot, h, g, 8)
    assert np.array_equal(Ys[:, 5], 4.0 * Y8[:, 5]) and np.count_nonzero(np.delete(Ys, 5, axis=1)) == 0


# ---------------------------------------------------------------------------- bias, activation, chain

def test_activations_closed_forms():
    """ReLU clamps at zero; GELU(0) = 0, GELU(x) -> x for large x and -> 0 for very negative x,
    GELU(1) = Phi(1) = 0.8413447460685429 (the normal distribution function at 1, a tabulated
    value), and GELU(x) - GELU(-x) = x (Phi(x) + Phi(-x) = 1)."""
    v = np.array([-3.0, -0.5, 0.0, 0.25, 2.0])
    assert np.array_equal(O.activation(v, O.ACT_RELU), [0.0, 0.0, 0.0, 0.25, 2.0])
    assert np.array_equal(O.activation(v, O.ACT_NONE), v)
    gl = O.activation(np.array([0.0, 1.0, 12.0, -12.0]), O.ACT_GELU)
    assert gl[0] == 0.0 and abs(gl[1] - 0.8413447460685429) < 1e-15
    assert abs(gl[2] - 12.0) < 1e-12 and abs(gl[3]) < 1e-12
    x = np.linspace(-4, 4, 41)
    assert np.allclose(O.activation(x, O.ACT_GELU) - O.activation(-x, O.ACT_GELU), x, atol=1e-14)


def test_bias_act_layer():
    """With X = 0 the layer gives act(bias) exactly; with zero bias and no activation it is the
    plain forward; the bias of neuron n shifts column n alone."""
    rng = np.random.default_rng(2)
    K, N, c, BK, BN = 32, 16, 2, 16, 8
    h, g = O.ss1_tables(K, N, c, BK, BN, 3)
    Wc = rng.standard_normal((N, K // c))
    X = rng.standard_normal((5, K))
    b = rng.standard_normal(N)
    for act in (O.ACT_NONE, O.ACT_RELU, O.ACT_GELU):
        Y0 = O.ss1_forward_bias_act(np.zeros((2, K)), Wc, h, g, BN, b, act)
        assert np.array_equal(Y0, np.tile(O.activation(b, act), (2, 1)))
    assert np.array_equal(O.ss1_forward_bias_act(X, Wc, h, g, BN, None, O.ACT_NONE), O.ss1_forward(X, Wc, h, g, BN))
    e = np.zeros(N)
    e[3] = 1.5
    d = O.ss1_forward_bias_act(X, Wc, h, g, BN, e, O.ACT_NONE) - O.ss1_forward(X, Wc, h, g, BN)
    assert np.allclose(d[:, 3], 1.5, atol=1e-14) and np.count_nonzero(np.delete(d, 3, axis=1)) == 0


def test_chain_is_composition():
    """Each output of the chain is the next layer's input: layer 2 of the chain equals one layer
    applied to layer 1's output."""
    rng = np.random.default_rng(4)
    dims = [32, 16, 16, 8]
    layers = []
    for i in range(3):
        h, g = O.ss1_tables(dims[i], dims[i + 1], 2, 16, 8, 4)
        layers.append((rng.standard_normal((dims[i + 1], dims[i] // 2)), h, g, 8, rng.standard_normal(dims[i + 1]),
                       O.ACT_RELU if i < 2 else O.ACT_NONE))
    X = rng.standard_normal((6, 32))
    outs = O.ss1_chain_forward(X, layers)
    assert [o.shape for o in outs] == [(6, 16), (6, 16), (6, 8)]
    W, h, g, BN, b, act = layers[1]
    assert np.array_equal(outs[1], O.ss1_forward_bias_act(outs[0], W, h, g, BN, b, act))
    assert (outs[0] >= 0).all() and (outs[1] >= 0).all()
