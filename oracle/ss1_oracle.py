"""CPU oracle for the forward pass of the SS1 (Sketch Structured Transform) linear layer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module. The CUDA library never calls it and
shares no code, table or constant generator with it: everything here is written from the
definitions below, in float64 / exact integers, with no blocking, fusion or reordering.

What the layer computes
-----------------------
Source: "SS1: Accelerating Inference with Fast and Expressive Sketch Structured Transform"
(atlas.scime.ai paper summary), section "Approach"; and the SS1 abstract on the dblp author
page (taxoreview.com, dblp:18/8339). Random parameter sharing is confined to the weight
vector of one neuron through K- and N-coalescing hash functions; the input is first
sketched -- shrunk by the compression factor c through signed additions -- and the sketch
is multiplied with the compressed weights.

The pages print no formula, so the following reading is used (the plainest one the text
supports):

* Neurons are grouped into N-blocks of BN consecutive outputs (nb = n // BN, the
  "N-coalescing" part: one hash per block, shared by its BN neurons). Inputs are split
  into K-chunks of BK consecutive coordinates (kc = k // BK).
* For every (nb, kc) a hash maps the BK coordinates of the chunk onto S = BK / c slots,
  exactly c coordinates per slot, each with a sign +1 / -1, drawn independently per
  (nb, kc) (the "K-coalescing" part; independence keeps neurons of different blocks
  apart).
* Compressed column j = kc * S + s holds slot s of chunk kc, so Wc has shape [N, K / c].
* The layer is exactly a dense linear layer whose weight is the tied, expanded matrix
      W_full[n, k] = g_nb(k) * Wc[n, h_nb(k)]            (nb = n // BN)
      Y[m, n]      = sum_k X[m, k] * W_full[n, k]
  and the sketch-then-multiply route of the page reaches the same Y because
      sum_k X[m,k] g(k) Wc[n,h(k)] = sum_j Wc[n,j] * (sum_{k: h(k)=j} g(k) X[m,k]).
  `ss1_forward` is that definition; `ss1_forward_sketch` is the page's two-step route.

Hash generator (the pages leave the hash family open; this is the fixed reading)
--------------------------------------------------------------------------------
* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
  OOPSLA 2014), used counter-style: draw(key, t) = mix64(key + (t + 1) * GAMMA mod 2^64).
* Block key: key(nb, kc) = seed XOR mix64(nb * KC + kc + 1).
* Permutation of the chunk: Fisher-Yates in Durstenfeld's form. Position i runs from BK-1
  down to 1; the t-th draw (t = BK-1-i) picks j in [0, i] by Lemire's multiply-shift
  reduction without rejection, j = ((r >> 32) * (i + 1)) >> 32, and perm[i], perm[j] swap.
* Signs: the draws t = BK-1 .. 2*BK-2 give g(k) = -1 when bit 63 of the draw is set,
  else +1, for k = 0 .. BK-1 in order.
* Fold: slot hl(k) = perm[k] mod S, so slot s receives the coordinates whose permuted
  position is s, s+S, ..., s+(c-1)S -- exactly c of them.
* c = 1 is the identity hash with all signs +1 and no draws, so the layer reduces to a
  plain dense GEMM Y = X Wc^T.

Parity pins (tests that tie this file to something other than itself): the SplitMix64
published test vector, permutation uniformity statistics, table invariants, the sketch
Gram identity S^T S = c I, a hand-worked example, the c = 1 dense reduction, agreement of
the two forward routes, the Frobenius identity of the tied weight, one-hot probing and
linearity. See tests/test_oracle_*.py.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "GAMMA",
    "mix64",
    "splitmix64_draws",
    "block_key",
    "block_permutation",
    "block_signs",
    "ss1_tables",
    "sketch_matrix",
    "expand_weight",
    "ss1_forward",
    "ss1_forward_rows",
    "ss1_forward_sketch",
    "project_dense",
    "ss1_backward_input",
    "ss1_backward_weight",
    "e4m3_decode",
    "e4m3_encode",
    "quantize_rows_e4m3",
    "ss1_forward_fp8",
    "ACT_NONE",
    "ACT_RELU",
    "ACT_GELU",
    "activation",
    "ss1_forward_bias_act",
    "ss1_chain_forward",
]

_U64 = np.uint64
GAMMA = 0x9E3779B97F4A7C15
_MUL1 = 0xBF58476D1CE4E5B9
_MUL2 = 0x94D049BB133111EB


def mix64(z):
    """SplitMix64 output mixer (Steele, Lea & Flood 2014), on uint64 arrays, wrapping.

    z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
    z ^= z >> 31.
    """
    z = np.asarray(z, dtype=_U64)
    with np.errstate(over="ignore"):
        z = z ^ (z >> _U64(30))
        z = z * _U64(_MUL1)
        z = z ^ (z >> _U64(27))
        z = z * _U64(_MUL2)
        z = z ^ (z >> _U64(31))
    return z


def splitmix64_draws(key, t):
    """The t-th SplitMix64 output (t = 0, 1, ...) of the stream whose state starts at key.

    Sequential SplitMix64 adds GAMMA to its state before each output, so output t is
    mix64(key + (t + 1) * GAMMA); written counter-style here. key: uint64 array.
    """
    key = np.asarray(key, dtype=_U64)
    with np.errstate(over="ignore"):
        state = key + _U64((t + 1) * GAMMA % (1 << 64))
    return mix64(state)


def block_key(seed: int, block_ids):
    """Per-(N-block, K-chunk) stream key: seed XOR mix64(block_id + 1), block_id = nb*KC+kc."""
    ids = np.asarray(block_ids, dtype=_U64)
    with np.errstate(over="ignore"):
        return _U64(seed & 0xFFFFFFFFFFFFFFFF) ^ mix64(ids + _U64(1))


def block_permutation(keys, BK: int):
    """Fisher-Yates (Durstenfeld) permutation of [0, BK) for every key.

    Draw t (t = 0 .. BK-2) serves position i = BK-1-t; j = ((r >> 32) * (i+1)) >> 32
    (Lemire multiply-shift, no rejection) and perm[i] <-> perm[j]. The blocks are
    independent streams, so they are stepped side by side as numpy rows; inside a block
    the steps run in the algorithm's order.
    Returns int64 [len(keys), BK].
    """
    keys = np.atleast_1d(np.asarray(keys, dtype=_U64))
    nblk = keys.shape[0]
    perm = np.tile(np.arange(BK, dtype=np.int64), (nblk, 1))
    rows = np.arange(nblk)
    for t in range(BK - 1):
        i = BK - 1 - t
        r = splitmix64_draws(keys, t)
        with np.errstate(over="ignore"):
            j = (((r >> _U64(32)) * _U64(i + 1)) >> _U64(32)).astype(np.int64)
        pi = perm[:, i].copy()
        perm[:, i] = perm[rows, j]
        perm[rows, j] = pi
    return perm


def block_signs(keys, BK: int):
    """Signs g(k) for k = 0..BK-1 from draws t = BK-1 .. 2BK-2: -1 if bit 63 set, else +1.

    Returns int8 [len(keys), BK].
    """
    keys = np.atleast_1d(np.asarray(keys, dtype=_U64))
    g = np.empty((keys.shape[0], BK), dtype=np.int8)
    for k in range(BK):
        r = splitmix64_draws(keys, BK - 1 + k)
        g[:, k] = np.where((r >> _U64(63)) != 0, -1, 1).astype(np.int8)
    return g


def _check_shape(K: int, N: int, c: int, BK: int, BN: int):
    if K < 1 or N < 1 or c < 1 or BK < 1 or BN < 1:
        raise ValueError("K, N, c, BK, BN must be positive")
    if K % BK or N % BN or BK % c:
        raise ValueError("need K % BK == 0, N % BN == 0, BK % c == 0")


def ss1_tables(K: int, N: int, c: int, BK: int, BN: int, seed: int):
    """Hash and sign tables of one SS1 layer.

    Returns (h, g):
      h: int32 [NB, K], h[nb, k] = kc*S + hl(k), the compressed column that input k feeds
         in N-block nb (kc = k // BK, S = BK // c);
      g: int8  [NB, K], the sign of input k in N-block nb.
    """
    _check_shape(K, N, c, BK, BN)
    NB, KC, S = N // BN, K // BK, BK // c
    h = np.empty((NB, K), dtype=np.int32)
    g = np.empty((NB, K), dtype=np.int8)
    if c == 1:
        h[:] = np.arange(K, dtype=np.int32)[None, :]
        g[:] = 1
        return h, g
    block_ids = np.arange(NB * KC, dtype=np.int64)          # block id = nb * KC + kc
    keys = block_key(seed, block_ids)
    perm = block_permutation(keys, BK)                       # [NB*KC, BK]
    sg = block_signs(keys, BK)                               # [NB*KC, BK]
    hl = perm % S                                            # the fold
    kc = block_ids % KC
    hglob = hl + (kc * S)[:, None]
    h[:] = hglob.reshape(NB, KC * BK).astype(np.int32)
    g[:] = sg.reshape(NB, KC * BK)
    return h, g


def sketch_matrix(h, g, nb: int, K: int, Kc: int):
    """Dense sketch operator of N-block nb: Sk[k, j] = g_nb(k) if h_nb(k) == j else 0.

    Shape [K, K/c] float64. X @ Sk is the sketch of X for that block.
    """
    Sk = np.zeros((K, Kc), dtype=np.float64)
    Sk[np.arange(K), h[nb].astype(np.int64)] = g[nb].astype(np.float64)
    return Sk


def expand_weight(Wc, h, g, BN: int, nb: int):
    """Rows nb*BN .. nb*BN+BN-1 of the tied dense weight: W_full[n, k] = g_nb(k) Wc[n, h_nb(k)].

    Returns float64 [BN, K].
    """
    Wc_blk = np.asarray(Wc, dtype=np.float64)[nb * BN:(nb + 1) * BN]
    return Wc_blk[:, h[nb].astype(np.int64)] * g[nb].astype(np.float64)[None, :]


def ss1_forward(X, Wc, h, g, BN: int):
    """The definition: Y = X W_full^T in float64, one N-block of W_full at a time.

    X: [M, K], Wc: [N, K/c] (any real dtype; widened to float64), h/g from ss1_tables.
    Returns float64 [M, N].
    """
    X = np.asarray(X, dtype=np.float64)
    Wc = np.asarray(Wc, dtype=np.float64)
    M, K = X.shape
    N = Wc.shape[0]
    NB = N // BN
    if h.shape != (NB, K) or g.shape != (NB, K) or N % BN:
        raise ValueError("tables do not match X / Wc / BN")
    Y = np.empty((M, N), dtype=np.float64)
    for nb in range(NB):
        Wf = expand_weight(Wc, h, g, BN, nb)
        Y[:, nb * BN:(nb + 1) * BN] = X @ Wf.T
    return Y


def ss1_forward_rows(X, Wc, h, g, BN: int, rows):
    """The definition evaluated only at the given rows of Y.

    Rows of Y are independent, so a sample of rows is exact for those rows.
    Returns float64 [len(rows), N].
    """
    X = np.asarray(X, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.int64)
    Ys = ss1_forward(X[rows], Wc, h, g, BN)
    return Ys


def ss1_forward_sketch(X, Wc, h, g, BN: int):
    """The page's route: per N-block, sketch the input by signed hashed additions, then
    multiply with the compressed weights of that block. float64 throughout.

    Xs_nb[m, j] = sum over k with h_nb(k) = j of g_nb(k) * X[m, k]   (count-sketch style)
    Y[m, n]     = sum_j Xs_nb[m, j] * Wc[n, j]                          (nb = n // BN)
    """
    X = np.asarray(X, dtype=np.float64)
    Wc = np.asarray(Wc, dtype=np.float64)
    M, K = X.shape
    N, Kc = Wc.shape
    NB = N // BN
    Y = np.empty((M, N), dtype=np.float64)
    for nb in range(NB):
        Xs_t = np.zeros((Kc, M), dtype=np.float64)
        signed_t = (X * g[nb].astype(np.float64)[None, :]).T        # [K, M]
        np.add.at(Xs_t, h[nb].astype(np.int64), signed_t)           # hashed additions
        Y[:, nb * BN:(nb + 1) * BN] = Xs_t.T @ Wc[nb * BN:(nb + 1) * BN].T
    return Y


def project_dense(W, h, g, BN: int, c: int):
    """Least-squares projection of a dense weight W[N, K] onto the SS1 weights of these tables.

    The pages say pre-trained layers can be projected onto SS1 but print no formula. The
    tied weight of block nb is Wc_nb Sk_nb^T, and Sk_nb^T Sk_nb = c I (every slot has
    exactly c unit entries), so the Frobenius-closest Wc is Wc_nb = W_nb Sk_nb / c:
        Wc[n, j] = (1/c) * sum over k with h_nb(k) = j of g_nb(k) * W[n, k].
    Returns float64 [N, K/c].
    """
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    NB = N // BN
    Kc = K // c
    Wc = np.empty((N, Kc), dtype=np.float64)
    for nb in range(NB):
        Sk = sketch_matrix(h, g, nb, K, Kc)
        Wc[nb * BN:(nb + 1) * BN] = (W[nb * BN:(nb + 1) * BN] @ Sk) / c
    return Wc


def ss1_backward_input(dY, Wc, h, g, BN: int):
    """Gradient of a loss with respect to X, given dY = dLoss/dY: since Y = X W_full^T,
    dX = dY W_full, computed in float64 one N-block of W_full at a time.

    The pages say the SS1 backward pass is not made cheaper ("Limitations") and give no
    formula; this is plain matrix calculus on the tied weight. dY: [M, N]; returns [M, K].
    """
    dY = np.asarray(dY, dtype=np.float64)
    Wc = np.asarray(Wc, dtype=np.float64)
    M, N = dY.shape
    K = h.shape[1]
    NB = N // BN
    dX = np.zeros((M, K), dtype=np.float64)
    for nb in range(NB):
        Wf = expand_weight(Wc, h, g, BN, nb)                   # [BN, K]
        dX += dY[:, nb * BN:(nb + 1) * BN] @ Wf
    return dX


def ss1_backward_weight(X, dY, h, g, BN: int, Kc: int):
    """Gradient with respect to the compressed weights. The gradient of the dense weight is
    dW_full = dY^T X; every W_full[n, k] is g_nb(k) * Wc[n, h_nb(k)], so by the chain rule
        dWc[n, j] = sum over k with h_nb(k) == j of g_nb(k) * dW_full[n, k].
    float64; X: [M, K], dY: [M, N]; returns [N, Kc].
    """
    X = np.asarray(X, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    N = dY.shape[1]
    NB = N // BN
    dWfull = dY.T @ X                                          # [N, K]
    dWc = np.zeros((N, Kc), dtype=np.float64)
    for nb in range(NB):
        rows = slice(nb * BN, (nb + 1) * BN)
        signed = dWfull[rows] * g[nb].astype(np.float64)[None, :]
        for k in range(h.shape[1]):                            # collect every input's term in its column
            dWc[rows, h[nb, k]] += signed[:, k]
    return dWc


# ---------------------------------------------------------------------------- FP8 weights
#
# The SS1 page ("Limitations") lists quantised SS1 kernels as not built, and ("Measured
# effects") reports post-training quantisation of SS1 models. This reading stores Wc as FP8
# E4M3 codes with one float32 scale per output neuron: Wc_deq[n, j] = scale[n] * e4m3(Wq[n, j]).
# E4M3 (the OCP 8-bit floating point format): 1 sign bit, 4 exponent bits with bias 7, 3
# mantissa bits; exponent field 0 holds subnormals m/8 * 2^-6; S.1111.111 is NaN; there are no
# infinities, so the largest finite magnitude is 1.75 * 2^8 = 448.

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Exact float64 value of each E4M3 code (uint8 array); NaN for 0x7F and 0xFF."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def e4m3_encode(x):
    """The E4M3 code nearest to each float (ties to the even code), magnitudes above 448
    saturated to +-448 (the conversion's 'satfinite' behaviour). x: finite floats."""
    x = np.asarray(x, dtype=np.float64)
    values = e4m3_decode(np.arange(0x7F))          # the 127 non-negative finite codes, increasing
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(values, a, side="left")   # first code with value >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - values[lo], values[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))   # an even code has an even mantissa
    code = np.where(a == values[hi], hi, np.where(pick_hi, hi, lo)).astype(np.int64)
    return (code | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)


def quantize_rows_e4m3(Wc):
    """Per-row FP8 quantisation: scale[n] = max_j |Wc[n, j]| / 448 computed in float32 (1 for an
    all-zero row), then codes = e4m3_encode(Wc / scale) with the quotient rounded to float32.
    Returns (codes uint8 [N, Kc], scale float32 [N])."""
    W32 = np.asarray(Wc, dtype=np.float32)
    amax = np.abs(W32).max(axis=1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = (W32 / scale[:, None]).astype(np.float32)
    return e4m3_encode(q), scale


def ss1_forward_fp8(X, Wq, scale, h, g, BN: int):
    """The layer with FP8 weights: the definition applied to Wc_deq = scale[n] * e4m3(Wq[n, j])."""
    Wd = e4m3_decode(Wq) * np.asarray(scale, dtype=np.float64)[:, None]
    return ss1_forward(X, Wd, h, g, BN)


# ---------------------------------------------------------------------------- epilogue, chain
#
# The SS1 page ("Measured effects") replaces the DLRM MLPerf top MLP's layers by SS1 layers. The
# layer itself has no bias or activation; an MLP adds both between layers. This reading: a
# per-neuron bias added to the fp64 sum, then the activation, ReLU (max(v, 0)) or GELU in its
# exact form v * Phi(v) = 0.5 v (1 + erf(v / sqrt(2))), written with the library erf.

ACT_NONE, ACT_RELU, ACT_GELU = 0, 1, 2


def activation(v, act: int):
    """The activation of the epilogue on float64 values."""
    v = np.asarray(v, dtype=np.float64)
    if act == ACT_NONE:
        return v
    if act == ACT_RELU:
        return np.maximum(v, 0.0)
    if act == ACT_GELU:
        from math import erf, sqrt
        return 0.5 * v * (1.0 + np.vectorize(erf)(v / sqrt(2.0)))
    raise ValueError(act)


def ss1_forward_bias_act(X, Wc, h, g, BN: int, bias=None, act: int = ACT_NONE):
    """act(SS1(X) + bias) in float64; bias: [N] or None."""
    Y = ss1_forward(X, Wc, h, g, BN)
    if bias is not None:
        Y = Y + np.asarray(bias, dtype=np.float64)[None, :]
    return activation(Y, act)


def ss1_chain_forward(X, layers):
    """A chain of SS1 layers, each the input of the next: layers is a list of
    (Wc, h, g, BN, bias, act). Returns every layer's output (float64, no intermediate rounding)."""
    outs = []
    cur = np.asarray(X, dtype=np.float64)
    for Wc, h, g, BN, bias, act in layers:
        cur = ss1_forward_bias_act(cur, Wc, h, g, BN, bias, act)
        outs.append(cur)
    return outs
