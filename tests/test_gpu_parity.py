"""CUDA path vs CPU oracle, element by element.

Small cases (whole output compared) span several tiles in M and N plus ragged M tails, for
every kernel that supports them. The workloads run at full size in the launch the
benchmark times (automatic kernel choice); there the oracle computes sampled rows.
"""

import numpy as np
import pytest
import torch

from structured_compressed_linear_b200.workloads import WORKLOADS, Layer, make_inputs
from tests.gpu_common import check_layer, get_ss1, sample_rows

pytestmark = pytest.mark.gpu

SIMT, TC, SMALLM = 2, 1, 3


def _small_cases():
    cases = []
    # fp32: the single-layer workload and ragged variants
    for M in (1, 3, 64, 65, 130):
        cases.append(Layer("fp32-small", M, 768, 768, 2, 64, 64, "fp32", "normal", "uniform_invsqrtk", 0))
    cases.append(Layer("fp32-small", 77, 512, 256, 4, 128, 128, "fp32", "normal", "uniform_invsqrtk", 5))
    cases.append(Layer("fp32-small", 33, 256, 192, 1, 64, 64, "fp32", "normal", "uniform_invsqrtk", 5))
    # bf16: every c, both BK of the workloads, ragged M, several N-blocks
    for c in (1, 2, 4, 8):
        for BK in (128, 256):
            for M in (1, 16, 200, 333):
                cases.append(Layer("bf16-small", M, 1024, 384, c, BK, 128, "bf16", "normal", "normal_002", 3))
    cases.append(Layer("bf16-small", 257, 1280, 640, 4, 128, 128, "bf16", "normal_outliers", "uniform_invsqrtk", 2))
    # an even count of N-blocks: the tensor-core kernel pairs N-blocks in one tile (every c, both BK)
    for c in (2, 4, 8):
        for BK in (128, 256):
            for M in (130, 333):
                cases.append(Layer("bf16-small", M, 768, 768, c, BK, 128, "bf16", "normal", "uniform_invsqrtk", 8))
    # decode-sized rows: every row-group width, ragged groups, narrow N-blocks, K past one segment
    for M in (2, 3, 5, 8, 9, 37, 64):
        cases.append(Layer("bf16-small", M, 3072, 320, 2, 128, 64, "bf16", "normal", "normal_002", 4))
    # a K-chunk that is not a power of two (S = 24): outside the small-M kernel's shapes
    cases.append(Layer("bf16-small", 4, 960, 256, 2, 48, 128, "bf16", "normal", "normal_002", 4))
    for c in (1, 4, 8):
        cases.append(Layer("bf16-small", 6, 4608, 256, c, 256, 32, "bf16", "normal_outliers", "normal_002", 6))
    # wide N: the widest neuron group per CTA
    cases.append(Layer("bf16-small", 8, 1024, 19456, 4, 128, 128, "bf16", "normal", "normal_002", 7))
    # c = 1 with N a multiple of 256: the persistent 128 x 256 tile kernel (BK plays no part)
    for M in (1, 130, 333):
        cases.append(Layer("bf16-small", M, 1024, 512, 1, 128, 128, "bf16", "normal", "normal_002", 3))
    cases.append(Layer("bf16-small", 200, 768, 768, 1, 256, 128, "bf16", "normal_outliers", "uniform_invsqrtk", 2))
    return cases


def tc_eligible(L: Layer) -> bool:
    """Documented preconditions of the tensor-core kernel (include/ss1.h)."""
    S = L.BK // L.c
    return (L.dtype == "bf16" and L.BN == 128 and L.BK in (64, 128, 256) and S % 16 == 0 and S >= 16
            and L.K % 8 == 0 and (L.K // L.c) % 8 == 0)


def smallm_eligible(L: Layer) -> bool:
    """Documented preconditions of the small-M kernel (include/ss1.h)."""
    S = L.BK // L.c
    return (L.dtype == "bf16" and 1 <= L.M <= 64 and S >= 8 and S & (S - 1) == 0 and L.BN % 8 == 0
            and L.K % 8 == 0 and (L.K // L.c) % 8 == 0)


def _kernels_for(L: Layer):
    ks = [SIMT]
    if tc_eligible(L):
        ks.append(TC)
    if smallm_eligible(L):
        ks.append(SMALLM)
    return ks


SMALL = [(L, k) for L in _small_cases() for k in _kernels_for(L)]


@pytest.mark.parametrize("L,kernel", SMALL, ids=[f"{L.tag}:{L.BK}:{L.dtype}:k{k}" for L, k in SMALL])
def test_small_parity(L, kernel):
    ss1 = get_ss1()
    check_layer(ss1, L, kernel=kernel)


FULL = [L for wid in sorted(WORKLOADS) for L in WORKLOADS[wid]]


@pytest.mark.parametrize("L", FULL, ids=[L.tag for L in FULL])
def test_workload_parity_sampled(L):
    """Full-size layers, automatic kernel choice, oracle on sampled rows (all outliers too)."""
    ss1 = get_ss1()
    X, Wc = make_inputs(L)
    must = []
    if L.x_dist == "normal_outliers":
        must = torch.nonzero(X.float().abs().amax(dim=1) > 8.0).flatten().tolist()[:64]
    rows = sample_rows(L.M, 48, seed=L.M + L.K, must=must)
    check_layer(ss1, L, kernel=0, rows=rows, X=X, Wc=Wc)


# Multi-wave shapes: more tiles than SMs, not a multiple of them (a partial last wave), ragged M,
# every BK and a c of each kind; the whole output is compared with the oracle.
MULTIWAVE = [
    Layer("multiwave", 8192, 768, 768, 2, 128, 128, "bf16", "normal", "uniform_invsqrtk", 1),
    Layer("multiwave", 8000, 768, 768, 2, 128, 128, "bf16", "normal", "uniform_invsqrtk", 1),
    Layer("multiwave", 4096, 1280, 1280, 4, 128, 128, "bf16", "normal_outliers", "uniform_invsqrtk", 2),
    Layer("multiwave", 4096, 4096, 1024, 2, 256, 128, "bf16", "normal", "normal_002", 3),
    Layer("multiwave", 5000, 3072, 1024, 8, 256, 128, "bf16", "normal", "normal_002", 3),
    # c = 1, 200 tiles of 128 x 256 on 148 SMs: CTAs take two tiles (both accumulators in turn)
    Layer("multiwave", 2500, 512, 2560, 1, 64, 128, "bf16", "normal", "uniform_invsqrtk", 4),
]


@pytest.mark.parametrize("L", MULTIWAVE, ids=[f"{L.tag}:{L.BK}" for L in MULTIWAVE])
def test_multiwave_full_parity(L):
    check_layer(get_ss1(), L, kernel=TC)


# Decode rows whose X range per CTA is too large to copy once, so the decode kernel's unit mode
# runs (each unit's X rows by TMA, boxes of 16 rows with the rows past M read as zero): fewer
# than 16 rows, a K-chunk of whole stages (c = 2) and a stage of whole K-chunks (c = 8).
UNITMODE = [
    Layer("unitmode", M, 4096, 14336, c, 256, 128, "bf16", "normal", "normal_002", 3)
    for c in (2, 8) for M in (8, 13)
]


@pytest.mark.parametrize("L", UNITMODE, ids=[L.tag for L in UNITMODE])
def test_decode_unit_mode_parity(L):
    check_layer(get_ss1(), L, kernel=SMALLM)


# BK = 64 on the tensor-core kernels (the dense kernel at c = 1, the gathering kernel at c = 2
# and 4): no workload uses it, but the automatic choice sends such layers there.
BK64 = [Layer("bk64", M, 1024, 384, c, 64, 128, "bf16", "normal", "normal_002", 12) for c in (1, 2, 4) for M in (130, 333)]


@pytest.mark.parametrize("L", BK64, ids=[f"{L.tag}:c{L.c}:M{L.M}" for L in BK64])
def test_bk64_tensor_core_parity(L):
    check_layer(get_ss1(), L, kernel=TC)
