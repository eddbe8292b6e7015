"""The device table generator reproduces the oracle's tables bit for bit (integer work)."""

import numpy as np
import pytest

import oracle as O
from structured_compressed_linear_b200.workloads import WORKLOADS
from tests.gpu_common import get_ss1

pytestmark = pytest.mark.gpu


def _shapes():
    seen = []
    for layers in WORKLOADS.values():
        for L in layers:
            key = (L.K, L.N, L.c, L.BK, L.BN, L.seed)
            if key not in seen:
                seen.append(key)
    # extra: small chunks, BK = 256 with c = 8 (S = 32), odd seeds, 64-bit seeds
    seen += [(64, 64, 2, 16, 16, 7), (512, 256, 8, 256, 128, 2**63 + 5), (256, 128, 4, 32, 32, 123456789)]
    return seen


@pytest.mark.parametrize("K,N,c,BK,BN,seed", _shapes())
def test_tables_bit_identical(K, N, c, BK, BN, seed):
    ss1 = get_ss1()
    layer = ss1.SS1Layer(K, N, c, BK, BN, seed)
    h_dev, g_dev = layer.tables()
    h_ref, g_ref = O.ss1_tables(K, N, c, BK, BN, seed)
    assert np.array_equal(h_dev, h_ref)
    assert np.array_equal(g_dev, g_ref)
    layer.close()
