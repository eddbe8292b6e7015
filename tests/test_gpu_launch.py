"""Launch shapes (ss1_last_launch): each path launches the kernel and grid it is meant to.

Regression guards for how the layer uses the machine: the large-M tensor-core kernel is one
persistent CTA per SM; the decode kernel splits K over a thread-block cluster when its N-blocks
alone would leave most SMs idle, with every cluster resident at once; the fp32 layer splits K
over a cluster too. Each launch is also checked against the oracle on a few rows, so a shape
change cannot hide a wrong result.
"""

import numpy as np
import pytest
import torch

import oracle as O
from tests._parity import row_normalised_max_err
from tests.gpu_common import get_ss1, to_np64

pytestmark = pytest.mark.gpu


def _run(ss1, K, N, c, BK, BN, M, dtype=torch.bfloat16, seed=5):
    layer = ss1.SS1Layer(K, N, c, BK, BN, seed=seed)
    gen = torch.Generator().manual_seed(seed)
    X = torch.randn(M, K, generator=gen).to(dtype)
    Wc = (torch.randn(N, K // c, generator=gen) / np.sqrt(K)).to(dtype)
    Y = layer.forward(X.cuda(), Wc.cuda())
    torch.cuda.synchronize()
    info = ss1.last_launch()
    rows = sorted({0, M - 1, M // 2})
    h, g = O.ss1_tables(K, N, c, BK, BN, seed)
    ref = O.ss1_forward(to_np64(X[rows]), to_np64(Wc), h, g, BN)
    tol = 2e-2 if dtype == torch.bfloat16 else 1e-4
    assert row_normalised_max_err(to_np64(Y.cpu()[rows]), ref) <= tol
    layer.close()
    return info


def test_large_m_is_one_persistent_cta_per_sm():
    ss1 = get_ss1()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    info = _run(ss1, 4096, 4096, 2, 256, 128, 1024)
    assert info["kernel"] == "tc3"
    assert info["grid"] == (min(sms, 8 * 32), 1) and info["cluster_y"] == 1


@pytest.mark.parametrize("N", [1024, 4096, 14336])
def test_decode_splits_k_over_resident_clusters(N):
    ss1 = get_ss1()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    info = _run(ss1, 4096, N, 2, 256, 128, 1)
    nb, splits = info["grid"]
    assert info["kernel"] == "dec" and nb == N // 128
    assert info["cluster_y"] == splits
    fit = info["resident_clusters"]
    assert fit[1] > 0, "the occupancy query behind the split choice ran"
    if nb * 2 <= sms:   # few N-blocks: K is split, and all clusters fit at once
        assert splits > 1
    assert fit[splits] >= nb or splits == 1


def test_fp32_layer_splits_k_over_a_cluster():
    ss1 = get_ss1()
    info = _run(ss1, 768, 768, 2, 64, 64, 64, dtype=torch.float32, seed=0)
    tiles, splits = info["grid"]
    assert info["kernel"] == "simt" and splits > 1 and info["cluster_y"] == splits
    assert info["resident_clusters"][splits] >= tiles
