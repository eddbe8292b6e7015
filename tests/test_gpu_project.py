"""ss1_project (dense -> SS1 projection) against the CPU oracle, through the C ABI.

The oracle's project_dense is the least-squares projection written out (pinned on CPU by the
round trip and the orthogonality of its residual). The CUDA kernel sums the c signed inputs
of a slot in fp32 and rounds once, so against the float64 oracle:
  * fp32 : every element within 1e-6 of its row's largest |Wc| (c <= 8 fp32 additions), and
           the per-row normalised error within 1e-4;
  * bf16 : every element within 2^-8 |ref| + 1e-30 (one round-to-nearest-even, 2^-9 relative,
           with a factor two for the fp32 sum before it), and the per-row error within 2e-2.
Projecting a tied weight must return its compressed weights bit for bit in both dtypes.
"""

import numpy as np
import pytest
import torch

import oracle as O
from tests._parity import row_normalised_max_err
from tests.gpu_common import get_ss1, to_np64

pytestmark = pytest.mark.gpu

# (K, N, c, BK, BN): the fast kernel at every c and BK of the workloads, narrow N-blocks (fewer
# rows per tile), and shapes whose rows are not 16-byte multiples (the plain kernel)
SHAPES = [
    (1024, 384, 1, 128, 128),
    (1024, 384, 2, 128, 128),
    (1024, 384, 4, 256, 128),
    (1024, 384, 8, 256, 128),
    (768, 768, 2, 64, 64),
    (4608, 256, 4, 256, 32),
    (960, 256, 2, 48, 16),
    (36, 48, 4, 12, 16),       # K * 2 bytes = 72: plain kernel
    (1280, 640, 4, 128, 128),
    (768, 96, 2, 96, 48),      # 16 (N-block, K-chunk) units: rows split in two, pairs cut by the range end
    (512, 160, 2, 64, 80),     # rows split in four ranges of 20: some warps end on a lone row
]


def _dense_weight(N, K, seed, dtype):
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(N, K, generator=gen) * 0.05).to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("K,N,c,BK,BN", SHAPES)
def test_project_matches_oracle(K, N, c, BK, BN, dtype):
    ss1 = get_ss1()
    layer = ss1.SS1Layer(K, N, c, BK, BN, seed=21)
    W = _dense_weight(N, K, K + N + c, dtype)
    Wc = layer.project(W.cuda())
    torch.cuda.synchronize()
    h, g = O.ss1_tables(K, N, c, BK, BN, 21)
    ref = O.project_dense(to_np64(W), h, g, BN, c)
    got = to_np64(Wc)
    assert np.isfinite(got).all()
    if dtype == torch.float32:
        scale = np.abs(ref).max(axis=1, keepdims=True)
        assert (np.abs(got - ref) <= 1e-6 * scale + 1e-30).all()
        assert row_normalised_max_err(got, ref) <= 1e-4
    else:
        assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30).all()
        assert row_normalised_max_err(got, ref) <= 2e-2
    layer.close()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("c,BK", [(2, 128), (4, 128), (8, 256), (2, 256)])
def test_project_of_tied_weight_is_exact(c, BK, dtype):
    """W = W_full(Wc0): every slot sums c copies of g^2 Wc0 = Wc0, so the result is Wc0 exactly."""
    ss1 = get_ss1()
    K, N, BN = 2048, 512, 128
    layer = ss1.SS1Layer(K, N, c, BK, BN, seed=5)
    gen = torch.Generator().manual_seed(c * BK)
    Wc0 = (torch.randn(N, K // c, generator=gen) * 0.05).to(dtype)
    h, g = O.ss1_tables(K, N, c, BK, BN, 5)
    Wfull = np.concatenate([O.expand_weight(to_np64(Wc0), h, g, BN, nb) for nb in range(N // BN)])
    W = torch.from_numpy(np.ascontiguousarray(Wfull)).to(dtype)   # exact: +-Wc0 entries
    Wc = layer.project(W.cuda())
    torch.cuda.synchronize()
    assert torch.equal(Wc.cpu(), Wc0)
    layer.close()


def test_project_full_size_sampled_blocks():
    """The Llama-3-8B gate/up projection (4096 x 14336, c = 2, BK = 256): the bench's launch,
    compared with the oracle on three whole N-blocks (first, middle, last)."""
    ss1 = get_ss1()
    K, N, c, BK, BN = 4096, 14336, 2, 256, 128
    layer = ss1.SS1Layer(K, N, c, BK, BN, seed=3)
    gen = torch.Generator(device="cuda").manual_seed(3)
    W = (torch.randn(N, K, device="cuda", generator=gen) * 0.02).to(torch.bfloat16)
    Wc = layer.project(W)
    torch.cuda.synchronize()
    h, g = O.ss1_tables(K, N, c, BK, BN, 3)
    for nb in (0, N // BN // 2, N // BN - 1):
        rows = slice(nb * BN, (nb + 1) * BN)
        ref = O.project_dense(to_np64(W[rows]), h[nb:nb + 1], g[nb:nb + 1], BN, c)
        got = to_np64(Wc[rows])
        assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30).all()
    layer.close()


def test_project_argument_errors():
    ss1 = get_ss1()
    lib = ss1.lib()
    layer = ss1.SS1Layer(512, 256, 2, 128, 128, seed=1)
    W = torch.zeros(256, 512, dtype=torch.bfloat16, device="cuda")
    Wc = torch.zeros(256, 256, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert lib.ss1_project(layer.handle, None, Wc.data_ptr(), 0, st) == -1
    assert lib.ss1_project(layer.handle, W.data_ptr(), Wc.data_ptr(), 5, st) == -1
    assert lib.ss1_project(layer.handle, W.data_ptr() + 1, Wc.data_ptr(), 0, st) == -5
    assert lib.ss1_project(layer.handle, W.data_ptr(), Wc.data_ptr(), 0, st) == 0
    torch.cuda.synchronize()
    layer.close()
