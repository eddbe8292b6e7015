"""FP8 (E4M3) compressed weights: ss1_quantize_fp8 and ss1_forward_fp8 against the CPU oracle.

Quantisation is integer work decided by float32 arithmetic that both sides do the same way
(the scale a correctly rounded float32 division, the codes round-to-nearest-even of the
correctly rounded float32 quotient), so codes and scales must match the oracle bit for bit.
The forward is compared with the oracle's forward on the dequantised weight (exact in float64)
at the layer's bf16 tolerance: per-row normalised error <= 2e-2.
"""

import numpy as np
import pytest
import torch

import oracle as O
from tests._parity import row_normalised_max_err
from tests.gpu_common import get_ss1, to_np64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("N,Kc", [(384, 512), (256, 2048), (7, 33), (1024, 7168)])
def test_quantize_matches_oracle_bit_for_bit(N, Kc, dtype):
    ss1 = get_ss1()
    gen = torch.Generator().manual_seed(N + Kc)
    Wc = (torch.randn(N, Kc, generator=gen) * torch.exp2(torch.randint(-9, 3, (N, 1), generator=gen).float())).to(dtype)
    Wc[0] = 0.0                      # an all-zero row: scale 1
    if N > 3:
        Wc[3, :5] = -0.0             # negative zeros keep their sign bit
    Wq, scale = ss1.quantize_fp8(Wc.cuda())
    torch.cuda.synchronize()
    ref_q, ref_s = O.quantize_rows_e4m3(Wc.float().numpy())
    assert np.array_equal(scale.cpu().numpy(), ref_s)
    assert np.array_equal(Wq.cpu().numpy(), ref_q)


# Decode-sized rows on the Llama-3-8B shapes (c = 2 and 8, BK = 256) and a narrow layer, every
# row-group width (16, 32, 64)
CASES = [(K, N, c, M) for (K, N) in [(4096, 1024), (1024, 384)] for c in (2, 8) for M in (1, 5, 16)]
CASES += [(1024, 384, 4, 33), (1024, 384, 2, 64), (14336, 4096, 2, 3), (4096, 14336, 8, 16)]


@pytest.mark.parametrize("K,N,c,M", CASES)
def test_forward_fp8_matches_oracle(K, N, c, M):
    ss1 = get_ss1()
    BK, BN = 256, 128
    layer = ss1.SS1Layer(K, N, c, BK, BN, seed=3)
    gen = torch.Generator().manual_seed(K + N + c + M)
    X = torch.randn(M, K, generator=gen).to(torch.bfloat16)
    Wc = (torch.randn(N, K // c, generator=gen) * 0.02).to(torch.bfloat16)
    Wq, scale = ss1.quantize_fp8(Wc.cuda())
    Y = layer.forward_fp8(X.cuda(), Wq, scale)
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    h, g = O.ss1_tables(K, N, c, BK, BN, 3)
    ref = O.ss1_forward_fp8(to_np64(X), Wq.cpu().numpy(), scale.cpu().numpy(), h, g, BN)
    got = to_np64(Y)
    assert np.isfinite(got).all()
    assert row_normalised_max_err(got, ref) <= 2e-2
    # repeated calls give the same bits (fixed reduction order of the K-splits)
    assert torch.equal(layer.forward_fp8(X.cuda(), Wq, scale), Y)
    layer.close()


def test_forward_fp8_one_hot_is_exact():
    """X = rows of the identity: every output is one product scale[n] * e4m3 value, the fp32 sum
    of a single term, so Y equals bf16(scale[n] * e4m3(Wq[n, h(k)]) * g(k)) exactly."""
    ss1 = get_ss1()
    K, N, c, BK, BN = 512, 256, 2, 256, 128
    layer = ss1.SS1Layer(K, N, c, BK, BN, seed=11)
    gen = torch.Generator().manual_seed(2)
    Wc = (torch.randn(N, K // c, generator=gen) * 0.05).to(torch.bfloat16)
    Wq, scale = ss1.quantize_fp8(Wc.cuda())
    h, g = O.ss1_tables(K, N, c, BK, BN, 11)
    Wd = O.e4m3_decode(Wq.cpu().numpy()) * scale.cpu().numpy().astype(np.float64)[:, None]
    Wfull = np.concatenate([O.expand_weight(Wd, h, g, BN, nb) for nb in range(N // BN)])   # [N, K]
    for r0 in range(0, K, 64):
        X = torch.eye(K, dtype=torch.bfloat16)[r0:r0 + 64].contiguous()
        Y = layer.forward_fp8(X.cuda(), Wq, scale)
        torch.cuda.synchronize()
        ref = torch.from_numpy(np.ascontiguousarray(Wfull.T[r0:r0 + 64])).to(torch.float32).to(torch.bfloat16)
        assert torch.equal(Y.cpu(), ref)
    layer.close()


def test_forward_fp8_errors():
    ss1 = get_ss1()
    lib = ss1.lib()
    layer = ss1.SS1Layer(1024, 384, 2, 256, 128, seed=1)
    X = torch.zeros(65, 1024, dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros(384, 512, dtype=torch.uint8, device="cuda")
    sc = torch.ones(384, dtype=torch.float32, device="cuda")
    Y = torch.zeros(65, 384, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    h = layer.handle
    assert lib.ss1_forward_fp8(h, X.data_ptr(), Wq.data_ptr(), sc.data_ptr(), Y.data_ptr(), 65, st) == -8   # M > 64
    assert lib.ss1_forward_fp8(h, X.data_ptr(), Wq.data_ptr(), sc.data_ptr(), Y.data_ptr(), 0, st) == 0     # no-op
    assert lib.ss1_forward_fp8(h, X.data_ptr() + 2, Wq.data_ptr(), sc.data_ptr(), Y.data_ptr(), 4, st) == -5
    assert lib.ss1_forward_fp8(h, X.data_ptr(), None, sc.data_ptr(), Y.data_ptr(), 4, st) == -1
    layer.close()
    other = ss1.SS1Layer(1024, 384, 2, 256, 64, seed=1)          # BN = 64: not the decode kernel's shape
    assert lib.ss1_forward_fp8(other.handle, X.data_ptr(), Wq.data_ptr(), sc.data_ptr(), Y.data_ptr(), 4, st) == -8
    other.close()
