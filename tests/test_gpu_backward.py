"""SS1 backward pass (ss1_backward_input, ss1_backward_weight) against the CPU oracle.

The oracle's ss1_backward_input / ss1_backward_weight are pinned on CPU by central finite
differences of a linear loss. The CUDA path multiplies exact copies of the operands (W_full^T
holds +-Wc entries; dY^T and X^T are copies) with fp32 accumulation and one rounding to the
output type; the weight gradient's dense product G = dY^T X is rounded once more (to the data
type) before its c-term tied sums. The bounds are the layer's: per-row normalised error
<= 2e-2 for bf16 and <= 1e-4 for fp32, rows of dX and rows of dWc alike.
"""

import numpy as np
import pytest
import torch

import oracle as O
from tests._parity import TOL, row_normalised_max_err
from tests.gpu_common import get_ss1, to_np64

pytestmark = pytest.mark.gpu

# (K, N, c, BK, BN, M, dtype): tensor-core shapes (bf16, K % 128 == 0, N % 64 == 0) at every c,
# ragged M, a bf16 shape the tensor-core kernel does not take (K % 128 != 0), and fp32
CASES = [
    (1024, 384, 2, 128, 128, 200, "bf16"),
    (1024, 256, 8, 256, 128, 333, "bf16"),
    (768, 768, 4, 128, 128, 130, "bf16"),
    (512, 256, 1, 128, 128, 65, "bf16"),
    (960, 256, 2, 48, 16, 37, "bf16"),
    (768, 768, 2, 64, 64, 64, "fp32"),
    (512, 256, 4, 128, 128, 77, "fp32"),
    (256, 192, 1, 64, 64, 1, "fp32"),
]


def _inputs(K, N, c, M, dtype, seed):
    gen = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    X = torch.randn(M, K, generator=gen).to(dt)
    dY = torch.randn(M, N, generator=gen).to(dt)
    Wc = (torch.randn(N, K // c, generator=gen) * 0.05).to(dt)
    return X, dY, Wc


@pytest.mark.parametrize("K,N,c,BK,BN,M,dtype", CASES)
def test_backward_matches_oracle(K, N, c, BK, BN, M, dtype):
    ss1 = get_ss1()
    layer = ss1.SS1Layer(K, N, c, BK, BN, seed=17)
    X, dY, Wc = _inputs(K, N, c, M, dtype, K + N + M)
    dX = layer.backward_input(dY.cuda(), Wc.cuda())
    dWc = layer.backward_weight(X.cuda(), dY.cuda())
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    h, g = O.ss1_tables(K, N, c, BK, BN, 17)
    ref_dx = O.ss1_backward_input(to_np64(dY), to_np64(Wc), h, g, BN)
    ref_dw = O.ss1_backward_weight(to_np64(X), to_np64(dY), h, g, BN, K // c)
    got_dx, got_dw = to_np64(dX), to_np64(dWc)
    assert np.isfinite(got_dx).all() and np.isfinite(got_dw).all()
    assert row_normalised_max_err(got_dx, ref_dx) <= TOL[dtype]
    assert row_normalised_max_err(got_dw, ref_dw) <= TOL[dtype]
    layer.close()


def test_backward_full_size_sampled():
    """Llama-3-8B q projection (4096 x 4096, c = 2, BK = 256) at M = 4096 rows, the benchmark's
    launch: dX on sampled rows, dWc on three whole N-blocks, against the oracle."""
    ss1 = get_ss1()
    K, N, c, BK, BN, M = 4096, 4096, 2, 256, 128, 4096
    layer = ss1.SS1Layer(K, N, c, BK, BN, seed=3)
    X, dY, Wc = _inputs(K, N, c, M, "bf16", 99)
    dX = layer.backward_input(dY.cuda(), Wc.cuda())
    dWc = layer.backward_weight(X.cuda(), dY.cuda())
    torch.cuda.synchronize()
    h, g = O.ss1_tables(K, N, c, BK, BN, 3)
    rows = np.array([0, 1, 127, 128, 2047, 4094, 4095])
    ref_dx = O.ss1_backward_input(to_np64(dY[rows]), to_np64(Wc), h, g, BN)
    assert row_normalised_max_err(to_np64(dX[torch.as_tensor(rows).cuda()]), ref_dx) <= 2e-2
    X64, dY64 = to_np64(X), to_np64(dY)
    for nb in (0, 17, N // BN - 1):
        cols = slice(nb * BN, (nb + 1) * BN)
        ref_dw = O.ss1_backward_weight(X64, dY64[:, cols], h[nb:nb + 1], g[nb:nb + 1], BN, K // c)
        assert row_normalised_max_err(to_np64(dWc[cols]), ref_dw) <= 2e-2
    layer.close()


def test_backward_zero_rows_and_errors():
    ss1 = get_ss1()
    lib = ss1.lib()
    K, N, c = 512, 256, 2
    layer = ss1.SS1Layer(K, N, c, 128, 128, seed=1)
    X = torch.zeros(0, K, dtype=torch.bfloat16, device="cuda")
    dY = torch.zeros(0, N, dtype=torch.bfloat16, device="cuda")
    dWc = layer.backward_weight(X, dY, out=torch.full((N, K // c), 3.0, dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert torch.count_nonzero(dWc).item() == 0          # no rows: zero gradient
    st = torch.cuda.current_stream().cuda_stream
    Wc = torch.zeros(N, K // c, dtype=torch.bfloat16, device="cuda")
    dY1 = torch.zeros(4, N, dtype=torch.bfloat16, device="cuda")
    dX1 = torch.zeros(4, K, dtype=torch.bfloat16, device="cuda")
    need_in, need_w = layer.backward_workspace(4)
    ws = torch.empty(max(need_in, need_w), dtype=torch.uint8, device="cuda")
    h = layer.handle
    assert lib.ss1_backward_input(h, dY1.data_ptr(), Wc.data_ptr(), dX1.data_ptr(), 4, 0, ws.data_ptr(), need_in - 1, st) == -1
    assert lib.ss1_backward_input(h, dY1.data_ptr(), Wc.data_ptr(), dX1.data_ptr(), 4, 0, ws.data_ptr() + 16, need_in, st) == -5
    assert lib.ss1_backward_input(h, dY1.data_ptr(), Wc.data_ptr(), dX1.data_ptr(), -1, 0, ws.data_ptr(), need_in, st) == -1
    assert lib.ss1_backward_input(h, dY1.data_ptr(), Wc.data_ptr(), dX1.data_ptr(), 4, 0, ws.data_ptr(), need_in, st) == 0
    torch.cuda.synchronize()
    layer.close()


def test_autograd_wrapper_matches_entry_points():
    """SS1Function (torch.autograd) routes its backward to the same entry points."""
    ss1 = get_ss1()
    K, N, c, M = 1024, 384, 2, 96
    layer = ss1.SS1Layer(K, N, c, 128, 128, seed=4)
    X, dY, Wc = _inputs(K, N, c, M, "bf16", 5)
    Xd = X.cuda().requires_grad_()
    Wd = Wc.cuda().requires_grad_()
    Y = ss1.SS1Function.apply(Xd, Wd, layer)
    Y.backward(dY.cuda())
    torch.cuda.synchronize()
    assert torch.equal(Xd.grad, layer.backward_input(dY.cuda(), Wc.cuda()))
    assert torch.equal(Wd.grad, layer.backward_weight(X.cuda(), dY.cuda()))
    assert torch.equal(Y.detach(), layer.forward(X.cuda(), Wc.cuda()))
    layer.close()
