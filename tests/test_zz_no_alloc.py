"""ss1_forward_noalloc (the forward that allocates nothing) against ss1_forward, on the GPU.

The file name sorts last, so the test runs after every other GPU test in a full run and also
passes alone. Each case makes two calls in a row through the C ABI and compares both outputs
with the handle-based ss1_forward on the same inputs. The status word starts non-zero to show
that the call clears it, and the second call must leave the device's free memory unchanged.
"""

import pytest
import torch

from structured_compressed_linear_b200.workloads import Layer, make_inputs
from tests.gpu_common import get_ss1

pytestmark = pytest.mark.gpu

CASES = [
    # tensor-core path: GPT-2 Small fc shape with a ragged row count
    Layer("noalloc-tc", 333, 768, 3072, 2, 128, 128, "bf16", "normal", "uniform_invsqrtk", 7),
    # decode path
    Layer("noalloc-smallm", 4, 1024, 1024, 4, 128, 128, "bf16", "normal", "uniform_invsqrtk", 8),
    # CUDA-core path in fp32
    Layer("noalloc-simt", 65, 512, 256, 2, 64, 64, "fp32", "normal", "uniform_invsqrtk", 9),
]

# Same kernels, same tables and the same reduction order on both sides: the outputs agree bit
# for bit.


@pytest.mark.parametrize("L", CASES, ids=lambda L: L.tag)
def test_noalloc_matches_forward_twice(L):
    ss1 = get_ss1()
    X, Wc = make_inputs(L)
    Xd, Wd = X.cuda(), Wc.cuda()
    layer = ss1.SS1Layer(L.K, L.N, L.c, L.BK, L.BN, L.seed)
    ref = layer.forward(Xd, Wd)
    torch.cuda.synchronize()
    assert layer.device_status()[0] == 0
    layer.close()

    status = torch.ones(1, dtype=torch.int32, device="cuda")
    outs = [torch.empty_like(ref), torch.empty_like(ref)]
    ss1.forward_noalloc(Xd, Wd, L.K, L.N, L.c, L.BK, L.BN, L.seed, out=outs[0], device_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    status.fill_(1)
    free_before = torch.cuda.mem_get_info()[0]
    ss1.forward_noalloc(Xd, Wd, L.K, L.N, L.c, L.BK, L.BN, L.seed, out=outs[1], device_status=status)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert status.item() == 0
    assert free_after == free_before, f"free device memory changed by {free_after - free_before} bytes"
    for Y in outs:
        assert torch.equal(Y, ref), f"max |diff| {(Y.float() - ref.float()).abs().max().item():.3e}"


def test_noalloc_rejects_oversized_tables():
    ss1 = get_ss1()
    lib = ss1.lib()
    # (N / BN) * K = 128 * 8192 > the static region's limit
    assert 128 * 8192 > ss1.NOALLOC_MAX_ENTRIES
    X = torch.zeros(1, 8192, dtype=torch.bfloat16, device="cuda")
    Wc = torch.zeros(16384, 4096, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(1, 16384, dtype=torch.bfloat16, device="cuda")
    rc = lib.ss1_forward_noalloc(8192, 16384, 2, 128, 128, 0, X.data_ptr(), Wc.data_ptr(), Y.data_ptr(), 1, 0, None,
                                 None)
    assert rc == -8
