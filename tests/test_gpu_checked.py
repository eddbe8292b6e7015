"""The bounds-checked debug build (libss1_checked.so) on every kernel path.

The checked build tests each global access that a kernel addresses by its own index arithmetic
against the extent of its buffer, records the first failure and skips the access (include/ss1.h,
ss1_bounds_check). It stands in for a memory checker. Each case runs one entry point through the
normal library and then through the checked one, on the same inputs: the outputs must agree bit
for bit (the tests change nothing in range) and the record must stay empty. Small and ragged
shapes reach every kernel: tc3, tc2, tc (c = 1), the decode kernel (bf16 and FP8, with and
without a K-split cluster), the CUDA-core small-M kernel, the CUDA-core general kernel (bf16 and
fp32, with a cluster K-split), the fused and separate bias/activation epilogues, a two-layer
chain, the allocation-free forward, the three projection kernels, both backward entry points
and the table generator (every ss1_create).
"""

import pytest
import torch

from tests.gpu_common import get_ss1

pytestmark = pytest.mark.gpu

BF16, F32 = torch.bfloat16, torch.float32


@pytest.fixture(scope="module")
def ss1():
    s = get_ss1()
    from structured_compressed_linear_b200 import build
    build.build(checked=True)
    s.load_library(s.CHECKED_LIB_PATH)
    yield s
    s.use_library(s.LIB_PATH)


def _inputs(K, N, c, M, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    X = torch.randn(M, K, generator=g).to(dtype).cuda()
    Wc = (torch.randn(N, K // c, generator=g) / K ** 0.5).to(dtype).cuda()
    return X, Wc


def _both(ss1, fn):
    """fn(ss1) under the normal library, then under the checked one; the checked record must be empty."""
    ss1.use_library(ss1.LIB_PATH)
    try:
        ref = fn(ss1)
        torch.cuda.synchronize()
        ss1.use_library(ss1.CHECKED_LIB_PATH)
        assert ss1.bounds_check() == (True, 0), "a record left over from an earlier call"
        got = fn(ss1)
        torch.cuda.synchronize()
        checked, record = ss1.bounds_check()
        kernel = ss1.last_launch()["kernel"]
    finally:
        ss1.use_library(ss1.LIB_PATH)
    assert checked
    assert record == 0, f"out-of-range access: site {record >> 48}, index {record & ((1 << 48) - 1)}"
    ref = ref if isinstance(ref, (list, tuple)) else [ref]
    got = got if isinstance(got, (list, tuple)) else [got]
    for a, b in zip(ref, got):
        assert torch.equal(a, b), "the checked build changed a result"
    return kernel


FORWARD = [
    # K, N, c, BK, BN, M, dtype, forced kernel (0: the automatic choice), kernel of the last launch
    (1024, 384, 2, 128, 128, 300, BF16, 0, "tc3"),
    (1024, 512, 8, 256, 128, 129, BF16, 0, "tc3"),
    (512, 256, 2, 64, 128, 300, BF16, 0, "tc2"),
    (512, 256, 1, 128, 128, 300, BF16, 0, "tc"),
    (1024, 384, 2, 128, 128, 5, BF16, 0, "dec"),
    (4096, 1024, 2, 256, 128, 1, BF16, 0, "dec"),
    (1024, 384, 8, 256, 128, 40, BF16, 3, "dec"),   # SMALLM forced: the decode kernel at M = 40
    (512, 192, 2, 64, 64, 7, BF16, 0, "smallm"),
    (640, 96, 2, 64, 48, 100, BF16, 0, "simt"),
    (768, 768, 2, 64, 64, 64, F32, 0, "simt"),
    (768, 256, 4, 64, 64, 200, F32, 0, "simt"),
]


@pytest.mark.parametrize("K,N,c,BK,BN,M,dtype,force,kernel", FORWARD)
def test_forward_in_bounds(ss1, K, N, c, BK, BN, M, dtype, force, kernel):
    X, Wc = _inputs(K, N, c, M, dtype, seed=K + N + M)

    def run(s):
        layer = s.SS1Layer(K, N, c, BK, BN, seed=11)
        Y = layer.forward(X, Wc, kernel=force)
        torch.cuda.synchronize()
        layer.close()
        return Y
    assert _both(ss1, run) == kernel


@pytest.mark.parametrize("K,N,c,BK,BN,M,dtype", [(1024, 384, 2, 128, 128, 300, BF16), (768, 256, 2, 64, 64, 50, F32)])
def test_bias_activation_in_bounds(ss1, K, N, c, BK, BN, M, dtype):
    X, Wc = _inputs(K, N, c, M, dtype, seed=3)
    bias = torch.randn(N, generator=torch.Generator().manual_seed(4)).to(dtype).cuda()

    def run(s):
        layer = s.SS1Layer(K, N, c, BK, BN, seed=5)
        Y = layer.forward_ex(X, Wc, bias=bias, act=s.Act.GELU)
        torch.cuda.synchronize()
        layer.close()
        return Y
    _both(ss1, run)


def test_chain_in_bounds(ss1):
    M = 200
    X, W0 = _inputs(1024, 512, 2, M, BF16, seed=6)
    _, W1 = _inputs(512, 256, 2, 1, BF16, seed=7)

    def run(s):
        layers = [s.SS1Layer(1024, 512, 2, 128, 128, seed=8), s.SS1Layer(512, 256, 2, 128, 128, seed=9)]
        outs = s.chain_forward(layers, X, [W0, W1], acts=[s.Act.RELU, s.Act.NONE])
        torch.cuda.synchronize()
        for ly in layers:
            ly.close()
        return outs
    _both(ss1, run)


@pytest.mark.parametrize("M", [1, 16, 33])
def test_fp8_in_bounds(ss1, M):
    K, N, c = 4096, 1024, 2
    X, Wc = _inputs(K, N, c, M, BF16, seed=M)

    def run(s):
        Wq, scale = s.quantize_fp8(Wc)
        layer = s.SS1Layer(K, N, c, 256, 128, seed=12)
        Y = layer.forward_fp8(X, Wq, scale)
        torch.cuda.synchronize()
        layer.close()
        return [Wq, scale, Y]
    assert _both(ss1, run) == "dec_fp8"


def test_noalloc_in_bounds(ss1):
    X, Wc = _inputs(1024, 384, 2, 70, BF16, seed=13)
    _both(ss1, lambda s: s.forward_noalloc(X, Wc, 1024, 384, 2, 128, 128, seed=14))


@pytest.mark.parametrize("K,N,c,BK,BN,dtype", [
    (1024, 384, 2, 128, 128, BF16),    # bf16 pair kernel
    (1024, 384, 4, 128, 128, F32),     # fp32 row kernel
    (768, 96, 2, 96, 48, BF16),        # row ranges split over CTAs
    (96, 32, 2, 12, 16, BF16),         # 24-byte chunks: the plain kernel
])
def test_projection_in_bounds(ss1, K, N, c, BK, BN, dtype):
    W = torch.randn(N, K, generator=torch.Generator().manual_seed(15)).to(dtype).cuda()

    def run(s):
        layer = s.SS1Layer(K, N, c, BK, BN, seed=16)
        Wc = layer.project(W)
        torch.cuda.synchronize()
        layer.close()
        return Wc
    _both(ss1, run)


@pytest.mark.parametrize("K,N,c,BK,BN,M,dtype", [(1024, 384, 2, 128, 128, 300, BF16), (768, 256, 4, 64, 64, 70, F32)])
def test_backward_in_bounds(ss1, K, N, c, BK, BN, M, dtype):
    X, Wc = _inputs(K, N, c, M, dtype, seed=17)
    dY = torch.randn(M, N, generator=torch.Generator().manual_seed(18)).to(dtype).cuda()

    def run(s):
        layer = s.SS1Layer(K, N, c, BK, BN, seed=19)
        dX = layer.backward_input(dY, Wc)
        dWc = layer.backward_weight(X, dY)
        torch.cuda.synchronize()
        layer.close()
        return [dX, dWc]
    _both(ss1, run)


def test_record_reports_the_first_failed_test(ss1):
    """The record itself, on given values (the self-test touches no memory): a failed test is
    reported as (63 << 48) | index, only the first one is kept, and reading clears it."""
    ss1.use_library(ss1.CHECKED_LIB_PATH)
    try:
        lib = ss1.lib()
        assert ss1.bounds_check() == (True, 0)
        assert lib.ss1_test_bounds_check(3, 4) == 0     # in range: nothing recorded
        assert ss1.bounds_check() == (True, 0)
        assert lib.ss1_test_bounds_check(5, 4) == 0
        assert lib.ss1_test_bounds_check(9, 4) == 0     # a second failure does not replace the first
        assert ss1.bounds_check() == (True, (63 << 48) | 5)
        assert ss1.bounds_check() == (True, 0)
        assert lib.ss1_test_bounds_check(-1, 4) == 0    # negative indices fail too
        assert ss1.bounds_check()[1] >> 48 == 63
    finally:
        ss1.use_library(ss1.LIB_PATH)
