"""Exactness properties and error conventions of the CUDA path through the C ABI."""

import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from tests.gpu_common import get_ss1, to_np64

pytestmark = pytest.mark.gpu

SIMT, TC, SMALLM = 2, 1, 3
BF16_KERNELS = [SIMT, TC, SMALLM]
SMALLM_MAX_ROWS = 64


def _rows(kernel, M):
    """Row count a test uses with this kernel: the small-M kernel takes at most 64 rows."""
    return min(M, SMALLM_MAX_ROWS) if kernel == SMALLM else M


def _layer(ss1, K=512, N=256, c=4, BK=128, BN=128, seed=3):
    return ss1.SS1Layer(K, N, c, BK, BN, seed)


@pytest.mark.parametrize("kernel", BF16_KERNELS)
@pytest.mark.parametrize("c,BK", [(1, 128), (2, 128), (4, 128), (8, 128), (8, 256), (2, 256)])
def test_one_hot_probe_bit_exact(kernel, c, BK):
    """X = I_K: every output is one product g * Wc (exact in bf16), so Y must equal the tied
    weight bit for bit. Pins the hash indexing and signs inside the kernel."""
    ss1 = get_ss1()
    K, N, BN = 512, 256, 128
    layer = _layer(ss1, K, N, c, BK, BN, seed=11)
    gen = torch.Generator().manual_seed(5)
    Wc = (torch.randn(N, K // c, generator=gen) * 0.1).to(torch.bfloat16)
    X = torch.eye(K, dtype=torch.bfloat16)
    step = _rows(kernel, K)
    Y = torch.cat([layer.forward(X[r:r + step].cuda(), Wc.cuda(), kernel=kernel) for r in range(0, K, step)])
    h, g = O.ss1_tables(K, N, c, BK, BN, 11)
    Wfull = np.concatenate([O.expand_weight(to_np64(Wc), h, g, BN, nb) for nb in range(N // BN)])
    assert np.array_equal(to_np64(Y), Wfull.T)
    layer.close()


@pytest.mark.parametrize("kernel", BF16_KERNELS)
def test_zero_negation_linearity(kernel):
    ss1 = get_ss1()
    layer = _layer(ss1)
    gen = torch.Generator().manual_seed(9)
    M = _rows(kernel, 300)
    X1 = torch.randn(M, 512, generator=gen).to(torch.bfloat16).cuda()
    X2 = torch.randn(M, 512, generator=gen).to(torch.bfloat16).cuda()
    Wc = (torch.randn(256, 128, generator=gen) * 0.05).to(torch.bfloat16).cuda()
    Y0 = layer.forward(torch.zeros_like(X1), Wc, kernel=kernel)
    assert torch.count_nonzero(Y0).item() == 0
    Yp = layer.forward(X1, Wc, kernel=kernel)
    Yn = layer.forward(-X1, Wc, kernel=kernel)
    assert torch.equal(Yn, -Yp)
    Ys = layer.forward((X1.float() + X2.float()).to(torch.bfloat16), Wc, kernel=kernel)
    Y2 = layer.forward(X2, Wc, kernel=kernel)
    ref = Yp.float() + Y2.float()
    scale = ref.abs().amax(dim=1, keepdim=True)
    assert float(((Ys.float() - ref).abs() / scale).max()) < 3e-2
    layer.close()


def test_guard_band_and_zero_rows():
    """Rows of the output buffer past M stay untouched; M = 0 is a no-op."""
    ss1 = get_ss1()
    layer = _layer(ss1)
    lib = ss1.lib()
    gen = torch.Generator().manual_seed(1)
    Wc = (torch.randn(256, 128, generator=gen) * 0.05).to(torch.bfloat16).cuda()
    for k in [0] + BF16_KERNELS:
        M = _rows(k, 129) - 2   # ragged against every row tile
        X = torch.randn(M, 512, generator=gen).to(torch.bfloat16).cuda()
        buf = torch.full((M + 7, 256), 7.0, dtype=torch.bfloat16, device="cuda")
        st = torch.cuda.current_stream().cuda_stream
        assert lib.ss1_forward_with(layer.handle, X.data_ptr(), Wc.data_ptr(), buf.data_ptr(), M, 0, k, st) == 0
        torch.cuda.synchronize()
        assert torch.all(buf[M:] == 7.0)
        assert lib.ss1_forward_with(layer.handle, X.data_ptr(), Wc.data_ptr(), buf.data_ptr(), 0, 0, k, st) == 0
    layer.close()


def test_error_conventions():
    ss1 = get_ss1()
    lib = ss1.lib()
    layer = _layer(ss1)
    X = torch.zeros(8, 512, dtype=torch.bfloat16, device="cuda")
    Wc = torch.zeros(256, 128, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(8, 256, dtype=torch.bfloat16, device="cuda")
    h = layer.handle
    st = torch.cuda.current_stream().cuda_stream
    assert lib.ss1_forward(h, X.data_ptr() + 2, Wc.data_ptr(), Y.data_ptr(), 4, 0, st) == -5
    assert lib.ss1_forward(h, None, Wc.data_ptr(), Y.data_ptr(), 4, 0, st) == -1
    assert lib.ss1_forward(h, X.data_ptr(), Wc.data_ptr(), Y.data_ptr(), -1, 0, st) == -1
    assert lib.ss1_forward(h, X.data_ptr(), Wc.data_ptr(), Y.data_ptr(), 4, 7, st) == -1
    assert lib.ss1_forward_with(h, X.data_ptr(), Wc.data_ptr(), Y.data_ptr(), 4, 0, 99, st) == -1
    # fp32 data cannot take the tensor-core or small-M path; the small-M path takes <= 64 rows
    assert lib.ss1_forward_with(h, X.data_ptr(), Wc.data_ptr(), Y.data_ptr(), 4, 1, TC, st) == -8
    assert lib.ss1_forward_with(h, X.data_ptr(), Wc.data_ptr(), Y.data_ptr(), 4, 1, SMALLM, st) == -8
    assert lib.ss1_forward_with(h, X.data_ptr(), Wc.data_ptr(), Y.data_ptr(), 65, 0, SMALLM, st) == -8
    k = ctypes.c_int()
    assert lib.ss1_select_kernel(h, 4096, 1, ctypes.byref(k)) == 0 and k.value == SIMT
    K_, N_ = ctypes.c_int64(), ctypes.c_int64()
    c_, bk, bn = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    assert lib.ss1_get_info(h, ctypes.byref(K_), ctypes.byref(N_), ctypes.byref(c_), ctypes.byref(bk),
                            ctypes.byref(bn)) == 0
    assert (K_.value, N_.value, c_.value, bk.value, bn.value) == (512, 256, 4, 128, 128)
    assert layer.device_status() == (0, 0)
    raw = layer._h
    layer.close()
    assert lib.ss1_forward(raw, X.data_ptr(), Wc.data_ptr(), Y.data_ptr(), 4, 0, st) == -7
    assert lib.ss1_destroy(raw) == -7
    torch.cuda.synchronize()


@pytest.mark.parametrize("c,BK", [(2, 256), (8, 256), (2, 128), (4, 128)])
def test_repeated_calls_bit_identical(c, BK):
    """The tensor-core kernel has a fixed reduction order: repeated calls give identical bits.
    Guards the ordering between one chunk's TMEM gathers and the next chunk's TMEM staging
    (a missing tcgen05 fence there showed up as run-to-run differences)."""
    ss1 = get_ss1()
    K, N, M = 4096, 1024, 2048
    layer = _layer(ss1, K, N, c, BK, 128, seed=17)
    gen = torch.Generator().manual_seed(23)
    X = torch.randn(M, K, generator=gen).to(torch.bfloat16).cuda()
    Wc = (torch.randn(N, K // c, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    first = layer.forward(X, Wc, kernel=TC)
    for _ in range(4):
        assert torch.equal(layer.forward(X, Wc, kernel=TC), first)
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    layer.close()


@pytest.mark.parametrize("M", [1, 5, 8, 40, 64])
def test_small_m_repeated_calls_bit_identical(M):
    """The small-M kernel reduces its K split in a fixed order: repeated calls agree bit for bit."""
    ss1 = get_ss1()
    K, N = 4096, 14336
    layer = _layer(ss1, K, N, 2, 256, 128, seed=19)
    gen = torch.Generator().manual_seed(29)
    X = torch.randn(M, K, generator=gen).to(torch.bfloat16).cuda()
    Wc = (torch.randn(N, K // 2, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    first = layer.forward(X, Wc, kernel=SMALLM)
    for _ in range(3):
        assert torch.equal(layer.forward(X, Wc, kernel=SMALLM), first)
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    layer.close()


def test_device_timeout_is_reported_and_cleared():
    """A bounded wait that runs out (on a barrier nothing completes) sets the handle's status
    word; the next forward reports SS1_ERR_DEVICE_TIMEOUT, ss1_device_status gives the site and
    clears it, and the same context then computes correctly again. No GPU fault is involved."""
    ss1 = get_ss1()
    lib = ss1.lib()
    K, N, c, BK, BN, seed = 512, 256, 4, 128, 128, 3
    layer = _layer(ss1, K, N, c, BK, BN, seed)
    gen = torch.Generator().manual_seed(13)
    X = torch.randn(8, K, generator=gen).to(torch.bfloat16)
    Wc = (torch.randn(N, K // c, generator=gen) * 0.05).to(torch.bfloat16)
    st = torch.cuda.current_stream().cuda_stream
    assert lib.ss1_test_device_timeout(layer.handle, 0, st) == -1
    assert lib.ss1_test_device_timeout(layer.handle, 5_000_000, st) == 0     # 5 ms limit
    torch.cuda.synchronize()
    with pytest.raises(ss1.SS1Error) as err:
        layer.forward(X.cuda(), Wc.cuda())
    assert err.value.status == -6
    assert layer.device_status() == (-6, (3 << 8) | 0x81)
    assert layer.device_status() == (0, 0)
    Y = layer.forward(X.cuda(), Wc.cuda())
    torch.cuda.synchronize()
    h, g = O.ss1_tables(K, N, c, BK, BN, seed)
    ref = O.ss1_forward(to_np64(X), to_np64(Wc), h, g, BN)
    got = to_np64(Y.cpu())
    assert float((np.abs(got - ref).max(1) / np.abs(ref).max(1)).max()) <= 2e-2
    layer.close()


@pytest.mark.parametrize("K,N,c", [(4096, 4096, 2), (4096, 1024, 8), (4096, 14336, 2)])
def test_decode_calls_on_one_handle_run_concurrently(K, N, c):
    """ss1_forward only reads the handle: decode-sized calls on one handle, issued on two streams
    with no ordering between them (many launches, so they overlap on the device), each match the
    oracle and agree with a serial call bit for bit. The decode kernel's K-split partial sums stay
    inside one thread-block cluster's shared memory."""
    ss1 = get_ss1()
    BK, BN = 256, 128
    layer = _layer(ss1, K, N, c, BK, BN, seed=31)
    gen = torch.Generator().manual_seed(K + N + c)
    Xs = [torch.randn(M, K, generator=gen).to(torch.bfloat16) for M in (1, 5, 16)]
    Wc = (torch.randn(N, K // c, generator=gen) * 0.02).to(torch.bfloat16)
    Wd = Wc.cuda()
    Xd = [x.cuda() for x in Xs]
    serial = [layer.forward(x, Wd) for x in Xd]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [[torch.empty_like(y) for y in serial] for _ in range(8)]
    for it in range(8):
        for i, (x, st) in enumerate(zip(Xd, streams)):
            layer.forward(x, Wd, out=outs[it][i], stream=st)
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    h, g = O.ss1_tables(K, N, c, BK, BN, 31)
    for i, x in enumerate(Xs):
        ref = O.ss1_forward(to_np64(x), to_np64(Wc), h, g, BN)
        got = to_np64(serial[i].cpu())
        assert float((np.abs(got - ref).max(1) / np.abs(ref).max(1)).max()) <= 2e-2
        for it in range(8):
            assert torch.equal(outs[it][i], serial[i])
    layer.close()


def test_forward_kernel_timeout_drains_and_recovers():
    """The tensor-core kernel's own time-out path: one build warp withholds an arrival and every
    wait is cut to 5 ms, so the sketch warp's wait runs out. The kernel must return (its copies
    and matrix multiplies drained, tensor memory freed), the handle must report the site, and the
    next forward on the same context must match the oracle. No GPU fault is involved."""
    ss1 = get_ss1()
    lib = ss1.lib()
    K, N, c, BK, BN, seed, M = 1024, 768, 2, 128, 128, 5, 4096
    layer = _layer(ss1, K, N, c, BK, BN, seed)
    gen = torch.Generator().manual_seed(21)
    X = torch.randn(M, K, generator=gen).to(torch.bfloat16)
    Wc = (torch.randn(N, K // c, generator=gen) * 0.03).to(torch.bfloat16)
    Xd, Wd = X.cuda(), Wc.cuda()
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert lib.ss1_test_forward_timeout(layer.handle, Xd.data_ptr(), Wd.data_ptr(), Y.data_ptr(), M, 0, st) == -1
    assert lib.ss1_test_forward_timeout(layer.handle, Xd.data_ptr(), Wd.data_ptr(), Y.data_ptr(), M, 5_000_000, st) == 0
    torch.cuda.synchronize()            # the kernel returned
    with pytest.raises(ss1.SS1Error) as err:
        layer.forward(Xd, Wd)
    assert err.value.status == -6
    st_, detail = layer.device_status()
    # kernel id 1 (the tensor-core kernel) and the site of the first wait to run out, with the
    # time-out marker bit: the epilogue's wait for the first accumulator, which starts at launch
    assert st_ == -6 and detail >> 8 == 1 and detail & 0x80 and 1 <= (detail & 0x7F) <= 12, hex(detail)
    assert layer.device_status() == (0, 0)
    out = layer.forward(Xd, Wd)
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    h, g = O.ss1_tables(K, N, c, BK, BN, seed)
    rows = np.array([0, 1, 127, 128, 2048, M - 1])
    ref = O.ss1_forward_rows(to_np64(X), to_np64(Wc), h, g, BN, rows)
    got = to_np64(out[torch.as_tensor(rows).cuda()])
    assert float((np.abs(got - ref).max(1) / np.abs(ref).max(1)).max()) <= 2e-2
    layer.close()
