"""Fused bias + activation (ss1_forward_ex) and layer chains (ss1_chain_forward) against the oracle.

The oracle's ss1_forward_bias_act / ss1_chain_forward are pinned on CPU (closed forms of ReLU
and GELU, X = 0 gives act(bias), per-neuron bias, composition). The tensor-core kernel applies
bias and activation to the fp32 sum and rounds once; the other kernels round Y, then add the
bias in fp32 and round again. Against the float64 oracle the bound is the layer's bf16 one
(per-row normalised error <= 2e-2). Chains are checked layer by layer with the GPU's previous
output as the oracle's input (each layer's own error), and end to end.
"""

import numpy as np
import pytest
import torch

import oracle as O
from tests._parity import row_normalised_max_err
from tests.gpu_common import get_ss1, to_np64

pytestmark = pytest.mark.gpu

SIMT, TC, SMALLM = 2, 1, 3


def _data(M, K, N, c, seed):
    gen = torch.Generator().manual_seed(seed)
    X = torch.randn(M, K, generator=gen).to(torch.bfloat16)
    Wc = (torch.randn(N, K // c, generator=gen) / np.sqrt(K)).to(torch.bfloat16)
    b = (torch.randn(N, generator=gen) * 0.5).to(torch.bfloat16)
    return X, Wc, b


CASES = [(kernel, c, BK, act, with_bias)
         for kernel in (TC, SIMT) for (c, BK) in ((2, 128), (8, 256), (4, 128))
         for act in (0, 1, 2) for with_bias in (True, False) if act or with_bias]
CASES += [(SMALLM, 2, 256, act, True) for act in (0, 1, 2)]


@pytest.mark.parametrize("kernel,c,BK,act,with_bias", CASES)
def test_forward_ex_matches_oracle(kernel, c, BK, act, with_bias):
    ss1 = get_ss1()
    K, N = 1024, 384
    M = 16 if kernel == SMALLM else 333
    layer = ss1.SS1Layer(K, N, c, BK, 128, seed=9)
    X, Wc, b = _data(M, K, N, c, c * 10 + act)
    Y = layer.forward_ex(X.cuda(), Wc.cuda(), b.cuda() if with_bias else None, act, kernel=kernel)
    torch.cuda.synchronize()
    assert layer.device_status() == (0, 0)
    h, g = O.ss1_tables(K, N, c, BK, 128, 9)
    ref = O.ss1_forward_bias_act(to_np64(X), to_np64(Wc), h, g, 128, to_np64(b) if with_bias else None, act)
    assert row_normalised_max_err(to_np64(Y), ref) <= 2e-2
    layer.close()


@pytest.mark.parametrize("act", [0, 1, 2])
def test_zero_input_gives_act_of_bias(act):
    """X = 0: every row is act(bias), rounded once to bf16 on the tensor-core path."""
    ss1 = get_ss1()
    K, N, c = 768, 768, 2
    layer = ss1.SS1Layer(K, N, c, 128, 128, seed=2)
    _, Wc, b = _data(1, K, N, c, 3)
    Y = layer.forward_ex(torch.zeros(130, K, dtype=torch.bfloat16, device="cuda"), Wc.cuda(), b.cuda(), act, kernel=TC)
    torch.cuda.synchronize()
    ref = torch.from_numpy(O.activation(to_np64(b), act)).float()
    got = Y.float().cpu()
    assert torch.all((got - ref[None, :]).abs() <= 2.0 ** -8 * ref.abs()[None, :] + 1e-6)
    layer.close()


def _chain(dims, c, BK, BN, acts, seed):
    ss1 = get_ss1()
    layers, Wcs, bs = [], [], []
    gen = torch.Generator().manual_seed(seed)
    for i in range(len(dims) - 1):
        K, N = dims[i], dims[i + 1]
        layers.append(ss1.SS1Layer(K, N, c, BK, BN[i] if isinstance(BN, list) else BN, seed + i))
        Wcs.append((torch.randn(N, K // c, generator=gen) / np.sqrt(K) * 2).to(torch.bfloat16))
        bs.append((torch.randn(N, generator=gen) * 0.1).to(torch.bfloat16))
    return ss1, layers, Wcs, bs


def _check_chain(ss1, layers, Wcs, bs, acts, X, rows=None):
    outs = ss1.chain_forward(layers, X.cuda(), [w.cuda() for w in Wcs], [b.cuda() for b in bs], acts)
    torch.cuda.synchronize()
    for ly in layers:
        assert ly.device_status() == (0, 0)
    sel = slice(None) if rows is None else torch.as_tensor(rows)
    prev = to_np64(X[sel])
    full = []
    for i, (ly, W, b, a) in enumerate(zip(layers, Wcs, bs, acts)):
        h, g = O.ss1_tables(ly.K, ly.N, ly.c, ly.BK, ly.BN, ly.seed)
        got = to_np64(outs[i].cpu()[sel])
        ref = O.ss1_forward_bias_act(prev, to_np64(W), h, g, ly.BN, to_np64(b), a)   # the GPU's previous output as input
        assert row_normalised_max_err(got, ref) <= 2e-2, f"layer {i}"
        full.append((to_np64(W), h, g, ly.BN, to_np64(b), a))
        prev = got
    end = O.ss1_chain_forward(to_np64(X[sel]), full)[-1]
    assert row_normalised_max_err(to_np64(outs[-1].cpu()[sel]), end) <= 3e-2
    return outs


@pytest.mark.parametrize("M", [1, 300, 1000])
def test_dlrm_shaped_chain_in_one_launch(M):
    """1024 -> 1024 -> 512 -> 256, c = 2, BK = BN = 128, ReLU between layers: one persistent launch."""
    acts = [1, 1, 0]
    ss1, layers, Wcs, bs = _chain([1024, 1024, 512, 256], 2, 128, 128, acts, 40)
    assert ss1.chain_fused(layers)
    X = torch.randn(M, 1024, generator=torch.Generator().manual_seed(M)).to(torch.bfloat16)
    _check_chain(ss1, layers, Wcs, bs, acts, X)
    for ly in layers:
        ly.close()


def test_chain_llama_mlp_gelu():
    """A two-layer MLP with GELU (4096 -> 2048 -> 4096, c = 8, BK = 256): fused."""
    acts = [2, 0]
    ss1, layers, Wcs, bs = _chain([4096, 2048, 4096], 8, 256, 128, acts, 50)
    assert ss1.chain_fused(layers)
    X = torch.randn(513, 4096, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    _check_chain(ss1, layers, Wcs, bs, acts, X)
    for ly in layers:
        ly.close()


def test_chain_that_cannot_fuse_runs_layer_by_layer():
    """An N-block size the tensor-core kernel does not take: the chain runs one layer at a time."""
    acts = [1, 0]
    ss1, layers, Wcs, bs = _chain([1024, 512, 256], 2, 128, [64, 128], acts, 60)
    assert not ss1.chain_fused(layers)
    X = torch.randn(200, 1024, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    _check_chain(ss1, layers, Wcs, bs, acts, X)
    for ly in layers:
        ly.close()


def test_dlrm_chain_full_size_sampled():
    """The workload's chain at M = 65536 (the launch the benchmark times), sampled rows."""
    acts = [1, 1, 0]
    ss1, layers, Wcs, bs = _chain([1024, 1024, 512, 256], 2, 128, 128, acts, 4)
    X = (torch.rand(65536, 1024, generator=torch.Generator().manual_seed(4)) * 2 - 1).to(torch.bfloat16)
    rows = [0, 1, 127, 128, 4095, 30000, 65534, 65535]
    _check_chain(ss1, layers, Wcs, bs, acts, X, rows=rows)
    for ly in layers:
        ly.close()
