"""Helpers for the GPU tests: library loading, oracle comparison on sampled rows."""

import numpy as np
import torch

import oracle as O
from structured_compressed_linear_b200.workloads import Layer, make_inputs, torch_dtype
from tests._parity import TOL, row_normalised_max_err


def get_ss1():
    from structured_compressed_linear_b200 import build
    build.build()
    from structured_compressed_linear_b200 import ss1
    ss1.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return ss1


def to_np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def sample_rows(M: int, n: int, seed: int, must=()):
    """First, last, ragged-tail and random rows (plus any rows in `must`)."""
    rng = np.random.default_rng(seed)
    rows = {0, M - 1, max(0, M - 2), M // 2}
    rows |= {r for r in (127, 128, 129) if r < M}
    rows |= set(int(r) for r in rng.choice(M, size=min(n, M), replace=False))
    rows |= set(int(r) for r in must)
    return np.array(sorted(r for r in rows if 0 <= r < M), dtype=np.int64)


def check_layer(ss1, L: Layer, kernel=0, rows=None, X=None, Wc=None, tables=None):
    """Run one layer on the GPU and compare (sampled) rows with the oracle. Returns err."""
    if X is None:
        X, Wc = make_inputs(L)
    Xd, Wd = X.cuda(), Wc.cuda()
    layer = ss1.SS1Layer(L.K, L.N, L.c, L.BK, L.BN, L.seed)
    Y = layer.forward(Xd, Wd, kernel=kernel)
    torch.cuda.synchronize()
    st, detail = layer.device_status()
    assert st == 0, f"device status {detail:#x}"
    h, g = tables if tables is not None else O.ss1_tables(L.K, L.N, L.c, L.BK, L.BN, L.seed)
    if rows is None:
        ref = O.ss1_forward(to_np64(X), to_np64(Wc), h, g, L.BN)
        got = to_np64(Y)
    else:
        ref = O.ss1_forward_rows(to_np64(X), to_np64(Wc), h, g, L.BN, rows)
        got = to_np64(Y[torch.as_tensor(rows, device=Y.device)])
    err = row_normalised_max_err(got, ref)
    layer.close()
    assert np.isfinite(got).all()
    assert err <= TOL[L.dtype], f"{L.tag} kernel={kernel}: err {err:.3e} > {TOL[L.dtype]}"
    return err
