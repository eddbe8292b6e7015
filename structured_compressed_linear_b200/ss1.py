"""ctypes binding of libss1.so (argument marshalling only).

Every step of the layer runs in the CUDA library; this module passes device pointers, sizes
and the current CUDA stream across the C ABI declared in include/ss1.h. PyTorch provides
device memory and streams. If the library is missing this module raises -- there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from enum import IntEnum
from typing import Optional, Tuple

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libss1.so")

SYMBOLS = ("ss1_create", "ss1_forward", "ss1_forward_with", "ss1_select_kernel", "ss1_destroy",
           "ss1_get_tables", "ss1_get_info", "ss1_device_status", "ss1_strerror", "ss1_forward_noalloc",
           "ss1_test_device_timeout")

#: (N / BN) * K limit of ss1_forward_noalloc (SS1_NOALLOC_MAX_ENTRIES in include/ss1.h).
NOALLOC_MAX_ENTRIES = 983040


class Kernel(IntEnum):
    AUTO = 0
    TC = 1
    SIMT = 2
    SMALLM = 3


class DType(IntEnum):
    BF16 = 0
    FP32 = 1


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """dlopen libss1.so and declare its signatures (works without a GPU)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run `python -m structured_compressed_linear_b200.build`")
    L = ctypes.CDLL(path)
    i64, i32, u64, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_uint64, ctypes.c_void_p
    L.ss1_create.argtypes = [i64, i64, i32, i32, i32, u64, ctypes.POINTER(vp)]
    L.ss1_forward.argtypes = [vp, vp, vp, vp, i64, i32, vp]
    L.ss1_forward_with.argtypes = [vp, vp, vp, vp, i64, i32, i32, vp]
    L.ss1_select_kernel.argtypes = [vp, i64, i32, ctypes.POINTER(i32)]
    L.ss1_destroy.argtypes = [vp]
    L.ss1_get_tables.argtypes = [vp, vp, vp]
    L.ss1_get_info.argtypes = [vp, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i32),
                               ctypes.POINTER(i32), ctypes.POINTER(i32)]
    L.ss1_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    L.ss1_strerror.argtypes = [i32]
    L.ss1_forward_noalloc.argtypes = [i64, i64, i32, i32, i32, u64, vp, vp, vp, i64, i32, vp, vp]
    L.ss1_test_device_timeout.argtypes = [vp, i64, vp]
    L.ss1_strerror.restype = ctypes.c_char_p
    for name in SYMBOLS:
        if name != "ss1_strerror":
            getattr(L, name).restype = i32
    if path == LIB_PATH:
        _lib = L
    return L


def lib() -> ctypes.CDLL:
    return load_library()


class SS1Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib().ss1_strerror(status).decode()} ({status})")


def _check(status: int, what: str):
    if status != 0:
        raise SS1Error(status, what)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return DType.BF16
    if t == torch.float32:
        return DType.FP32
    raise TypeError(f"unsupported dtype {t}; SS1 takes bfloat16 or float32")


class SS1Layer:
    """One SS1 layer's hash tables on the current CUDA device.

    forward(X[M, K], Wc[N, K/c]) -> Y[M, N]; X, Wc, Y share a dtype (bf16 or fp32) and live
    on the device the layer was created on.
    """

    def __init__(self, K: int, N: int, c: int, BK: int, BN: int, seed: int):
        self.K, self.N, self.c, self.BK, self.BN, self.seed = K, N, c, BK, BN, seed
        h = ctypes.c_void_p()
        _check(lib().ss1_create(K, N, c, BK, BN, seed & 0xFFFFFFFFFFFFFFFF, ctypes.byref(h)), "ss1_create")
        self._h = h
        self.device = torch.cuda.current_device()

    @property
    def handle(self) -> ctypes.c_void_p:
        if self._h is None:
            raise RuntimeError("layer destroyed")
        return self._h

    def forward(self, X: torch.Tensor, Wc: torch.Tensor, out: Optional[torch.Tensor] = None,
                kernel: int = Kernel.AUTO, stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        if X.dim() != 2 or X.shape[1] != self.K:
            raise ValueError(f"X must be [M, {self.K}]")
        if Wc.shape != (self.N, self.K // self.c):
            raise ValueError(f"Wc must be [{self.N}, {self.K // self.c}]")
        if X.dtype != Wc.dtype or not X.is_cuda or not Wc.is_cuda:
            raise ValueError("X and Wc must be CUDA tensors of one dtype")
        if not (X.is_contiguous() and Wc.is_contiguous()):
            raise ValueError("X and Wc must be contiguous")
        if X.device.index != self.device or Wc.device.index != self.device:
            raise ValueError(f"X and Wc must be on cuda:{self.device}, where the layer's tables are")
        M = X.shape[0]
        if out is None:
            out = torch.empty((M, self.N), dtype=X.dtype, device=X.device)
        elif out.shape != (M, self.N) or out.dtype != X.dtype or not out.is_contiguous() or out.device != X.device:
            raise ValueError("out must be a contiguous [M, N] tensor of X's dtype on X's device")
        st = stream if stream is not None else torch.cuda.current_stream(X.device)
        _check(lib().ss1_forward_with(self.handle, X.data_ptr(), Wc.data_ptr(), out.data_ptr(), M,
                                      _dtype_code(X.dtype), int(kernel), st.cuda_stream), "ss1_forward")
        return out

    __call__ = forward

    def select_kernel(self, M: int, dtype: torch.dtype = torch.bfloat16) -> Kernel:
        k = ctypes.c_int()
        _check(lib().ss1_select_kernel(self.handle, M, _dtype_code(dtype), ctypes.byref(k)), "ss1_select_kernel")
        return Kernel(k.value)

    def tables(self) -> Tuple[np.ndarray, np.ndarray]:
        NB = self.N // self.BN
        h = np.empty((NB, self.K), dtype=np.int32)
        g = np.empty((NB, self.K), dtype=np.int8)
        _check(lib().ss1_get_tables(self.handle, h.ctypes.data, g.ctypes.data), "ss1_get_tables")
        return h, g

    def device_status(self) -> Tuple[int, int]:
        d = ctypes.c_int32()
        st = lib().ss1_device_status(self.handle, ctypes.byref(d))
        return st, d.value

    def close(self):
        if getattr(self, "_h", None) is not None:
            lib().ss1_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def forward_noalloc(X: torch.Tensor, Wc: torch.Tensor, K: int, N: int, c: int, BK: int, BN: int, seed: int,
                    out: Optional[torch.Tensor] = None, device_status: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Y = SS1(X) through ss1_forward_noalloc: no handle, the tables rebuilt in the library's
    static device region on `stream`. Calls must not overlap on the device (they share that
    region). `device_status`, if given, is a CUDA int32 tensor of one element that receives the
    kernels' bounded-wait status."""
    if X.dim() != 2 or X.shape[1] != K:
        raise ValueError(f"X must be [M, {K}]")
    if Wc.shape != (N, K // c):
        raise ValueError(f"Wc must be [{N}, {K // c}]")
    if X.dtype != Wc.dtype or not X.is_cuda or not Wc.is_cuda:
        raise ValueError("X and Wc must be CUDA tensors of one dtype")
    if not (X.is_contiguous() and Wc.is_contiguous()):
        raise ValueError("X and Wc must be contiguous")
    if X.device != Wc.device or X.device.index != torch.cuda.current_device():
        raise ValueError("X and Wc must be on the current CUDA device (the library runs there)")
    M = X.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=X.dtype, device=X.device)
    elif out.shape != (M, N) or out.dtype != X.dtype or not out.is_contiguous() or out.device != X.device:
        raise ValueError("out must be a contiguous [M, N] tensor of X's dtype on X's device")
    if device_status is not None and (device_status.dtype != torch.int32 or device_status.device != X.device
                                      or device_status.numel() < 1):
        raise ValueError("device_status must be an int32 tensor on X's device")
    st = stream if stream is not None else torch.cuda.current_stream(X.device)
    status_ptr = device_status.data_ptr() if device_status is not None else None
    _check(lib().ss1_forward_noalloc(K, N, c, BK, BN, seed & 0xFFFFFFFFFFFFFFFF, X.data_ptr(), Wc.data_ptr(),
                                     out.data_ptr(), M, _dtype_code(X.dtype), status_ptr, st.cuda_stream),
           "ss1_forward_noalloc")
    return out
