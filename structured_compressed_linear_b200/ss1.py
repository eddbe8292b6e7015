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
#: The bounds-checked debug build of the same sources (ss1_bounds_check in include/ss1.h).
CHECKED_LIB_PATH = os.path.join(_HERE, "libss1_checked.so")

SYMBOLS = ("ss1_create", "ss1_forward", "ss1_forward_with", "ss1_select_kernel", "ss1_destroy",
           "ss1_get_tables", "ss1_get_info", "ss1_device_status", "ss1_strerror", "ss1_forward_noalloc",
           "ss1_test_device_timeout", "ss1_project", "ss1_backward_workspace", "ss1_backward_input",
           "ss1_backward_weight", "ss1_quantize_fp8", "ss1_forward_fp8", "ss1_forward_ex", "ss1_chain_forward",
           "ss1_chain_fused", "ss1_test_forward_timeout", "ss1_last_launch", "ss1_bounds_check",
           "ss1_test_bounds_check")

#: (N / BN) * K limit of ss1_forward_noalloc (SS1_NOALLOC_MAX_ENTRIES in include/ss1.h).
NOALLOC_MAX_ENTRIES = 983040


class Kernel(IntEnum):
    AUTO = 0
    TC = 1
    SIMT = 2
    SMALLM = 3


class Act(IntEnum):
    NONE = 0
    RELU = 1
    GELU = 2


#: Layers one chain_forward call takes at most (SS1_CHAIN_MAX_LAYERS in include/ss1.h).
CHAIN_MAX_LAYERS = 4


class DType(IntEnum):
    BF16 = 0
    FP32 = 1


_lib = None


class _LaunchInfo(ctypes.Structure):
    """ss1_launch_info of include/ss1.h."""
    _fields_ = [("kernel", ctypes.c_char_p), ("grid_x", ctypes.c_int), ("grid_y", ctypes.c_int),
                ("cluster_y", ctypes.c_int), ("threads", ctypes.c_int), ("smem_bytes", ctypes.c_int),
                ("resident_clusters", ctypes.c_int * 17)]


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
    L.ss1_project.argtypes = [vp, vp, vp, i32, vp]
    sz = ctypes.c_size_t
    L.ss1_backward_workspace.argtypes = [vp, i64, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.ss1_backward_input.argtypes = [vp, vp, vp, vp, i64, i32, vp, sz, vp]
    L.ss1_backward_weight.argtypes = [vp, vp, vp, vp, i64, i32, vp, sz, vp]
    L.ss1_quantize_fp8.argtypes = [vp, i32, i64, i64, vp, vp, vp]
    L.ss1_forward_fp8.argtypes = [vp, vp, vp, vp, vp, i64, vp]
    L.ss1_forward_ex.argtypes = [vp, vp, vp, vp, i32, vp, i64, i32, i32, vp]
    L.ss1_chain_forward.argtypes = [ctypes.POINTER(vp), i32, vp, ctypes.POINTER(vp), ctypes.POINTER(vp),
                                    ctypes.POINTER(i32), ctypes.POINTER(vp), i64, vp]
    L.ss1_chain_fused.argtypes = [ctypes.POINTER(vp), i32, ctypes.POINTER(i32)]
    L.ss1_test_forward_timeout.argtypes = [vp, vp, vp, vp, i64, i64, vp]
    L.ss1_last_launch.argtypes = [ctypes.POINTER(_LaunchInfo)]
    L.ss1_bounds_check.argtypes = [ctypes.POINTER(i32), ctypes.POINTER(u64)]
    L.ss1_test_bounds_check.argtypes = [i64, i64]
    L.ss1_strerror.restype = ctypes.c_char_p
    for name in SYMBOLS:
        if name != "ss1_strerror":
            getattr(L, name).restype = i32
    if path == LIB_PATH:
        _lib = L
    return L


_active = None


def lib() -> ctypes.CDLL:
    """The library every call of this module goes through (libss1.so unless use_library chose another)."""
    return _active if _active is not None else load_library()


def use_library(path: str) -> ctypes.CDLL:
    """Route this module's calls through the library at `path` (CHECKED_LIB_PATH: the checked
    build); use_library(LIB_PATH) switches back. A handle belongs to the library that made it:
    destroy layers before switching."""
    global _active
    _active = None if path == LIB_PATH else load_library(path)
    return lib()


def bounds_check() -> tuple[bool, int]:
    """(checked build?, first failed index test since the last call or 0) of the active library."""
    checked, record = ctypes.c_int(0), ctypes.c_uint64(0)
    _check(lib().ss1_bounds_check(ctypes.byref(checked), ctypes.byref(record)), "ss1_bounds_check")
    return bool(checked.value), int(record.value)


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
        self._lib = lib()   # the library that owns the handle, for every later call
        _check(self._lib.ss1_create(K, N, c, BK, BN, seed & 0xFFFFFFFFFFFFFFFF, ctypes.byref(h)), "ss1_create")
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
        _check(self._lib.ss1_forward_with(self.handle, X.data_ptr(), Wc.data_ptr(), out.data_ptr(), M,
                                      _dtype_code(X.dtype), int(kernel), st.cuda_stream), "ss1_forward")
        return out

    __call__ = forward

    def project(self, W: torch.Tensor, out: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """Wc[N, K/c] closest to the dense weight W[N, K] (ss1_project)."""
        if W.dim() != 2 or W.shape != (self.N, self.K):
            raise ValueError(f"W must be [{self.N}, {self.K}]")
        if not W.is_cuda or not W.is_contiguous() or W.device.index != self.device:
            raise ValueError(f"W must be a contiguous CUDA tensor on cuda:{self.device}")
        shape = (self.N, self.K // self.c)
        if out is None:
            out = torch.empty(shape, dtype=W.dtype, device=W.device)
        elif out.shape != shape or out.dtype != W.dtype or not out.is_contiguous() or out.device != W.device:
            raise ValueError("out must be a contiguous [N, K/c] tensor of W's dtype on W's device")
        st = stream if stream is not None else torch.cuda.current_stream(W.device)
        _check(self._lib.ss1_project(self.handle, W.data_ptr(), out.data_ptr(), _dtype_code(W.dtype), st.cuda_stream),
               "ss1_project")
        return out

    def backward_workspace(self, M: int, dtype: torch.dtype = torch.bfloat16) -> Tuple[int, int]:
        """Workspace bytes of backward_input and backward_weight (ss1_backward_workspace)."""
        a, b = ctypes.c_size_t(), ctypes.c_size_t()
        _check(self._lib.ss1_backward_workspace(self.handle, M, _dtype_code(dtype), ctypes.byref(a), ctypes.byref(b)),
               "ss1_backward_workspace")
        return a.value, b.value

    def _check_cuda(self, **tensors):
        for name, t in tensors.items():
            if not t.is_cuda or not t.is_contiguous() or t.device.index != self.device:
                raise ValueError(f"{name} must be a contiguous CUDA tensor on cuda:{self.device}")

    def backward_input(self, dY: torch.Tensor, Wc: torch.Tensor, out: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None,
                       stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """dX[M, K] = dY[M, N] W_full (ss1_backward_input)."""
        if dY.dim() != 2 or dY.shape[1] != self.N or Wc.shape != (self.N, self.K // self.c) or dY.dtype != Wc.dtype:
            raise ValueError(f"dY must be [M, {self.N}] and Wc [{self.N}, {self.K // self.c}] of one dtype")
        self._check_cuda(dY=dY, Wc=Wc)
        M = dY.shape[0]
        out = torch.empty((M, self.K), dtype=dY.dtype, device=dY.device) if out is None else out
        need = self.backward_workspace(M, dY.dtype)[0]
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dY.device)
        st = stream if stream is not None else torch.cuda.current_stream(dY.device)
        _check(self._lib.ss1_backward_input(self.handle, dY.data_ptr(), Wc.data_ptr(), out.data_ptr(), M,
                                        _dtype_code(dY.dtype), workspace.data_ptr(), workspace.numel(),
                                        st.cuda_stream), "ss1_backward_input")
        return out

    def backward_weight(self, X: torch.Tensor, dY: torch.Tensor, out: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """dWc[N, K/c] from the forward's input X[M, K] and dY[M, N] (ss1_backward_weight)."""
        if X.dim() != 2 or X.shape[1] != self.K or dY.shape != (X.shape[0], self.N) or X.dtype != dY.dtype:
            raise ValueError(f"X must be [M, {self.K}] and dY [M, {self.N}] of one dtype")
        self._check_cuda(X=X, dY=dY)
        M = X.shape[0]
        out = torch.empty((self.N, self.K // self.c), dtype=X.dtype, device=X.device) if out is None else out
        need = self.backward_workspace(M, X.dtype)[1]
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=X.device)
        st = stream if stream is not None else torch.cuda.current_stream(X.device)
        _check(self._lib.ss1_backward_weight(self.handle, X.data_ptr(), dY.data_ptr(), out.data_ptr(), M,
                                         _dtype_code(X.dtype), workspace.data_ptr(), workspace.numel(),
                                         st.cuda_stream), "ss1_backward_weight")
        return out

    def forward_ex(self, X: torch.Tensor, Wc: torch.Tensor, bias: Optional[torch.Tensor] = None, act: int = Act.NONE,
                   out: Optional[torch.Tensor] = None, kernel: int = Kernel.AUTO,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """act(SS1(X) + bias) (ss1_forward_ex); bias [N] of X's dtype or None."""
        if X.dim() != 2 or X.shape[1] != self.K or Wc.shape != (self.N, self.K // self.c) or X.dtype != Wc.dtype:
            raise ValueError(f"X must be [M, {self.K}] and Wc [{self.N}, {self.K // self.c}] of one dtype")
        self._check_cuda(X=X, Wc=Wc)
        if bias is not None:
            if bias.shape != (self.N,) or bias.dtype != X.dtype:
                raise ValueError(f"bias must be [{self.N}] of X's dtype")
            self._check_cuda(bias=bias)
        M = X.shape[0]
        out = torch.empty((M, self.N), dtype=X.dtype, device=X.device) if out is None else out
        st = stream if stream is not None else torch.cuda.current_stream(X.device)
        _check(self._lib.ss1_forward_ex(self.handle, X.data_ptr(), Wc.data_ptr(), bias.data_ptr() if bias is not None else None,
                                    int(act), out.data_ptr(), M, _dtype_code(X.dtype), int(kernel), st.cuda_stream),
               "ss1_forward_ex")
        return out

    def forward_fp8(self, X: torch.Tensor, Wq: torch.Tensor, scale: torch.Tensor, out: Optional[torch.Tensor] = None,
                    stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
        """Y[M, N] (bf16) with FP8 weights: Wq uint8 E4M3 codes [N, K/c], scale float32 [N] (ss1_forward_fp8)."""
        if X.dim() != 2 or X.shape[1] != self.K or X.dtype != torch.bfloat16:
            raise ValueError(f"X must be bf16 [M, {self.K}]")
        if Wq.shape != (self.N, self.K // self.c) or Wq.dtype != torch.uint8:
            raise ValueError(f"Wq must be uint8 [{self.N}, {self.K // self.c}]")
        if scale.shape != (self.N,) or scale.dtype != torch.float32:
            raise ValueError(f"scale must be float32 [{self.N}]")
        self._check_cuda(X=X, Wq=Wq, scale=scale)
        M = X.shape[0]
        out = torch.empty((M, self.N), dtype=torch.bfloat16, device=X.device) if out is None else out
        st = stream if stream is not None else torch.cuda.current_stream(X.device)
        _check(self._lib.ss1_forward_fp8(self.handle, X.data_ptr(), Wq.data_ptr(), scale.data_ptr(), out.data_ptr(), M,
                                     st.cuda_stream), "ss1_forward_fp8")
        return out

    def select_kernel(self, M: int, dtype: torch.dtype = torch.bfloat16) -> Kernel:
        k = ctypes.c_int()
        _check(self._lib.ss1_select_kernel(self.handle, M, _dtype_code(dtype), ctypes.byref(k)), "ss1_select_kernel")
        return Kernel(k.value)

    def tables(self) -> Tuple[np.ndarray, np.ndarray]:
        NB = self.N // self.BN
        h = np.empty((NB, self.K), dtype=np.int32)
        g = np.empty((NB, self.K), dtype=np.int8)
        _check(self._lib.ss1_get_tables(self.handle, h.ctypes.data, g.ctypes.data), "ss1_get_tables")
        return h, g

    def device_status(self) -> Tuple[int, int]:
        d = ctypes.c_int32()
        st = self._lib.ss1_device_status(self.handle, ctypes.byref(d))
        return st, d.value

    def close(self):
        if getattr(self, "_h", None) is not None:
            self._lib.ss1_destroy(self._h)
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


def quantize_fp8(Wc: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(Wq uint8 [N, Kc], scale float32 [N]) from bf16 or fp32 Wc[N, Kc] (ss1_quantize_fp8)."""
    if Wc.dim() != 2 or not Wc.is_cuda or not Wc.is_contiguous():
        raise ValueError("Wc must be a contiguous 2-D CUDA tensor")
    N, Kc = Wc.shape
    Wq = torch.empty((N, Kc), dtype=torch.uint8, device=Wc.device)
    scale = torch.empty((N,), dtype=torch.float32, device=Wc.device)
    st = stream if stream is not None else torch.cuda.current_stream(Wc.device)
    _check(lib().ss1_quantize_fp8(Wc.data_ptr(), _dtype_code(Wc.dtype), N, Kc, Wq.data_ptr(), scale.data_ptr(),
                                  st.cuda_stream), "ss1_quantize_fp8")
    return Wq, scale


def last_launch() -> dict:
    """Shape of the main kernel launched by the last layer call on this thread (ss1_last_launch)."""
    info = _LaunchInfo()
    _check(lib().ss1_last_launch(ctypes.byref(info)), "ss1_last_launch")
    return {"kernel": (info.kernel or b"").decode(), "grid": (info.grid_x, info.grid_y), "cluster_y": info.cluster_y,
            "threads": info.threads, "smem_bytes": info.smem_bytes,
            "resident_clusters": list(info.resident_clusters)}


def _ptr_array(ts):
    return (ctypes.c_void_p * len(ts))(*[t.data_ptr() if t is not None else None for t in ts])


def chain_fused(layers) -> bool:
    """Whether chain_forward runs these layers as one persistent launch (ss1_chain_fused)."""
    hs = (ctypes.c_void_p * len(layers))(*[ly.handle.value for ly in layers])
    f = ctypes.c_int()
    _check(layers[0]._lib.ss1_chain_fused(hs, len(layers), ctypes.byref(f)), "ss1_chain_fused")
    return bool(f.value)


def chain_forward(layers, X: torch.Tensor, Wcs, biases=None, acts=None, outs=None,
                  stream: Optional[torch.cuda.Stream] = None):
    """Every layer's output of a chain of bf16 SS1 layers (ss1_chain_forward)."""
    n = len(layers)
    if not (1 <= n <= CHAIN_MAX_LAYERS) or len(Wcs) != n:
        raise ValueError(f"1 .. {CHAIN_MAX_LAYERS} layers, one Wc each")
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.shape[1] != layers[0].K or not X.is_contiguous():
        raise ValueError(f"X must be contiguous bf16 [M, {layers[0].K}]")
    M = X.shape[0]
    if outs is None:
        outs = [torch.empty((M, ly.N), dtype=torch.bfloat16, device=X.device) for ly in layers]
    for ly, W, Y in zip(layers, Wcs, outs):
        if W.shape != (ly.N, ly.K // ly.c) or W.dtype != torch.bfloat16 or not W.is_contiguous():
            raise ValueError("each Wc must be contiguous bf16 [N, K/c] of its layer")
        if Y.shape != (M, ly.N) or Y.dtype != torch.bfloat16 or not Y.is_contiguous():
            raise ValueError("each output must be contiguous bf16 [M, N] of its layer")
    hs = (ctypes.c_void_p * n)(*[ly.handle.value for ly in layers])
    bias_arr = _ptr_array(biases) if biases is not None else None
    act_arr = (ctypes.c_int * n)(*[int(a) for a in acts]) if acts is not None else None
    st = stream if stream is not None else torch.cuda.current_stream(X.device)
    _check(layers[0]._lib.ss1_chain_forward(hs, n, X.data_ptr(), _ptr_array(Wcs), bias_arr, act_arr, _ptr_array(outs), M,
                                   st.cuda_stream), "ss1_chain_forward")
    return outs


class SS1Function(torch.autograd.Function):
    """Autograd wrapper: Y = SS1(X; Wc) with the CUDA forward and backward entry points.

    Usage: Y = SS1Function.apply(X, Wc, layer) with `layer` an SS1Layer."""

    @staticmethod
    def forward(ctx, X, Wc, layer):
        ctx.layer = layer
        ctx.save_for_backward(X, Wc)
        return layer.forward(X.contiguous(), Wc.contiguous())

    @staticmethod
    def backward(ctx, dY):
        X, Wc = ctx.saved_tensors
        dY = dY.contiguous()
        dX = ctx.layer.backward_input(dY, Wc) if ctx.needs_input_grad[0] else None
        dWc = ctx.layer.backward_weight(X, dY) if ctx.needs_input_grad[1] else None
        return dX, dWc, None
