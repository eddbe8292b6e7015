"""SS1 (Sketch Structured Transform) linear-layer forward for NVIDIA B200 (sm_100a).

The compute path lives in the C-ABI library `libss1.so` (hand-written CUDA, built in-tree by
`build.py`); `ss1` is a thin ctypes binding over it. PyTorch is used only for device memory
and streams. Nothing here falls back to a CPU or library implementation: if the CUDA
library is missing, the binding raises.
"""

from .workloads import WORKLOADS, BENCH_WORKLOAD, Layer, make_inputs  # noqa: F401

__all__ = ["WORKLOADS", "BENCH_WORKLOAD", "Layer", "make_inputs", "SS1Layer", "lib"]


def __getattr__(name):
    # the binding is imported lazily so that CPU-only users of the workloads never dlopen CUDA
    if name in ("SS1Layer", "lib", "Kernel"):
        from . import ss1
        return getattr(ss1, name)
    raise AttributeError(name)
