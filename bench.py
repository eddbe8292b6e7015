"""Benchmark of the SS1 layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload ID] [--m ROWS]
    python bench.py --decode-block C [--m ROWS] [--steps K]   (one Llama-3-8B block's decode latency)

One step = the forward of every layer of the workload (default: the four GPT-2 Small shaped
SS1 layers, M = 8192 tokens, c = 2, BK = BN = 128, bf16 with fp32 accumulation) on seeded
synthetic inputs already resident in HBM. L2 is flushed (a 256 MiB write, outside the event
brackets) before every timed step. Each layer launch is bracketed by CUDA events on the
launching stream; ms_per_step is the mean over the K timed steps of the summed layer times,
max over ranks. Rank 0 prints one JSON line.

Multi-GPU (torchrun): the rows of X are independent, so every rank runs its own batch of M
rows with replicated weights and tables and no data-path collective (weak scaling); the value
is the whole-job dense-equivalent throughput, all ranks' work over the slowest rank's time.

--impl reference times the CPU oracle (the plain float64 definition) on the host cores on a
bounded row sample of the same workload and prints the same line with "impl": "reference".
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SS1 layer ms & dense-equiv TFLOP/s on 1 B200; achieved fraction of roofline"
UNIT = "TFLOP/s (dense-equivalent 2*M*N*K per layer)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=None)
    ap.add_argument("--m", type=int, default=None,
                    help="time the workload's layers with this row count (default: its largest)")
    ap.add_argument("--decode-block", type=int, choices=[2, 8], default=None, metavar="C",
                    help="time one Llama-3-8B block's seven projections back to back at compression C "
                         "(rows: --m, default 1) instead of the workload step")
    ap.add_argument("--op", choices=["forward", "project", "backward", "chain"], default="forward",
                    help="project: time ss1_project (dense W[N, K] -> Wc[N, K/c]) on the workload's layer shapes; "
                         "backward: time ss1_backward_input + ss1_backward_weight on the workload's layers; "
                         "chain: the DLRM top-MLP chain (bias + ReLU between layers) as one ss1_chain_forward")
    ap.add_argument("--graph", action="store_true",
                    help="capture the launches in CUDA graphs and replay them (GPU time without the host's "
                         "per-launch cost): --decode-block, the whole block; otherwise each layer, as R calls "
                         "with Wc rotated over R copies larger than L2")
    ap.add_argument("--only", default=None, metavar="KxNcC",
                    help="keep only the workload's layers of this shape and compression, e.g. 4096x14336c2 "
                         "(a smaller step for profiling one kernel launch)")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 (E4M3) weights with per-neuron scales (ss1_forward_fp8; decode-sized rows only)")
    ap.add_argument("--nvtx", action="store_true",
                    help="name each layer launch with an NVTX range (for profilers that filter on them)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# The CUDA-core FP32 peak that the fp32 (SIMT) path is held to: 148 SMs x 128 FP32 lanes x
# 2 flops per FMA x 1.965 GHz, the B200's maximum SM clock.
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def compute_peak_tflops(L, peaks):
    """Arithmetic peak for a layer's kernel: the bf16 tensor peak, or the FP32 ALU peak for fp32 data."""
    return FP32_ALU_TFLOPS if L.dtype == "fp32" else peaks["bf16_tflops"]


def layer_work(L, fp8=False):
    """Algorithmic work of one layer: dense-equivalent flops, actual flops, bytes moved. With FP8
    weights Wc is one byte per weight plus one float scale per neuron."""
    e = 2 if L.dtype == "bf16" else 4
    dense = 2.0 * L.M * L.N * L.K
    adds = float(L.M) * (L.N // L.BN) * L.K * (1.0 - 1.0 / L.c)
    actual = 2.0 * L.M * L.N * L.K / L.c + adds
    wbytes = (L.N * L.K // L.c + 4.0 * L.N) if fp8 else float(e) * (L.N * L.K // L.c)
    byts = float(e) * (L.M * L.K + L.M * L.N) + wbytes
    return dense, actual, byts


_COMMENT_OR_STRING = re.compile(r'"(?:\\.|[^"\\\n])*"|//[^\n]*|/\*.*?\*/', re.S)


def code_only(text):
    """C++ / CUDA source without its comments and blank lines (string literals kept)."""
    text = _COMMENT_OR_STRING.sub(lambda m: m.group(0) if m.group(0).startswith('"') else "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_hash(names):
    """Hash of the code (comments and blank lines excluded) of the named files under csrc/."""
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "structured_compressed_linear_b200", "csrc")
    for name in names:
        with open(os.path.join(pkg, name), encoding="utf-8") as f:
            h.update(code_only(f.read()).encode())
    return h.hexdigest()[:16]


def layer_key(L):
    return [L.M, L.K, L.N, L.c, L.BK, L.BN]


def traffic_record(kernel_name, layers, path=None):
    """ncu DRAM bytes of one step of `kernel_name` over `layers`, from profiles/dram_traffic.json.

    The record holds only for the layers it was taken on and for the code it was taken on: its
    `sources` (the kernel's own files) must hash as they did then. Otherwise None."""
    p = path or os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    rec = d.get(kernel_name)
    if not rec or rec.get("layers") != [layer_key(L) for L in layers]:
        return None
    if rec.get("source_hash") != source_hash(rec.get("sources", [])):
        return None
    return rec


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index):
        self.ok = False
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append(mhz)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def prepare_oracle(layers, max_rows=None):
    """Inputs and tables for the CPU oracle's row sample (prepared once, not timed)."""
    import oracle as O
    from structured_compressed_linear_b200.workloads import make_inputs
    prepared = []
    for L in layers:
        X, Wc = make_inputs(L if max_rows is None else L.with_M(min(L.M, max_rows)))
        h, g = O.ss1_tables(L.K, L.N, L.c, L.BK, L.BN, L.seed)
        prepared.append((L, X.double().numpy(), Wc.double().numpy(), h, g))
    return prepared


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max(i.get("num_threads", 0) for i in threadpool_info())
        if n:
            return n
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def _oracle_pass(prepared, rows):
    import oracle as O
    t0 = time.perf_counter()
    dense = 0.0
    for L, X, Wc, h, g in prepared:
        r = min(rows, X.shape[0])
        O.ss1_forward(X[:r], Wc, h, g, L.BN)
        dense += 2.0 * r * L.N * L.K
    return dense, time.perf_counter() - t0


def oracle_sample_rate(prepared, budget_s, rows_per_layer=None):
    """Times the CPU oracle (float64 definition) on a row sample of every layer.

    Without a given sample size, the sample grows until one pass takes about budget_s
    (or covers every prepared row). Returns (dense-equivalent TFLOP/s, seconds, rows)."""
    max_rows = max(p[1].shape[0] for p in prepared)
    if rows_per_layer is None:
        rows = 64
        while True:
            _, dt = _oracle_pass(prepared, rows)
            if dt >= budget_s / 2 or rows >= max_rows:
                break
            rows = int(min(max_rows, rows * max(2.0, 0.8 * budget_s / max(dt, 1e-6))))
        rows_per_layer = rows
    dense, dt = 0.0, 0.0
    while dt < min(budget_s, 3.0) or dense == 0.0:      # repeat short samples for a stable time
        d, t = _oracle_pass(prepared, rows_per_layer)
        dense, dt = dense + d, dt + t
    return dense / dt / 1e12, dt, rows_per_layer


# One Llama-3-8B transformer block's projections, in order: q, k, v, o, gate, up, down (K, N).
LLAMA_BLOCK = [(4096, 4096), (4096, 1024), (4096, 1024), (4096, 4096), (4096, 14336), (4096, 14336), (14336, 4096)]


def run_decode_block(args, peaks, peak_src, dev):
    """Decode latency of one Llama-3-8B block: its seven projections back to back at M rows,
    through the public API, as a model's decode step runs them. Wc is rotated over enough
    copies that they exceed L2, so no flush runs between blocks, and one event pair brackets
    all timed blocks. The roofline is the block's bytes (X + Wc + Y) at the HBM copy rate."""
    import torch
    from structured_compressed_linear_b200 import ss1
    M, c = args.m or 1, args.decode_block
    layers = [ss1.SS1Layer(K, N, c, 256, 128, 3) for K, N in LLAMA_BLOCK]
    wc_bytes = sum(N * (K // c) * (1 if args.fp8 else 2) + (4 * N if args.fp8 else 0) for K, N in LLAMA_BLOCK)
    ncopy = max(2, -(-300_000_000 // wc_bytes))
    gen = torch.Generator(device=dev).manual_seed(3)
    Ws = [[(torch.randn(N, K // c, device=dev, generator=gen) * 0.02).to(torch.bfloat16) for K, N in LLAMA_BLOCK]
          for _ in range(ncopy)]
    if args.fp8:
        Ws = [[ss1.quantize_fp8(w) for w in copy] for copy in Ws]
    Xs = [torch.randn(M, K, device=dev, generator=gen).to(torch.bfloat16) for K, _ in LLAMA_BLOCK]
    Ys = [torch.empty(M, N, device=dev, dtype=torch.bfloat16) for _, N in LLAMA_BLOCK]
    kernels = ["SMALLM-FP8"] if args.fp8 else sorted({layer.select_kernel(M).name for layer in layers})

    def block(cp):
        for i, layer in enumerate(layers):
            if args.fp8:
                layer.forward_fp8(Xs[i], Ws[cp][i][0], Ws[cp][i][1], out=Ys[i])
            else:
                layer.forward(Xs[i], Ws[cp][i], out=Ys[i])

    for s in range(max(3, args.warmup) * ncopy):
        block(s % ncopy)
    torch.cuda.synchronize()
    graph = None
    if args.graph:   # one graph holding a block on every Wc copy, replayed; set-up already done above
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for cp in range(ncopy):
                block(cp)
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    if graph is not None:
        reps = max(1, args.steps // ncopy)
        for _ in range(reps):
            graph.replay()
        nblocks = reps * ncopy
    else:
        for s in range(args.steps):
            block(s % ncopy)
        nblocks = args.steps
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / nblocks * 1e3
    for layer in layers:
        st, detail = layer.device_status()
        if st != 0:
            raise RuntimeError(f"device status {detail:#x} after the decode block")
    byts = wc_bytes + sum(2 * (M * K + M * N) for K, N in LLAMA_BLOCK)
    achieved = byts / (us * 1e-6) / 1e9
    print(json.dumps({
        "metric": "SS1 decode block latency (Llama-3-8B q, k, v, o, gate, up, down back to back)"
                  + (", FP8 weights" if args.fp8 else ""),
        "value": us, "unit": "us per block", "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup),
        "higher_is_better": False, "dtype": "bf16 activations, " + ("e4m3 weights" if args.fp8 else "bf16 weights"),
        "data": "synthetic",
        "config": {"workload": f"llama-3-8b block at M={M}, c={c}, BK=256, BN=128", "kernels": kernels,
                   "l2": f"Wc rotated over {ncopy} copies ({ncopy * wc_bytes / 1e6:.0f} MB), no flush",
                   "launch": "CUDA graph replay" if graph is not None else "one API call per layer from Python"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "algorithmic_bytes": byts,
                     "peak_source": peak_src},
    }), flush=True)
    for layer in layers:
        layer.close()


def run_project(args, layers, wid, peaks, peak_src, dev):
    """ss1_project on every distinct layer shape of the workload: W[N, K] (seeded, N(0, 0.02^2))
    -> Wc[N, K/c]. HBM-bound: the algorithmic bytes are W read once and Wc written once. L2 is
    flushed before every timed step; each launch is bracketed by CUDA events."""
    import torch
    from structured_compressed_linear_b200 import ss1
    shapes = []
    for L in layers:
        key = (L.K, L.N, L.c, L.BK, L.BN, L.dtype)
        if key not in [x[0] for x in shapes]:
            shapes.append((key, L))
    objs = []
    gen = torch.Generator(device=dev).manual_seed(7)
    for (K, N, c, BK, BN, dt), L in shapes:
        dtype = torch.bfloat16 if dt == "bf16" else torch.float32
        W = (torch.randn(N, K, device=dev, generator=gen) * 0.02).to(dtype)
        layer = ss1.SS1Layer(K, N, c, BK, BN, L.seed)
        objs.append((L, layer, W, torch.empty((N, K // c), dtype=dtype, device=dev)))
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        for _L, layer, W, Wc in objs:
            layer.project(W, out=Wc)
    torch.cuda.synchronize()
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in objs]
           for _ in range(args.steps)]
    sampler = ClockSampler(dev.index or 0)
    with sampler:
        for s_ in range(args.steps):
            flush.zero_()
            for i, (_L, layer, W, Wc) in enumerate(objs):
                evs[s_][i][0].record(stream)
                layer.project(W, out=Wc)
                evs[s_][i][1].record(stream)
        torch.cuda.synchronize()
    per = []
    total_bytes, total_ms = 0.0, 0.0
    for i, (L, layer, W, Wc) in enumerate(objs):
        ms = statistics.mean(evs[s_][i][0].elapsed_time(evs[s_][i][1]) for s_ in range(args.steps))
        e = W.element_size()
        byts = float(e) * (L.N * L.K + L.N * (L.K // L.c))
        total_bytes += byts
        total_ms += ms
        per.append({"K": L.K, "N": L.N, "c": L.c, "BK": L.BK, "BN": L.BN, "us": ms * 1e3,
                    "gbs": byts / (ms * 1e-3) / 1e9, "frac": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]})
        layer.close()
    achieved = total_bytes / (total_ms * 1e-3) / 1e9
    print(json.dumps({
        "metric": "SS1 dense -> SS1 projection (ss1_project) GB/s on 1 B200; achieved fraction of HBM roofline",
        "value": achieved, "unit": "GB/s (W read + Wc written, algorithmic)", "n_gpus": 1, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": total_ms, "higher_is_better": True, "dtype": layers[0].dtype,
        "data": "synthetic (seeded)", "config": {"workload": f"workload {wid} layer shapes", "l2": "flushed before every step"},
        "layers": per,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "peak_source": peak_src,
                     "kernel": "project_pairs_kernel" if layers[0].dtype == "bf16" else "project_rows_kernel",
                     "algorithmic_bytes": total_bytes},
        "gpu_launches": args.steps * len(objs), "clocks": sampler.summary(),
    }), flush=True)


def backward_work(L):
    """Algorithmic work of one layer's backward pass (both gradients): dense-equivalent flops
    2 * 2 M N K; the method's own flops: the two compressed products 2 * 2 M N K / c, the
    un-sketch adds of dX (M K NB) and the sketch adds of dWc (M NB K (1 - 1/c))."""
    NB = L.N // L.BN
    dense = 4.0 * L.M * L.N * L.K
    actual = 4.0 * L.M * L.N * L.K / L.c + float(L.M) * L.K * NB + float(L.M) * NB * L.K * (1.0 - 1.0 / L.c)
    return dense, actual


def run_backward(args, layers, wid, peaks, peak_src, dev):
    """ss1_backward_input + ss1_backward_weight on every layer of the workload, seeded dY and
    X, workspaces allocated once. L2 flushed before every step; CUDA events around each call."""
    import torch
    from structured_compressed_linear_b200 import ss1
    from structured_compressed_linear_b200.workloads import make_inputs
    objs = []
    for L in layers:
        X, Wc = make_inputs(L)
        gen = torch.Generator().manual_seed(L.M + L.N)
        dY = torch.randn(L.M, L.N, generator=gen).to(X.dtype)
        layer = ss1.SS1Layer(L.K, L.N, L.c, L.BK, L.BN, L.seed)
        wi, ww = layer.backward_workspace(L.M, X.dtype)
        objs.append((L, layer, X.to(dev), Wc.to(dev), dY.to(dev), torch.empty(L.M, L.K, dtype=X.dtype, device=dev),
                     torch.empty(L.N, L.K // L.c, dtype=X.dtype, device=dev),
                     torch.empty(max(wi, ww, 1), dtype=torch.uint8, device=dev)))
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None):
        for i, (L, layer, X, Wc, dY, dX, dWc, ws) in enumerate(objs):
            if evs is not None:
                evs[i][0].record(stream)
            layer.backward_input(dY, Wc, out=dX, workspace=ws)
            if evs is not None:
                evs[i][1].record(stream)
            layer.backward_weight(X, dY, out=dWc, workspace=ws)
            if evs is not None:
                evs[i][2].record(stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in objs] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index or 0)
    with sampler:
        for s_ in range(args.steps):
            flush.zero_()
            step(evs[s_])
        torch.cuda.synchronize()
    per, tot_ms, tot_dense, tot_actual = [], 0.0, 0.0, 0.0
    for i, (L, layer, *_r) in enumerate(objs):
        ms_in = statistics.mean(evs[s_][i][0].elapsed_time(evs[s_][i][1]) for s_ in range(args.steps))
        ms_w = statistics.mean(evs[s_][i][1].elapsed_time(evs[s_][i][2]) for s_ in range(args.steps))
        dense, actual = backward_work(L)
        ms = ms_in + ms_w
        tot_ms += ms
        tot_dense += dense
        tot_actual += actual
        per.append({"K": L.K, "N": L.N, "M": L.M, "c": L.c, "dX_us": ms_in * 1e3, "dWc_us": ms_w * 1e3,
                    "dense_tflops": dense / (ms * 1e-3) / 1e12,
                    "roofline_frac": actual / (peaks["bf16_tflops"] * 1e12) / (ms * 1e-3)})
        st, detail = layer.device_status()
        if st != 0:
            raise RuntimeError(f"device status {detail:#x}")
        layer.close()
    achieved = tot_actual / (tot_ms * 1e-3) / 1e12
    print(json.dumps({
        "metric": "SS1 backward (dX and dWc) dense-equiv TFLOP/s on 1 B200; achieved fraction of roofline",
        "value": tot_dense / (tot_ms * 1e-3) / 1e12, "unit": "TFLOP/s (dense-equivalent 4*M*N*K per layer)",
        "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": tot_ms,
        "higher_is_better": True, "dtype": layers[0].dtype, "data": "synthetic (seeded)",
        "config": {"workload": f"workload {wid} layers at M = {layers[0].M}", "l2": "flushed before every step"},
        "layers": per,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "peak_source": peak_src,
                     "note": "algorithmic flops: the compressed products and the sketch adds; the kernels run the "
                             "dense products (the pages: the backward pass is not made cheaper)"},
        "gpu_launches": None, "clocks": sampler.summary(),
    }), flush=True)


def run_chain(args, layers, wid, peaks, peak_src, dev):
    """The DLRM top-MLP chain of the sweep workload (1024 -> 1024 -> 512 -> 256 at M = 65536, or --m, c = 2):
    bias + ReLU after the first two layers, one ss1_chain_forward per step (one persistent launch
    when the layers allow it), against the same layers as three ss1_forward_ex calls. L2 flushed
    before every step; CUDA events around the chain."""
    import torch
    from structured_compressed_linear_b200 import ss1
    from structured_compressed_linear_b200.workloads import WORKLOADS, make_inputs
    chain = [L for L in WORKLOADS[5] if L.workload == "dlrm-top-mlp"]
    if args.m:
        chain = [L.with_M(args.m) for L in chain]
    X, _ = make_inputs(chain[0])
    lays, Wcs, bs = [], [], []
    gen = torch.Generator().manual_seed(5)
    for L in chain:
        lays.append(ss1.SS1Layer(L.K, L.N, L.c, L.BK, L.BN, L.seed))
        Wcs.append(make_inputs(L)[1].to(dev))
        bs.append((torch.randn(L.N, generator=gen) * 0.1).to(torch.bfloat16).to(dev))
    acts = [ss1.Act.RELU, ss1.Act.RELU, ss1.Act.NONE]
    Xd = X.to(dev)
    outs = [torch.empty(L.M, L.N, dtype=torch.bfloat16, device=dev) for L in chain]
    fused = ss1.chain_fused(lays)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def as_chain():
        ss1.chain_forward(lays, Xd, Wcs, bs, acts, outs)

    def by_layer():
        cur = Xd
        for ly, W, b, a, o in zip(lays, Wcs, bs, acts, outs):
            ly.forward_ex(cur, W, b, a, out=o)
            cur = o

    def timed(fn):
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            ts.append((e0, e1))
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in ts)

    sampler = ClockSampler(dev.index or 0)
    with sampler:
        ms_chain = timed(as_chain)
        ms_layers = timed(by_layer)
    for ly in lays:
        st, detail = ly.device_status()
        if st != 0:
            raise RuntimeError(f"device status {detail:#x}")
        ly.close()
    dense = sum(layer_work(L)[0] for L in chain)
    actual = sum(layer_work(L)[1] for L in chain)
    t_roof = sum(max(layer_work(L)[1] / (peaks["bf16_tflops"] * 1e12), layer_work(L)[2] / (peaks["hbm_gbs"] * 1e9))
                 for L in chain)
    print(json.dumps({
        "metric": "SS1 DLRM top-MLP chain (1024-1024-512-256, bias + ReLU) dense-equiv TFLOP/s on 1 B200",
        "value": dense / (ms_chain * 1e-3) / 1e12, "unit": "TFLOP/s (dense-equivalent 2*M*N*K per layer)",
        "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_chain,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded, the sweep workload's chain)",
        "config": {"workload": f"dlrm-top-mlp chain at M = {chain[0].M}, c = 2, BK = BN = 128",
                   "one_launch": fused, "l2": "flushed before every step"},
        "layer_by_layer_ms": ms_layers,
        "roofline": {"bound": "per layer, the slower of tensor and HBM", "achieved_tflops": actual / (ms_chain * 1e-3) / 1e12,
                     "frac": t_roof / (ms_chain * 1e-3), "frac_layer_by_layer": t_roof / (ms_layers * 1e-3),
                     "peak_source": peak_src},
        "gpu_launches": args.steps * (1 if fused else len(chain)), "clocks": sampler.summary(),
    }), flush=True)


def run_reference(args, layers, wid, rank, world):
    if rank != 0:
        return
    cfg = workload_config(layers, wid, world)
    prepared = prepare_oracle(layers, max_rows=4096)
    threads = oracle_threads()
    n = len(prepared)
    # Step s times layer s mod n of the workload with all its prepared rows: the same rows the
    # cpu_baseline leg times, so the rate is the same quantity (the oracle's cost per row falls
    # as rows are added, its per-layer expansion of W_full being fixed), and each step stays
    # bounded (one layer pass) whatever K and W are.
    all_rows = 1 << 30
    for w in range(args.warmup):
        _oracle_pass([prepared[w % n]], all_rows)
    work, secs = 0.0, 0.0
    for s in range(args.steps):
        d, t = _oracle_pass([prepared[s % n]], all_rows)
        work += d
        secs += t
    value = work / secs / 1e12
    step_ms = secs / args.steps * 1e3
    full_ms = sum(2.0 * L.M * L.N * L.K for L in layers) / (value * 1e12) * 1e3
    rows = max(p[1].shape[0] for p in prepared)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "full_step_ms_extrapolated": full_ms,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"step s: layer s mod {n} of the workload, its first {rows} rows (all rows up "
                                   f"to 4096; float64 definition, numpy BLAS); ms_per_step is that pass, "
                                   f"full_step_ms_extrapolated the whole workload at the measured rate (rows "
                                   f"are independent)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def rank_rows(X, rank):
    """Rank r's rows: rank 0 keeps the seeded rows, others a rank-seeded permutation of them."""
    import torch
    if rank == 0:
        return X
    g = torch.Generator().manual_seed(1000 + rank)
    return X[torch.randperm(X.shape[0], generator=g)]


def max_over_ranks(values, world):
    """Element-wise max of a float64 tensor over all ranks (the slowest rank's timings)."""
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(values, op=dist.ReduceOp.MAX)
    return values


def whole_job_value(dense_flops_per_rank_step, step_ms, world):
    """Dense-equivalent TFLOP/s of the whole job: every rank's work over the slowest rank's time."""
    return world * dense_flops_per_rank_step / (step_ms * 1e-3) / 1e12


def workload_config(layers, wid, world):
    L0 = layers[0]
    return {
        "workload": f"{L0.workload} (workload {wid}): " + ", ".join(f"{L.K}x{L.N}" for L in layers)
                    + f" at M={L0.M} per GPU, c={L0.c}, BK={L0.BK}, BN={L0.BN}",
        "layers": [{"M": L.M, "K": L.K, "N": L.N, "c": L.c, "BK": L.BK, "BN": L.BN} for L in layers],
        "dtype_in": L0.dtype, "accumulate": "fp32", "parallelism": f"replicas x{world} (rows sharded, no collective)",
        "l2": "flushed before every timed step (256 MiB write outside the event brackets)",
    }


def select_layers(workload, m, only=None):
    """The layers one bench step runs: the workload's layers at row count m, or at its largest;
    with `only` ("KxNcC"), just the layers of that shape and compression."""
    from structured_compressed_linear_b200.workloads import WORKLOADS, BENCH_WORKLOAD
    wid = workload or BENCH_WORKLOAD
    layers = WORKLOADS[wid]
    if m is not None:
        layers = [L for L in layers if L.M == m]
        if not layers:
            raise SystemExit(f"workload {wid} has no layers with M = {m}")
    elif len({L.M for L in layers}) != 1:
        layers = [L for L in layers if L.M == max(x.M for x in layers)]
    if only is not None:
        layers = [L for L in layers if f"{L.K}x{L.N}c{L.c}" == only]
        if not layers:
            raise SystemExit(f"workload {wid} has no layer {only}")
    return wid, layers


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.decode_block is not None:   # a latency measurement on one GPU, not the workload step
        if rank != 0:
            return
        import torch
        from structured_compressed_linear_b200 import build
        build.build()
        torch.cuda.set_device(local)
        peaks, peak_src = load_peaks()
        run_decode_block(args, peaks, peak_src, torch.device("cuda", local))
        return

    if args.op == "chain":   # the MLP chain at its own row count (--m overrides it)
        wid, layers = 5, []
    else:
        wid, layers = select_layers(args.workload, args.m, args.only)

    if args.op in ("project", "backward", "chain"):   # one GPU: projection, backward, or the MLP chain
        if rank != 0:
            return
        import torch
        from structured_compressed_linear_b200 import build
        build.build()
        torch.cuda.set_device(local)
        peaks, peak_src = load_peaks()
        run = {"project": run_project, "backward": run_backward, "chain": run_chain}[args.op]
        run(args, layers, wid, peaks, peak_src, torch.device("cuda", local))
        return

    if args.impl == "reference":
        run_reference(args, layers, wid, rank, world)
        return

    import torch
    import torch.distributed as dist
    from structured_compressed_linear_b200 import build
    build.build()
    from structured_compressed_linear_b200 import ss1
    from structured_compressed_linear_b200.workloads import make_inputs, instance_seed  # noqa: F401

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    peaks, peak_src = load_peaks()
    # inputs: every rank its own rows (seed offset by rank), shared weights and tables
    objs = []
    for L in layers:
        X, Wc = make_inputs(L)
        X = rank_rows(X, rank)
        layer = ss1.SS1Layer(L.K, L.N, L.c, L.BK, L.BN, L.seed)
        Xd, Wd = X.to(dev), Wc.to(dev)
        Yd = torch.empty((L.M, L.N), dtype=Xd.dtype, device=dev)
        objs.append((L, layer, Xd, Wd, Yd, X))
    kernels = [ss1.Kernel(layer.select_kernel(L.M, Xd.dtype)).name for (L, layer, Xd, *_r) in objs]
    fp8 = None
    if args.fp8:   # per-neuron FP8 weights for the decode kernel
        if any(L.M > 64 or L.BN != 128 for L in layers):
            raise SystemExit("--fp8 runs decode-sized layers (M <= 64, BN = 128)")
        fp8 = [ss1.quantize_fp8(Wd) for (_L, _l, _X, Wd, *_r) in objs]
        kernels = ["SMALLM-FP8"] * len(objs)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(evs=None, launches=None):
        for i, (L, layer, Xd, Wd, Yd, _) in enumerate(objs):
            if args.nvtx:
                torch.cuda.nvtx.range_push(f"ss1_forward {L.K}x{L.N} M={L.M} c={L.c}")
            if evs is not None:
                evs[i][0].record(stream)
            if fp8 is not None:
                layer.forward_fp8(Xd, fp8[i][0], fp8[i][1], out=Yd)
            else:
                layer.forward(Xd, Wd, out=Yd)
            if evs is not None:
                evs[i][1].record(stream)
            if launches is not None:
                launches.append(ss1.last_launch())
            if args.nvtx:
                torch.cuda.nvtx.range_pop()

    launches = []
    for w in range(max(args.warmup, 3)):
        flush.zero_()
        step(launches=launches if w == 0 else None)
    torch.cuda.synchronize()
    for (L, layer, *_r) in objs:
        st, detail = layer.device_status()
        if st != 0:
            raise RuntimeError(f"device status {detail:#x} during warm-up")

    K = args.steps
    graph_calls = None
    if args.graph:
        # Per layer, one CUDA graph of R calls with Wc rotated over R copies that together exceed
        # L2 (no flush needed); the per-layer time is a replay's event time / R. The host's cost of
        # each launch drops out; what remains is the kernels back to back on the device.
        graphs = []
        for (L, layer, Xd, Wd, Yd, _) in objs:
            w_bytes = Wd.numel() * Wd.element_size() if fp8 is None else Wd.numel()
            R = max(2, -(-300_000_000 // w_bytes))
            copies = [Wd] + [Wd.clone() for _ in range(R - 1)] if fp8 is None else None
            if fp8 is not None:
                i = len(graphs)
                copies = [fp8[i]] + [(fp8[i][0].clone(), fp8[i][1].clone()) for _ in range(R - 1)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for r in range(R):
                    if fp8 is not None:
                        layer.forward_fp8(Xd, copies[r][0], copies[r][1], out=Yd)
                    else:
                        layer.forward(Xd, copies[r], out=Yd)
            for _ in range(max(args.warmup, 3)):
                g.replay()
            graphs.append((g, R, copies))
        torch.cuda.synchronize()
        graph_calls = [R for (_g, R, _c) in graphs]
        evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in objs]
               for _ in range(K)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(local)
        with sampler:
            for s in range(K):
                for i, (g, _R, _c) in enumerate(graphs):
                    evs[s][i][0].record(stream)
                    g.replay()
                    evs[s][i][1].record(stream)
            torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        per_layer_ms = [[evs[s][i][0].elapsed_time(evs[s][i][1]) / graph_calls[i] for s in range(K)]
                        for i in range(len(objs))]
        del graphs
    else:
        evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in objs]
               for _ in range(K)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        sampler = ClockSampler(local)
        with sampler:
            for s in range(K):
                flush.zero_()
                step(evs[s])
            torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        per_layer_ms = [[evs[s][i][0].elapsed_time(evs[s][i][1]) for s in range(K)] for i in range(len(objs))]
    layer_ms = [statistics.mean(v) for v in per_layer_ms]
    step_ms = sum(layer_ms)
    t = max_over_ranks(torch.tensor([step_ms] + layer_ms, dtype=torch.float64, device=dev), world)
    step_ms, layer_ms = float(t[0]), [float(x) for x in t[1:]]

    # end to end through the public API: pinned host X -> device, forward, device -> pinned host Y.
    # Three streams: copies in, forwards, copies out, with device X and Y double-buffered per layer,
    # so that a step's inputs travel to the device while the previous step's results travel back
    # (PCIe carries both directions at once) and the forwards run in between.
    e2e = None
    if not args.no_e2e and fp8 is None:
        hostX = [x.pin_memory() for (*_r, x) in objs]
        hostY = [torch.empty((L.M, L.N), dtype=Xd.dtype).pin_memory() for (L, _l, Xd, *_r) in objs]
        h2d = sum(x.numel() * x.element_size() for x in hostX)
        d2h = sum(y.numel() * y.element_size() for y in hostY)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        nbuf = 2
        bufX = [[torch.empty_like(Xd) for _ in range(nbuf)] for (_L, _l, Xd, *_r) in objs]
        bufY = [[torch.empty_like(Yd) for _ in range(nbuf)] for (_L, _l, _X, _W, Yd, _x) in objs]
        ev = {k: [[torch.cuda.Event() for _ in range(nbuf)] for _ in objs] for k in ("in", "fwd", "out")}
        used = [[False] * nbuf for _ in objs]

        def e2e_step(s):
            b = s % nbuf
            for li, hx in enumerate(hostX):
                if used[li][b]:
                    s_in.wait_event(ev["fwd"][li][b])     # the forward that read this buffer is done
                with torch.cuda.stream(s_in):
                    bufX[li][b].copy_(hx, non_blocking=True)
                ev["in"][li][b].record(s_in)
            for li, ((L, layer, _X, Wd, _Y, _x), hy) in enumerate(zip(objs, hostY)):
                stream.wait_event(ev["in"][li][b])
                if used[li][b]:
                    stream.wait_event(ev["out"][li][b])  # the copy that read this Y buffer is done
                layer.forward(bufX[li][b], Wd, out=bufY[li][b], stream=stream)
                ev["fwd"][li][b].record(stream)
                s_out.wait_event(ev["fwd"][li][b])
                with torch.cuda.stream(s_out):
                    hy.copy_(bufY[li][b], non_blocking=True)
                ev["out"][li][b].record(s_out)
                used[li][b] = True

        def drain():   # the compute stream waits for every copy back
            for li in range(len(objs)):
                for b in range(nbuf):
                    if used[li][b]:
                        stream.wait_event(ev["out"][li][b])

        for s in range(3):
            e2e_step(s)
        drain()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ke = max(3, min(K, 20))
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for s in range(ke):
            e2e_step(s)
        drain()
        e1.record(stream)
        torch.cuda.synchronize()
        te = max_over_ranks(torch.tensor([e0.elapsed_time(e1) / ke], dtype=torch.float64, device=dev), world)
        e2e = (float(te[0]), h2d, d2h)

    isfp8 = fp8 is not None
    dense_step = sum(layer_work(L, isfp8)[0] for L in layers)
    value = whole_job_value(dense_step, step_ms, world)

    # roofline of the dominant kernel over the step (sum over its launches, one per layer)
    hbm_peak = peaks["hbm_gbs"] * 1e9
    dom = max(set(kernels), key=kernels.count)
    dom_layers = [(L, ms) for L, k, ms in zip(layers, kernels, layer_ms) if k == dom]

    def t_compute(L):
        return layer_work(L)[1] / (compute_peak_tflops(L, peaks) * 1e12)

    t_tc = sum(t_compute(L) for L, _ in dom_layers)
    t_hbm = sum(layer_work(L, isfp8)[2] / hbm_peak for L, _ in dom_layers)
    t_kernel = sum(ms for _, ms in dom_layers) * 1e-3
    ns_frac = sum(max(t_compute(L), layer_work(L, isfp8)[2] / hbm_peak) for L in layers) / (step_ms * 1e-3)
    alu = all(L.dtype == "fp32" for L, _ in dom_layers)
    if t_tc >= t_hbm:
        achieved = sum(layer_work(L)[1] for L, _ in dom_layers) / t_kernel / 1e12
        roof = {"bound": "alu" if alu else "tensor", "achieved": achieved,
                "peak": FP32_ALU_TFLOPS if alu else peaks["bf16_tflops"], "unit": "TFLOP/s"}
    else:
        achieved = sum(layer_work(L, isfp8)[2] for L, _ in dom_layers) / t_kernel / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["peak_source"] = f"{peak_src} (burst figure; MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    if roof["bound"] == "alu":
        roof["peak_source"] = "derived: 148 SMs x 128 FP32 lanes x 2 flops x 1.965 GHz"
    rec = traffic_record(dom, [L for L, _ in dom_layers])
    roof["traffic"] = rec["dram_bytes_per_step"] if rec else None
    roof["kernel"] = dom
    roof["launches_per_step"] = kernels.count(dom)
    roof["per"] = "one step: the sum over that kernel's launches (one per layer)"
    roof["algorithmic_bytes"] = sum(layer_work(L, isfp8)[2] for L, k in zip(layers, kernels) if k == dom)
    roof["algorithmic_flops"] = sum(layer_work(L)[1] for L, k in zip(layers, kernels) if k == dom)
    roof["frac_slower_of_tensor_and_hbm"] = ns_frac

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("bf16 activations, e4m3 weights" if isfp8 else "bf16") if layers[0].dtype == "bf16" else "fp32",
        "data": "synthetic (seeded, shapes of the workload)",
        "config": workload_config(layers, wid, world),
        "layers": [{"K": L.K, "N": L.N, "M": L.M, "c": L.c, "kernel": k, "ms": ms,
                    "dense_tflops": layer_work(L)[0] / (ms * 1e-3) / 1e12,
                    "actual_tflops": layer_work(L)[1] / (ms * 1e-3) / 1e12,
                    "gbs": layer_work(L, isfp8)[2] / (ms * 1e-3) / 1e9,
                    "roofline_frac": max(t_compute(L), layer_work(L, isfp8)[2] / hbm_peak) / (ms * 1e-3),
                    "launch": {"kernel": ln["kernel"], "grid": list(ln["grid"]), "cluster_y": ln["cluster_y"]}}
                   for L, k, ms, ln in zip(layers, kernels, layer_ms, launches)],
        "roofline": roof,
        "gpu_launches": K * (sum(graph_calls) if graph_calls else len(objs)),
        "clocks": sampler.summary(),
    }
    if graph_calls:
        line["config"]["l2"] = "no flush: each layer's Wc rotated over copies larger than L2"
        line["config"]["timing"] = (f"CUDA graph per layer of {graph_calls} calls (Wc copy r in call r), "
                                    "replayed; layer time = replay event time / calls")
    if e2e is not None:
        ms_e, h2d, d2h = e2e
        line["e2e"] = {"value": whole_job_value(dense_step, ms_e, world), "unit": UNIT, "ms_per_step": ms_e,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "note": "X copied from pinned host memory and Y read back every step (copies in, forwards and "
                               "copies out on three streams, device X and Y double-buffered); Wc resident"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, dt, rows = oracle_sample_rate(prepare_oracle(layers), 10.0)
        rows = min(rows, layers[0].M)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                                "sample": f"first {rows} of {layers[0].M} rows of each layer (all {len(layers)} layers), "
                                          f"float64 definition with numpy BLAS, {dt:.1f} s timed"}
    for (L, layer, *_r) in objs:
        st, detail = layer.device_status()
        if st != 0:
            raise RuntimeError(f"device status {detail:#x}")
        layer.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
