"""Benchmark of the fused RMSNorm + projection (FlashNorm form) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--m M]
    python bench.py --impl reference ...      # the fp64 CPU oracle, as the reference arm

Default workload: decode QKV projection, d = 4096, N = 6144; one step is one
pass of the hot path over each batch size of the workload, M in {1, 8, 32, 64}
(four calls).  Inputs are seeded synthetic data (the ``workloads`` recipe) with
random-init weights; the folded weight is replicated into enough copies that
the copies together exceed twice the 126 MB L2, and every call reads the next
copy, so no call finds its weight in L2.

Metric: achieved HBM GB/s at decode M (algorithmic bytes: x, W' and y, each
read or written once, per call), or tensor TFLOP/s at prefill M (2 M d N_cols
per call), with the dominant kernel's fraction of the measured roofline.

Multi-GPU (torchrun): one process per GPU; every rank runs its own batch
against its own weight replica (rows of a batch are independent, so the path
shards by rows with no collective; weak scaling).  Timing is on the device
with CUDA events, and the job time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import faulthandler
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as WL  # noqa: E402

METRIC = "fused norm+proj HBM GB/s (decode) & TFLOP/s (prefill); % of roofline"
L2_BYTES = 126 * 1024 * 1024
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# environment
# ---------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(local_units: float, local_ms: float, world: int, device):
    """Whole-job throughput inputs: units summed over ranks, time as the
    maximum over ranks (the slowest rank finishes the job)."""
    if world == 1:
        return local_units, local_ms
    import torch.distributed as dist
    u = torch.tensor([local_units], dtype=torch.float64, device=device)
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(u.item()), float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# ---------------------------------------------------------------------------
_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = None
            props = torch.cuda.get_device_properties(device_index)
            ids = [getattr(props, k, None) for k in ("pci_domain_id", "pci_bus_id", "pci_device_id")]
            if all(isinstance(v, int) for v in ids):
                # NVML wants the "domain:bus:device.function" string, never an integer
                bus_id = f"{ids[0]:08x}:{ids[1]:02x}:{ids[2]:02x}.0"
                try:
                    handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus_id)
                except pynvml.NVMLError:
                    handle = None
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nvml, self._h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that, never guess
            self._nvml = None
            self.error = str(e)
        self.period = period_s

    def _run(self):
        nv, h = self._nvml, self._h
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except AttributeError:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                self.samples.append((sm, reasons))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "no NVML")}
        mhz = [s for s, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        reasons = sorted(name for b, name in _REASONS.items() if bits & b and name != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


# ---------------------------------------------------------------------------
# workload setup
# ---------------------------------------------------------------------------
def algorithmic(M: int, d: int, N: int, swiglu: bool, wbytes_per_elem: int = 2, out: str = "bf16"):
    """Bytes (x and W' read once, the output written once) and flops of one call.
    NVFP4 output: half a byte per element plus one scale byte per 16."""
    ncols = 2 * N if swiglu else N
    out_bytes = M * N // 2 + M * N // 16 if out == "nvfp4" else M * N * 2
    by = M * d * 2 + d * ncols * wbytes_per_elem + out_bytes
    fl = 2.0 * M * d * ncols
    return by, fl


def scale_bytes(wl: WL.Workload) -> int:
    """Bytes of the weight's block scales: fp32 per 128x128 block, or one
    ue8m0 byte per 32 k values per column (MXFP8)."""
    if wl.wtype == "fp8_e4m3_b128":
        return (wl.d // 128) * (wl.ncols // 128) * 4
    if wl.wtype == "mxfp8_e4m3":
        return wl.d * wl.ncols // 32
    return 0


def kernel_source_hash(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "rmsnorm_linear_projection_flashnorm_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profile_traffic(profile_name: str, src_hash: str, M=None):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source; None otherwise.  A summary may give the bytes
    per M ("dram_bytes_per_launch_M256"); the plain key is the figure for the
    workload's own mix of M (the main line).  A record whose M the summary
    does not cover gets None."""
    path = os.path.join(ROOT, "profiles", profile_name)
    try:
        kv = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip().strip("-* ")] = v.strip().strip("`")
        if kv.get("source_sha256") != src_hash:
            return None
        if M is not None:
            v = kv.get(f"dram_bytes_per_launch_M{M}")
            return float(v) if v is not None else None
        return float(kv["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class Setup:
    """Operands of one workload on the device: folded weight copies (rotated so
    that consecutive calls never find their weight in L2), activations for each
    M, outputs, the workspace.  gen="host" draws the inputs with the seeded
    host recipe (and keeps pinned host copies for the end-to-end timing);
    gen="device" draws the same distributions on the device (large prefill
    shapes, where host generation would dominate the run)."""

    def __init__(self, wl: WL.Workload, Ms, device, out: str = "bf16", gen: str = "host"):
        import rmsnorm_linear_projection_flashnorm_b200 as fnb
        from rmsnorm_linear_projection_flashnorm_b200 import torch_api as T
        self.fnb, self.T = fnb, T
        self.wl, self.Ms, self.dev = wl, list(Ms), device
        d, N, sw = wl.d, wl.N, wl.swiglu
        self.wtype = {"bf16": fnb.FN_W_BF16, "fp8_e4m3_b128": fnb.FN_W_FP8_E4M3_B128,
                      "mxfp8_e4m3": fnb.FN_W_MXFP8_E4M3}[wl.wtype]
        Mmax = max(self.Ms)
        if gen == "device":
            x_all, g, W = WL.device_inputs(wl, Mmax, device)
            W0, W1 = (W if sw else (W, None))
        else:
            g = WL.gain(d, wl.seed).to(device)
            if sw:
                W0, W1 = (w.to(device) for w in WL.weights(d, N, wl.seed, halves=2))
            else:
                W0, W1 = WL.weights(d, N, wl.seed).to(device), None
            x_all = WL.activations(Mmax, d, wl.seed, wl.outliers)
        Wp, scales = T.fold(W0, g, W1, wtype=self.wtype)
        wp_bytes = Wp.numel() * Wp.element_size()
        self.copies = max(2, math.ceil(2 * L2_BYTES / wp_bytes) + 1)
        self.Wp = [Wp] + [Wp.clone() for _ in range(self.copies - 1)]
        self.scales = [scales] + ([scales.clone() for _ in range(self.copies - 1)] if scales is not None else
                                  [None] * (self.copies - 1))
        # unfused chain operands (original, unfolded weights) are made on first use
        self.g = g
        self._W_src = (W0, W1)
        self.W_unf = None
        if gen == "device":
            self.x_host = None
            self.x = {M: x_all[:M].contiguous() for M in self.Ms}
        else:
            self.x_host = {M: x_all[:M].contiguous().pin_memory() for M in self.Ms}
            self.x = {M: self.x_host[M].to(device) for M in self.Ms}
        self.out = out
        if out == "nvfp4":
            # codes [M, N/2] and scale bytes [M, N/16], copied to one host buffer
            # per M; a fixed global scale (its value does not change the work)
            self.y = {M: torch.empty((M, N // 2 + N // 16), dtype=torch.uint8, device=device) for M in self.Ms}
            self.y_host = {M: torch.empty((M, N // 2 + N // 16), dtype=torch.uint8).pin_memory() for M in self.Ms} \
                if gen == "host" else None
            self.yq = {M: torch.empty((M, N // 2), dtype=torch.uint8, device=device) for M in self.Ms}
            self.ysf = {M: torch.empty((M, N // 16), dtype=torch.uint8, device=device) for M in self.Ms}
            self.gscale = torch.tensor([448.0 * 6.0 / 8.0], dtype=torch.float32, device=device)
        else:
            self.y = {M: torch.empty((M, N), dtype=torch.bfloat16, device=device) for M in self.Ms}
            self.y_host = {M: torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for M in self.Ms} \
                if gen == "host" else None
        self.ws = T.Workspace(device)
        for M in self.Ms:
            self.ws.get(M, d, N, self.wtype, sw)
        self.fn = fnb.fn_norm_proj_swiglu if sw else fnb.fn_norm_proj
        self.i = 0
        torch.cuda.synchronize()

    def call(self, M, x=None, y=None, stream=None):
        wl, c = self.wl, self.i % self.copies
        self.i += 1
        x = self.x[M] if x is None else x
        y = self.y[M] if y is None else y
        if self.out == "nvfp4":
            st = self.fnb.fn_norm_proj_swiglu_nvfp4(x, M, wl.d, self.Wp[c], self.scales[c], self.wtype, wl.N,
                                                    WL.EPS, self.gscale, self.yq[M], self.ysf[M], self.ws.buf,
                                                    self.ws.buf.numel(), stream)
        else:
            st = self.fn(x, M, wl.d, self.Wp[c], self.scales[c], self.wtype, wl.N, WL.EPS, y, self.ws.buf,
                         self.ws.buf.numel(), stream)
        if st != 0:
            raise RuntimeError(f"norm_proj failed: {self.fnb.status_string(st)}")

    def fetch(self, M):
        """Copy the call's output to pinned host memory (asynchronous)."""
        if self.out == "nvfp4":
            n = self.yq[M].shape[1]
            self.y_host[M][:, :n].copy_(self.yq[M], non_blocking=True)
            self.y_host[M][:, n:].copy_(self.ysf[M], non_blocking=True)
        else:
            self.y_host[M].copy_(self.y[M], non_blocking=True)

    def chain(self, M, stream=None):
        """Unfused chain: standalone RMSNorm kernel -> cuBLAS GEMM -> (silu * up).
        bf16 weights: the norm applies g and the GEMM uses the original W.  fp8
        weights: a dequantisation kernel first turns the stored e4m3 W' (g
        already folded in) into bf16, the norm runs without a gain, and the
        GEMM's interleaved gate/up columns are separated for silu * up."""
        wl, c = self.wl, self.i % self.copies
        self.i += 1
        fp8 = self.wtype != self.fnb.FN_W_BF16
        if fp8:
            if self.W_unf is None:
                self.W_unf = torch.empty_like(self.Wp[0], dtype=torch.bfloat16)
                self.g_one = torch.ones_like(self.g)
            ncols = self.Wp[c].shape[1]
            deq = self.fnb.fn_dequant_mxfp8 if self.wtype == self.fnb.FN_W_MXFP8_E4M3 else self.fnb.fn_dequant_fp8
            st = deq(self.Wp[c], self.scales[c], wl.d, ncols, self.W_unf, stream)
            if st != 0:
                raise RuntimeError(self.fnb.status_string(st))
            W, g = self.W_unf, self.g_one
        else:
            if self.W_unf is None:
                W0, W1 = self._W_src
                Wcat = torch.cat([W0, W1], dim=1) if self.wl.swiglu else W0
                self.W_unf = [Wcat] + [Wcat.clone() for _ in range(self.copies - 1)]
            W, g = self.W_unf[c], self.g
        h = torch.empty((M, wl.d), dtype=torch.bfloat16, device=self.dev)
        st = self.fnb.fn_rmsnorm(self.x[M], M, wl.d, g, WL.EPS, h, stream)
        if st != 0:
            raise RuntimeError(self.fnb.status_string(st))
        z = torch.matmul(h, W)
        if wl.swiglu:
            if fp8:   # stored layout: 128-column gate and up blocks alternate
                z4 = z.view(M, wl.N // 128, 2, 128)
                return (torch.nn.functional.silu(z4[:, :, 0]) * z4[:, :, 1]).reshape(M, wl.N)
            return torch.nn.functional.silu(z[:, :wl.N]) * z[:, wl.N:]
        return z


def run_cpu_baseline(wl: WL.Workload, Ms, budget_s: float = 10.0):
    """The fp64 oracle (unfolded: RMSNorm, then the matmul with the original W
    and g) on this host's cores, on a bounded sample: whole passes over the
    workload's batch sizes until `budget_s` of CPU time has been spent."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        threads = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:
        threads = None
    cores = len(os.sched_getaffinity(0))
    d, N = wl.d, wl.N
    g = WL.gain(d, wl.seed)
    if wl.swiglu:
        W0, W1 = WL.weights(d, N, wl.seed, halves=2)
    else:
        W0, W1 = WL.weights(d, N, wl.seed), None
    x_all = WL.activations(max(Ms), d, wl.seed, wl.outliers)
    nbytes = 0
    passes = 0
    t0 = time.perf_counter()
    while True:
        for M in Ms:
            x = x_all[:M]
            if wl.swiglu:
                O.norm_proj_swiglu(x, g, W0, W1, WL.EPS)
            else:
                O.norm_proj(x, g, W0, WL.EPS)
            nbytes += algorithmic(M, d, N, wl.swiglu)[0]
        passes += 1
        el = time.perf_counter() - t0
        if el >= budget_s or passes >= 1000:
            break
    return {"value": nbytes / el / 1e9, "unit": "GB/s", "cores": threads or cores, "host_cores": cores,
            "kind": "oracle",
            "sample": f"{passes} full pass(es) over M={list(Ms)} of {wl.name} (d={d}, N={N}), "
                      f"fp64 NumPy, {el:.1f} s"}


# ---------------------------------------------------------------------------
# the reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle as O
    wl = WL.WORKLOADS[args.workload]
    Ms = [args.m] if args.m else list(wl.Ms)
    d, N = wl.d, wl.N
    g = WL.gain(d, wl.seed)
    if wl.swiglu:
        W0, W1 = WL.weights(d, N, wl.seed, halves=2)
    else:
        W0, W1 = WL.weights(d, N, wl.seed), None
    x_all = WL.activations(max(Ms), d, wl.seed, wl.outliers)

    def step(j):
        M = Ms[j % len(Ms)]
        x = x_all[:M]
        if wl.swiglu:
            O.norm_proj_swiglu(x, g, W0, W1, WL.EPS)
        else:
            O.norm_proj(x, g, W0, WL.EPS)
        return algorithmic(M, d, N, wl.swiglu)[0]

    for j in range(args.warmup):
        step(j)
    nbytes = 0
    t0 = time.perf_counter()
    for j in range(args.steps):
        nbytes += step(j)
    el = time.perf_counter() - t0
    value = nbytes / el / 1e9
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded workloads recipe; random-init weights)",
        "config": {"workload": wl.name, "M": Ms, "d": d, "N": N, "swiglu": wl.swiglu,
                   "step": "one oracle call per step, cycling through M"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{args.steps} oracle calls cycling M={Ms}"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the fused path
# ---------------------------------------------------------------------------
def _stage(msg: str) -> None:
    if os.environ.get("FN_BENCH_TRACE"):
        print(f"[bench] {msg}", file=sys.stderr, flush=True)


def roofline_entry(units_per_call: float, us_per_call: float, hbm_bound: bool, peaks, peaks_kind, clocks_summary,
                   kernel: str, traffic):
    """Roofline record of one call: algorithmic bytes (decode) or flops (prefill)
    of a call over its in-stream duration, against the measured peak.  A
    tensor-bound run that saw the power cap (or ran well below the maximum SM
    clock) is compared with the sustained GEMM peak, otherwise with the burst
    peak."""
    if hbm_bound:
        peak = float(peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]))
        achieved = units_per_call / (us_per_call / 1e6) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": traffic, "kernel": kernel, "peak_source": f"hbm_gbs ({peaks_kind})",
                "bytes_per_launch": units_per_call, "avg_launch_us": us_per_call}
    ck = clocks_summary
    capped = "sw_power_cap" in ck.get("reasons", []) or bool(
        ck.get("sm_mhz") and ck.get("sm_max_mhz") and ck["sm_mhz"] < 0.9 * ck["sm_max_mhz"])
    burst = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"]))
    peak = sustained if capped else burst
    achieved = units_per_call / (us_per_call / 1e6) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": traffic, "kernel": kernel,
            "peak_source": f"bf16_tflops{'_sustained' if capped else ''} ({peaks_kind})",
            "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
            "flops_per_launch": units_per_call, "avg_launch_us": us_per_call}


def kernel_for(wl: WL.Workload, M: int, out: str, per_m: bool = True):
    """Name of the dominant kernel of a call, its sources and its ncu summary file."""
    # the library's promotion-kernel thresholds: fp8 from 33 rows, MXFP8 above 64
    promotion = out == "bf16" and ((wl.wtype == "fp8_e4m3_b128" and M >= 33) or (wl.wtype == "mxfp8_e4m3" and M > 64))
    # bf16 plain projections with bf16 output at these workloads' sizes (the decode QKV
    # shape) take the cluster decode kernel, which needs no fix-up kernel
    grouped = wl.wtype == "bf16" and not wl.swiglu and out == "bf16"
    if M <= 64 and grouped:
        kname, sources = "decode_cl_kernel", ["decode_cl.cu", "decode_common.cuh", "ptx.cuh"]
        label = "decode_cl_kernel (k split inside clusters, partials reduced in distributed shared memory)"
    elif M <= 64 and not promotion:
        kname, src = {"bf16": ("decode_kernel", "decode.cu"), "fp8_e4m3_b128": ("decode_fp8_kernel", "decode_fp8.cu"),
                      "mxfp8_e4m3": ("decode_mx_kernel", "decode_mx.cu")}[wl.wtype]
        sources = [src, "decode_common.cuh", "ptx.cuh", "nvfp4.cuh"]
        label = f"{kname} (+ decode_fixup_kernel where a tile's k range is split)"
    elif promotion:
        # x split once per call, then the block-scale promotion kernel
        kname, sources = "tc8_kernel", ["tc8.cu", "ptx.cuh"]
        label = "tc8_kernel (after xsplit_rows_kernel)" if wl.wtype == "fp8_e4m3_b128" else \
            "tc8_kernel, block-scaled MMAs (after xsplit_mx_rows_kernel)"
    else:
        once = wl.wtype == "mxfp8_e4m3" or (wl.wtype != "bf16" and M >= 1024)
        # bf16 weights (or a bf16 copy) at M >= 512 with bf16 output run on pairs of SMs
        pair = (wl.wtype == "bf16" or once) and M >= 512 and out == "bf16"
        kname = "tc2_kernel" if pair else "tc_kernel"
        sources = ["tc2.cu" if pair else "tc.cu", "ptx.cuh"] + ([] if pair else ["nvfp4.cuh"])
        label = kname + (" (after the dequantise-once kernel)" if once else "")
    src_hash = kernel_source_hash(sources)
    prof = f"{kname}_{wl.name}{'_nvfp4' if out == 'nvfp4' else ''}.md"
    return kname, label, src_hash, profile_traffic(prof, src_hash, M if per_m else None)


# Same-run records for the rest of the metric: the prefill half (tensor-bound
# shapes) and the other decode workloads, each with its own roofline, clocks
# and unfused chain.
SUB_RECORDS = (
    ("ffn_swiglu", 4096), ("prefill_swiglu_large", 16384), ("fp8_swiglu", 8192), ("fp8_swiglu", 256),
    ("mxfp8_swiglu", 8192), ("mxfp8_swiglu", 256),
    ("ffn_swiglu", 16), ("fp8_swiglu", 1), ("fp8_swiglu", 64), ("mxfp8_swiglu", 1), ("mxfp8_swiglu", 64),
)


def run_sub_record(name: str, M: int, dev, peaks, peaks_kind, world: int, target_s: float = 0.25):
    """One call shape timed on its own: direct calls on the launching stream
    (inputs drawn on the device; weights rotated over copies that together
    exceed twice the L2), CUDA events around n calls, NVML clocks during them,
    then the unfused chain over the same rotation."""
    wl = WL.WORKLOADS[name]
    S = Setup(wl, [M], dev, "bf16", gen="device")
    stream = torch.cuda.current_stream()
    wbyte = 2 if wl.wtype == "bf16" else 1
    by, fl = algorithmic(M, wl.d, wl.N, wl.swiglu, wbyte)
    by += scale_bytes(wl)
    hbm_bound = M <= 64

    def timed(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / n * 1e3          # us per call

    for _ in range(3):
        S.call(M)
    est = timed(lambda: S.call(M), 3)
    n = int(min(2000, max(10, math.ceil(target_s / (est * 1e-6)))))
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        us = timed(lambda: S.call(M), n)
    units, ms = aggregate((by if hbm_bound else fl) * n, us * n / 1e3, world, dev)
    ck = clocks.summary()
    _, label, src_hash, traffic = kernel_for(wl, M, "bf16")
    rec = {"workload": name, "M": M, "d": wl.d, "N": wl.N, "swiglu": wl.swiglu, "weights": wl.wtype,
           "calls": n, "us_per_call": ms * 1e3 / n,
           "value": units / (ms / 1e3) / (1e9 if hbm_bound else 1e12), "unit": "GB/s" if hbm_bound else "TFLOP/s",
           "roofline": roofline_entry(by if hbm_bound else fl, ms * 1e3 / n, hbm_bound, peaks, peaks_kind, ck,
                                      label, traffic),
           "clocks": ck, "l2": f"{S.copies} rotating W' copies", "kernel_source_sha256": src_hash}
    for _ in range(2):
        S.chain(M)
    n_c = int(min(n, max(5, math.ceil(target_s / (timed(lambda: S.chain(M), 2) * 1e-6)))))
    with ClockSampler(dev.index if dev.index is not None else 0) as cclk:
        chain_us = timed(lambda: S.chain(M), n_c)
    chain_us = max_over_ranks(chain_us, world, dev)
    rec["unfused_chain"] = {"us_per_call": chain_us, "fused_speedup": chain_us / rec["us_per_call"],
                            "clocks": cclk.summary(),
                            "what": (f"fn_dequant_{'mx' if wl.wtype == 'mxfp8_e4m3' else ''}fp8 (e4m3 W' -> bf16) -> "
                                     "fn_rmsnorm (no gain) -> torch.matmul (cuBLAS)" if wl.wtype != "bf16" else
                                     "fn_rmsnorm -> torch.matmul (cuBLAS) with unfolded W")
                                    + (" -> silu(gate)*up" if wl.swiglu else "")}
    del S
    torch.cuda.empty_cache()
    return rec


def main():
    faulthandler.enable()
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="fused", choices=["fused", "reference"])
    ap.add_argument("--workload", default="decode_qkv", choices=list(WL.WORKLOAD_ORDER))
    ap.add_argument("--m", type=int, default=0, help="run a single batch size of the workload")
    ap.add_argument("--skip-cpu", action="store_true", help="omit the CPU oracle baseline")
    ap.add_argument("--skip-chain", action="store_true", help="omit the unfused-chain baseline")
    ap.add_argument("--sub", default="all", choices=["all", "none"],
                    help="same-run records of the prefill and other decode shapes")
    ap.add_argument("--out", default="bf16", choices=["bf16", "nvfp4"],
                    help="output format; nvfp4 (SwiGLU workloads) runs the quantising epilogue")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import rmsnorm_linear_projection_flashnorm_b200 as fnb
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        fnb.build()
    barrier(world)
    fnb.lib()

    wl = WL.WORKLOADS[args.workload]
    if args.out == "nvfp4" and not wl.swiglu:
        raise SystemExit("--out nvfp4 needs a SwiGLU workload")
    Ms = [args.m] if args.m else list(wl.Ms)
    _stage("setup")
    S = Setup(wl, Ms, dev, args.out)
    _stage("setup done")
    stream = torch.cuda.current_stream()
    peaks, peaks_kind = load_peaks()
    wbyte = 2 if wl.wtype == "bf16" else 1
    bytes_per_step = sum(algorithmic(M, wl.d, wl.N, wl.swiglu, wbyte, args.out)[0] + scale_bytes(wl) for M in Ms)
    flops_per_step = sum(algorithmic(M, wl.d, wl.N, wl.swiglu, wbyte, args.out)[1] for M in Ms)
    hbm_bound = max(Ms) <= 64

    # warm-up
    for _ in range(args.warmup):
        for M in Ms:
            S.call(M)
    torch.cuda.synchronize()
    _stage("warm-up done")

    # Timed region: K steps, each a replay of a CUDA graph of G steps (the way a
    # decode loop issues many layers' projections per graph), so consecutive
    # calls overlap through programmatic dependent launch exactly as they do in
    # such a loop.  Graph p holds calls p*G*len(Ms) .. of the weight-copy
    # rotation, so consecutive calls always read different copies.  The
    # per-call time is the timed region over the calls it holds: in-stream,
    # kernel boundaries included, and consistent with ms_per_step.
    K = args.steps
    n_calls = len(Ms)
    G = max(1, min(K, math.ceil(16 / n_calls)))
    per_graph = G * n_calls
    n_graphs = S.copies // math.gcd(per_graph, S.copies)
    cap_stream = torch.cuda.Stream()

    def capture(start_call, steps, Ms_):
        S.i = start_call % S.copies
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=cap_stream):
            for _ in range(steps):
                for M in Ms_:
                    S.call(M)
        return gr

    launches0 = fnb.fn_kernel_launches()
    graphs = [capture(gi * per_graph, G, Ms) for gi in range(n_graphs)]
    kernels_per_step = (fnb.fn_kernel_launches() - launches0) // (n_graphs * G)
    tail = [capture(j * n_calls, 1, Ms) for j in range(K % G)]
    _stage(f"{n_graphs} graphs of {G} steps captured, {kernels_per_step} kernels per step")
    for gi in range(max(args.warmup, n_graphs)):
        graphs[gi % n_graphs].replay()
    for gr in tail:
        gr.replay()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_start.record(stream)
        for k in range(K // G):
            graphs[k % n_graphs].replay()
        for gr in tail:
            gr.replay()
        t_end.record(stream)
        torch.cuda.synchronize()
    _stage("timed region done")
    barrier(world)
    elapsed_ms = t_start.elapsed_time(t_end)
    job_units, job_ms = aggregate(float(bytes_per_step if hbm_bound else flops_per_step) * K, elapsed_ms,
                                  world, dev)
    gpu_launches = K * kernels_per_step
    us_per_call = max_over_ranks(elapsed_ms, world, dev) / (K * n_calls) * 1e3
    kname, label, src_hash, traffic = kernel_for(wl, max(Ms), args.out, per_m=len(Ms) == 1)
    ck = clocks.summary()
    units_per_call = (bytes_per_step if hbm_bound else flops_per_step) / n_calls
    roofline = roofline_entry(units_per_call, us_per_call, hbm_bound, peaks, peaks_kind, ck,
                              f"{label}: one fn_norm_proj call, averaged over M={Ms}", traffic)
    roofline["timing"] = "timed region / calls (in-stream, graph replays, kernel boundaries included)"
    value = job_units / (job_ms / 1e3) / (1e9 if hbm_bound else 1e12)
    unit = "GB/s" if hbm_bound else "TFLOP/s"

    # the same timing per batch size (one M per graph), for the breakdown
    per_m = None
    if len(Ms) > 1:
        per_m = {}
        reps = max(1, min(K // G, 50))
        for M in Ms:
            gs = [capture(gi * 16, 1, [M] * 16) for gi in range(max(1, S.copies // math.gcd(16, S.copies)))]
            for gr in gs:
                gr.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            for r in range(reps):
                gs[r % len(gs)].replay()
            e1.record(stream)
            torch.cuda.synchronize()
            us_m = max_over_ranks(e0.elapsed_time(e1), world, dev) / (reps * 16) * 1e3
            by_m = algorithmic(M, wl.d, wl.N, wl.swiglu, wbyte, args.out)[0] + scale_bytes(wl)
            per_m[str(M)] = {"us_per_call": us_m, "GB/s": by_m / (us_m / 1e6) / 1e9,
                             "frac": by_m / (us_m / 1e6) / 1e9 / roofline["peak"]} if hbm_bound else \
                {"us_per_call": us_m}
            del gs

    # End to end through the public API: every step copies its inputs from pinned
    # host memory, makes the fused calls and copies the results back to pinned
    # host memory.  The copies run on their own streams, so a call's input copy
    # and the previous call's output copy overlap the calls (a call waits for its
    # own input, an output copy for its own call).  The step is captured once as a
    # CUDA graph, as a serving loop would; every replay moves all of its bytes.
    e2e_steps = max(1, min(K, 2000))
    h2d = sum(S.x_host[M].numel() * 2 for M in Ms)
    d2h = sum(S.y_host[M].numel() * S.y_host[M].element_size() for M in Ms)
    xs = {M: torch.empty_like(S.x[M]) for M in Ms}
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    # The step's calls are independent: the smallest batch goes first and last
    # comes the next smallest, so only small copies sit at the step's ends (the
    # first input copy and the last output copy overlap no call).
    order = sorted(Ms)
    order = order[:1] + sorted(order[1:], reverse=True)

    def e2e_step():
        cur = torch.cuda.current_stream()
        copy_in.wait_stream(cur)
        copy_out.wait_stream(cur)
        landed = {}
        with torch.cuda.stream(copy_in):
            for M in order:
                xs[M].copy_(S.x_host[M], non_blocking=True)
                landed[M] = torch.cuda.Event()
                landed[M].record(copy_in)
        for M in order:
            cur.wait_event(landed[M])
            S.call(M, x=xs[M])
            done = torch.cuda.Event()
            done.record(cur)
            copy_out.wait_event(done)
            with torch.cuda.stream(copy_out):
                S.fetch(M)
        cur.wait_stream(copy_out)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e2e_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(e2e_graph, stream=cap_stream):
        e2e_step()
    for _ in range(3):
        e2e_graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_units, e2e_ms = aggregate(float(bytes_per_step if hbm_bound else flops_per_step) * e2e_steps,
                                  e0.elapsed_time(e1), world, dev)
    e2e_val = e2e_units / (e2e_ms / 1e3)
    _stage("e2e done")
    e2e = {"value": e2e_val / (1e9 if hbm_bound else 1e12), "unit": unit, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "step": "one CUDA graph replay per step: pinned-host x -> device copies (copy stream), the fused "
                   "calls, device -> pinned-host output copies (second copy stream), each call ordered after "
                   "its input copy and each output copy after its call; calls in the order M = "
                   + ", ".join(str(M) for M in order)}
    del e2e_graph

    # unfused chain (same rotation of weight copies): rmsnorm -> cuBLAS -> silu*up
    chain = None
    if not args.skip_chain and args.out == "bf16":
        for _ in range(3):
            for M in Ms:
                S.chain(M)
        torch.cuda.synchronize()
        c_steps = max(1, min(K, 2000))
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(c_steps):
            for M in Ms:
                S.chain(M)
        c1.record(stream)
        torch.cuda.synchronize()
        chain_ms = max_over_ranks(c0.elapsed_time(c1) / c_steps, world, dev)
        chain = {"ms_per_step": chain_ms, "fused_speedup": chain_ms / (job_ms / K),
                 "what": ("fn_dequant_fp8 kernel (e4m3 W' -> bf16) -> fn_rmsnorm kernel (no gain) -> "
                          "torch.matmul (cuBLAS)" if wl.wtype != "bf16" else
                          "fn_rmsnorm kernel -> torch.matmul (cuBLAS) with unfolded W")
                         + (" -> silu(gate)*up" if wl.swiglu else "")}
    _stage("chain done")
    l2_desc = (f"{S.copies} rotating W' copies "
               f"({S.copies * S.Wp[0].numel() * S.Wp[0].element_size() / 1e6:.0f} MB > L2)")
    del S, xs
    torch.cuda.empty_cache()

    subs = None
    if args.sub == "all" and not args.m and args.workload == "decode_qkv" and args.out == "bf16":
        subs = {}
        for name, M in SUB_RECORDS:
            _stage(f"sub-record {name} M={M}")
            subs[f"{name}_M{M}"] = run_sub_record(name, M, dev, peaks, peaks_kind, world)

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        cpu = run_cpu_baseline(wl, Ms)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": job_ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": ("bf16" if wl.wtype == "bf16" else "bf16 (e4m3 weights)")
                     + (", NVFP4 output" if args.out == "nvfp4" else ""),
            "data": "synthetic (seeded workloads recipe; random-init weights)",
            "config": {"workload": wl.name, "M": Ms, "d": wl.d, "N": wl.N, "swiglu": wl.swiglu, "output": args.out,
                       "weights": wl.wtype, "parallelism": f"replicas x{world} (rows shard, no collective)",
                       "l2": l2_desc,
                       "step": f"{len(Ms)} fused calls, one per M; CUDA graphs of {G} steps",
                       "kernels_per_step": kernels_per_step},
            "roofline": roofline, "per_m": per_m, "cpu_baseline": cpu, "e2e": e2e, "clocks": ck,
            "gpu_launches": gpu_launches, "unfused_chain": chain,
            "kernel_source_sha256": src_hash, "sub_records": subs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
