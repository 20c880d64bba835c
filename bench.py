#!/usr/bin/env python
"""Benchmark of the ConvRot packed-INT4 quantized linear on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the hot path over one batch: fused rotate+quant (K1)
of x (8192 x 3840 bf16, G = 64) into packed int4, then the tcgen05 W4A4 GEMM
with the rowwise-scale epilogue (K2) against packed int4 weights
(3840 x 3840) -> bf16 y. `value` = 2*M*N*K per step / step time, in TOPS, summed
over ranks (weak scaling: every rank runs its own replica, no collective on
the data path) and divided by the slowest rank's time.

Also reported on the same JSON line: per-kernel times and the roofline of the
dominant kernel (K2, against the int8 tensor peak derived from the measured
bf16 peak), the end-to-end number through the C ABI with host buffers, the
W4A8 / AWQ W4A16 decode GEMVs in weight GB/s, SM clocks sampled during the
timed region, and the CPU oracle timed on a bounded sample (cpu_baseline).
`--impl reference` times the CPU oracle itself as the reference arm.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_quantized_linear_rotate_b200 import workloads as WL  # noqa: E402

METRIC = "W4A4 linear TOPS (M=8192) + W4A8/W4A16 GEMV weight GB/s, % of B200 roofline"
L2_BYTES = 126 * 1024 * 1024
INT8_PER_BF16 = 2.0      # nominal dense int8 / bf16 tensor throughput ratio (4.5 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(files) -> str:
    """Hash of the named files under csrc/ (a kernel's own header and the device helpers it uses)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "bit_quantized_linear_rotate_b200", "csrc")
    for f in sorted(files):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def load_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on this kernel's exact sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(e.get("sources", [])):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml as N
            N.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            try:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self._h = N.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self._h = N.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self._h, N.NVML_CLOCK_SM)
            self._N = N
        except Exception:
            self._h = None

    def _run(self):
        N = self._N
        get_r = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            N.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(N.nvmlDeviceGetClockInfo(self._h, N.NVML_CLOCK_SM))
                r = get_r(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    dev = "cuda" if torch.cuda.is_available() and dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_e2e(e2e: dict, ops_per_step: float, world: int) -> dict:
    """Whole-job end-to-end figure: the slowest rank's step time, the units
    and copied bytes of all ranks (every rank feeds its own replica)."""
    ms = max_over_ranks(e2e["ms_per_step"], world)
    out = dict(e2e)
    out["ms_per_step"] = ms
    out["value"] = ops_per_step * world / (ms * 1e-3) / 1e12
    out["h2d_bytes_per_step"] = e2e["h2d_bytes_per_step"] * world
    out["d2h_bytes_per_step"] = e2e["d2h_bytes_per_step"] * world
    return out


def barrier(world: int):
    if world > 1:
        dist.barrier()


# ------------------------------------------------------------ CPU oracle legs

def oracle_linear_sample(w, rows: int):
    """Times the oracle (as it stands) on the first `rows` rows of the workload."""
    import oracle as O
    d = WL.linear_inputs(w)
    x = d["x"][:rows].float().numpy().astype(np.float64)
    wp = d["w_packed"].numpy()
    sw = d["w_scale"].float().numpy().astype(np.float64)
    t0 = time.perf_counter()
    O.linear_w4a4(x, wp, sw, w.G)
    dt = time.perf_counter() - t0
    return dt


def cpu_baseline(w, rows: int, min_seconds: float = 10.0, max_passes: int = 8):
    """The oracle on `rows` rows of the workload, repeated until about `min_seconds` of CPU work."""
    rows = min(rows, w.M)
    total, passes = 0.0, 0
    while passes < max_passes and (passes == 0 or total < min_seconds):
        total += oracle_linear_sample(w, rows)
        passes += 1
    ops = 2.0 * rows * w.N * w.K * passes
    out = {"value": ops / total / 1e12, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
           "sample": f"first {rows} of {w.M} rows of {w.name} (full K, N), {passes} passes, {total:.1f} s"}
    out["single_thread"] = oracle_single_thread(w)
    return out


def oracle_single_thread(w, rows: int = 256):
    """The same oracle with its BLAS limited to one thread, on a short row sample."""
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return None
    with threadpool_limits(limits=1):
        dt = oracle_linear_sample(w, rows)
    return {"value": 2.0 * rows * w.N * w.K / dt / 1e12, "unit": "TOPS", "cores": 1,
            "sample": f"first {rows} of {w.M} rows of {w.name}, one pass, {dt:.1f} s"}


# ------------------------------------------------------------------ GPU legs

def time_linear(ck, w, steps: int, warmup: int, world: int, dev):
    """The linear step as its two C-ABI calls (what ck_linear_w4a4 runs), timed per kernel."""
    d = WL.linear_inputs(w)
    per_copy = d["x"].numel() * 2 + d["w_packed"].numel() + w.M * w.N * 2
    R = max(2, -(-2 * L2_BYTES // per_copy))
    xs = [d["x"].to(dev) for _ in range(R)]
    wps = [d["w_packed"].to(dev) for _ in range(R)]
    sw = d["w_scale"].to(dev)
    ys = [torch.empty(w.M, w.N, device=dev, dtype=torch.bfloat16) for _ in range(R)]
    ws = torch.empty(ck.linear_w4a4_workspace_bytes(w.M, w.K), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream()

    def step(i, ev=None):
        c = i % R
        if ev is not None:
            ev[0].record(stream)
        ck.linear_w4a4_quantize(xs[c], w.G, ws)
        if ev is not None:
            ev[1].record(stream)
        ck.linear_w4a4_matmul(w.M, w.K, wps[c], sw, ws, out=ys[c])
        if ev is not None:
            ev[2].record(stream)

    for i in range(warmup):
        step(i)
    ck.device_error_check()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    # the timed region: steps back to back (the kernels are programmatic dependents of
    # each other, so no event is recorded between them here)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        start.record(stream)
        for i in range(steps):
            step(i)
        stop.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ck.device_error_check()
    total_ms = start.elapsed_time(stop)
    # per-kernel breakdown in a second pass, with events between the kernels
    nb = min(steps, 200)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nb)]
    for i in range(nb):
        step(i, evs[i])
    torch.cuda.synchronize()
    k1 = [e[0].elapsed_time(e[1]) for e in evs]
    k2 = [e[1].elapsed_time(e[2]) for e in evs]

    # the same product through the other operand paths: int8 codes in natural order with signed
    # weight decode (ck_gemm_w4a8), pre-decoded int8 weights (ck_unpack_int4 once, then
    # ck_gemm_s8), and packed int4 activations (ck_gemm_w4a4)
    qa, sa = ck.rotate_quant_rowwise_i8(xs[0], w.G, 4)
    w8s = [ck.unpack_int4(wp) for wp in wps]
    qp, _ = ck.rotate_quant_rowwise(xs[0], w.G, 4)
    variants = {
        "gemm_w4a8_natural_us": 1e3 * time_rotating(lambda c: ck.gemm_w4a8(qa, sa, wps[c], sw, out=ys[c]), R, 20, 3),
        "gemm_s8_predecoded_us": 1e3 * time_rotating(lambda c: ck.gemm_s8(qa, sa, w8s[c], sw, out=ys[c]), R, 20, 3),
        "gemm_w4a4_packed_a_us": 1e3 * time_rotating(lambda c: ck.gemm_w4a4(qp, sa, wps[c], sw, out=ys[c]), R, 20, 3),
        "unpack_int4_us": 1e3 * time_rotating(lambda c: ck.unpack_int4(wps[c], out=w8s[c]), R, 20, 3),
    }
    del w8s
    return {"total_ms": total_ms, "k1_ms": statistics.mean(k1), "k2_ms": statistics.mean(k2),
            "copies": R, "clocks": clk.summary(), "variants": variants}


def time_linear_e2e(ck, w, steps: int, warmup: int, dev):
    """ck_linear_w4a4 fed from host memory: every step copies its x in (pinned H2D), runs the
    linear and copies its y out (D2H), as a host-fed serving loop would. Upload, compute and
    download run on three streams with two device buffers, so step i + 1's upload and step
    i - 1's download overlap step i's linear; the rate is the whole pipeline's."""
    d = WL.linear_inputs(w)
    x_h = d["x"].pin_memory()
    y_h = [torch.empty(w.M, w.N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    x_d = [torch.empty_like(d["x"], device=dev) for _ in range(2)]
    y_d = [torch.empty(w.M, w.N, device=dev, dtype=torch.bfloat16) for _ in range(2)]
    wp, sw = d["w_packed"].to(dev), d["w_scale"].to(dev)
    ws = torch.empty(ck.linear_w4a4_workspace_bytes(w.M, w.K), device=dev, dtype=torch.uint8)
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    x_ready, x_free = [ev(), ev()], [ev(), ev()]
    y_ready, y_free = [ev(), ev()], [ev(), ev()]
    started = [False, False]

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(x_free[b])          # the linear of step i - 2 has read x_d[b]
            x_d[b].copy_(x_h, non_blocking=True)
            x_ready[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(x_ready[b])
            if started[b]:
                s_cmp.wait_event(y_free[b])         # step i - 2's y has left y_d[b]
            ck.linear_w4a4(x_d[b], wp, sw, w.G, workspace=ws, out=y_d[b], stream=s_cmp)
            x_free[b].record(s_cmp)
            y_ready[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(y_ready[b])
            y_h[b].copy_(y_d[b], non_blocking=True)
            y_free[b].record(s_out)
        started[b] = True

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(warmup, warmup + steps):
        step(i)
    s_in.wait_stream(s_out)
    e.record(s_in)
    torch.cuda.synchronize()
    ms = a.elapsed_time(e) / steps
    return {"value": 2.0 * w.M * w.N * w.K / (ms * 1e-3) / 1e12, "unit": "TOPS",
            "h2d_bytes_per_step": x_h.numel() * 2, "d2h_bytes_per_step": y_h[0].numel() * 2,
            "ms_per_step": ms, "pipeline": "H2D / linear / D2H on three streams, two device buffers"}


def time_rotating(fn, n_copies: int, iters: int, warmup: int, graph: bool = True):
    """Device ms per call of fn(copy) over rotating buffer copies.

    With graph=True the calls are captured once in a CUDA graph (as a decode
    loop would run them) and the graph is replayed, so the timing is the
    kernels' back-to-back device time rather than the host's launch rate.
    """
    for i in range(warmup):
        fn(i % n_copies)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if not graph:
        a.record()
        for i in range(iters):
            fn(i % n_copies)
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters
    per_graph = n_copies * max(1, 20 // n_copies)
    cg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cg, capture_error_mode="relaxed"):
        for i in range(per_graph):
            fn(i % n_copies)
    cg.replay()
    torch.cuda.synchronize()
    reps = max(1, iters // per_graph)
    a.record()
    for _ in range(reps):
        cg.replay()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (reps * per_graph)
    del cg
    return ms


def time_gemvs(ck, dev, hbm_gbs: float, iters: int = 200):
    out = {}
    w = WL.GEMV_W4A8
    for M in w.Ms:
        d = WL.gemv_w4a8_inputs(w, M)
        R = max(2, -(-2 * L2_BYTES // d["w_packed"].numel()))
        wps = [d["w_packed"].to(dev) for _ in range(R)]
        sw = d["w_scale"].to(dev)
        xq, xs = ck.rotate_quant_rowwise(d["x"].to(dev), 1, 8)      # rowwise int8, no rotation
        y = torch.empty(M, w.N, device=dev, dtype=torch.bfloat16)
        ms = time_rotating(lambda c: ck.gemv_w4a8(xq, xs, wps[c], sw, out=y), R, iters, 10)
        wbytes = w.N * w.K // 2
        allb = wbytes + 2 * w.N + M * w.K + 4 * M + 2 * M * w.N
        out[f"w4a8_M{M}"] = {"us": ms * 1e3, "weight_GBps": wbytes / (ms * 1e-3) / 1e9,
                             "all_GBps": allb / (ms * 1e-3) / 1e9,
                             "frac_hbm": wbytes / (ms * 1e-3) / 1e9 / hbm_gbs, "copies": R,
                             "traffic": load_traffic("w4a8_rowsplit_kernel" if M <= 8 else "w4a8_rowsplit_kernel_m16")}
        # the same product on the tcgen05 alternative (not the default path)
        ms = time_rotating(lambda c: ck.gemv_w4a8_tc(xq, xs, wps[c], sw, out=y), R, iters, 10)
        out[f"w4a8_tc_M{M}"] = {"us": ms * 1e3, "weight_GBps": wbytes / (ms * 1e-3) / 1e9,
                                "frac_hbm": wbytes / (ms * 1e-3) / 1e9 / hbm_gbs, "copies": R,
                                "traffic": load_traffic("gemv_w4a8_tc_kernel")}
        del wps
    w = WL.GEMV_AWQ
    for M in w.Ms:
        d = WL.gemv_awq_inputs(w, M)
        per = d["qweight"].numel() + 2 * (d["wscales"].numel() + d["wzeros"].numel())
        R = max(2, -(-2 * L2_BYTES // per))
        qws = [d["qweight"].to(dev) for _ in range(R)]
        wss = [d["wscales"].to(dev) for _ in range(R)]
        wzs = [d["wzeros"].to(dev) for _ in range(R)]
        x = d["x"].to(dev)
        y = torch.empty(M, w.N, device=dev, dtype=torch.bfloat16)
        ms = time_rotating(lambda c: ck.gemv_awq_w4a16(x, qws[c], wss[c], wzs[c], group_size=w.G, out=y),
                           R, iters, 10)
        wbytes = w.N * w.K // 2
        allb = per + 2 * M * w.K + 2 * M * w.N
        out[f"awq_M{M}"] = {"us": ms * 1e3, "weight_GBps": wbytes / (ms * 1e-3) / 1e9,
                            "all_GBps": allb / (ms * 1e-3) / 1e9,
                            "frac_hbm": wbytes / (ms * 1e-3) / 1e9 / hbm_gbs, "copies": R,
                            "traffic": load_traffic("awq_stream_kernel")}
    return out


def time_other_configs(ck, dev, peaks):
    """The other linear workloads and the standalone rotate+quant at the pages' shapes.

    Graph-replayed over rotating input copies (no copy stays in L2 between calls)."""
    out = {}
    int8_peak = peaks["bf16_tflops"] * INT8_PER_BF16
    for w in (WL.LINEAR_M32, WL.LINEAR_MLP_DOWN):
        d = WL.linear_inputs(w)
        per = d["x"].numel() * 2 + d["w_packed"].numel()
        R = max(2, -(-2 * L2_BYTES // per))
        xs = [d["x"].to(dev) for _ in range(R)]
        wps = [d["w_packed"].to(dev) for _ in range(R)]
        sw = d["w_scale"].to(dev)
        y = torch.empty(w.M, w.N, device=dev, dtype=torch.bfloat16)
        ws = torch.empty(ck.linear_w4a4_workspace_bytes(w.M, w.K), device=dev, dtype=torch.uint8)
        ms = time_rotating(lambda c: ck.linear_w4a4(xs[c], wps[c], sw, w.G, workspace=ws, out=y), R, 100, 5)
        ops = 2.0 * w.M * w.N * w.K
        out[w.name] = {"us": round(ms * 1e3, 2), "TOPS": round(ops / (ms * 1e-3) / 1e12, 1),
                       "frac_int8": round(ops / (ms * 1e-3) / 1e12 / int8_peak, 4),
                       "weight_GBps": round(d["w_packed"].numel() / (ms * 1e-3) / 1e9, 1), "copies": R}
        del xs, wps
    # the W4A8 linear (int8 activation codes) and the W4A4 linear on weights unpacked once to int8
    # (the weight-cache trade: 2x the packed weight bytes resident, no decode in the GEMM)
    for w in (WL.LINEAR_M8192, WL.LINEAR_MLP_DOWN):
        d = WL.linear_inputs(w)
        per = d["x"].numel() * 2 + 3 * d["w_packed"].numel()
        R = max(2, -(-2 * L2_BYTES // per))
        xs = [d["x"].to(dev) for _ in range(R)]
        wps = [d["w_packed"].to(dev) for _ in range(R)]
        w8s = [ck.unpack_int4(wp) for wp in wps]
        sw = d["w_scale"].to(dev)
        y = torch.empty(w.M, w.N, device=dev, dtype=torch.bfloat16)
        ws = torch.empty(ck.linear_w4a4_workspace_bytes(w.M, w.K), device=dev, dtype=torch.uint8)
        ops = 2.0 * w.M * w.N * w.K
        tail = w.name.split("linear_", 1)[1]
        for name, fn in ((f"w4a8_linear_{tail}", lambda c: ck.linear_w4a8(xs[c], wps[c], sw, w.G, workspace=ws, out=y)),
                         (f"w4a4_linear_predecoded_{tail}",
                          lambda c: ck.linear_w4a4_predecoded(xs[c], w8s[c], sw, w.G, workspace=ws, out=y))):
            ms = time_rotating(fn, R, 50, 5)
            out[name] = {"us": round(ms * 1e3, 2), "TOPS": round(ops / (ms * 1e-3) / 1e12, 1),
                         "frac_int8": round(ops / (ms * 1e-3) / 1e12 / int8_peak, 4), "copies": R}
            if "predecoded" in name:
                out[name]["weight_bytes_resident"] = w.N * w.K
                out[name]["weight_bytes_packed"] = w.N * w.K // 2
        del xs, wps, w8s
    # rotate+quant (int8 codes, as the pages' RotateQuant measures) at the pages' activation shapes,
    # plus the MLP-down standalone case (G = 16, bits 4 and 8)
    cases = [(32, 3840, 64, 8), (8192, 3840, 64, 8), (32, 10240, 64, 8), (8192, 10240, 64, 8),
             (8192, 10240, 16, 8), (8192, 10240, 16, 4)]
    for M, K, G, bits in cases:
        g = torch.Generator().manual_seed(M + K + G)
        x0 = WL.activations(M, K, max(1, K // 100), g)
        R = max(2, -(-2 * L2_BYTES // (x0.numel() * 2)))
        xs = [x0.to(dev) for _ in range(R)]
        q = torch.empty((M, K // 2) if bits == 4 else (M, K), device=dev,
                        dtype=torch.uint8 if bits == 4 else torch.int8)
        sc = torch.empty(M, device=dev, dtype=torch.float32)
        ms = time_rotating(lambda c: ck.rotate_quant_rowwise(xs[c], G, bits, q_out=q, scale_out=sc), R, 100, 5)
        nbytes = M * K * 2 + q.numel() + 4 * M
        out[f"rotate_quant_M{M}_K{K}_G{G}_int{bits}"] = {
            "us": round(ms * 1e3, 2), "GBps": round(nbytes / (ms * 1e-3) / 1e9, 1),
            "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4), "copies": R}
        if (M, K, G) == (8192, 3840, 64) and bits == 8:
            # the linear's own quantize phase (permuted codes + row sums), back to back
            ws = torch.empty(ck.linear_w4a4_workspace_bytes(M, K), device=dev, dtype=torch.uint8)
            ms = time_rotating(lambda c: ck.linear_w4a4_quantize(xs[c], G, ws), R, 100, 5)
            nbytes = M * K * 2 + M * K + 8 * M
            # the same time on the survey's algorithmic bytes of a1-a3: x, the packed int4 codes
            # and the row scales (the phase stores its codes one per byte plus row sums instead)
            alg = M * K * 2 + M * K // 2 + 4 * M
            out[f"linear_quantize_M{M}_K{K}_G{G}"] = {
                "us": round(ms * 1e3, 2), "GBps": round(nbytes / (ms * 1e-3) / 1e9, 1),
                "frac_hbm": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                "frac_hbm_packed_codes_bytes": round(alg / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4), "copies": R}
        del xs
    return out


# --------------------------------------------------------------------- arms

def run_ours(args, world, rank, local):
    from bit_quantized_linear_rotate_b200 import ck
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = WL.LINEAR_M8192
    peaks, peak_src = load_peaks()
    t = time_linear(ck, w, args.steps, args.warmup, world, dev)
    ms_step = max_over_ranks(t["total_ms"], world) / args.steps
    ops = 2.0 * w.M * w.N * w.K
    value = ops * world / (ms_step * 1e-3) / 1e12
    int8_peak = peaks["bf16_tflops"] * INT8_PER_BF16
    k2_tops = ops / (t["k2_ms"] * 1e-3) / 1e12
    k1_bytes = w.M * w.K * 2 + w.M * w.K + 8 * w.M       # bf16 in, int8 codes out, scales + row sums
    k1_gbs = k1_bytes / (t["k1_ms"] * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "s8",
        "data": "synthetic",
        "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "G": w.G,
                   "step": "ck_linear_w4a4_quantize + ck_linear_w4a4_matmul (= ck_linear_w4a4)",
                   "parallelism": f"replicas x{world}",
                   "l2": f"inputs rotated over {t['copies']} copies (> 2x L2)"},
        "roofline": {"bound": "tensor", "achieved": round(k2_tops, 1), "peak": round(int8_peak, 1),
                     "unit": "TOPS", "frac": round(k2_tops / int8_peak, 4),
                     "traffic": load_traffic("gemm_w4_kernel"),
                     "kernel": "gemm_w4_kernel (K2)",
                     "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {INT8_PER_BF16} (int8/bf16 nominal)"},
        "kernels": {"rotate_quant_us": round(t["k1_ms"] * 1e3, 2), "gemm_us": round(t["k2_ms"] * 1e3, 2),
                    "rotate_quant_GBps": round(k1_gbs, 1),
                    "rotate_quant_frac_hbm": round(k1_gbs / peaks["hbm_gbs"], 4),
                    "rotate_quant_traffic": load_traffic("rotate_quant_kernel"),
                    **{k: round(v, 2) for k, v in t["variants"].items()}},
        "gpu_launches": 2 * args.steps,
        "clocks": t["clocks"],
    }
    if not args.skip_e2e:
        barrier(world)
        e2e = time_linear_e2e(ck, w, max(3, min(args.steps, 50)), 3, dev)
        line["e2e"] = aggregate_e2e(e2e, ops, world)
    if not args.skip_siblings:
        line["siblings"] = time_gemvs(ck, dev, peaks["hbm_gbs"])
        line["other_configs"] = time_other_configs(ck, dev, peaks)
    if rank == 0 and world == 1 and not args.skip_cpu:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_rows)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_reference(args, world, rank):
    if rank != 0:
        return
    w = WL.LINEAR_M8192
    # size each step's row sample so that the whole run stays around a minute of CPU time
    probe_rows = 64
    per_row = oracle_linear_sample(w, probe_rows) / probe_rows
    rows = int(max(16, min(args.cpu_rows, 60.0 / max(1, args.steps + args.warmup) / per_row)))
    for _ in range(args.warmup):
        oracle_linear_sample(w, rows)
    times = [oracle_linear_sample(w, rows) for _ in range(args.steps)]
    dt = sum(times)
    ops = 2.0 * rows * w.N * w.K * args.steps
    v = ops / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "M": w.M, "K": w.K, "N": w.N, "G": w.G,
                       "step": "CPU oracle linear_w4a4 on a bounded row sample"},
            "cpu_baseline": {"value": v, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"first {rows} of {w.M} rows per step"},
            "e2e": {"value": v, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=8192, help="rows of the CPU oracle sample (at most M)")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-siblings", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        # the CPU oracle runs on rank 0 only; other ranks exit without work or collectives
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")))
        return
    world, rank, local = dist_setup()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
