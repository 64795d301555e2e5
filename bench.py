"""Benchmark of the NVFP4 hot path on the video-DiT layers (M=32768 tokens,
hidden 3072: QKV 3072->9216, MLP fc1 3072->12288, fc2 12288->3072).

One step = for every layer: NVFP4-quantize the bf16 activation X (tensor amax
pass + quantize pass) and run the W4A4 GEMM Y = X W^T with a bf16 epilogue.
Weights are quantized once, before timing (static weights).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Rank 0 prints one JSON line.  value = GEMM FLOPs of all ranks' steps / max
over ranks of the device time of the K steps (quantization included).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "video_dit"
METRIC = "NVFP4 W4A4 GEMM TFLOPS and % of dense FP4 peak; quantize GB/s vs HBM"
FP4_OVER_BF16 = 4.0          # nominal dense FP4 / dense bf16 tensor throughput (9 / 2.25 PFLOP/s)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# quantize, algorithmic bytes per element: 2 (amax read) + 2 (read) + 0.5 (codes) + 1/16 (scales)
QUANT_BYTES_PER_ELEM = 4.5625
# fake quantization (bf16 in, bf16 out, 1-bit clip mask): 2 (amax read) + 2 (read) + 2 (y) + 1/8 (mask);
# with a given tensor scale no amax read; the masked STE backward reads the gradient and the mask and
# writes the gradient
QAT_FWD_DYNAMIC_BYTES = 6.125
QAT_FWD_GIVEN_BYTES = 4.125
QAT_BWD_BYTES = 4.125
# MX quantize: 2 (read) + 0.5 (codes) + 1/32 (E8M0 scales), no amax pass
MX_QUANT_BYTES_PER_ELEM = 2.53125


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK, "fallback"


class ClockSampler:
    """nvidia-smi samples (clocks and throttle reasons), kept only when they
    fall inside the timed region (host monotonic time between mark_start and
    mark_end)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int, period_ms: int = 20):
        self.idx = gpu_index
        self.period_ms = period_ms
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return

        def reader():
            for line in self.proc.stdout:
                self.lines.append((time.monotonic(), line))
        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, power, smax, reasons = [], [], None, set()
        for t, line in self.lines:
            if self.t0 is not None and not (self.t0 <= t <= self.t1):
                continue
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(self.NAMES, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "power_w": round(statistics.median(power), 1) if power else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus: int):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if os.environ.get("NVFP4_BENCH_BACKEND", "nccl") == "nccl" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- oracle leg
# ----------------------------------------------------------------- CPU oracle legs
def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OracleRunner:
    """The CPU oracle as it stands, spread over host threads by rows.

    Rows are independent once the tensor scale is known, so a tensor's rows
    are cut into slices (for the quantizer multiples of 128 rows, so that the
    slices' scale buffers concatenate into the whole tensor's layout) and each
    thread calls the unchanged oracle on one slice; the oracle's C library
    releases the GIL while it runs.  The tensor scale of a whole tensor is the largest of
    its slices' scales (the division by 2688 is monotone and rounds once)."""

    def __init__(self, threads: int):
        from concurrent.futures import ThreadPoolExecutor
        self.threads = max(1, threads)
        self.pool = ThreadPoolExecutor(self.threads) if self.threads > 1 else None

    def _slices(self, rows: int, align: int = 128):
        per = -(-rows // self.threads)
        per = max(align, -(-per // align) * align)
        return [slice(r, min(rows, r + per)) for r in range(0, rows, per)]

    def _map(self, fn, items):
        items = list(items)
        if self.pool is None or len(items) == 1:
            return [fn(i) for i in items]
        return list(self.pool.map(fn, items))

    def tensor_scale(self, x):
        import numpy as np
        import oracle
        return max(self._map(lambda sl: np.float32(oracle.tensor_scale(x[sl])), self._slices(x.shape[0])))

    def quantize(self, x, scale=None):
        """(codes, sf, g) of oracle.quantize(x) with a data-derived (or given) scale."""
        import numpy as np
        import oracle
        g = self.tensor_scale(x) if scale is None else np.float32(scale)
        parts = self._map(lambda sl: oracle.quantize(x[sl], scale=float(g)), self._slices(x.shape[0]))
        return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts]), np.float32(g)

    def gemm(self, a, b):
        """Y = A B^T of two oracle-quantized operands, FP64, rows spread over threads."""
        import numpy as np
        import oracle
        ac, asf, ga = a
        bc, bsf, gb = b
        return np.concatenate(self._map(lambda sl: oracle.gemm_w4a4(ac, asf, ga, bc, bsf, gb, rows=sl),
                                        self._slices(ac.shape[0], align=1)))


def _timed(fn):
    t0 = time.perf_counter()
    out = fn()
    return out, time.perf_counter() - t0


_VIDEO = {}


def host_tensors(workload: str, layer: str):
    """(X, W) of one layer in host memory, drawn by synth on the GPU when
    there is one (the very tensors the GPU arm multiplies, and far faster
    than the host generator), else on the host."""
    import torch
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x, w = synth.layer_tensors(workload, layer, device=dev)
    return x.cpu(), w.cpu()


def video_tensors(runner: OracleRunner):
    """The video workload in host memory: X per layer, and W per layer
    quantized once by the oracle with its own tensor scale (untimed)."""
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    if not _VIDEO:
        for L in synth.WORKLOADS[WORKLOAD].layers:
            x, w = host_tensors(WORKLOAD, L.name)
            _VIDEO[L.name] = (x, runner.quantize(w))
    return _VIDEO


def oracle_step(runner: OracleRunner, rows: int, offset: int = 0):
    """One step of the hot path on the host: for every video layer, quantize
    `rows` rows of its input (data-derived tensor scale over those rows) and
    form those rows of Y = X W^T against all output features.  Returns (GEMM
    FLOPs, seconds)."""
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    data = video_tensors(runner)
    flops, secs = 0, 0.0
    for L in synth.WORKLOADS[WORKLOAD].layers:
        x, wq = data[L.name]
        r0 = (offset * rows) % max(1, L.M - rows + 1)
        xs = x[r0:r0 + rows]
        _, dt = _timed(lambda: runner.gemm(runner.quantize(xs), wq))
        secs += dt
        flops += 2 * xs.shape[0] * L.N * L.K
    return flops, secs


def oracle_quantize_rates(runner: OracleRunner, single: OracleRunner):
    """The oracle's quantize (data-derived scale, 4.5625 algorithmic bytes per
    element as on the GPU) on the full fc1 and fc2 inputs with every host
    core, and on one core on their first 8192 and 2048 rows (25 M values)."""
    data = video_tensors(runner)
    out = {}
    for name in ("fc1", "fc2"):
        x = data[name][0]
        _, t_all = _timed(lambda: runner.quantize(x))
        xs = x[: (1 << 25) // x.shape[1]]
        _, t_one = _timed(lambda: single.quantize(xs))
        out[f"{name}_input_{x.shape[0]}x{x.shape[1]}"] = {
            "all_cores_gbs": round(QUANT_BYTES_PER_ELEM * x.numel() / t_all / 1e9, 4),
            "one_core_gbs": round(QUANT_BYTES_PER_ELEM * xs.numel() / t_one / 1e9, 4),
            "one_core_rows": int(xs.shape[0])}
    return out


def oracle_gemm_rates(runner: OracleRunner, single: OracleRunner, step_rows: int, step_secs_per_row: dict):
    """The FP64 GEMM oracle: PR1 in full on one core, the four DiT-XL/2
    layers in full on every core, and the video layers extrapolated to M rows
    from the step sample."""
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    out = {}
    x, w = host_tensors("pr1", "linear")
    a, b = single.quantize(x), single.quantize(w)
    _, dt = _timed(lambda: single.gemm(a, b))
    out["pr1_128x256x256_one_core_gflops"] = round(2 * 128 * 256 * 256 / dt / 1e9, 3)
    fl, secs = 0, 0.0
    for L in synth.WORKLOADS["dit_xl2"].layers:
        x, w = host_tensors("dit_xl2", L.name)
        a, b = runner.quantize(x), runner.quantize(w)
        _, dt = _timed(lambda: runner.gemm(a, b))
        fl += 2 * L.M * L.N * L.K
        secs += dt
    out["dit_xl2_4_layers_all_cores_gflops"] = round(fl / secs / 1e9, 3)
    out["video_step_extrapolated_s"] = round(sum(step_secs_per_row.values()) * 32768, 1)
    out["video_step_extrapolated_from_rows"] = step_rows
    return out


def epsilon_report(runner: OracleRunner):
    """Lemma III.2's relative error bound (NVFP4-DiT README: 2^-3) next to
    what the quantizer does on each workload's tensors (oracle quantize and
    exact dequantize): the largest per-element |x - Q(x)| / |x| (x != 0), the
    distribution of ||x - Q(x)|| / ||x|| over 16-value blocks, and the
    tensor-level ||x - Q(x)||_F / ||x||_F.  Activations and weights of every
    layer; tensors beyond 1024 rows on their first 1024 rows, quantized with
    the whole tensor's scale."""
    import numpy as np
    import oracle
    from nvfp4_w4a4_gemm_quantize_b200 import synth

    def stats(t, rows=1024):
        g = runner.tensor_scale(t)
        ts = t[:rows]
        codes, sf, _ = runner.quantize(ts, scale=g)
        xv = oracle.bf16_to_f32(oracle.bf16_bits(ts)).astype(np.float64)
        e = oracle.dequantize(codes, sf, g) - xv
        nz = xv != 0
        blk_e = np.sqrt((e.reshape(-1, 16) ** 2).sum(1))
        blk_x = np.sqrt((xv.reshape(-1, 16) ** 2).sum(1))
        rb = blk_e[blk_x > 0] / blk_x[blk_x > 0]
        return {"elem_max": float(np.max(np.abs(e[nz]) / np.abs(xv[nz]))),
                "block_p50": float(np.percentile(rb, 50)), "block_p90": float(np.percentile(rb, 90)),
                "block_p99": float(np.percentile(rb, 99)), "block_max": float(rb.max()),
                "block_frac_above_eps": float((rb > 0.125).mean()),
                "tensor": float(np.sqrt((e ** 2).sum() / (xv ** 2).sum())),
                "rows": int(ts.shape[0]), "of_rows": int(t.shape[0])}

    rep = {"eps_page": 0.125}
    for wl in ("pr1", "dit_xl2", "pixart1024", "video_dit", "w4a16"):
        r = {}
        for L in synth.WORKLOADS[wl].layers:
            if wl == WORKLOAD:
                x, w = _VIDEO[L.name][0], None
            else:
                x, w = host_tensors(wl, L.name)
            if wl != "w4a16":                        # W4A16 keeps its activations in bf16
                r[f"{L.name}.x"] = stats(x)
            if w is not None:
                r[f"{L.name}.w"] = stats(w)
        rep[wl] = r
    return rep


def cpu_baseline_leg(args):
    """The cpu_baseline object of the JSON line (rank 0, N = 1): the oracle on
    the host cores -- the headline value on a row sample of the bench step,
    plus the quantize and GEMM rates and the error report."""
    cores = host_cores()
    runner, single = OracleRunner(cores), OracleRunner(1)
    video_tensors(runner)
    rows = max(16, min(args.ref_rows * cores, 2048))
    per_row = {}
    fl, secs = 0, 0.0
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    for L in synth.WORKLOADS[WORKLOAD].layers:
        x, wq = _VIDEO[L.name]
        _, dt = _timed(lambda: runner.gemm(runner.quantize(x[:rows]), wq))
        per_row[L.name] = dt / rows
        fl += 2 * rows * L.N * L.K
        secs += dt
    return {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": (f"oracle quantize (data-derived scale over the sampled rows) + FP64 GEMM of the first "
                       f"{rows} of 32768 activation rows of each {WORKLOAD} layer against all output features, "
                       f"rows spread over {cores} host threads"),
            "quantize": oracle_quantize_rates(runner, single),
            "gemm": oracle_gemm_rates(runner, single, rows, per_row),
            "epsilon": epsilon_report(runner)}


REF_BUDGET_S = 60.0     # CPU seconds the reference arm's timed steps may take in all


def ref_rows_for_budget(probe_rows: int, probe_secs: float, steps: int, budget_s: float = REF_BUDGET_S) -> int:
    """Rows per layer of one reference-arm step, from the time of a warm-up
    step on probe_rows rows: the cost is close to proportional to the rows,
    so they are scaled to keep all `steps` timed steps within the budget (at
    least one row, at most the layer)."""
    rows = int(probe_rows * budget_s / max(1, steps) / max(probe_secs, 1e-9))
    return max(1, min(rows, 32768))


def run_reference(args):
    rank, world = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    cores = host_cores()
    runner = OracleRunner(cores)
    video_tensors(runner)
    probe = max(16, min(args.ref_rows * cores, 2048))
    s = 0.0
    for _ in range(max(1, args.warmup)):
        _, s = oracle_step(runner, probe)
    rows = ref_rows_for_budget(probe, s, args.steps)
    fl, secs = 0, 0.0
    for i in range(args.steps):
        f, dt = oracle_step(runner, rows, offset=i)
        fl += f
        secs += dt
    v = fl / secs / 1e12
    desc = (f"oracle quantize + FP64 GEMM of {rows} of 32768 activation rows of each {WORKLOAD} layer per step "
            f"(a different row window each step) against all output features, rows spread over {cores} host "
            f"threads")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": step_config(world),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def step_config(world: int) -> dict:
    return {"workload": f"{WORKLOAD}: M=32768, qkv 3072->9216, fc1 3072->12288, fc2 12288->3072 "
                        "(dynamic-scale activation quantize + W4A4 GEMM, bf16 out)",
            "l2": "inputs larger than L2 (X 201-805 MB per layer, >2 GB streamed per step)",
            "parallelism": f"replica per GPU x{world}"}


# ----------------------------------------------------------------- extra measurements
def time_device(fn, iters=10, warmup=3):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def reference_points(dev, layers, w4a16_layers):
    """cuBLAS bf16 on the same shapes (a reference point, never the product
    path) and this library's W4A16 kernel on the weights-only workload."""
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    out = {"cublas_bf16_tflops": {}, "w4a16": {}}
    for L in layers:
        x, w = synth.layer_tensors(WORKLOAD, L.name, device=dev)
        x = x[: L.M]
        ms = time_device(lambda: torch.matmul(x, w.t()))
        out["cublas_bf16_tflops"][L.name] = round(2 * L.M * L.N * L.K / (ms * 1e-3) / 1e12, 1)
        del x, w
    out["w4a16"] = w4a16_points(dev, w4a16_layers)
    out["qat"] = qat_points(dev, layers)
    out["mlp_fc1_gelu"] = mlp_fusion_points(dev, layers)
    out["layernorm_nvfp4"] = layernorm_points(dev)
    out["small_layers"] = small_layer_points(dev)
    out["grouped"] = grouped_points(dev)
    out["mx_and_block_size"] = mx_points(dev, layers)
    out["attention"] = attention_points(dev)
    torch.cuda.empty_cache()
    return out


def time_arm(fn):
    """One arm of a comparison under the 1 kW power cap, where the clock
    follows the recent draw: after a 1 s idle, a 10-launch burst (ms), then 50
    launches in a row (ms, sustained)."""
    import time
    time.sleep(1.0)
    return time_device(fn, iters=10), time_device(fn, iters=50, warmup=0)


def w4a16_points(dev, w4a16_layers):
    """The W4A16 GEMM (bf16 activations x NVFP4 weights, dequantized in the
    mainloop) on the weights-only workload, with cuBLAS bf16 on the same
    shapes beside it (the dequantized product is exact in bf16, so the bf16
    tensor rate is its bar).  Both run under the 1 kW power cap, where the
    clock follows the recent draw: each arm is timed after a 1 s idle, as a
    10-launch burst and then 50 launches in a row (sustained)."""
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    arm = time_arm
    out = {}
    for L in w4a16_layers:
        x, w = synth.layer_tensors("w4a16", L.name, device=dev)
        x = x[: L.M].contiguous()
        W = nv.quantize(w)
        y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device=dev)
        ours = arm(lambda: nv.gemm_w4a16(x, W, out=y))
        ref = arm(lambda: torch.matmul(x, w.t()))
        tf = lambda ms: round(2 * L.M * L.N * L.K / (ms * 1e-3) / 1e12, 1)
        out[L.name] = {"shape": f"{L.M}x{L.K}x{L.N}", "ms": round(ours[0], 4), "tflops": tf(ours[0]),
                       "tflops_sustained": tf(ours[1]), "cublas_bf16_tflops": tf(ref[0]),
                       "cublas_bf16_tflops_sustained": tf(ref[1])}
        del x, w, W, y
    return out


def qat_points(dev, layers):
    """Quantization-aware training kernels on the fc1 / fc2 inputs (the
    fake-quantized forward with its clip mask, dynamic and given tensor
    scale, and the masked straight-through backward); HBM-bound, algorithmic
    bytes per element as the QAT_* constants state."""
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    hbm = load_peaks()[0].get("hbm_gbs", FALLBACK["hbm_gbs"])
    res_all = {}
    for name in ("fc1", "fc2"):
        if name not in [L.name for L in layers]:
            continue
        x, = synth.layer_tensors(WORKLOAD, name, device=dev, want=("x",))
        x = x[: [L.M for L in layers if L.name == name][0]].contiguous()
        rows, k = x.shape
        y = torch.empty_like(x)
        m = torch.empty(rows, k // 8, dtype=torch.uint8, device=dev)
        g = torch.zeros(1, dtype=torch.float32, device=dev)
        wsb = nv.nvfp4_quantize_workspace_bytes(rows, k)
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
        gx = torch.empty_like(x)
        runs = {
            "fake_quantize_dynamic": (lambda: nv.nvfp4_fake_quantize(x, rows, k, k, y, 0, m, g, 0, ws, wsb),
                                      QAT_FWD_DYNAMIC_BYTES),
            "fake_quantize_given": (lambda: nv.nvfp4_fake_quantize(x, rows, k, k, y, 0, m, g, 1, None, 0),
                                    QAT_FWD_GIVEN_BYTES),
            "ste_backward": (lambda: nv.nvfp4_ste_backward(x, m, rows, k, 0, gx), QAT_BWD_BYTES),
        }
        res = {"shape": f"{rows}x{k}"}
        full = name == "fc2" and rows == 32768
        traffic_keys = {"fake_quantize_dynamic": "dram_bytes_per_launch_dynamic",
                        "fake_quantize_given": "dram_bytes_per_launch_given",
                        "ste_backward": "dram_bytes_per_launch_ste"}
        for key, (fn, bpe) in runs.items():
            ms = time_device(fn)
            gbs = bpe * rows * k / (ms * 1e-3) / 1e9
            res[key] = {"ms": round(ms, 4), "gbs": round(gbs, 1), "frac": round(gbs / hbm, 4), "bytes_per_elem": bpe,
                        "traffic": profiled_traffic("fake_quantize_ste_fc2_32768x12288.txt", traffic_keys[key])
                        if full else None}
        res_all[name] = res
        del x, y, m, gx, ws
    torch.cuda.empty_cache()
    return res_all


def mlp_fusion_points(dev, layers):
    """The MLP's first layer with GELU and the second layer's NVFP4 input
    produced in the GEMM epilogue (one kernel), against the same result made
    in three steps: the GEMM writing bf16, GELU (torch, a reference point
    only), and the dynamic-scale quantize of the activation."""
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    L = [l for l in layers if l.name == "fc1"]
    if not L:
        return None
    L = L[0]
    x, w = synth.layer_tensors(WORKLOAD, "fc1", device=dev)
    A, W = nv.quantize(x[: L.M].contiguous()), nv.quantize(w)
    del x, w
    y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device=dev)
    q = nv.NVFP4Tensor.empty(L.M, L.N, dev)
    amax = torch.zeros(1, dtype=torch.float32, device=dev)
    ws = torch.empty(nv.nvfp4_quantize_workspace_bytes(L.M, L.N), dtype=torch.uint8, device=dev)
    nv.gemm_w4a4(A, W, out=y, act=nv.NVFP4_ACT_GELU_TANH)
    q.scale.copy_(torch.max(torch.abs(y.float())).reshape(1) / 2688.0)
    gy = q.scale.clone()
    fused = time_device(lambda: nv.gemm_w4a4_nvfp4_out(A, W, gy, y_amax=amax, out=q, act=nv.NVFP4_ACT_GELU_TANH))
    g_ms = time_device(lambda: nv.gemm_w4a4(A, W, out=y))
    a_ms = time_device(lambda: torch.nn.functional.gelu(y, approximate="tanh"))
    h = torch.nn.functional.gelu(y, approximate="tanh")
    q_ms = time_device(lambda: nv.quantize(h, out=q, workspace=ws))
    del y, h, q, A, W
    torch.cuda.empty_cache()
    fl = 2 * L.M * L.N * L.K
    return {"shape": f"{L.M}x{L.K}x{L.N}", "fused_ms": round(fused, 4),
            "fused_tflops": round(fl / (fused * 1e-3) / 1e12, 1),
            "three_step_ms": round(g_ms + a_ms + q_ms, 4),
            "three_step_parts_ms": {"gemm_bf16": round(g_ms, 4), "gelu_torch": round(a_ms, 4),
                                    "quantize": round(q_ms, 4)}}


def layernorm_points(dev):
    """The block input's LayerNorm (adaLN: a per-sample affine) emitted as the
    QKV projection's NVFP4 input in one kernel, data-derived tensor scale,
    against LayerNorm + modulation in torch (bf16, a reference point only)
    followed by the dynamic-scale quantize.  Video block input (32768 x 3072,
    16 samples of 2048 tokens) and PixArt-1024's (8192 x 1152, 2 samples)."""
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    out = {}
    hbm = load_peaks()[0].get("hbm_gbs", FALLBACK["hbm_gbs"])
    for name, (M, K, groups, dist, seed) in {"video_dit": (32768, 3072, 16, "token_scaled", 31),
                                             "pixart1024": (8192, 1152, 2, "student_t3", 32)}.items():
        x = synth.random_bf16((M, K), seed=seed, dist=dist, device=dev)
        gen = torch.Generator(device=dev).manual_seed(seed)
        scale = 0.1 * torch.randn(groups, K, generator=gen, device=dev)
        shift = 0.1 * torch.randn(groups, K, generator=gen, device=dev)
        gamma, beta = (1.0 + scale).contiguous(), shift.contiguous()
        q = nv.NVFP4Tensor.empty(M, K, dev)
        ws = torch.empty(nv.nvfp4_quantize_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
        rpg = M // groups
        fused = time_device(lambda: nv.layernorm_quantize(x, gamma, beta, rpg, 1e-6, out=q, workspace=ws))
        g16 = gamma.to(torch.bfloat16).repeat_interleave(rpg, dim=0)
        b16 = beta.to(torch.bfloat16).repeat_interleave(rpg, dim=0)

        def ln_torch():
            return torch.nn.functional.layer_norm(x, (K,), eps=1e-6) * g16 + b16
        h = ln_torch()
        ln_ms = time_device(ln_torch)
        q_ms = time_device(lambda: nv.quantize(h, out=q, workspace=ws))
        gbs = QUANT_BYTES_PER_ELEM * M * K / (fused * 1e-3) / 1e9
        out[name] = {"shape": f"{M}x{K}", "samples": groups, "fused_ms": round(fused, 4),
                     "fused_gbs": round(gbs, 1), "fused_frac_hbm": round(gbs / hbm, 4),
                     "bytes_per_elem": QUANT_BYTES_PER_ELEM,
                     "two_step_ms": round(ln_ms + q_ms, 4),
                     "two_step_parts_ms": {"layernorm_modulate_torch_bf16": round(ln_ms, 4), "quantize": round(q_ms, 4)}}
        del x, h, q, g16, b16
        torch.cuda.empty_cache()
    return out


def time_flushed(fn, flush, iters=20, warmup=3):
    """Median device time of fn with L2 flushed before every run (a write of a
    buffer larger than L2), for operands that would otherwise stay in L2."""
    import torch
    for _ in range(warmup):
        fn()
    ts = []
    for _ in range(iters):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def small_layer_points(dev):
    """Every DiT-XL/2 (M = 2048) and PixArt-1024 (M = 8192, cross-attention
    M = 600) layer: the W4A4 GEMM (bf16 out) on each kernel the shape allows
    (the library's choice, the single-CTA kernel, CTA pairs with 192- and
    256-wide tiles), the dynamic-scale quantize of its input, and cuBLAS bf16
    (a reference point), L2 flushed before every run.  Roofline per layer:
    t = max(FLOPs / FP4 peak, (codes + scales of A and B + bf16 Y) / HBM peak)
    with the measured peaks; frac = t / measured."""
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    peaks, _ = load_peaks()
    fp4 = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"]) * FP4_OVER_BF16 * 1e12
    hbm = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"]) * 1e9
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    kernels = {"auto": {}, "single": {"NVFP4_GEMM_KERNEL": "single"},
               "pair192": {"NVFP4_GEMM_KERNEL": "pair", "NVFP4_PAIR_TILE_N": "192"},
               "pair256": {"NVFP4_GEMM_KERNEL": "pair", "NVFP4_PAIR_TILE_N": "256"}}
    out = {}
    for wl in ("dit_xl2", "pixart1024"):
        for L in synth.WORKLOADS[wl].layers:
            x, w = synth.layer_tensors(wl, L.name, device=dev)
            A, B = nv.quantize(x), nv.quantize(w)
            y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device=dev)
            fl = 2 * L.M * L.N * L.K
            byts = (L.M + L.N) * L.K * (0.5 + 1 / 16) + 2 * L.M * L.N
            t_roof = max(fl / fp4, byts / hbm) * 1e3
            r = {"shape": f"{L.M}x{L.K}x{L.N}", "roofline_ms": round(t_roof, 5),
                 "bound": "tensor" if fl / fp4 > byts / hbm else "hbm"}
            for name, env in kernels.items():
                if name == "pair192" and L.N % 192 or name == "pair256" and L.N % 256:
                    continue
                saved = {k: os.environ.get(k) for k in env}
                os.environ.update(env)
                try:
                    ms = time_flushed(lambda: nv.gemm_w4a4(A, B, out=y), flush)
                finally:
                    for k, v in saved.items():
                        if v is None:
                            os.environ.pop(k, None)
                        else:
                            os.environ[k] = v
                r[name] = {"ms": round(ms, 5), "tflops": round(fl / (ms * 1e-3) / 1e12, 1),
                           "frac": round(t_roof / ms, 3)}
            q = nv.NVFP4Tensor.empty(L.M, L.K, dev)
            ws = torch.empty(nv.nvfp4_quantize_workspace_bytes(L.M, L.K), dtype=torch.uint8, device=dev)
            qms = time_flushed(lambda: nv.quantize(x, out=q, workspace=ws), flush)
            r["quantize_ms"] = round(qms, 5)
            r["quantize_frac_hbm"] = round(QUANT_BYTES_PER_ELEM * L.M * L.K / hbm * 1e3 / qms, 3)
            bms = time_flushed(lambda: torch.matmul(x, w.t()), flush)
            r["cublas_bf16_ms"] = round(bms, 5)
            out[f"{wl}.{L.name}"] = r
            del x, w, A, B, y, q
    del flush
    torch.cuda.empty_cache()
    return out


def grouped_points(dev):
    """One PixArt-1024 block's independent projections as one grouped launch
    vs separate launches: the image-token QKV with the text-token
    cross-attention K and V, and the same with the MLP's fc1 added (every N a
    multiple of 192, so the group runs on the CTA-pair kernel), L2 flushed
    before every run."""
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ops = {}
    for name in ("qkv", "xattn_k", "xattn_v", "fc1"):
        x, w = synth.layer_tensors("pixart1024", name, device=dev)
        A, B = nv.quantize(x), nv.quantize(w)
        ops[name] = (A, B, torch.empty(A.rows, B.rows, dtype=torch.bfloat16, device=dev),
                     2 * x.shape[0] * x.shape[1] * w.shape[0])
        del x, w
    out = {}
    for label, names in (("qkv_xattn", ("qkv", "xattn_k", "xattn_v")),
                         ("qkv_xattn_fc1", ("qkv", "xattn_k", "xattn_v", "fc1"))):
        sel = [ops[n] for n in names]
        probs = [dict(a_codes=A.codes, a_sf=A.sf, a_scale=A.scale, b_codes=B.codes, b_sf=B.sf, b_scale=B.scale,
                      M=A.rows, N=B.rows, K=A.k, y=y) for A, B, y, _ in sel]
        fl = sum(f for *_, f in sel)

        def separate():
            for A, B, y, _ in sel:
                nv.gemm_w4a4(A, B, out=y)

        sep = time_flushed(separate, flush)
        grp = time_flushed(lambda: nv.nvfp4_gemm_w4a4_grouped(probs), flush)
        out[label] = {"problems": ", ".join(f"{n} {ops[n][0].rows}x{ops[n][0].k}x{ops[n][1].rows}" for n in names),
                      "separate_us": round(sep * 1e3, 1), "grouped_us": round(grp * 1e3, 1),
                      "grouped_tflops": round(fl / (grp * 1e-3) / 1e12, 1)}
    del flush, ops
    torch.cuda.empty_cache()
    return out


def mx_points(dev, layers):
    """The MX variant (block 32, E8M0 scales) on the fc2 input and the fc1 /
    fc2 products, next to NVFP4; and the Eq. 9 block-size measurement on the
    fc2 input (the relative squared error of every candidate block size)."""
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    hbm = load_peaks()[0].get("hbm_gbs", FALLBACK["hbm_gbs"])
    res = {}
    names = [L.name for L in layers]
    if "fc2" in names:
        L = layers[names.index("fc2")]
        x, = synth.layer_tensors(WORKLOAD, "fc2", device=dev, want=("x",))
        x = x[: L.M].contiguous()
        n = x.numel()
        mq = nv.MXTensor.empty(*x.shape, dev)
        ms = time_device(lambda: nv.mx_quantize(x, out=mq))
        gbs = MX_QUANT_BYTES_PER_ELEM * n / (ms * 1e-3) / 1e9
        res["mx_quantize_fc2"] = {"ms": round(ms, 4), "gbs": round(gbs, 1), "frac": round(gbs / hbm, 4),
                                  "bytes_per_elem": MX_QUANT_BYTES_PER_ELEM}
        g = nv.quantize(x).scale
        e = torch.empty(8, dtype=torch.float64, device=dev)
        ms = time_device(lambda: nv.nvfp4_block_size_errors(x, x.shape[0], x.shape[1], x.shape[1], g, e), iters=3,
                         warmup=1)
        rel = (e[:7] / e[7]).cpu().tolist()
        res["block_size_errors_fc2"] = {"ms": round(ms, 3),
                                        "relative_sq_error": {str(b): round(v, 6) for b, v in zip((1, 2, 4, 8, 16, 32, 64), rel)},
                                        "selected": {str(lam): nv.nvfp4_select_block_size(e.cpu().tolist(), lam)
                                                     for lam in (0.001, 0.01, 0.1)}}
        del x, mq, e
    for name in ("fc1", "fc2"):
        if name not in names:
            continue
        L = layers[names.index(name)]
        x, w = synth.layer_tensors(WORKLOAD, name, device=dev)
        x = x[: L.M].contiguous()
        A, W = nv.mx_quantize(x), nv.mx_quantize(w)
        y = torch.empty(L.M, L.N, dtype=torch.bfloat16, device=dev)
        ms = time_device(lambda: nv.mx_gemm(A, W, out=y))
        res[f"mx_gemm_{name}"] = {"shape": f"{L.M}x{L.K}x{L.N}", "ms": round(ms, 4),
                                  "tflops": round(2 * L.M * L.N * L.K / (ms * 1e-3) / 1e12, 1)}
        del x, w, A, W, y
    torch.cuda.empty_cache()
    return res


def attention_points(dev, heads=384):
    """Attention over NVFP4 Q, K, V (Eq. 10) at the video DiT's spatial
    attention: 16 frames x 24 heads (d = 128) of 2048 tokens each, i.e. 384
    independent heads; torch's bf16 scaled-dot-product attention on bf16
    tensors of the same shape as a library reference point.  Both arms are
    timed after a 1 s idle, as a burst and then sustained (time_arm)."""
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import synth
    H, L, D = heads, 2048, 128
    xs = [synth.random_bf16((H * L, D), seed=90 + i, dist="normal", device=dev) for i in range(3)]
    Q, K, V = (nv.quantize(x) for x in xs)
    o = torch.empty(H * L, D, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(nv.nvfp4_attention_workspace_bytes(H, L, D), dtype=torch.uint8, device=dev)
    ms, ms_s = time_arm(lambda: nv.attention(Q, K, V, H, out=o, workspace=ws))
    q4, k4, v4 = (x.view(1, H, L, D) for x in xs)
    ms_ref, ms_ref_s = time_arm(lambda: torch.nn.functional.scaled_dot_product_attention(q4, k4, v4))
    fl = 4 * H * L * L * D
    del xs, Q, K, V, o, ws, q4, k4, v4
    torch.cuda.empty_cache()
    return {"shape": f"{H} heads x {L} tokens x d {D}", "ms": round(ms, 4), "tflops": round(fl / (ms * 1e-3) / 1e12, 1),
            "ms_sustained": round(ms_s, 4), "torch_sdpa_bf16_ms": round(ms_ref, 4),
            "torch_sdpa_bf16_tflops": round(fl / (ms_ref * 1e-3) / 1e12, 1),
            "torch_sdpa_bf16_ms_sustained": round(ms_ref_s, 4)}


def reduced(wl, args):
    """A reduced case for profiling captures: selected layers and/or fewer
    tokens (rows of X) per layer."""
    if not (args.layers or args.m):
        return wl
    import dataclasses
    keep = [L for L in wl.layers if not args.layers or L.name in args.layers.split(",")]
    keep = [dataclasses.replace(L, M=min(args.m, L.M) if args.m else L.M) for L in keep]
    return dataclasses.replace(wl, layers=tuple(keep))


def kernel_source_hash(files=None) -> str:
    """SHA-256 over CUDA sources of the library (names and contents): the
    given file names under csrc/, or all of them.  A DRAM traffic figure
    recorded under profiles/ is reported only while this matches the hash
    recorded beside it: a change to any of those sources voids it."""
    import hashlib
    d = os.path.join(ROOT, "nvfp4_w4a4_gemm_quantize_b200", "csrc")
    names = sorted(files) if files else sorted(n for n in os.listdir(d) if n.endswith((".cu", ".cuh", ".h")))
    h = hashlib.sha256()
    for name in names:
        h.update(name.encode())
        h.update(open(os.path.join(d, name), "rb").read())
    return h.hexdigest()


def profiled_traffic(summary: str, key: str = "dram_bytes_per_launch"):
    """DRAM bytes per launch (read + write) from an ncu summary under
    profiles/ (the line `key: <bytes>`), or None when it is absent or was
    taken on other sources (the summary lists its `source_files` and their
    `source_sha256`)."""
    p = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(p):
        return None
    kv = {}
    for line in open(p):
        if ":" in line:
            k, v = line.split(":", 1)
            kv.setdefault(k.strip(), v.strip())
    files = kv.get("source_files", "").split() or None
    try:
        if kv.get("source_sha256") != kernel_source_hash(files):
            return None
        return int(kv[key])
    except (KeyError, ValueError, OSError):
        return None


# ----------------------------------------------------------------- our leg
def run_ours(args):
    import torch
    import nvfp4_w4a4_gemm_quantize_b200 as nv
    from nvfp4_w4a4_gemm_quantize_b200 import build, synth

    rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        build.build()
    barrier(world)
    wl = reduced(synth.WORKLOADS[WORKLOAD], args)
    wl16 = reduced(synth.WORKLOADS["w4a16"], args)
    peaks, peak_src = load_peaks()
    if args.qat or args.only:
        # profiling aid: one group of reference points alone
        groups = {"qat": lambda: qat_points(dev, wl.layers), "mlp": lambda: mlp_fusion_points(dev, wl.layers),
                  "layernorm": lambda: layernorm_points(dev), "small": lambda: small_layer_points(dev),
                  "grouped": lambda: grouped_points(dev), "mx": lambda: mx_points(dev, wl.layers),
                  "attention": lambda: attention_points(dev, args.heads or 384),
                  "w4a16": lambda: w4a16_points(dev, wl16.layers)}
        name = "qat" if args.qat else args.only
        if name not in groups:
            raise SystemExit(f"--only: one of {sorted(groups)}")
        res = groups[name]()
        if rank == 0:
            print(json.dumps({name: res, "peak_gbs": peaks.get("hbm_gbs", FALLBACK["hbm_gbs"]),
                              "peak_source": peak_src}))
        return 0

    # ---- data (resident in HBM before timing); each rank its own batch
    xs, Ws, Aq, Ys = [], [], [], []
    for L in wl.layers:
        x, w = synth.layer_tensors(WORKLOAD, L.name, device=dev)
        x = x[: L.M].contiguous()
        if rank:
            x = x.roll(rank * 977, dims=0)
        xs.append(x)
        Ws.append(nv.quantize(w))                        # static weights, quantized once
        del w
        Aq.append(nv.NVFP4Tensor.empty(L.M, L.K, dev))
        Ys.append(torch.empty(L.M, L.N, dtype=torch.bfloat16, device=dev))
    ws = torch.empty(nv.nvfp4_quantize_workspace_bytes(1, 64), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    gemm_flops = sum(2 * L.M * L.N * L.K for L in wl.layers)
    q_elems = sum(L.M * L.K for L in wl.layers)

    ev = lambda: torch.cuda.Event(enable_timing=True)
    gemm_ev = [[(ev(), ev()) for _ in wl.layers] for _ in range(args.steps)]
    quant_ev = [[(ev(), ev()) for _ in wl.layers] for _ in range(args.steps)]

    def step(i=None):
        for li, L in enumerate(wl.layers):
            if i is not None:
                quant_ev[i][li][0].record(stream)
            nv.quantize(xs[li], out=Aq[li], workspace=ws)
            if i is not None:
                quant_ev[i][li][1].record(stream)
                gemm_ev[i][li][0].record(stream)
            nv.gemm_w4a4(Aq[li], Ws[li], out=Ys[li])
            if i is not None:
                gemm_ev[i][li][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    launches0 = nv.nvfp4_launch_count()
    t0, t1 = ev(), ev()
    sampler.mark_start()
    t0.record(stream)
    for i in range(args.steps):
        step(i)
    t1.record(stream)
    torch.cuda.synchronize()
    sampler.mark_end()
    launches = nv.nvfp4_launch_count() - launches0
    barrier(world)
    clocks = sampler.stop()
    dev_ms = t0.elapsed_time(t1)
    max_ms = max_over_ranks(dev_ms, world, dev)

    gemm_all = [[gemm_ev[i][li][0].elapsed_time(gemm_ev[i][li][1]) for i in range(args.steps)]
                for li in range(len(wl.layers))]
    quant_all = [[quant_ev[i][li][0].elapsed_time(quant_ev[i][li][1]) for i in range(args.steps)]
                 for li in range(len(wl.layers))]
    gemm_ms = [sum(v) / len(v) for v in gemm_all]
    quant_ms = [sum(v) / len(v) for v in quant_all]

    def pct(v):
        """p10 / median / p90 of per-step times (ms)."""
        q = sorted(v)
        at = lambda f: q[min(len(q) - 1, int(round(f * (len(q) - 1))))]
        return [round(at(0.1), 4), round(at(0.5), 4), round(at(0.9), 4)]

    # ---- end to end through the public API with host buffers
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for y in Ys]
    h2d = sum(x.numel() * x.element_size() for x in xh)
    d2h = sum(y.numel() * y.element_size() for y in yh)

    # copies in and out run on their own streams (PCIe is full duplex), layer
    # by layer, so the inputs of the next layer and the outputs of the last one
    # move while a layer computes; events keep each buffer's reuse in order
    nl = len(wl.layers)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nl)]      # X landed on the device
    ev_used = [torch.cuda.Event() for _ in range(nl)]    # X read by the quantize kernel
    ev_done = [torch.cuda.Event() for _ in range(nl)]    # Y computed
    ev_out = [torch.cuda.Event() for _ in range(nl)]     # Y copied to the host

    def e2e_step():
        for li in range(nl):
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_used[li])
                xs[li].copy_(xh[li], non_blocking=True)
                ev_in[li].record(s_in)
            stream.wait_event(ev_in[li])
            nv.quantize(xs[li], out=Aq[li], workspace=ws)
            ev_used[li].record(stream)
            stream.wait_event(ev_out[li])
            nv.gemm_w4a4(Aq[li], Ws[li], out=Ys[li])
            ev_done[li].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[li])
                yh[li].copy_(Ys[li], non_blocking=True)
                ev_out[li].record(s_out)

    e2e_steps = max(1, min(args.steps, 5))
    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = ev(), ev()
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for _ in range(e2e_steps):
        e2e_step()
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps

    extra = None
    if rank == 0 and world == 1 and not args.no_reference_points:
        del xh, yh
        extra = reference_points(dev, wl.layers, wl16.layers)

    # ---- cpu baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_leg(args)

    if rank == 0:
        # the GEMM is timed inside a long step (back-to-back steps under the
        # power cap) once the timed region lasts half a second or more: then
        # the sustained bf16 figure is its denominator, else the burst one
        sustained = max_ms >= 500.0
        bf16_key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
        fp4_peak = peaks.get(bf16_key, FALLBACK[bf16_key]) * FP4_OVER_BF16
        hbm_peak = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
        # dominant kernel: the GEMM of the largest layer (fc1, the 32768x3072x12288 shape)
        names = [L.name for L in wl.layers]
        li = names.index("fc1") if "fc1" in names else 0
        L = wl.layers[li]
        g_flops = 2 * L.M * L.N * L.K
        g_tflops = g_flops / (gemm_ms[li] * 1e-3) / 1e12
        q_gbs = [QUANT_BYTES_PER_ELEM * l.M * l.K / (quant_ms[j] * 1e-3) / 1e9 for j, l in enumerate(wl.layers)]
        # quantize: the largest activation (fc2's input, 32768 x 12288)
        qi = names.index("fc2") if "fc2" in names else 0
        full = not (args.layers or args.m)
        g_traffic = profiled_traffic("gemm_w4a4_fc1_32768x3072x12288.txt") if full else None
        q_traffic = profiled_traffic("quantize_fc2_32768x12288.txt") if full else None
        per_layer = {l.name: {"gemm_ms": round(gemm_ms[j], 4),
                              "gemm_tflops": round(2 * l.M * l.N * l.K / (gemm_ms[j] * 1e-3) / 1e12, 1),
                              "gemm_ms_p10_p50_p90": pct(gemm_all[j]),
                              "quant_ms": round(quant_ms[j], 4), "quant_gbs": round(q_gbs[j], 1),
                              "quant_ms_p10_p50_p90": pct(quant_all[j])}
                     for j, l in enumerate(wl.layers)}
        value = world * args.steps * gemm_flops / (max_ms * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
            "data": "synthetic",
            "config": step_config(world),
            "roofline": {"bound": "tensor", "kernel": f"gemm_w4a4 {L.name} {L.M}x{L.K}x{L.N}",
                         "achieved": round(g_tflops, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                         "frac": round(g_tflops / fp4_peak, 4),
                         "peak_source": f"{peak_src} bf16 {'sustained' if sustained else 'burst'} x "
                                        f"{FP4_OVER_BF16:g} (nominal FP4/bf16 ratio; timed region "
                                        f"{max_ms / 1e3:.2f} s)",
                         "traffic": g_traffic},
            "quantize": {"bound": "hbm", "kernel": f"amax + quantize {wl.layers[qi].name} input "
                                                   f"{wl.layers[qi].M}x{wl.layers[qi].K}",
                         "achieved": round(q_gbs[qi], 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(q_gbs[qi] / hbm_peak, 4), "bytes_per_elem": QUANT_BYTES_PER_ELEM,
                         "peak_source": peak_src, "traffic": q_traffic},
            "layers": per_layer,
            "e2e": {"value": round(world * gemm_flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches),
            "clocks": clocks,
            "cpu_baseline": cpu,
            "reference_points": extra,
        }
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=16, help="oracle rows per host core and layer")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-reference-points", action="store_true")
    ap.add_argument("--layers", default="", help="profiling: comma-separated subset of layers")
    ap.add_argument("--m", type=int, default=0, help="profiling: tokens (rows of X) per layer")
    ap.add_argument("--qat", action="store_true", help="profiling: time only the QAT kernels (fc1 / fc2 inputs)")
    ap.add_argument("--heads", type=int, default=0, help="profiling: attention heads (default 384)")
    ap.add_argument("--only", default="", help="profiling: time one group of reference points "
                                               "(qat, mlp, layernorm, small, grouped, mx, attention, w4a16)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
