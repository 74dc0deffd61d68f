"""Benchmark of the NVFP4 W4A4 linear-layer hot path on B200.

One step = one forward of the FLUX double-stream MLP-up layer
(M=4608 tokens, K=3072, N=12288, bf16 bias): runtime NVFP4 quantization of
the bf16 activations with the calibrated input scale, then the block-scaled
NVFP4 GEMM with the fused alpha*acc + bias -> bf16 epilogue.  Inputs are
seeded synthetic tensors of that shape (weights quantized once, untimed).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` is whole-job TFLOP/s (2*M*N*K per
step per GPU) with inputs resident in HBM; L2 is flushed between timed steps
(256 MiB written then read back, so L2 holds clean unrelated lines) and every
step is bracketed by CUDA events on the launching stream.  Under
torchrun each rank runs its own token batch (weak scaling, no data
collective); the step time is the max over ranks.
``--impl reference`` times the CPU oracle on a bounded row sample instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 GEMM TFLOP/s and % dense-FP4 peak; quantize GB/s and % HBM peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP4_PER_BF16 = 4.0  # nominal dense ratio: 9 PFLOP/s FP4 vs 2.25 PFLOP/s bf16
QUANT_BYTES_PER_ELEM = 2.0 + 0.5 + 1.0 / 16.0
MX_QUANT_BYTES_PER_ELEM = 2.0 + 1.0 + 1.0 / 32.0  # bf16 in, E4M3 code + E8M0 scale out
FP8_PER_BF16 = 2.0


PROFILES = os.path.join(ROOT, "profiles")
GEMM_PROFILE = os.path.join(PROFILES, "gemm_nvf4_flux_mlp_up_m4608_k3072_n12288.txt")
GEMM_SOURCES = ("gemm.cu", "device.cuh", "internal.h")


def gemm_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        with open(os.path.join(ROOT, "nvfp4_block_scaled_12_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gemm_dram_traffic():
    """DRAM bytes per launch of the GEMM kernel from the committed ncu
    summary, or None when the kernel's sources changed since the capture."""
    try:
        fields = {}
        with open(GEMM_PROFILE) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("sources_sha256") != gemm_sources_sha256():
            return None
        return int(fields["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


QUANT_PROFILE = os.path.join(PROFILES, "quantize_laplace_m4608_k12288.txt")
QUANT_SOURCES = ("quantize.cu", "device.cuh", "internal.h")


def quantize_dram_traffic():
    """DRAM bytes per launch of the standalone quantize from the committed
    ncu summary, or None when the kernel's sources changed since."""
    try:
        import hashlib
        fields = {}
        with open(QUANT_PROFILE) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip()
        h = hashlib.sha256()
        for name in QUANT_SOURCES:
            with open(os.path.join(ROOT, "nvfp4_block_scaled_12_b200", "csrc", name), "rb") as f:
                h.update(f.read())
        if fields.get("sources_sha256") != h.hexdigest():
            return None
        return int(fields["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=5)

    def summary(self, t0=None, t1=None):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 8:
                continue
            try:
                rows.append((ts, float(parts[0]), float(parts[1]), parts))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}
        inside = [r for r in rows if t0 is None or (t0 <= r[0] <= t1)] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, _, _, parts in inside:
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside)}


# ---------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_activation_seed(rank: int, base_seed: int) -> int:
    """Each rank draws its own token batch (weak scaling, no data exchange)."""
    return base_seed + 100 * rank


def max_over_ranks(value: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- CPU oracle
ORACLE_COLS = 1024  # weight rows (output columns) in the oracle's sample block


def oracle_sample(rows: int, step: int = 0):
    """Time the oracle on a block of the MLP-up layer: `rows` activation rows
    (a different slice each step) x ORACLE_COLS output columns.  Timed: the
    runtime activation quantize of those rows and the fp64
    dequantize-then-matmul + bias.  The weight block is quantized once,
    untimed (weight preparation is offline).  Returns (seconds, flops)."""
    import oracle as O
    import synth
    wl = synth.MLP_UP
    x = synth_cache("x", lambda: wl.activations().float().numpy())
    gx = synth_cache("gx", lambda: O.global_scale(O.tensor_amax(x)))
    wq = synth_cache("wq", lambda: _oracle_weight(O, wl))
    bias = synth_cache("bias", lambda: wl.bias_vec().float().numpy()[:ORACLE_COLS])
    r0 = (step * rows) % (wl.m - rows + 1)
    t0 = time.perf_counter()
    xc, xs = O.quantize_nvfp4(x[r0:r0 + rows], gx)
    O.gemm_ref(xc, xs, gx, wq[0], wq[1], wq[2], bias)
    dt = time.perf_counter() - t0
    return dt, 2.0 * rows * ORACLE_COLS * wl.k


_CACHE = {}


def synth_cache(key, fn):
    if key not in _CACHE:
        _CACHE[key] = fn()
    return _CACHE[key]


def _oracle_weight(O, wl):
    w = wl.weight().float().numpy()
    gw = O.global_scale(O.tensor_amax(w))  # per-tensor scale over the whole weight
    wc, ws = O.quantize_nvfp4(w[:ORACLE_COLS], gw)
    return wc, ws, gw


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [int(i.get("num_threads", 0)) for i in threadpool_info()]
        return max(n) if n else os.cpu_count() or 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def cpu_baseline(budget_s: float = 10.0, rows: int = 256):
    """The oracle as it stands, on a bounded sample of the workload."""
    oracle_sample(8)  # build the cached inputs (untimed)
    total_t, total_f, n = 0.0, 0.0, 0
    while total_t < budget_s and n < 400:
        dt, fl = oracle_sample(rows, n)
        total_t += dt
        total_f += fl
        n += 1
    return {"value": total_f / total_t / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} blocks of {rows} activation rows x {ORACLE_COLS} output columns of "
                      f"M=4608,K=3072,N=12288 (quantize + fp64 GEMM + bias), {total_t:.1f} s"}


def quantize_cpu_baseline(budget_s: float = 8.0):
    """The oracle's quantizer as it stands (numpy, elementwise: one core) on
    the whole standalone-quantize workload bf16 [4608, 12288], swizzled scales
    included, repeated until about ``budget_s`` seconds; GB/s on the same
    2.5625 bytes per element as the GPU figure."""
    import oracle as O
    import synth
    x = synth_cache("xq", lambda: synth.quantize_input().float().numpy())
    g = O.global_scale(O.tensor_amax(x))
    total, n = 0.0, 0
    while total < budget_s and n < 8:
        t0 = time.perf_counter()
        _, sf = O.quantize_nvfp4(x, g)
        O.swizzle_sf(sf)
        total += time.perf_counter() - t0
        n += 1
    gbs = n * x.size * QUANT_BYTES_PER_ELEM / total / 1e9
    return {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} full passes over bf16 [4608,12288] (codes + swizzled scales), {total:.1f} s; "
                      "numpy elementwise, one core"}


def single_stream_g_next() -> float:
    """The output projection's calibrated input scale of the single-stream
    pair, stored by tests/golden/make_golden.py (computed by the oracle)."""
    with open(os.path.join(ROOT, "tests", "golden", "single_stream_pair.json")) as f:
        return float(json.load(f)["g_next"])


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    rows = 128
    oracle_sample(8)  # build the cached inputs (untimed)
    for i in range(args.warmup):
        oracle_sample(rows, i)
    times, flops = [], 0.0
    for i in range(args.steps):
        dt, fl = oracle_sample(rows, args.warmup + i)
        times.append(dt)
        flops += fl
    tot = sum(times)
    val = flops / tot / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "flux_mlp_up_m4608_k3072_n12288", "m": 4608, "k": 3072, "n": 12288,
                   "step_sample_rows": rows, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{rows} activation rows x {ORACLE_COLS} output columns per step of "
                                   "M=4608,K=3072,N=12288"},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm
def extra_workloads(F, torch, synth, device, stream, median_ms, hbm, fp4_peak):
    """The other measured configurations, one GPU: the FLUX single-stream
    block pair (fused quantize epilogue vs a bf16 round trip) and the
    attention-projection token sweep.  Timed like the rest (median, L2
    flushed before every repetition)."""
    out = {}
    # --- single-stream pair: GEMM1 [4608,3072] x [21504,3072]^T whose epilogue
    # writes Q and GELU(MLP) as NVFP4 (GEMM2's input) and K,V as bf16, then
    # GEMM2 [4608,15360] x [3072,15360]^T
    w1l, w2l = synth.SINGLE_IN, synth.SINGLE_OUT
    M = w1l.m
    q0, q1 = synth.SINGLE_Q
    kv0, kv1 = synth.SINGLE_KV
    m0, m1 = synth.SINGLE_MLP
    x = w1l.activations().to(device)
    xq = F.quantize(x, F.global_scale(x))
    w1 = w1l.weight().to(device)
    w1q = F.quantize(w1, F.global_scale(w1))
    w2 = w2l.weight().to(device)
    w2q = F.quantize(w2, F.global_scale(w2))
    del w1, w2
    k2 = w2l.k
    g2 = single_stream_g_next()  # the output projection's calibrated input scale
    b2 = w2l.bias_vec().to(device)
    a2 = F.NVFP4Tensor(torch.empty(M, k2 // 2, dtype=torch.uint8, device=device),
                       torch.empty(F.nvfp4_sf_bytes(M, k2), dtype=torch.uint8, device=device), g2, M, k2)
    y_kv = torch.empty(M, kv1 - kv0, dtype=torch.bfloat16, device=device)
    y2 = torch.empty(M, w2l.n, dtype=torch.bfloat16, device=device)
    fused_ranges = [(q0, q1, F.ACT_NONE, F.DST_NVFP4, 0), (kv0, kv1, F.ACT_NONE, F.DST_BF16, 0),
                    (m0, m1, F.ACT_GELU_TANH, F.DST_NVFP4, q1 - q0)]
    y_qm = torch.empty(M, k2, dtype=torch.bfloat16, device=device)  # unfused: [Q | GELU(MLP)] in bf16
    y_all = torch.empty(M, k2 + (kv1 - kv0), dtype=torch.bfloat16, device=device)
    bf16_ranges = [(q0, q1, F.ACT_NONE, F.DST_BF16, 0), (m0, m1, F.ACT_GELU_TANH, F.DST_BF16, q1 - q0),
                   (kv0, kv1, F.ACT_NONE, F.DST_BF16, k2)]

    def gemm1_fused():
        F.gemm_quant(xq, w1q, fused_ranges, y_bf16=y_kv, g_next=g2, next_out=a2, stream=stream)

    def gemm1_bf16():
        F.gemm_quant(xq, w1q, bf16_ranges, y_bf16=y_all, stream=stream)

    def gemm2():
        F.gemm(a2, w2q, bias=b2, y=y2, stream=stream)

    def unfused():
        gemm1_bf16()
        y_qm.copy_(y_all[:, :k2])  # the quantizer reads rows of K contiguous elements
        F.quantize(y_qm, g2, out=a2, stream=stream)
        gemm2()

    f1, f2 = 2 * M * w1l.n * w1l.k, 2 * M * w2l.n * w2l.k
    t1f = median_ms(gemm1_fused)
    t1b = median_ms(gemm1_bf16)
    t2 = median_ms(gemm2)
    tf = median_ms(lambda: (gemm1_fused(), gemm2()))
    tu = median_ms(unfused)
    out["single_stream_pair"] = {
        "gemm1_fused_ms": t1f, "gemm1_fused_tflops": f1 / (t1f * 1e-3) / 1e12,
        "gemm1_bf16_out_ms": t1b, "gemm2_ms": t2, "gemm2_tflops": f2 / (t2 * 1e-3) / 1e12,
        "pair_fused_ms": tf, "pair_unfused_ms": tu,
        "note": "GEMM1 4608x3072x21504 + bias (Q, GELU(MLP) -> NVFP4 in the epilogue with the oracle-calibrated "
                "scale; K,V -> bf16), GEMM2 4608x15360x3072 + bias; unfused = GEMM1 writing bf16, column copy, "
                "quantize, GEMM2"}
    del y_qm, y_all, y_kv, y2, a2, w1q, w2q, xq, x
    # --- attention-projection sweep, K = N = 3072
    sweep = []
    for wl in synth.SWEEP:
        x = wl.activations().to(device)
        g = F.global_scale(x)
        xq = F.quantize(x, g)
        w = wl.weight().to(device)
        wq = F.quantize(w, F.global_scale(w))
        y = torch.empty(wl.m, wl.n, dtype=torch.bfloat16, device=device)
        tq = median_ms(lambda: F.quantize(x, g, out=xq, stream=stream))
        tg = median_ms(lambda: F.gemm(xq, wq, y=y, stream=stream))
        w16 = F.dequantize(wq, stream=stream)
        tw = median_ms(lambda: F.linear_w4a16(x, wq, None, y=y, stream=stream))

        def dequant_then_linear():  # the pages' fallback: dequantize, then a library bf16 linear
            F.dequantize(wq, out=w16, stream=stream)
            torch.nn.functional.linear(x, w16)

        twc = median_ms(dequant_then_linear)
        flops = 2 * wl.m * wl.n * wl.k
        # min(compute, memory) roofline: A + B + scales in, Y out
        bytes_ = wl.m * wl.k / 2 + wl.n * wl.k / 2 + (wl.m + wl.n) * wl.k / 16 + wl.m * wl.n * 2
        t_roof = max(flops / (fp4_peak * 1e12), bytes_ / (hbm * 1e9)) * 1e3
        sweep.append({"m": wl.m, "quantize_ms": tq, "gemm_ms": tg, "gemm_tflops": flops / (tg * 1e-3) / 1e12,
                      "frac_of_roofline": t_roof / tg, "w4a16_linear_ms": tw,
                      "w4a16_dequantize_then_cublas_ms": twc})
        del x, xq, w, wq, y, w16
    out["proj_sweep_k3072_n3072"] = sweep
    return out


def run_ours(args):
    import torch
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    import nvfp4_block_scaled_12_b200 as F
    import synth

    wl = synth.MLP_UP
    M, K, N = wl.m, wl.k, wl.n
    flops = 2.0 * M * N * K
    # each rank gets its own token batch (independent seeds): weak scaling
    x = synth.activations_with_outlier_channels(M, K, seed=rank_activation_seed(rank, wl.seed)).to(device)
    w = wl.weight().to(device)
    bias = wl.bias_vec().to(device)
    g_x = F.global_scale(x)              # calibrated input_scale (offline)
    wq = F.quantize(w, F.global_scale(w))  # ModelOpt-style weight prep (offline)
    xq = F.quantize(x, g_x)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def flush_l2():
        # write 256 MiB (twice L2), then read it back: L2 ends up holding clean
        # lines of an unrelated buffer, so the timed kernels read their inputs
        # from HBM and do not pay for write-backs of the flush itself
        flush.zero_()
        flush.view(torch.int64).sum()

    def step():
        F.quantize(x, g_x, out=xq, stream=stream)
        F.gemm(xq, wq, bias=bias, y=y, stream=stream)

    for _ in range(max(args.warmup, 0)):
        flush_l2()
        step()
    torch.cuda.synchronize(device)
    F.nvfp4_check_fault()

    # The step is timed whole (one event pair around quantize + GEMM: an event
    # recorded between the two kernels costs the step ~3 us); the split into
    # the two kernels comes from two more loops that time each one alone, the
    # same way (L2 flushed before every launch, outside the events).
    def timed_loop(body):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in evs:
            flush_l2()  # between timed steps, outside the events
            a.record(stream)
            body()
            b.record(stream)
        return evs

    sampler = ClockSampler(local if not os.environ.get("CUDA_VISIBLE_DEVICES") else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
    sampler.start()
    time.sleep(0.2)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    # the clock record covers all three timed loops (the step, and each kernel
    # alone for the split and the roofline)
    t_wall0 = time.time()
    ev_step = timed_loop(step)
    ev_q = timed_loop(lambda: F.quantize(x, g_x, out=xq, stream=stream))
    ev_g = timed_loop(lambda: F.gemm(xq, wq, bias=bias, y=y, stream=stream))
    torch.cuda.synchronize(device)
    t_wall1 = time.time()
    if world > 1:
        torch.distributed.barrier()
    sampler.stop()
    F.nvfp4_check_fault()

    def mean_ms(evs):
        return sum(a.elapsed_time(b) for a, b in evs) / len(evs)

    step_ms = mean_ms(ev_step)
    step_ms_max = max_over_ranks(step_ms, world, device)
    gemm_ms = max_over_ranks(mean_ms(ev_g), world, device)
    quant_ms = max_over_ranks(mean_ms(ev_q), world, device)

    # end to end through the public API with host buffers: pinned x in,
    # pinned y out, copies inside the timed region
    x_host = x.cpu().pin_memory()
    y_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        x_dev.copy_(x_host, non_blocking=True)
        F.quantize(x_dev, g_x, out=xq, stream=stream)
        F.gemm(xq, wq, bias=bias, y=y, stream=stream)
        y_host.copy_(y, non_blocking=True)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        x_dev.copy_(x_host, non_blocking=True)
        F.quantize(x_dev, g_x, out=xq, stream=stream)
        F.gemm(xq, wq, bias=bias, y=y, stream=stream)
        y_host.copy_(y, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_serial_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, device)

    # the same steps pipelined the way a serving loop would run them: the
    # input copy, the compute and the result copy of a step each on their own
    # stream, device tensors double-buffered, so step i's result copy overlaps
    # step i+1's input copy and compute (every step still moves its input in
    # and its result out inside the timed region)
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    xd2 = [torch.empty_like(x) for _ in range(2)]
    xq2 = [F.quantize(x, g_x, stream=stream) for _ in range(2)]
    y2 = [torch.empty(M, N, dtype=torch.bfloat16, device=device) for _ in range(2)]
    done_in = [torch.cuda.Event() for _ in range(2)]
    done_mm = [torch.cuda.Event() for _ in range(2)]
    done_out = [torch.cuda.Event() for _ in range(2)]

    def pipelined(n):
        for i in range(n):
            b = i % 2
            if i >= 2:
                s_in.wait_event(done_mm[b])        # x_dev[b] free again
            with torch.cuda.stream(s_in):
                xd2[b].copy_(x_host, non_blocking=True)
            done_in[b].record(s_in)
            stream.wait_event(done_in[b])
            if i >= 2:
                stream.wait_event(done_out[b])     # y[b] copied out
            F.quantize(xd2[b], g_x, out=xq2[b], stream=stream)
            F.gemm(xq2[b], wq, bias=bias, y=y2[b], stream=stream)
            done_mm[b].record(stream)
            s_out.wait_event(done_mm[b])
            with torch.cuda.stream(s_out):
                y_host.copy_(y2[b], non_blocking=True)
            done_out[b].record(s_out)

    pipelined(4)
    torch.cuda.synchronize(device)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record(s_in)
    pipelined(e2e_steps)
    s_in.wait_stream(s_out)
    p1.record(s_in)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(p0.elapsed_time(p1) / e2e_steps, world, device)

    # the standalone activation-quantize workload, bf16 [4608, 12288]
    xl = synth.quantize_input().to(device)
    gl = F.global_scale(xl)
    xlq = F.quantize(xl, gl)
    ql_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
    for a, b in ql_ev:
        flush_l2()
        a.record(stream)
        F.quantize(xl, gl, out=xlq, stream=stream)
        b.record(stream)
    torch.cuda.synchronize(device)
    ql_ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in ql_ev[3:]), world, device)
    F.nvfp4_check_fault()

    # the dynamic-scale variant (per-tensor scale measured in the same
    # launch): its quantize alone, on both shapes, and the MLP-up linear
    # layer built on it (quantize_dynamic + GEMM reading g on the device)
    ws = torch.empty(F.NVFP4_DYNAMIC_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
    xq_dyn = F.quantize_dynamic(x, workspace=ws, stream=stream)
    xlq_dyn = F.quantize_dynamic(xl, workspace=ws, stream=stream)

    def median_ms(fn, n=20, skip=3):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, b in evs:
            flush_l2()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(device)
        return max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in evs[skip:]), world, device)

    qd_ms = median_ms(lambda: F.quantize_dynamic(x, out=xq_dyn, workspace=ws, stream=stream))
    qdl_ms = median_ms(lambda: F.quantize_dynamic(xl, out=xlq_dyn, workspace=ws, stream=stream))

    def linear_dynamic():
        F.quantize_dynamic(x, out=xq_dyn, workspace=ws, stream=stream)
        F.gemm(xq_dyn, wq, bias=bias, y=y, stream=stream)

    ld_ms = median_ms(linear_dynamic)
    # the one-pass dynamic scale: the amax of a layer's input emitted by the
    # previous layer's GEMM epilogue (timed here on the MLP-up GEMM itself),
    # then the quantize that derives g from it on the device
    amax_x = torch.empty(1, dtype=torch.float32, device=device)
    amax_xl = torch.empty(1, dtype=torch.float32, device=device)
    amax_x.fill_(float(x.float().abs().max()))
    amax_xl.fill_(float(xl.float().abs().max()))
    xq_fa = F.quantize_from_amax(x, amax_x, stream=stream)
    xlq_fa = F.quantize_from_amax(xl, amax_xl, stream=stream)
    qa_ms = median_ms(lambda: F.quantize_from_amax(x, amax_x, out=xq_fa, stream=stream))
    qal_ms = median_ms(lambda: F.quantize_from_amax(xl, amax_xl, out=xlq_fa, stream=stream))
    amax_y = torch.zeros(1, dtype=torch.float32, device=device)
    ga_ms = median_ms(lambda: F.gemm(xq, wq, bias=bias, y=y, amax_out=amax_y, stream=stream))

    def linear_from_amax():
        F.quantize_from_amax(x, amax_x, out=xq_fa, stream=stream)
        F.gemm(xq_fa, wq, bias=bias, y=y, stream=stream)

    lfa_ms = median_ms(linear_from_amax)
    F.nvfp4_check_fault()
    # the MXFP8 variant on the same MLP-up shape: E4M3 activations and
    # weights with one E8M0 scale per 32 elements, no per-tensor scale
    wq8 = F.quantize_mxfp8(w, stream=stream)
    xq8 = F.quantize_mxfp8(x, stream=stream)
    q8_ms = median_ms(lambda: F.quantize_mxfp8(x, out=xq8, stream=stream))
    g8_ms = median_ms(lambda: F.gemm_mxfp8(xq8, wq8, bias=bias, y=y, stream=stream))
    # row-wise FP8 (W8A8) on the same shape: E4M3 with one fp32 scale per row
    wr8 = F.quantize_fp8row(w, stream=stream)
    xr8 = F.quantize_fp8row(x, stream=stream)
    qr_ms = median_ms(lambda: F.quantize_fp8row(x, out=xr8, stream=stream))
    gr_ms = median_ms(lambda: F.gemm_fp8row(xr8, wr8, bias=bias, y=y, stream=stream))
    # W4A16: the weight dequantized to bf16 by this library, then a regular
    # bf16 linear (a library GEMM) on the unquantized activations
    w16 = F.dequantize(wq, stream=stream)
    dq_ms = median_ms(lambda: F.dequantize(wq, out=w16, stream=stream))
    lw_ms = median_ms(lambda: F.linear_w4a16(x, wq, bias, y=y, stream=stream))

    def dequant_then_linear():  # the pages' fallback: dequantize, then a library bf16 linear
        F.dequantize(wq, out=w16, stream=stream)
        torch.nn.functional.linear(x, w16, bias)

    lwc_ms = median_ms(dequant_then_linear)
    F.nvfp4_check_fault()
    extras = {}
    if world == 1 and not args.no_extras:
        hbm_, bf16_, _ = peaks()
        extras = extra_workloads(F, torch, synth, device, stream, median_ms, hbm_, bf16_ * FP4_PER_BF16)
        F.nvfp4_check_fault()

    if rank == 0:
        hbm, bf16, src = peaks()
        fp4_peak = bf16 * FP4_PER_BF16
        gemm_tf = flops / (gemm_ms * 1e-3) / 1e12
        quant_gbs = M * K * QUANT_BYTES_PER_ELEM / (quant_ms * 1e-3) / 1e9
        clocks = sampler.summary(t_wall0, t_wall1)
        line = {
            "metric": METRIC,
            "value": world * flops / (step_ms_max * 1e-3) / 1e12,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": step_ms_max,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "fp4(e2m1)xfp4->f32 accum, bf16 out",
            "data": "synthetic",
            "config": {"workload": "flux_mlp_up_m4608_k3072_n12288", "m": M, "k": K, "n": N,
                       "bias": True, "global_batch_tokens": world * M, "parallelism": f"dp{world} (token shards)",
                       "l2": "flushed between timed steps: 256 MiB written then read, outside the events"},
            "roofline": {"bound": "tensor", "achieved": gemm_tf, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": gemm_tf / fp4_peak, "traffic": gemm_dram_traffic(),
                         "peak_source": f"{src} bf16 burst x {FP4_PER_BF16:g} (nominal FP4/bf16 dense ratio)"},
            "kernels": {
                "gemm": {"ms": gemm_ms, "tflops": gemm_tf, "frac_of_fp4_peak": gemm_tf / fp4_peak},
                "quantize": {"ms": quant_ms, "gbs": quant_gbs, "frac_of_hbm": quant_gbs / hbm,
                             "bytes": M * K * QUANT_BYTES_PER_ELEM, "hbm_peak_gbs": hbm, "peak_source": src},
                "quantize_4608x12288": {
                    "ms": ql_ms, "gbs": xl.numel() * QUANT_BYTES_PER_ELEM / (ql_ms * 1e-3) / 1e9,
                    "frac_of_hbm": xl.numel() * QUANT_BYTES_PER_ELEM / (ql_ms * 1e-3) / 1e9 / hbm,
                    "note": "standalone quantize workload (Laplace, spikes, zero blocks), median of 17, L2 flushed"},
                "quantize_dynamic": {
                    "ms": qd_ms, "gbs": M * K * QUANT_BYTES_PER_ELEM / (qd_ms * 1e-3) / 1e9,
                    "frac_of_hbm": M * K * QUANT_BYTES_PER_ELEM / (qd_ms * 1e-3) / 1e9 / hbm,
                    "note": "MLP-up activations with the scale measured in the same cooperative launch (amax pass, "
                            "grid-wide max, quantize pass mostly from L2); bytes counted once, 2.5625 B/elem; "
                            "median of 17, L2 flushed"},
                "quantize_dynamic_4608x12288": {
                    "ms": qdl_ms, "gbs": xl.numel() * QUANT_BYTES_PER_ELEM / (qdl_ms * 1e-3) / 1e9,
                    "frac_of_hbm": xl.numel() * QUANT_BYTES_PER_ELEM / (qdl_ms * 1e-3) / 1e9 / hbm,
                    "note": "standalone quantize workload, scale measured in the same launch; median of 17"},
                "linear_dynamic": {
                    "ms": ld_ms, "tflops": flops / (ld_ms * 1e-3) / 1e12,
                    "note": "MLP-up step with the measured scale: quantize_dynamic + GEMM reading g on the device"},
                "quantize_from_amax": {
                    "ms": qa_ms, "gbs": M * K * QUANT_BYTES_PER_ELEM / (qa_ms * 1e-3) / 1e9,
                    "frac_of_hbm": M * K * QUANT_BYTES_PER_ELEM / (qa_ms * 1e-3) / 1e9 / hbm,
                    "ms_4608x12288": qal_ms,
                    "frac_of_hbm_4608x12288": xl.numel() * QUANT_BYTES_PER_ELEM / (qal_ms * 1e-3) / 1e9 / hbm,
                    "gemm_with_amax_ms": ga_ms, "linear_ms": lfa_ms,
                    "note": "one-pass dynamic scale: g derived on the device from an amax the previous layer's "
                            "GEMM epilogue emitted (gemm_with_amax_ms: the MLP-up GEMM measuring max|Y| of its "
                            "own output); linear = that quantize + the GEMM reading g on the device"},
                "mxfp8": {
                    "quantize_ms": q8_ms,
                    "quantize_gbs": M * K * MX_QUANT_BYTES_PER_ELEM / (q8_ms * 1e-3) / 1e9,
                    "quantize_frac_of_hbm": M * K * MX_QUANT_BYTES_PER_ELEM / (q8_ms * 1e-3) / 1e9 / hbm,
                    "gemm_ms": g8_ms, "gemm_tflops": flops / (g8_ms * 1e-3) / 1e12,
                    "gemm_frac_of_fp8_peak": flops / (g8_ms * 1e-3) / 1e12 / (bf16 * FP8_PER_BF16),
                    "note": "MLP-up shape with MXFP8 operands (E4M3, E8M0 per 32); quantize bytes 2 + 1 + 1/32 "
                            "per element; FP8 peak = measured bf16 burst x 2 (nominal FP8/bf16 dense ratio)"},
                "fp8row": {
                    "quantize_ms": qr_ms,
                    "quantize_gbs": (M * K * 3 + M * 4) / (qr_ms * 1e-3) / 1e9,
                    "quantize_frac_of_hbm": (M * K * 3 + M * 4) / (qr_ms * 1e-3) / 1e9 / hbm,
                    "gemm_ms": gr_ms, "gemm_tflops": flops / (gr_ms * 1e-3) / 1e12,
                    "gemm_frac_of_fp8_peak": flops / (gr_ms * 1e-3) / 1e12 / (bf16 * FP8_PER_BF16),
                    "note": "MLP-up shape with row-wise FP8 (E4M3, fp32 scale per row of A and of W); quantize "
                            "bytes 2 + 1 per element + 4 per row"},
                "w4a16": {
                    "dequantize_ms": dq_ms,
                    "dequantize_gbs": N * K * QUANT_BYTES_PER_ELEM / (dq_ms * 1e-3) / 1e9,
                    "dequantize_frac_of_hbm": N * K * QUANT_BYTES_PER_ELEM / (dq_ms * 1e-3) / 1e9 / hbm,
                    "linear_ms": lw_ms, "linear_tflops": flops / (lw_ms * 1e-3) / 1e12,
                    "linear_frac_of_bf16_peak": flops / (lw_ms * 1e-3) / 1e12 / bf16,
                    "dequantize_then_cublas_ms": lwc_ms,
                    "note": "MLP-up shape; linear = this library's W4A16 GEMM (weight tiles dequantized in shared "
                            "memory, tcgen05 kind::f16, bias fused); dequantize_then_cublas = the dequantize kernel "
                            "(weight [12288,3072] NVFP4 -> bf16, 0.5 + 1/16 in, 2 out per element) then torch "
                            "linear (cuBLAS bf16); bf16 peak = measured burst"},
                **extras,
            },
            "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
                    "ms_per_step": e2e_ms,
                    "note": "pinned host x in, pinned host y out, every step; input copy, compute and result copy "
                            "on three streams with double-buffered device tensors",
                    "serial_value": world * flops / (e2e_serial_ms * 1e-3) / 1e12,
                    "serial_ms_per_step": e2e_serial_ms},
            "gpu_launches": 2 * args.steps,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"],
                       "samples": clocks["samples"]},
        }
        ql_gbs = xl.numel() * QUANT_BYTES_PER_ELEM / (ql_ms * 1e-3) / 1e9
        line["quantize_roofline"] = {
            "workload": "laplace_quantize_m4608_k12288", "bound": "hbm", "achieved": ql_gbs, "peak": hbm,
            "unit": "GB/s", "frac": ql_gbs / hbm, "traffic": quantize_dram_traffic(),
            "bytes": xl.numel() * QUANT_BYTES_PER_ELEM, "ms": ql_ms,
            "peak_source": f"{src} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else src}
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline()
            line["quantize_cpu_baseline"] = quantize_cpu_baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the single-stream pair and token-sweep measurements")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
