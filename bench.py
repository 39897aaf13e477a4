"""Benchmark of the weight-only block-32 qgemv/qgemm path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Default workload ("decoder_block_m1"): one Qwen3-0.6B-style decoder block at decode, M = 1,
int4 block-32 weights: the 7 projections q[2048x1024], k[1024x1024], v[1024x1024],
o[1024x2048], gate/up[3072x1024], down[1024x3072]. q|k|v share their input, as do gate|up,
so their packed rows are stored concatenated and one step is 4 qgemv calls: qkv[4096x1024],
o, gate_up[6144x1024], down (--unfused: 7 calls). Consecutive steps walk the 28 blocks of a
seeded synthetic decoder (247.7 MB of packed weights, more than the 126 MB L2), so every
step streams its weights from HBM. Metric: weight GB/s (packed codes + scales per step /
time).

Timed region: K steps replayed from CUDA graphs on one stream, bracketed by a barrier and
device synchronisation, timed with CUDA events on that stream; the max over ranks is
reported. Under torchrun every rank runs its own replica (no data-path collective).

Also on the JSON line: `e2e` (the same steps through the public API with x copied from
pinned host memory and y read back every step), `roofline` (the qgemv kernel against the
measured HBM copy bandwidth), `cpu_baseline` (the CPU oracle on the host cores, a bounded
sample), `parity` (GPU vs oracle on the sampled step), `kernel_roofline_lm_head` (one qgemv
launch over the 165 MB int8 lm_head, the kernel alone against HBM), and `prefill` (the tcgen05
qgemm over all projections of all 28 blocks at M = 512, TFLOP/s against the measured bf16
peak).
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from weight_only_bit_qgemv_b200 import workloads  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def measured_traffic(workload: str, root: str | None = None):
    """DRAM bytes per launch for `workload` from profiles/traffic.txt (an ncu capture), or None
    when there is none or a kernel source it was taken with has changed since."""
    import hashlib

    root = root or os.path.dirname(os.path.abspath(__file__))
    path = os.path.join(root, "profiles", "traffic.txt")
    csrc = os.path.join(root, "weight_only_bit_qgemv_b200", "csrc")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    for line in lines:
        f = line.split()
        if not f or f[0].startswith("#") or f[0] != workload:
            continue
        for dep in f[3:]:
            name, digest = dep.split("=")
            try:
                now = hashlib.sha256(open(os.path.join(csrc, name), "rb").read()).hexdigest()[:16]
            except OSError:
                return None
            if now != digest:
                return None
        return int(f[1])
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------------------
# distributed plumbing (replicas only)
# --------------------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    if world == 1:
        return value
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank: float, ms_per_rank: float, world: int):
    """(whole-job units/s, max ms) with the max-over-ranks time as the job's time."""
    ms = max_over_ranks(ms_per_rank, world)
    return units_per_rank * world / (ms / 1e3), ms


# --------------------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        time.sleep(0.25)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------------------
# the workload
# --------------------------------------------------------------------------------------

#: Launch groups of one decoder block. A real decoder feeds q, k and v the same input and
#: gate and up the same input, so their weights are stored row-concatenated and run as one
#: qgemv each (qkv [4096x1024], gate_up [6144x1024]); every packed byte is unchanged.
FUSED_GROUPS = (("qkv", (0, 1, 2)), ("o", (3,)), ("gate_up", (4, 5)), ("down", (6,)))
UNFUSED_GROUPS = tuple((nm, (i,)) for i, (nm, _, _) in enumerate(workloads.DECODER_PROJ))


def group_shape(members):
    n = sum(workloads.DECODER_PROJ[i][1] for i in members)
    k = workloads.DECODER_PROJ[members[0]][2]
    return n, k


def group_x_seed(members):
    """Activation seed of a launch group (one input per group, shared by its members)."""
    return workloads.X_SEED + members[0]


def group_weight(layer, members):
    """float32 weight of a group: its members' seeded weights, rows concatenated."""
    ws = []
    for i in members:
        _, n, k = workloads.DECODER_PROJ[i]
        ws.append(workloads.weight(n, k, seed=workloads.layer_seed(layer, i)))
    return torch.cat(ws, 0) if len(ws) > 1 else ws[0]


def build_decoder(bits: int, device, groups, n_layers: int = workloads.N_LAYERS):
    import weight_only_bit_qgemv_b200 as woq

    return [[woq.pack(group_weight(layer, mem), bits, device) for _, mem in groups]
            for layer in range(n_layers)]


def decode_step_bytes(layer):
    return sum(w.nbytes for w in layer)


def time_graph_steps(step_fn, n_cycle: int, steps: int, warmup: int, stream, world):
    """Capture step_fn(i) for i in [0, n_cycle) into a graph; replay to cover `steps` steps.

    Returns (ms for the K timed steps, launches of our kernels per step).
    """
    import weight_only_bit_qgemv_b200 as woq

    def capture(count, start):
        g = torch.cuda.CUDAGraph()
        c0 = woq.launch_count()
        with torch.cuda.graph(g, stream=stream):
            for i in range(count):
                step_fn((start + i) % n_cycle)
        return g, woq.launch_count() - c0

    with torch.cuda.stream(stream):
        for i in range(min(2, n_cycle)):  # eager warm-up (allocations, attribute setup)
            step_fn(i)
    stream.synchronize()
    full, launches_full = capture(n_cycle, 0)
    rem = steps % n_cycle
    g_rem = capture(rem, 0)[0] if rem else None
    per_step = launches_full / n_cycle

    # warm-up steps, untimed
    w_full, w_rem = divmod(warmup, n_cycle)
    g_wrem = capture(w_rem, 0)[0] if w_rem else None
    with torch.cuda.stream(stream):
        for _ in range(w_full):
            full.replay()
        if g_wrem is not None:
            g_wrem.replay()
    stream.synchronize()

    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(steps // n_cycle):
            full.replay()
        if g_rem is not None:
            g_rem.replay()
        end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end), per_step


def run_decode(args, world, rank, local, peaks, peak_kind):
    import weight_only_bit_qgemv_b200 as woq

    device = torch.device("cuda", local)
    bits = 4
    groups = UNFUSED_GROUPS if args.unfused else FUSED_GROUPS
    layers = build_decoder(bits, device, groups)
    M = args.m
    xs = [workloads.activations(M, group_shape(mem)[1], seed=group_x_seed(mem)).to(device)
          for _, mem in groups]
    ys = [torch.empty(M, group_shape(mem)[0], device=device) for _, mem in groups]
    step_bytes = decode_step_bytes(layers[0])
    total_bytes = sum(decode_step_bytes(l) for l in layers)

    def step(i):
        for g, w in enumerate(layers[i]):
            woq.qgemv(xs[g], w, out=ys[g])

    stream = torch.cuda.Stream(device)
    with ClockSampler(local) as clk:
        ms, per_step = time_graph_steps(step, len(layers), args.steps, args.warmup, stream, world)
    clocks = clk.summary()
    value, ms_max = aggregate_throughput(step_bytes * args.steps, ms, world)
    gbs = value / 1e9

    # the qgemv kernel against the HBM roofline: every launch in the timed region is it
    launches = per_step * args.steps
    achieved = step_bytes * args.steps / (ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": (measured_traffic("decoder_block_m1")
                            if M == 1 and not args.unfused else None),
                "peak_source": peak_kind,
                "bytes_per_launch": round(step_bytes / per_step),
                "avg_launch_us": round(ms * 1e3 / launches, 3)}

    e2e = run_decode_e2e(layers, groups, device, min(args.steps, 2000), stream, world, M)

    out = {
        "metric": "decode qgemv weight GB/s (% of HBM peak); prefill qgemm TFLOP/s (% peak)",
        "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"decoder_block_m{M}", "bits": 4, "block": 32, "m": M,
                   "launches": [f"{nm}[{group_shape(mem)[0]}x{group_shape(mem)[1]}]"
                                for nm, mem in groups],
                   "fused_qkv_gate_up": not args.unfused,
                   "layers_cycled": len(layers), "weight_bytes_per_step": step_bytes,
                   "l2": f"inputs larger than L2: steps walk {len(layers)} blocks, "
                         f"{total_bytes / 1e6:.1f} MB of packed weights > 126 MB L2",
                   "launch": "CUDA graph of qgemv C-ABI calls, programmatic dependent launch",
                   "parallelism": f"replicas x{world}"},
        "hbm_frac": round(gbs / world / peaks["hbm_gbs"], 4),
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "roofline": roofline,
    }
    return out, layers, groups, xs


def run_decode_e2e(layers, groups, device, steps, stream, world, M=1):
    """Same steps through the public API, x from pinned host memory, y read back each step.

    Each block's step (the host->device copy of its x rows, its qgemv calls, the
    device->host copy of its outputs) is captured once into a CUDA graph from those API
    calls, as a serving loop would; every timed step replays its block's graph and the host
    waits for the step's outputs before the next one.
    """
    import weight_only_bit_qgemv_b200 as woq

    # A step's inputs sit in one pinned staging buffer and its outputs in another, so that a
    # step moves them in one copy each way (every group's slice starts on a 16-byte boundary).
    xs = [workloads.activations(M, group_shape(mem)[1], seed=group_x_seed(mem)) for _, mem in groups]
    x_sizes = [t.numel() for t in xs]
    y_sizes = [M * group_shape(mem)[0] for _, mem in groups]
    host_x = torch.cat([t.reshape(-1) for t in xs]).pin_memory()
    host_y = torch.empty(sum(y_sizes)).pin_memory()
    dx_all = torch.empty_like(host_x, device=device)
    dy_all = torch.empty_like(host_y, device=device)
    dx = [v.view(M, -1) for v in torch.split(dx_all, x_sizes)]
    dy = [v.view(M, -1) for v in torch.split(dy_all, y_sizes)]
    h2d = host_x.numel() * 4
    d2h = host_y.numel() * 4

    def ops(layer):
        dx_all.copy_(host_x, non_blocking=True)
        for g, w in enumerate(layer):
            woq.qgemv(dx[g], w, out=dy[g])
        host_y.copy_(dy_all, non_blocking=True)

    graphs = []
    with torch.cuda.stream(stream):
        ops(layers[0])  # warm-up outside capture
        stream.synchronize()
        for layer in layers:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                ops(layer)
            graphs.append(g)

        def step(i):
            graphs[i % len(graphs)].replay()
            stream.synchronize()

        for i in range(5):
            step(i)
        barrier(world)
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(steps):
            step(i)
        end.record(stream)
        end.synchronize()
    barrier(world)
    ms = start.elapsed_time(end)
    del graphs
    value, _ = aggregate_throughput(decode_step_bytes(layers[0]) * steps, ms, world)
    return {"value": round(value / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms / steps,
            "launch": "per step: replay of a CUDA graph captured from the qgemv API calls and "
                      "one pinned-memory copy each way; the host waits for each step's outputs"}


def run_lm_head_roofline(device, peaks, peak_kind, reps=20):
    """qgemv on the int8 lm_head [151936x1024] at M = 1: one 165 MB launch, the kernel alone.

    Two packed copies alternate so that every launch streams its weights from HBM.
    """
    import weight_only_bit_qgemv_b200 as woq

    n, k = workloads.LM_HEAD
    w0 = woq.pack(workloads.weight(n, k, seed=workloads.LM_HEAD_SEED), 8, device)
    w1 = woq.PackedWeight(w0.packed.clone(), w0.scales.clone(), 8, n, k)
    x = workloads.activations(1, k, seed=workloads.X_SEED).to(device)
    y = torch.empty(1, n, device=device)
    for _ in range(3):
        woq.qgemv(x, w0, out=y)
        woq.qgemv(x, w1, out=y)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
    s = torch.cuda.current_stream()
    ev[0].record(s)
    for r in range(reps):
        woq.qgemv(x, w0 if r % 2 == 0 else w1, out=y)
        ev[r + 1].record(s)
    ev[-1].synchronize()
    times = [ev[r].elapsed_time(ev[r + 1]) for r in range(reps)]
    med = statistics.median(times)
    gbs = w0.nbytes / (med / 1e3) / 1e9
    # The fused greedy pick over the same weights (zero keys, GEMV with argmax, finish):
    # no logits written.
    # Timed as a decode loop runs it: calls captured in a CUDA graph (programmatic dependent
    # launch between the three kernels), replayed.
    gs = torch.cuda.Stream(device)
    for _ in range(3):
        woq.qgemv_argmax(x, w0, stream=gs)
    gs.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=gs):
        for r in range(reps):
            woq.qgemv_argmax(x, w0 if r % 2 == 0 else w1, stream=gs)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(gs):  # replay() launches on the current stream
        for _ in range(2):
            graph.replay()
        gs.synchronize()
        e0.record(gs)
        graph.replay()
        e1.record(gs)
    e1.synchronize()
    amed = e0.elapsed_time(e1) / reps
    del graph
    argmax = {"call_us": round(amed * 1e3, 2), "achieved": round(w0.nbytes / (amed / 1e3) / 1e9, 1),
              "unit": "GB/s", "launches_per_call": 3,
              "timing": f"{reps} calls replayed from one CUDA graph, CUDA events"}
    return {"workload": "lm_head_m1_int8", "weight_bytes": w0.nbytes, "launch_us_median": med * 1e3,
            "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "traffic": measured_traffic("lm_head_m1_int8"),
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_source": peak_kind,
            "timing": f"median of {reps} single launches, CUDA events, two alternating copies",
            "greedy_argmax": argmax}


def run_prefill(layers, groups, device, m: int, reps: int, peaks, peak_kind, world):
    """tcgen05 qgemm through every projection of every block at M = m (one pass = one rep)."""
    import weight_only_bit_qgemv_b200 as woq

    Xs = [workloads.activations(m, group_shape(mem)[1], seed=group_x_seed(mem)).to(device)
          for _, mem in groups]
    Ys = [torch.empty(m, group_shape(mem)[0], device=device) for _, mem in groups]
    ws = torch.empty(max(woq.qgemm_workspace_bytes(m, w, "bf16_tc") for w in layers[0]),
                     dtype=torch.uint8, device=device)
    flops = 2.0 * m * sum(n * k for _, n, k in workloads.DECODER_PROJ) * len(layers)

    def step(i):
        for layer in layers:
            for g, w in enumerate(layer):
                woq.qgemm(Xs[g], w, path="bf16_tc", out=Ys[g], workspace=ws)

    stream = torch.cuda.Stream(device)
    ms, per_step = time_graph_steps(step, 1, reps, 2, stream, world)
    tflops = flops * reps / (ms / 1e3) / 1e12
    return {"workload": f"prefill_m{m}", "m": m, "gemm_calls_per_pass": len(layers) * len(groups),
            "flop_per_pass": flops, "passes": reps, "ms_per_pass": ms / reps,
            "tflops": round(tflops, 1), "peak_tflops": peaks["bf16_tflops"],
            "frac": round(tflops / peaks["bf16_tflops"], 4), "peak_source": peak_kind,
            "launches_per_pass": int(per_step)}


def run_batched_decode(layers, groups, device, m: int, steps: int, peaks, peak_kind, world):
    """Batched decode: m activation rows through every fused projection of every block via
    qgemm's automatic path (the FP32-accurate split tensor-core GEMM for 24 <= m < 128, the
    CUDA-core kernel below), replayed from CUDA graphs like the M = 1 decode."""
    import weight_only_bit_qgemv_b200 as woq

    xs = [workloads.activations(m, group_shape(mem)[1], seed=group_x_seed(mem)).to(device)
          for _, mem in groups]
    ys = [torch.empty(m, group_shape(mem)[0], device=device) for _, mem in groups]
    need = max(woq.qgemm_workspace_bytes(m, w, "auto") for w in layers[0])
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=device)

    def step(i):
        for g, w in enumerate(layers[i]):
            woq.qgemm(xs[g], w, path="auto", out=ys[g], workspace=ws)

    stream = torch.cuda.Stream(device)
    ms, per_step = time_graph_steps(step, len(layers), steps, max(3, steps // 10), stream, world)
    us_block = ms * 1e3 / steps
    step_bytes = decode_step_bytes(layers[0])
    flops = 2.0 * m * sum(n * k for _, n, k in workloads.DECODER_PROJ)
    path = "split_tc" if 24 <= m < 128 else ("bf16_tc" if m >= 128 else "fp32")
    return {"workload": f"decoder_block_m{m}", "m": m, "qgemm_path": path,
            "blocks_timed": steps, "us_per_block": round(us_block, 2),
            "tokens_per_s": round(m * 1e6 / (us_block * len(layers)), 1),
            "weight_gbs": round(step_bytes / (us_block * 1e-6) / 1e9, 1),
            "hbm_frac": round(step_bytes / (us_block * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
            "algorithmic_tflops": round(flops / (us_block * 1e-6) / 1e12, 2),
            "peak_source": peak_kind, "launches_per_block": int(per_step)}


def run_fused_epilogues(layers, groups, device, steps: int, world):
    """The decode-step projections whose neighbours fuse (NEXT-4 rows): gate|up with the SwiGLU
    (qgemv_swiglu, the gate|up outputs never written) and down with the residual add
    (qgemv_residual, in place on the hidden state), each against the plain qgemv of the same
    weights; M = 1, all 28 blocks cycled, CUDA graphs as the decode steps. Timing only: the
    decode step's gate|up matrix is packed as gate rows then up rows, not interleaved, which
    changes which rows pair up but not the work."""
    import weight_only_bit_qgemv_b200 as woq

    names = [nm for nm, _ in groups]
    if "gate_up" not in names or "down" not in names:
        return None
    gu, dn = names.index("gate_up"), names.index("down")
    n_gu, k_gu = group_shape(groups[gu][1])
    n_dn, k_dn = group_shape(groups[dn][1])
    x_gu = workloads.activations(1, k_gu, seed=11).to(device)
    x_dn = workloads.activations(1, k_dn, seed=12).to(device)
    y_gu = torch.empty(1, n_gu, device=device)
    y_sw = torch.empty(1, n_gu // 2, device=device)
    h = torch.zeros(1, n_dn, device=device)
    y_dn = torch.empty(1, n_dn, device=device)
    stream = torch.cuda.Stream(device)
    warm = max(3, steps // 10)

    def timed(fn):
        ms, per_step = time_graph_steps(fn, len(layers), steps, warm, stream, world)
        return ms * 1e3 / steps, int(per_step)

    out = {"m": 1, "calls_timed": steps}
    for key, plain, fused, idx in (
        ("swiglu_gate_up", lambda i: woq.qgemv(x_gu, layers[i][gu], out=y_gu),
         lambda i: woq.qgemv_swiglu(x_gu, layers[i][gu], out=y_sw), gu),
        ("residual_down", lambda i: woq.qgemv(x_dn, layers[i][dn], out=y_dn),
         lambda i: woq.qgemv_residual(x_dn, layers[i][dn], h, out=h), dn),
    ):
        nbytes = layers[0][idx].nbytes
        us_plain, _ = timed(plain)
        us_fused, launches = timed(fused)
        out[key] = {"shape": f"[{layers[0][idx].n}x{layers[0][idx].k}]", "us_per_call": round(us_fused, 3),
                    "plain_qgemv_us": round(us_plain, 3), "launches_per_call": launches,
                    "weight_gbs": round(nbytes / (us_fused * 1e-6) / 1e9, 1)}
    return out


# --------------------------------------------------------------------------------------
# CPU oracle (cpu_baseline leg and the reference arm)
# --------------------------------------------------------------------------------------

def oracle_decode_pass(packed_layer, xs_np, rows=None):
    """One decode step of a block through the oracle; ``rows`` limits each projection."""
    import oracle

    outs = []
    for p, (pk, sc, bits) in enumerate(packed_layer):
        if rows is not None:
            pk, sc = pk[:rows[p]], sc[:rows[p]]
        outs.append(oracle.qgemv_ref(xs_np[p], pk, sc, bits))
    return outs


def oracle_layer_inputs(groups, bits=4, layer=0):
    """The block's 7 projections, quantised and packed by the oracle itself, and their x rows
    (members of a launch group share its input)."""
    import oracle

    x_of = {}
    for _, mem in groups:
        x = workloads.activations(1, group_shape(mem)[1], seed=group_x_seed(mem)).numpy()
        for i in mem:
            x_of[i] = x
    out = []
    for p, (_, n, k) in enumerate(workloads.DECODER_PROJ):
        W = workloads.weight(n, k, seed=workloads.layer_seed(layer, p)).numpy()
        q, s = oracle.quantise(W, bits)
        out.append((oracle.pack(q, bits), s, bits))
    return out, [x_of[p] for p in range(len(workloads.DECODER_PROJ))]


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(packed_layer, xs, budget_s: float):
    """Median seconds per decode-block pass of the oracle; the outputs of the last pass."""
    oracle_decode_pass(packed_layer, xs)  # discarded warm-up
    times, outs = [], None
    t_end = time.perf_counter() + budget_s
    while len(times) < 3 or time.perf_counter() < t_end:
        t0 = time.perf_counter()
        outs = oracle_decode_pass(packed_layer, xs)
        times.append(time.perf_counter() - t0)
        if len(times) >= 50:
            break
    return statistics.median(times), len(times), outs


def cpu_baseline_leg(layer0_gpu, groups, xs_gpu, budget_s):
    import weight_only_bit_qgemv_b200 as woq

    packed, xs = oracle_layer_inputs(groups)
    sec, passes, outs = time_oracle(packed, xs, budget_s)
    nbytes = sum(pk.nbytes + sc.nbytes for pk, sc, _ in packed)
    # parity of the GPU step against the oracle on the same inputs (block 0)
    errs = []
    for g, (w, (_, mem)) in enumerate(zip(layer0_gpu, groups)):
        y = woq.qgemv(xs_gpu[g], w).cpu().numpy()
        ref = np.concatenate([outs[i] for i in mem], axis=1)
        errs.append(float(np.max(np.abs(y - ref)) / np.max(np.abs(ref))))
    return ({"value": round(nbytes / sec / 1e9, 4), "unit": "GB/s", "cores": blas_threads(),
             "kind": "oracle",
             "sample": f"{passes} passes of decoder block 0 (7 projections, M=1, int4) through the "
                       f"NumPy float64 oracle, median pass {sec * 1e3:.1f} ms"},
            {"max_rel_err": max(errs), "tolerance": 1e-4, "checked": "block 0, every output"})


def run_reference(args, world, rank, budget_s=90.0):
    """The oracle as it stands, on the host cores, same metric and config (rank 0 only).

    Each of the K (+W) steps is a bounded sample of the decode step: the first rows of each
    of the 7 projections, sized from one untimed full pass so the whole run takes about
    ``budget_s`` seconds.
    """
    if rank != 0:
        return None
    packed, xs = oracle_layer_inputs(FUSED_GROUPS)
    t0 = time.perf_counter()
    oracle_decode_pass(packed, xs)
    full = time.perf_counter() - t0
    frac = min(1.0, budget_s / (args.steps + args.warmup) / full)
    rows = [max(1, int(round(frac * n))) for (_, n, k) in workloads.DECODER_PROJ]
    nbytes = sum(r * (pk.shape[1] + 2 * sc.shape[1]) for r, (pk, sc, _) in zip(rows, packed))
    for _ in range(args.warmup):
        oracle_decode_pass(packed, xs, rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_decode_pass(packed, xs, rows)
    sec = time.perf_counter() - t0
    value = nbytes * args.steps / sec / 1e9
    sample = (f"each step: rows {rows} of the 7 projections of decoder block 0 (M=1, int4), "
              f"{nbytes} weight bytes, through the NumPy float64 oracle; one full block pass "
              f"took {full * 1e3:.0f} ms")
    return {"impl": "reference",
            "metric": "decode qgemv weight GB/s (% of HBM peak); prefill qgemm TFLOP/s (% peak)",
            "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sec * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "decoder_block_m1", "bits": 4, "block": 32, "m": 1},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------------------------

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=28000)
    ap.add_argument("--warmup", type=int, default=280)
    ap.add_argument("--impl", default="woq", choices=["woq", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-m", type=int, default=512)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--unfused", action="store_true", help="7 launches per block instead of 4")
    ap.add_argument("--m", type=int, default=1, help="activation rows per decode step (1..64)")
    ap.add_argument("--no-lm-head", action="store_true")
    ap.add_argument("--no-fused-epilogues", action="store_true")
    ap.add_argument("--batched-m", type=int, default=64,
                    help="rows of the batched-decode leg (qgemm auto path); <= 1 skips it")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local = dist_setup()
    if args.impl == "reference":
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0

    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    peaks, peak_kind = load_peaks()
    out, layers, groups, xs = run_decode(args, world, rank, local, peaks, peak_kind)
    device = torch.device("cuda", local)
    if not args.no_lm_head:
        out["kernel_roofline_lm_head"] = run_lm_head_roofline(device, peaks, peak_kind)
    if not args.no_prefill:
        out["prefill"] = run_prefill(layers, groups, device, args.prefill_m, 3, peaks, peak_kind,
                                     world)
    if args.batched_m > 1:
        out["batched_decode"] = run_batched_decode(layers, groups, device, args.batched_m,
                                                   280, peaks, peak_kind, world)
    if not args.no_fused_epilogues:
        fe = run_fused_epilogues(layers, groups, device, 2800, world)
        if fe is not None:
            out["fused_epilogues"] = fe
    if rank == 0 and not args.no_cpu_baseline and args.m == 1:
        cb, parity = cpu_baseline_leg(layers[0], groups, xs, args.cpu_budget)
        out["cpu_baseline"] = cb
        out["parity"] = parity
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
