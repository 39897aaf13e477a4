"""Benchmark of the weight-only block-32 qgemv/qgemm path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--legs chain,int5,single,lm_head,prefill,batched,epilogues,cpu]

Headline workload ("decoder_block_m1"): one Qwen3-0.6B-style decoder block at decode, M = 1,
int4 block-32 weights: the 7 projections q[2048x1024], k[1024x1024], v[1024x1024],
o[1024x2048], gate/up[3072x1024], down[1024x3072]. q|k|v share their input, as do gate|up,
so their packed rows are stored concatenated and one step is 4 qgemv calls: qkv[4096x1024],
o, gate_up[6144x1024], down (--unfused: 7 calls). Consecutive steps walk the 28 blocks of a
seeded synthetic decoder (247.7 MB of packed weights, more than the 126 MB L2), and L2 is
flushed before the timed region, so every step streams its weights from HBM. Metric: weight
GB/s (packed codes + scales per step / time).

Timed region: K steps replayed from CUDA graphs on one stream, bracketed by a barrier and
device synchronisation, timed with CUDA events on that stream; every graph the timed region
replays has been replayed once, untimed, before it; the max over ranks is reported. Under
torchrun every rank runs its own replica (no data-path collective).

Also on the JSON line: `per_kernel` (each projection's launch timed alone, L2-cold), `e2e`
(the same steps through the public API with x copied from pinned host memory and y read back
every step), `roofline` (the decode kernel against the measured HBM copy bandwidth),
`cpu_baseline` (the CPU oracle on the host cores, all cores and one core, a bounded sample),
`parity` (GPU vs oracle on the sampled step), and `configs`: one object per workload
configuration of the benchmark (a single qgemv; the decoder block; the int8 lm_head; prefill
M = 512 over all 28 blocks; batched decode M = 64 and prefill M = 4096 over all 28 blocks
plus the lm_head), each with its own dtype, roofline and CPU baseline, beside the decoder
block as one `qgemv_chain` launch, the int4 and int5 lm_head, the int5 decoder block and the
fused epilogues. `--legs` runs a subset (the headline always runs); each leg runs inside an
NVTX range named after its workload, for `ncu --nvtx-include`.
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
METRIC = "decode qgemv weight GB/s (% of HBM peak); prefill qgemm TFLOP/s (% peak)"


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
# timing helpers
# --------------------------------------------------------------------------------------

class L2Flush:
    """Writes a buffer twice the size of L2, so that what follows starts with L2 cold."""

    def __init__(self, device):
        self.buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    def __call__(self, stream):
        with torch.cuda.stream(stream):
            self.buf.fill_(1.0)


def capture_graph(fn, count, stream, start=0):
    """CUDA graph of fn(start), ..., fn(start + count - 1); returns (graph, our launches)."""
    import weight_only_bit_qgemv_b200 as woq

    g = torch.cuda.CUDAGraph()
    c0 = woq.launch_count()
    with torch.cuda.graph(g, stream=stream):
        for i in range(count):
            fn(start + i)
    return g, woq.launch_count() - c0


def time_replays(graphs, stream, world, flush):
    """Device ms of replaying `graphs` in order, timed with CUDA events on `stream`.

    Every distinct graph is replayed once, untimed, first (its upload and first-launch costs
    stay out of the timed region); then L2 is flushed, the ranks meet at a barrier, and the
    replays run between two events, with a device synchronisation on both sides."""
    seen = []
    with torch.cuda.stream(stream):
        for g in graphs:
            if all(g is not h for h in seen):
                g.replay()
                seen.append(g)
    flush(stream)
    stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for g in graphs:
            g.replay()
        end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end)


def time_graph_steps(step_fn, n_cycle: int, steps: int, warmup: int, stream, world, flush):
    """Time `steps` steps of step_fn(i % n_cycle), replayed from CUDA graphs.

    Graphs: `full` holds steps 0..n_cycle-1, `rem` steps 0..(steps % n_cycle)-1; the timed
    region replays full (steps // n_cycle) times, then rem. Untimed first: each of them once,
    and full again until at least `warmup` steps have run. Returns (ms, our launches per step).
    """
    with torch.cuda.stream(stream):
        for i in range(min(2, n_cycle)):  # eager warm-up (attribute setup, lazy module loads)
            step_fn(i)
    stream.synchronize()
    full, launches_full = capture_graph(step_fn, n_cycle, stream)
    rem = steps % n_cycle
    g_rem = capture_graph(step_fn, rem, stream)[0] if rem else None
    timed = [full] * (steps // n_cycle) + ([g_rem] if g_rem is not None else [])
    done = (n_cycle if steps >= n_cycle else 0) + rem
    with torch.cuda.stream(stream):
        while done < warmup:
            full.replay()
            done += n_cycle
    ms = time_replays(timed, stream, world, flush)
    del full, g_rem
    return ms, launches_full / n_cycle


def time_graph_median(fn, count, stream, world, flush, reps=3):
    """Median over `reps` of the device ms of one replay of a graph of fn(0..count-1), each
    replay after an L2 flush. Returns (median ms, our launches per replay)."""
    with torch.cuda.stream(stream):
        fn(0)
    stream.synchronize()
    g, launches = capture_graph(fn, count, stream)
    times = [time_replays([g], stream, world, flush) for _ in range(reps)]
    del g
    return statistics.median(times), launches


def roofline(achieved, peak, unit, bound, peak_kind, traffic=None, **extra):
    out = {"bound": bound, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
           "frac": round(achieved / peak, 4), "traffic": traffic,
           "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else peak_kind}
    out.update(extra)
    return out


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


def block_flops(m):
    return 2.0 * m * sum(n * k for _, n, k in workloads.DECODER_PROJ)


def run_decode(args, world, local, peaks, peak_kind, flush):
    """Configuration 2 (the headline): one decoder block per step at M = args.m."""
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
        ms, per_step = time_graph_steps(step, len(layers), args.steps, args.warmup, stream, world,
                                        flush)
    clocks = clk.summary()
    value, ms_max = aggregate_throughput(step_bytes * args.steps, ms, world)
    gbs = value / 1e9

    # Each projection's launch alone: a graph of it over the 28 blocks, after an L2 flush.
    per_kernel = []
    for g, (nm, mem) in enumerate(groups):
        def one(i, g=g):
            woq.qgemv(xs[g], layers[i % len(layers)][g], out=ys[g])

        kms, _ = time_graph_median(one, len(layers), stream, world, flush)
        us = kms * 1e3 / len(layers)
        nb = layers[0][g].nbytes
        per_kernel.append({"launch": f"{nm}[{group_shape(mem)[0]}x{group_shape(mem)[1]}]",
                           "us": round(us, 3), "weight_bytes": nb,
                           "gbs": round(nb / (us * 1e-6) / 1e9, 1),
                           "hbm_frac": round(nb / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)})
    sum_us = sum(p["us"] for p in per_kernel)
    step_us = ms * 1e3 / args.steps
    dom = max(per_kernel, key=lambda p: p["us"])

    # The decode kernel against the HBM roofline: every launch in the timed region is a
    # qgemv launch; achieved = algorithmic bytes per launch / the timed region's average launch.
    launches = per_step * args.steps
    achieved = step_bytes * args.steps / (ms / 1e3) / 1e9
    roof = roofline(achieved, peaks["hbm_gbs"], "GB/s", "hbm", peak_kind,
                    traffic=(measured_traffic("decoder_block_m1") if M == 1 and not args.unfused
                             else None),
                    bytes_per_launch=round(step_bytes / per_step),
                    avg_launch_us=round(ms * 1e3 / launches, 3),
                    dominant_kernel={"launch": dom["launch"], "us_alone": dom["us"],
                                     "gbs_alone": dom["gbs"], "frac_alone": dom["hbm_frac"]})

    e2e = run_decode_e2e(layers, groups, device, min(args.steps, 2000), stream, world, M)

    out = {
        "metric": METRIC,
        "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"decoder_block_m{M}", "bits": 4, "block": 32, "m": M,
                   "launches": [f"{nm}[{group_shape(mem)[0]}x{group_shape(mem)[1]}]"
                                for nm, mem in groups],
                   "fused_qkv_gate_up": not args.unfused,
                   "layers_cycled": len(layers), "weight_bytes_per_step": step_bytes,
                   "l2": f"L2 flushed before the timed region, and steps walk {len(layers)} blocks, "
                         f"{total_bytes / 1e6:.1f} MB of packed weights > 126 MB L2",
                   "launch": "CUDA graph of qgemv C-ABI calls, programmatic dependent launch",
                   "parallelism": f"replicas x{world}"},
        "hbm_frac": round(gbs / world / peaks["hbm_gbs"], 4),
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "roofline": roof,
        "per_kernel": {"timing": "each launch group alone: a CUDA graph of its 28 blocks' launches "
                                 "after an L2 flush, median of 3, per launch",
                       "kernels": per_kernel, "sum_us": round(sum_us, 3),
                       "step_us": round(step_us, 3),
                       "share_of_step": {p["launch"]: round(p["us"] / step_us, 3) for p in per_kernel}},
    }
    return out, layers, groups, xs


def build_chain_layers(layers, bits, device):
    """Per block: qkv, o and down as packed for the decode step, gate|up packed again with its
    rows interleaved (row 2i gate i, row 2i+1 up i), as the fused SwiGLU reads them."""
    import weight_only_bit_qgemv_b200 as woq

    out = []
    for layer, packed in enumerate(layers):
        Wg = workloads.weight(3072, 1024, seed=workloads.layer_seed(layer, 4))
        Wu = workloads.weight(3072, 1024, seed=workloads.layer_seed(layer, 5))
        gu = woq.pack(woq.interleave_rows(Wg, Wu), bits, device)
        out.append([packed[0], packed[1], gu, packed[3]])
    return out


class ChainStep:
    """One decoder block's step as one qgemv_chain launch, with the block's real dependencies:
    y_qkv = qkv(x0); h1 = o(attn) + h0; a = SwiGLU(gate|up(h1)); h2 = down(a) + h1. The
    attention between qkv and o is not part of this path: attn is an input, and o still waits
    for qkv. h0 is fixed, so every step of a block computes the same values."""

    def __init__(self, clayers, m, device):
        import weight_only_bit_qgemv_b200 as woq

        self.x0 = workloads.activations(m, 1024, seed=workloads.X_SEED).to(device)
        self.attn = workloads.activations(m, 2048, seed=workloads.X_SEED + 3).to(device)
        self.h0 = workloads.activations(m, 1024, seed=workloads.X_SEED + 10).to(device)
        self.y_qkv = torch.empty(m, 4096, device=device)
        self.h1 = torch.empty(m, 1024, device=device)
        self.a = torch.empty(m, 3072, device=device)
        self.h2 = torch.empty(m, 1024, device=device)
        self.ws = woq.chain_workspace(device)
        self.items = [[woq.ChainItem(L[0], self.x0, self.y_qkv),
                       woq.ChainItem(L[1], self.attn, self.h1, self.h0, "residual"),
                       woq.ChainItem(L[2], self.h1, self.a, None, "swiglu"),
                       woq.ChainItem(L[3], self.a, self.h2, self.h1, "residual")] for L in clayers]

    def __call__(self, i, stream=None):
        import weight_only_bit_qgemv_b200 as woq

        woq.qgemv_chain(self.items[i % len(self.items)], self.ws, stream=stream)


def run_decode_chain(args, world, local, peaks, peak_kind, flush, layers):
    """The decoder block step at M = args.m as one qgemv_chain launch per block."""
    import weight_only_bit_qgemv_b200 as woq

    device = torch.device("cuda", local)
    clayers = build_chain_layers(layers, 4, device)
    M = args.m
    step = ChainStep(clayers, M, device)
    step_bytes = decode_step_bytes(clayers[0])
    total_bytes = sum(decode_step_bytes(l) for l in clayers)
    stream = torch.cuda.Stream(device)
    with ClockSampler(local) as clk:
        ms, per_step = time_graph_steps(step, len(clayers), args.steps, args.warmup, stream, world,
                                        flush)
    clocks = clk.summary()
    value, ms_max = aggregate_throughput(step_bytes * args.steps, ms, world)
    gbs = value / 1e9
    launches = per_step * args.steps
    step_us = ms * 1e3 / args.steps
    roof = roofline(gbs / world, peaks["hbm_gbs"], "GB/s", "hbm", peak_kind,
                    traffic=measured_traffic("decoder_block_m1_chain") if M == 1 else None,
                    bytes_per_launch=round(step_bytes / per_step),
                    avg_launch_us=round(ms * 1e3 / launches, 3),
                    dominant_kernel={"launch": "qgemv_chain_kernel (the whole step)",
                                     "us": round(step_us, 3)})
    e2e = run_chain_e2e(step, clayers, device, min(args.steps, 2000), stream, world, M)
    return {
        "value": round(gbs, 1), "ms_per_step": ms_max / args.steps,
        "config": {"workload": f"decoder_block_m{M}", "bits": 4, "block": 32, "m": M,
                   "launches": ["qgemv_chain: qkv[4096x1024] -> o[1024x2048]+residual -> "
                                "gate|up[6144x1024]+SwiGLU -> down[1024x3072]+residual"],
                   "step": "one qgemv_chain launch per block; items wait for their predecessors",
                   "layers_cycled": len(clayers), "weight_bytes_per_step": step_bytes,
                   "l2": f"L2 flushed before the timed region, and steps walk {len(clayers)} "
                         f"blocks, {total_bytes / 1e6:.1f} MB of packed weights > 126 MB L2",
                   "launch": "CUDA graph of qgemv_chain C-ABI calls, programmatic dependent launch",
                   "parallelism": f"replicas x{world}"},
        "hbm_frac": round(gbs / world / peaks["hbm_gbs"], 4),
        "clocks": clocks, "e2e": e2e, "gpu_launches": int(launches), "roofline": roof,
        "per_kernel": {"timing": "one launch per step: the step time is the kernel's",
                       "kernels": [{"launch": "qgemv_chain", "us": round(step_us, 3),
                                    "weight_bytes": step_bytes,
                                    "gbs": round(step_bytes / (step_us * 1e-6) / 1e9, 1)}],
                       "sum_us": round(step_us, 3), "step_us": round(step_us, 3)},
    }, clayers, step


def run_chain_e2e(step, clayers, device, steps, stream, world, M=1):
    """The chain step through the public API with its inputs copied from pinned host memory and
    its outputs (y_qkv, h2) read back every step; one captured graph per block, replayed."""
    h_in = torch.cat([step.x0.reshape(-1), step.attn.reshape(-1), step.h0.reshape(-1)]).cpu().pin_memory()
    d_in = torch.empty_like(h_in, device=device)
    n0, n1 = step.x0.numel(), step.attn.numel()
    h_out = torch.empty(step.y_qkv.numel() + step.h2.numel()).pin_memory()

    def ops(i):
        d_in.copy_(h_in, non_blocking=True)
        step.x0.view(-1).copy_(d_in[:n0])
        step.attn.view(-1).copy_(d_in[n0:n0 + n1])
        step.h0.view(-1).copy_(d_in[n0 + n1:])
        step(i)
        h_out[:step.y_qkv.numel()].copy_(step.y_qkv.view(-1), non_blocking=True)
        h_out[step.y_qkv.numel():].copy_(step.h2.view(-1), non_blocking=True)

    graphs = []
    with torch.cuda.stream(stream):
        ops(0)
        stream.synchronize()
        for i in range(len(clayers)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                ops(i)
            graphs.append(g)
        for g in graphs:  # every graph replayed once, untimed
            g.replay()
            stream.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(steps):
            graphs[i % len(graphs)].replay()
            stream.synchronize()
        end.record(stream)
        end.synchronize()
    barrier(world)
    ms = start.elapsed_time(end)
    del graphs
    value, _ = aggregate_throughput(decode_step_bytes(clayers[0]) * steps, ms, world)
    return {"value": round(value / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h_in.numel() * 4,
            "d2h_bytes_per_step": h_out.numel() * 4, "steps": steps, "ms_per_step": ms / steps,
            "launch": "per step: replay of a CUDA graph captured from the API calls (one pinned "
                      "copy in, device-side scatter, the qgemv_chain call, copies out); the host "
                      "waits for each step's outputs"}


def chain_parity(step, clayers_np):
    """Block 0's chain step against the oracle, item by item on the inputs each item read."""
    import oracle

    step(0)
    torch.cuda.synchronize()
    g = lambda t: t.cpu().numpy().astype(np.float64)  # noqa: E731
    (pq, sq), (po, so), (pg, sg), (pd, sd) = clayers_np
    refs = [(g(step.y_qkv), oracle.qgemv_ref(g(step.x0), pq, sq, 4)),
            (g(step.h1), oracle.residual_ref(g(step.attn), po, so, 4, g(step.h0))),
            (g(step.a), oracle.swiglu_ref(g(step.h1), pg, sg, 4)),
            (g(step.h2), oracle.residual_ref(g(step.a), pd, sd, 4, g(step.h1)))]
    errs = [float(np.max(np.abs(y - r)) / np.max(np.abs(r))) for y, r in refs]
    return {"max_rel_err": max(errs), "tolerance": 1e-4,
            "checked": "block 0's chain step, every output of every item"}


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

        for i in range(len(graphs)):  # every graph replayed once, untimed
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


def run_single_qgemv(device, peaks, peak_kind, stream, world, flush):
    """Configuration 1: one qgemv, x [1, 1024], W [3072, 1024] int4 (W seed 0, x seed 0).

    The weight is 1.77 MB, far below L2, so a CUDA graph of calls rotates over distinct copies
    of it whose total is more than twice L2: every call streams its weights from HBM. Reported:
    the average call in that graph (programmatic dependent launch between calls), and the
    latency of one call alone (L2 flushed first, the GPU kept busy while it is enqueued)."""
    import weight_only_bit_qgemv_b200 as woq

    n, k = 3072, 1024
    w0 = woq.pack(workloads.weight(n, k, seed=0), 4, device)
    copies = -(-2 * L2_BYTES // w0.nbytes) + 1
    ws = [w0] + [woq.PackedWeight(w0.packed.clone(), w0.scales.clone(), 4, n, k)
                 for _ in range(copies - 1)]
    x = workloads.activations(1, k, seed=0).to(device)
    y = torch.empty(1, n, device=device)
    ms, launches = time_graph_median(lambda i: woq.qgemv(x, ws[i % copies], out=y), copies,
                                     stream, world, flush)
    call_us = ms * 1e3 / copies
    # one call alone
    lat = []
    with torch.cuda.stream(stream):
        for r in range(7):
            flush(stream)
            torch.cuda._sleep(40000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            woq.qgemv(x, ws[r % copies], out=y, stream=stream)
            e1.record(stream)
            e1.synchronize()
            lat.append(e0.elapsed_time(e1) * 1e3)
    gbs = w0.nbytes / (call_us * 1e-6) / 1e9
    return {"workload": "single_qgemv_m1_int4_3072x1024", "dtype": "f32", "weight_bytes": w0.nbytes,
            "us_per_call": round(call_us, 3), "gbs": round(gbs, 1),
            "single_call_latency_us": round(statistics.median(lat), 3),
            "calls_in_graph": copies, "launches_per_call": launches / copies,
            "timing": f"CUDA graph of {copies} calls rotating over {copies} copies "
                      f"({copies * w0.nbytes / 1e6:.0f} MB > 2x L2), after an L2 flush, median of 3; "
                      "single call: median of 7, each after an L2 flush",
            "roofline": roofline(gbs, peaks["hbm_gbs"], "GB/s", "hbm", peak_kind)}


def run_lm_head(device, peaks, peak_kind, bits, reps=20):
    """Configuration 3: qgemv on the lm_head [151936x1024] at M = 1: one 165 MB (int8) launch,
    the kernel alone; two packed copies alternate so that every launch streams from HBM."""
    import weight_only_bit_qgemv_b200 as woq

    n, k = workloads.LM_HEAD
    w0 = woq.pack(workloads.weight(n, k, seed=workloads.LM_HEAD_SEED), bits, device)
    w1 = woq.PackedWeight(w0.packed.clone(), w0.scales.clone(), bits, n, k)
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
    out = {"workload": f"lm_head_m1_int{bits}", "dtype": "f32", "weight_bytes": w0.nbytes,
           "launch_us_median": round(med * 1e3, 3), "gbs": round(gbs, 1),
           "timing": f"median of {reps} single launches, CUDA events, two alternating copies",
           "roofline": roofline(gbs, peaks["hbm_gbs"], "GB/s", "hbm", peak_kind,
                                traffic=measured_traffic(f"lm_head_m1_int{bits}"))}
    if bits == 8:
        # The fused greedy pick over the same weights (zero keys, GEMV with argmax, finish):
        # no logits written. Timed as a decode loop runs it: calls captured in a CUDA graph
        # (programmatic dependent launch between the three kernels), replayed.
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
        out["greedy_argmax"] = {"call_us": round(amed * 1e3, 2),
                                "gbs": round(w0.nbytes / (amed / 1e3) / 1e9, 1),
                                "launches_per_call": 3,
                                "timing": f"{reps} calls replayed from one CUDA graph, CUDA events"}
    return out


def run_prefill(layers, groups, device, m: int, peaks, peak_kind, stream, world, flush,
                lm_head=None):
    """tcgen05 qgemm through every projection of every block at M = m (one pass), plus the
    int8 lm_head if given. Median of 3 passes, each replayed from a CUDA graph after an L2
    flush."""
    import weight_only_bit_qgemv_b200 as woq

    Xs = [workloads.activations(m, group_shape(mem)[1], seed=group_x_seed(mem)).to(device)
          for _, mem in groups]
    Ys = [torch.empty(m, group_shape(mem)[0], device=device) for _, mem in groups]
    ws_need = [woq.qgemm_workspace_bytes(m, w, "bf16_tc") for w in layers[0]]
    flops = block_flops(m) * len(layers)
    if lm_head is not None:
        X_lm = workloads.activations(m, lm_head.k, seed=workloads.X_SEED).to(device)
        Y_lm = torch.empty(m, lm_head.n, device=device)
        ws_need.append(woq.qgemm_workspace_bytes(m, lm_head, "bf16_tc"))
        flops += 2.0 * m * lm_head.n * lm_head.k
    ws = torch.empty(max(ws_need), dtype=torch.uint8, device=device)

    def pass_(i):
        for layer in layers:
            for g, w in enumerate(layer):
                woq.qgemm(Xs[g], w, path="bf16_tc", out=Ys[g], workspace=ws)
        if lm_head is not None:
            woq.qgemm(X_lm, lm_head, path="bf16_tc", out=Y_lm, workspace=ws)

    ms, launches = time_graph_median(pass_, 1, stream, world, flush)
    tflops = flops / (ms / 1e3) / 1e12
    calls = len(layers) * len(groups) + (1 if lm_head is not None else 0)
    return {"workload": f"prefill_m{m}" + ("_plus_lm_head" if lm_head is not None else ""),
            "dtype": "bf16 operands, f32 accumulate", "m": m, "gemm_calls_per_pass": calls,
            "flop_per_pass": flops, "ms_per_pass": round(ms, 4), "tflops": round(tflops, 1),
            "launches_per_pass": int(launches),
            "timing": "one pass replayed from a CUDA graph after an L2 flush, median of 3",
            "roofline": roofline(tflops, peaks["bf16_tflops"], "TFLOP/s", "tensor", peak_kind,
                                 peak_note="bf16 burst (kernel timed alone)")}


def run_batched_decode(layers, groups, device, m: int, peaks, peak_kind, stream, world, flush,
                       lm_head=None):
    """Batched decode: m activation rows through every fused projection of every block via
    qgemm's automatic path (the FP32-accurate split tensor-core GEMM for 16 <= m < 128), then
    the int8 lm_head if given. One decoder step = 28 blocks (+ lm_head), replayed from a CUDA
    graph after an L2 flush, median of 3."""
    import weight_only_bit_qgemv_b200 as woq

    xs = [workloads.activations(m, group_shape(mem)[1], seed=group_x_seed(mem)).to(device)
          for _, mem in groups]
    ys = [torch.empty(m, group_shape(mem)[0], device=device) for _, mem in groups]
    need = [woq.qgemm_workspace_bytes(m, w, "auto") for w in layers[0]]
    if lm_head is not None:
        x_lm = workloads.activations(m, lm_head.k, seed=workloads.X_SEED).to(device)
        y_lm = torch.empty(m, lm_head.n, device=device)
        need.append(woq.qgemm_workspace_bytes(m, lm_head, "auto"))
    ws = torch.empty(max(max(need), 256), dtype=torch.uint8, device=device)

    def blocks_only(i):
        for g, w in enumerate(layers[i % len(layers)]):
            woq.qgemm(xs[g], w, path="auto", out=ys[g], workspace=ws)

    ms_blocks, launches_blocks = time_graph_median(blocks_only, len(layers), stream, world, flush)
    us_block = ms_blocks * 1e3 / len(layers)
    step_bytes = decode_step_bytes(layers[0])
    block_gbs = step_bytes / (us_block * 1e-6) / 1e9
    path = "split_tc" if 16 <= m < 128 else ("bf16_tc" if m >= 128 else "fp32")
    out = {"workload": f"decoder_m{m}" + ("_plus_lm_head" if lm_head is not None else ""),
           "dtype": "f32 (split tensor-core form: bf16 hi+lo operands, f32 accumulate)"
                    if path == "split_tc" else "f32",
           "m": m, "qgemm_path": path, "us_per_block": round(us_block, 2),
           "launches_per_block": launches_blocks / len(layers),
           "block_weight_gbs": round(block_gbs, 1),
           "block_algorithmic_tflops": round(block_flops(m) / (us_block * 1e-6) / 1e12, 2)}
    total_bytes = step_bytes * len(layers)
    total_us = us_block * len(layers)
    if lm_head is not None:
        def lm(i):
            woq.qgemm(x_lm, lm_head, path="auto", out=y_lm, workspace=ws)

        ms_lm, _ = time_graph_median(lm, 1, stream, world, flush)
        out["lm_head_us"] = round(ms_lm * 1e3, 2)
        out["lm_head_gbs"] = round(lm_head.nbytes / (ms_lm * 1e-3) / 1e9, 1)
        total_bytes += lm_head.nbytes
        total_us += ms_lm * 1e3
    gbs = total_bytes / (total_us * 1e-6) / 1e9
    out.update({"decoder_step_us": round(total_us, 1),
                "tokens_per_s": round(m * 1e6 / total_us, 1),
                "weight_gbs": round(gbs, 1),
                "timing": "blocks: a CUDA graph of the 28 blocks' calls after an L2 flush, median "
                          "of 3; lm_head: one call, same rule",
                "roofline": roofline(gbs, peaks["hbm_gbs"], "GB/s", "hbm", peak_kind)})
    return out


def run_decode_int5(device, peaks, peak_kind, stream, world, flush, steps=280):
    """The headline decode step (4 qgemv calls per block, 28 blocks cycled) with int5 weights:
    0.6875 bytes per weight against int4's 0.5625."""
    import weight_only_bit_qgemv_b200 as woq

    layers = build_decoder(5, device, FUSED_GROUPS)
    xs = [workloads.activations(1, group_shape(mem)[1], seed=group_x_seed(mem)).to(device)
          for _, mem in FUSED_GROUPS]
    ys = [torch.empty(1, group_shape(mem)[0], device=device) for _, mem in FUSED_GROUPS]

    def step(i):
        for g, w in enumerate(layers[i]):
            woq.qgemv(xs[g], w, out=ys[g])

    ms, per_step = time_graph_steps(step, len(layers), steps, 28, stream, world, flush)
    step_bytes = decode_step_bytes(layers[0])
    gbs = step_bytes * steps / (ms / 1e3) / 1e9
    return {"workload": "decoder_block_m1_int5", "dtype": "f32", "bits": 5,
            "weight_bytes_per_step": step_bytes, "us_per_step": round(ms * 1e3 / steps, 3),
            "gbs": round(gbs, 1), "launches_per_step": per_step,
            "timing": f"{steps} steps from CUDA graphs after an L2 flush, 28 blocks cycled",
            "roofline": roofline(gbs, peaks["hbm_gbs"], "GB/s", "hbm", peak_kind)}


def run_fused_epilogues(layers, groups, device, stream, world, flush):
    """The decode-step projections whose neighbours fuse: gate|up with the SwiGLU
    (qgemv_swiglu, the gate|up outputs never written) and down with the residual add
    (qgemv_residual, in place on the hidden state), each against the plain qgemv of the same
    weights; M = 1, all 28 blocks cycled. Timing only: the decode step's gate|up matrix is
    packed as gate rows then up rows, not interleaved, which changes which rows pair up but
    not the work."""
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
    nl = len(layers)

    def timed(fn):
        ms, launches = time_graph_median(fn, nl, stream, world, flush)
        return ms * 1e3 / nl, launches / nl

    out = {"m": 1}
    for key, plain, fused, idx in (
        ("swiglu_gate_up", lambda i: woq.qgemv(x_gu, layers[i % nl][gu], out=y_gu),
         lambda i: woq.qgemv_swiglu(x_gu, layers[i % nl][gu], out=y_sw), gu),
        ("residual_down", lambda i: woq.qgemv(x_dn, layers[i % nl][dn], out=y_dn),
         lambda i: woq.qgemv_residual(x_dn, layers[i % nl][dn], h, out=h), dn),
    ):
        nbytes = layers[0][idx].nbytes
        us_plain, _ = timed(plain)
        us_fused, launches = timed(fused)
        out[key] = {"shape": f"[{layers[0][idx].n}x{layers[0][idx].k}]", "us_per_call": round(us_fused, 3),
                    "plain_qgemv_us": round(us_plain, 3), "launches_per_call": launches,
                    "weight_gbs": round(nbytes / (us_fused * 1e-6) / 1e9, 1)}
    return out


# --------------------------------------------------------------------------------------
# CPU oracle (cpu_baseline legs and the reference arm)
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


def oracle_pack(W: np.ndarray, bits: int):
    """(packed, scale bits, bits) of a float32 weight, quantised and packed by the oracle."""
    import oracle

    q, s = oracle.quantise(W, bits)
    return oracle.pack(q, bits), s, bits


def oracle_layer_inputs(groups, bits=4, layer=0, m=1):
    """The block's 7 projections, quantised and packed by the oracle itself, and their x rows
    (members of a launch group share its input)."""
    x_of = {}
    for _, mem in groups:
        x = workloads.activations(m, group_shape(mem)[1], seed=group_x_seed(mem)).numpy()
        for i in mem:
            x_of[i] = x
    out = []
    for p, (_, n, k) in enumerate(workloads.DECODER_PROJ):
        W = workloads.weight(n, k, seed=workloads.layer_seed(layer, p)).numpy()
        out.append(oracle_pack(W, bits))
    return out, [x_of[p] for p in range(len(workloads.DECODER_PROJ))]


def oracle_chain_block0():
    """Block 0's chain matrices packed by the oracle: qkv (rows of q, k, v), o, gate|up with
    rows interleaved, down."""
    W = [workloads.weight(n, k, seed=workloads.layer_seed(0, i)).numpy()
         for i, (_, n, k) in enumerate(workloads.DECODER_PROJ)]
    gu = np.stack([W[4], W[5]], axis=1).reshape(6144, 1024)
    return [oracle_pack(w, 4)[:2] for w in (np.concatenate(W[0:3], 0), W[3], gu, W[6])]


def all_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_cpu(fn, threads: int, runs: int = 3):
    """Median seconds of fn() with BLAS limited to `threads` threads: one discarded run, then
    the median of `runs`. Returns (seconds, threads actually used, last result)."""
    from threadpoolctl import threadpool_limits

    with threadpool_limits(limits=threads, user_api="blas"):
        used = blas_threads()
        res = fn()
        ts = []
        for _ in range(runs):
            t0 = time.perf_counter()
            res = fn()
            ts.append(time.perf_counter() - t0)
    return statistics.median(ts), used, res


def cpu_baseline(fn, work: float, unit: str, scale: float, sample: str):
    """The oracle timed on all host cores and on one core. `work` units per run (bytes or
    FLOP), reported in `unit` after dividing by `scale` (1e9 for GB/s, 1e12 for TFLOP/s)."""
    n_all = all_cores()
    sec_all, used_all, res = time_cpu(fn, n_all)
    sec_one, used_one, _ = time_cpu(fn, 1)
    return ({"value": round(work / sec_all / scale, 5), "unit": unit, "cores": used_all,
             "kind": "oracle", "sample": sample,
             "seconds_per_run": round(sec_all, 4),
             "one_core": {"value": round(work / sec_one / scale, 5), "cores": used_one,
                          "seconds_per_run": round(sec_one, 4)},
             "timing": "one discarded run, then the median of 3 (all cores in the affinity set, "
                       "then BLAS limited to one thread)"}, res)


def cpu_legs(groups, layer0_gpu, xs_gpu):
    """The oracle as it stands on the host cores, one bounded sample per configuration; also the
    parity of the headline GPU step against the oracle's outputs (block 0)."""
    import oracle
    import weight_only_bit_qgemv_b200 as woq

    legs = {}
    # configuration 1: the single qgemv, in full
    n, k = 3072, 1024
    pk1 = oracle_pack(workloads.weight(n, k, seed=0).numpy(), 4)
    x1 = workloads.activations(1, k, seed=0).numpy()
    b1 = pk1[0].nbytes + pk1[1].nbytes
    legs["single_qgemv_m1"], _ = cpu_baseline(
        lambda: oracle.qgemv_ref(x1, *pk1), b1, "GB/s", 1e9,
        "the whole [3072x1024] int4 qgemv at M=1 through the NumPy float64 oracle")
    # configuration 2: decoder block 0, in full (and parity of the GPU step)
    packed, xs = oracle_layer_inputs(groups)
    nbytes = sum(pk.nbytes + sc.nbytes for pk, sc, _ in packed)
    legs["decoder_block_m1"], outs = cpu_baseline(
        lambda: oracle_decode_pass(packed, xs), nbytes, "GB/s", 1e9,
        "decoder block 0 (7 projections, M=1, int4) through the NumPy float64 oracle")
    errs = []
    for g, (w, (_, mem)) in enumerate(zip(layer0_gpu, groups)):
        y = woq.qgemv(xs_gpu[g], w).cpu().numpy()
        ref = np.concatenate([outs[i] for i in mem], axis=1)
        errs.append(float(np.max(np.abs(y - ref)) / np.max(np.abs(ref))))
    parity = {"max_rel_err": max(errs), "tolerance": 1e-4, "checked": "block 0, every output"}
    # configuration 3: lm_head int8, the first 8192 of its 151936 rows
    rows = 8192
    n, k = workloads.LM_HEAD
    W = workloads.weight(n, k, seed=workloads.LM_HEAD_SEED)[:rows].numpy()
    pk3 = oracle_pack(W, 8)
    x3 = workloads.activations(1, k, seed=workloads.X_SEED).numpy()
    legs["lm_head_m1_int8"], _ = cpu_baseline(
        lambda: oracle.qgemv_ref(x3, *pk3), pk3[0].nbytes + pk3[1].nbytes, "GB/s", 1e9,
        f"rows 0..{rows - 1} of the int8 lm_head [151936x1024] at M=1 (the rate is per byte, "
        "so it stands for the whole matrix)")
    # the same lm_head sample as int4 and int5, and decoder block 0 as int5
    for bits in (4, 5):
        pkb = oracle_pack(W, bits)
        legs[f"lm_head_m1_int{bits}"], _ = cpu_baseline(
            lambda pkb=pkb: oracle.qgemv_ref(x3, *pkb), pkb[0].nbytes + pkb[1].nbytes, "GB/s", 1e9,
            f"rows 0..{rows - 1} of the int{bits} lm_head [151936x1024] at M=1 (the rate is per "
            "byte, so it stands for the whole matrix)")
    packed5, xs5 = oracle_layer_inputs(groups, bits=5)
    legs["decoder_block_m1_int5"], _ = cpu_baseline(
        lambda: oracle_decode_pass(packed5, xs5), sum(pk.nbytes + sc.nbytes for pk, sc, _ in packed5),
        "GB/s", 1e9, "decoder block 0 (7 projections, M=1, int5) through the NumPy float64 oracle")
    # configuration 4: prefill M=512, block 0's 7 projections (1/28 of a pass)
    packed512, xs512 = oracle_layer_inputs(groups, m=512)
    legs["prefill_m512"], _ = cpu_baseline(
        lambda: oracle_decode_pass(packed512, xs512), block_flops(512), "TFLOP/s", 1e12,
        "decoder block 0's 7 projections at M=512 (1/28 of the pass; a rate, so it stands for "
        "the pass)")
    # configuration 5: batched decode M=64 (block 0) and prefill M=4096 (block 0's q projection)
    packed64, xs64 = oracle_layer_inputs(groups, m=64)
    legs["decoder_m64"], _ = cpu_baseline(
        lambda: oracle_decode_pass(packed64, xs64), nbytes, "GB/s", 1e9,
        "decoder block 0's 7 projections at M=64 (weight bytes per second; a rate, so it stands "
        "for the 28 blocks)")
    q0 = packed[0]
    x4096 = workloads.activations(4096, 1024, seed=workloads.X_SEED).numpy()
    legs["prefill_m4096"], _ = cpu_baseline(
        lambda: oracle.qgemv_ref(x4096, *q0), 2.0 * 4096 * 2048 * 1024, "TFLOP/s", 1e12,
        "block 0's q projection [2048x1024] at M=4096 (a rate, so it stands for the pass)")
    return legs, parity


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
    return {"impl": "reference", "metric": METRIC,
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
    ap.add_argument("--steps", type=int, default=2800)
    ap.add_argument("--warmup", type=int, default=280)
    ap.add_argument("--impl", default="woq", choices=["woq", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true", help="7 launches per block instead of 4")
    ap.add_argument("--decode-step", default="best", choices=["best", "chain", "calls"],
                    help="headline decode step: one qgemv_chain launch, 4 qgemv calls, or the faster")
    ap.add_argument("--m", type=int, default=1, help="activation rows per decode step (1..64)")
    ap.add_argument("--no-lm-head", action="store_true")
    ap.add_argument("--no-fused-epilogues", action="store_true")
    ap.add_argument("--no-batched", action="store_true", help="skip the M=64 / M=4096 legs")
    ap.add_argument("--legs", default="all",
                    help="comma list of legs to run (the headline decode always runs): chain, int5, "
                         "single, lm_head, prefill, batched, epilogues, cpu; default all")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    legs = {"chain", "int5", "single", "lm_head", "prefill", "batched", "epilogues", "cpu"}
    if args.legs != "all":
        want = {x.strip() for x in args.legs.split(",") if x.strip()}
        if not want <= legs | {"decode"}:
            ap.error(f"--legs takes {sorted(legs)}")
        legs = want
    args.no_prefill = args.no_prefill or "prefill" not in legs
    args.no_lm_head = args.no_lm_head or "lm_head" not in legs
    args.no_batched = args.no_batched or "batched" not in legs
    args.no_fused_epilogues = args.no_fused_epilogues or "epilogues" not in legs
    args.no_cpu_baseline = args.no_cpu_baseline or "cpu" not in legs
    world, rank, local = dist_setup()
    if args.impl == "reference":
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0

    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    import weight_only_bit_qgemv_b200 as woq

    peaks, peak_kind = load_peaks()
    device = torch.device("cuda", local)
    flush = L2Flush(device)
    stream = torch.cuda.Stream(device)
    nvtx = torch.cuda.nvtx
    nvtx.range_push("decode")
    out, layers, groups, xs = run_decode(args, world, local, peaks, peak_kind, flush)
    nvtx.range_pop()
    configs = {}
    chain_step = None
    if not args.unfused and args.m <= 8 and "chain" in legs:
        nvtx.range_push("chain")
        ch, clayers, chain_step = run_decode_chain(args, world, local, peaks, peak_kind, flush, layers)
        nvtx.range_pop()
        calls = {k: out[k] for k in ("value", "ms_per_step", "config", "hbm_frac", "clocks", "e2e",
                                     "gpu_launches", "roofline", "per_kernel")}
        if args.decode_step == "chain" or (args.decode_step == "best" and ch["value"] > out["value"]):
            out.update(ch)
            configs["decoder_block_m1_separate_calls"] = dict(calls, dtype="f32",
                                                              note="the same block as 4 qgemv calls")
        else:
            configs["decoder_block_m1_chain"] = dict(ch, dtype="f32",
                                                     note="the same block as one qgemv_chain launch")
    configs["decoder_block_m1"] = {"workload": out["config"]["workload"], "dtype": "f32",
                                   "gbs": out["value"], "us_per_step": round(out["ms_per_step"] * 1e3, 3),
                                   "roofline": out["roofline"], "note": "the headline line itself"}
    if "single" in legs:
        nvtx.range_push("single_qgemv_m1")
        configs["single_qgemv_m1"] = run_single_qgemv(device, peaks, peak_kind, stream, world, flush)
        nvtx.range_pop()
    lm8 = None
    if not args.no_lm_head:
        for bits in (8, 4, 5):
            nvtx.range_push(f"lm_head_m1_int{bits}")
            configs[f"lm_head_m1_int{bits}"] = run_lm_head(device, peaks, peak_kind, bits)
            nvtx.range_pop()
    if not args.no_batched:
        n, k = workloads.LM_HEAD
        lm8 = woq.pack(workloads.weight(n, k, seed=workloads.LM_HEAD_SEED), 8, device)
    if not args.no_prefill:
        nvtx.range_push("prefill_m512")
        configs["prefill_m512"] = run_prefill(layers, groups, device, 512, peaks, peak_kind,
                                              stream, world, flush)
        nvtx.range_pop()
    if not args.no_batched:
        nvtx.range_push("decoder_m64_plus_lm_head")
        configs["decoder_m64_plus_lm_head"] = run_batched_decode(
            layers, groups, device, 64, peaks, peak_kind, stream, world, flush, lm_head=lm8)
        nvtx.range_pop()
        if not args.no_prefill:
            nvtx.range_push("prefill_m4096_plus_lm_head")
            configs["prefill_m4096_plus_lm_head"] = run_prefill(
                layers, groups, device, 4096, peaks, peak_kind, stream, world, flush, lm_head=lm8)
            nvtx.range_pop()
    if args.m == 1 and not args.unfused and "int5" in legs:
        nvtx.range_push("decoder_block_m1_int5")
        configs["decoder_block_m1_int5"] = run_decode_int5(device, peaks, peak_kind, stream, world, flush)
        nvtx.range_pop()
    if not args.no_fused_epilogues:
        nvtx.range_push("fused_epilogues")
        fe = run_fused_epilogues(layers, groups, device, stream, world, flush)
        nvtx.range_pop()
        if fe is not None:
            out["fused_epilogues"] = fe
    if rank == 0 and not args.no_cpu_baseline and args.m == 1 and not args.unfused:
        cpu, parity = cpu_legs(groups, layers[0], xs)
        out["cpu_baseline"] = cpu.pop("decoder_block_m1")
        out["parity"] = parity
        if chain_step is not None:
            out["parity_chain"] = chain_parity(chain_step, oracle_chain_block0())
        configs["decoder_block_m1"]["cpu_baseline"] = out["cpu_baseline"]
        key_of = {"single_qgemv_m1": "single_qgemv_m1", "lm_head_m1_int8": "lm_head_m1_int8",
                  "lm_head_m1_int4": "lm_head_m1_int4", "lm_head_m1_int5": "lm_head_m1_int5",
                  "decoder_block_m1_int5": "decoder_block_m1_int5",
                  "prefill_m512": "prefill_m512", "decoder_m64": "decoder_m64_plus_lm_head",
                  "prefill_m4096": "prefill_m4096_plus_lm_head"}
        for leg, cfg in key_of.items():
            if cfg in configs:
                configs[cfg]["cpu_baseline"] = cpu[leg]
    out["configs"] = configs
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
