"""Benchmark of the ParoQuant runtime hot path on B200 (one JSON line on rank 0).

Default workload: one Qwen2.5-1.5B-shaped decoder layer at decode (M = 1):
the seven linears q, k, v, o, gate, up, down, each preceded by its own K = 8
stage pairwise-rotation transform (group-128 asymmetric INT4 weights).  One
step = the seven fused rotate+INT4 linears of one layer.  Steps cycle over 28
distinct layers (0.70 GB of packed weights, several times the 126 MB L2), so
every step streams its weights from HBM.

value     = algorithmic HBM bytes of the step / step time  (GB/s, device clock)
e2e       = the same with the per-step host->device copy of the inputs (pinned)
            and device->host copy of the outputs inside the timed region
roofline  = the INT4 linear kernel alone, algorithmic bytes / its time, against
            the measured HBM copy bandwidth
cpu_baseline = the fp64 CPU oracle on a bounded sample of the same workload

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1..4] [--impl ours|reference]
Multi-GPU (torchrun): every rank runs its own layers (weak scaling, no data-path
collective); the time is the max over ranks.
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

from synth import LAYER_SHAPES, device_weights, linear_problem  # noqa: E402

METRIC = "rot+W4 linear: decode HBM GB/s (% peak), prefill TFLOP/s, rotation overhead %"

# DRAM bytes (read + write) per launch of the kernel the roofline times, from
# one ncu capture of `bench.py --profile --variants batched_plain --config N`
# (metrics dram__bytes_read.sum, dram__bytes_write.sum; the first launch after
# four skipped), with the sha256 prefix
# of the kernel's sources at capture time: once the sources change, the figure
# no longer describes the kernel and the bench reports null.
TRAFFIC = {
    1: {"bytes": 24964608, "src": ("w4_stream.cu", "w4_stream.cuh"), "sha": "2cbfd0012327d0d7"},
    2: {"bytes": 131985408 + 3412992, "src": ("w4_stream.cu", "w4_stream.cuh"), "sha": "2cbfd0012327d0d7"},
    3: {"bytes": 346587136 + 137527040, "src": ("w4_tc.cu", "w4_tc.cuh"), "sha": "a093d18620409e5a"},
    4: {"bytes": 25542400, "src": ("w4_stream.cu", "w4_stream.cuh"), "sha": "2cbfd0012327d0d7"},
}


def measured_traffic(config, M):
    """The captured DRAM bytes per launch of this config's timed kernel, or None
    when the workload is not the captured one or the kernel changed since."""
    import hashlib
    t = TRAFFIC.get(config)
    if t is None or M is not None:
        return None
    h = hashlib.sha256()
    for f in t["src"]:
        with open(os.path.join(ROOT, "rotation_int4_weight_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return t["bytes"] if h.hexdigest()[:16] == t["sha"] else None
K_STAGES = 8
GROUP = 128
PREFILL_M = 512                          # from this many tokens on the metric is TFLOP/s
TABLE_BYTES_PER_CH = K_STAGES * 6 + 4   # pairs 4 B + cos/sin 8 B per pair per stage, + fp32 scale


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0)) or None, "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------- workloads
def workload(config: int, M: int | None):
    """(name, shapes, M, layers cycled, steps_are_whole_stack)"""
    if config == 0:
        return "tiny 512x512 layer", LAYER_SHAPES["tiny"], M or 4, 1, False
    if config == 1:
        return "qwen2.5-1.5b decoder layer, 7 linears", LAYER_SHAPES["qwen2.5-1.5b"], M or 1, 28, False
    if config == 2:
        return "llama-3-8b decoder layer, 7 linears", LAYER_SHAPES["llama-3-8b"], M or 1, 8, False
    if config == 3:
        return "llama-3-8b decoder layer, 7 linears, prefill", LAYER_SHAPES["llama-3-8b"], M or 2048, 1, False
    if config == 4:
        return "qwen2.5-1.5b 28-layer linear stack (196 linears)", LAYER_SHAPES["qwen2.5-1.5b"], M or 16, 28, True
    raise SystemExit(f"unknown config {config}")


def linear_bytes(d_in, d_out, M, rotate=True, unfused=False):
    b = d_in * d_out // 2 + 4 * d_out * (d_in // GROUP) + 2 * M * d_in + 2 * M * d_out
    if rotate:
        b += TABLE_BYTES_PER_CH * d_in
    if unfused:
        b += 4 * M * d_in
    return b


class Linear:
    """Device tensors of one linear layer: tables, packed weights (rotated and plain), x, y."""

    def __init__(self, p, dev, plan=True):
        import torch
        import rotation_int4_weight_b200 as paro
        self.d_in, self.d_out, self.M = p.d_in, p.d_out, p.M
        pairs, cos_t, sin_t = p.pairs, p.cos_t, p.sin_t
        if plan and p.d_in % 64 == 0:  # load-time: conflict-free order of the pairs (same transform)
            pairs, cos_t, sin_t = paro.paro_plan_pair_order(pairs, cos_t, sin_t)
        self.pairs = torch.from_numpy(pairs.view(np.int16)).to(dev)
        self.cos = torch.from_numpy(cos_t).to(dev)
        self.sin = torch.from_numpy(sin_t).to(dev)
        self.scale = torch.from_numpy(p.scale).to(dev)
        W = device_weights(p, dev)
        ws = torch.empty_like(W)
        self.qw, self.sc, self.z = paro.paro_pack_weights(W, self.pairs, self.cos, self.sin, self.scale, workspace=ws)
        self.qw0, self.sc0, self.z0 = paro.paro_pack_weights(W)
        del W, ws
        self.x = torch.from_numpy(p.x).to(dev).to(torch.bfloat16)
        self.xr = torch.empty_like(self.x)
        self.y = torch.empty(p.M, p.d_out, dtype=torch.bfloat16, device=dev)
        self.ws = torch.empty(max(paro.paro_workspace_bytes(p.M, p.d_in), 256), dtype=torch.uint8, device=dev)
        self.x_host = torch.empty(self.x.shape, dtype=torch.bfloat16, pin_memory=True)
        self.x_host.copy_(self.x)
        self.y_host = torch.empty(self.y.shape, dtype=torch.bfloat16, pin_memory=True)

    # each call below is one public C-ABI call
    def fused(self, paro):
        paro.paro_rotate_w4_linear(self.x, self.pairs, self.cos, self.sin, self.scale, self.qw, self.sc, self.z,
                                   out=self.y, workspace=self.ws)

    def unfused(self, paro):
        paro.paro_rotate(self.x, self.pairs, self.cos, self.sin, self.scale, out=self.xr)
        paro.paro_w4_linear(self.xr, self.qw, self.sc, self.z, out=self.y)

    def plain(self, paro):
        # the same INT4 linear without a transform; with many tokens the fused
        # call with K = 0 (the transform kernel then only rounds x to fp16, the
        # input format of the tensor-core kernel), with few the plain call
        if self.M > 64:
            paro.paro_rotate_w4_linear(self.x, None, None, None, None, self.qw0, self.sc0, self.z0, out=self.y,
                                       workspace=self.ws)
        else:
            paro.paro_w4_linear(self.x, self.qw0, self.sc0, self.z0, out=self.y)

    def rotate(self, paro):
        paro.paro_rotate(self.x, self.pairs, self.cos, self.sin, self.scale, out=self.xr)

    def rotate_backward(self, paro):
        # gradients of the transform for a synthetic upstream gradient (the
        # calibration-time step; buffers made on first use)
        import torch
        if getattr(self, "grad", None) is None:
            g = torch.Generator(device=self.x.device)
            g.manual_seed(self.d_in * 7 + self.d_out)
            self.grad = torch.randn(self.x.shape, generator=g, dtype=torch.float32, device=self.x.device)
            need = paro.lib.paro_rotate_backward_workspace_bytes(self.M, self.d_in, self.pairs.shape[0], 1)
            self.bws = torch.empty(max(need, 16), dtype=torch.uint8, device=self.x.device)
        paro.paro_rotate_backward(self.x, self.grad, self.pairs, self.cos, self.sin, self.scale, workspace=self.bws)

    def fused_e2e(self, paro):
        self.x.copy_(self.x_host, non_blocking=True)
        self.fused(paro)
        self.y_host.copy_(self.y, non_blocking=True)


# kernels launched per linear of each variant (batched: 2 per call of up to 7 linears)
LAUNCHES = {"fused": 2, "unfused": 2, "plain": 1, "rotate": 1, "fused_e2e": 2,  # plain: 2 when M > 64
            "rotate_backward": 2}
BATCH = 7  # linears per batched call (one decoder layer)


class Unit:
    """The linears of one step; runs them per linear or as batched calls."""

    def __init__(self, lins, paro):
        import torch
        self.lins = lins
        # the step's inputs and outputs live in one contiguous device buffer each
        # (every linear's x and y are views into them), so the end-to-end variant
        # moves them with one host->device and one device->host copy per step
        dev = lins[0].x.device
        self.x_all = torch.empty(sum(l.x.numel() for l in lins), dtype=torch.bfloat16, device=dev)
        self.y_all = torch.empty(sum(l.y.numel() for l in lins), dtype=torch.bfloat16, device=dev)
        ox = oy = 0
        for l in lins:
            nx, ny = l.x.numel(), l.y.numel()
            vx = self.x_all[ox:ox + nx].view(l.x.shape)
            vx.copy_(l.x)
            l.x = vx
            l.y = self.y_all[oy:oy + ny].view(l.y.shape)
            ox += nx
            oy += ny
        self.x_host = torch.empty(self.x_all.shape, dtype=torch.bfloat16, pin_memory=True)
        self.x_host.copy_(self.x_all)
        self.y_host = torch.empty(self.y_all.shape, dtype=torch.bfloat16, pin_memory=True)
        self.calls = []
        for i in range(0, len(lins), BATCH):
            grp = lins[i:i + BATCH]
            descs = [paro.paro_linear(l.x, l.pairs, l.cos, l.sin, l.scale, l.qw, l.sc, l.z, l.y) for l in grp]
            plain = [paro.paro_linear(l.x, None, None, None, None, l.qw0, l.sc0, l.z0, l.y) for l in grp]
            need = paro.paro_batched_workspace_bytes(descs)
            ws = __import__("torch").empty(max(need, 256), dtype=__import__("torch").uint8, device=lins[0].x.device)
            self.calls.append((grp, descs, plain, ws))

    def run(self, paro, variant):
        if variant in ("batched", "batched_e2e", "batched_plain"):
            if variant == "batched_e2e":
                self.x_all.copy_(self.x_host, non_blocking=True)
            for grp, descs, plain, ws in self.calls:
                paro.paro_rotate_w4_linear_batched(plain if variant == "batched_plain" else descs, workspace=ws)
            if variant == "batched_e2e":
                self.y_host.copy_(self.y_all, non_blocking=True)
        else:
            for lin in self.lins:
                getattr(lin, variant)(paro)

    def launches(self, variant):
        if variant == "batched_plain":
            return len(self.calls)
        if variant.startswith("batched"):
            # one token per linear: the transforms run inside the INT4 kernel (one
            # launch per call); otherwise a transform launch and an INT4 launch
            return (1 if all(l.M == 1 for l in self.lins) else 2) * len(self.calls)
        return LAUNCHES[variant] * len(self.lins)


def rank_seed(config, rank):
    """Seed of a rank's inputs: every rank draws its own layers (weak scaling)."""
    return 0x5A17 + config + 1000 * rank


def max_over_ranks(torch, dist, ms, device):
    """The step time of the whole job: the slowest rank's (all ranks call this)."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(per_rank_amount, world, ms):
    """Units all ranks processed per second, each rank doing `per_rank_amount`
    per step in `ms` milliseconds (the max over ranks)."""
    return per_rank_amount * world / (ms * 1e-3)


def build_layers(config, M, n_layers, rank, dev, plan=True):
    name, shapes, M, _, _ = workload(config, M)
    base = rank_seed(config, rank)
    layers = []
    for li in range(n_layers):
        lins = []
        for si, (nm, d_in, d_out) in enumerate(shapes):
            p = linear_problem(base, li * 16 + si, d_in, d_out, M, K_STAGES, GROUP, name=nm, host_weights=False)
            lins.append(Linear(p, dev, plan))
        layers.append(lins)
    return layers


def capture(torch, paro, units, variant):
    """CUDA graphs of a variant: one per unit (a unit = the linears of one step)
    and one that runs every unit once in order (a full cycle), so that the host
    enqueues many steps per replay and never limits the device."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for unit in units:           # warm the launch path outside capture
            unit.run(paro, variant)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    per_unit = []
    for unit in units:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            unit.run(paro, variant)
        per_unit.append(g)
    cycle = None
    if len(units) > 1:
        cycle = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cycle):
            for unit in units:
                unit.run(paro, variant)
    return per_unit, cycle


def _replay(graphs, first, count):
    """Replay `count` steps starting at unit index `first` (mod the number of units)."""
    per_unit, cycle = graphs
    n = len(per_unit)
    i = 0
    while i < count and (first + i) % n != 0:
        per_unit[(first + i) % n].replay()
        i += 1
    while cycle is not None and count - i >= n:
        cycle.replay()
        i += n
    while i < count:
        per_unit[(first + i) % n].replay()
        i += 1


def time_graphs(torch, graphs, steps, warmup, dist=None):
    """Run `warmup` untimed steps, then time exactly `steps` steps on the device
    (CUDA events on the launching stream, barrier + synchronize on both sides).
    Returns ms per step, the max over ranks."""
    _replay(graphs, 0, warmup)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record()
    _replay(graphs, warmup, steps)
    end.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(torch, dist, start.elapsed_time(end) / steps, "cuda")
    if dist is not None:
        dist.barrier()
    return ms


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while the timed region runs."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index  # nvidia-smi -i accepts an index, a UUID or a PCI bus id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
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
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def _smi_id(torch):
    try:
        u = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(torch.cuda.current_device())


# ----------------------------------------------------------------------------- CPU oracle baseline
def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        return 1


def oracle_problems(config, M):
    """The linears of one unit of the workload, packed by the oracle (untimed build step).
    Rows of M beyond 64 are dropped (bytes are counted for the rows run)."""
    import oracle
    name, shapes, M, _, _ = workload(config, M)
    sub_m = min(M, 64)
    probs = []
    for si, (nm, d_in, d_out) in enumerate(shapes):
        p = linear_problem(0x5A17 + config, si, d_in, d_out, sub_m, K_STAGES, GROUP, name=nm, host_weights=True)
        qw, sc, z = oracle.pack_weights(p.W, None, None, None, None)  # code values do not change the timing
        probs.append((p, qw, sc, z))
    return probs, sub_m, M


def oracle_run(probs, idx, rows=None):
    """One oracle linear of the unit (cycling), on its first `rows` output rows
    (all when None): returns (seconds, algorithmic bytes of the rows run)."""
    import oracle
    p, qw, sc, z = probs[idx % len(probs)]
    r = p.d_out if rows is None else max(1, min(rows[idx % len(probs)], p.d_out))
    t0 = time.perf_counter()
    oracle.rotate_w4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale, qw[:r], sc[:r], z[:r])
    return time.perf_counter() - t0, linear_bytes(p.d_in, r, p.M)


def _oracle_passes(probs, seconds):
    tot_t, tot_b, reps = 0.0, 0, 0
    while tot_t < seconds or reps == 0:
        for i in range(len(probs)):
            t, b = oracle_run(probs, i)
            tot_t += t
            tot_b += b
        reps += 1
    return tot_b / tot_t / 1e9, reps, tot_t


def oracle_sample(config, M, seconds=12.0, one_core_seconds=None):
    """Time the fp64 CPU oracle over whole passes of one unit's linears for about
    `seconds` on all host threads; returns (GB/s, threads, description, one-core
    figure).  With one_core_seconds, the same passes are timed again with the
    numeric libraries held to one thread: (GB/s, description), else None."""
    probs, sub_m, M = oracle_problems(config, M)
    gbs, reps, tot_t = _oracle_passes(probs, seconds)
    unit = (f" over the {len(probs)} linears of one unit at M={sub_m}"
            + (f" (workload M={M}; bytes counted for M={sub_m})" if sub_m != M else ""))
    sample = f"{reps} pass(es){unit}, {tot_t:.1f} s"
    one = None
    if one_core_seconds is not None:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            gbs1, reps1, t1 = _oracle_passes(probs, one_core_seconds)
        one = (gbs1, f"{reps1} pass(es){unit}, one thread, {t1:.1f} s")
    return gbs, _oracle_threads(), sample, one


def reference_rows(probs, steps, warmup, seconds=60.0):
    """Output rows per oracle step so that `warmup + steps` steps take about
    `seconds` of CPU time: the cost of a row is measured on one full linear of
    each shape (untimed), rows are a multiple of 16, at least 16."""
    per_step = seconds / max(1, steps + warmup)
    rows = []
    for i, (p, *_rest) in enumerate(probs):
        t_full, _ = oracle_run(probs, i)
        t_row = t_full / p.d_out
        r = int(per_step / t_row) // 16 * 16
        rows.append(max(16, min(p.d_out, r)))
    return rows


def run_reference(args):
    """The reference arm: the CPU oracle, timed as it stands on this host's cores.
    Each step runs one linear of the workload's unit (cycling q, k, v, o, gate,
    up, down) on a bounded sample of its output rows, sized so that the whole
    run takes about a minute; value = bytes of all timed steps / their time.
    Under torchrun only rank 0 runs; the other ranks exit without work."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    name, shapes, M, _, _ = workload(args.config, args.M)
    probs, sub_m, M = oracle_problems(args.config, args.M)
    rows = reference_rows(probs, args.steps, args.warmup)
    for i in range(args.warmup):
        oracle_run(probs, i, rows)
    tot_t, tot_b, tot_f = 0.0, 0, 0
    for i in range(args.steps):
        k = args.warmup + i
        t, b = oracle_run(probs, k, rows)
        p = probs[k % len(probs)][0]
        tot_t += t
        tot_b += b
        tot_f += 2 * p.M * p.d_in * min(rows[k % len(probs)], p.d_out)
    prefill = M >= PREFILL_M
    value = tot_f / tot_t / 1e12 if prefill else tot_b / tot_t / 1e9
    unit = "TFLOP/s" if prefill else "GB/s"
    sample = (f"{args.steps} steps of one linear each (cycling the {len(probs)} linears), M={sub_m}, "
              f"first {rows} output rows of each, {tot_t:.1f} s")
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit, "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot_t / args.steps, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": f"{name}: rotate + INT4 linear, M={M}, K={K_STAGES}, group={GROUP} "
                                  f"(fp64 CPU oracle)"},
           "cpu_baseline": {"kind": "oracle", "value": round(value, 6), "unit": unit, "cores": _oracle_threads(),
                            "sample": sample},
           "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for about half a second of device time)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--M", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--variants", default="batched,batched_plain,fused,plain,unfused,rotate,rotate_backward")
    ap.add_argument("--no-plan", action="store_true",
                    help="use the pair tables as drawn instead of the conflict-free order of paro_plan_pair_order")
    ap.add_argument("--profile", action="store_true",
                    help="run only the listed variants (no end-to-end leg, no CPU baseline): a fixed, short "
                         "launch sequence for ncu; its numbers are not bench values")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.steps is None:
        args.steps = {0: 20000, 1: 56000, 2: 8000, 3: 200, 4: 128}.get(args.config, 1000)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as tdist
        from datetime import timedelta
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        dist = tdist
    else:
        torch.cuda.set_device(0)
    import rotation_int4_weight_b200 as paro
    dev = torch.device("cuda", torch.cuda.current_device())
    hbm, bf16, bf16_sus, peak_kind = peaks()

    name, shapes, M, n_layers, stack = workload(args.config, args.M)
    layers = build_layers(args.config, M, n_layers, rank, dev, plan=not args.no_plan)
    torch.cuda.synchronize()
    units = [Unit(sum(layers, []), paro)] if stack else [Unit(l, paro) for l in layers]
    step_lins = units[0].lins
    flops_step = sum(2 * M * l.d_in * l.d_out for l in step_lins)

    def bytes_of(variant):
        if variant == "plain":
            return sum(linear_bytes(l.d_in, l.d_out, M, rotate=False) for l in step_lins)
        if variant == "rotate":
            return sum(4 * M * l.d_in + TABLE_BYTES_PER_CH * l.d_in for l in step_lins)
        if variant == "rotate_backward":
            # x (bf16) and the upstream gradient in, dx out (fp32), the tables and
            # the outputs dtheta, dscale; the per-block partial sums round trip
            def bwd(l):
                R = 4 if 8 * 4 * l.d_in <= 226 * 1024 else (2 if 8 * 2 * l.d_in <= 226 * 1024 else 1)
                n = K_STAGES * l.d_in // 2 + l.d_in
                return 10 * M * l.d_in + TABLE_BYTES_PER_CH * l.d_in + 4 * n + 2 * 4 * n * -(-M // R)
            return sum(bwd(l) for l in step_lins)
        return sum(linear_bytes(l.d_in, l.d_out, M, unfused=(variant == "unfused")) for l in step_lins)

    variants = [v for v in args.variants.split(",") if v]
    if "batched" not in variants and not args.profile:
        variants.insert(0, "batched")
    results = {}
    clocks = None
    for v in variants:
        graphs = capture(torch, paro, units, v)
        if v == "batched" and not args.profile:
            with ClockSampler(_smi_id(torch)) as cs:
                ms = time_graphs(torch, graphs, args.steps, args.warmup, dist)
            clocks = cs.summary()
        else:
            ms = time_graphs(torch, graphs, args.steps, args.warmup, dist)
        results[v] = ms
        del graphs
    if args.profile:
        if rank == 0:
            print(json.dumps({"profile_run": True, "variants_ms_per_step": results}), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return
    # end to end: per step the inputs come from pinned host memory and outputs go back
    graphs = capture(torch, paro, units, "batched_e2e")
    ms_e2e = time_graphs(torch, graphs, args.steps, args.warmup, dist)
    del graphs
    h2d = units[0].x_all.numel() * 2
    d2h = units[0].y_all.numel() * 2

    ms = results["batched"]
    step_bytes = bytes_of("fused")
    value = whole_job_rate(step_bytes, world, ms) / 1e9
    e2e_value = whole_job_rate(step_bytes + h2d + d2h, world, ms_e2e) / 1e9
    plain_ms = results.get("plain")
    # dominant kernel: the INT4 linear, timed alone (plain weights, no transform:
    # one launch per batched call when that variant ran, else one per linear)
    w4_ms = results.get("batched_plain", plain_ms)
    w4_gbs = bytes_of("plain") / (w4_ms * 1e-3) / 1e9 if w4_ms else None
    # launches of the timed kernel per step (one per batched call), for the
    # per-launch figures next to the captured traffic
    w4_launches = units[0].launches("batched_plain") if "batched_plain" in results else len(step_lins)
    traffic = measured_traffic(args.config, args.M)
    rot_gbs = bytes_of("rotate") / (results["rotate"] * 1e-3) / 1e9 if "rotate" in results else None
    bwd_ms = results.get("rotate_backward")
    prefill = M >= PREFILL_M

    out = {
        "metric": METRIC,
        "value": round(value if not prefill else whole_job_rate(flops_step, world, ms) / 1e12, 3),
        "unit": "GB/s" if not prefill else "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {
            "workload": f"{name}: fused rotate + INT4 linear (one batched C-ABI call per {BATCH} linears), "
                        f"M={M}, K={K_STAGES}, group={GROUP}, asymmetric INT4, bf16 activations",
            "linears_per_step": len(step_lins), "distinct_units_cycled": len(units),
            "l2": ("inputs larger than L2: each step streams a different layer's weights "
                   f"({len(units)} units, {sum(bytes_of('fused') for _ in units) / 1e9:.2f} GB)") if len(units) > 1
                  else "inputs larger than L2 per step" if step_bytes > 126e6 else "L2-resident (single unit)",
            "graphs": "each step is one CUDA-graph replay of the step's C-ABI calls",
            "pair_order": "as drawn" if args.no_plan else "paro_plan_pair_order (conflict-free; same transform)",
        },
        "roofline": {
            "bound": "hbm", "achieved": round(w4_gbs, 1) if w4_gbs else None, "peak": hbm, "unit": "GB/s",
            "frac": round(w4_gbs / hbm, 4) if w4_gbs else None, "traffic": traffic,
            "algorithmic_bytes_per_launch": int(bytes_of("plain") / w4_launches),
            "kernel": ("w4_stream_kernel" if M <= 16 else "w4_gemv_kernel")
                      + " (INT4 linear; one launch per batched call of a step's linears, timed alone "
                        "with plain weights), algorithmic bytes / device time",
            "peak_kind": f"{peak_kind} HBM copy bandwidth",
        },
        "e2e": {"value": round(e2e_value, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(ms_e2e, 6)},
        "gpu_launches": units[0].launches("batched") * args.steps,
        "clocks": clocks,
        "variants_ms_per_step": {k: round(v, 6) for k, v in results.items()},
        "rotation_overhead_pct": (round(100 * (ms - results["batched_plain"]) / results["batched_plain"], 2)
                                  if "batched_plain" in results else None),
        "rotation_overhead_vs_per_linear_plain_pct": round(100 * (ms - plain_ms) / plain_ms, 2) if plain_ms else None,
        "rotation_overhead_unfused_pct": (round(100 * (results["unfused"] - plain_ms) / plain_ms, 2)
                                          if plain_ms and "unfused" in results else None),
        "rotation_overhead_per_linear_fused_pct": (round(100 * (results["fused"] - plain_ms) / plain_ms, 2)
                                                   if plain_ms and "fused" in results else None),
        "rotate_kernel_gbs": round(rot_gbs, 1) if rot_gbs else None,
        "rotate_backward": ({"ms_per_step": round(bwd_ms, 6),
                             "gbs": round(bytes_of("rotate_backward") / (bwd_ms * 1e-3) / 1e9, 1),
                             "what": "dL/dx, dL/dtheta, dL/ds of the step's transforms for a synthetic upstream "
                                     "gradient (paro_rotate_backward, one call per linear)",
                             "bound": "shared memory: each stage moves 8 B per element forward and 16 B back "
                                      "(x and its gradient)"} if bwd_ms else None),
        "tokens_per_s": round(M * world / (ms * 1e-3), 1),
        "tflops": round(flops_step * world / (ms * 1e-3) / 1e12, 3),
        "hbm_frac_of_measured": round(value / hbm, 4),
    }
    if prefill:
        tf = flops_step / (w4_ms * 1e-3) / 1e12 if w4_ms else None
        out["roofline"] = {"bound": "tensor", "achieved": round(tf, 2) if tf else None,
                           "peak": bf16, "unit": "TFLOP/s",
                           "frac": round(tf / bf16, 4) if tf else None, "traffic": traffic,
                           "peak_sustained": bf16_sus,
                           "frac_of_sustained": round(tf / bf16_sus, 4) if tf and bf16_sus else None,
                           "algorithmic_bytes_per_launch": int(bytes_of("plain") / w4_launches),
                           "kernel": "INT4 linear, 2*M*d_in*d_out / device time",
                           "peak_kind": f"{peak_kind} bf16 dense (f16 operands: same nominal rate)"}
    if rank == 0 and not args.no_cpu:
        gbs, cores, sample, one = oracle_sample(args.config, args.M, one_core_seconds=4.0)
        out["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                               "sample": sample,
                               "one_core": {"value": round(one[0], 4), "unit": "GB/s", "cores": 1,
                                            "sample": one[1]}}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
