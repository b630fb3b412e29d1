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
roofline  = the step's dominant kernel (at one token per linear the step is a
            single launch of the fused stream-K kernel), algorithmic bytes per
            launch / its share of the timed region, against the measured HBM
            copy bandwidth
sub_records = the rest of the metric: the Llama-3-8B-shaped layer at 2048
            tokens (TFLOP/s of the tensor-core INT4 linear, rotation overhead),
            the 196-linear Qwen2.5-1.5B-shaped stack at 16 tokens, and the
            Llama-3-8B-shaped layer at 1, 4, 8 and 16 tokens
cpu_baseline = the fp64 CPU oracle on a bounded sample of the same workload

Timing: every timed region is exactly --steps steps, replayed as CUDA graphs
whose calls chain by programmatic dependent launch (all graphs launched once
beforehand); the region is repeated back to back for at least a second (the
headline) and the median repetition is reported, with SM clocks sampled over
all repetitions.

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
# one ncu capture (metrics dram__bytes_read.sum, dram__bytes_write.sum) of
#   config 1: `bench.py --profile --variants batched --config 1 --steps 28 --warmup 3 --no-cpu`
#             (the fused one-launch step; the 21st launch),
#   config 3: `... --variants batched,batched_plain --config 3 --steps 2` (the
#             tensor-core launch on fp16 activations, the same kernel in both
#             variants; the rounding pass of the plain step is not included),
#   config 4: `... --variants batched_plain --config 4 --steps 8` (the INT4 launch alone;
#             the first launch after four skipped),
# with the sha256 prefix of the kernel's sources at capture time: once the
# sources change, the figure no longer describes the kernel and the bench
# reports null.  (Config 2's fused step was not captured.)
TRAFFIC = {
    1: {"bytes": 25990656 + 0, "src": ("w4_stream.cu", "w4_stream.cuh", "rotate_decode_cta.cuh"), "sha": "f5a614ede539d503"},
    3: {"bytes": 353620736 + 133817088, "src": ("w4_tc.cu", "w4_tc.cuh"), "sha": "58523abd4a64b532"},
    4: {"bytes": 25540864 + 0, "src": ("w4_stream.cu", "w4_stream.cuh"), "sha": "8c2412e535f4abba"},
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
        self.ws = torch.zeros(max(paro.paro_workspace_bytes(p.M, p.d_in), 256), dtype=torch.uint8, device=dev)
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

    def dense(self, paro):
        # the contrast the pages draw: a dense d x d rotation (bf16 matrix
        # multiply on the tensor cores) before the same INT4 linear
        if getattr(self, "Q", None) is None:
            import torch
            g = torch.Generator(device=self.x.device)
            g.manual_seed(self.d_in * 131 + self.d_out)
            self.Q = (torch.randn(self.d_in, self.d_in, generator=g, device=self.x.device)
                      * self.d_in ** -0.5).to(torch.bfloat16)
        paro.paro_dense_rotate(self.x, self.Q, out=self.xr)
        paro.paro_w4_linear(self.xr, self.qw0, self.sc0, self.z0, out=self.y)

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

    def w4a4(self, paro):
        # the weight-activation variant on the same packed weights: transform,
        # per-token INT4 codes of x~, the INT4 x INT4 linear
        if getattr(self, "ws4", None) is None:
            import torch
            need = paro.lib.paro_w4a4_workspace_bytes(self.M, self.d_in, self.d_out, 1)
            self.ws4 = torch.empty(max(need, 256), dtype=torch.uint8, device=self.x.device)
            self.w4a4_launches = 3 + (1 if paro.lib.paro_w4a4_workspace_bytes(self.M, self.d_in, self.d_out, 0)
                                      else 0)
        paro.paro_rotate_w4a4_linear(self.x, self.pairs, self.cos, self.sin, self.scale, self.qw, self.sc, self.z,
                                     out=self.y, workspace=self.ws4)

    def fused_e2e(self, paro):
        self.x.copy_(self.x_host, non_blocking=True)
        self.fused(paro)
        self.y_host.copy_(self.y, non_blocking=True)


# kernels launched per linear of each variant (batched: 2 per call of up to 7 linears)
LAUNCHES = {"fused": 2, "unfused": 2, "plain": 1, "rotate": 1, "fused_e2e": 2,  # plain: 2 when M > 64
            "rotate_backward": 2, "dense": 2}
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
            ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=lins[0].x.device)
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
        if variant == "fused":
            # the single-linear call at one token is the same one-launch form
            return sum(1 if l.M == 1 else 2 for l in self.lins)
        if variant == "w4a4":
            # transform, codes, linear, and an ordered reduction when the linear
            # splits a tile's groups over several CTAs
            return sum(getattr(l, "w4a4_launches", 4) for l in self.lins)
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


def warm_eager(torch, paro, units, variant):
    """Run every unit of a variant once outside capture (library-side set-up,
    first-launch costs), on a side stream, and wait for it."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for unit in units:
            unit.run(paro, variant)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()


def capture_units(torch, paro, units, variant):
    """One CUDA graph running the given units in order (their launches chain by
    programmatic dependent launch inside the graph)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for unit in units:
            unit.run(paro, variant)
    return g


def chained_plan(torch, paro, units, variant, steps):
    """Graphs that run `steps` steps in unit order 0, 1, ..., L-1, 0, ... (L
    units) in as few graph launches as possible: a full-cycle graph replayed
    steps // L times, then a graph of the first steps % L units.  Returns (the
    sequence of graph launches, the distinct graphs)."""
    L = len(units)
    warm_eager(torch, paro, units, variant)
    full = capture_units(torch, paro, units, variant) if steps >= L else None
    r = steps % L
    rem = capture_units(torch, paro, units[:r], variant) if r else None
    seq = [full] * (steps // L) + ([rem] if rem is not None else [])
    return seq, [g for g in (full, rem) if g is not None]


def isolated_plan(torch, paro, units, variant, steps):
    """One graph launch per step (no chaining across steps): every step waits
    for the previous one to finish before its first kernel starts."""
    warm_eager(torch, paro, units, variant)
    per_unit = [capture_units(torch, paro, [u], variant) for u in units]
    return [per_unit[i % len(units)] for i in range(steps)], per_unit


def l2_bytes(torch):
    try:
        return int(torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size)
    except Exception:  # pragma: no cover
        return 126 * 2 ** 20


class Timed:
    """Device time of one variant: exactly `steps` steps per timed region,
    bracketed by a barrier and a synchronize on both sides, timed with CUDA
    events on the launching stream.  The region is repeated back to back
    (the same count on every rank) until it has run for `min_seconds`; each
    repetition's time is the max over ranks, and the median repetition is the
    figure.  When `steps` steps move less than twice the L2 size, a buffer
    larger than L2 is written between repetitions (outside the timing)."""

    def __init__(self, median, lo, hi, reps, warmup_steps, l2):
        self.ms, self.lo, self.hi, self.reps, self.warmup_steps, self.l2 = median, lo, hi, reps, warmup_steps, l2

    def summary(self):
        return {"ms_per_step": round(self.ms, 6), "reps": self.reps, "rep_min_ms": round(self.lo, 6),
                "rep_max_ms": round(self.hi, 6), "l2": self.l2}


def time_plan(torch, plan, steps, warmup, dist, step_bytes, min_seconds=0.25, flush=None):
    seq, distinct = plan
    for g in distinct:                 # every graph launched once before any timing
        g.replay()
    done = 0
    while done < max(warmup, 1):       # at least `warmup` untimed steps
        for g in seq:
            g.replay()
        done += steps
    torch.cuda.synchronize()
    need_flush = flush is not None and steps * step_bytes < 2 * l2_bytes(torch)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)

    def one():
        if need_flush:
            flush.zero_()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        start.record()
        for g in seq:
            g.replay()
        end.record()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        return start.elapsed_time(end)

    first = max_over_ranks(torch, dist, one(), "cuda")
    n = max(3, min(2000, int(min_seconds * 1e3 / max(first, 1e-3)) + 1))
    n = int(max_over_ranks(torch, dist, float(n), "cuda"))
    reps = [one() for _ in range(n)]
    if dist is not None:
        t = torch.tensor(reps, dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        reps = t.tolist()
    per_step = sorted(r / steps for r in reps)
    l2 = ("L2 flushed between repetitions (a 256 MB write)" if need_flush
          else "each timed region streams more than twice the L2 size")
    return Timed(statistics.median(per_step), per_step[0], per_step[-1], n, done, l2)


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
def bytes_of(step_lins, M, variant):
    """Algorithmic bytes of one step of a variant (each table read once per call)."""
    if variant in ("plain", "batched_plain"):
        return sum(linear_bytes(l.d_in, l.d_out, M, rotate=False) for l in step_lins)
    if variant == "rotate":
        return sum(4 * M * l.d_in + TABLE_BYTES_PER_CH * l.d_in for l in step_lins)
    if variant == "dense":
        # the d x d bf16 matrix and the x~ round trip on top of the plain linear
        return sum(linear_bytes(l.d_in, l.d_out, M, rotate=False) + 2 * l.d_in * l.d_in + 4 * M * l.d_in
                   for l in step_lins)
    if variant == "rotate_backward":
        # x (bf16) and the upstream gradient in, dx out (fp32), the tables and
        # the outputs dtheta, dscale; the per-block partial sums round trip
        def bwd(l):
            R = 4 if 8 * 4 * l.d_in <= 226 * 1024 else (2 if 8 * 2 * l.d_in <= 226 * 1024 else 1)
            n = K_STAGES * l.d_in // 2 + l.d_in
            return 10 * M * l.d_in + TABLE_BYTES_PER_CH * l.d_in + 4 * n + 2 * 4 * n * -(-M // R)
        return sum(bwd(l) for l in step_lins)
    return sum(linear_bytes(l.d_in, l.d_out, M, unfused=(variant == "unfused")) for l in step_lins)


def run_workload(torch, paro, args, config, M_arg, variants, dist, rank, dev, flush, clock_variant=None,
                 isolated=False, e2e=False, min_seconds=0.25, per_linear=False):
    """Build one workload, time its variants; returns a dict of results."""
    name, shapes, M, n_layers, stack = workload(config, M_arg)
    layers = build_layers(config, M, n_layers, rank, dev, plan=not args.no_plan)
    torch.cuda.synchronize()
    units = [Unit(sum(layers, []), paro)] if stack else [Unit(l, paro) for l in layers]
    del layers
    step_lins = units[0].lins
    out = {"name": name, "M": M, "units": units, "step_lins": step_lins, "timed": {}, "clocks": None}
    for v in variants:
        plan = chained_plan(torch, paro, units, v, args.steps)
        sb = bytes_of(step_lins, M, v)
        if v == clock_variant:
            with ClockSampler(_smi_id(torch)) as cs:
                t = time_plan(torch, plan, args.steps, args.warmup, dist, sb, min_seconds=1.0, flush=flush)
            out["clocks"] = cs.summary()
        else:
            t = time_plan(torch, plan, args.steps, args.warmup, dist, sb, min_seconds=min_seconds, flush=flush)
        out["timed"][v] = t
        del plan
    if isolated:
        plan = isolated_plan(torch, paro, units, "batched", args.steps)
        out["isolated"] = time_plan(torch, plan, args.steps, args.warmup, dist, bytes_of(step_lins, M, "batched"),
                                    min_seconds=min_seconds, flush=flush)
        del plan
    if e2e:
        plan = chained_plan(torch, paro, units, "batched_e2e", args.steps)
        out["e2e"] = time_plan(torch, plan, args.steps, args.warmup, dist, bytes_of(step_lins, M, "batched"),
                               min_seconds=min_seconds, flush=flush)
        del plan
    if per_linear and not stack:
        # each linear of the layer alone: a batched call of that one linear per
        # step (fused, and plain), cycling over the same layers as above (last:
        # the units made here take over the linears' x and y views)
        out["per_linear"] = {}
        for i, (lname, _, _) in enumerate(shapes):
            lin_units = [Unit([u.lins[i]], paro) for u in units]
            rec = {}
            for v in ("batched", "batched_plain"):
                plan = chained_plan(torch, paro, lin_units, v, args.steps)
                sb = bytes_of([step_lins[i]], M, v)
                tl = time_plan(torch, plan, args.steps, args.warmup, dist, sb, min_seconds=0.1, flush=flush)
                rec["fused" if v == "batched" else "plain"] = tl
                del plan
            out["per_linear"][lname] = (step_lins[i], rec)
            del lin_units
    return out


def overhead(t, a, b):
    return round(100 * (t[a].ms - t[b].ms) / t[b].ms, 2) if a in t and b in t else None


def sub_record(r, world, hbm, bf16, bf16_sus):
    """One workload's figures for the JSON line (value in its metric's unit)."""
    t, M, lins = r["timed"], r["M"], r["step_lins"]
    ms = t["batched"].ms
    flops = sum(2 * M * l.d_in * l.d_out for l in lins)
    prefill = M >= PREFILL_M
    rec = {"workload": f"{r['name']}: fused rotate + INT4 linear, M={M}, K={K_STAGES}, group={GROUP}",
           "linears_per_step": len(lins), "distinct_units_cycled": len(r["units"]),
           "ms_per_step": round(ms, 6), "reps": t["batched"].reps, "l2": t["batched"].l2,
           "rotation_overhead_pct": overhead(t, "batched", "batched_plain")}
    if "dense" in t:
        rec["per_linear"] = {k: round(t[k].ms, 6) for k in ("plain", "fused", "dense") if k in t}
        rec["rotation_overhead_per_linear_fused_pct"] = overhead(t, "fused", "plain")
        rec["dense_rotation_overhead_pct"] = overhead(t, "dense", "plain")
    if prefill:
        tf = whole_job_rate(flops, world, ms) / 1e12
        rec.update(value=round(tf, 2), unit="TFLOP/s", frac_of_bf16=round(tf / bf16, 4))
        if "batched_plain" in t:
            tp = flops / (t["batched_plain"].ms * 1e-3) / 1e12
            rec["roofline"] = {"bound": "tensor", "kernel": "w4_tc_kernel (tcgen05) on plain weights: the step "
                                                            "is one bf16->fp16 rounding launch into the workspace "
                                                            "and one tensor-core launch; 2*M*d_in*d_out / step time",
                               "achieved": round(tp, 2), "peak": bf16, "unit": "TFLOP/s", "frac": round(tp / bf16, 4),
                               "peak_sustained": bf16_sus,
                               "frac_of_sustained": round(tp / bf16_sus, 4) if bf16_sus else None,
                               "traffic": measured_traffic(3, None),
                               "traffic_what": "DRAM bytes of the tensor-core launch (the rounding pass apart)"}
        if "rotate" in t:
            gb = bytes_of(lins, M, "rotate") / (t["rotate"].ms * 1e-3) / 1e9
            rec["rotate_kernel"] = {"gbs": round(gb, 1), "frac_of_hbm": round(gb / hbm, 4),
                                    "ms_per_step": round(t["rotate"].ms, 6),
                                    "what": "paro_rotate alone, one call per linear (bf16 in and out)"}
    else:
        gb = whole_job_rate(bytes_of(lins, M, "batched"), world, ms) / 1e9
        rec.update(value=round(gb, 1), unit="GB/s", frac_of_hbm=round(gb / hbm, 4),
                   tokens_per_s=round(M * world / (ms * 1e-3), 1))
        if "batched_plain" in t:
            gp = bytes_of(lins, M, "batched_plain") / (t["batched_plain"].ms * 1e-3) / 1e9
            rec["int4_alone"] = {"gbs": round(gp, 1), "frac_of_hbm": round(gp / hbm, 4),
                                 "ms_per_step": round(t["batched_plain"].ms, 6),
                                 "what": "the same step on plain INT4 weights (no transform)"}
    return rec


def run_timeline(torch, args):
    """Phases of the fused one-token decode launch from the instrumented build
    (global-timer stamps per CTA; see rotation_int4_weight_b200/_build.py).
    The last launch of a chain of chained graphs is read back; times are in us
    from the moment its CTAs' wait for the previous launch ended."""
    import ctypes
    import importlib.util
    pkg = os.path.join(os.path.dirname(os.path.abspath(__file__)), "rotation_int4_weight_b200")
    spec = importlib.util.spec_from_file_location("_paro_build", os.path.join(pkg, "_build.py"))
    builder = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(builder)
    builder.build(timeline=True)
    os.environ["PARO_TIMELINE"] = "1"
    import rotation_int4_weight_b200 as paro
    if not paro.LIB_PATH.endswith("libparo_timeline.so"):
        raise SystemExit("the package was loaded before --timeline could select the instrumented library")
    read = paro.lib.paro_timeline_read
    read.restype, read.argtypes = ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t]
    dev = torch.device("cuda", 0)
    name, shapes, M, n_layers, stack = workload(args.config, args.M)
    if stack or M != 1:
        raise SystemExit("--timeline covers the fused one-token form: a config at M = 1")
    layers = build_layers(args.config, M, n_layers, 0, dev, plan=not args.no_plan)
    units = [Unit(l, paro) for l in layers]
    seq, distinct = chained_plan(torch, paro, units, "batched", args.steps)
    for _ in range(args.warmup):
        for g in seq:
            g.replay()
    torch.cuda.synchronize()
    status = paro.paro_get_device_status()
    buf = np.zeros(2 * 256 * 8, dtype=np.uint64)
    rc = read(buf.ctypes.data, buf.nbytes)
    if rc != 0 or status != 0:
        raise SystemExit(f"timeline read {rc}, device status {status}")
    t = buf.reshape(2, 256, 8).astype(np.int64)
    last = t[0] if t[0, :, 0].max() > t[1, :, 0].max() else t[1]
    rot = [i for i in range(256) if last[i, 5] == 1]
    t0 = min(last[i, 1] for i in rot)
    us = lambda v: round((float(v) - t0) / 1e3, 2)
    out = {"workload": name, "steps_chained": args.steps, "time_origin": "end of the transform CTAs' wait for "
           "the previous launch", "transform_ctas": [], "int4_ctas": []}
    for i in rot:
        r = last[i]
        out["transform_ctas"].append({"cta": i, "entry": us(r[0]), "wait_done": us(r[1]), "staged": us(r[2]),
                                      "stages_done": us(r[3]), "flag": us(r[4])})
    int4 = np.array([i for i in range(256) if last[i, 5] == 2])
    for pi in sorted(set(int(v) for v in last[int4, 7])):
        g = int4[last[int4, 7] == pi]
        rec = {"last_linear": pi, "ctas": int(len(g)),
               "units_warp0": [int(last[g, 6].min()), int(last[g, 6].max())]}
        for k, nm in enumerate(["entry", "wait_done", "first_unit", "units_done", "end"]):
            col = [us(v) for v in last[g, k]]
            rec[nm] = {"min": min(col), "median": round(float(np.median(col)), 2), "max": max(col)}
        out["int4_ctas"].append(rec)
    print(json.dumps({"timeline": out}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20, help="steps per timed region")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--M", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-sub", action="store_true", help="skip the prefill, stack and Llama decode sub-records")
    ap.add_argument("--variants",
                    default="batched,batched_plain,fused,plain,unfused,rotate,rotate_backward,dense,w4a4")
    ap.add_argument("--no-plan", action="store_true",
                    help="use the pair tables as drawn instead of the conflict-free order of paro_plan_pair_order")
    ap.add_argument("--profile", action="store_true",
                    help="run only the listed variants once each (no repetitions, no end-to-end leg, no "
                         "sub-records, no CPU baseline): a short launch sequence for ncu; not bench values")
    ap.add_argument("--timeline", action="store_true",
                    help="one-token configs: load the instrumented library (built on first use) and print the "
                         "global-timer phases of the last fused launch of a chain of steps, per CTA group; "
                         "not bench values")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.steps < 1:
        raise SystemExit("--steps must be >= 1")
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
    if args.timeline:
        if world > 1:
            raise SystemExit("--timeline runs on one GPU")
        return run_timeline(torch, args)
    import rotation_int4_weight_b200 as paro
    dev = torch.device("cuda", torch.cuda.current_device())
    hbm, bf16, bf16_sus, peak_kind = peaks()

    if args.profile:
        # a fixed, short launch sequence: each listed variant's chained graphs,
        # warmed and then replayed once
        name, shapes, M, n_layers, stack = workload(args.config, args.M)
        layers = build_layers(args.config, M, n_layers, rank, dev, plan=not args.no_plan)
        units = [Unit(sum(layers, []), paro)] if stack else [Unit(l, paro) for l in layers]
        res = {}
        for v in [v for v in args.variants.split(",") if v]:
            seq, distinct = chained_plan(torch, paro, units, v, args.steps)
            for _ in range(args.warmup):
                for g in distinct:
                    g.replay()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for g in seq:
                g.replay()
            b.record()
            torch.cuda.synchronize()
            res[v] = a.elapsed_time(b) / args.steps
            del seq, distinct
        if rank == 0:
            print(json.dumps({"profile_run": True, "variants_ms_per_step": res}), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return

    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    variants = [v for v in args.variants.split(",") if v]
    if "batched" not in variants:
        variants.insert(0, "batched")
    head = run_workload(torch, paro, args, args.config, args.M, variants, dist, rank, dev, flush,
                        clock_variant="batched", isolated=True, e2e=True, per_linear=True)
    t, M, step_lins, units = head["timed"], head["M"], head["step_lins"], head["units"]
    ms = t["batched"].ms
    step_bytes = bytes_of(step_lins, M, "batched")
    flops_step = sum(2 * M * l.d_in * l.d_out for l in step_lins)
    prefill = M >= PREFILL_M
    value = (whole_job_rate(flops_step, world, ms) / 1e12 if prefill
             else whole_job_rate(step_bytes, world, ms) / 1e9)
    h2d = units[0].x_all.numel() * 2
    d2h = units[0].y_all.numel() * 2
    ms_e2e = head["e2e"].ms
    e2e_value = (whole_job_rate(flops_step, world, ms_e2e) / 1e12 if prefill
                 else whole_job_rate(step_bytes + h2d + d2h, world, ms_e2e) / 1e9)
    launches = units[0].launches("batched")
    # the dominant kernel: at one token per linear the whole step is one launch
    # of the stream-K kernel in its fused form (transform CTAs + INT4 CTAs);
    # otherwise the INT4 launch, timed alone on plain weights
    one_launch = launches == len(units[0].calls) and not prefill
    if prefill:
        kt = t.get("batched_plain", t["batched"])
        ach = flops_step / (kt.ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 2), "peak": bf16, "unit": "TFLOP/s",
                "frac": round(ach / bf16, 4), "traffic": measured_traffic(args.config, args.M),
                "peak_sustained": bf16_sus, "frac_of_sustained": round(ach / bf16_sus, 4) if bf16_sus else None,
                "kernel": "w4_tc_kernel, 2*M*d_in*d_out per launch / (timed region / launches)",
                "peak_kind": f"{peak_kind} bf16 dense (f16 operands: same nominal rate)"}
    else:
        kv = "batched" if one_launch else "batched_plain"
        kt = t.get(kv, t["batched"])
        per_launch_bytes = bytes_of(step_lins, M, kv) / units[0].launches(kv)
        per_launch_ms = kt.ms / units[0].launches(kv)
        ach = per_launch_bytes / (per_launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm, "unit": "GB/s", "frac": round(ach / hbm, 4),
                "traffic": measured_traffic(args.config, args.M),
                "algorithmic_bytes_per_launch": int(per_launch_bytes),
                "kernel": ("w4_stream_kernel, fused form (one launch per step: transform CTAs and INT4 CTAs)"
                           if one_launch else "w4_stream_kernel (INT4 linear, plain weights, one launch per "
                                              "batched call)")
                          + "; algorithmic bytes per launch / (timed region / launches)",
                "peak_kind": f"{peak_kind} HBM copy bandwidth"}
    plain_ms = t["plain"].ms if "plain" in t else None
    iso = head["isolated"]
    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s" if prefill else "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {
            "workload": f"{head['name']}: fused rotate + INT4 linear (one batched C-ABI call per {BATCH} linears), "
                        f"M={M}, K={K_STAGES}, group={GROUP}, asymmetric INT4, bf16 activations",
            "linears_per_step": len(step_lins), "distinct_units_cycled": len(units),
            "timing": (f"each timed region is exactly {args.steps} steps, replayed as CUDA graphs of up to "
                       f"{len(units)} steps whose calls chain by programmatic dependent launch; every graph is "
                       f"launched before timing; the region is repeated {t['batched'].reps} times back to back "
                       "(barrier + synchronize around each) and the median repetition is reported"),
            "l2": t["batched"].l2,
            "pair_order": "as drawn" if args.no_plan else "paro_plan_pair_order (conflict-free; same transform)",
        },
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s" if prefill else "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 6),
                "what": "per step: host->device copy of the step's inputs from pinned memory, the C-ABI call, "
                        "device->host copy of its outputs, all inside the timed region"},
        "gpu_launches": launches * args.steps,
        "clocks": head["clocks"],
        "timed_region": t["batched"].summary(),
        "isolated_step": {"ms_per_step": round(iso.ms, 6),
                          "value": round((flops_step / 1e12 if prefill else step_bytes / 1e9) / (iso.ms * 1e-3), 3),
                          "what": "one graph launch per step, so no step overlaps the previous one"},
        "variants_ms_per_step": {k: round(v.ms, 6) for k, v in t.items()},
        "rotation_overhead_pct": overhead(t, "batched", "batched_plain"),
        "rotation_overhead_unfused_pct": overhead(t, "unfused", "plain"),
        "rotation_overhead_per_linear_fused_pct": overhead(t, "fused", "plain"),
        "dense_rotation_overhead_pct": overhead(t, "dense", "plain"),
        "w4a4": ({"ms_per_step": round(t["w4a4"].ms, 6),
                  "vs_w4a16_fused_pct": overhead(t, "w4a4", "fused"),
                  "what": "the weight-activation variant per linear (paro_rotate_w4a4_linear: transform, per-token "
                          "INT4 codes, INT4 x INT4 linear on the same packed weights); vs_w4a16_fused_pct: its "
                          "time against the weight-only fused per-linear calls"} if "w4a4" in t else None),
        "dense_rotation": ("the contrast the pages draw: a dense d x d bf16 rotation (paro_dense_rotate, tensor "
                           "cores) then the same INT4 linear, per linear; its overhead against the plain per-"
                           "linear INT4 calls sits beside rotation_overhead_per_linear_fused_pct"),
        "rotate_kernel_gbs": (round(bytes_of(step_lins, M, "rotate") / (t["rotate"].ms * 1e-3) / 1e9, 1)
                              if "rotate" in t else None),
        "rotate_backward": ({"ms_per_step": round(t["rotate_backward"].ms, 6),
                             "gbs": round(bytes_of(step_lins, M, "rotate_backward")
                                          / (t["rotate_backward"].ms * 1e-3) / 1e9, 1),
                             "what": "dL/dx, dL/dtheta, dL/ds of the step's transforms for a synthetic upstream "
                                     "gradient (paro_rotate_backward, one call per linear)"}
                            if "rotate_backward" in t else None),
        "tokens_per_s": round(M * world / (ms * 1e-3), 1),
        "hbm_frac_of_measured": None if prefill else round(value / hbm, 4),
    }
    if head.get("per_linear") and not prefill:
        pl = {}
        for lname, (lin, rec) in head["per_linear"].items():
            e = {}
            for k, tl in rec.items():
                gb = bytes_of([lin], M, "batched" if k == "fused" else "batched_plain") / (tl.ms * 1e-3) / 1e9
                e[k] = {"us": round(tl.ms * 1e3, 2), "gbs": round(gb, 1), "frac_of_hbm": round(gb / hbm, 4)}
            if "fused" in e and "plain" in e:
                e["rotation_overhead_pct"] = round(100 * (e["fused"]["us"] - e["plain"]["us"]) / e["plain"]["us"], 1)
            pl[lname] = e
        out["per_linear"] = pl
        out["per_linear_what"] = ("each linear of the layer alone, one batched call of that linear per step, chained "
                                  "over the same distinct layers; fused = with its transform, plain = plain weights")
    del head, units, step_lins, t
    torch.cuda.empty_cache()
    if not args.no_sub and args.config == 1 and args.M is None:
        subs = {}
        for key, cfg, m, vs in [("prefill_llama_m2048", 3, None, "batched,batched_plain,rotate,plain,fused,dense"),
                                ("stack_qwen_196_linears_m16", 4, None, "batched,batched_plain"),
                                ("decode_llama_m1", 2, 1, "batched,batched_plain"),
                                ("decode_llama_m4", 2, 4, "batched,batched_plain"),
                                ("decode_llama_m8", 2, 8, "batched,batched_plain"),
                                ("decode_llama_m16", 2, 16, "batched,batched_plain")]:
            r = run_workload(torch, paro, args, cfg, m, vs.split(","), dist, rank, dev, flush, min_seconds=0.5)
            subs[key] = sub_record(r, world, hbm, bf16, bf16_sus)
            if cfg == 4:
                subs[key]["tokens_per_s_note"] = "one step = all 196 linears at 16 tokens"
            del r
            torch.cuda.empty_cache()
        out["sub_records"] = subs
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
