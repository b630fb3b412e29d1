"""Seeded synthetic problems shaped like the workloads of the ParoQuant pages.

Distributions (one linear layer, d = d_in):
  * every rotation stage is a uniformly random perfect matching of the d
    channels: a random permutation p of 0..d-1 cut into pairs (p[2t], p[2t+1]),
    orientation kept as drawn;
  * angles theta ~ U(-pi, pi) per pair and stage; the boundary takes the fp32
    round-to-nearest values of cos(theta) and sin(theta), computed in fp64;
  * channel scales s = exp(0.3 * N(0, 1)), rounded to fp32;
  * weights W ~ N(0, 0.02^2) in fp32, with 4 distinct input columns x10;
  * activations x ~ N(0, 1) with 4 distinct channels x20 (drawn independently
    of the weight columns), rounded to bf16 (round to nearest even).

Random streams come from numpy's PCG64 seeded through SeedSequence with
(base, tag, layer, index) so that every quantity of every layer has its own
stream and the draw does not depend on which other layers are generated.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# Decoder-layer linears as (name, d_in, d_out).
LAYER_SHAPES = {
    "qwen2.5-1.5b": [
        ("q", 1536, 1536), ("k", 1536, 256), ("v", 1536, 256), ("o", 1536, 1536),
        ("gate", 1536, 8960), ("up", 1536, 8960), ("down", 8960, 1536),
    ],
    "llama-3-8b": [
        ("q", 4096, 4096), ("k", 4096, 1024), ("v", 4096, 1024), ("o", 4096, 4096),
        ("gate", 4096, 14336), ("up", 4096, 14336), ("down", 14336, 4096),
    ],
    "tiny": [("tiny", 512, 512)],
}

_TAG_PAIRS, _TAG_THETA, _TAG_SCALE, _TAG_W, _TAG_WCOL, _TAG_X, _TAG_XCH = 1, 2, 3, 4, 5, 6, 7


def _rng(base: int, tag: int, layer: int, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([base, tag, layer, index])))


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returns fp32 holding bf16 values."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return (r & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


@dataclasses.dataclass
class LinearProblem:
    name: str
    d_in: int
    d_out: int
    M: int
    K: int
    group: int
    seed: int
    layer: int
    pairs: np.ndarray   # uint16 [K, d_in/2, 2]; stage 0 is applied first
    theta: np.ndarray   # float64 [K, d_in/2]
    cos_t: np.ndarray   # float32 [K, d_in/2]
    sin_t: np.ndarray   # float32 [K, d_in/2]
    scale: np.ndarray   # float32 [d_in]
    x: np.ndarray       # float32 [M, d_in], every value exactly a bf16
    W: np.ndarray | None  # float32 [d_out, d_in] or None when drawn on the device
    w_outlier_cols: np.ndarray
    x_outlier_ch: np.ndarray


def linear_problem(base: int, layer: int, d_in: int, d_out: int, M: int, K: int = 8,
                   group: int = 128, name: str = "", host_weights: bool = True) -> LinearProblem:
    """Draw one seeded linear layer problem (tables, scales, weights, activations)."""
    if d_in % 2:
        raise ValueError("d_in must be even")
    half = d_in // 2
    pairs = np.empty((K, half, 2), dtype=np.uint16)
    for k in range(K):
        p = _rng(base, _TAG_PAIRS, layer, k).permutation(d_in)
        pairs[k] = p.reshape(half, 2).astype(np.uint16)
    theta = _rng(base, _TAG_THETA, layer).uniform(-math.pi, math.pi, size=(K, half))
    cos_t = np.cos(theta).astype(np.float32)
    sin_t = np.sin(theta).astype(np.float32)
    scale = np.exp(0.3 * _rng(base, _TAG_SCALE, layer).standard_normal(d_in)).astype(np.float32)

    wcols = _rng(base, _TAG_WCOL, layer).choice(d_in, size=4, replace=False)
    W = None
    if host_weights:
        W = (_rng(base, _TAG_W, layer).standard_normal((d_out, d_in), dtype=np.float32)
             * np.float32(0.02))
        W[:, wcols] *= np.float32(10.0)
    xch = _rng(base, _TAG_XCH, layer).choice(d_in, size=min(4, d_in), replace=False)
    x = _rng(base, _TAG_X, layer).standard_normal((M, d_in), dtype=np.float32)
    x[:, xch] *= np.float32(20.0)
    x = bf16_round(x)
    return LinearProblem(name=name, d_in=d_in, d_out=d_out, M=M, K=K, group=group, seed=base,
                         layer=layer, pairs=pairs, theta=theta, cos_t=cos_t, sin_t=sin_t,
                         scale=scale, x=x, W=W, w_outlier_cols=wcols, x_outlier_ch=xch)


def config_problems(config: int, M: int | None = None, layers: int | None = None,
                    host_weights: bool = True, only: list[str] | None = None):
    """Yield the seeded problems of one workload configuration.

    0: one 512x512 layer, M=4.  1: the seven Qwen2.5-1.5B-shaped linears, M=1.
    2: the seven Llama-3-8B-shaped linears (M from {1,4,8,16}, default 1).
    3: the Llama-3-8B-shaped linears at M=2048.
    4: 28 Qwen2.5-1.5B-shaped decoder layers x 7 linears at M=16.
    """
    base = 0x5A17 + config
    if config == 0:
        shapes, M, nl = LAYER_SHAPES["tiny"], 4 if M is None else M, 1
    elif config == 1:
        shapes, M, nl = LAYER_SHAPES["qwen2.5-1.5b"], 1 if M is None else M, 1
    elif config == 2:
        shapes, M, nl = LAYER_SHAPES["llama-3-8b"], 1 if M is None else M, 1
    elif config == 3:
        shapes, M, nl = LAYER_SHAPES["llama-3-8b"], 2048 if M is None else M, 1
    elif config == 4:
        shapes, M, nl = LAYER_SHAPES["qwen2.5-1.5b"], 16 if M is None else M, 28
    else:
        raise ValueError(f"unknown configuration {config}")
    if layers is not None:
        nl = layers
    for li in range(nl):
        for si, (nm, d_in, d_out) in enumerate(shapes):
            if only is not None and nm not in only:
                continue
            yield linear_problem(base, li * 16 + si, d_in, d_out, M, 8, 128, name=nm,
                                 host_weights=host_weights)


def device_weights(prob: LinearProblem, device):
    """Draw the weights of `prob` on a CUDA device (same distribution, not the same
    values as the host draw); used where the host draw would take too long."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed((prob.seed << 20) ^ (prob.layer << 4) ^ 0xA5)
    W = torch.randn(prob.d_out, prob.d_in, generator=g, device=device, dtype=torch.float32)
    W.mul_(0.02)
    cols = torch.as_tensor(prob.w_outlier_cols, device=device, dtype=torch.long)
    W[:, cols] *= 10.0
    return W
