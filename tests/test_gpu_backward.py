"""GPU parity of paro_rotate_backward (gradients of the activation transform)
against the fp64 oracle (oracle/backward.py, itself pinned by finite
differences in tests/test_backward_pins.py), on seeded synthetic problems.

Tolerances (fp32 kernel against fp64): every stage rotates and, going back,
un-rotates each value once (2K roundings of about 2^-24 relative, K <= 16), and
the sums over tokens add per-block fp32 partials, so the relative error is a
few 1e-6 at most; the tests allow 1e-5 of the norm of each output (per row for
dx, per stage for dtheta, the whole vector for dscale) and 1e-4 of its largest
entry elementwise.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import rotation_int4_weight_b200 as paro
from oracle.backward import rotate_backward as oracle_backward
from synth import linear_problem

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _rel(got, ref):
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


def _check(got, ref):
    assert _rel(got, ref) <= 1e-5, _rel(got, ref)
    assert float(np.abs(got - ref).max()) <= 1e-4 * float(np.abs(ref).max()) + 1e-30


def _run(M, d, K, with_scale, seed=5, planned=False):
    p = linear_problem(seed, 0, d, 16, M, K=K, host_weights=False)
    pairs, cos_t, sin_t = p.pairs, p.cos_t, p.sin_t
    if planned and K and d % 64 == 0:
        pairs, cos_t, sin_t = paro.paro_plan_pair_order(pairs, cos_t, sin_t)
    scale = p.scale if with_scale else None
    G = np.random.default_rng(seed + 100).standard_normal((M, d)).astype(np.float32)
    x = torch.from_numpy(p.x).to(DEV).to(torch.bfloat16)
    x_host = x.float().cpu().numpy()
    dev = dict(pairs=torch.from_numpy(pairs.view(np.int16)).to(DEV) if K else None,
               cos_t=torch.from_numpy(cos_t).to(DEV) if K else None,
               sin_t=torch.from_numpy(sin_t).to(DEV) if K else None,
               scale=torch.from_numpy(scale).to(DEV) if with_scale else None)
    (dx, dth, dsc), ws = paro.paro_rotate_backward(x, torch.from_numpy(G).to(DEV), **dev)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    ref = oracle_backward(x_host, G, pairs, cos_t, sin_t, scale)
    return (x, G, dev, ws), (dx, dth, dsc), ref


@pytest.mark.parametrize("M,d,K,with_scale", [
    (1, 512, 8, True), (5, 1536, 3, True),      # 4 rows a block: one full block and a ragged one
    (17, 4096, 8, True), (3, 8960, 8, False),   # 2 rows a block at d = 8960
    (2, 14336, 8, True), (1, 28672, 2, True),   # the widest: one row a block
    (6, 1024, 0, True),                         # scale only
    (64, 2048, 16, True),                       # sixteen stages, sixteen blocks
])
def test_backward_matches_oracle(M, d, K, with_scale):
    _, (dx, dth, dsc), (rdx, rdth, rdsc) = _run(M, d, K, with_scale)
    gx = dx.cpu().numpy()
    for m in range(M):
        _check(gx[m], rdx[m])
    if K:
        gt = dth.cpu().numpy()
        for k in range(K):
            _check(gt[k], rdth[k])
    else:
        assert dth is None
    if with_scale:
        _check(dsc.cpu().numpy(), rdsc)
    else:
        assert dsc is None


def test_backward_with_planned_order_and_repeats_bit_exactly():
    (x, G, dev, ws), (dx, dth, dsc), (rdx, rdth, rdsc) = _run(33, 4096, 8, True, seed=9, planned=True)
    for m in range(33):
        _check(dx.cpu().numpy()[m], rdx[m])
    for k in range(8):
        _check(dth.cpu().numpy()[k], rdth[k])
    _check(dsc.cpu().numpy(), rdsc)
    # the partial sums over blocks are added in a fixed order: a second call
    # gives the same bits
    (dx2, dth2, dsc2), _ = paro.paro_rotate_backward(x, torch.from_numpy(G).to(DEV), **dev, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(dx, dx2) and torch.equal(dth, dth2) and torch.equal(dsc, dsc2)
