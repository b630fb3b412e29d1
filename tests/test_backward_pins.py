"""Pins of the oracle's transform gradients (oracle/backward.py) against
finite differences of the forward oracle and closed forms.  CPU only.

The gradients are those of L = sum(G * x~) for x~ = diag(1/s) R_K ... R_1 x
(page "ParoQuant: pairwise rotations that survive deployment", section "A
rotation small enough to execute"; the angles and scales are the optimizable
parameters of page "ParoQuant: Pairwise Rotation Quantization for Efficient
Reasoning LLM Inference", abstract).  L is linear in x and G, so dL/dx is
exact for any step; the angle and scale derivatives are checked by central
differences in fp64 (truncation ~eps^2, rounding ~1e-16/eps).
"""
from __future__ import annotations

import math

import numpy as np
import pytest

import oracle
from oracle.backward import rotate_backward

EPS = 1e-6


def _case(seed, M, d, K, with_scale=True):
    rng = np.random.default_rng(seed)
    pairs = np.stack([rng.permutation(d).reshape(d // 2, 2) for _ in range(K)]).astype(np.uint16) if K else \
        np.zeros((0, d // 2, 2), np.uint16)
    theta = rng.uniform(-math.pi, math.pi, size=(K, d // 2))
    x = rng.standard_normal((M, d))
    G = rng.standard_normal((M, d))
    s = np.exp(0.3 * rng.standard_normal(d)) if with_scale else None
    return x, G, pairs, theta, s


def _loss(x, G, pairs, theta, s):
    return float((G * oracle.rotate(x, pairs, np.cos(theta), np.sin(theta), s)).sum())


@pytest.mark.parametrize("seed,M,d,K,with_scale", [(1, 3, 8, 3, True), (2, 1, 12, 4, False), (3, 5, 6, 1, True),
                                                   (4, 2, 16, 6, True)])
def test_gradients_match_central_differences(seed, M, d, K, with_scale):
    x, G, pairs, theta, s = _case(seed, M, d, K, with_scale)
    dx, dth, ds = rotate_backward(x, G, pairs, np.cos(theta), np.sin(theta), s)
    # every angle
    for k in range(K):
        for p in range(d // 2):
            tp, tm = theta.copy(), theta.copy()
            tp[k, p] += EPS
            tm[k, p] -= EPS
            fd = (_loss(x, G, pairs, tp, s) - _loss(x, G, pairs, tm, s)) / (2 * EPS)
            assert abs(fd - dth[k, p]) <= 1e-7 * (1 + abs(fd)), (k, p, fd, dth[k, p])
    # every input entry
    for m in range(M):
        for c in range(d):
            xp, xm = x.copy(), x.copy()
            xp[m, c] += EPS
            xm[m, c] -= EPS
            fd = (_loss(xp, G, pairs, theta, s) - _loss(xm, G, pairs, theta, s)) / (2 * EPS)
            assert abs(fd - dx[m, c]) <= 1e-7 * (1 + abs(fd))
    # every channel scale
    if with_scale:
        for c in range(d):
            sp, sm = s.copy(), s.copy()
            sp[c] += EPS
            sm[c] -= EPS
            fd = (_loss(x, G, pairs, theta, sp) - _loss(x, G, pairs, theta, sm)) / (2 * EPS)
            assert abs(fd - ds[c]) <= 1e-7 * (1 + abs(fd))
    else:
        assert ds is None


def test_one_pair_worked_by_hand():
    # d = 2, one stage with the pair (0, 1) at angle t, x = (1, 0), G = (1, 0), s = (2, 4):
    # x~ = (cos t / 2, -sin t / 4), L = cos t / 2, so dL/dt = -sin t / 2,
    # dL/ds = (-(cos t / 2) / 2, 0) and dL/dx = R^T (G / s) = (cos t / 2, sin t / 2)
    t = 0.3
    pairs = np.array([[[0, 1]]], np.uint16)
    dx, dth, ds = rotate_backward(np.array([[1.0, 0.0]]), np.array([[1.0, 0.0]]), pairs, np.array([[math.cos(t)]]),
                                  np.array([[math.sin(t)]]), np.array([2.0, 4.0]))
    assert dth[0, 0] == pytest.approx(-math.sin(t) / 2, abs=1e-15)
    np.testing.assert_allclose(ds, [-math.cos(t) / 4, 0.0], atol=1e-15)
    np.testing.assert_allclose(dx[0], [math.cos(t) / 2, math.sin(t) / 2], atol=1e-15)


def test_scale_only_closed_form():
    x, G, pairs, theta, s = _case(7, 4, 10, 0)
    dx, dth, ds = rotate_backward(x, G, pairs, np.cos(theta), np.sin(theta), s)
    assert dth.shape == (0, 5)
    np.testing.assert_allclose(dx, G / s, rtol=1e-15)
    np.testing.assert_allclose(ds, -(G * x).sum(axis=0) / s ** 2, rtol=1e-14)


def test_input_gradient_keeps_the_norm_without_scale():
    # without the scale the transform is orthogonal: dL/dx = R^T G has the norm of G
    x, G, pairs, theta, _ = _case(9, 6, 64, 8, with_scale=False)
    dx, _, _ = rotate_backward(x, G, pairs, np.cos(theta), np.sin(theta), None)
    np.testing.assert_allclose(np.linalg.norm(dx, axis=1), np.linalg.norm(G, axis=1), rtol=1e-13)
    # and it is the transpose: <dL/dx, v> = <G, R v> for any v
    v = np.random.default_rng(10).standard_normal(x.shape)
    lhs = (dx * v).sum()
    rhs = (G * oracle.rotate(v, pairs, np.cos(theta), np.sin(theta), None)).sum()
    assert lhs == pytest.approx(rhs, rel=1e-12)
