"""Pins of the weight-activation (W4A4) oracle (oracle/w4a4.py) to what the
arithmetic fixes, independent of the oracle's own formulas: a worked example
with exactly representable values, the rounding bound of the codes, the
grouped integer form of the linear against dequantise-then-multiply, and
brute-force loops on a tiny case.  No GPU."""
import numpy as np
import pytest

import oracle
from synth import linear_problem


def test_quantize_worked_example():
    # row 0: largest magnitude 7, so s = 1 and the codes are rint(x), ties to even;
    # row 1: largest magnitude 14, s = 2; row 2: all zero, s = 1 and codes 0
    x = np.array([[3.5, -7.0, 1.75, 0.0, 5.25, -3.5, 0.5, 1.0],
                  [7.0, -14.0, 3.0, -1.0, 0.0, 13.0, 5.0, -5.0],
                  [0.0] * 8], dtype=np.float32)
    q, s = oracle.quantize_activations(x)
    assert s.tolist() == [1.0, 2.0, 1.0]
    assert q.tolist() == [[4, -7, 2, 0, 5, -4, 0, 1],
                          [4, -7, 2, 0, 0, 6, 2, -2],
                          [0] * 8]
    assert q.dtype == np.int8


def test_quantize_bounds_on_random_rows():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((9, 640)) * rng.uniform(0.01, 50, (9, 1))).astype(np.float32)
    x[3, 17] = 300.0  # an outlier sets its row's scale
    q, s = oracle.quantize_activations(x)
    assert q.min() >= -8 and q.max() <= 7
    amax = np.abs(x).max(axis=1)
    assert np.allclose(s, amax / 7, rtol=2 ** -23)
    err = np.abs(q * s[:, None].astype(np.float64) - x)
    assert (err <= s[:, None] / 2 * (1 + 1e-6)).all()       # round to nearest: at most half a step
    assert (np.abs(q[np.arange(9), np.abs(x).argmax(axis=1)]) == 7).all()  # the largest maps to +-7


def test_w4a4_linear_equals_dequantise_then_multiply():
    p = linear_problem(41, 0, 512, 96, 5, K=8)
    qw, sw, zw = oracle.pack_weights(p.W, p.pairs, p.cos_t, p.sin_t, p.scale)
    qx, sx = oracle.quantize_activations(oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale))
    y = oracle.w4a4_linear(qx, sx, qw, sw, zw)
    ref = oracle.linear(oracle.dequantize_activations(qx, sx), oracle.dequantize(qw, sw, zw))
    assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()


def test_w4a4_linear_against_python_loops():
    rng = np.random.default_rng(6)
    M, d_in, d_out = 2, 256, 3
    codes = rng.integers(0, 16, (d_out, d_in)).astype(np.uint8)
    qw = oracle.pack_nibbles(codes)
    sw = rng.uniform(0.001, 0.05, (d_out, 2)).astype(np.float16)
    zw = rng.integers(0, 16, (d_out, 2)).astype(np.float16)
    qx = rng.integers(-8, 8, (M, d_in)).astype(np.int8)
    sx = rng.uniform(0.1, 2.0, M).astype(np.float32)
    y = oracle.w4a4_linear(qx, sx, qw, sw, zw)
    for m in range(M):
        for n in range(d_out):
            acc = 0.0
            for k in range(d_in):
                g = k // 128
                acc += float(sx[m]) * float(sw[n, g]) * (int(codes[n, k]) - int(zw[n, g])) * int(qx[m, k])
            assert y[m, n] == pytest.approx(acc, rel=1e-12, abs=1e-12)


def test_w4a4_path_stays_near_the_weight_only_path():
    # 4-bit activations add at most half a code step per element: the W4A4
    # output stays within the sum of |w^| * s_x / 2 of the W4A16 output
    p = linear_problem(42, 0, 1536, 64, 3, K=8)
    qw, sw, zw = oracle.pack_weights(p.W, p.pairs, p.cos_t, p.sin_t, p.scale)
    xt = oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale)
    y4, qx, sx = oracle.rotate_w4a4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale, qw, sw, zw)
    w_hat = oracle.dequantize(qw, sw, zw)
    y16 = oracle.linear(xt.astype(np.float32), w_hat)
    bound = np.abs(w_hat).sum(axis=1)[None, :] * (sx[:, None].astype(np.float64) / 2)
    assert (np.abs(y4 - y16) <= bound * (1 + 1e-6) + 1e-9).all()
