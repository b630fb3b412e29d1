"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties one oracle function to something other than itself: a worked
example, an invariant, a closed form, an exhaustive enumeration or a
brute-force computation written differently from the oracle.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from synth import bf16_round, linear_problem

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _tables(g):
    pairs = np.array([st["pairs"] for st in g["stages"]], dtype=np.uint16)
    cos_t = np.array([st["cos"] for st in g["stages"]], dtype=np.float64)
    sin_t = np.array([st["sin"] for st in g["stages"]], dtype=np.float64)
    return pairs, cos_t, sin_t


def _random_tables(rng, d, K):
    pairs = np.stack([rng.permutation(d).reshape(d // 2, 2) for _ in range(K)]).astype(np.uint16)
    theta = rng.uniform(-math.pi, math.pi, size=(K, d // 2))
    return pairs, np.cos(theta), np.sin(theta)


# ---------------------------------------------------------------- rotation
def test_hand_example_stages_and_scale():
    g = _load("hand_example_4ch_2stage.json")
    pairs, c, s = _tables(g)
    x = np.array([g["x"]])
    tol = g["tolerance"]
    y1 = oracle.givens_stage(x, pairs[0], c[0], s[0])
    np.testing.assert_allclose(y1[0], g["after_stage_1"], rtol=0, atol=tol)
    y2 = oracle.givens_stage(y1, pairs[1], c[1], s[1])
    np.testing.assert_allclose(y2[0], g["after_stage_2"], rtol=0, atol=tol)
    xt = oracle.rotate(x, pairs, c, s, np.array(g["scale"]))
    np.testing.assert_allclose(xt[0], g["x_tilde"], rtol=0, atol=tol)


def test_hand_example_fold_preserves_dot():
    g = _load("hand_example_4ch_2stage.json")
    pairs, c, s = _tables(g)
    w = np.array([g["w"]])
    wt = oracle.fold_weights(w, pairs, c, s, np.array(g["scale"]))
    np.testing.assert_allclose(wt[0], g["w_tilde"], rtol=0, atol=g["tolerance"])
    xt = oracle.rotate(np.array([g["x"]]), pairs, c, s, np.array(g["scale"]))
    assert abs(float(xt[0] @ wt[0]) - g["w_tilde_dot_x_tilde"]) < g["tolerance"]
    assert abs(float(np.dot(g["w"], g["x"])) - g["w_dot_x"]) < g["tolerance"]


def test_pair_norm_preserved():
    rng = np.random.default_rng(1)
    d = 64
    pairs, c, s = _random_tables(rng, d, 1)
    x = rng.standard_normal((3, d))
    y = oracle.givens_stage(x, pairs[0], c[0], s[0])
    i, j = pairs[0, :, 0].astype(int), pairs[0, :, 1].astype(int)
    n0 = np.hypot(x[:, i], x[:, j])
    n1 = np.hypot(y[:, i], y[:, j])
    np.testing.assert_allclose(n1, n0, rtol=1e-15, atol=0)
    # the rotation really moves the values (not a no-op)
    assert np.max(np.abs(y - x)) > 0.1


def test_zero_angle_is_identity_and_quarter_turn_is_signed_swap():
    rng = np.random.default_rng(2)
    d = 16
    pairs = rng.permutation(d).reshape(1, d // 2, 2).astype(np.uint16)
    x = rng.standard_normal((2, d))
    y = oracle.givens_stage(x, pairs[0], np.ones(d // 2), np.zeros(d // 2))
    assert np.array_equal(y, x)
    y = oracle.givens_stage(x, pairs[0], np.zeros(d // 2), np.ones(d // 2))
    i, j = pairs[0, :, 0].astype(int), pairs[0, :, 1].astype(int)
    assert np.array_equal(y[:, i], x[:, j])
    assert np.array_equal(y[:, j], -x[:, i])


def test_orientation_flip_with_negated_sine_is_bit_identical():
    rng = np.random.default_rng(3)
    d, K = 128, 4
    pairs, c, s = _random_tables(rng, d, K)
    x = rng.standard_normal((5, d))
    flipped = pairs[:, :, ::-1].copy()
    a = oracle.rotate(x, pairs, c, s)
    b = oracle.rotate(x, flipped, c, -s)
    assert np.array_equal(a, b)


def test_order_of_pairs_within_stage_is_irrelevant():
    rng = np.random.default_rng(4)
    d, K = 256, 8
    pairs, c, s = _random_tables(rng, d, K)
    x = rng.standard_normal((3, d))
    perm = np.stack([rng.permutation(d // 2) for _ in range(K)])
    p2 = np.stack([pairs[k][perm[k]] for k in range(K)])
    c2 = np.stack([c[k][perm[k]] for k in range(K)])
    s2 = np.stack([s[k][perm[k]] for k in range(K)])
    assert np.array_equal(oracle.rotate(x, pairs, c, s), oracle.rotate(x, p2, c2, s2))


def _dense_stage(d, pairs_k, c_k, s_k):
    """Dense d x d matrix of one stage, built from the printed 2x2 block."""
    R = np.eye(d)
    for (i, j), c, s in zip(pairs_k.astype(int), c_k, s_k):
        R[i, i], R[i, j] = c, s
        R[j, i], R[j, j] = -s, c
    return R


def test_rotation_equals_dense_matrix_product_and_is_orthogonal():
    rng = np.random.default_rng(5)
    d, K = 32, 8
    pairs, c, s = _random_tables(rng, d, K)
    scale = np.exp(0.3 * rng.standard_normal(d))
    R = np.eye(d)
    for k in range(K):
        R = _dense_stage(d, pairs[k], c[k], s[k]) @ R   # R_k ... R_1
    np.testing.assert_allclose(R.T @ R, np.eye(d), atol=1e-13)
    x = rng.standard_normal((4, d))
    expect = (np.diag(1.0 / scale) @ R @ x.T).T
    np.testing.assert_allclose(oracle.rotate(x, pairs, c, s, scale), expect, rtol=0, atol=1e-12)
    W = rng.standard_normal((6, d))
    expect_w = (np.diag(scale) @ R @ W.T).T
    np.testing.assert_allclose(oracle.fold_weights(W, pairs, c, s, scale), expect_w, rtol=0, atol=1e-12)


def test_inverse_after_forward_is_identity():
    rng = np.random.default_rng(6)
    d, K = 512, 8
    pairs, c, s = _random_tables(rng, d, K)
    scale = np.exp(0.3 * rng.standard_normal(d))
    x = rng.standard_normal((4, d))
    xt = oracle.rotate(x, pairs, c, s, scale)
    y = xt * scale                        # undo diag(1/s)
    for k in reversed(range(K)):          # R_k^T is the stage with sin negated
        y = oracle.givens_stage(y, pairs[k], c[k], -s[k])
    np.testing.assert_allclose(y, x, rtol=0, atol=1e-12 * np.abs(x).max())


def test_fold_then_transform_reproduces_unquantised_linear():
    # fp64 cos/sin of the drawn angles: exactly orthogonal up to fp64 rounding
    p = linear_problem(99, 0, 512, 96, 4, K=8)
    c, s = np.cos(p.theta), np.sin(p.theta)
    xt = oracle.rotate(p.x, p.pairs, c, s, p.scale)
    wt = oracle.fold_weights(p.W, p.pairs, c, s, p.scale)
    y_fold = oracle.linear(xt, wt)
    y_ref = p.x.astype(np.float64) @ p.W.astype(np.float64).T
    err = np.abs(y_fold - y_ref).max() / np.abs(y_ref).max()
    assert err < 1e-10


def test_pack_weights_scale_only_branch():
    """K = 0 with a channel scale: the packed weights are those of W diag(s),
    column c multiplied by s_c (the fold with no stage, page "ParoQuant:
    pairwise rotations that survive deployment", section "A rotation small
    enough to execute"), so that W~ (x / s) = W x up to quantisation."""
    p = linear_problem(98, 0, 256, 32, 3, K=8)
    W, s = p.W, p.scale
    # the closed form, one column at a time
    ws = np.empty(W.shape, dtype=np.float64)
    for c in range(p.d_in):
        ws[:, c] = W[:, c].astype(np.float64) * float(s[c])
    q, sc, z = oracle.quantize_groups(ws.astype(np.float32))
    qw, scw, zw = oracle.pack_weights(W, None, None, None, s)
    assert np.array_equal(qw, oracle.pack_nibbles(q))
    assert np.array_equal(scw.view(np.uint16), sc.view(np.uint16))
    assert np.array_equal(zw, z.astype(np.float16))
    # the same as a fold with zero stages, and as pack_weights given empty tables
    empty = (p.pairs[:0], p.cos_t[:0], p.sin_t[:0])
    assert np.array_equal(oracle.fold_weights(W, *empty, s), ws)
    qe, sce, ze = oracle.pack_weights(W, *empty, s)
    assert np.array_equal(qe, qw) and np.array_equal(sce, scw) and np.array_equal(ze, zw)
    # a divide (or no scale at all) would give other codes
    assert not np.array_equal(oracle.pack_weights(W, None, None, None, None)[0], qw)
    # and the scaled activations undo it: W^ (x / s) stays within the quantisation
    # bound of W x, row by row
    xs = p.x.astype(np.float64) / s.astype(np.float64)
    y = oracle.linear(xs, oracle.dequantize(qw, scw, zw))
    y_ref = p.x.astype(np.float64) @ W.astype(np.float64).T
    step = np.repeat(scw.astype(np.float64), 128, axis=1)          # [d_out, d_in]
    bound = np.abs(xs) @ (step / 2 + 15 * step * 2.0 ** -11).T     # [M, d_out]
    assert np.all(np.abs(y - y_ref) <= bound + 1e-12)


def test_non_disjoint_stage_is_rejected():
    pairs = np.array([[0, 1], [1, 2]], dtype=np.uint16)
    with pytest.raises(ValueError):
        oracle.givens_stage(np.zeros((1, 4)), pairs, np.ones(2), np.zeros(2))


# ---------------------------------------------------------------- quantisation
def test_worked_group():
    g = _load("quant_group_worked.json")
    v = np.full((1, g["group_size"]), g["rest_of_group"], dtype=np.float32)
    v[0, :4] = np.array(g["values_head"], dtype=np.float32)
    q, sc, z = oracle.quantize_groups(v, g["group_size"])
    assert sc.view(np.uint16)[0, 0] == int(g["scale_fp16_bits"], 16)
    assert float(sc[0, 0]) == g["scale_value"]
    assert int(z[0, 0]) == g["zero"]
    assert q[0, :4].tolist() == g["codes_head"]
    assert np.all(q[0, 4:] == g["code_of_rest"])
    qw = oracle.pack_nibbles(q)
    deq = oracle.dequantize(qw, sc, z.astype(np.float16), g["group_size"])
    assert deq[0, 1] == g["dequant_of_0.45"]
    assert deq[0, 2] == 0.0


def test_degenerate_groups():
    v = np.zeros((4, 128), dtype=np.float32)
    v[1, :] = 0.5          # constant positive group: range [0, 0.5]
    v[2, 7] = -1e-30       # a range so small its fp16 scale is zero
    v[3, :] = -0.5         # constant negative group: range [-0.5, 0]
    q, sc, z = oracle.quantize_groups(v)
    assert float(sc[0, 0]) == 1.0 and z[0, 0] == 0 and np.all(q[0] == 0)
    assert z[1, 0] == 0 and np.all(q[1] == 15)
    assert float(sc[1, 0]) == float(np.float16(np.float32(0.5) / np.float32(15)))
    assert float(sc[2, 0]) == 1.0 and z[2, 0] == 0 and np.all(q[2] == 0)
    assert float(sc[3, 0]) == float(sc[1, 0]) and z[3, 0] == 15 and np.all(q[3] == 0)


def test_quantisation_error_bound_and_exact_zero():
    rng = np.random.default_rng(7)
    v = (rng.standard_normal((64, 1024)) * 0.02).astype(np.float32)
    v[:, 5] *= 10
    q, sc, z = oracle.quantize_groups(v)
    assert q.max() <= 15 and z.max() <= 15
    deq = oracle.dequantize(oracle.pack_nibbles(q), sc, z.astype(np.float16))
    scale_full = np.repeat(sc.astype(np.float64), 128, axis=1)
    err = np.abs(deq - v.astype(np.float64))
    # half a step of rounding plus the fp16 rounding of the scale stretched over <= 15 steps
    bound = scale_full / 2 + 15 * scale_full * 2.0 ** -11
    assert np.all(err <= bound)
    # zero is on the grid: an exact 0 weight gets the zero point and dequantises to 0
    v0 = v.copy()
    v0[:, 0::128] = 0.0
    q0, sc0, z0 = oracle.quantize_groups(v0)
    assert np.array_equal(q0[:, 0::128], z0)
    deq0 = oracle.dequantize(oracle.pack_nibbles(q0), sc0, z0.astype(np.float16))
    assert np.all(deq0[:, 0::128] == 0.0)
    # the grid ends cover the range
    vg = v.reshape(64, 8, 128).astype(np.float64)
    lo = (0 - z.astype(np.float64)) * sc
    hi = (15 - z.astype(np.float64)) * sc
    assert np.all(lo <= np.minimum(vg.min(axis=2), 0) + sc.astype(np.float64) / 2 + 1e-12)
    assert np.all(hi >= np.maximum(vg.max(axis=2), 0) - sc.astype(np.float64) / 2 - 1e-12)


def test_pack_word_layout():
    q = np.arange(1, 9, dtype=np.uint8).reshape(1, 8)
    assert oracle.pack_nibbles(q)[0, 0] == 0x87654321


def test_pack_against_little_endian_bytes():
    rng = np.random.default_rng(8)
    q = rng.integers(0, 16, size=(7, 256), dtype=np.uint8)
    words = oracle.pack_nibbles(q)
    # independent route: byte b of a little-endian word holds columns 2b (low) and 2b+1 (high)
    by = words.astype("<u4").view(np.uint8).reshape(7, 256 // 2)
    lo = by & 0xF
    hi = by >> 4
    rebuilt = np.empty_like(q)
    rebuilt[:, 0::2] = lo
    rebuilt[:, 1::2] = hi
    assert np.array_equal(rebuilt, q)
    assert np.array_equal(oracle.unpack_nibbles(words), q)


def test_dequant_exhaustive_codes_and_zeros():
    codes = np.array(list(itertools.product(range(16), range(16))), dtype=np.int64)  # (q, z)
    n = codes.shape[0]
    q = np.repeat(codes[:, :1], 128, axis=1).astype(np.uint8)
    sc = np.full((n, 1), 0.04998779296875, dtype=np.float16)
    z = codes[:, 1:2].astype(np.float16)
    deq = oracle.dequantize(oracle.pack_nibbles(q), sc, z)
    for r, (qq, zz) in enumerate(codes.tolist()):
        assert np.all(deq[r] == (qq - zz) * 0.04998779296875)


# ---------------------------------------------------------------- linear
def test_linear_against_python_loops():
    rng = np.random.default_rng(9)
    M, d_in, d_out = 3, 256, 5
    q = rng.integers(0, 16, size=(d_out, d_in), dtype=np.uint8)
    sc = (rng.uniform(0.001, 0.01, size=(d_out, d_in // 128))).astype(np.float16)
    z = rng.integers(0, 16, size=(d_out, d_in // 128)).astype(np.float16)
    x = rng.standard_normal((M, d_in))
    y = oracle.w4_linear(x, oracle.pack_nibbles(q), sc, z)
    for m in range(M):
        for n in range(d_out):
            acc = 0.0
            for k in range(d_in):
                acc += (int(q[n, k]) - float(z[n, k // 128])) * float(sc[n, k // 128]) * x[m, k]
            assert abs(acc - y[m, n]) <= 1e-12 * max(1.0, abs(acc))


def test_rotate_w4_linear_is_composition():
    p = linear_problem(11, 0, 256, 16, 2, K=4)
    qw, sc, z = oracle.pack_weights(p.W, p.pairs, p.cos_t, p.sin_t, p.scale)
    y = oracle.rotate_w4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale, qw, sc, z)
    xt = oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale)
    assert np.array_equal(y, oracle.linear(xt, oracle.dequantize(qw, sc, z)))
    # the quantised product stays within the per-weight error bound of the
    # unquantised folded product: |y - W~ x~| <= sum_k |x~_k| * err_bound_k
    wt = oracle.fold_weights(p.W, p.pairs, p.cos_t, p.sin_t, p.scale).astype(np.float32)
    y_fp = oracle.linear(xt, wt.astype(np.float64))
    step = np.repeat(sc.astype(np.float64), 128, axis=1)
    bound = np.abs(xt) @ (step / 2 + 15 * step * 2.0 ** -11).T
    assert np.all(np.abs(y - y_fp) <= bound + 1e-12)


# ---------------------------------------------------------------- inputs
def test_synthetic_problem_structure():
    p = linear_problem(5, 3, 512, 64, 4, K=8)
    for k in range(8):
        assert np.array_equal(np.sort(p.pairs[k].reshape(-1)), np.arange(512))
    assert np.array_equal(bf16_round(p.x), p.x)
    assert p.x.dtype == np.float32 and p.W.dtype == np.float32
    q = linear_problem(5, 3, 512, 64, 4, K=8)
    assert np.array_equal(p.pairs, q.pairs) and np.array_equal(p.W, q.W)
    r = linear_problem(5, 4, 512, 64, 4, K=8)
    assert not np.array_equal(p.pairs, r.pairs)
    assert abs(float(p.cos_t[0, 0]) ** 2 + float(p.sin_t[0, 0]) ** 2 - 1) < 1e-6


def test_bf16_round_ties_to_even():
    a = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9], dtype=np.float32)
    r = bf16_round(a)
    assert r.tolist() == [1.0, 1.0 + 2 ** -6, 1.0]
