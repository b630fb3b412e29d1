"""Oracle of the weight-activation (W4A4) variant of the path (numpy).

TEST INFRASTRUCTURE ONLY, like the rest of this package: imported by the test
suite and the bench's CPU-baseline leg, never by the CUDA library, and sharing
no code with it.

Source: page "ParoQuant: Pairwise Rotation Quantization for Efficient Reasoning
LLM Inference", section "Abstract (arXiv)": besides weight-only quantization,
the method is said to match the accuracy of weight-activation quantization
methods.  The pages give no detail of that setting, so this file takes the
plainest reading of "4-bit weights and 4-bit activations" on top of the
weight-only path:
  * the weights are the W4A16 path's packed INT4 weights unchanged (group-128
    asymmetric codes q_w in 0..15 with an integer zero point z and an fp16
    scale s_w per group, the transform folded in);
  * the activations are the transformed x~ (the activation-side transform
    first, as in the weight-only path), quantised per token (one scale per
    row of x~), symmetrically, to signed 4-bit codes: s_x = max_k |x~_k| / 7
    and q_x = clamp(rint(x~_k / s_x), -8, 7), in fp32 IEEE arithmetic with
    round-half-to-even; a row that is all zero takes s_x = 1 (codes 0);
  * the linear: y[m, n] = s_x[m] * sum_g s_w[n, g] * sum_{k in g}
    (q_w[n, k] - z[n, g]) * q_x[m, k], the inner sums exact integers.
"""
from __future__ import annotations

import numpy as np

from .paro import unpack_nibbles


def quantize_activations(xt):
    """Per-token symmetric INT4 codes of x~ [M, d] (any float type, taken as
    fp32): returns (codes int8 [M, d] in -8..7, scales fp32 [M])."""
    x = np.asarray(xt, dtype=np.float32)
    M, d = x.shape
    q = np.zeros((M, d), dtype=np.int8)
    s = np.ones(M, dtype=np.float32)
    for m in range(M):
        amax = np.float32(np.max(np.abs(x[m]))) if d else np.float32(0)
        if amax == 0:
            continue  # all-zero row: scale 1, codes 0
        s[m] = np.float32(amax / np.float32(7.0))
        r = np.rint(x[m] / s[m])  # fp32 division, then round half to even
        q[m] = np.clip(r, -8, 7).astype(np.int8)
    return q, s


def dequantize_activations(q, s):
    """x^ = q * s_x per row, fp64."""
    return np.asarray(q, dtype=np.float64) * np.asarray(s, dtype=np.float64)[:, None]


def w4a4_linear(qx, sx, qweight, scales, zeros, group_size=128):
    """y [M, d_out] (fp64) from activation codes and scales and the packed INT4
    weights, group by group: the integer sums first, then the scales."""
    qx = np.asarray(qx, dtype=np.int64)
    codes = unpack_nibbles(qweight).astype(np.int64)  # [d_out, d_in], 0..15
    sw = np.asarray(scales, dtype=np.float64)
    z = np.asarray(zeros, dtype=np.float64).astype(np.int64)
    M, d_in = qx.shape
    d_out = codes.shape[0]
    G = d_in // group_size
    y = np.zeros((M, d_out), dtype=np.float64)
    for g in range(G):
        k0, k1 = g * group_size, (g + 1) * group_size
        ints = qx[:, k0:k1] @ (codes[:, k0:k1] - z[:, g][:, None]).T  # [M, d_out], exact
        y += ints.astype(np.float64) * sw[:, g][None, :]
    return y * np.asarray(sx, dtype=np.float64)[:, None]


def rotate_w4a4_linear(x, pairs, cos_t, sin_t, scale, qweight, scales, zeros, xt_bf16=None):
    """The whole W4A4 path: transform, per-token INT4 codes, W4A4 linear.
    xt_bf16: the transformed activations to quantise, when the caller fixes
    them (the device path hands x~ to the quantiser in bf16); else the oracle's
    own fp64 transform rounded to fp32."""
    from .paro import rotate
    xt = rotate(x, pairs, cos_t, sin_t, scale) if xt_bf16 is None else xt_bf16
    qx, sx = quantize_activations(xt)
    return w4a4_linear(qx, sx, qweight, scales, zeros), qx, sx
