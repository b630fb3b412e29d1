"""Plain, slow CPU oracle of the ParoQuant runtime hot path (numpy).

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
bench's CPU-baseline leg, never by the CUDA library.  It shares no code with
the CUDA path.

Sources (page title, section):
  * "ParoQuant: pairwise rotations that survive deployment",
    section "A rotation small enough to execute": the Givens rotation of one
    channel pair (the printed 2x2 matrix), disjoint pairs inside a stage,
    several stages, channel-wise scaling after the rotations, the weight-side
    transform folded in at build time and the activation-side transform run
    right before the packed INT4 linear;
  * same page, section "My reduced-calibration experiment": INT4 weights in
    groups of 128 input columns;
  * same page, section "From fake quantization to a real TensorRT engine":
    real INT4 packing, one rotation operator and one group-wise INT4 GEMM per
    linear layer.

Where the pages leave a step open, this file takes these readings:
  * stage k = 0 (R_1) is applied first; the channel scale comes after all
    stages and divides: x~ = diag(1/s) R_K ... R_1 x;
  * a pair (i, j) is rotated as printed: x_i' = c x_i + s x_j,
    x_j' = -s x_i + c x_j, with (i, j) in stored order;
  * the weight side gets the inverse-transpose of the activation transform,
    which for orthogonal R is the same stages followed by a multiply by s:
    w~_n = diag(s) R_K ... R_1 w_n, so that W~ x~ = W x;
  * quantisation is asymmetric with an integer zero point: per group of 128
    input columns, range [min(0, min v), max(0, max v)], fp16 scale
    (max - min) / 15, zero rint(-min / scale) in 0..15, codes
    clamp(rint(v / scale) + zero, 0, 15); an all-zero group (scale rounds to
    fp16 zero) takes scale 1 and zero 0.  All of this in fp32 IEEE arithmetic
    with round-half-to-even, in exactly this operation order;
  * packing: eight 4-bit codes per uint32 along the input dimension, code of
    column 8w+e in bits [4e, 4e+4) of word w, words row-major [d_out][d_in/8].
Rotation, fold, dequantisation and the matmul run in fp64.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32


def check_stage_disjoint(pairs_k: np.ndarray, d: int) -> None:
    """A stage is a set of disjoint pairs: no channel may appear twice."""
    flat = np.asarray(pairs_k, dtype=np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= d):
        raise ValueError("pair index out of range")
    if np.unique(flat).size != flat.size:
        raise ValueError("pairs of one stage are not disjoint")


def givens_stage(x: np.ndarray, pairs_k: np.ndarray, c_k: np.ndarray, s_k: np.ndarray) -> np.ndarray:
    """One stage of independent Givens rotations, applied to the last axis of x.

    For every pair (i, j) of the stage, with (c, s) = (cos theta, sin theta):
        x_i <- c * x_i + s * x_j
        x_j <- -s * x_i + c * x_j
    both computed from the values before the stage (the pairs are disjoint, so
    the result does not depend on the order of the pairs).
    """
    x = np.asarray(x, dtype=np.float64)
    check_stage_disjoint(pairs_k, x.shape[-1])
    i = np.asarray(pairs_k[:, 0], dtype=np.intp)
    j = np.asarray(pairs_k[:, 1], dtype=np.intp)
    c = np.asarray(c_k, dtype=np.float64)
    s = np.asarray(s_k, dtype=np.float64)
    a = x[..., i]
    b = x[..., j]
    out = x.copy()
    out[..., i] = c * a + s * b
    out[..., j] = (-s) * a + c * b
    return out


def rotate(x: np.ndarray, pairs: np.ndarray, cos_t: np.ndarray, sin_t: np.ndarray,
           scale: np.ndarray | None = None) -> np.ndarray:
    """Activation-side transform x~ = diag(1/s) R_K ... R_1 x, one row per token.

    x: [M, d] (any float dtype, used as fp64); pairs: [K, d/2, 2];
    cos_t, sin_t: [K, d/2]; scale: [d] or None (no scaling).  Returns fp64.
    """
    y = np.asarray(x, dtype=np.float64)
    for k in range(np.asarray(pairs).shape[0]):
        y = givens_stage(y, pairs[k], cos_t[k], sin_t[k])
    if scale is not None:
        y = y / np.asarray(scale, dtype=np.float64)
    return y


def fold_weights(W: np.ndarray, pairs: np.ndarray, cos_t: np.ndarray, sin_t: np.ndarray,
                 scale: np.ndarray | None = None) -> np.ndarray:
    """Build-time weight transform w~_n = diag(s) R_K ... R_1 w_n for every row n.

    Since x~ = D^-1 R x with R orthogonal, W x = (W R^T D) x~, whose row n is
    D R w_n: the same stages as the activations, then a multiply by s.  fp64.
    """
    y = np.asarray(W, dtype=np.float64)
    for k in range(np.asarray(pairs).shape[0]):
        y = givens_stage(y, pairs[k], cos_t[k], sin_t[k])
    if scale is not None:
        y = y * np.asarray(scale, dtype=np.float64)
    return y


def quantize_groups(wt: np.ndarray, group: int = 128):
    """Asymmetric INT4 quantisation of fp32 weights in groups along the input dim.

    Returns (q uint8 [d_out, d_in], scales fp16 [d_out, d_in/group],
    zeros uint8 [d_out, d_in/group]).  fp32 IEEE arithmetic, half-to-even.
    """
    wt = np.asarray(wt, dtype=np.float32)
    n, d = wt.shape
    if d % group:
        raise ValueError("d_in must be a multiple of the group size")
    v = wt.reshape(n, d // group, group)
    mn = np.minimum(v.min(axis=2), F32(0.0))
    mx = np.maximum(v.max(axis=2), F32(0.0))
    s32 = (mx - mn) / F32(15.0)
    sc = s32.astype(np.float16)
    degenerate = sc == np.float16(0.0)
    sc = np.where(degenerate, np.float16(1.0), sc)
    scf = sc.astype(np.float32)
    z = np.clip(np.rint((-mn) / scf), F32(0.0), F32(15.0))
    z = np.where(degenerate, F32(0.0), z)
    q = np.clip(np.rint(v / scf[..., None]) + z[..., None], F32(0.0), F32(15.0))
    return q.reshape(n, d).astype(np.uint8), sc, z.astype(np.uint8)


def pack_nibbles(q: np.ndarray) -> np.ndarray:
    """Pack 4-bit codes [d_out, d_in] into uint32 [d_out, d_in/8]; column 8w+e -> bits 4e..4e+3."""
    q = np.asarray(q, dtype=np.uint32)
    n, d = q.shape
    if d % 8:
        raise ValueError("d_in must be a multiple of 8")
    q8 = q.reshape(n, d // 8, 8)
    words = np.zeros((n, d // 8), dtype=np.uint32)
    for e in range(8):
        words |= (q8[:, :, e] & np.uint32(0xF)) << np.uint32(4 * e)
    return words


def unpack_nibbles(qweight: np.ndarray) -> np.ndarray:
    """Inverse of pack_nibbles: uint32 [d_out, d_in/8] -> uint8 codes [d_out, d_in]."""
    w = np.asarray(qweight, dtype=np.uint32)
    n, nw = w.shape
    out = np.empty((n, nw, 8), dtype=np.uint8)
    for e in range(8):
        out[:, :, e] = (w >> np.uint32(4 * e)) & np.uint32(0xF)
    return out.reshape(n, nw * 8)


def pack_weights(W: np.ndarray, pairs: np.ndarray | None, cos_t, sin_t, scale, group: int = 128):
    """Build-time path: fold (fp64) -> round to fp32 -> quantise -> pack.

    Returns (qweight uint32 [d_out, d_in/8], scales fp16 [d_out, G], zeros fp16 [d_out, G]).
    pairs=None (or K = 0) and scale=None give the plain INT4 weights without rotation.
    """
    if pairs is not None and np.asarray(pairs).shape[0] > 0:
        wt = fold_weights(W, pairs, cos_t, sin_t, scale)
    elif scale is not None:
        wt = np.asarray(W, dtype=np.float64) * np.asarray(scale, dtype=np.float64)
    else:
        wt = np.asarray(W, dtype=np.float64)
    q, sc, z = quantize_groups(wt.astype(np.float32), group)
    return pack_nibbles(q), sc, z.astype(np.float16)


def dequantize(qweight: np.ndarray, scales: np.ndarray, zeros: np.ndarray, group: int = 128) -> np.ndarray:
    """w^ = (q - z) * scale per group, exact in fp64.  Returns [d_out, d_in]."""
    q = unpack_nibbles(qweight).astype(np.float64)
    n, d = q.shape
    sc = np.asarray(scales, dtype=np.float64)
    z = np.asarray(zeros, dtype=np.float64)
    return ((q.reshape(n, d // group, group) - z[..., None]) * sc[..., None]).reshape(n, d)


def linear(xt: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """y[m, n] = sum_k w^[n, k] x~[m, k] in fp64 (library matmul)."""
    return np.asarray(xt, dtype=np.float64) @ np.asarray(w_hat, dtype=np.float64).T


def w4_linear(x: np.ndarray, qweight, scales, zeros, group: int = 128) -> np.ndarray:
    """The group-wise INT4 weight-only linear on already-transformed activations."""
    return linear(x, dequantize(qweight, scales, zeros, group))


def rotate_w4_linear(x, pairs, cos_t, sin_t, scale, qweight, scales, zeros, group: int = 128):
    """The runtime path: activation transform right before the packed INT4 linear."""
    return w4_linear(rotate(x, pairs, cos_t, sin_t, scale), qweight, scales, zeros, group)
