"""Plain, slow CPU oracle of the gradients of the activation-side transform.

TEST INFRASTRUCTURE ONLY: imported by the test suite and the bench's CPU
baseline, never by the CUDA library; it shares no code with the CUDA path.

Sources (page title, section):
  * "ParoQuant: Pairwise Rotation Quantization for Efficient Reasoning LLM
    Inference", abstract: the Givens rotations and the channel-wise scaling
    are optimizable parameters;
  * "ParoQuant: pairwise rotations that survive deployment", opening section
    (each pair has a learned Givens rotation plus channel-wise scaling) and
    section "From fake quantization to a real TensorRT engine" (the pairs are
    learned at calibration time, before the weights are transformed);
  * same page, section "A rotation small enough to execute": the forward
    transform whose gradients these are.

The pages give no backward pass.  This file takes the plain reading: for an
upstream gradient G = dL/dx~ of the transform x~ = diag(1/s) R_K ... R_1 x
(one row per token), the chain rule gives dL/dx, dL/dtheta for the angle of
every pair of every stage, and dL/ds for the channel scale, with
(c, s) = (cos theta, sin theta) and the rotation of a pair as printed
(x_i' = c x_i + s x_j, x_j' = -s x_i + c x_j):
  * d x_i'/d theta = -s x_i + c x_j = x_j',  d x_j'/d theta = -c x_i - s x_j = -x_i',
    so dL/dtheta = sum over tokens of (h_i x_j' - h_j x_i'), h = dL/dx' of the stage;
  * dL/dx of a stage is its transpose: g_i = c h_i - s h_j, g_j = s h_i + c h_j;
  * x~_c = x_c / s_c gives dL/ds_c = -sum over tokens of G_c x~_c / s_c and
    dL/dx_c = G_c / s_c at the output of the last stage.
The forward values of every stage are kept (not recomputed), and everything
runs in fp64.
"""
from __future__ import annotations

import numpy as np

from .paro import check_stage_disjoint, givens_stage


def rotate_backward(x: np.ndarray, grad: np.ndarray, pairs: np.ndarray, cos_t: np.ndarray, sin_t: np.ndarray,
                    scale: np.ndarray | None = None):
    """Gradients of L with dL/dx~ = grad through x~ = diag(1/s) R_K ... R_1 x.

    x, grad: [M, d]; pairs: [K, d/2, 2]; cos_t, sin_t: [K, d/2]; scale: [d] or
    None.  Returns (dx [M, d], dtheta [K, d/2], dscale [d] or None), fp64.
    """
    x = np.asarray(x, dtype=np.float64)
    G = np.asarray(grad, dtype=np.float64)
    K = np.asarray(pairs).shape[0]
    # forward, keeping the output of every stage: acts[k] = R_k ... R_1 x
    acts = [x]
    for k in range(K):
        acts.append(givens_stage(acts[-1], pairs[k], cos_t[k], sin_t[k]))
    dscale = None
    if scale is not None:
        s = np.asarray(scale, dtype=np.float64)
        xt = acts[K] / s
        dscale = -(G * xt).sum(axis=0) / s
        h = G / s
    else:
        h = G.copy()
    dtheta = np.zeros((K, np.asarray(pairs).shape[1]), dtype=np.float64)
    for k in range(K - 1, -1, -1):
        check_stage_disjoint(pairs[k], x.shape[-1])
        i = np.asarray(pairs[k][:, 0], dtype=np.intp)
        j = np.asarray(pairs[k][:, 1], dtype=np.intp)
        c = np.asarray(cos_t[k], dtype=np.float64)
        sn = np.asarray(sin_t[k], dtype=np.float64)
        xo = acts[k + 1]  # the stage's output
        hi, hj = h[:, i], h[:, j]
        dtheta[k] = (hi * xo[:, j] - hj * xo[:, i]).sum(axis=0)
        g = h.copy()
        g[:, i] = c * hi - sn * hj
        g[:, j] = sn * hi + c * hj
        h = g
    return h, dtheta, dscale
