"""The dense-rotation contrast (paro_dense_rotate) against the oracle.

The dense matrix Q is that of the layer's own pairwise transform, diag(1/s)
R_K ... R_1, written out by the oracle and rounded to bf16, so the contrast
computes the same x~ as the pairwise path up to the rounding of Q and of the
bf16 output (page "ParoQuant: pairwise rotations that survive deployment",
section "Why it differs from a dense learned rotation")."""
import numpy as np
import pytest
import torch

import oracle
from synth import bf16_round, linear_problem
from tests.tolerances import assert_linear_close

pytestmark = pytest.mark.gpu

paro = pytest.importorskip("rotation_int4_weight_b200")
DEV = "cuda"


def dense_q(p):
    """Q with x~ = x Q^T: column i of Q is the transform of the i-th unit vector."""
    return oracle.rotate(np.eye(p.d_in), p.pairs, p.cos_t, p.sin_t, p.scale).T


def _dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV).to(torch.bfloat16)


@pytest.mark.parametrize("M,d", [(1, 512), (5, 1536), (300, 1024), (129, 4096)])
def test_dense_rotate_matches_the_oracle_product(M, d):
    p = linear_problem(501, M + d, d, 64, M)
    q32 = bf16_round(dense_q(p).astype(np.float32))
    got = paro.paro_dense_rotate(_dev_bf16(p.x), _dev_bf16(q32))
    assert paro.paro_get_device_status() == 0
    ref = p.x.astype(np.float64) @ q32.astype(np.float64).T
    assert_linear_close(got.float().cpu().numpy(), ref)
    # and Q is the pairwise transform: x Q^T agrees with it to bf16 rounding of Q
    xt = oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale)
    assert np.abs(ref - xt).max() <= 2e-2 * np.abs(xt).max()


@pytest.mark.parametrize("M", [1, 300])
def test_dense_contrast_before_the_same_int4_linear(M):
    """The INT4 linear on the dense path's own x~ matches the oracle on that x~;
    end to end, the bf16 matrix and the bf16 x~ leave the result within a few
    percent of the row rms of the exact transform's result (the contrast
    method's own rounding: the weights were folded with the exact transform)."""
    p = linear_problem(502, M, 1536, 512, M)
    tables = (torch.from_numpy(p.pairs.view(np.int16)).to(DEV), torch.from_numpy(p.cos_t).to(DEV),
              torch.from_numpy(p.sin_t).to(DEV), torch.from_numpy(p.scale).to(DEV))
    qw, sc, z = paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV), *tables)
    q = _dev_bf16(bf16_round(dense_q(p).astype(np.float32)))
    xt = paro.paro_dense_rotate(_dev_bf16(p.x), q)
    y = paro.paro_w4_linear(xt, qw, sc, z)
    assert paro.paro_get_device_status() == 0
    packed = (qw.cpu().numpy().view(np.uint32), sc.cpu().numpy(), z.cpu().numpy())
    y = y.float().cpu().numpy()
    assert_linear_close(y, oracle.w4_linear(xt.float().cpu().numpy(), *packed))
    exact = oracle.rotate_w4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale, *packed)
    rms = np.sqrt(np.mean(exact ** 2, axis=1, keepdims=True))
    assert np.max(np.abs(y - exact) / rms) < 0.1


def test_dense_rotate_rejects_widths_off_the_tile():
    x = torch.zeros(2, 96, dtype=torch.bfloat16, device=DEV)
    q = torch.zeros(96, 96, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(paro.ParoError, match="PARO_ERR_UNSUPPORTED"):
        paro.paro_dense_rotate(x, q)
