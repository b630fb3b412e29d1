"""The weight-activation (W4A4) variant on the GPU against its oracle
(oracle/w4a4.py), on the same seeded inputs (needs a B200).

Bit-exact: the activation codes and scales, computed by both sides in fp32
from the same bf16 input.  The linear: its inner sums are exact integers on
both sides, so the GPU's bf16 output may differ from the oracle's fp64 value
only by the fp32 rounding of the scaled group sums and the final bf16
rounding: at most one bf16 ulp of the value plus 1e-6 of the row's largest
output (asserted for every output element).
"""
import numpy as np
import pytest
import torch

import oracle
from synth import linear_problem

pytestmark = pytest.mark.gpu

paro = pytest.importorskip("rotation_int4_weight_b200")
DEV = "cuda"


def _bf16_ulp(v):
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_w4a4_close(got, ref):
    got = np.asarray(got, dtype=np.float64)
    bound = _bf16_ulp(ref) + 1e-6 * np.abs(ref).max(axis=1, keepdims=True)
    err = np.abs(got - ref)
    assert (err <= bound).all(), float((err - bound).max())


def _tables(p):
    return (torch.from_numpy(p.pairs.view(np.int16)).to(DEV), torch.from_numpy(p.cos_t).to(DEV),
            torch.from_numpy(p.sin_t).to(DEV), torch.from_numpy(p.scale).to(DEV))


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV).to(torch.bfloat16)


@pytest.mark.parametrize("M,d", [(1, 128), (3, 1536), (16, 8960), (33, 640), (2, 14336)])
def test_quantize_activations_bit_exact(M, d):
    rng = np.random.default_rng(M * 1000 + d)
    x = rng.standard_normal((M, d)) * rng.uniform(0.01, 30, (M, 1))
    x[0, d // 3] = 250.0                    # an outlier row
    if M > 2:
        x[2] = 0.0                          # an all-zero row: scale 1, codes 0
    xb = _bf16(x)
    q, sx = paro.paro_quantize_activations(xb)
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_activations(xb.float().cpu().numpy())
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def _packed(p):
    W = torch.from_numpy(p.W).to(DEV)
    return paro.paro_pack_weights(W, *_tables(p))


@pytest.mark.parametrize("M,d_in,d_out", [
    (1, 1536, 1536),     # several shares per 64-row tile
    (4, 8960, 1536),     # the widest Qwen2.5-1.5B input
    (16, 1536, 8960),    # two token tiles in one CTA
    (9, 512, 272),       # ragged output tail, one tile of nine tokens
    (33, 640, 96),       # three token blocks
    (2, 128, 19008),     # one share per tile (more tiles than two per SM)
])
def test_w4a4_linear_matches_oracle(M, d_in, d_out):
    p = linear_problem(71, 0, d_in, d_out, M, K=8)
    qw, sc, z = _packed(p)
    rng = np.random.default_rng(d_out)
    qx = torch.from_numpy(rng.integers(-8, 8, (M, d_in)).astype(np.int8)).to(DEV)
    sx = torch.from_numpy(rng.uniform(0.05, 3.0, M).astype(np.float32)).to(DEV)
    y = paro.paro_w4a4_linear(qx, sx, qw, sc, z)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    ref = oracle.w4a4_linear(qx.cpu().numpy(), sx.cpu().numpy(), qw.cpu().numpy().view(np.uint32),
                             sc.cpu().numpy(), z.cpu().numpy())
    assert_w4a4_close(y.float().cpu().numpy(), ref)
    y2 = paro.paro_w4a4_linear(qx, sx, qw, sc, z)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))  # fixed summation order


@pytest.mark.parametrize("M,d_in,d_out", [(1, 1536, 256), (1, 8960, 1536), (16, 1536, 1536), (5, 4096, 1040)])
def test_rotate_w4a4_linear_end_to_end(M, d_in, d_out):
    p = linear_problem(72, 0, d_in, d_out, M, K=8)
    tables = _tables(p)
    qw, sc, z = _packed(p)
    x = _bf16(p.x)
    y = paro.paro_rotate_w4a4_linear(x, *tables, qw, sc, z)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    # the same transform kernel alone gives the bf16 x~ the call quantised
    xt = paro.paro_rotate(x, *tables).float().cpu().numpy()
    ref, qx, sx = oracle.rotate_w4a4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale, qw.cpu().numpy().view(np.uint32),
                                            sc.cpu().numpy(), z.cpu().numpy(), xt_bf16=xt)
    assert_w4a4_close(y.float().cpu().numpy(), ref)


def test_w4a4_rejects_bad_shapes_without_launching():
    qx = torch.zeros(2, 200, dtype=torch.int8, device=DEV)
    sx = torch.ones(2, dtype=torch.float32, device=DEV)
    qw = torch.zeros(64, 25, dtype=torch.int32, device=DEV)
    sc = torch.ones(64, 1, dtype=torch.float16, device=DEV)
    with pytest.raises(paro.ParoError, match="multiple of 128"):
        paro.paro_w4a4_linear(qx, sx, qw, sc, sc)
    with pytest.raises(paro.ParoError, match="multiple of 8"):
        paro.paro_quantize_activations(torch.zeros(2, 12, dtype=torch.bfloat16, device=DEV))
