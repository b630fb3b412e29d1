"""Failure detection on the GPU without a fault: bounded waits that run out,
and an fp16 range overflow, reported through the device status word.

A hand-over flag that nothing sets is made on the host: the test hook
paro_set_test_hooks makes the decode transforms skip publishing their
"x~ is written" flags and bounds the INT4 kernel's flag waits to a fraction
of a millisecond.  The call must then report PARO_ERR_TIMEOUT, leave every
output tile unwritten, and leave the context usable: the same call after the
hooks are reset matches the oracle.  Nothing traps or hangs (every wait in
the kernels is bounded).
"""
import numpy as np
import pytest
import torch

import oracle
from synth import linear_problem
from tests.tolerances import assert_linear_close

pytestmark = pytest.mark.gpu

paro = pytest.importorskip("rotation_int4_weight_b200")
DEV = "cuda"
TIMEOUT, RANGE = 4, 5


def _layer(seed, shapes, M):
    probs, devs = [], []
    for i, (d_in, d_out) in enumerate(shapes):
        p = linear_problem(seed, i, d_in, d_out, M)
        tables = (torch.from_numpy(p.pairs.view(np.int16)).to(DEV), torch.from_numpy(p.cos_t).to(DEV),
                  torch.from_numpy(p.sin_t).to(DEV), torch.from_numpy(p.scale).to(DEV))
        qw, sc, z = paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV), *tables)
        x = torch.from_numpy(p.x).to(DEV).to(torch.bfloat16)
        y = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device=DEV)
        probs.append(p)
        devs.append(dict(x=x, tables=tables, qw=qw, sc=sc, z=z, y=y))
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    return probs, devs, layers


@pytest.mark.parametrize("M", [1, 4, 16])
def test_dropped_ready_flags_time_out_without_writing_output(M):
    # M = 1: the fused one-launch form; 4 and 16: the transform launch, then the
    # INT4 launch that waits for each linear's transform CTAs
    shapes = [(1536, 1536), (1536, 256), (8960, 1536), (1536, 2048)]
    probs, devs, layers = _layer(301 + M, shapes, M)
    assert paro.paro_get_device_status() == 0
    try:
        paro.paro_set_test_hooks(200_000, True)
        ws = paro.paro_rotate_w4_linear_batched(layers)
        torch.cuda.synchronize()
    finally:
        paro.paro_set_test_hooks(0, False)
    assert paro.paro_get_device_status() == TIMEOUT
    for d in devs:
        assert torch.isnan(d["y"].float()).all(), "a tile was written although its activations never came"
    assert paro.paro_get_device_status() == 0  # read and cleared
    # the context is still usable: the same call, hooks reset, is correct
    paro.paro_rotate_w4_linear_batched(layers, workspace=ws)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    for p, d in zip(probs, devs):
        ref = oracle.rotate_w4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale,
                                      d["qw"].cpu().numpy().view(np.uint32), d["sc"].cpu().numpy(),
                                      d["z"].cpu().numpy())
        assert_linear_close(d["y"].float().cpu().numpy(), ref)


def test_short_flag_wait_alone_still_completes_a_small_call():
    # with the flags published, a bound of a few million cycles is plenty for a
    # small layer: the hook by itself does not make calls fail
    probs, devs, layers = _layer(311, [(512, 512), (1024, 128)], 1)
    try:
        paro.paro_set_test_hooks(20_000_000, False)
        paro.paro_rotate_w4_linear_batched(layers)
        torch.cuda.synchronize()
    finally:
        paro.paro_set_test_hooks(0, False)
    assert paro.paro_get_device_status() == 0
    for d in devs:
        assert torch.isfinite(d["y"].float()).all()


def _huge_x(M, d, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, d, generator=g) * 1e6  # far beyond the fp16 range (65504)
    return x.to(DEV).to(torch.bfloat16)


@pytest.mark.parametrize("M", [1, 4, 300])
def test_fp16_overflow_of_the_transformed_activations_is_reported(M):
    p = linear_problem(321, M, 1536, 256, M)
    tables = (torch.from_numpy(p.pairs.view(np.int16)).to(DEV), torch.from_numpy(p.cos_t).to(DEV),
              torch.from_numpy(p.sin_t).to(DEV), torch.from_numpy(p.scale).to(DEV))
    qw, sc, z = paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV), *tables)
    assert paro.paro_get_device_status() == 0
    paro.paro_rotate_w4_linear(_huge_x(M, 1536, M), *tables, qw, sc, z)
    assert paro.paro_get_device_status() == RANGE
    # the same call on ordinary activations reports nothing
    paro.paro_rotate_w4_linear(torch.from_numpy(p.x).to(DEV).to(torch.bfloat16), *tables, qw, sc, z)
    assert paro.paro_get_device_status() == 0
    # bf16 output of the standalone transform has the range: nothing to report
    paro.paro_rotate(_huge_x(M, 1536, M + 1), *tables)
    assert paro.paro_get_device_status() == 0


def test_fp16_overflow_of_bf16_inputs_on_the_tensor_cores_is_reported():
    # many tokens, no transform: the tensor-core kernel rounds bf16 inputs to fp16
    p = linear_problem(331, 0, 512, 256, 256)
    qw, sc, z = paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV))
    assert paro.paro_get_device_status() == 0
    paro.paro_w4_linear(_huge_x(256, 512, 7), qw, sc, z)
    assert paro.paro_get_device_status() == RANGE
    paro.paro_w4_linear(torch.from_numpy(p.x).to(DEV).to(torch.bfloat16), qw, sc, z)
    assert paro.paro_get_device_status() == 0


@pytest.mark.parametrize("M", [1, 4])
def test_bad_pair_index_in_a_layer_is_reported_and_others_are_correct(M):
    # a channel index >= d in one linear's tables: the transform clamps it into
    # range (every access stays inside the rows) and reports
    # PARO_ERR_INVALID_ARG (that linear's result is void), but still hands its
    # x~ over, so the call ends at once (no bounded wait runs out) and every
    # other linear of the call is correct
    shapes = [(1536, 256), (8960, 1536), (1536, 512)]
    probs, devs, layers = _layer(331 + M, shapes, M)
    bad = probs[1].pairs.copy()
    bad[4, 100, 0] = 9000  # >= d = 8960, in stage 4
    devs[1]["tables"] = (torch.from_numpy(bad.view(np.int16)).to(DEV),) + devs[1]["tables"][1:]
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    assert paro.paro_get_device_status() == 0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    paro.paro_rotate_w4_linear_batched(layers)
    end.record()
    torch.cuda.synchronize()
    assert start.elapsed_time(end) < 100.0  # milliseconds: no wait ran to its bound
    assert paro.paro_get_device_status() == 1  # PARO_ERR_INVALID_ARG
    for i in (0, 2):
        p, d = probs[i], devs[i]
        ref = oracle.rotate_w4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale,
                                      d["qw"].cpu().numpy().view(np.uint32), d["sc"].cpu().numpy(),
                                      d["z"].cpu().numpy())
        assert_linear_close(d["y"].float().cpu().numpy(), ref)
