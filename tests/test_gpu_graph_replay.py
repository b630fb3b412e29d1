"""Calls captured in a CUDA graph and replayed with new inputs each time.

A decode loop captures its layer calls once and replays them every step with
new activations in the same buffers.  Every hand-over between CTAs (the
transform's "x~ is written" flags, the partial sums of tiles split between
CTAs) must then be recognised as this replay's, never the previous one's:
each replay here is compared with the oracle on the inputs it was given."""
import numpy as np
import pytest
import torch

import oracle
from synth import linear_problem
from tests.tolerances import assert_linear_close

pytestmark = pytest.mark.gpu

paro = pytest.importorskip("rotation_int4_weight_b200")
DEV = "cuda"


def _layer(seed, shapes, M, rotate=True):
    probs, devs = [], []
    for i, (d_in, d_out) in enumerate(shapes):
        p = linear_problem(seed, i, d_in, d_out, M)
        tables = ((torch.from_numpy(p.pairs.view(np.int16)).to(DEV), torch.from_numpy(p.cos_t).to(DEV),
                   torch.from_numpy(p.sin_t).to(DEV), torch.from_numpy(p.scale).to(DEV)) if rotate
                  else (None, None, None, None))
        qw, sc, z = paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV), *tables)
        x = torch.empty(M, d_in, dtype=torch.bfloat16, device=DEV)
        y = torch.empty(M, d_out, dtype=torch.bfloat16, device=DEV)
        probs.append(p)
        devs.append(dict(x=x, tables=tables, qw=qw, sc=sc, z=z, y=y))
    return probs, devs


def _new_inputs(probs, devs, step):
    xs = []
    for i, (p, d) in enumerate(zip(probs, devs)):
        rng = np.random.default_rng(1000 * step + i)
        x = rng.standard_normal(p.x.shape).astype(np.float32)
        x[:, p.x_outlier_ch] *= 20
        xb = torch.from_numpy(x).to(torch.bfloat16)
        d["x"].copy_(xb.to(DEV))
        xs.append(xb.float().numpy())
    return xs


@pytest.mark.parametrize("M,rotate", [(1, True), (4, True), (16, True), (1, False), (8, False)])
def test_replayed_batched_call_uses_each_replays_inputs(M, rotate):
    shapes = [(1536, 1536), (1536, 256), (8960, 1536), (1536, 2048)]
    probs, devs = _layer(601 + M, shapes, M, rotate)
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    need = paro.paro_batched_workspace_bytes(layers)
    ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=DEV)
    _new_inputs(probs, devs, 0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        paro.paro_rotate_w4_linear_batched(layers, workspace=ws)  # outside capture once
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        paro.paro_rotate_w4_linear_batched(layers, workspace=ws)
    packed = [(d["qw"].cpu().numpy().view(np.uint32), d["sc"].cpu().numpy(), d["z"].cpu().numpy()) for d in devs]
    for step in range(1, 4):
        xs = _new_inputs(probs, devs, step)
        g.replay()
        torch.cuda.synchronize()
        assert paro.paro_get_device_status() == 0
        for p, d, x, pk in zip(probs, devs, xs, packed):
            xt = oracle.rotate(x, p.pairs, p.cos_t, p.sin_t, p.scale) if rotate else x
            assert_linear_close(d["y"].float().cpu().numpy(), oracle.w4_linear(xt, *pk))
    del g


@pytest.mark.parametrize("M", [1, 4])
def test_replayed_single_linear_call_uses_each_replays_inputs(M):
    probs, devs = _layer(611 + M, [(8960, 1536)], M)
    d, p = devs[0], probs[0]
    ws = torch.zeros(paro.paro_workspace_bytes(M, p.d_in), dtype=torch.uint8, device=DEV)

    def call():
        paro.paro_rotate_w4_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], out=d["y"], workspace=ws)

    _new_inputs(probs, devs, 0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    pk = (d["qw"].cpu().numpy().view(np.uint32), d["sc"].cpu().numpy(), d["z"].cpu().numpy())
    for step in range(1, 4):
        x = _new_inputs(probs, devs, step)[0]
        g.replay()
        torch.cuda.synchronize()
        assert paro.paro_get_device_status() == 0
        ref = oracle.rotate_w4_linear(x, p.pairs, p.cos_t, p.sin_t, p.scale, *pk)
        assert_linear_close(d["y"].float().cpu().numpy(), ref)
    del g
