"""The allocation-free entry point, paro_rotate_w4_linear_noalloc, called
through the C ABI.

It serves callers that cannot allocate device memory at call time (a plugin
inside an engine that owns all device memory, a path that must not trigger
the synchronisation cudaFree can cause, a program that reserves its memory at
start-up), so it takes no workspace and uses the library's built-in scratch
array instead.  It runs the same kernels as paro_rotate_w4_linear given a
workspace of the scratch array's size, so the two must agree bit for bit; both
are also compared with the oracle.  This file is collected last on purpose: a
run that stops at the first failure has already run every other test.  It
passes alone in a fresh process and after the other tests: it relies on no
state they leave.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from synth import linear_problem
from tests.tolerances import assert_linear_close

pytestmark = pytest.mark.gpu

paro = pytest.importorskip("rotation_int4_weight_b200")
DEV = "cuda"
MAX_ELEMS = 1 << 18  # M * d_in limit of the built-in scratch array
SCRATCH_BYTES = 4 << 20  # the scratch array's size, PARO_NOALLOC_SCRATCH_BYTES in include/paro.h


def _setup(seed, M, d_in, d_out):
    p = linear_problem(seed, 0, d_in, d_out, M)
    pairs = torch.from_numpy(p.pairs.view(np.int16)).to(DEV)
    cos_t = torch.from_numpy(p.cos_t).to(DEV)
    sin_t = torch.from_numpy(p.sin_t).to(DEV)
    scale = torch.from_numpy(p.scale).to(DEV)
    W = torch.from_numpy(p.W).to(DEV)
    qw, sc, z = paro.paro_pack_weights(W, pairs, cos_t, sin_t, scale)
    x = torch.from_numpy(p.x).to(DEV).to(torch.bfloat16)
    return dict(p=p, x=x, pairs=pairs, cos=cos_t, sin=sin_t, scale=scale, qw=qw, sc=sc, z=z, M=M, d_in=d_in,
                d_out=d_out, K=p.K)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _call_noalloc(a, y, stream):
    return paro.lib.paro_rotate_w4_linear_noalloc(
        _ptr(a["x"]), a["K"], _ptr(a["pairs"]), _ptr(a["cos"]), _ptr(a["sin"]), _ptr(a["scale"]),
        _ptr(a["qw"]), _ptr(a["sc"]), _ptr(a["z"]), _ptr(y), a["M"], a["d_in"], a["d_out"], 128,
        ctypes.c_void_p(stream.cuda_stream))


def _call_with_workspace(a):
    """The workspace-taking call, given a workspace of the scratch array's size
    (the no-alloc call's kernel choice depends on the bytes it can use)."""
    ws = torch.zeros(SCRATCH_BYTES, dtype=torch.uint8, device=DEV)
    return paro.paro_rotate_w4_linear(a["x"], a["pairs"], a["cos"], a["sin"], a["scale"], a["qw"], a["sc"], a["z"],
                                      workspace=ws)


def _oracle(a):
    p = a["p"]
    qwn = a["qw"].cpu().numpy().view(np.uint32)
    return oracle.rotate_w4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale, qwn, a["sc"].cpu().numpy(),
                                   a["z"].cpu().numpy())


@pytest.mark.parametrize("cases", [
    # a decode call, then a smaller one after it: stale scratch must not matter
    [(71, 16, 4096, 1024), (72, 3, 1536, 272)],
    # one token of the widest width the scratch takes, then one token of a narrow linear
    [(74, 1, 16384, 64), (75, 1, 512, 80)],
    # exactly at the size limit (M * d_in == 2^18), then the tensor-core path (M >= 128)
    [(76, 64, 4096, 128), (77, 512, 512, 256)],
])
def test_noalloc_matches_the_workspace_call_on_two_calls_in_a_row(cases):
    stream = torch.cuda.current_stream()
    for seed, M, d_in, d_out in cases:
        a = _setup(seed, M, d_in, d_out)
        assert M * d_in <= MAX_ELEMS
        y = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device=DEV)
        assert _call_noalloc(a, y, stream) == 0, paro.lib.paro_last_error()
        ref = _call_with_workspace(a)
        torch.cuda.synchronize()
        assert paro.paro_get_device_status() == 0
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), (seed, M, d_in, d_out)
        assert_linear_close(y.float().cpu().numpy(), _oracle(a))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    a = _setup(73, 2, 1536, 256)
    a["M"] = MAX_ELEMS // a["d_in"] + 1   # shape only: rejected before anything is read
    y = torch.empty(1, dtype=torch.bfloat16, device=DEV)
    assert _call_noalloc(a, y, torch.cuda.current_stream()) == 2  # PARO_ERR_UNSUPPORTED
    assert "exceeds the built-in scratch" in paro.lib.paro_last_error().decode()
