"""Host-side checks of the C ABI: the library loads, exports every declared
entry point, and rejects invalid calls before touching the GPU.  No kernel is
launched by these tests (no CUDA device is needed)."""
import ctypes
import os
import re
import shutil
import subprocess
import sys

import pytest

import rotation_int4_weight_b200 as paro

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, UNSUPPORTED = 0, 1, 2

A = ctypes.c_void_p(1 << 20)        # aligned fake device pointers, never dereferenced
B = ctypes.c_void_p((1 << 20) + 4096 * 1024)
C = ctypes.c_void_p((1 << 21) + 8192 * 1024)
D = ctypes.c_void_p((1 << 22) + 8192 * 1024)
E = ctypes.c_void_p((1 << 23) + 8192 * 1024)
W = ctypes.c_void_p((1 << 24))
MIS = ctypes.c_void_p((1 << 20) + 2)  # misaligned


def declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"PARO_API\s+[\w\s\*]+?\b(paro_\w+)\s*\(", txt))
    return names


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert {"paro_pack_weights", "paro_rotate", "paro_w4_linear", "paro_rotate_w4_linear"} <= names
    out = subprocess.run(["nm", "-D", "--defined-only", paro.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (paro_\w+)", out))
    assert names <= exported, f"declared but not exported: {names - exported}"
    assert names <= set(paro.EXPORTED), f"declared but not bound: {names - set(paro.EXPORTED)}"
    for n in names:
        assert hasattr(paro.lib, n)


def test_default_library_carries_no_timeline_stamps():
    # the global-timer stamps exist only in the instrumented build
    # (_build.py --timeline, loaded with PARO_TIMELINE=1); the library the
    # package loads by default exports nothing beyond the header
    assert paro.LIB_PATH.endswith("libparo.so")
    out = subprocess.run(["nm", "-D", "--defined-only", paro.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (paro_\w+)", out))
    assert "paro_timeline_read" not in exported
    assert exported == declared_symbols(), exported ^ declared_symbols()


def test_status_strings_and_version():
    assert paro.paro_weight_layout_version() == 1
    for code, name in [(0, "PARO_OK"), (1, "PARO_ERR_INVALID_ARG"), (2, "PARO_ERR_UNSUPPORTED"),
                       (3, "PARO_ERR_CUDA"), (4, "PARO_ERR_TIMEOUT"), (5, "PARO_ERR_RANGE")]:
        assert paro.lib.paro_status_string(code).decode() == name


def test_test_hooks_validate_and_reset():
    assert paro.lib.paro_set_test_hooks(-1, 0) == INVALID
    assert paro.lib.paro_set_test_hooks(100000, 1) == OK
    assert paro.lib.paro_set_test_hooks(0, 0) == OK


@pytest.mark.parametrize("args,expect", [
    ((A, B, C, 4, 96), UNSUPPORTED), ((A, B, C, -1, 512), INVALID), ((A, B, C, 4, 0), INVALID),
    ((None, B, C, 4, 512), INVALID), ((MIS, B, C, 4, 512), INVALID), ((A, B, A, 4, 512), INVALID),
    ((A, B, C, 0, 512), OK),
])
def test_dense_rotate_validation(args, expect):
    assert paro.lib.paro_dense_rotate(*args, None) == expect


def test_workspace_bytes():
    """The fp16 transformed activations (2 M d_in bytes, rounded up to 256), plus,
    up to 16 tokens, the stream-K kernel's flags and partial tiles: the same
    bytes as the batched call takes for that one linear."""
    def xt(M, d):
        return (2 * M * d + 255) // 256 * 256
    assert paro.paro_workspace_bytes(0, 512) == 0
    assert paro.paro_workspace_bytes(17, 512) == xt(17, 512)
    assert paro.paro_workspace_bytes(2048, 4096) == xt(2048, 4096)
    extra8 = paro.paro_workspace_bytes(1, 512) - xt(1, 512)
    extra16 = paro.paro_workspace_bytes(16, 512) - xt(16, 512)
    assert extra8 > 0 and extra8 % 256 == 0 and extra16 > 0 and extra16 % 256 == 0
    for M, d in [(1, 512), (3, 1536), (8, 8960), (9, 128), (16, 4096)]:
        w = paro.paro_workspace_bytes(M, d)
        assert w % 256 == 0
        assert w - xt(M, d) == (extra8 if M <= 8 else extra16)
        one = [paro.ParoLinear(1 << 20, 2 << 20, M, d, 512, 8, 1, 2, 3, 4, 1 << 22, 5, 6)]
        assert paro.paro_batched_workspace_bytes(one) == w


def rot(x=A, y=B, M=4, d=512, K=8, pairs=C, c=D, s=E, scale=W):
    return paro.lib.paro_rotate(x, y, M, d, K, pairs, c, s, scale, None)


def lin(x=A, q=B, sc=C, z=D, y=E, M=4, d_in=512, d_out=512, g=128):
    return paro.lib.paro_w4_linear(x, q, sc, z, y, M, d_in, d_out, g, None)


def fused(x=A, K=8, pairs=C, c=D, s=E, scale=W, q=B, sc=C, z=D, y=E, M=4, d_in=512, d_out=512, g=128,
          ws=ctypes.c_void_p(1 << 26), wsb=1 << 20):
    return paro.lib.paro_rotate_w4_linear(x, K, pairs, c, s, scale, q, sc, z, y, M, d_in, d_out, g, ws, wsb, None)


def pack(Wp=W, d_out=512, d_in=512, g=128, K=8, pairs=C, c=D, s=E, scale=A, ws=ctypes.c_void_p(1 << 27),
         q=B, sc=C, z=D):
    return paro.lib.paro_pack_weights(Wp, d_out, d_in, g, K, pairs, c, s, scale, ws, q, sc, z, None)


@pytest.mark.parametrize("kwargs,expect", [
    (dict(d=7), INVALID), (dict(d=0), INVALID), (dict(d=49154), UNSUPPORTED), (dict(M=-1), INVALID),
    (dict(K=-1), INVALID), (dict(K=17), UNSUPPORTED), (dict(pairs=None), INVALID), (dict(c=None), INVALID),
    (dict(x=None), INVALID), (dict(y=None), INVALID), (dict(x=MIS), INVALID),
    (dict(pairs=ctypes.c_void_p((1 << 20) + 2)), INVALID), (dict(scale=ctypes.c_void_p((1 << 24) + 2)), INVALID),
    (dict(y=ctypes.c_void_p((1 << 20) + 16)), INVALID),  # partial overlap with x
    (dict(M=0, x=None, y=None), OK),                       # empty batch: nothing enqueued
])
def test_rotate_validation(kwargs, expect):
    assert rot(**kwargs) == expect
    if expect != OK:
        assert paro.lib.paro_last_error().decode()


@pytest.mark.parametrize("kwargs,expect", [
    (dict(d_in=500), INVALID), (dict(d_in=0), INVALID), (dict(d_out=8), UNSUPPORTED), (dict(d_out=0), INVALID),
    (dict(g=64), UNSUPPORTED), (dict(g=0), INVALID), (dict(M=-2), INVALID), (dict(q=None), INVALID),
    (dict(q=MIS), INVALID), (dict(x=MIS), INVALID), (dict(sc=ctypes.c_void_p((1 << 21) + 1)), INVALID),
    (dict(y=A), INVALID),                                  # output aliases the input
    (dict(M=0, x=None, y=None), OK),
])
def test_w4_linear_validation(kwargs, expect):
    assert lin(**kwargs) == expect


@pytest.mark.parametrize("kwargs,expect", [
    (dict(ws=None), INVALID), (dict(wsb=100), INVALID), (dict(ws=ctypes.c_void_p((1 << 26) + 16)), INVALID),
    (dict(K=20), UNSUPPORTED), (dict(d_in=50000 * 128 // 128 * 128 + 128 * 400), UNSUPPORTED),
    (dict(d_out=24), UNSUPPORTED), (dict(pairs=None), INVALID), (dict(y=A), INVALID),
    (dict(M=0, x=None, y=None), OK),
])
def test_fused_validation(kwargs, expect):
    assert fused(**kwargs) == expect


@pytest.mark.parametrize("kwargs,expect", [
    (dict(Wp=None), INVALID), (dict(d_in=100), INVALID), (dict(g=256), UNSUPPORTED), (dict(d_out=0), INVALID),
    (dict(ws=None), INVALID), (dict(ws=W), INVALID), (dict(K=-3), INVALID), (dict(q=None), INVALID),
    (dict(d_in=65536), UNSUPPORTED),
])
def test_pack_validation(kwargs, expect):
    assert pack(**kwargs) == expect


@pytest.mark.parametrize("args,expect", [
    # (M, d, K, pairs, cos, sin, scale, dtheta, dscale, workspace bytes)
    ((-1, 512, 8, A, B, C, D, E, E, 1 << 30), INVALID),     # negative M
    ((4, 511, 8, A, B, C, D, E, E, 1 << 30), INVALID),      # odd width
    ((4, 30000, 2, A, B, C, D, E, E, 1 << 30), UNSUPPORTED),  # wider than the kernel's shared memory
    ((4, 512, 17, A, B, C, D, E, E, 1 << 30), UNSUPPORTED),   # more than 16 stages
    ((4, 512, 8, None, B, C, D, E, E, 1 << 30), INVALID),   # K > 0 without pairs
    ((4, 512, 8, A, B, C, D, None, E, 1 << 30), INVALID),   # K > 0 without a dtheta output
    ((4, 512, 8, A, B, C, D, E, None, 1 << 30), INVALID),   # a scale without a dscale output
    ((4, 512, 8, A, B, C, D, E, E, 16), INVALID),           # workspace too small
    ((0, 512, 8, A, B, C, D, E, E, 0), OK),                 # no tokens: nothing enqueued
])
def test_rotate_backward_validation(args, expect):
    M, d, K, pr, cs, sn, sc, dth, dsc, wsb = args
    st = paro.lib.paro_rotate_backward(A, B, M, d, K, pr, cs, sn, sc, W, dth, dsc, C, wsb, None)
    assert st == expect, paro.lib.paro_last_error()


def test_rotate_backward_workspace_bytes():
    # one partial per block of 4 rows (d <= 7168), 2 rows (d <= 14336) or 1 row
    assert paro.lib.paro_rotate_backward_workspace_bytes(5, 512, 8, 1) == 2 * (8 * 256 + 512) * 4
    assert paro.lib.paro_rotate_backward_workspace_bytes(5, 512, 8, 0) == 2 * 8 * 256 * 4
    assert paro.lib.paro_rotate_backward_workspace_bytes(3, 8960, 2, 1) == 2 * (2 * 4480 + 8960) * 4
    assert paro.lib.paro_rotate_backward_workspace_bytes(3, 20000, 1, 0) == 3 * 10000 * 4
    assert paro.lib.paro_rotate_backward_workspace_bytes(0, 512, 8, 1) == 0
    assert paro.lib.paro_rotate_backward_workspace_bytes(4, 30000, 8, 1) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    pkg = tmp_path / "rotation_int4_weight_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "rotation_int4_weight_b200", "__init__.py"), pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import rotation_int4_weight_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libparo.so is missing" in r.stderr


def test_product_path_does_not_touch_the_oracle():
    pkg = os.path.join(ROOT, "rotation_int4_weight_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.replace("oracle-free", ""), f
                assert "import synth" not in txt and "from synth" not in txt, f


def test_batched_validation_on_host():
    L = paro.ParoLinear
    good = dict(d_x=1 << 20, d_y=1 << 22, M=1, d_in=512, d_out=512, K=8, d_pairs=1 << 24, d_cos=1 << 25,
                d_sin=1 << 26, d_scale=None, d_qweight=1 << 27, d_scales=1 << 28, d_zeros=1 << 29)
    arr = (L * 2)(L(**good), L(**dict(good, d_out=500, d_y=(1 << 22) + 4096)))
    ptr = ctypes.cast(arr, ctypes.c_void_p)
    assert paro.lib.paro_rotate_w4_linear_batched(ptr, 2, 128, ctypes.c_void_p(1 << 30), 1 << 20, None) == UNSUPPORTED
    assert "layer 1" in paro.lib.paro_last_error().decode()
    arr = (L * 1)(L(**dict(good, K=-1)))
    assert paro.lib.paro_rotate_w4_linear_batched(ctypes.cast(arr, ctypes.c_void_p), 1, 128, None, 0, None) == INVALID
    assert paro.lib.paro_rotate_w4_linear_batched(None, 9, 128, None, 0, None) == INVALID
    arr9 = (L * 9)(*[L(**dict(good, d_y=(1 << 22) + 4096 * i)) for i in range(9)])
    assert paro.lib.paro_rotate_w4_linear_batched(ctypes.cast(arr9, ctypes.c_void_p), 9, 128, None, 0, None) == UNSUPPORTED
    arr = (L * 1)(L(**good))
    assert paro.lib.paro_rotate_w4_linear_batched(ctypes.cast(arr, ctypes.c_void_p), 1, 128, None, 0, None) == INVALID
    # the transformed activations (1024 bytes), then the stream-K kernel's
    # counter word (rounded to 256 bytes) and its per-SM partial tiles
    wb = paro.lib.paro_batched_workspace_bytes(ctypes.cast(arr, ctypes.c_void_p), 1)
    assert wb > 1024 + 256 and wb % 256 == 0
    too_many = (L * 1)(L(**dict(good, M=17)))
    assert paro.lib.paro_batched_workspace_bytes(ctypes.cast(too_many, ctypes.c_void_p), 1) == 17 * 1024
    assert paro.lib.paro_rotate_w4_linear_batched(None, 0, 128, None, 0, None) == OK


# ---------------------------------------------------------------- pair-order planner (host only)
def _tables(d, K=8, seed=0):
    import numpy as np
    from synth import linear_problem
    p = linear_problem(seed, 1, d, 16, 2, K=K)
    return p, p.pairs, p.cos_t, p.sin_t


@pytest.mark.parametrize("d", [64, 512, 1536, 8960])
def test_planned_order_is_conflict_free_and_the_same_transform(d):
    import numpy as np
    import oracle
    p, pairs, c, s = _tables(d)
    po, co, so = paro.paro_plan_pair_order(pairs, c, s)
    for k in range(pairs.shape[0]):
        # every aligned group of 32 pairs hits 32 distinct banks with i and with j,
        # and so does every aligned 16 (8) mod 16 (8): the phases of 8- and
        # 16-byte shared-memory accesses of channel-major rows
        for n in (32, 16, 8):
            g = po[k].reshape(-1, n, 2) % n
            assert all(len(set(b[:, 0])) == n and len(set(b[:, 1])) == n for b in g), n
        # the same set of rotations: each (i, j, c, s) or its flip (j, i, c, -s)
        orig = {(int(a), int(b)): (float(cc), float(ss)) for (a, b), cc, ss in zip(pairs[k], c[k], s[k])}
        for (a, b), cc, ss in zip(po[k], co[k], so[k]):
            if (int(a), int(b)) in orig:
                assert orig[(int(a), int(b))] == (float(cc), float(ss))
            else:
                assert orig[(int(b), int(a))] == (float(cc), -float(ss))
    # reordering disjoint pairs and flipping them leaves the oracle's result bit-identical
    assert np.array_equal(oracle.rotate(p.x, pairs, c, s, p.scale), oracle.rotate(p.x, po, co, so, p.scale))


def test_planner_rejects_bad_tables():
    import numpy as np
    p, pairs, c, s = _tables(512)
    bad = pairs.copy()
    bad[2, 5, 0] = bad[2, 6, 1]  # a channel twice in stage 2
    with pytest.raises(paro.ParoError, match="perfect matching"):
        paro.paro_plan_pair_order(bad, c, s)
    p2, pairs2, c2, s2 = _tables(96)  # 96 is not a multiple of 64
    with pytest.raises(paro.ParoError) as e:
        paro.paro_plan_pair_order(pairs2, c2, s2)
    assert e.value.status == UNSUPPORTED


@pytest.mark.parametrize("fn,args,expect", [
    # paro_quantize_activations(x, q, sx, M, d, stream)
    ("paro_quantize_activations", (A, B, C, 0, 512, None), OK),            # M == 0: nothing enqueued
    ("paro_quantize_activations", (A, B, C, 2, 12, None), INVALID),        # d % 8
    ("paro_quantize_activations", (MIS, B, C, 2, 512, None), INVALID),     # x not 16-byte aligned
    ("paro_quantize_activations", (A, A, C, 2, 512, None), INVALID),       # q overlaps x
    ("paro_quantize_activations", (None, B, C, 2, 512, None), INVALID),
    # paro_w4a4_linear(q, sx, qweight, scales, zeros, y, M, d_in, d_out, group, ws, ws_bytes, stream)
    ("paro_w4a4_linear", (A, B, W, C, D, E, 0, 512, 256, 128, None, 0, None), OK),
    ("paro_w4a4_linear", (A, B, W, C, D, E, 2, 200, 256, 128, None, 0, None), INVALID),   # d_in % 128
    ("paro_w4a4_linear", (A, B, W, C, D, E, 2, 512, 250, 128, None, 0, None), UNSUPPORTED),  # d_out % 16
    ("paro_w4a4_linear", (A, B, W, C, D, E, 2, 512, 256, 64, None, 0, None), UNSUPPORTED),   # group 64
    ("paro_w4a4_linear", (MIS, B, W, C, D, E, 2, 512, 256, 128, None, 0, None), INVALID),   # q misaligned
    ("paro_w4a4_linear", (A, B, W, C, D, W, 2, 512, 256, 128, None, 0, None), INVALID),     # y overlaps weights
])
def test_w4a4_validation(fn, args, expect):
    st = getattr(paro.lib, fn)(*args)
    assert st == expect, (fn, args, paro.lib.paro_last_error())


def test_w4a4_workspace_bytes():
    # the fused call's workspace: bf16 x~, its codes and scales (each rounded up
    # to 256 bytes), then the linear's fp32 partial sums (0 when it needs none)
    r = lambda b: (b + 255) // 256 * 256
    for M, d_in, d_out in [(1, 1536, 1536), (16, 8960, 1536), (3, 512, 96)]:
        lin = paro.lib.paro_w4a4_workspace_bytes(M, d_in, d_out, 0)
        fused = paro.lib.paro_w4a4_workspace_bytes(M, d_in, d_out, 1)
        assert fused == r(2 * M * d_in) + r(M * d_in) + r(4 * M) + lin
        assert lin % (4 * M * d_out) == 0   # shares x M x d_out fp32 values
    assert paro.lib.paro_w4a4_workspace_bytes(0, 512, 512, 1) == 0
