"""CUDA path against the fp64 oracle on the same seeded inputs (needs a B200).

Bit-exact: packing, unpacking, pair indexing.  Within the criteria of
tests/tolerances.py: the rotation and the linear.  Sizes span several tiles
and ragged tails.  Every decode case (up to 16 tokens) is compared on every
token and every output column; with more tokens, on sampled token rows that
include one of every 256-token tile, and every output column.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import config_problems, linear_problem
from tests.tolerances import assert_linear_close, assert_rotation_close, linear_errors, rotation_errors

pytestmark = pytest.mark.gpu

paro = pytest.importorskip("rotation_int4_weight_b200")
DEV = "cuda"


def dev_tables(p):
    pairs = torch.from_numpy(p.pairs.view(np.int16)).to(DEV)
    return (pairs, torch.from_numpy(p.cos_t).to(DEV), torch.from_numpy(p.sin_t).to(DEV),
            torch.from_numpy(p.scale).to(DEV))


def dev_x(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(DEV).to(torch.bfloat16)


def host(t):
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def oracle_pack_from_fp32(wt32):
    q, sc, z = oracle.quantize_groups(wt32)
    return oracle.pack_nibbles(q), sc, z.astype(np.float16)


def gpu_pack(W32, tables=None):
    W = torch.from_numpy(np.ascontiguousarray(W32)).to(DEV)
    if tables is None:
        return paro.paro_pack_weights(W)
    return paro.paro_pack_weights(W, *tables)


def to_np_pack(qw, sc, z):
    return (qw.cpu().numpy().view(np.uint32), sc.cpu().numpy(), z.cpu().numpy())


def oracle_all_columns(xt, qwn, scn, zn, chunk=2048):
    """The oracle's linear over every output column, dequantising `chunk` weight
    rows at a time (bounded host memory at the full layer sizes)."""
    out = np.empty((xt.shape[0], qwn.shape[0]), dtype=np.float64)
    for r0 in range(0, qwn.shape[0], chunk):
        r1 = min(r0 + chunk, qwn.shape[0])
        out[:, r0:r1] = oracle.linear(xt, oracle.dequantize(qwn[r0:r1], scn[r0:r1], zn[r0:r1]))
    return out


# ---------------------------------------------------------------- packing
@pytest.mark.parametrize("shape", [(512, 512), (48, 1536), (272, 8960 // 2)])
def test_pack_is_bit_exact_on_the_same_fp32_weights(shape):
    d_out, d_in = shape
    p = linear_problem(21, d_in, d_in, d_out, 1)
    wt32 = oracle.fold_weights(p.W, p.pairs, p.cos_t, p.sin_t, p.scale).astype(np.float32)
    ref = oracle_pack_from_fp32(wt32)
    got = to_np_pack(*gpu_pack(wt32))
    assert np.array_equal(got[0], ref[0])
    assert np.array_equal(got[1].view(np.uint16), ref[1].view(np.uint16))
    assert np.array_equal(got[2].view(np.uint16), ref[2].view(np.uint16))


def test_pack_degenerate_groups_bit_exact():
    v = np.zeros((16, 512), dtype=np.float32)
    v[1, :128] = 0.5
    v[2, 130] = -1e-30
    v[3, 256:384] = -0.5
    v[4, :] = np.linspace(-3, 1, 512, dtype=np.float32)
    v[5, ::2] = 1e-3
    ref = oracle_pack_from_fp32(v)
    got = to_np_pack(*gpu_pack(v))
    assert np.array_equal(got[0], ref[0])
    assert np.array_equal(got[1].view(np.uint16), ref[1].view(np.uint16))
    assert np.array_equal(got[2].view(np.uint16), ref[2].view(np.uint16))


def test_brute_force_unpack_of_gpu_pack():
    """Every nibble, scale and zero of a GPU-packed layer unpacks to the oracle's codes."""
    p = next(config_problems(0))
    wt32 = oracle.fold_weights(p.W, p.pairs, p.cos_t, p.sin_t, p.scale).astype(np.float32)
    qw, sc, z = to_np_pack(*gpu_pack(wt32))
    q_ref, sc_ref, z_ref = oracle.quantize_groups(wt32)
    by = qw.astype("<u4").view(np.uint8).reshape(qw.shape[0], -1)
    codes = np.empty((qw.shape[0], by.shape[1] * 2), dtype=np.uint8)
    codes[:, 0::2], codes[:, 1::2] = by & 0xF, by >> 4
    assert np.array_equal(codes, q_ref)
    assert np.array_equal(z.astype(np.float32).astype(np.uint8), z_ref)
    assert np.array_equal(sc.view(np.uint16), sc_ref.view(np.uint16))


@pytest.mark.parametrize("cfg,only", [(0, None), (1, ["k", "down"])])
def test_pack_with_fold(cfg, only):
    for p in config_problems(cfg, only=only):
        tables = dev_tables(p)
        W = torch.from_numpy(p.W).to(DEV)
        ws = torch.empty(p.d_out, p.d_in, dtype=torch.float32, device=DEV)
        qw, sc, z = paro.paro_pack_weights(W, *tables, workspace=ws)
        fold_ref = oracle.fold_weights(p.W, p.pairs, p.cos_t, p.sin_t, p.scale)
        fold_gpu = ws.cpu().numpy().astype(np.float64)
        rel = np.linalg.norm(fold_gpu - fold_ref, axis=1) / np.linalg.norm(fold_ref, axis=1)
        assert rel.max() <= 1e-5
        # the GPU's fp32 fold packs bit-exactly like the oracle's quantiser
        ref_from_gpu_fold = oracle_pack_from_fp32(ws.cpu().numpy())
        got = to_np_pack(qw, sc, z)
        assert np.array_equal(got[0], ref_from_gpu_fold[0])
        # against the oracle's own fp64 fold only rare rounding ties may flip a code
        q_ref = oracle.unpack_nibbles(oracle.pack_weights(p.W, p.pairs, p.cos_t, p.sin_t, p.scale)[0])
        flips = np.count_nonzero(oracle.unpack_nibbles(got[0]) != q_ref)
        assert flips <= max(2, q_ref.size // 100000)


# ---------------------------------------------------------------- rotation
@pytest.mark.parametrize("M,d", [(1, 512), (3, 512), (4, 512), (5, 1536), (17, 1536), (9, 8960), (2, 14336),
                                 (7, 130), (33, 4096),
                                 # many tokens (the channel-major kernel), ragged last row blocks
                                 (130, 14336), (67, 8960), (129, 1536)])
def test_rotate_parity(M, d):
    p = linear_problem(31, M * 1000 + d, d, 16, M)
    x = dev_x(p.x)
    got = host(paro.paro_rotate(x, *dev_tables(p)))
    ref = oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale)
    assert_rotation_close(got, ref)


def test_rotate_signed_permutation_is_bit_exact():
    """c = 0, s = 1 makes every stage an exact signed permutation: bit-exact pair indexing."""
    p = linear_problem(32, 0, 4096, 16, 6)
    c = np.zeros_like(p.cos_t)
    s = np.ones_like(p.sin_t)
    tables = (torch.from_numpy(p.pairs.view(np.int16)).to(DEV), torch.from_numpy(c).to(DEV),
              torch.from_numpy(s).to(DEV), None)
    got = host(paro.paro_rotate(dev_x(p.x), *tables))
    ref = oracle.rotate(p.x, p.pairs, c, s, None)
    assert np.array_equal(got, ref.astype(np.float32))


def test_rotate_pair_order_within_stage_is_bit_irrelevant():
    p = linear_problem(33, 0, 1536, 16, 8)
    rng = np.random.default_rng(0)
    perm = np.stack([rng.permutation(p.d_in // 2) for _ in range(p.K)])
    pairs2 = np.stack([p.pairs[k][perm[k]] for k in range(p.K)])
    c2 = np.stack([p.cos_t[k][perm[k]] for k in range(p.K)])
    s2 = np.stack([p.sin_t[k][perm[k]] for k in range(p.K)])
    x = dev_x(p.x)
    a = paro.paro_rotate(x, *dev_tables(p))
    b = paro.paro_rotate(x, torch.from_numpy(pairs2.view(np.int16)).to(DEV), torch.from_numpy(c2).to(DEV),
                         torch.from_numpy(s2).to(DEV), torch.from_numpy(p.scale).to(DEV))
    assert torch.equal(a, b)


def test_rotate_in_place_and_k0():
    p = linear_problem(34, 0, 1536, 16, 5)
    x = dev_x(p.x)
    ref = paro.paro_rotate(x, *dev_tables(p))
    y = x.clone()
    paro.paro_rotate(y, *dev_tables(p), out=y)
    assert torch.equal(y, ref)
    # K = 0, no scale: the identity
    assert torch.equal(paro.paro_rotate(x), x)
    # K = 0 with scale only
    got = host(paro.paro_rotate(x, scale=torch.from_numpy(p.scale).to(DEV)))
    assert_rotation_close(got, p.x / p.scale.astype(np.float64))


def test_rotate_bad_pair_index_is_reported_not_faulted():
    p = linear_problem(35, 0, 512, 16, 2)
    bad = p.pairs.copy()
    bad[3, 7, 1] = 600  # >= d
    assert paro.paro_get_device_status() == 0
    paro.paro_rotate(dev_x(p.x), torch.from_numpy(bad.view(np.int16)).to(DEV), *dev_tables(p)[1:])
    assert paro.paro_get_device_status() == 1
    assert paro.paro_get_device_status() == 0  # cleared


# ---------------------------------------------------------------- linear
def _packed(p, rotate=True):
    if rotate:
        return paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV), *dev_tables(p))
    return paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV))


@pytest.mark.parametrize("M,d_in,d_out", [(1, 512, 512), (3, 512, 512), (8, 1536, 256), (9, 1536, 272),
                                          (16, 512, 1024), (17, 384, 96), (40, 1024, 64), (2, 8960, 1536)])
def test_w4_linear_parity(M, d_in, d_out):
    p = linear_problem(41, M * 7 + d_out, d_in, d_out, M)
    qw, sc, z = _packed(p, rotate=False)
    got = host(paro.paro_w4_linear(dev_x(p.x), qw, sc, z))
    ref = oracle.w4_linear(p.x, *to_np_pack(qw, sc, z))
    assert_linear_close(got, ref)


@pytest.mark.parametrize("M,d_in,d_out", [(1, 512, 512), (4, 512, 512), (16, 1536, 256), (11, 4096, 1024),
                                          (24, 1536, 1536)])
def test_rotate_w4_linear_parity(M, d_in, d_out):
    p = linear_problem(51, M * 13 + d_in, d_in, d_out, M)
    qw, sc, z = _packed(p)
    got = host(paro.paro_rotate_w4_linear(dev_x(p.x), *dev_tables(p), qw, sc, z))
    ref = oracle.rotate_w4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale, *to_np_pack(qw, sc, z))
    assert_linear_close(got, ref)
    # and the unfused composition agrees with the same reference
    xr = paro.paro_rotate(dev_x(p.x), *dev_tables(p))
    got2 = host(paro.paro_w4_linear(xr, qw, sc, z))
    assert_linear_close(got2, ref)


def test_empty_batch_is_a_noop():
    p = linear_problem(52, 0, 512, 512, 1)
    qw, sc, z = _packed(p)
    x = torch.empty(0, 512, dtype=torch.bfloat16, device=DEV)
    assert paro.paro_w4_linear(x, qw, sc, z).shape == (0, 512)
    assert paro.paro_rotate_w4_linear(x, *dev_tables(p), qw, sc, z).shape == (0, 512)
    assert paro.paro_rotate(x, *dev_tables(p)).shape == (0, 512)


# ---------------------------------------------------------------- full-size layers, sampled rows
def _full_size_check(p, M_rows, seed=0):
    """Full-size fused call against the oracle on every output column; every
    token up to 16 tokens, beyond that M_rows tokens with at least one in every
    256-token tile of the tensor-core kernel."""
    qw, sc, z = _packed(p)
    y = host(paro.paro_rotate_w4_linear(dev_x(p.x), *dev_tables(p), qw, sc, z))
    rows = np.arange(p.M) if p.M <= 16 else _sampled_rows(p.M, M_rows, seed)
    xt = oracle.rotate(p.x[rows], p.pairs, p.cos_t, p.sin_t, p.scale)
    ref = oracle_all_columns(xt, *to_np_pack(qw, sc, z))
    got = y[rows]
    assert np.isfinite(got).all(), p.name
    metric, literal = linear_errors(got, ref)
    assert metric <= 1e-2, (p.name, metric, literal)


@pytest.mark.parametrize("cfg", [1, 2])
def test_full_size_decode_layers(cfg):
    for p in config_problems(cfg, M=1 if cfg == 1 else 16):
        _full_size_check(p, 16)


def test_full_size_prefill_layer_sampled():
    p = next(config_problems(3, only=["k"]))
    _full_size_check(p, 64)


# ---------------------------------------------------------------- batched layer call
def _batch_case(shapes_m, seed):
    probs, devs = [], []
    for i, (d_in, d_out, M) in enumerate(shapes_m):
        p = linear_problem(seed, i, d_in, d_out, M)
        tables = dev_tables(p)
        qw, sc, z = paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV), *tables)
        x = dev_x(p.x)
        y = torch.empty(M, d_out, dtype=torch.bfloat16, device=DEV)
        probs.append(p)
        devs.append(dict(x=x, tables=tables, qw=qw, sc=sc, z=z, y=y))
    return probs, devs


@pytest.mark.parametrize("shapes_m", [
    [(1536, 1536, 1), (1536, 256, 1), (1536, 256, 1), (1536, 1536, 1), (1536, 8960, 1), (1536, 8960, 1),
     (8960, 1536, 1)],
    [(512, 512, 1), (1024, 272, 3), (4096, 1024, 16), (512, 96, 20), (384, 64, 9)],
])
def test_batched_matches_oracle_and_single_calls(shapes_m):
    probs, devs = _batch_case(shapes_m, 61)
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    paro.paro_rotate_w4_linear_batched(layers)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    for p, d in zip(probs, devs):
        got = host(d["y"])
        single = host(paro.paro_rotate_w4_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"]))
        ref = oracle_all_columns(oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale),
                                 *to_np_pack(d["qw"], d["sc"], d["z"]))
        assert_linear_close(got, ref)
        assert_linear_close(got, single)


def test_batched_rejects_bad_layer_without_launching():
    probs, devs = _batch_case([(512, 512, 1), (512, 512, 2)], 62)
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    layers[1].d_out = 520  # not a multiple of 16
    before = devs[0]["y"].clone()
    with pytest.raises(paro.ParoError, match="layer 1"):
        paro.paro_rotate_w4_linear_batched(layers)
    torch.cuda.synchronize()
    assert torch.equal(devs[0]["y"], before)  # nothing ran


# ---------------------------------------------------------------- tensor-core (tcgen05) path, M >= 128
def _sampled_rows(M, n, seed, tile=256):
    """n seeded token rows of M, at least one in every `tile`-token tile (the
    tensor-core kernel's token tile), the rest drawn at random."""
    rng = np.random.default_rng(seed)
    per_tile = [int(rng.integers(t0, min(t0 + tile, M))) for t0 in range(0, M, tile)]
    rest = np.setdiff1d(np.arange(M), per_tile)
    extra = rng.choice(rest, size=max(0, min(n, M) - len(per_tile)), replace=False) if rest.size else []
    return np.sort(np.concatenate([per_tile, extra]).astype(np.int64))


@pytest.mark.parametrize("M,d_in,d_out", [(128, 256, 256), (200, 512, 272), (384, 1536, 1024), (129, 4096, 512)])
def test_w4_linear_tensor_core_bf16(M, d_in, d_out):
    p = linear_problem(81, M + d_out, d_in, d_out, M)
    qw, sc, z = _packed(p, rotate=False)
    got = host(paro.paro_w4_linear(dev_x(p.x), qw, sc, z))
    rows = _sampled_rows(M, 48, 1)
    ref = oracle.w4_linear(p.x[rows], *to_np_pack(qw, sc, z))
    assert_linear_close(got[rows], ref)
    assert paro.paro_get_device_status() == 0


@pytest.mark.parametrize("M,d_in,d_out", [(128, 512, 256), (300, 1536, 272), (640, 4096, 1024)])
def test_rotate_w4_linear_tensor_core_f16(M, d_in, d_out):
    p = linear_problem(82, M + d_out, d_in, d_out, M)
    qw, sc, z = _packed(p)
    got = host(paro.paro_rotate_w4_linear(dev_x(p.x), *dev_tables(p), qw, sc, z))
    rows = _sampled_rows(M, 48, 2)
    ref = oracle.rotate_w4_linear(p.x[rows], p.pairs, p.cos_t, p.sin_t, p.scale, *to_np_pack(qw, sc, z))
    assert_linear_close(got[rows], ref)
    assert paro.paro_get_device_status() == 0


# ---------------------------------------------------------------- planned (conflict-free) pair order
@pytest.mark.parametrize("M,d", [(1, 1536), (4, 4096), (300, 4096), (2, 8960)])
def test_planned_tables_match_the_oracle(M, d):
    p = linear_problem(91, M + d, d, 256, M)
    po, co, so = paro.paro_plan_pair_order(p.pairs, p.cos_t, p.sin_t)
    tables = (torch.from_numpy(po.view(np.int16)).to(DEV), torch.from_numpy(co).to(DEV),
              torch.from_numpy(so).to(DEV), torch.from_numpy(p.scale).to(DEV))
    got = host(paro.paro_rotate(dev_x(p.x), *tables))
    assert_rotation_close(got, oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale))
    qw, sc, z = paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV), *tables)
    y = host(paro.paro_rotate_w4_linear(dev_x(p.x), *tables, qw, sc, z))
    ref = oracle.rotate_w4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale, *to_np_pack(qw, sc, z))
    assert_linear_close(y, ref)


# ---------------------------------------------------------------- stream-K decode kernel (M <= 16)
def _stream_case(shapes_m, seed, rotate):
    probs, devs = [], []
    for i, (d_in, d_out, M) in enumerate(shapes_m):
        p = linear_problem(seed, i, d_in, d_out, M)
        tables = dev_tables(p) if rotate else (None, None, None, None)
        qw, sc, z = _packed(p, rotate)
        y = torch.full((M, d_out), float("nan"), dtype=torch.bfloat16, device=DEV)
        probs.append(p)
        devs.append(dict(x=dev_x(p.x), tables=tables, qw=qw, sc=sc, z=z, y=y))
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    return probs, devs, layers


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("shapes_m", [
    # a Qwen2.5-1.5B-shaped layer at 16 tokens: tiles split between warps and CTAs
    [(1536, 1536, 16), (1536, 256, 16), (1536, 256, 16), (1536, 1536, 16), (1536, 8960, 16), (1536, 8960, 16),
     (8960, 1536, 16)],
    # mixed token counts, ragged output tails (d_out not a multiple of 64)
    [(512, 80, 1), (1024, 272, 3), (384, 112, 9), (128, 64, 16), (4096, 1040, 8)],
    # fewer units than warps in the only CTA
    [(128, 64, 1)],
    # one row block whose 96 groups are spread over twelve CTAs
    [(12288, 64, 2)],
])
def test_stream_decode_matches_oracle_and_repeats_bit_exactly(shapes_m, rotate):
    probs, devs, layers = _stream_case(shapes_m, 71, rotate)
    ws = paro.paro_rotate_w4_linear_batched(layers)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    first = [d["y"].clone() for d in devs]
    for p, d in zip(probs, devs):
        got = host(d["y"])
        assert np.isfinite(got).all(), p.name
        xt = oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale) if rotate else p.x
        assert_linear_close(got, oracle_all_columns(xt, *to_np_pack(d["qw"], d["sc"], d["z"])))
    # the arrival counters left by the first call are reused as they are: the
    # second call must give the same bits (fixed summation order)
    for d in devs:
        d["y"].fill_(float("nan"))
    paro.paro_rotate_w4_linear_batched(layers, workspace=ws)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    for f, d in zip(first, devs):
        assert torch.equal(f.view(torch.int16), d["y"].view(torch.int16))


def test_stream_decode_full_size_llama_layer_split():
    """The seven Llama-3-8B-shaped linears at 8 tokens in one batched call: the
    two-launch decode path (transform CTAs publish per-CTA flags, the INT4
    launch waits per linear) with the widest linear's units on CTAs of their
    own, since the layer gives every CTA a long INT4 share.  Sampled output
    columns against the oracle, then a repeat that must give the same bits."""
    M = 8
    probs, devs = [], []
    for p in config_problems(2, M=M):
        tables = dev_tables(p)
        qw, sc, z = paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV), *tables)
        p.W = None  # the host weights are not needed again
        y = torch.full((M, p.d_out), float("nan"), dtype=torch.bfloat16, device=DEV)
        probs.append(p)
        devs.append(dict(x=dev_x(p.x), tables=tables, qw=qw, sc=sc, z=z, y=y))
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    ws = paro.paro_rotate_w4_linear_batched(layers)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    first = [d["y"].clone() for d in devs]
    for p, d in zip(probs, devs):
        got = host(d["y"])
        assert np.isfinite(got).all(), p.name
        ref = oracle_all_columns(oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale),
                                 *to_np_pack(d["qw"], d["sc"], d["z"]))
        assert_linear_close(got, ref)
    for d in devs:
        d["y"].fill_(float("nan"))
    paro.paro_rotate_w4_linear_batched(layers, workspace=ws)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    for f, d in zip(first, devs):
        assert torch.equal(f.view(torch.int16), d["y"].view(torch.int16))


# ---------------------------------------------------------------- fused decode (one token per linear)
# With every linear at M = 1 the batched call runs the transforms in the INT4
# kernel's first CTAs (one per linear), which publish x~ with a flag that the
# INT4 CTAs wait for before requesting a linear's activations.
@pytest.mark.parametrize("spec", [
    # (d_in, d_out, K, transform): the widest linears take two-slot and one-slot
    # stage rings inside the fused kernel; one linear has no transform (its x is
    # only rounded to fp16); ragged output tails
    [(14336, 272, 8, True), (16384, 64, 16, True), (512, 80, 0, False), (1536, 1040, 3, True)],
    # the most linears a call takes: eight transform CTAs
    [(512, 64, 8, True), (1024, 128, 2, True), (384, 96, 8, True), (2048, 64, 1, True),
     (512, 208, 8, True), (640, 64, 5, True), (4096, 64, 8, True), (128, 64, 8, True)],
])
def test_fused_decode_matches_oracle_and_repeats_bit_exactly(spec):
    probs, devs = [], []
    for i, (d_in, d_out, K, rot) in enumerate(spec):
        p = linear_problem(83, i, d_in, d_out, 1, K=K)
        tables = dev_tables(p) if rot else (None, None, None, None)
        qw, sc, z = _packed(p, rot)
        y = torch.full((1, d_out), float("nan"), dtype=torch.bfloat16, device=DEV)
        probs.append((p, rot))
        devs.append(dict(x=dev_x(p.x), tables=tables, qw=qw, sc=sc, z=z, y=y))
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    ws = paro.paro_rotate_w4_linear_batched(layers)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    first = [d["y"].clone() for d in devs]
    for (p, rot), d in zip(probs, devs):
        got = host(d["y"])
        xt = oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale) if rot else p.x
        ref = oracle.linear(xt, oracle.dequantize(*to_np_pack(d["qw"], d["sc"], d["z"])))
        assert_linear_close(got, ref)
    for d in devs:
        d["y"].fill_(float("nan"))
    paro.paro_rotate_w4_linear_batched(layers, workspace=ws)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    for f, d in zip(first, devs):
        assert torch.equal(f.view(torch.int16), d["y"].view(torch.int16))


@pytest.mark.parametrize("shapes", [
    # Llama-3-8B-shaped layer (the widest linear's units on CTAs of their own)
    [(4096, 4096), (4096, 1024), (4096, 1024), (4096, 4096), (4096, 14336), (4096, 14336), (14336, 4096)],
    # ragged output tails; the widest linear's tiles split between CTAs
    [(1024, 1040), (2048, 272), (512, 3088), (6144, 4112)],
])
def test_fused_layer_matches_oracle_and_repeats_bit_exactly(shapes):
    probs, devs = _batch_case([(d_in, d_out, 1) for d_in, d_out in shapes], 64)
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    ws = paro.paro_rotate_w4_linear_batched(layers)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    first = [d["y"].clone() for d in devs]
    for p, d in zip(probs, devs):
        ref = oracle_all_columns(oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale),
                                 *to_np_pack(d["qw"], d["sc"], d["z"]))
        assert_linear_close(host(d["y"]), ref)
    for d in devs:
        d["y"].fill_(float("nan"))
    paro.paro_rotate_w4_linear_batched(layers, workspace=ws)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    for f, d in zip(first, devs):
        assert torch.equal(f.view(torch.int16), d["y"].view(torch.int16))


# ---------------------------------------------------------------- grouped tensor-core launch (batched, M >= 128)
@pytest.mark.parametrize("shapes_m", [
    # mixed K, ragged token counts and ragged output tails in one launch
    [(512, 272, 128), (1536, 528, 300), (4096, 1024, 200)],
    # more tiles than SMs: every CTA walks several tiles, the longest K first
    [(4096, 14336, 640), (4096, 1024, 640), (14336, 512, 384)],
])
def test_batched_prefill_grouped_matches_oracle_and_single_calls(shapes_m):
    probs, devs = _batch_case(shapes_m, 63)
    layers = [paro.paro_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"], d["y"]) for d in devs]
    paro.paro_rotate_w4_linear_batched(layers)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    for i, (p, d) in enumerate(zip(probs, devs)):
        got = host(d["y"])
        assert np.isfinite(got).all(), p.name
        rows = _sampled_rows(p.M, 24, 7 + i)
        ref = oracle.rotate_w4_linear(p.x[rows], p.pairs, p.cos_t, p.sin_t, p.scale, *to_np_pack(d["qw"], d["sc"], d["z"]))
        assert_linear_close(got[rows], ref)
        # a tile's sum does not depend on the launch it ran in
        single = paro.paro_rotate_w4_linear(d["x"], *d["tables"], d["qw"], d["sc"], d["z"])
        assert torch.equal(single.view(torch.int16), d["y"].view(torch.int16))


def test_batched_prefill_plain_bf16_grouped():
    """No transforms, every linear on the tensor cores: one launch reads the bf16 inputs."""
    shapes_m = [(4096, 1040, 256), (1536, 528, 300), (512, 256, 128)]
    probs, devs, layers = _stream_case(shapes_m, 64, rotate=False)
    paro.paro_rotate_w4_linear_batched(layers)
    torch.cuda.synchronize()
    assert paro.paro_get_device_status() == 0
    for i, (p, d) in enumerate(zip(probs, devs)):
        got = host(d["y"])
        assert np.isfinite(got).all(), p.name
        rows = _sampled_rows(p.M, 24, 11 + i)
        ref = oracle.w4_linear(p.x[rows], *to_np_pack(d["qw"], d["sc"], d["z"]))
        assert_linear_close(got[rows], ref)
        single = paro.paro_w4_linear(d["x"], d["qw"], d["sc"], d["z"])
        assert torch.equal(single.view(torch.int16), d["y"].view(torch.int16))
