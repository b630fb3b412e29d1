"""Host logic of the column-parallel split (rotation_int4_weight_b200.column_parallel)
on CPU: row ranges, slicing of packed weights, and, with two gloo ranks, the
all-gather that assembles y.  Each rank computes its rows with a CPU stand-in
that is row by row deterministic (the oracle's transform and dequantisation,
then an elementwise product summed along each weight row), so the gathered
result must equal the single-rank one bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from rotation_int4_weight_b200 import column_parallel as cp
from synth import linear_problem


def test_row_ranges_cover_d_out_in_aligned_equal_slices():
    for d_out, world in [(1536, 1), (1536, 2), (256, 8), (8960, 8), (14336, 4)]:
        rr = [cp.row_range(d_out, world, r) for r in range(world)]
        assert rr[0][0] == 0 and rr[-1][1] == d_out
        assert all(a[1] == b[0] for a, b in zip(rr, rr[1:]))
        assert len({n1 - n0 for n0, n1 in rr}) == 1
        assert all(n0 % 16 == 0 and n1 % 16 == 0 for n0, n1 in rr)
    with pytest.raises(ValueError):
        cp.row_range(272, 2, 0)      # 136 rows is not a multiple of 16
    with pytest.raises(ValueError):
        cp.row_range(256, 2, 2)


def test_shard_packed_takes_contiguous_rows():
    qw = torch.arange(64 * 4, dtype=torch.int32).view(64, 4)
    sc = torch.arange(64, dtype=torch.float16).view(64, 1)
    z = -sc
    a, b, c = cp.shard_packed(qw, sc, z, 4, 2)
    assert torch.equal(a, qw[32:48]) and torch.equal(b, sc[32:48]) and torch.equal(c, z[32:48])
    assert a.is_contiguous()


def _reference_rows(p, packed):
    """y[m, n] for the rows of `packed`, row by row deterministic."""
    qw, sc, z = packed
    xt = oracle.rotate(p.x, p.pairs, p.cos_t, p.sin_t, p.scale)
    w = oracle.dequantize(qw.numpy().view(np.uint32), sc.numpy(), z.numpy())
    return np.stack([(xt[m][None, :] * w).sum(axis=1) for m in range(xt.shape[0])])


def _packed(p):
    qw, sc, z = oracle.pack_weights(p.W, p.pairs, p.cos_t, p.sin_t, p.scale)
    return torch.from_numpy(qw.view(np.int32)), torch.from_numpy(sc), torch.from_numpy(z)


def _worker(rank, world, port, M, q):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        p = linear_problem(401, 0, 512, 256, M)
        packed = _packed(p)

        def compute(x, shard):
            return torch.from_numpy(_reference_rows(p, shard))

        lin = cp.ColumnParallelLinear((None,) * 4, packed, world, rank, compute=compute)
        y = lin(torch.zeros(M, 512))
        q.put((rank, y.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M", [1, 3])
def test_two_gloo_ranks_gather_the_single_rank_result_bit_exactly(M):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, M, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=120) for _ in range(2))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    p = linear_problem(401, 0, 512, 256, M)
    full = _reference_rows(p, _packed(p))
    assert res[0].shape == (M, 256)
    assert np.array_equal(res[0], full) and np.array_equal(res[1], full)
