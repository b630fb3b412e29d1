"""Column-parallel split of the rotate + INT4 linear across the ranks of a
process group (one process per GPU, torch.distributed over NCCL).

Rank r of N holds output rows [r d_out / N, (r + 1) d_out / N) of the packed
weights W~ and the whole transform (pairs, cos, sin, scale), which is small
and replicated.  Every rank transforms the full activation row itself (the
transform couples all d_in channels through its perfect matchings, page
"ParoQuant: pairwise rotations that survive deployment", section "A rotation
small enough to execute", so splitting d_in would need x~ exchanged first and
the partial outputs summed), computes its slice of y with the library's
calls, and one all-gather assembles y [M, d_out] on every rank.  Each output
element is computed on exactly one rank from the same inputs, so the split
changes no arithmetic of the transform; the INT4 linear's summation order
within a row may differ from an unsplit call (its work split depends on the
rows it is given), within the linear's tolerance.

Only plumbing lives here: row ranges, slicing of packed weights, the gather
and its reordering.  The arithmetic runs in libparo.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch

ROW_ALIGN = 16  # the INT4 calls take d_out in multiples of 16


def row_range(d_out: int, world: int, rank: int) -> tuple[int, int]:
    """Output rows [n0, n1) of `rank`: equal slices, each a multiple of 16 rows."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    if d_out % (ROW_ALIGN * world):
        raise ValueError(f"d_out = {d_out} does not split into {world} slices of a multiple of {ROW_ALIGN} rows")
    s = d_out // world
    return rank * s, (rank + 1) * s


def shard_packed(qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, world: int, rank: int):
    """This rank's rows of packed weights (layout version 1 is row-major in every
    array, so a row slice is a contiguous block of each)."""
    n0, n1 = row_range(qweight.shape[0], world, rank)
    return (qweight[n0:n1].contiguous(), scales[n0:n1].contiguous(), zeros[n0:n1].contiguous())


def gather_columns(y_local: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """All-gather of every rank's y slice [M, s] into y [M, world * s], ranks in
    column order (one collective; for M == 1 the gathered buffer already is y)."""
    import torch.distributed as dist
    M, s = y_local.shape
    buf = torch.empty(world * M * s, dtype=y_local.dtype, device=y_local.device)
    dist.all_gather_into_tensor(buf, y_local.contiguous().view(-1), group=group)
    if M == 1:
        return buf.view(1, world * s)
    return buf.view(world, M, s).permute(1, 0, 2).reshape(M, world * s)


class ColumnParallelLinear:
    """One linear split by output rows over the ranks of `group`.

    `compute(x, shard)` returns this rank's y slice [M, s] for activations x;
    by default it is the library's fused rotate + INT4 call on the rank's
    packed rows.  The tables and x are the same on every rank.
    """

    def __init__(self, tables: Sequence, packed: Sequence[torch.Tensor], world: int, rank: int, group=None,
                 compute: Callable | None = None):
        self.world, self.rank, self.group = world, rank, group
        self.tables = tuple(tables)
        self.d_out = packed[0].shape[0]
        self.rows = row_range(self.d_out, world, rank)
        self.shard = shard_packed(*packed, world, rank)
        self.compute = compute or self._paro_compute
        self._ws = None

    def _paro_compute(self, x, shard):
        import rotation_int4_weight_b200 as paro
        need = paro.paro_workspace_bytes(x.shape[0], x.shape[1])
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=x.device)
        return paro.paro_rotate_w4_linear(x, *self.tables, *shard, workspace=self._ws)

    def local(self, x: torch.Tensor) -> torch.Tensor:
        """This rank's slice of y, [M, d_out / world]."""
        return self.compute(x, self.shard)

    def __call__(self, x: torch.Tensor) -> torch.Tensor:
        y = self.local(x)
        if self.world == 1:
            return y
        return gather_columns(y, self.world, self.group)
