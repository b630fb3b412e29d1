"""The column-parallel split on one GPU: two ranks emulated one after the other
(each computes its slice of y through the library on its own packed rows; no
collective runs, since ranks that wait for one another never share a GPU
here).  The concatenated slices must match the oracle and the unsplit call."""
import numpy as np
import pytest
import torch

import oracle
from rotation_int4_weight_b200 import column_parallel as cp
from synth import linear_problem
from tests.tolerances import assert_linear_close

pytestmark = pytest.mark.gpu

paro = pytest.importorskip("rotation_int4_weight_b200")
DEV = "cuda"


@pytest.mark.parametrize("M,d_in,d_out,world", [(1, 1536, 1536, 2), (4, 1536, 8960, 2), (16, 4096, 1024, 4),
                                                (300, 1536, 512, 2)])
def test_emulated_ranks_match_the_oracle_and_the_unsplit_call(M, d_in, d_out, world):
    p = linear_problem(411, M, d_in, d_out, M)
    tables = (torch.from_numpy(p.pairs.view(np.int16)).to(DEV), torch.from_numpy(p.cos_t).to(DEV),
              torch.from_numpy(p.sin_t).to(DEV), torch.from_numpy(p.scale).to(DEV))
    packed = paro.paro_pack_weights(torch.from_numpy(p.W).to(DEV), *tables)
    x = torch.from_numpy(p.x).to(DEV).to(torch.bfloat16)
    parts = [cp.ColumnParallelLinear(tables, packed, world, r).local(x) for r in range(world)]
    y = torch.cat(parts, dim=1)
    assert y.shape == (M, d_out)
    assert paro.paro_get_device_status() == 0
    ref = oracle.rotate_w4_linear(p.x, p.pairs, p.cos_t, p.sin_t, p.scale, packed[0].cpu().numpy().view(np.uint32),
                                  packed[1].cpu().numpy(), packed[2].cpu().numpy())
    assert_linear_close(y.float().cpu().numpy(), ref)
    whole = paro.paro_rotate_w4_linear(x, *tables, *packed)
    assert_linear_close(y.float().cpu().numpy(), whole.float().cpu().numpy().astype(np.float64))
