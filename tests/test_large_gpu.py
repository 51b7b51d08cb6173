"""Tensors past 2^31 elements (4.3 GB per BF16 tensor): 64-bit addressing end to end (GPU).

The batch is a seeded 65536 x 128 block tiled 257 times along the rows (16,842,752 rows,
2,156,003,328 elements per tensor, so the last 257 - 256 = 1 tile lies entirely past
element 2^31).  Every output row depends on its own row only, so each tile of y, rstd, dx
and dg must equal the block's own outputs bit for bit -- a property that holds at any
size; the block's outputs are checked against the FP64 oracle on sampled rows, and dw
against 257 x the oracle's dw of the block (a sum over rows).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import Case, dev_to_f64, sample_rows
from tolerance import bf16_check, dw_fp32_check, rstd_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn

BLOCK, TILES, N = 65536, 257, 128


def _enough_memory(need_bytes):
    free, _ = torch.cuda.mem_get_info()
    return free > need_bytes


@pytest.mark.parametrize("det", [True, False])
def test_past_2_31_elements(det):
    M = BLOCK * TILES
    assert M * N > 2 ** 31
    tensor = M * N * 2
    if not _enough_memory(7 * tensor + (4 << 30)):
        pytest.skip("needs about 35 GB of free device memory")
    case = Case(BLOCK, N, seed=77)
    small = gn.gnorm_ckpt_step(case.x, case.g, case.w, case.eps, case.dy, dw_fp32=True,
                               deterministic=det)
    rows = sample_rows(BLOCK, n_random=512)
    ry, rr, rdx, rdg = case.oracle_rows(rows)
    sel = torch.from_numpy(rows).cuda()
    for got, ref, name in ((small[0], ry, "y"), (small[2], rdx, "dx"), (small[3], rdg, "dg")):
        rep = bf16_check(dev_to_f64(got[sel]), ref)
        assert rep["ok"], (name, rep)
    assert rstd_check(dev_to_f64(small[1][sel]), rr)["ok"]

    x, g, dy = (t.repeat(TILES, 1) for t in (case.x, case.g, case.dy))
    try:
        y, rstd, dx, dg, dw = gn.gnorm_ckpt_step(x, g, case.w, case.eps, dy, dw_fp32=True,
                                                 deterministic=det)
        torch.cuda.synchronize()
        assert gn.gnorm_device_error(reset=True) == 0
        for big, ref, name in ((y, small[0], "y"), (dx, small[2], "dx"), (dg, small[3], "dg")):
            tiles = big.view(TILES, BLOCK, N)
            for t in range(TILES):
                assert torch.equal(tiles[t], ref), (name, t)
        assert torch.equal(rstd.view(TILES, BLOCK), small[1].expand(TILES, BLOCK))
        rep = dw_fp32_check(dev_to_f64(dw), TILES * case.oracle_dw())
        assert rep["ok"], rep
    finally:
        del x, g, dy
        torch.cuda.empty_cache()
