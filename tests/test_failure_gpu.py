"""Bounded waits: a wait that runs out reports and returns; the context stays usable (GPU).

Every pipeline wait in the kernels gives up after a time limit, sets a bit in the device
error word and lets the kernel return.  The self-test entry point makes one such wait run
out on purpose (a barrier nothing arrives on, 20 ms limit); nothing faults, traps or hangs.
"""
from __future__ import annotations

import pytest
import torch

from gpu_util import Case, dev_to_f64
from tolerance import bf16_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn


def test_wait_runs_out_reports_and_context_survives():
    assert gn.gnorm_device_error(reset=True) == 0
    waited = gn.gnorm_selftest_wait_timeout(20000)
    assert 20e6 <= waited < 1e9, waited          # gave up after its 20 ms limit
    assert gn.gnorm_device_error(reset=True) == 4  # and said so
    assert gn.gnorm_device_error(reset=False) == 0
    case = Case(300, 256, seed=31)                # the next real call works as usual
    y, rstd = gn.gnorm_fwd(case.x, case.g, case.w, case.eps)
    torch.cuda.synchronize()
    ry, _, _, _ = case.oracle_rows()
    assert bf16_check(dev_to_f64(y), ry)["ok"]
    assert gn.gnorm_device_error(reset=True) == 0
