"""Randomised shapes, strides, weight and dw types, modes and eps against the oracle (GPU).

hypothesis draws the cases (seeded by the test database / derandomised run); each runs the
checkpointed step through the descriptor entry point and is checked element by element.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from gpu_util import bits_to_dev, dev_to_f64
from synthetic import bf16_bits_to_f64, make_inputs
from tolerance import bf16_check, dw_fp32_check, rstd_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn


def _place(t, pad):
    """t [M, N] in a buffer with `pad` extra columns per row (a row-strided view)."""
    if pad == 0:
        return t
    buf = torch.zeros(t.shape[0], t.shape[1] + pad, dtype=t.dtype, device=t.device)
    buf[:, :t.shape[1]] = t
    return buf[:, :t.shape[1]]


@settings(max_examples=40, deadline=None, derandomize=True,
          suppress_health_check=list(HealthCheck))
@given(
    n8=st.sampled_from([1, 2, 3, 8, 15, 16, 17, 32, 33, 64, 65, 128, 255, 256, 511, 512]),
    M=st.integers(min_value=0, max_value=3000),
    pads=st.tuples(*[st.sampled_from([0, 0, 8, 64]) for _ in range(6)]),
    w_fp32=st.booleans(), dw_fp32=st.booleans(), det=st.booleans(),
    eps=st.sampled_from([1e-6, 1e-3, 0.5]), g_std=st.sampled_from([1.0, 3.0]),
    seed=st.integers(min_value=0, max_value=10_000),
)
def test_random_cases(n8, M, pads, w_fp32, dw_fp32, det, eps, g_std, seed):
    N = 8 * n8
    d = make_inputs(M, N, seed=seed, g_std=g_std)
    x, g, dy = (bits_to_dev(d[k]).view(M, N) for k in ("x", "g", "dy"))
    wh = bf16_bits_to_f64(d["w"])
    if w_fp32:
        w32 = (wh + 1e-3 * np.random.default_rng(seed).standard_normal(N)).astype(np.float32)
        w = torch.from_numpy(w32).cuda()
        wh = w32.astype(np.float64)
    else:
        w = bits_to_dev(d["w"])
    x, g, dy = _place(x, pads[0]), _place(g, pads[1]), _place(dy, pads[2])
    y = _place(torch.empty(M, N, dtype=torch.bfloat16, device="cuda"), pads[3])
    dx = _place(torch.empty(M, N, dtype=torch.bfloat16, device="cuda"), pads[4])
    dg = _place(torch.empty(M, N, dtype=torch.bfloat16, device="cuda"), pads[5])
    y, rstd, dx, dg, dw = gn.gnorm_ckpt_step(x, g, w, eps, dy, y=y, dx=dx, dg=dg,
                                             dw_fp32=dw_fp32, deterministic=det)
    torch.cuda.synchronize()
    xo, go, dyo = (bf16_bits_to_f64(d[k]) for k in ("x", "g", "dy"))
    ry, rr = oracle.fwd(xo, go, wh, eps)
    rdx, rdg, rdw = oracle.bwd(dyo, xo, go, wh, rr)
    if M:
        assert bf16_check(dev_to_f64(y.contiguous()), ry)["ok"]
        assert rstd_check(dev_to_f64(rstd), rr)["ok"]
        assert bf16_check(dev_to_f64(dx.contiguous()), rdx)["ok"]
        assert bf16_check(dev_to_f64(dg.contiguous()), rdg)["ok"]
    got = dev_to_f64(dw)
    if M == 0:
        assert np.all(got == 0)
    else:
        rep = dw_fp32_check(got, rdw) if dw_fp32 else bf16_check(got, rdw)
        assert rep["ok"], rep
