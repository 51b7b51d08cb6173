"""The Python binding rejects tensors it must not hand to the library (no GPU needed).

A host tensor passed where the library expects device memory would reach a kernel as a
device pointer; a device tensor passed to the host-buffer step would reach a host copy.
The binding checks placement, dtype and shape first and raises before any CUDA call.
"""
from __future__ import annotations

import pytest
import torch

import gated_norm_b200 as gn


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_device_entry_points_reject_host_tensors():
    x = _bf16(4, 128)
    w = _bf16(128)
    with pytest.raises(ValueError, match="CUDA"):
        gn.gnorm_fwd(x, x, w, 1e-6)
    with pytest.raises(ValueError, match="CUDA"):
        gn.gnorm_bwd(x, x, x, w, torch.zeros(4))
    with pytest.raises(ValueError, match="CUDA"):
        gn.gnorm_ckpt_step(x, x, w, 1e-6, x)
    with pytest.raises(ValueError, match="CUDA"):
        gn.gnorm_dw_reduce(torch.zeros(2, 128))


def test_host_step_checks_its_tensors():
    M, N = 4, 128
    x, w = _bf16(M, N), _bf16(N)
    with pytest.raises(ValueError):
        gn.gnorm_ckpt_step_host(x.float(), x, w, 1e-6, x)        # not BF16
    with pytest.raises(ValueError):
        gn.gnorm_ckpt_step_host(x[0], x, w, 1e-6, x)              # not 2-D
    with pytest.raises(ValueError):
        gn.gnorm_ckpt_step_host(x, _bf16(M, N + 8), w, 1e-6, x)   # g of another shape
    with pytest.raises(ValueError):
        gn.gnorm_ckpt_step_host(x, x, _bf16(N + 8), 1e-6, x)      # w of another length
    with pytest.raises(ValueError):
        gn.gnorm_ckpt_step_host(x, x, w, 1e-6, x.t().contiguous().t())  # not contiguous
    # outputs are checked before the device is touched
    with pytest.raises(ValueError):
        gn.gnorm_ckpt_step_host(x, x, w, 1e-6, x, y=_bf16(M, N + 8), device="cuda:0")
    with pytest.raises(ValueError):
        gn.gnorm_ckpt_step_host(x, x, w, 1e-6, x, dw=torch.zeros(N), dw_fp32=False,
                                device="cuda:0")                  # FP32 dw for a BF16 one
    with pytest.raises(ValueError):
        gn.gnorm_ckpt_step_host(x, x, w, 1e-6, x, rstd=torch.zeros(M + 1), device="cuda:0")
