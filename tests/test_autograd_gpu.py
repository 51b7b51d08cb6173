"""The autograd wrapper against torch autograd of the same composition in FP64 (GPU)."""
from __future__ import annotations

import pytest
import torch

from gpu_util import Case, dev_to_f64
from tolerance import bf16_check, dw_fp32_check

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn


def _reference_grads(x, g, w, dy, eps):
    xr, gr, wr = (t.detach().double().cpu().requires_grad_(True) for t in (x, g, w))
    out = torch.nn.functional.rms_norm(xr, (x.shape[-1],), weight=wr, eps=eps) * \
        torch.nn.functional.silu(gr)
    out.backward(dy.detach().double().cpu())
    return out.detach(), xr.grad, gr.grad, wr.grad


@pytest.mark.parametrize("w_dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", [(4, 33, 128), (257, 256), (9, 4096)])
def test_autograd_matches_torch(shape, w_dtype):
    N = shape[-1]
    torch.manual_seed(0)
    x = torch.randn(shape, device="cuda").to(torch.bfloat16).requires_grad_(True)
    g = (2 * torch.randn(shape, device="cuda")).to(torch.bfloat16).requires_grad_(True)
    w = (1 + 0.1 * torch.randn(N, device="cuda")).to(w_dtype).requires_grad_(True)
    dy = torch.randn(shape, device="cuda").to(torch.bfloat16)
    y = gn.gated_rmsnorm(x, g, w, 1e-6)
    y.backward(dy)
    torch.cuda.synchronize()
    ry, rdx, rdg, rdw = _reference_grads(x, g, w, dy, 1e-6)
    flat = lambda t: t.reshape(-1, N).numpy()
    assert bf16_check(dev_to_f64(y.reshape(-1, N)), flat(ry))["ok"]
    assert bf16_check(dev_to_f64(x.grad.reshape(-1, N)), flat(rdx))["ok"]
    assert bf16_check(dev_to_f64(g.grad.reshape(-1, N)), flat(rdg))["ok"]
    assert w.grad.dtype == w_dtype
    got_dw = dev_to_f64(w.grad)
    rep = dw_fp32_check(got_dw, rdw.numpy()) if w_dtype == torch.float32 else \
        bf16_check(got_dw, rdw.numpy())
    assert rep["ok"], rep


def test_module_in_a_training_step():
    torch.manual_seed(1)
    norm = gn.GatedRMSNorm(256, device="cuda", dtype=torch.float32)
    opt = torch.optim.SGD(norm.parameters(), lr=0.1)
    x = torch.randn(512, 256, device="cuda").to(torch.bfloat16)
    g = torch.randn(512, 256, device="cuda").to(torch.bfloat16)
    before = norm.weight.detach().clone()
    loss = norm(x, g).float().square().mean()
    loss.backward()
    opt.step()
    torch.cuda.synchronize()
    assert torch.isfinite(loss)
    assert not torch.equal(before, norm.weight.detach())
