"""Calls on several streams at once, and from several host threads (GPU).

The entry points keep no state between calls apart from the caller's buffers (the device
error word aside), so checkpointed steps enqueued on four streams at once, each with its
own workspace, must give bitwise the results of the same steps run one after the other;
so must host-buffer steps issued from two threads, each with its own stream and device
buffer.
"""
from __future__ import annotations

import threading

import numpy as np
import pytest
import torch

from gpu_util import Case

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import gated_norm_b200 as gn


def _serial(cases, det):
    out = []
    for c in cases:
        ws = torch.zeros(gn.gnorm_bwd_workspace_bytes(c.M, c.N, det), dtype=torch.uint8,
                         device="cuda")
        out.append(gn.gnorm_ckpt_step(c.x, c.g, c.w, c.eps, c.dy, dw_fp32=True,
                                      deterministic=det, workspace_buf=ws))
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("det", [True, False])
def test_four_streams_at_once(det):
    shapes = [(4099, 128), (2500, 256), (300, 4096), (65536, 64)]
    cases = [Case(M, N, seed=40 + i) for i, (M, N) in enumerate(shapes)]
    ref = _serial(cases, det)
    streams = [torch.cuda.Stream() for _ in cases]
    wss = [torch.zeros(gn.gnorm_bwd_workspace_bytes(c.M, c.N, det), dtype=torch.uint8,
                       device="cuda") for c in cases]
    torch.cuda.synchronize()
    for rep in range(3):
        outs = []
        for c, s, ws in zip(cases, streams, wss):
            with torch.cuda.stream(s):
                outs.append(gn.gnorm_ckpt_step(c.x, c.g, c.w, c.eps, c.dy, dw_fp32=True,
                                               deterministic=det, workspace_buf=ws, stream=s))
        torch.cuda.synchronize()
        for got, exp in zip(outs, ref):
            for a, b in zip(got[:4], exp[:4]):
                assert torch.equal(a, b)
            if det:
                assert torch.equal(got[4], exp[4])
            else:
                assert torch.allclose(got[4], exp[4], rtol=1e-4, atol=1e-4 * exp[4].abs().max())
    assert gn.gnorm_device_error(reset=True) == 0


def test_host_steps_from_two_threads():
    cases = [Case(3001, 128, seed=50), Case(1300, 512, seed=51)]  # one chunk each
    ref = _serial(cases, True)

    def host(c):
        def cpu(bits):
            t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
            return t.pin_memory()
        return tuple(cpu(c.host[k]) for k in ("x", "g", "w", "dy"))

    inputs = [host(c) for c in cases]
    bufs = [torch.empty(gn.gnorm_ckpt_step_host_bytes(c.M, c.N, True), dtype=torch.uint8,
                        device="cuda") for c in cases]
    results = [None, None]
    errors = []

    def run(i):
        try:
            torch.cuda.set_device(0)
            s = torch.cuda.Stream()
            x, g, w, dy = inputs[i]
            for _ in range(3):
                out = gn.gnorm_ckpt_step_host(x, g, w, cases[i].eps, dy, dw_fp32=True,
                                              dev_buf=bufs[i], stream=s)
            s.synchronize()
            results[i] = out
        except Exception as e:  # reported below, in the main thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for got, exp in zip(results, ref):
        for a, b in zip(got[:4], exp[:4]):
            assert torch.equal(a, b.cpu())
        assert torch.equal(got[4], exp[4].cpu())  # one chunk each: dw equals the device step's
    assert gn.gnorm_device_error(reset=True) == 0
