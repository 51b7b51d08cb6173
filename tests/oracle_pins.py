"""Pins for the FP64 oracle: checks against facts that do not come from the oracle.

Each pin takes an oracle-like object (anything with ``fwd(x, g, w, eps)`` and
``bwd(dy, x, g, w, rstd)``) and returns ``(ok, detail)``.  The test suite runs
every pin against the real oracle (all must hold) and against deliberately
broken copies of it (each must be caught by at least one pin), so a plausible
mistake anywhere in the oracle -- a dropped term, a wrong sign, a transposed
reduction, eps in the wrong place -- fails one of them.

The independent facts are: a hand-derived worked example (closed forms), the
library routines ``torch.nn.functional.rms_norm`` / ``silu`` and torch
autograd in FP64, central finite differences, the g -> +inf limit and the
orthogonality of dx to x when eps = 0.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_n4.json")


def _rng_case(seed, M, N, g_std=1.0, x_scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, N)) * x_scale
    g = rng.standard_normal((M, N)) * g_std
    w = 1.0 + 0.1 * rng.standard_normal(N)
    dy = rng.standard_normal((M, N))
    return x, g, w, dy


def _max_rel(a, b, floor=1e-300):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    scale = np.maximum(np.max(np.abs(b)), floor)
    return float(np.max(np.abs(a - b)) / scale) if a.size else 0.0


def load_golden():
    with open(GOLDEN) as f:
        d = json.load(f)
    env = {"L": math.log(3.0)}

    def ev(v):
        if isinstance(v, list):
            return [ev(e) for e in v]
        if isinstance(v, str):
            return float(eval(v, {"__builtins__": {}}, env))  # closed-form strings only
        return float(v)

    return {k: (np.array(ev(v)) if k not in ("about", "derivation", "eps") else v)
            for k, v in d.items()}


# --------------------------------------------------------------------------- pins

def pin_golden(orc):
    """Hand-derived worked example (tests/golden/closed_form_n4.json)."""
    d = load_golden()
    y, rstd = orc.fwd(d["x"], d["g"], d["w"], d["eps"])
    dx, dg, dw = orc.bwd(d["dy"], d["x"], d["g"], d["w"], rstd)
    errs = {
        "rstd": _max_rel(rstd, d["rstd"]),
        "y": _max_rel(y, d["y"]),
        "dx": _max_rel(dx, d["dx"]),
        "dg": _max_rel(dg, d["dg"]),
        "dw": _max_rel(dw, d["dw"]),
    }
    return all(e < 1e-13 for e in errs.values()), errs


def pin_library_forward(orc):
    """y = rms_norm(x, w, eps) * silu(g) with torch's FP64 library routines."""
    x, g, w, _ = _rng_case(1, 5, 24)
    eps = 1e-6
    y, rstd = orc.fwd(x, g, w, eps)
    xt, gt, wt = (torch.from_numpy(a) for a in (x, g, w))
    ref = torch.nn.functional.rms_norm(xt, (x.shape[1],), weight=wt, eps=eps) * \
        torch.nn.functional.silu(gt)
    ref_rstd = torch.rsqrt(torch.mean(xt * xt, dim=1) + eps)  # torch library reduction
    e_y = _max_rel(y, ref.numpy())
    e_r = _max_rel(rstd, ref_rstd.numpy())
    return e_y < 1e-13 and e_r < 1e-13, {"y": e_y, "rstd": e_r}


def pin_autograd_backward(orc):
    """dx, dg, dw equal torch autograd (FP64) of rms_norm(x, w) * silu(g)."""
    x, g, w, dy = _rng_case(2, 6, 40, g_std=2.0)
    eps = 1e-5
    xt = torch.tensor(x, requires_grad=True)
    gt = torch.tensor(g, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    out = torch.nn.functional.rms_norm(xt, (x.shape[1],), weight=wt, eps=eps) * \
        torch.nn.functional.silu(gt)
    out.backward(torch.tensor(dy))
    _, rstd = orc.fwd(x, g, w, eps)
    dx, dg, dw = orc.bwd(dy, x, g, w, rstd)
    errs = {
        "dx": _max_rel(dx, xt.grad.numpy()),
        "dg": _max_rel(dg, gt.grad.numpy()),
        "dw": _max_rel(dw, wt.grad.numpy()),
    }
    return all(e < 1e-12 for e in errs.values()), errs


def pin_finite_differences(orc):
    """Central differences of L = sum(dy * y) w.r.t. x, g and w (M<=4, N in 8/16/24)."""
    worst = {}
    ok = True
    h = 1e-6
    for (M, N, seed) in ((1, 8, 3), (3, 16, 4), (4, 24, 5)):
        x, g, w, dy = _rng_case(seed, M, N)
        eps = 1e-3

        def loss(xx, gg, ww):
            yy, _ = orc.fwd(xx, gg, ww, eps)
            return float(np.sum(dy * yy))

        _, rstd = orc.fwd(x, g, w, eps)
        dx, dg, dw = orc.bwd(dy, x, g, w, rstd)
        for name, base, grad in (("dx", x, dx), ("dg", g, dg), ("dw", w, dw)):
            fd = np.zeros_like(base)
            it = np.nditer(base, flags=["multi_index"])
            for _ in it:
                idx = it.multi_index
                p = base.copy(); p[idx] += h
                m = base.copy(); m[idx] -= h
                args_p = {"dx": (p, g, w), "dg": (x, p, w), "dw": (x, g, p)}[name]
                args_m = {"dx": (m, g, w), "dg": (x, m, w), "dw": (x, g, m)}[name]
                fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
            e = _max_rel(grad, fd)
            worst[f"{name}@{M}x{N}"] = e
            ok = ok and e < 1e-7
    return ok, worst


def pin_gate_limit(orc):
    """g in [20, 40]: sigmoid(g) = 1 - O(2e-9), so y -> rmsnorm(x) * w * g."""
    rng = np.random.default_rng(6)
    M, N = 4, 32
    x = rng.standard_normal((M, N))
    g = rng.uniform(20.0, 40.0, (M, N))
    w = 1.0 + 0.1 * rng.standard_normal(N)
    eps = 1e-6
    y, _ = orc.fwd(x, g, w, eps)
    xt = torch.from_numpy(x)
    rms = torch.nn.functional.rms_norm(xt, (N,), eps=eps).numpy()
    ref = rms * w[None, :] * g
    e = float(np.max(np.abs(y - ref) / np.abs(ref)))
    return e < 1e-8, {"y": e}


def pin_zero_gate(orc):
    """g = 0: y = 0 exactly and dg = dy * xhat * w / 2 (silu'(0) = 1/2)."""
    x, _, w, dy = _rng_case(7, 3, 16)
    g = np.zeros_like(x)
    y, rstd = orc.fwd(x, g, w, 1e-6)
    _, dg, dw = orc.bwd(dy, x, g, w, rstd)
    xhat = torch.nn.functional.rms_norm(torch.from_numpy(x), (x.shape[1],), eps=1e-6).numpy()
    ref_dg = 0.5 * dy * xhat * w[None, :]
    ok = bool(np.all(y == 0.0)) and bool(np.all(dw == 0.0)) and _max_rel(dg, ref_dg) < 1e-14
    return ok, {"max|y|": float(np.max(np.abs(y))), "dg": _max_rel(dg, ref_dg)}


def pin_orthogonality(orc):
    """sum_j dx_j x_j = r * sum_j(u_j x_j) * eps / (ms + eps); 0 when eps = 0.

    A scale-invariant function of x has a gradient orthogonal to x; eps breaks
    the invariance by exactly this amount.
    """
    errs = {}
    ok = True
    for eps in (0.0, 0.5):
        x, g, w, dy = _rng_case(8, 5, 32)
        _, rstd = orc.fwd(x, g, w, eps)
        dx, _, _ = orc.bwd(dy, x, g, w, rstd)
        lhs = np.sum(dx * x, axis=1)
        ms = np.mean(x * x, axis=1)
        r = 1.0 / np.sqrt(ms + eps)
        u = dy * w[None, :] * torch.nn.functional.silu(torch.from_numpy(g)).numpy()
        rhs = r * np.sum(u * x, axis=1) * eps / (ms + eps)
        scale = np.max(np.abs(r * np.sum(u * x, axis=1)))
        e = float(np.max(np.abs(lhs - rhs)) / scale)
        errs[f"eps={eps}"] = e
        ok = ok and e < 1e-13
    return ok, errs


def pin_scale_invariance(orc):
    """y(50 x) = y(x) up to eps: exactly y(x) * sqrt(ms + eps) / sqrt(ms + eps / 2500)."""
    x, g, w, _ = _rng_case(9, 4, 64)
    eps = 1e-2
    y1, _ = orc.fwd(x, g, w, eps)
    y50, _ = orc.fwd(50.0 * x, g, w, eps)
    ms = np.mean(x * x, axis=1)
    factor = np.sqrt(ms + eps) / np.sqrt(ms + eps / 2500.0)
    e = _max_rel(y50, y1 * factor[:, None])
    return e < 1e-13, {"y": e}


def pin_dw_linearity(orc):
    """dw is linear in dy and a sum over rows (split rows, add)."""
    x, g, w, dy = _rng_case(10, 8, 16)
    dy2 = np.random.default_rng(11).standard_normal(dy.shape)
    _, rstd = orc.fwd(x, g, w, 1e-6)
    _, _, dw_a = orc.bwd(dy, x, g, w, rstd)
    _, _, dw_b = orc.bwd(dy2, x, g, w, rstd)
    _, _, dw_ab = orc.bwd(2.0 * dy - 3.0 * dy2, x, g, w, rstd)
    _, _, dw_top = orc.bwd(dy[:3], x[:3], g[:3], w, rstd[:3])
    _, _, dw_bot = orc.bwd(dy[3:], x[3:], g[3:], w, rstd[3:])
    e1 = _max_rel(dw_ab, 2.0 * dw_a - 3.0 * dw_b)
    e2 = _max_rel(dw_top + dw_bot, dw_a)
    return e1 < 1e-13 and e2 < 1e-13, {"linear": e1, "split": e2}


ALL_PINS = [
    pin_golden,
    pin_library_forward,
    pin_autograd_backward,
    pin_finite_differences,
    pin_gate_limit,
    pin_zero_gate,
    pin_orthogonality,
    pin_scale_invariance,
    pin_dw_linearity,
]
