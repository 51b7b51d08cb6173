"""The FP64 oracle against its pins, and the pins against planted mistakes.

CPU only.  Every pin must hold for the oracle; every broken copy of the oracle
below must fail at least one pin (so the pins can tell a right oracle from a
plausibly wrong one).  Mistakes are planted in copies of the oracle on the CPU,
never in the GPU path.
"""
from __future__ import annotations

import types

import numpy as np
import pytest
import scipy.special

import oracle
from oracle import gated_norm_ref as ref
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_pin_holds(pin):
    ok, detail = pin(oracle)
    assert ok, f"{pin.__name__}: {detail}"


def test_sigmoid_closed_forms_and_library():
    L = np.log(3.0)
    s = oracle.sigmoid(np.array([0.0, L, -L, 800.0, -800.0]))
    assert s[0] == 0.5
    assert abs(s[1] - 0.75) < 1e-16 and abs(s[2] - 0.25) < 1e-16
    assert s[3] == 1.0 and s[4] == 0.0  # saturates without overflow
    t = np.linspace(-60.0, 60.0, 2001)
    np.testing.assert_allclose(oracle.sigmoid(t), scipy.special.expit(t), rtol=1e-15, atol=0)
    np.testing.assert_allclose(oracle.sigmoid(-t), 1.0 - oracle.sigmoid(t), rtol=0, atol=3e-16)
    assert np.isnan(oracle.sigmoid(np.array([np.nan])))[0]


def test_degenerate_rows():
    """All-zero row: r = 1/sqrt(eps), y = 0, dx = r * u; NaN propagates."""
    N = 16
    x = np.zeros((1, N))
    g = np.linspace(-2, 2, N)[None, :]
    w = np.ones(N)
    dy = np.ones((1, N))
    y, rstd = oracle.fwd(x, g, w, 1e-6)
    assert rstd[0] == 1.0 / np.sqrt(1e-6)
    assert np.all(y == 0.0)
    dx, _, _ = oracle.bwd(dy, x, g, w, rstd)
    np.testing.assert_allclose(dx[0], rstd[0] * scipy.special.expit(g[0]) * g[0], rtol=1e-15)
    xn = np.ones((1, N)); xn[0, 3] = np.nan
    yn, rn = oracle.fwd(xn, g, w, 1e-6)
    assert np.isnan(rn[0]) and np.all(np.isnan(yn))


def test_infinities_and_huge_gates_follow_ieee_and_the_library():
    """Non-finite inputs follow IEEE arithmetic through the definition, as the library
    routines of the comparators' form do (torch sigmoid / silu / rms_norm in FP64): silu(+inf)
    = +inf, silu(-inf) = -inf * 0 = NaN; an infinite x gives r = 0, so that row's y is 0
    except NaN at the infinite element.  For a huge finite gate (sigmoid rounds to exactly 1
    in FP64) the gate derivative's bracket 1 + g (1 - sigmoid) is exactly 1, so
    dg = dy * xhat * w (closed form)."""
    import torch

    g = np.array([-np.inf, np.inf, -1e30, 1e30, 3e7, np.nan])
    tg = torch.tensor(g, dtype=torch.float64)
    with np.errstate(invalid="ignore"):
        np.testing.assert_array_equal(oracle.silu(g), torch.nn.functional.silu(tg).numpy())
    np.testing.assert_array_equal(oracle.sigmoid(g), torch.sigmoid(tg).numpy())
    N = 8
    rng = np.random.default_rng(5)
    x = rng.standard_normal((2, N))
    x[1, 3] = np.inf
    gg = rng.standard_normal((2, N))
    w = 1 + 0.1 * rng.standard_normal(N)
    with np.errstate(invalid="ignore"):
        y, r = oracle.fwd(x, gg, w, 1e-6)
    assert r[1] == 0.0 and np.isnan(y[1, 3])
    assert np.all(y[1, np.arange(N) != 3] == 0.0)
    ty = torch.nn.functional.rms_norm(torch.tensor(x[:1]), (N,), eps=1e-6).numpy()
    np.testing.assert_allclose(y[0], (ty * w * gg[:1] * scipy.special.expit(gg[:1]))[0],
                               rtol=1e-13)
    big = np.full((1, N), 3e7)
    dy = rng.standard_normal((1, N))
    _, rb = oracle.fwd(x[:1], big, w, 1e-6)
    _, dg, _ = oracle.bwd(dy, x[:1], big, w, rb)
    np.testing.assert_array_equal(dg, dy * (x[:1] * rb[:, None]) * w[None, :])


def test_ckpt_step_is_two_forwards_then_backward():
    rng = np.random.default_rng(12)
    x, g, dy = (rng.standard_normal((3, 8)) for _ in range(3))
    w = rng.standard_normal(8)
    y, rstd, dx, dg, dw = oracle.ckpt_step(x, g, w, 1e-6, dy)
    y1, r1 = oracle.fwd(x, g, w, 1e-6)
    dx1, dg1, dw1 = oracle.bwd(dy, x, g, w, r1)
    for a, b in ((y, y1), (rstd, r1), (dx, dx1), (dg, dg1), (dw, dw1)):
        assert np.array_equal(a, b)


def test_dw_rows_matches_bwd():
    rng = np.random.default_rng(13)
    x, g, dy = (rng.standard_normal((7, 24)) for _ in range(3))
    w = 1 + 0.1 * rng.standard_normal(24)
    _, rstd = oracle.fwd(x, g, w, 1e-6)
    _, _, dw = oracle.bwd(dy, x, g, w, rstd)
    parts = oracle.dw_rows(dy[:4], x[:4], g[:4], rstd[:4]) + \
        oracle.dw_rows(dy[4:], x[4:], g[4:], rstd[4:])
    np.testing.assert_allclose(parts, dw, rtol=1e-14, atol=1e-14)


# ----------------------------------------------------------------- planted mistakes

def _mutant(fwd=None, bwd=None):
    return types.SimpleNamespace(fwd=fwd or ref.fwd, bwd=bwd or ref.bwd)


def _fwd_eps_outside(x, g, w, eps):
    x, g, w = (np.asarray(a, dtype=np.float64) for a in (x, g, w))
    rstd = 1.0 / (np.sqrt(np.mean(x * x, axis=1)) + eps)
    return x * rstd[:, None] * w * g * ref.sigmoid(g), rstd


def _fwd_sum_not_mean(x, g, w, eps):
    x, g, w = (np.asarray(a, dtype=np.float64) for a in (x, g, w))
    rstd = 1.0 / np.sqrt(np.sum(x * x, axis=1) + eps)
    return x * rstd[:, None] * w * g * ref.sigmoid(g), rstd


def _fwd_sigmoid_gate(x, g, w, eps):
    y, rstd = ref.fwd(x, g, w, eps)
    g = np.asarray(g, dtype=np.float64)
    with np.errstate(invalid="ignore", divide="ignore"):
        return np.where(g != 0, y / g, 0.0), rstd


def _fwd_no_weight(x, g, w, eps):
    return ref.fwd(x, g, np.ones_like(np.asarray(w, dtype=np.float64)), eps)


def _bwd_variant(kind):
    def bwd(dy, x, g, w, rstd):
        dy, x, g, w, rstd = (np.asarray(a, dtype=np.float64) for a in (dy, x, g, w, rstd))
        r = rstd[:, None]
        xhat = x * r
        sig = ref.sigmoid(g)
        s = g * sig
        u = dy * w * s if kind != "u_no_w" else dy * s
        cx = xhat if kind != "c_uses_x" else x
        c = np.mean(u * cx, axis=1)
        if kind == "dx_sign":
            dx = r * (u + xhat * c[:, None])
        elif kind == "dx_no_r":
            dx = u - xhat * c[:, None]
        else:
            dx = r * (u - xhat * c[:, None])
        if kind == "dg_no_silu_deriv":
            dg = dy * xhat * w * sig
        elif kind == "dg_sign":
            dg = dy * xhat * w * sig * (1.0 - g * (1.0 - sig))
        elif kind == "dg_no_w":
            dg = dy * xhat * sig * (1.0 + g * (1.0 - sig))
        else:
            dg = dy * xhat * w * sig * (1.0 + g * (1.0 - sig))
        if kind == "dw_sigmoid":
            dw = np.sum(dy * xhat * sig, axis=0)
        elif kind == "dw_raw_x":
            dw = np.sum(dy * x * s, axis=0)
        elif kind == "dw_has_w":
            dw = np.sum(dy * xhat * s * w, axis=0)
        else:
            dw = np.sum(dy * xhat * s, axis=0)
        return dx, dg, dw
    return bwd


MUTANTS = {
    "eps_outside_sqrt": _mutant(fwd=_fwd_eps_outside),
    "sum_instead_of_mean": _mutant(fwd=_fwd_sum_not_mean),
    "sigmoid_gate_not_silu": _mutant(fwd=_fwd_sigmoid_gate),
    "forward_drops_weight": _mutant(fwd=_fwd_no_weight),
    "u_drops_weight": _mutant(bwd=_bwd_variant("u_no_w")),
    "c_uses_x_not_xhat": _mutant(bwd=_bwd_variant("c_uses_x")),
    "dx_wrong_sign": _mutant(bwd=_bwd_variant("dx_sign")),
    "dx_drops_rstd": _mutant(bwd=_bwd_variant("dx_no_r")),
    "dg_drops_silu_derivative": _mutant(bwd=_bwd_variant("dg_no_silu_deriv")),
    "dg_wrong_sign": _mutant(bwd=_bwd_variant("dg_sign")),
    "dg_drops_weight": _mutant(bwd=_bwd_variant("dg_no_w")),
    "dw_sigmoid_not_silu": _mutant(bwd=_bwd_variant("dw_sigmoid")),
    "dw_unnormalised_x": _mutant(bwd=_bwd_variant("dw_raw_x")),
    "dw_extra_weight": _mutant(bwd=_bwd_variant("dw_has_w")),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    orc = MUTANTS[name]
    failed = []
    for pin in ALL_PINS:
        try:
            ok, _ = pin(orc)
        except Exception:  # a crash also counts as caught
            ok = False
        if not ok:
            failed.append(pin.__name__)
    assert failed, f"no pin catches the planted mistake {name}"
