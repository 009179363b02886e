"""Pins for the decay-activation oracle (oracle/activation.py, CPU only).

The activation g = -s softplus(a) is checked against identities of softplus
that hold exactly, and the oracle's reverse pass with raw decay logits is
checked against central finite differences of the composed forward
(logits -> g -> recurrence) in fp64; planted mistakes in the derivative
must fail that check.
"""
import math

import numpy as np
import pytest

from oracle import activation, ref

from test_oracle_pins import rand_pair, rel


def test_softplus_identities():
    assert activation.softplus(0.0) == pytest.approx(math.log(2.0), abs=1e-15)
    x = np.linspace(-30, 30, 121)
    # softplus(x) - softplus(-x) = x;  softplus(-40) = exp(-40) to rounding
    assert np.max(np.abs(activation.softplus(x) - activation.softplus(-x) - x)) < 1e-13
    assert activation.softplus(-40.0) == pytest.approx(math.exp(-40.0), rel=1e-12)
    assert activation.softplus(800.0) == 800.0  # no overflow
    g = activation.decay_from_logits(x, 0.1)
    assert np.all(g < 0.0)
    assert activation.decay_from_logits(0.0, 0.3) == pytest.approx(-0.3 * math.log(2.0))
    # derivative: central differences of the activation itself
    h = 1e-6
    fd = (activation.decay_from_logits(x + h, 0.1)
          - activation.decay_from_logits(x - h, 0.1)) / (2 * h)
    assert np.max(np.abs(fd - activation.decay_grad(x, 0.1))) < 1e-9
    assert activation.decay_grad(0.0, 0.1) == pytest.approx(-0.05)


def _batched(a):
    """One pair as a B = H = 1 batch in the library layouts."""
    out = {}
    for n in ("q", "k", "v", "g", "bx"):
        out[n] = a[n][None, :, None, :]
    out["w"] = a["w"][None, :, None]
    out["u_down"] = a["u_down"][None]
    out["u_up"] = a["u_up"][None]
    out["S0"] = None if a["S0"] is None else a["S0"][None, None]
    out["m0"] = None if a["m0"] is None else a["m0"][None, None]
    return out


def _loss(inp, L, s, d_o, dS, dm):
    o, S, m = ref.fwd_batch(inp, L, threads=1, decay_scale=s)[(0, 0)]
    return float((o * d_o).sum() + (S * dS).sum() + (m * dm).sum())


def _fd_check(s, monkey=None):
    rng = np.random.default_rng(17)
    T, DK, DV, R, L = 12, 4, 4, 2, 4
    a = rand_pair(rng, T, DK, DV, R, ub_std=0.8)
    a["g"] = rng.standard_normal((T, DK))  # raw logits
    inp = _batched(a)
    d_o = rng.standard_normal((T, DV))
    dS = rng.standard_normal((DV, DK))
    dm = rng.standard_normal(DV)
    gr = ref.bwd_batch(inp, L, d_o[None, :, None, :], dS[None, None],
                       dm[None, None], threads=1, decay_scale=s)[(0, 0)]
    h = 1e-6
    fd = np.zeros((T, DK))
    for t in range(T):
        for j in range(DK):
            p = dict(inp, g=inp["g"].copy())
            p["g"][0, t, 0, j] += h
            lp = _loss(p, L, s, d_o, dS, dm)
            p["g"][0, t, 0, j] -= 2 * h
            lm = _loss(p, L, s, d_o, dS, dm)
            fd[t, j] = (lp - lm) / (2 * h)
    return rel(gr["dg"], fd)


def test_reverse_pass_through_activation_matches_finite_differences():
    assert _fd_check(0.3) < 1e-6


@pytest.mark.parametrize("mistake", ["sign", "mirrored", "unscaled"])
def test_planted_derivative_mistakes_fail(mistake, monkeypatch):
    wrong = {
        "sign": lambda a, s: +s / (1.0 + np.exp(-np.asarray(a, float))),
        "mirrored": lambda a, s: -s / (1.0 + np.exp(np.asarray(a, float))),
        "unscaled": lambda a, s: -1.0 / (1.0 + np.exp(-np.asarray(a, float))),
    }[mistake]
    monkeypatch.setattr(activation, "decay_grad", wrong)
    assert _fd_check(0.3) > 1e-3
