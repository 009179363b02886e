"""Pins for the q / k L2-normalisation oracle (oracle/normalize.py, CPU).

Normalising q and k per token makes the recurrence invariant to any
positive per-token scaling of the raw q and k, and leaves already-unit rows
unchanged: both hold exactly (to rounding) in the composed oracle.  Its
reverse pass is checked against central finite differences of the composed
forward (raw q, k -> unit rows -> recurrence) in fp64; planted mistakes in
the normalisation's derivative must fail.
"""
import numpy as np
import pytest

from oracle import normalize, ref

from test_activation_oracle import _batched
from test_oracle_pins import rand_pair, rel


def _fwd(inp, L, norm=True):
    return ref.fwd_batch(inp, L, threads=1, qk_norm=norm)[(0, 0)]


def test_scale_invariance_and_unit_rows():
    rng = np.random.default_rng(5)
    a = rand_pair(rng, 12, 6, 5, 3, ub_std=0.8)
    base = _fwd(_batched(a), 4, norm=False)  # q, k already unit rows
    assert max(rel(x, y) for x, y in zip(_fwd(_batched(a), 4), base)) < 1e-13
    b = dict(a)
    b["q"] = a["q"] * rng.uniform(0.1, 10.0, (12, 1))
    b["k"] = a["k"] * rng.uniform(0.1, 10.0, (12, 1))
    assert max(rel(x, y) for x, y in zip(_fwd(_batched(b), 4), base)) < 1e-12


def _fd_check():
    rng = np.random.default_rng(23)
    T, DK, DV, R, L = 8, 4, 3, 2, 4
    a = rand_pair(rng, T, DK, DV, R, ub_std=0.8)
    a["q"] = a["q"] * rng.uniform(0.5, 2.0, (T, 1))  # raw, not unit
    a["k"] = a["k"] * rng.uniform(0.5, 2.0, (T, 1))
    inp = _batched(a)
    d_o = rng.standard_normal((T, DV))
    dS = rng.standard_normal((DV, DK))

    def loss(p):
        o, S, _ = _fwd(p, L)
        return float((o * d_o).sum() + (S * dS).sum())

    gr = ref.bwd_batch(inp, L, d_o[None, :, None, :], dS[None, None], None,
                       threads=1, qk_norm=True)[(0, 0)]
    h = 1e-6
    worst = 0.0
    for name in ("q", "k"):
        fd = np.zeros((T, DK))
        for t in range(T):
            for j in range(DK):
                p = dict(inp, **{name: inp[name].copy()})
                p[name][0, t, 0, j] += h
                lp = loss(p)
                p[name][0, t, 0, j] -= 2 * h
                fd[t, j] = (lp - loss(p)) / (2 * h)
        worst = max(worst, rel(gr["d" + name], fd))
    return worst


def test_reverse_pass_through_normalisation_matches_finite_differences():
    assert _fd_check() < 1e-6


@pytest.mark.parametrize("mistake", ["no_projection", "no_norm_division"])
def test_planted_normalisation_mistakes_fail(mistake, monkeypatch):
    def wrong(x, dy):
        x = np.asarray(x, np.float64)
        n = np.linalg.norm(x, axis=1, keepdims=True)
        y = x / n
        if mistake == "no_projection":
            return dy / n
        return dy - y * np.sum(y * dy, axis=1, keepdims=True)
    monkeypatch.setattr(normalize, "l2_normalise_grad", wrong)
    assert _fd_check() > 1e-3
