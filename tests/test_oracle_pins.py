"""Pins for the fp64 oracle (CPU only).

Each test ties the oracle to something other than itself: a hand-computed
example, the pages' chunkability theorem (an independent WY-form solve),
textbook special cases the pages say CARVE generalises (gated delta rule,
original delta rule), the closed form of unnormalised linear attention, the
chunk-0 "no content signal" rule, resume and permutation invariances, a
stability bound, and central finite differences for the reverse pass.
"""
import math
import os

import numpy as np
import pytest

from oracle import ref
from oracle.chunked import chunked_fwd_pair

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    den = max(np.abs(b).max(), 1e-300)
    return float(np.abs(a - b).max() / den)


def rand_pair(rng, T, DK, DV, R, ub_std=0.5, s0=True, m0=True, gscale=0.3):
    q = rng.standard_normal((T, DK))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, DK))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    return dict(
        q=q, k=k, v=rng.standard_normal((T, DV)),
        g=-np.log1p(np.exp(rng.standard_normal((T, DK)))) * gscale,
        bx=rng.standard_normal((T, DK)),
        w=1.0 / (1.0 + np.exp(-rng.standard_normal(T))),
        u_down=rng.standard_normal((R, DV)) * ub_std,
        u_up=rng.standard_normal((DK, R)) * ub_std,
        S0=rng.standard_normal((DV, DK)) * 0.5 if s0 else None,
        m0=rng.standard_normal(DV) * 0.5 if m0 else None)


def run(a, L, erase=0):
    return ref.fwd_pair(a["q"], a["k"], a["v"], a["g"], a["bx"], a["w"],
                        a["u_down"], a["u_up"], L, a["S0"], a["m0"], erase)


# ---------------------------------------------------------------- golden ----

def _tok(s):
    sign = -1.0 if s.startswith("-") else 1.0
    s = s.lstrip("-")
    if s.startswith("ln"):
        return sign * math.log(float(s[2:]))
    if "/" in s:
        n, d = s.split("/")
        return sign * float(n) / float(d)
    return sign * float(s)


def load_golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            parts = line.split()
            key, r, c = parts[0], int(parts[1]), int(parts[2])
            vals = [_tok(x) for x in parts[3:]]
            assert len(vals) == r * c, key
            out[key] = np.array(vals).reshape(r, c)
    return out


def test_hand_computed_two_chunk_example():
    gd = load_golden("hand_two_chunks.txt")
    L = int(gd["L"][0, 0])
    a = dict(q=gd["q"], k=gd["k"], v=gd["v"], g=gd["g"], bx=gd["bx"],
             w=gd["w"][:, 0], u_down=gd["u_down"], u_up=gd["u_up"],
             S0=gd["S0"], m0=None)
    o, S_T, m_T = run(a, L)
    np.testing.assert_allclose(o, gd["expect_o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S_T, gd["expect_S_T"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(m_T, gd["expect_m_T"][0], rtol=0, atol=1e-12)
    # first chunk alone: state and chunk mean after chunk 0
    a0 = {n: (x[:2] if n in ("q", "k", "v", "g", "bx", "w") else x)
          for n, x in a.items()}
    o0, S1, m1 = run(a0, L)
    np.testing.assert_allclose(S1, gd["expect_S_after_chunk0"], atol=1e-12)
    np.testing.assert_allclose(m1, gd["expect_m_after_chunk0"][0], atol=1e-12)


# ------------------------------------------------------- chunkability -------

@pytest.mark.parametrize("L", [1, 2, 3, 16])
def test_chunked_solve_equals_token_recurrence(L):
    rng = np.random.default_rng(100 + L)
    a = rand_pair(rng, T=37, DK=5, DV=4, R=2)
    o, S, m = run(a, L)
    oc, Sc, mc = chunked_fwd_pair(**a, L=L)
    assert rel(oc, o) < 1e-12
    assert rel(Sc, S) < 1e-12
    assert rel(mc, m) < 1e-12


@pytest.mark.parametrize("L", [1, 2, 3, 16])
def test_other_erase_form_chunked_solve_equals_token_recurrence(L):
    # the other key-axis erase, S' (I - (b (.) k) k^T): its single-key WY
    # chunk form against the token loop
    rng = np.random.default_rng(200 + L)
    a = rand_pair(rng, T=37, DK=5, DV=4, R=2)
    o, S, m = run(a, L, erase=1)
    oc, Sc, mc = chunked_fwd_pair(**a, L=L, erase=1)
    assert rel(oc, o) < 1e-12 and rel(Sc, S) < 1e-12 and rel(mc, m) < 1e-12


def test_erase_forms_coincide_for_a_channel_constant_gate():
    # k (b k)^T = (b k) k^T when b is the same on every key channel (U_b = 0
    # and a channel-constant erase logit); with per-channel b they differ
    rng = np.random.default_rng(9)
    a = rand_pair(rng, T=30, DK=6, DV=4, R=2)
    diff = max(rel(x, y) for x, y in zip(run(a, 4, 1), run(a, 4, 0)))
    assert diff > 1e-3
    a["bx"] = np.repeat(rng.standard_normal((30, 1)), 6, axis=1)
    a["u_down"] = np.zeros_like(a["u_down"])
    a["u_up"] = np.zeros_like(a["u_up"])
    assert max(rel(x, y) for x, y in zip(run(a, 4, 1), run(a, 4, 0))) < 1e-13


@pytest.mark.parametrize("block", [1, 2, 4, 8])
def test_chunk_solved_in_blocks_equals_recurrence(block):
    # the gate is constant over a chunk, so a chunk may be solved as blocks
    rng = np.random.default_rng(7)
    a = rand_pair(rng, T=40, DK=6, DV=3, R=2)
    o, S, m = run(a, 8)
    oc, Sc, mc = chunked_fwd_pair(**a, L=8, block=block)
    assert rel(oc, o) < 1e-12 and rel(Sc, S) < 1e-12 and rel(mc, m) < 1e-12


# ---------------------------------------------------- special cases ---------

def test_reduces_to_gated_delta_rule_with_scalar_gates():
    """U_b = 0, scalar-broadcast decay and erase logit, w = sigmoid(bx):
    S_t = a_t S_{t-1} (I - beta_t k k^T) + beta_t v k^T (textbook form
    S_t = a S + beta (v - a S k) k^T), outputs read S_{t-1} q_t."""
    rng = np.random.default_rng(3)
    T, DK, DV = 29, 6, 5
    a = rand_pair(rng, T, DK, DV, R=3)
    gs = -np.abs(rng.standard_normal(T)) * 0.2
    xs = rng.standard_normal(T)
    a["g"] = np.repeat(gs[:, None], DK, axis=1)
    a["bx"] = np.repeat(xs[:, None], DK, axis=1)
    beta = 1.0 / (1.0 + np.exp(-xs))
    a["w"] = beta
    a["u_down"] = np.zeros_like(a["u_down"])
    a["u_up"] = np.zeros_like(a["u_up"])
    a["m0"] = None
    o, S_T, _ = run(a, 4)
    S = a["S0"].copy()
    o_ref = np.zeros((T, DV))
    for t in range(T):
        o_ref[t] = S @ a["q"][t]
        al = math.exp(gs[t])
        kt = a["k"][t]
        S = al * S + beta[t] * np.outer(a["v"][t] - al * (S @ kt), kt)
    assert rel(o, o_ref) < 1e-12
    assert rel(S_T, S) < 1e-12


def test_reduces_to_original_delta_rule():
    rng = np.random.default_rng(4)
    T, DK, DV = 23, 4, 4
    a = rand_pair(rng, T, DK, DV, R=2, m0=False)
    a["g"] = np.zeros((T, DK))
    beta = 0.7
    a["bx"] = np.full((T, DK), math.log(beta / (1 - beta)))
    a["w"] = np.full(T, beta)
    a["u_down"] *= 0
    o, S_T, _ = run(a, 5)
    S = a["S0"].copy()
    for t in range(T):
        kt = a["k"][t]
        S = S + beta * np.outer(a["v"][t] - S @ kt, kt)
    assert rel(S_T, S) < 1e-12


def test_linear_attention_closed_form_independent_of_Ub():
    """g = 0, bx = -inf (sigmoid = 0 exactly), w = 1:
    S_T = S0 + V^T K and o_t = S0 q_t + sum_{i<t} v_i (k_i . q_t)."""
    rng = np.random.default_rng(5)
    T, DK, DV = 33, 5, 6
    a = rand_pair(rng, T, DK, DV, R=2, ub_std=3.0)
    a["g"] = np.zeros((T, DK))
    a["bx"] = np.full((T, DK), -np.inf)
    a["w"] = np.ones(T)
    o, S_T, _ = run(a, 4)
    K, Q, V, S0 = a["k"], a["q"], a["v"], a["S0"]
    assert rel(S_T, S0 + V.T @ K) < 1e-12
    o_ref = Q @ S0.T + np.tril(Q @ K.T, -1) @ V
    assert rel(o, o_ref) < 1e-12


def test_no_content_signal_within_first_chunk():
    """Tokens of chunk 0 never see U_b (the summary's stated limitation)."""
    rng = np.random.default_rng(6)
    a = rand_pair(rng, T=16, DK=4, DV=4, R=2, ub_std=2.0, m0=False)
    o1, S1, _ = run(a, 16)
    z = dict(a, u_down=np.zeros_like(a["u_down"]))
    o0, S0_, _ = run(z, 16)
    assert np.array_equal(o1, o0) and np.array_equal(S1, S0_)
    # one more token opens chunk 1, where the gate must change the state
    b = rand_pair(np.random.default_rng(6), T=17, DK=4, DV=4, R=2, ub_std=2.0,
                  m0=False)
    _, Sb1, _ = run(b, 16)
    _, Sb0, _ = run(dict(b, u_down=np.zeros_like(b["u_down"])), 16)
    assert rel(Sb1, Sb0) > 1e-6


def test_zero_Ub_is_independent_of_chunk_length():
    rng = np.random.default_rng(8)
    a = rand_pair(rng, T=48, DK=5, DV=4, R=2, m0=False)
    a["u_down"] *= 0
    outs = [run(a, L) for L in (1, 4, 16, 48)]
    for o, S, _ in outs[1:]:
        assert rel(o, outs[0][0]) < 1e-12 and rel(S, outs[0][1]) < 1e-12


def test_resume_from_state_and_mean():
    rng = np.random.default_rng(9)
    L = 4
    a = rand_pair(rng, T=24, DK=4, DV=3, R=2)
    o, S, m = run(a, L)
    cut = 12
    head = {n: (x[:cut] if n in ("q", "k", "v", "g", "bx", "w") else x)
            for n, x in a.items()}
    oh, Sh, mh = run(head, L)
    tail = {n: (x[cut:] if n in ("q", "k", "v", "g", "bx", "w") else x)
            for n, x in a.items()}
    tail["S0"], tail["m0"] = Sh, mh
    ot, St, mt = run(tail, L)
    assert rel(np.vstack([oh, ot]), o) < 1e-14
    assert rel(St, S) < 1e-14 and rel(mt, m) < 1e-14


def test_value_channel_permutation_equivariance():
    rng = np.random.default_rng(10)
    a = rand_pair(rng, T=20, DK=4, DV=6, R=3)
    o, S, m = run(a, 4)
    perm = rng.permutation(6)
    b = dict(a, v=a["v"][:, perm], S0=a["S0"][perm], m0=a["m0"][perm],
             u_down=a["u_down"][:, perm])
    ob, Sb, mb = run(b, 4)
    assert rel(ob, o[:, perm]) < 1e-13
    assert rel(Sb, S[perm]) < 1e-13 and rel(mb, m[perm]) < 1e-13


def test_scalar_gate_state_norm_bound():
    """Scalar b (U_b = 0, broadcast bx) and unit k: ||I - beta k k^T||_2 <= 1,
    so ||S_t|| <= a_max ||S_{t-1}|| + w_t ||v_t||, hence
    ||S_t|| <= ||S0|| + max_t(w_t ||v_t||) / (1 - a_max) for every t."""
    rng = np.random.default_rng(11)
    T, DK, DV = 400, 6, 5
    a = rand_pair(rng, T, DK, DV, R=2, m0=False)
    gs = -np.log1p(np.exp(rng.standard_normal(T))) * 0.1
    a["g"] = np.repeat(gs[:, None], DK, axis=1)
    a["bx"] = np.repeat(rng.standard_normal(T)[:, None], DK, axis=1)
    a["u_down"] *= 0
    amax = float(np.exp(gs.max()))
    bound = (np.linalg.norm(a["S0"], 2)
             + float((a["w"] * np.linalg.norm(a["v"], axis=1)).max())
             / (1 - amax))
    for Tp in (1, 7, 50, 200, 400):
        sub = {n: (x[:Tp] if n in ("q", "k", "v", "g", "bx", "w") else x)
               for n, x in a.items()}
        _, S, _ = run(sub, 8)
        assert np.linalg.norm(S, 2) <= bound * (1 + 1e-12)


def test_per_channel_gate_state_stays_bounded():
    """Per-key-channel erase is not a per-step contraction in general (the
    Lyapunov theorem is not stated on the pages); check empirically that the
    state norm shows no growth trend over a long run."""
    rng = np.random.default_rng(12)
    T, DK, DV = 4096, 8, 8
    a = rand_pair(rng, T, DK, DV, R=2, ub_std=0.02, m0=False)
    a["g"] = -np.log1p(np.exp(rng.standard_normal((T, DK)))) * 0.1
    norms = []
    for Tp in (512, 1024, 2048, 4096):
        sub = {n: (x[:Tp] if n in ("q", "k", "v", "g", "bx", "w") else x)
               for n, x in a.items()}
        norms.append(np.linalg.norm(run(sub, 64)[1]))
    assert max(norms[1:]) < 2.0 * max(norms[0], 1.0)


# ---------------------------------------------------------- backward --------

def _loss_parts(a, L, Ro, RS, Rm, erase=0):
    o, S, m = run(a, L, erase)
    return float((o * Ro).sum() + (S * RS).sum() + (m * Rm).sum())


@pytest.mark.parametrize("erase", [0, 1])
def test_backward_matches_central_finite_differences(erase):
    rng = np.random.default_rng(13)
    T, DK, DV, R, L = 12, 4, 4, 2, 4
    a = rand_pair(rng, T, DK, DV, R, ub_std=0.8)
    Ro = rng.standard_normal((T, DV))
    RS = rng.standard_normal((DV, DK))
    Rm = rng.standard_normal(DV)
    gr = ref.bwd_pair(a["q"], a["k"], a["v"], a["g"], a["bx"], a["w"],
                      a["u_down"], a["u_up"], L, Ro, a["S0"], a["m0"], RS, Rm,
                      erase)
    names = dict(q="dq", k="dk", v="dv", g="dg", bx="dbx", w="dw",
                 u_down="du_down", u_up="du_up", S0="dS0", m0="dm0")
    for name, gname in names.items():
        x = a[name]
        scale = max(float(np.abs(x).max()), 1.0)
        h = 1e-6 * scale
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            fp = _loss_parts(dict(a, **{name: xp}), L, Ro, RS, Rm, erase)
            fm = _loss_parts(dict(a, **{name: xm}), L, Ro, RS, Rm, erase)
            fd[idx] = (fp - fm) / (2 * h)
        err = rel(gr[gname], fd)
        assert err < 1e-6, (name, err)


def test_backward_linear_attention_closed_form():
    """g = 0, bx = -inf, w = 1 and zero upstream dS_T, dm_T:
    dq_t = S_{t-1}^T do_t,  dv_i = sum_{t>i} do_t (k_i . q_t),
    dS0 = sum_t do_t q_t^T."""
    rng = np.random.default_rng(14)
    T, DK, DV = 19, 4, 5
    a = rand_pair(rng, T, DK, DV, R=2)
    a["g"] = np.zeros((T, DK))
    a["bx"] = np.full((T, DK), -np.inf)
    a["w"] = np.ones(T)
    do = rng.standard_normal((T, DV))
    gr = ref.bwd_pair(a["q"], a["k"], a["v"], a["g"], a["bx"], a["w"],
                      a["u_down"], a["u_up"], 4, do, a["S0"], a["m0"])
    K, Q, V, S0 = a["k"], a["q"], a["v"], a["S0"]
    P = np.tril(Q @ K.T, -1)              # P[t, i] = q_t . k_i, i < t
    assert rel(gr["dv"], P.T @ do) < 1e-12
    assert rel(gr["dS0"], do.T @ Q) < 1e-12
    Sprev = np.cumsum(np.einsum("tv,tk->tvk", V, K), axis=0)
    Sprev = np.concatenate([np.zeros((1, DV, DK)), Sprev[:-1]]) + S0[None]
    assert rel(gr["dq"], np.einsum("tvk,tv->tk", Sprev, do)) < 1e-12
