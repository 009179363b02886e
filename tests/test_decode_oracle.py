"""Pins for the decode-step oracle (``oracle/decode.py``, CPU only).

The decode step is the token loop of the recurrence with the chunk
bookkeeping carried between calls, so T steps of it must reproduce the
token-recurrence oracle (``oracle/carve_oracle.c``, itself pinned in
test_oracle_pins.py) over the same T tokens: every output o_t, the final
state, and the content signal -- the decode carry m is the mean of the last
complete chunk, and osum / L is the C oracle's m_T after a partial chunk.
Planted mistakes in copies of the step must break the pin.
"""
import numpy as np
import pytest

from oracle import decode, ref

from test_oracle_pins import rand_pair, rel


def _decode_all(a, L, T, pos0=0, S=None, m=None, osum=None):
    DV, DK = a["v"].shape[1], a["q"].shape[1]
    S = np.zeros((DV, DK)) if S is None else S
    m = np.zeros(DV) if m is None else m
    osum = np.zeros(DV) if osum is None else osum
    return decode.decode_steps(S, m, osum, pos0, a["q"][:T], a["k"][:T],
                               a["v"][:T], a["g"][:T], a["bx"][:T],
                               a["w"][:T], a["u_down"], a["u_up"], L)


@pytest.mark.parametrize("T,L", [(12, 4), (13, 4), (9, 3), (5, 8), (16, 1)])
def test_decode_steps_equal_token_recurrence(T, L):
    rng = np.random.default_rng(100 + T * 7 + L)
    a = rand_pair(rng, T, 6, 5, 3, ub_std=0.8)
    o, S, m, osum = _decode_all(a, L, T, S=a["S0"].copy(), m=a["m0"].copy())
    o_ref, S_ref, m_ref = ref.fwd_pair(a["q"], a["k"], a["v"], a["g"],
                                       a["bx"], a["w"], a["u_down"],
                                       a["u_up"], L, a["S0"], a["m0"])
    assert rel(o, o_ref) < 1e-12
    assert rel(S, S_ref) < 1e-12
    if T % L == 0:
        assert rel(m, m_ref) < 1e-12
        assert np.all(osum == 0.0)
    else:
        # a partial last chunk: the C oracle reports its sum / L
        assert rel(osum / L, m_ref) < 1e-12
        Tc = T - T % L  # decode's m is the last complete chunk's mean
        m_c = ref.fwd_pair(a["q"][:Tc], a["k"][:Tc], a["v"][:Tc], a["g"][:Tc],
                           a["bx"][:Tc], a["w"][:Tc], a["u_down"], a["u_up"],
                           L, a["S0"], a["m0"])[2] if Tc else a["m0"]
        assert rel(m, m_c) < 1e-12


def test_decode_steps_other_erase_form_equal_token_recurrence():
    rng = np.random.default_rng(61)
    a = rand_pair(rng, 13, 6, 5, 3, ub_std=0.8)
    DV = 5
    o, S, m, osum = decode.decode_steps(
        a["S0"].copy(), a["m0"].copy(), np.zeros(DV), 0, a["q"], a["k"],
        a["v"], a["g"], a["bx"], a["w"], a["u_down"], a["u_up"], 4, erase=1)
    o_ref, S_ref, m_ref = ref.fwd_pair(a["q"], a["k"], a["v"], a["g"],
                                       a["bx"], a["w"], a["u_down"],
                                       a["u_up"], 4, a["S0"], a["m0"], erase=1)
    assert rel(o, o_ref) < 1e-12 and rel(S, S_ref) < 1e-12
    assert rel(osum / 4, m_ref) < 1e-12  # 13 tokens: a partial last chunk


def test_decode_resumes_mid_chunk():
    # stopping after 6 tokens (mid-chunk, L = 4) and continuing from the
    # carried (S, m, osum, pos) equals one run over all 14 tokens
    rng = np.random.default_rng(7)
    a = rand_pair(rng, 14, 4, 4, 2, ub_std=1.0)
    o_all, S_all, m_all, s_all = _decode_all(a, 4, 14)
    o1, S1, m1, s1 = _decode_all(a, 4, 6)
    b = {k: (v[6:] if k in ("q", "k", "v", "g", "bx", "w") else v)
         for k, v in a.items()}
    o2, S2, m2, s2 = _decode_all(b, 4, 8, pos0=6, S=S1, m=m1, osum=s1)
    assert rel(np.concatenate([o1, o2]), o_all) == 0.0
    assert rel(S2, S_all) == 0.0 and rel(m2, m_all) == 0.0


def _broken(kind):
    def step(S, m, osum, pos, q, k, v, g, bx, w, u_down, u_up, L, erase=0):
        p = u_up @ (u_down @ m)
        b = decode.sigmoid(bx + p)
        o = S @ q
        S1 = S * np.exp(g)[None, :]
        if kind == "read_after_write":
            o = None
        e = S1 @ k
        kap = k if kind == "ungated_erase" else b * k
        S_new = S1 - np.outer(e, kap) + w * np.outer(v, k)
        if kind == "read_after_write":
            o = S_new @ q
        osum_new = osum + o
        m_new = np.array(m)
        end = (pos % L == 0) if kind == "chunk_end" else ((pos + 1) % L == 0)
        if end:
            m_new = osum_new / L
            osum_new = np.zeros_like(osum_new)
        return o, S_new, m_new, osum_new
    return step


@pytest.mark.parametrize("kind", ["read_after_write", "ungated_erase",
                                  "chunk_end"])
def test_planted_mistakes_break_the_pin(kind, monkeypatch):
    rng = np.random.default_rng(3)
    a = rand_pair(rng, 12, 6, 5, 3, ub_std=0.8)
    monkeypatch.setattr(decode, "decode_step", _broken(kind))
    o, S, m, _ = _decode_all(a, 4, 12, S=a["S0"].copy(), m=a["m0"].copy())
    o_ref, S_ref, m_ref = ref.fwd_pair(a["q"], a["k"], a["v"], a["g"],
                                       a["bx"], a["w"], a["u_down"],
                                       a["u_up"], 4, a["S0"], a["m0"])
    assert max(rel(o, o_ref), rel(S, S_ref), rel(m, m_ref)) > 1e-6
