"""GPU parity of the recurrent decode step (carve_decode_step) against the
decode oracle (oracle/decode.py, pinned to the token-recurrence oracle).

Each case runs T consecutive decode steps on the GPU from a random state
(S, m, osum) and compares every output o_t and the final S, m, osum of
every (sequence, head) pair element by element with T oracle steps on the
same rounded inputs: max|delta| / max|ref| <= 1e-2 for bf16 inputs (fp32
state), <= 1e-4 for fp32 inputs.  Sequences of a batch sit at different
positions, so their chunks end at different steps.  A last check runs a
whole sequence through the chunk forward and through the decode step and
compares the two GPU paths.
"""
import numpy as np
import pytest
import torch

from chunk_gated_delta_02_b200 import carve
from chunk_gated_delta_02_b200.inputs import make_inputs
from oracle import decode

from _parity import TOL, assert_within, rel

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "fp32": torch.float32}


def _tokens(B, H, T, DK, DV, R, seed, dtype, ub_scale=25.0):
    """T tokens per sequence with the workloads' distributions, token-major
    ([T, B, H, D]), and the U_b factors (scaled up so the gate moves)."""
    inp = make_inputs(B=B, T=T, H=H, DK=DK, DV=DV, R=R, seed=seed, dtype=dtype)
    tok = {n: inp[n].transpose(0, 1).contiguous() for n in
           ("q", "k", "v", "g", "bx", "w")}
    ud = (inp["u_down"].float() * ub_scale).to(dtype)
    uu = (inp["u_up"].float() * ub_scale).to(dtype)
    return tok, ud, uu


def _run(case, dtype, seed=71):
    B, H, T, DK, DV, R, L, pos0 = case
    tok, ud, uu = _tokens(B, H, T, DK, DV, R, seed, dtype)
    gen = torch.Generator().manual_seed(seed + 1)
    S0 = torch.randn((B, H, DV, DK), generator=gen) * 0.3
    m0 = torch.randn((B, H, DV), generator=gen) * 0.3
    os0 = torch.randn((B, H, DV), generator=gen) * 0.3
    pos = torch.tensor(pos0, dtype=torch.int32)
    # GPU: T steps, the caller advancing pos
    dev = "cuda"
    S, m, osum = S0.to(dev), m0.to(dev), os0.to(dev)
    posd = pos.to(dev)
    udd, uud = ud.to(dev), uu.to(dev)
    outs = []
    for t in range(T):
        o = carve.decode_step(*(tok[n][t].to(dev) for n in
                                ("q", "k", "v", "g", "bx", "w")),
                              udd, uud, L, posd, S, m, osum)
        outs.append(o.float().cpu())
        posd += 1
    torch.cuda.synchronize()
    o_gpu = torch.stack(outs)  # [T, B, H, DV]
    # oracle, pair by pair
    errs = {}
    acc = {n: ([], []) for n in ("o", "S", "m", "osum")}
    f64 = lambda x: x.double().numpy()
    for b in range(B):
        for h in range(H):
            sl = lambda n: f64(tok[n][:, b, h])
            o_r, S_r, m_r, s_r = decode.decode_steps(
                f64(S0[b, h]), f64(m0[b, h]), f64(os0[b, h]), int(pos[b]),
                sl("q"), sl("k"), sl("v"), sl("g"), sl("bx"), sl("w"),
                f64(ud[h]), f64(uu[h]), L)
            for n, g_, r_ in (("o", o_gpu[:, b, h], o_r), ("S", S[b, h], S_r),
                              ("m", m[b, h], m_r), ("osum", osum[b, h], s_r)):
                acc[n][0].append(np.asarray(g_.double().cpu()).ravel())
                acc[n][1].append(np.asarray(r_).ravel())
    for n, (g_, r_) in acc.items():
        errs[n] = rel(np.concatenate(g_), np.concatenate(r_))
    return errs


CASES = [
    # B, H, T, DK, DV, R, L, pos0 per sequence
    (2, 3, 11, 64, 64, 8, 4, [0, 2]),
    (3, 2, 9, 128, 128, 32, 4, [0, 1, 3]),
    (1, 2, 7, 128, 256, 32, 3, [5]),
    (2, 1, 6, 32, 48, 0, 2, [0, 1]),        # R = 0: no content signal
    (1, 1, 5, 256, 64, 16, 64, [62]),       # chunk end mid-run
    (2, 2, 8, 16, 16, 4, 1, [0, 0]),        # L = 1: every token ends a chunk
]


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:7])))
def test_decode_steps_match_oracle(case, dt):
    errs = _run(case, DT[dt])
    assert_within(errs, TOL[DT[dt]], "decode %s %s" % (case[:7], dt))


def test_decode_layer_1p3b_shape():
    # the 1.3B-layer shape (B = 8, H = 16, dk = dv = 128, r = 32, L = 64),
    # 66 steps from position 0 so that the first chunk ends inside the run
    errs = _run((8, 16, 66, 128, 128, 32, 64, [0] * 8), torch.bfloat16)
    assert_within(errs, 1e-2, "decode 1.3B-layer shape, 66 steps")


def test_decode_continues_the_chunk_forward():
    # 256 tokens through carve_chunk_fwd equal their first 192 through
    # carve_chunk_fwd followed by the last 64 through the decode step,
    # started from that forward's (S_T, m_T) with osum = 0 and pos = 192
    B, H, DK, DV, R, L = 2, 2, 128, 128, 32, 64
    T0 = 192
    inp = make_inputs(B=B, T=T0 + L, H=H, DK=DK, DV=DV, R=R, seed=81,
                      dtype=torch.bfloat16)
    inp["u_down"] = (inp["u_down"].float() * 25).to(torch.bfloat16)
    inp["u_up"] = (inp["u_up"].float() * 25).to(torch.bfloat16)
    d = {n: (x.cuda() if x is not None else None) for n, x in inp.items()}
    o_all, S_all, m_all, _ = carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"],
                                             d["bx"], d["w"], d["u_down"],
                                             d["u_up"], L)
    head = {n: (d[n][:, :T0].contiguous() if n in ("q", "k", "v", "g", "bx",
                                                     "w") else d[n])
            for n in d}
    _, S, m, _ = carve.chunk_fwd(head["q"], head["k"], head["v"], head["g"],
                                 head["bx"], head["w"], d["u_down"], d["u_up"],
                                 L)
    osum = torch.zeros_like(m)
    pos = torch.full((B,), T0, dtype=torch.int32, device="cuda")
    outs = []
    for t in range(T0, T0 + L):
        outs.append(carve.decode_step(
            *(d[n][:, t].contiguous() for n in ("q", "k", "v", "g", "bx", "w")),
            d["u_down"], d["u_up"], L, pos, S, m, osum))
        pos += 1
    torch.cuda.synchronize()
    o_dec = torch.stack(outs, 1)
    assert rel(o_dec.float().cpu(), o_all[:, T0:].float().cpu()) < 1e-2
    assert rel(S.cpu(), S_all.cpu()) < 1e-2
    assert rel(m.cpu(), m_all.cpu()) < 1e-2
    assert float(osum.abs().max()) == 0.0


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_decode_copy_wait_gives_up(dt, monkeypatch):
    # Test-only knobs: CTA 0 (pair (0, 0), value rows 0 .. dv/4 - 1)
    # announces its first group of copies but issues none, so its bounded
    # wait (lowered to 2e5 cycles) gives up.  That CTA writes NaN to its
    # rows of o and leaves its rows of S, m and the output sums as they
    # were; every other output equals a normal step's bit for bit, and a
    # normal step afterwards does too.  Sequence 0 is at a chunk's last
    # token, so the CTA that gave up still meets its cluster's barrier.
    B, H, DK, DV, R, L = 2, 2, 128, 128, 16, 4
    dtype = DT[dt]
    tok, ud, uu = _tokens(B, H, 1, DK, DV, R, 91, dtype)
    gen = torch.Generator().manual_seed(92)
    S0 = (torch.randn((B, H, DV, DK), generator=gen) * 0.3).cuda()
    m0 = (torch.randn((B, H, DV), generator=gen) * 0.3).cuda()
    os0 = (torch.randn((B, H, DV), generator=gen) * 0.3).cuda()
    pos = torch.tensor([L - 1, 1], dtype=torch.int32, device="cuda")
    x = [tok[n][0].cuda() for n in ("q", "k", "v", "g", "bx", "w")]
    udd, uud = ud.cuda(), uu.cuda()

    def step():
        S, m, osum = S0.clone(), m0.clone(), os0.clone()
        o = carve.decode_step(*x, udd, uud, L, pos, S, m, osum)
        torch.cuda.synchronize()
        return o.float(), S, m, osum

    o_r, S_r, m_r, s_r = step()
    monkeypatch.setenv("CARVE_TEST_WAIT_CYCLES", "200000")
    monkeypatch.setenv("CARVE_TEST_STALL_BLOCK", "0")
    o_s, S_s, m_s, s_s = step()
    monkeypatch.delenv("CARVE_TEST_WAIT_CYCLES")
    monkeypatch.delenv("CARVE_TEST_STALL_BLOCK")
    rq = DV // 4
    assert bool(torch.isnan(o_s[0, 0, :rq]).all())
    keep = torch.ones_like(o_r, dtype=torch.bool)
    keep[0, 0, :rq] = False
    assert torch.equal(o_s[keep], o_r[keep])
    assert not bool(torch.isnan(o_r).any())
    for got, ref, before in ((S_s, S_r, S0), (m_s, m_r, m0), (s_s, s_r, os0)):
        assert torch.equal(got[0, 0, :rq], before[0, 0, :rq])
        assert not torch.equal(ref[0, 0, :rq], before[0, 0, :rq])
        k2 = torch.ones(got.shape[:3], dtype=torch.bool, device=got.device)
        k2[0, 0, :rq] = False
        assert torch.equal(got[k2], ref[k2])
    o_n, S_n, m_n, s_n = step()
    assert torch.equal(o_n, o_r) and torch.equal(S_n, S_r)
    assert torch.equal(m_n, m_r) and torch.equal(s_n, s_r)
