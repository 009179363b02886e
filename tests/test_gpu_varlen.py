"""GPU parity of the forward on ragged lengths: sequences whose length is not
a multiple of the chunk length L, and packed batches of sequences of
different lengths (carve_chunk_fwd_varlen with cu_seqlens).

Each sequence is compared with the fp64 oracle run on that sequence's own
tokens (chunks from its own start, a short last chunk whose mean still
divides by L): every output, S_T and m_T, max|delta| / max|ref| <= 1e-2
(bf16) or 1e-4 (fp32).  Tokens outside every sequence keep what the output
buffer held, and malformed offsets are reported in the status word.
"""
import numpy as np
import pytest
import torch

from chunk_gated_delta_02_b200 import carve
from chunk_gated_delta_02_b200.inputs import make_inputs
from oracle import ref

from _parity import TOL, Gathered, assert_within, fwd_errors, inputs

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "fp32": torch.float32}


@pytest.mark.parametrize("case", [
    # B, H, T, DK, DV, R, L, dtype
    (2, 2, 200, 128, 128, 32, 64, "bf16"),   # tensor cores: 3 blocks + 8 tokens
    (1, 2, 100, 128, 128, 16, 32, "bf16"),   # short chunks, partial last one
    (1, 1, 130, 128, 256, 8, 64, "bf16"),    # dv = 256 clusters
    (2, 1, 90, 64, 64, 8, 64, "bf16"),       # generic kernels
    (2, 1, 90, 64, 64, 8, 16, "fp32"),
    (1, 2, 5, 128, 128, 32, 64, "bf16"),     # shorter than one block
], ids=lambda c: "x".join(map(str, c)))
def test_sequence_length_not_a_multiple_of_L(case):
    B, H, T, DK, DV, R, L, dt = case
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    inp = inputs(cfg, 101, DT[dt])
    if R > 0:
        inp["u_down"] = (inp["u_down"].float() * 25).to(DT[dt])
        inp["u_up"] = (inp["u_up"].float() * 25).to(DT[dt])
    gen = torch.Generator().manual_seed(102)
    inp["S0"] = torch.randn((B, H, DV, DK), generator=gen) * 0.3
    inp["m0"] = torch.randn((B, H, DV), generator=gen) * 0.3
    assert_within(fwd_errors(inp, L), TOL[DT[dt]], "T %% L != 0 %s" % (case,))


def _packed(lengths, H, DK, DV, R, seed, dtype, gap=0):
    """Packed [T, H, D] tokens of sequences of the given lengths (with `gap`
    unowned tokens before the first and after the last), per-sequence S0,
    m0, and the offsets."""
    T = sum(lengths) + 2 * gap
    inp = make_inputs(B=1, T=T, H=H, DK=DK, DV=DV, R=R, seed=seed, dtype=dtype)
    tok = {n: inp[n][0].contiguous() for n in ("q", "k", "v", "g", "bx", "w")}
    tok["u_down"] = (inp["u_down"].float() * 25).to(dtype)
    tok["u_up"] = (inp["u_up"].float() * 25).to(dtype)
    N = len(lengths)
    gen = torch.Generator().manual_seed(seed + 1)
    tok["S0"] = torch.randn((N, H, DV, DK), generator=gen) * 0.3
    tok["m0"] = torch.randn((N, H, DV), generator=gen) * 0.3
    cu = np.concatenate([[0], np.cumsum(lengths)]) + gap
    return tok, torch.tensor(cu, dtype=torch.int32), T


def _oracle_seq(tok, cu, n, h, L):
    s, e = int(cu[n]), int(cu[n + 1])
    f = lambda x: x.double().numpy()
    return ref.fwd_pair(f(tok["q"][s:e, h]), f(tok["k"][s:e, h]),
                        f(tok["v"][s:e, h]), f(tok["g"][s:e, h]),
                        f(tok["bx"][s:e, h]), f(tok["w"][s:e, h]),
                        f(tok["u_down"][h]), f(tok["u_up"][h]), L,
                        f(tok["S0"][n, h]), f(tok["m0"][n, h]))


VARLEN = [
    # lengths, H, DK, DV, R, L, dtype
    ([0, 1, 63, 64, 65, 130, 200], 2, 128, 128, 32, 64, "bf16"),
    ([17, 0, 96, 33], 2, 128, 128, 16, 32, "bf16"),
    ([70, 5, 128], 1, 128, 256, 32, 64, "bf16"),
    ([0, 1, 63, 64, 65, 130], 2, 64, 64, 8, 64, "bf16"),
    ([20, 47, 3], 1, 64, 32, 4, 16, "fp32"),
    ([300, 129], 2, 128, 128, 32, 128, "bf16"),
]


@pytest.mark.parametrize("case", VARLEN, ids=lambda c: "%s-%d" % (
    "x".join(map(str, c[0])), c[5]))
def test_packed_sequences_match_oracle(case):
    lengths, H, DK, DV, R, L, dt = case
    dtype = DT[dt]
    tok, cu, T = _packed(lengths, H, DK, DV, R, 111, dtype, gap=3)
    d = {n: x.cuda() for n, x in tok.items()}
    sentinel = torch.full((T, H, DV), 7.0, dtype=dtype, device="cuda")
    o, S_T, m_T, ws = carve.chunk_fwd_varlen(
        d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"], d["u_down"],
        d["u_up"], L, cu.cuda(), d["S0"], d["m0"], o=sentinel)
    assert carve.get_status(ws) == 0
    o, S_T, m_T = o.cpu(), S_T.cpu(), m_T.cpu()
    acc = Gathered()
    for n in range(len(lengths)):
        s, e = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            oo, SS, mm = _oracle_seq(tok, cu, n, h, L)
            acc.add("o", o[s:e, h].double().numpy(), oo)
            acc.add("S_T", S_T[n, h].double().numpy(), SS)
            acc.add("m_T", m_T[n, h].double().numpy(), mm)
    assert_within(acc.errors(), TOL[dtype], "varlen %s L=%d" % (lengths, L))
    # the 3 tokens before the first and after the last sequence are untouched
    assert bool((o[:3] == 7.0).all()) and bool((o[-3:] == 7.0).all())
    # an empty sequence returns its initial state
    for n, ln in enumerate(lengths):
        if ln == 0:
            assert torch.equal(S_T[n], tok["S0"][n])
            assert torch.equal(m_T[n], tok["m0"][n])


def test_malformed_offsets_are_reported():
    tok, cu, T = _packed([10, 20], 1, 128, 128, 8, 121, torch.bfloat16)
    d = {n: x.cuda() for n, x in tok.items()}
    bad = torch.tensor([0, 25, 12], dtype=torch.int32, device="cuda")  # decreasing
    _, _, _, ws = carve.chunk_fwd_varlen(
        d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"], d["u_down"],
        d["u_up"], 64, bad)
    assert carve.STATUS[carve.get_status(ws)] == "CARVE_ERR_INVALID_ARG"
    torch.cuda.synchronize()
    assert int(ws[8:12].view(torch.int32).item()) == 90


def test_uniform_offsets_equal_the_batched_forward():
    # B sequences of T tokens through the packed entry point (offsets
    # 0, T, 2T, ...) equal the batched forward on the same memory
    B, H, T, L = 3, 2, 192, 64
    cfg = dict(B=B, H=H, T=T, DK=128, DV=128, R=32, L=L)
    inp = inputs(cfg, 131, torch.bfloat16)
    d = {n: (x.cuda() if x is not None else None) for n, x in inp.items()}
    o1, S1, m1, _ = carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["bx"],
                                    d["w"], d["u_down"], d["u_up"], L)
    flat = {n: d[n].reshape((B * T,) + d[n].shape[2:]) for n in
            ("q", "k", "v", "g", "bx", "w")}
    cu = torch.arange(0, B * T + 1, T, dtype=torch.int32, device="cuda")
    o2, S2, m2, _ = carve.chunk_fwd_varlen(flat["q"], flat["k"], flat["v"],
                                           flat["g"], flat["bx"], flat["w"],
                                           d["u_down"], d["u_up"], L, cu)
    torch.cuda.synchronize()
    assert torch.equal(o1.reshape(B * T, H, -1), o2)
    assert torch.equal(S1, S2) and torch.equal(m1, m2)
