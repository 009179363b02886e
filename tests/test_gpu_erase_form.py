"""GPU parity of the other key-axis erase form (erase_form = 1):
S_t = S' (I - (b (.) k) k^T) + w v k^T, run on the generic kernels (forward,
training backward) and the decode step, against the fp64 oracle's erase-1
entry points (pinned by their own WY chunk form and finite differences):
max|delta| / max|ref| <= 1e-2 (bf16) or 1e-4 (fp32).
"""
import numpy as np
import pytest
import torch

from chunk_gated_delta_02_b200 import carve
from oracle import decode

from _parity import (TOL, assert_within, bwd_errors, fwd_errors,
                     grad_outputs, inputs, rel)

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "fp32": torch.float32}

CASES = [
    # B, H, T, DK, DV, R, L, dtype
    (1, 2, 128, 64, 64, 8, 64, "bf16"),
    (1, 2, 128, 64, 64, 8, 64, "fp32"),
    (2, 1, 96, 32, 48, 4, 16, "fp32"),
    (1, 2, 192, 128, 128, 32, 64, "bf16"),
    (1, 1, 256, 64, 64, 8, 128, "fp32"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_other_erase_form_fwd_bwd(case):
    B, H, T, DK, DV, R, L, dt = case
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    assert carve.fwd_path(carve.make_shape(B, T, H, DK, DV, R, L, DT[dt],
                                           erase_form=1)) == "generic"
    inp = inputs(cfg, 151, DT[dt])
    if R > 0:
        inp["u_down"] = (inp["u_down"].float() * 25).to(DT[dt])
        inp["u_up"] = (inp["u_up"].float() * 25).to(DT[dt])
    gen = torch.Generator().manual_seed(152)
    inp["S0"] = torch.randn((B, H, DV, DK), generator=gen) * 0.3
    inp["m0"] = torch.randn((B, H, DV), generator=gen) * 0.3
    tol = TOL[DT[dt]]
    assert_within(fwd_errors(inp, L, erase_form=1), tol,
                  "erase form 1 fwd %s" % (case,))
    gro = grad_outputs(cfg, 153, DT[dt])
    assert_within(bwd_errors(inp, L, gro, du_heads=range(H), erase_form=1),
                  tol, "erase form 1 bwd %s" % (case,))


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_other_erase_form_decode(dt):
    B, H, T, DK, DV, R, L = 2, 2, 7, 128, 64, 16, 4
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    inp = inputs(cfg, 154, DT[dt])
    inp["u_down"] = (inp["u_down"].float() * 25).to(DT[dt])
    inp["u_up"] = (inp["u_up"].float() * 25).to(DT[dt])
    tok = {n: inp[n].transpose(0, 1).contiguous() for n in
           ("q", "k", "v", "g", "bx", "w")}
    gen = torch.Generator().manual_seed(155)
    S0 = torch.randn((B, H, DV, DK), generator=gen) * 0.3
    Sd = S0.cuda()
    m = torch.zeros((B, H, DV), device="cuda")
    osum = torch.zeros((B, H, DV), device="cuda")
    pos = torch.zeros((B,), dtype=torch.int32, device="cuda")
    ud, uu = inp["u_down"].cuda(), inp["u_up"].cuda()
    outs = []
    for t in range(T):
        outs.append(carve.decode_step(*(tok[n][t].cuda() for n in
                                        ("q", "k", "v", "g", "bx", "w")),
                                      ud, uu, L, pos, Sd, m, osum,
                                      erase_form=1).float().cpu())
        pos += 1
    torch.cuda.synchronize()
    f64 = lambda x: x.double().numpy()
    acc = {"o": ([], []), "S": ([], [])}
    for b in range(B):
        for h in range(H):
            sl = lambda n: f64(tok[n][:, b, h])
            o_r, S_r, _, _ = decode.decode_steps(
                f64(S0[b, h]), np.zeros(DV), np.zeros(DV), 0, sl("q"),
                sl("k"), sl("v"), sl("g"), sl("bx"), sl("w"),
                f64(inp["u_down"][h]), f64(inp["u_up"][h]), L, erase=1)
            acc["o"][0].append(np.stack([o[b, h].double().numpy()
                                         for o in outs]).ravel())
            acc["o"][1].append(o_r.ravel())
            acc["S"][0].append(Sd[b, h].double().cpu().numpy().ravel())
            acc["S"][1].append(S_r.ravel())
    errs = {n: rel(np.concatenate(g_), np.concatenate(r_))
            for n, (g_, r_) in acc.items()}
    assert_within(errs, TOL[DT[dt]], "erase form 1 decode " + dt)
