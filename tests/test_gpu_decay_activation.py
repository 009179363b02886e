"""GPU parity of the fused decay activation (decay_scale > 0).

The kernels take raw decay logits a in place of the log-decay and apply
g = -s softplus(a) themselves (forward: in the key-side transform; backward:
dL/da = dL/dg * (-s sigmoid(a)) in the per-channel epilogue).  Each case
draws a with the workloads' own recipe (a ~ N(0, 1), s = 0.1: the same
random numbers the unfused inputs push through -0.1 softplus) and compares
with the fp64 oracle run on the same logits, where the activation is a
separate step (oracle/activation.py): max|delta| / max|ref| <= 1e-2 (bf16),
<= 1e-4 (fp32), for o, S_T, m_T and every gradient, dg being dL/da.
"""
import numpy as np
import pytest
import torch

from chunk_gated_delta_02_b200 import carve
from chunk_gated_delta_02_b200.inputs import (DECAY_SCALE, WORKLOADS,
                                              sample_pairs)
from oracle import activation, decode

from _parity import (TOL, assert_within, bwd_errors, fwd_errors,
                     grad_outputs, inputs, rel, run_fwd)

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "fp32": torch.float32}
S = DECAY_SCALE


def _raw(cfg, seed, dtype, ub=25.0):
    inp = inputs(cfg, seed, dtype, raw_decay=True)
    if cfg["R"] > 0:
        inp["u_down"] = (inp["u_down"].float() * ub).to(dtype)
        inp["u_up"] = (inp["u_up"].float() * ub).to(dtype)
    return inp


CASES = [
    # B, H, T, DK, DV, R, L, dtype: generic and tensor-core families
    (1, 2, 128, 64, 64, 8, 64, "bf16"),
    (1, 2, 128, 64, 64, 8, 64, "fp32"),
    (2, 1, 96, 32, 48, 4, 16, "fp32"),
    (1, 2, 192, 128, 128, 32, 64, "bf16"),   # tensor-core fwd + bwd
    (2, 1, 256, 128, 128, 16, 128, "bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_fused_activation_fwd_bwd(case):
    B, H, T, DK, DV, R, L, dt = case
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    inp = _raw(cfg, 91, DT[dt])
    tol = TOL[DT[dt]]
    assert_within(fwd_errors(inp, L, decay_scale=S), tol,
                  "fused decay fwd %s" % (case,))
    gro = grad_outputs(cfg, 92, DT[dt])
    assert_within(bwd_errors(inp, L, gro, du_heads=range(H), decay_scale=S),
                  tol, "fused decay bwd %s" % (case,))


@pytest.mark.parametrize("case", [(1, 2, 128, 256, 32, 64), (1, 2, 256, 128, 16, 32),
                                  (1, 1, 128, 256, 8, 16)],
                         ids=lambda c: "x".join(map(str, c)))
def test_fused_activation_tensor_core_forward_shapes(case):
    # dv = 256 (two CTAs per pair) and chunks shorter than 64 tokens
    B, H, T, DV, R, L = case
    cfg = dict(B=B, H=H, T=T, DK=128, DV=DV, R=R, L=L)
    assert carve.fwd_path(carve.make_shape(B, T, H, 128, DV, R, L,
                                           torch.bfloat16, S)) == "tc"
    inp = _raw(cfg, 93, torch.bfloat16)
    assert_within(fwd_errors(inp, L, decay_scale=S), 1e-2,
                  "fused decay tc fwd %s" % (case,))


def test_fused_activation_layer_1p3b_training():
    cfg = WORKLOADS["layer_1p3b"]
    inp = inputs(cfg, 94, torch.bfloat16, raw_decay=True)
    gro = grad_outputs(cfg, 94, torch.bfloat16)
    pairs = sample_pairs(cfg["B"], cfg["H"], 2, seed=94)
    assert_within(bwd_errors(inp, cfg["L"], gro, pairs=pairs, du_heads=[3],
                             decay_scale=S), 1e-2,
                  "fused decay 1.3B-layer fwd+bwd")


def test_fused_activation_matches_host_activation():
    # the same logits activated on the host in fp32 and passed as g: the
    # two GPU runs agree to the bf16 rounding of the host-side g
    cfg = dict(B=2, H=2, T=192, DK=128, DV=128, R=32, L=64)
    inp = _raw(cfg, 95, torch.bfloat16)
    _, o_f, S_f, m_f, _ = run_fwd(inp, 64, decay_scale=S)
    host = dict(inp)
    host["g"] = (-S * torch.nn.functional.softplus(inp["g"].float())).to(
        torch.bfloat16)
    _, o_h, S_h, m_h, _ = run_fwd(host, 64)
    assert rel(o_f.float().cpu(), o_h.float().cpu()) < 1e-2
    assert rel(S_f.cpu(), S_h.cpu()) < 1e-2


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_fused_activation_decode(dt):
    B, H, T, DK, DV, R, L = 2, 2, 7, 128, 128, 16, 4
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    inp = _raw(cfg, 96, DT[dt])
    tok = {n: inp[n].transpose(0, 1).contiguous() for n in
           ("q", "k", "v", "g", "bx", "w")}
    gen = torch.Generator().manual_seed(97)
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
                                      decay_scale=S).float().cpu())
        pos += 1
    torch.cuda.synchronize()
    f64 = lambda x: x.double().numpy()
    acc = {"o": ([], []), "S": ([], [])}
    for b in range(B):
        for h in range(H):
            sl = lambda n: f64(tok[n][:, b, h])
            o_r, S_r, _, _ = decode.decode_steps(
                f64(S0[b, h]), np.zeros(DV), np.zeros(DV), 0, sl("q"), sl("k"),
                sl("v"), activation.decay_from_logits(sl("g"), S), sl("bx"),
                sl("w"), f64(inp["u_down"][h]), f64(inp["u_up"][h]), L)
            acc["o"][0].append(np.stack([o[b, h].double().numpy()
                                         for o in outs]).ravel())
            acc["o"][1].append(o_r.ravel())
            acc["S"][0].append(Sd[b, h].double().cpu().numpy().ravel())
            acc["S"][1].append(S_r.ravel())
    errs = {n: rel(np.concatenate(g_), np.concatenate(r_))
            for n, (g_, r_) in acc.items()}
    assert_within(errs, TOL[DT[dt]], "fused decay decode " + dt)
