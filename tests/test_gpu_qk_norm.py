"""GPU parity of the fused q / k L2 normalisation (qk_l2norm = 1).

The kernels receive raw q and k (here the workloads' unit rows scaled by a
random factor in [0.5, 2] per token, then rounded to the input dtype) and
divide them by their per-token norms themselves; the backward returns the
gradients of the raw q and k.  Compared with the fp64 oracle, which
normalises as a separate step (oracle/normalize.py): max|delta| / max|ref|
<= 1e-2 (bf16) or 1e-4 (fp32) for every output and gradient.
"""
import numpy as np
import pytest
import torch

from chunk_gated_delta_02_b200 import carve
from oracle import decode, normalize

from _parity import (TOL, assert_within, bwd_errors, fwd_errors,
                     grad_outputs, inputs, rel, run_fwd)

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "fp32": torch.float32}


def _raw_qk(cfg, seed, dtype, ub=25.0):
    inp = inputs(cfg, seed, dtype)
    gen = torch.Generator().manual_seed(seed + 5)
    for n in ("q", "k"):
        f = 0.5 + 1.5 * torch.rand(inp[n].shape[:-1] + (1,), generator=gen)
        inp[n] = (inp[n].double() * f).to(dtype)
    if cfg["R"] > 0:
        inp["u_down"] = (inp["u_down"].float() * ub).to(dtype)
        inp["u_up"] = (inp["u_up"].float() * ub).to(dtype)
    return inp


CASES = [
    # B, H, T, DK, DV, R, L, dtype
    (1, 2, 128, 64, 64, 8, 64, "bf16"),
    (1, 2, 128, 64, 64, 8, 64, "fp32"),
    (2, 1, 96, 32, 48, 4, 16, "fp32"),
    (1, 2, 192, 128, 128, 32, 64, "bf16"),   # tensor-core forward and backward
    (2, 2, 256, 128, 128, 16, 128, "bf16"),  # the same, two blocks per chunk
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_fused_normalisation_fwd_bwd(case):
    B, H, T, DK, DV, R, L, dt = case
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    if DK == DV == 128 and dt == "bf16":
        assert carve.fwd_path(carve.make_shape(B, T, H, DK, DV, R, L, torch.bfloat16,
                                               0.0, True)) == "tc"
    inp = _raw_qk(cfg, 141, DT[dt])
    tol = TOL[DT[dt]]
    assert_within(fwd_errors(inp, L, qk_l2norm=True), tol,
                  "fused qk norm fwd %s" % (case,))
    gro = grad_outputs(cfg, 142, DT[dt])
    assert_within(bwd_errors(inp, L, gro, du_heads=range(H), qk_l2norm=True),
                  tol, "fused qk norm bwd %s" % (case,))


@pytest.mark.parametrize("case", [(1, 2, 256, 128, 32, 64), (1, 2, 128, 256, 16, 64),
                                  (1, 1, 160, 128, 8, 32), (2, 1, 100, 128, 8, 64)],
                         ids=lambda c: "x".join(map(str, c)))
def test_fused_normalisation_tensor_core_forward(case):
    B, H, T, DV, R, L = case
    cfg = dict(B=B, H=H, T=T, DK=128, DV=DV, R=R, L=L)
    assert carve.fwd_path(carve.make_shape(B, T, H, 128, DV, R, L,
                                           torch.bfloat16, 0.0, True)) == "tc"
    inp = _raw_qk(cfg, 143, torch.bfloat16)
    assert_within(fwd_errors(inp, L, qk_l2norm=True), 1e-2,
                  "fused qk norm tc fwd %s" % (case,))


def test_fused_normalisation_equals_unit_inputs():
    # raw rows with the flag against the unit rows without it (both GPU)
    cfg = dict(B=2, H=2, T=192, DK=128, DV=128, R=32, L=64)
    unit = inputs(cfg, 144, torch.bfloat16)
    raw = dict(unit)
    gen = torch.Generator().manual_seed(145)
    for n in ("q", "k"):
        f = 0.5 + 1.5 * torch.rand(unit[n].shape[:-1] + (1,), generator=gen)
        raw[n] = (unit[n].double() * f).to(torch.bfloat16)
    _, o_u, S_u, _, _ = run_fwd(unit, 64)
    _, o_r, S_r, _, _ = run_fwd(raw, 64, qk_l2norm=True)
    assert rel(o_r.float().cpu(), o_u.float().cpu()) < 1e-2
    assert rel(S_r.cpu(), S_u.cpu()) < 1e-2


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_fused_normalisation_decode(dt):
    B, H, T, DK, DV, R, L = 2, 2, 6, 128, 64, 16, 4
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    inp = _raw_qk(cfg, 146, DT[dt])
    tok = {n: inp[n].transpose(0, 1).contiguous() for n in
           ("q", "k", "v", "g", "bx", "w")}
    gen = torch.Generator().manual_seed(147)
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
                                      qk_l2norm=True).float().cpu())
        pos += 1
    torch.cuda.synchronize()
    f64 = lambda x: x.double().numpy()
    acc = {"o": ([], []), "S": ([], [])}
    for b in range(B):
        for h in range(H):
            sl = lambda n: f64(tok[n][:, b, h])
            o_r, S_r, _, _ = decode.decode_steps(
                f64(S0[b, h]), np.zeros(DV), np.zeros(DV), 0,
                normalize.l2_normalise(sl("q")), normalize.l2_normalise(sl("k")),
                sl("v"), sl("g"), sl("bx"), sl("w"), f64(inp["u_down"][h]),
                f64(inp["u_up"][h]), L)
            acc["o"][0].append(np.stack([o[b, h].double().numpy()
                                         for o in outs]).ravel())
            acc["o"][1].append(o_r.ravel())
            acc["S"][0].append(Sd[b, h].double().cpu().numpy().ravel())
            acc["S"][1].append(S_r.ravel())
    errs = {n: rel(np.concatenate(g_), np.concatenate(r_))
            for n, (g_, r_) in acc.items()}
    assert_within(errs, TOL[DT[dt]], "fused qk norm decode " + dt)


@pytest.mark.parametrize("case", [(1, 2, 192, 128, 128, 32, 64),
                                  (2, 2, 128, 64, 64, 8, 64)],
                         ids=lambda c: "x".join(map(str, c)))
def test_fused_normalisation_with_fused_activation(case):
    # both fused prologues at once: raw q, k and raw decay logits (the
    # tensor-core kernels' instances with both at dk = dv = 128, the generic
    # kernels at 64); the oracle applies the activation and the
    # normalisation as separate steps before the recurrence
    from chunk_gated_delta_02_b200.inputs import DECAY_SCALE
    B, H, T, DK, DV, R, L = case
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    if DK == DV == 128:
        assert carve.fwd_path(carve.make_shape(B, T, H, DK, DV, R, L, torch.bfloat16,
                                               DECAY_SCALE, True)) == "tc"
    inp = inputs(cfg, 151, torch.bfloat16, raw_decay=True)
    gen = torch.Generator().manual_seed(152)
    for n in ("q", "k"):
        f = 0.5 + 1.5 * torch.rand(inp[n].shape[:-1] + (1,), generator=gen)
        inp[n] = (inp[n].double() * f).to(torch.bfloat16)
    for n in ("u_down", "u_up"):
        inp[n] = (inp[n].float() * 25.0).to(torch.bfloat16)
    assert_within(fwd_errors(inp, L, decay_scale=DECAY_SCALE, qk_l2norm=True),
                  1e-2, "fused qk norm + decay fwd %s" % (case,))
    gro = grad_outputs(cfg, 153, torch.bfloat16)
    assert_within(bwd_errors(inp, L, gro, du_heads=range(H), decay_scale=DECAY_SCALE,
                             qk_l2norm=True),
                  1e-2, "fused qk norm + decay bwd %s" % (case,))


def test_fused_normalisation_layer_1p3b_training():
    # the 1.3B-layer shape (B = 8, H = 16, T = 4096) with raw q, k and the
    # fused normalisation, trained on the tensor cores: the oracle checks
    # two sampled pairs (the corners) and the dU of head 3 over the batch
    from chunk_gated_delta_02_b200.inputs import WORKLOADS, sample_pairs
    cfg = WORKLOADS["layer_1p3b"]
    inp = inputs(cfg, 161, torch.bfloat16)
    gen = torch.Generator().manual_seed(162)
    for n in ("q", "k"):
        f = 0.5 + 1.5 * torch.rand(inp[n].shape[:-1] + (1,), generator=gen)
        inp[n] = (inp[n].double() * f).to(torch.bfloat16)
    gro = grad_outputs(cfg, 163, torch.bfloat16)
    pairs = sample_pairs(cfg["B"], cfg["H"], 2, seed=161)
    assert_within(bwd_errors(inp, cfg["L"], gro, pairs=pairs, du_heads=[3],
                             qk_l2norm=True), 1e-2,
                  "fused qk norm 1.3B-layer fwd+bwd")
