"""GPU parity: libcarve (through its C ABI) against the fp64 oracle.

Small cases compare every output element of every (sequence, head) pair;
the full-size workloads compare every element of a sampled set of pairs
(each pair is an independent recurrence, so a pair is an output the oracle
can compute on its own).  Tolerance: max|delta| / max|ref| <= 1e-2 with
bf16 inputs and fp32 state, <= 1e-4 with fp32 inputs.
"""
import numpy as np
import pytest
import torch

from chunk_gated_delta_02_b200 import carve
from chunk_gated_delta_02_b200.inputs import WORKLOADS, sample_pairs
from oracle import ref

from _parity import (TOL, assert_within, bwd_errors, fwd_errors,
                     grad_outputs, inputs, run_fwd, to_dev)

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "fp32": torch.float32}


# ------------------------------------------------------------ tiny ----------

@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_tiny_fwd(dt):
    cfg = WORKLOADS["tiny"]
    errs = fwd_errors(inputs(cfg, 0, DT[dt]), cfg["L"])
    assert_within(errs, TOL[DT[dt]], "tiny fwd " + dt)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_tiny_fwd_bwd(dt):
    cfg = WORKLOADS["tiny"]
    inp = inputs(cfg, 0, DT[dt])
    gro = grad_outputs(cfg, 0, DT[dt])
    errs = bwd_errors(inp, cfg["L"], gro, du_heads=range(cfg["H"]))
    assert_within(errs, TOL[DT[dt]], "tiny bwd " + dt)


# ------------------------------------------- shapes, tails, edge cases ------

SHAPES = [
    # B, H, T, DK, DV, R, L
    (2, 3, 64, 64, 64, 8, 64),       # one chunk: no content signal
    (2, 3, 192, 64, 64, 8, 64),      # three chunks
    (1, 2, 96, 32, 64, 4, 8),        # many short chunks, DK != DV
    (1, 2, 128, 128, 64, 16, 16),
    (1, 1, 160, 64, 32, 0, 32),      # R = 0 (no content projection)
    (1, 2, 256, 64, 64, 8, 128),     # chunk solved as two blocks
    (2, 1, 64, 16, 16, 1, 1),        # L = 1
    (1, 1, 256, 64, 256, 8, 64),     # widest value dimension
    (1, 2, 192, 128, 128, 32, 64),   # tensor-core forward (bf16)
    (2, 1, 256, 128, 128, 8, 128),   # tensor-core forward, two blocks/chunk
]


def _rand_state(inp, seed, scale=0.3):
    B, _, H, DK = inp["q"].shape
    DV = inp["v"].shape[-1]
    gen = torch.Generator().manual_seed(seed)
    inp["S0"] = torch.randn((B, H, DV, DK), generator=gen) * scale
    inp["m0"] = torch.randn((B, H, DV), generator=gen) * scale
    return inp


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_shapes_fwd_bwd(shape, dt):
    B, H, T, DK, DV, R, L = shape
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    # a larger U_b than the workloads' so the content gate moves b visibly
    inp = inputs(cfg, 11, DT[dt])
    if R > 0:
        inp["u_down"] = (inp["u_down"].float() * 25).to(DT[dt])
        inp["u_up"] = (inp["u_up"].float() * 25).to(DT[dt])
    _rand_state(inp, 12)
    tag = "x".join(map(str, shape)) + " " + dt
    assert_within(fwd_errors(inp, L), TOL[DT[dt]], "fwd " + tag)
    gro = grad_outputs(cfg, 13, DT[dt])
    gen = torch.Generator().manual_seed(14)
    gro["dS_T"] = torch.randn((B, H, DV, DK), generator=gen)
    gro["dm_T"] = torch.randn((B, H, DV), generator=gen)
    assert_within(bwd_errors(inp, L, gro, du_heads=range(H)), TOL[DT[dt]],
                  "bwd " + tag)


def test_empty_sequence_returns_initial_state():
    cfg = dict(B=2, H=2, T=0, DK=64, DV=64, R=4, L=64)
    inp = _rand_state(inputs(cfg, 1, torch.bfloat16), 2)
    _, o, S_T, m_T, _ = run_fwd(inp, 64)
    assert o.numel() == 0
    assert torch.equal(S_T.cpu(), inp["S0"])
    assert torch.equal(m_T.cpu(), inp["m0"])


def test_resume_across_calls_matches_single_call():
    cfg = dict(B=1, H=2, T=256, DK=64, DV=64, R=8, L=64)
    inp = inputs(cfg, 3, torch.float32)
    _, o, S_T, m_T, _ = run_fwd(inp, 64)
    cut = 128
    head = {k: (x[:, :cut] if k in ("q", "k", "v", "g", "bx", "w") else x)
            for k, x in inp.items()}
    tail = {k: (x[:, cut:] if k in ("q", "k", "v", "g", "bx", "w") else x)
            for k, x in inp.items()}
    _, o1, S1, m1, _ = run_fwd(head, 64)
    tail["S0"], tail["m0"] = S1.cpu(), m1.cpu()
    _, o2, S2, m2, _ = run_fwd(tail, 64)
    assert torch.allclose(torch.cat([o1, o2], 1), o, rtol=0, atol=1e-6)
    assert torch.allclose(S2, S_T, rtol=0, atol=1e-6)
    assert torch.allclose(m2, m_T, rtol=0, atol=1e-6)


def test_scalar_gates_zero_Ub_matches_oracle():
    """The reduction case: scalar-broadcast decay and erase logit, U_b = 0."""
    cfg = dict(B=2, H=2, T=256, DK=64, DV=64, R=8, L=64)
    inp = inputs(cfg, 5, torch.bfloat16, ub_zero=True)
    for n in ("g", "bx"):
        inp[n] = inp[n][..., :1].expand_as(inp[n]).contiguous()
    assert_within(fwd_errors(inp, 64), 1e-2, "scalar gates")


def test_autograd_wrapper_matches_direct_backward():
    cfg = dict(B=1, H=2, T=128, DK=64, DV=64, R=8, L=64)
    inp = _rand_state(inputs(cfg, 6, torch.float32), 7)
    d = to_dev(inp)
    leaves = {k: v.clone().requires_grad_(True) for k, v in d.items()}
    o, S_T, m_T = carve.carve(leaves["q"], leaves["k"], leaves["v"],
                              leaves["g"], leaves["bx"], leaves["w"],
                              leaves["u_down"], leaves["u_up"], 64,
                              leaves["S0"], leaves["m0"])
    gen = torch.Generator().manual_seed(8)
    do = torch.randn(o.shape, generator=gen).cuda()
    (o * do).sum().backward()
    res = ref.bwd_batch(inp, 64, do.cpu())
    for (b, h), r in res.items():
        for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"),
                          ("bx", "dbx")):
            got = leaves[name].grad[b, :, h].double().cpu().numpy()
            err = np.abs(got - r[key]).max() / np.abs(r[key]).max()
            assert err < 1e-4, (name, err)


# ------------------------------------------------------- workloads ----------

def test_layer_1p3b_fwd():
    cfg = WORKLOADS["layer_1p3b"]
    pairs = sample_pairs(cfg["B"], cfg["H"], 4)
    errs = fwd_errors(inputs(cfg, 1, torch.bfloat16), cfg["L"], pairs)
    assert_within(errs, 1e-2, "1.3B layer fwd")


def test_layer_1p3b_fwd_zero_Ub():
    cfg = WORKLOADS["layer_1p3b"]
    pairs = sample_pairs(cfg["B"], cfg["H"], 3, seed=1)
    errs = fwd_errors(inputs(cfg, 1, torch.bfloat16, ub_zero=True), cfg["L"],
                      pairs)
    assert_within(errs, 1e-2, "1.3B layer fwd, U_b = 0")


@pytest.mark.parametrize("L", [16, 32, 64, 128])
def test_chunk_sweep_fwd(L):
    cfg = dict(WORKLOADS["layer_1p3b"], L=L)
    shape = carve.make_shape(cfg["B"], cfg["T"], cfg["H"], cfg["DK"],
                             cfg["DV"], cfg["R"], L, torch.bfloat16)
    assert carve.fwd_path(shape) == "tc"  # every L of the sweep
    pairs = sample_pairs(cfg["B"], cfg["H"], 2, seed=L)
    errs = fwd_errors(inputs(cfg, 2, torch.bfloat16), L, pairs)
    assert_within(errs, 1e-2, "chunk sweep L=%d" % L)


def test_long_context_fwd():
    cfg = WORKLOADS["long_context"]
    pairs = [(0, 0), (0, cfg["H"] - 1)]
    errs = fwd_errors(inputs(cfg, 3, torch.bfloat16), cfg["L"], pairs)
    assert_within(errs, 1e-2, "long context fwd")


def test_training_fwd_bwd():
    cfg = WORKLOADS["layer_1p3b"]
    inp = inputs(cfg, 4, torch.bfloat16)
    gro = grad_outputs(cfg, 4, torch.bfloat16)
    pairs = sample_pairs(cfg["B"], cfg["H"], 3, seed=4)
    errs = bwd_errors(inp, cfg["L"], gro, pairs=pairs, du_heads=[5])
    assert_within(errs, 1e-2, "training fwd+bwd")


# ------------------------------------------ tensor-core vs generic path -----

TC_CASES = [
    # B, H, T, R, L
    (1, 1, 64, 32, 64),
    (2, 3, 320, 32, 64),
    (1, 2, 384, 8, 128),
    (1, 1, 128, 0, 64),
]


@pytest.mark.parametrize("case", TC_CASES, ids=lambda c: "x".join(map(str, c)))
def test_tensor_core_forward_matches_oracle_and_generic(case, monkeypatch):
    B, H, T, R, L = case
    cfg = dict(B=B, H=H, T=T, DK=128, DV=128, R=R, L=L)
    inp = inputs(cfg, 21, torch.bfloat16)
    if R > 0:
        inp["u_down"] = (inp["u_down"].float() * 25).to(torch.bfloat16)
        inp["u_up"] = (inp["u_up"].float() * 25).to(torch.bfloat16)
    _rand_state(inp, 22)
    shape = carve.make_shape(B, T, H, 128, 128, R, L, torch.bfloat16)
    assert carve.fwd_path(shape) == "tc"
    assert_within(fwd_errors(inp, L), 1e-2, "tensor-core fwd %s" % (case,))
    _, o_tc, S_tc, m_tc, _ = run_fwd(inp, L, training=True)
    monkeypatch.setenv("CARVE_FWD_PATH", "generic")
    assert carve.fwd_path(shape) == "generic"
    _, o_g, S_g, m_g, _ = run_fwd(inp, L, training=True)
    from _parity import rel as _rel
    assert _rel(o_tc.float().cpu(), o_g.float().cpu()) < 1e-2
    assert _rel(S_tc.cpu(), S_g.cpu()) < 1e-2
    assert _rel(m_tc.cpu(), m_g.cpu()) < 1e-2


SHORT_CHUNK_CASES = [
    # B, H, T, DV, R, L  (chunks shorter than the 64-row tiles: the chunk is
    # the block, rows past it stay zero)
    (1, 2, 256, 128, 32, 16),
    (2, 1, 320, 128, 8, 32),
    (1, 1, 192, 128, 16, 48),
    (1, 1, 64, 128, 0, 32),
    (1, 2, 128, 256, 32, 16),
    (1, 1, 160, 256, 16, 32),
]


@pytest.mark.parametrize("case", SHORT_CHUNK_CASES,
                         ids=lambda c: "x".join(map(str, c)))
def test_tensor_core_forward_short_chunks(case, monkeypatch):
    B, H, T, DV, R, L = case
    cfg = dict(B=B, H=H, T=T, DK=128, DV=DV, R=R, L=L)
    inp = inputs(cfg, 61, torch.bfloat16)
    if R > 0:  # a gate that really moves between chunks
        inp["u_down"] = (inp["u_down"].float() * 25).to(torch.bfloat16)
        inp["u_up"] = (inp["u_up"].float() * 25).to(torch.bfloat16)
    _rand_state(inp, 62)
    shape = carve.make_shape(B, T, H, 128, DV, R, L, torch.bfloat16)
    assert carve.fwd_path(shape) == "tc"
    assert_within(fwd_errors(inp, L), 1e-2, "tc fwd short chunks %s" % (case,))
    _, o_tc, S_tc, m_tc, _ = run_fwd(inp, L)
    monkeypatch.setenv("CARVE_FWD_PATH", "generic")
    _, o_g, S_g, m_g, _ = run_fwd(inp, L)
    from _parity import rel as _rel
    assert _rel(o_tc.float().cpu(), o_g.float().cpu()) < 1e-2
    assert _rel(S_tc.cpu(), S_g.cpu()) < 1e-2
    assert _rel(m_tc.cpu(), m_g.cpu()) < 1e-2


TC_DV256_CASES = [
    # B, H, T, R, L  (dv = 256: a cluster of two CTAs per (b, h))
    (1, 1, 64, 32, 64),
    (1, 2, 320, 32, 64),
    (2, 1, 256, 16, 128),
]


@pytest.mark.parametrize("case", TC_DV256_CASES, ids=lambda c: "x".join(map(str, c)))
def test_tensor_core_forward_dv256_matches_oracle_and_generic(case, monkeypatch):
    B, H, T, R, L = case
    cfg = dict(B=B, H=H, T=T, DK=128, DV=256, R=R, L=L)
    inp = inputs(cfg, 41, torch.bfloat16)
    if R > 0:  # a gate the value halves really have to share
        inp["u_down"] = (inp["u_down"].float() * 25).to(torch.bfloat16)
        inp["u_up"] = (inp["u_up"].float() * 25).to(torch.bfloat16)
    _rand_state(inp, 42)
    shape = carve.make_shape(B, T, H, 128, 256, R, L, torch.bfloat16)
    assert carve.fwd_path(shape) == "tc"
    assert_within(fwd_errors(inp, L), 1e-2, "tc fwd dv=256 %s" % (case,))
    _, o_tc, S_tc, m_tc, _ = run_fwd(inp, L)
    monkeypatch.setenv("CARVE_FWD_PATH", "generic")
    _, o_g, S_g, m_g, _ = run_fwd(inp, L)
    from _parity import rel as _rel
    assert _rel(o_tc.float().cpu(), o_g.float().cpu()) < 1e-2
    assert _rel(S_tc.cpu(), S_g.cpu()) < 1e-2
    assert _rel(m_tc.cpu(), m_g.cpu()) < 1e-2


BWD_CASES = [
    # B, H, T, R, L
    (1, 1, 128, 32, 64),
    (2, 2, 256, 16, 128),
    (1, 1, 192, 0, 64),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "x".join(map(str, c)))
def test_tensor_core_backward_matches_oracle_and_generic(case, monkeypatch):
    B, H, T, R, L = case
    cfg = dict(B=B, H=H, T=T, DK=128, DV=128, R=R, L=L)
    inp = inputs(cfg, 31, torch.bfloat16)
    if R > 0:
        inp["u_down"] = (inp["u_down"].float() * 25).to(torch.bfloat16)
        inp["u_up"] = (inp["u_up"].float() * 25).to(torch.bfloat16)
    _rand_state(inp, 32)
    gro = grad_outputs(cfg, 33, torch.bfloat16)
    gen = torch.Generator().manual_seed(34)
    gro["dS_T"] = torch.randn((B, H, 128, 128), generator=gen)
    gro["dm_T"] = torch.randn((B, H, 128), generator=gen)
    assert_within(bwd_errors(inp, L, gro, du_heads=range(H)), 1e-2,
                  "tensor-core bwd %s" % (case,))
    d, _, _, _, ws = run_fwd(inp, L, training=True)
    dd = to_dev(gro)
    g_tc = carve.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                           d["u_down"], d["u_up"], L, dd["d_o"], ws,
                           dd["dS_T"], dd["dm_T"])
    # the generic backward needs the generic forward's fp32 checkpoints,
    # which a tensor-core workspace does not hold: refused on the host
    assert carve.get_status(ws) == 0
    monkeypatch.setenv("CARVE_BWD_PATH", "generic")
    with pytest.raises(carve.CarveError) as exc:
        carve.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                        d["u_down"], d["u_up"], L, dd["d_o"], ws,
                        dd["dS_T"], dd["dm_T"])
    assert carve.STATUS[exc.value.code] == "CARVE_ERR_WORKSPACE"
    assert carve.get_status(ws) == 0
    monkeypatch.setenv("CARVE_FWD_PATH", "generic")
    _, _, _, _, ws_g = run_fwd(inp, L, training=True)
    g_ge = carve.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                           d["u_down"], d["u_up"], L, dd["d_o"], ws_g,
                           dd["dS_T"], dd["dm_T"])
    assert carve.get_status(ws_g) == 0
    torch.cuda.synchronize()
    from _parity import rel as _rel
    for name in g_tc:
        if g_tc[name] is not None and g_tc[name].numel():
            assert _rel(g_tc[name].float().cpu(), g_ge[name].float().cpu()) < 1e-2, name


# ------------------------------- full size, every pair: tc vs generic ----

def _all_pairs(a, b):
    from _parity import rel as _rel
    return _rel(a.float().cpu(), b.float().cpu())


def test_layer_1p3b_every_pair_tensor_core_vs_generic(monkeypatch):
    """Every (sequence, head) pair of the full 1.3B-layer forward and
    training backward: the tensor-core kernels against the generic CUDA-core
    kernels (both GPU paths; the oracle comparison of sampled pairs is in
    the tests above).  Catches pair-indexing faults in unsampled pairs."""
    cfg = WORKLOADS["layer_1p3b"]
    inp = inputs(cfg, 9, torch.bfloat16)
    gro = grad_outputs(cfg, 9, torch.bfloat16)
    d, dd = to_dev(inp), to_dev(gro)
    L = cfg["L"]
    res = {}
    for path in ("tc", "generic"):
        if path == "generic":
            monkeypatch.setenv("CARVE_FWD_PATH", "generic")
        o, S_T, m_T, ws = carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"],
                                          d["bx"], d["w"], d["u_down"],
                                          d["u_up"], L, training=True)
        gr = carve.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                             d["u_down"], d["u_up"], L, dd["d_o"], ws)
        torch.cuda.synchronize()
        assert carve.get_status(ws) == 0
        res[path] = dict(gr, o=o, S_T=S_T, m_T=m_T)
        del ws
    errs = {k: _all_pairs(res["tc"][k], res["generic"][k])
            for k in res["tc"] if res["tc"][k] is not None}
    assert_within(errs, 1e-2, "1.3B layer, all 128 pairs, tc vs generic")
