"""Helpers for the GPU parity tests: run libcarve on CUDA, the fp64 oracle on
the CPU, on the same seeded inputs, and compare element by element.

The comparison measure is the pages' tolerance form max|delta| / max|ref|
per tensor, over every compared (sequence, head) pair.
"""
import numpy as np
import torch

from chunk_gated_delta_02_b200 import carve
from chunk_gated_delta_02_b200.inputs import make_grad_outputs, make_inputs
from oracle import ref

TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}
TOKEN_KEYS = ("q", "k", "v", "g", "bx", "w")


def to_dev(inp, device="cuda"):
    return {k: (None if x is None else x.to(device).contiguous())
            for k, x in inp.items()}


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = float(np.abs(b).max()) if b.size else 0.0
    if den == 0.0:
        return float(np.abs(a).max()) if a.size else 0.0
    return float(np.abs(a - b).max() / den)


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


class Gathered:
    """Accumulates (gpu, oracle) pairs per tensor name across pairs."""

    def __init__(self):
        self.g, self.r = {}, {}

    def add(self, name, gpu, oracle):
        self.g.setdefault(name, []).append(np.asarray(gpu, np.float64).ravel())
        self.r.setdefault(name, []).append(np.asarray(oracle, np.float64).ravel())

    def errors(self):
        return {n: rel(np.concatenate(self.g[n]), np.concatenate(self.r[n]))
                for n in self.g}


def run_fwd(inp, L, training=False, decay_scale=0.0, qk_l2norm=False,
            erase_form=0):
    d = to_dev(inp)
    o, S_T, m_T, ws = carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["bx"],
                                      d["w"], d["u_down"], d["u_up"], L,
                                      d["S0"], d["m0"], training=training,
                                      decay_scale=decay_scale,
                                      qk_l2norm=qk_l2norm,
                                      erase_form=erase_form)
    torch.cuda.synchronize()
    return d, o, S_T, m_T, ws


def fwd_errors(inp, L, pairs=None, decay_scale=0.0, qk_l2norm=False,
               erase_form=0):
    """GPU forward over the whole batch; oracle on `pairs` (default all).
    decay_scale > 0: inp["g"] holds raw decay logits (both sides activate)."""
    _, o, S_T, m_T, ws = run_fwd(inp, L, decay_scale=decay_scale,
                                 qk_l2norm=qk_l2norm, erase_form=erase_form)
    assert carve.get_status(ws) == 0
    res = ref.fwd_batch(inp, L, pairs=pairs, decay_scale=decay_scale,
                        qk_norm=qk_l2norm, erase=erase_form)
    acc = Gathered()
    o_c, S_c, m_c = o.cpu(), S_T.cpu(), m_T.cpu()
    for (b, h), (oo, SS, mm) in res.items():
        acc.add("o", np64(o_c[b, :, h, :]), oo)
        acc.add("S_T", np64(S_c[b, h]), SS)
        acc.add("m_T", np64(m_c[b, h]), mm)
    return acc.errors()


def bwd_errors(inp, L, grads, pairs=None, du_heads=(), decay_scale=0.0,
               qk_l2norm=False, erase_form=0):
    """GPU training forward + backward; oracle reverse pass on `pairs`.
    du_down / du_up (summed over the batch) are compared for each head in
    `du_heads`, for which the oracle runs every sequence of that head."""
    d, o, S_T, m_T, ws = run_fwd(inp, L, training=True,
                                 decay_scale=decay_scale, qk_l2norm=qk_l2norm,
                                 erase_form=erase_form)
    dd = to_dev(grads)
    gr = carve.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                         d["u_down"], d["u_up"], L, dd["d_o"], ws,
                         dd.get("dS_T"), dd.get("dm_T"),
                         decay_scale=decay_scale, qk_l2norm=qk_l2norm,
                         erase_form=erase_form)
    torch.cuda.synchronize()
    assert carve.get_status(ws) == 0
    B, _, H, _ = inp["q"].shape
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(H)]
    need = sorted(set(pairs) | {(b, h) for h in du_heads for b in range(B)})
    res = ref.bwd_batch(inp, L, grads["d_o"], grads.get("dS_T"),
                        grads.get("dm_T"), pairs=need, decay_scale=decay_scale,
                        qk_norm=qk_l2norm, erase=erase_form)
    g = {k: (None if v is None else v.cpu()) for k, v in gr.items()}
    acc = Gathered()
    for (b, h) in pairs:
        r = res[(b, h)]
        for name in ("dq", "dk", "dg", "dbx", "dv"):
            acc.add(name, np64(g[name][b, :, h, :]), r[name])
        acc.add("dw", np64(g["dw"][b, :, h]), r["dw"])
        acc.add("dS0", np64(g["dS0"][b, h]), r["dS0"])
        acc.add("dm0", np64(g["dm0"][b, h]), r["dm0"])
    for h in du_heads:
        acc.add("du_down", np64(g["du_down"][h]),
                sum(res[(b, h)]["du_down"] for b in range(B)))
        acc.add("du_up", np64(g["du_up"][h]),
                sum(res[(b, h)]["du_up"] for b in range(B)))
    return acc.errors()


# (what, tol, {tensor: max|delta| / max|ref|}) of every comparison made in
# this process; tests/conftest.py prints them at the end of the run so that
# the log shows the headroom under each tolerance.
MARGINS = []


def record(what, tol, errs):
    MARGINS.append((what, tol, dict(errs)))


def assert_within(errs, tol, what=""):
    record(what, tol, errs)
    bad = {k: v for k, v in errs.items() if not (v <= tol)}
    assert not bad, "%s exceeds %.1e: %s (all: %s)" % (what, tol, bad, errs)


def inputs(cfg, seed, dtype, **over):
    c = dict(cfg)
    c.update(over)
    return make_inputs(seed=seed, dtype=dtype, **c)


def grad_outputs(cfg, seed, dtype):
    return make_grad_outputs(seed=seed, dtype=dtype, **cfg)
