"""Seeded synthetic inputs for the CARVE recurrent core.

This module only draws random numbers and shapes them into the value
distributions of the workloads below; it contains none of the recurrence's
arithmetic, so both the CUDA path and the fp64 oracle may consume its
output.  The oracle always receives the values exactly as rounded to the
compute dtype.

Distributions (one (sequence, head) pair each; N(0, s) has std s):
  q, k   ~ N(0, 1), then L2-normalised over the key dimension (fp64, no eps)
  v      ~ N(0, 1)
  g      = -softplus(N(0, 1)) * 0.1          log-decay per key channel (<= 0)
  bx     ~ N(0, 1)                           erase-gate logit per key channel
  w      = sigmoid(N(0, 1))                  scalar write gate per token, head
  u_down ~ N(0, 0.02)  [H, R, DV]            low-rank content projection U_b
  u_up   ~ N(0, 0.02)  [H, DK, R]            (U_b = u_up @ u_down)
  S0     ~ N(0, s0_std) [B, H, DV, DK] fp32, or zeros
The 1.3B-layer shape is one mixer layer of the 1.3B CARVE model the pages
evaluate (16 heads of dk = dv = 128); the pages' datasets are not used.
"""
import math

import torch

# Named workloads (shapes only; L is the chunk length, R the rank of U_b).
WORKLOADS = {
    "tiny": dict(B=1, H=2, T=256, DK=64, DV=64, L=64, R=16, s0_std=0.0),
    "layer_1p3b": dict(B=8, H=16, T=4096, DK=128, DV=128, L=64, R=32,
                       s0_std=0.0),
    "long_context": dict(B=1, H=16, T=65536, DK=128, DV=256, L=64, R=32,
                         s0_std=0.01),
}

_SLAB = 1 << 22  # elements per fp64 slab, bounds host memory at full size


def _normal(gen, shape, std=1.0):
    x = torch.randn(shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        x = x.double().mul_(std)
    return x


def _rows_l2_normalise(x):
    # L2 normalisation over the last dimension in fp64, slab by slab.
    flat = x.reshape(-1, x.shape[-1])
    out = torch.empty_like(flat, dtype=torch.float64)
    step = max(1, _SLAB // flat.shape[1])
    for i in range(0, flat.shape[0], step):
        y = flat[i:i + step].double()
        out[i:i + step] = y / y.norm(dim=1, keepdim=True)
    return out.reshape(x.shape)


def _map_fp64(x, fn):
    flat = x.reshape(-1)
    out = torch.empty(flat.shape, dtype=torch.float64)
    for i in range(0, flat.numel(), _SLAB):
        out[i:i + _SLAB] = fn(flat[i:i + _SLAB].double())
    return out.reshape(x.shape)


# scale of the log-decay draw g = -softplus(z) * DECAY_SCALE; with
# raw_decay=True the raw z itself is returned as g and the kernels apply
# the activation with this scale
DECAY_SCALE = 0.1


def make_inputs(B, T, H, DK, DV, R, seed, dtype=torch.bfloat16, s0_std=0.0,
                ub_zero=False, raw_decay=False, **_unused):
    """Draw one batch.  Returns a dict of CPU tensors:
    q k g bx [B, T, H, DK], v [B, T, H, DV], w [B, T, H], u_down [H, R, DV],
    u_up [H, DK, R] in ``dtype``; S0 [B, H, DV, DK] fp32 or None.
    raw_decay=True: g holds the N(0, 1) draw z instead of -softplus(z) * 0.1
    (the same random numbers; for the kernels' fused decay activation)."""
    gen = torch.Generator().manual_seed(int(seed))
    out = {}
    out["q"] = _rows_l2_normalise(_normal(gen, (B, T, H, DK))).to(dtype)
    out["k"] = _rows_l2_normalise(_normal(gen, (B, T, H, DK))).to(dtype)
    out["v"] = _normal(gen, (B, T, H, DV)).to(dtype)
    z = _normal(gen, (B, T, H, DK))
    out["g"] = (z.to(dtype) if raw_decay else
                _map_fp64(z, lambda x: -torch.nn.functional.softplus(x)
                          * DECAY_SCALE).to(dtype))
    out["bx"] = _normal(gen, (B, T, H, DK)).to(dtype)
    out["w"] = _map_fp64(_normal(gen, (B, T, H)), torch.sigmoid).to(dtype)
    ud = _normal(gen, (H, R, DV), 0.02)
    uu = _normal(gen, (H, DK, R), 0.02)
    if ub_zero:
        ud, uu = torch.zeros_like(ud), torch.zeros_like(uu)
    out["u_down"] = ud.to(dtype)
    out["u_up"] = uu.to(dtype)
    if s0_std > 0.0:
        out["S0"] = _normal(gen, (B, H, DV, DK), s0_std).float()
    else:
        out["S0"] = None
    out["m0"] = None
    return out


def make_grad_outputs(B, T, H, DK, DV, seed, dtype=torch.bfloat16, **_unused):
    """Upstream gradient dO ~ N(0, 1) [B, T, H, DV] in ``dtype``; dS_T = 0."""
    gen = torch.Generator().manual_seed(int(seed) + 7919)
    return {"d_o": _normal(gen, (B, T, H, DV)).to(dtype), "dS_T": None}


def workload(name, **overrides):
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    return cfg


def sample_pairs(B, H, n, seed=0):
    """A deterministic spread of n (b, h) pairs: the corners plus a stride."""
    pairs = [(0, 0), (B - 1, H - 1)]
    step = max(1, (B * H) // max(1, n))
    i = (seed * 7 + 3) % (B * H)
    while len(pairs) < min(n, B * H):
        bh = (i // H, i % H)
        if bh not in pairs:
            pairs.append(bh)
        i = (i + step + 1) % (B * H)
    return pairs[:n]


def tokens(cfg):
    return cfg["B"] * cfg["T"]


def n_chunks(cfg):
    return math.ceil(cfg["T"] / cfg["L"])
