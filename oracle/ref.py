"""ctypes wrapper around the fp64 oracle (``carve_oracle.c``).

Test infrastructure only; see ``oracle/__init__.py``.

Per-pair functions take contiguous fp64 numpy arrays for ONE
(sequence, head) pair:  q, k, g, bx [T, DK];  v [T, DV];  w [T];
u_down [R, DV];  u_up [DK, R];  S0 [DV, DK] or None;  m0 [DV] or None.

Batched functions take arrays in the library's layouts
(q [B, T, H, DK], v [B, T, H, DV], w [B, T, H], u_down [H, R, DV],
u_up [H, DK, R], S0 [B, H, DV, DK], m0 [B, H, DV]) as numpy or torch CPU
tensors of any float dtype; values are upcast to fp64 exactly.  Pairs run
in a thread pool (ctypes releases the GIL during the C call).
"""
import ctypes
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import build as _build

_lib = None
_DP = ctypes.POINTER(ctypes.c_double)


def _load():
    global _lib
    if _lib is None:
        # CARVE_ORACLE_LIB lets the mutation test point the pins at a
        # deliberately broken copy of the oracle (CPU only).
        lib = ctypes.CDLL(os.environ.get("CARVE_ORACLE_LIB") or _build.build())
        i, d = ctypes.c_int, _DP
        lib.carve_oracle_fwd.argtypes = [i, i, i, i, i] + [d] * 13
        lib.carve_oracle_fwd.restype = i
        lib.carve_oracle_bwd.argtypes = [i, i, i, i, i] + [d] * 23
        lib.carve_oracle_bwd.restype = i
        lib.carve_oracle_fwd_erase.argtypes = [i, i, i, i, i, i] + [d] * 13
        lib.carve_oracle_fwd_erase.restype = i
        lib.carve_oracle_bwd_erase.argtypes = [i, i, i, i, i, i] + [d] * 23
        lib.carve_oracle_bwd_erase.restype = i
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_DP)


def _c64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def fwd_pair(q, k, v, g, bx, w, u_down, u_up, L, S0=None, m0=None, erase=0):
    """Returns (o [T, DV], S_T [DV, DK], m_T [DV]) in fp64.  erase = 1: the
    other key-axis erase form (see carve_oracle.c)."""
    q, k, v, g, bx, w, u_down, u_up, S0, m0 = map(
        _c64, (q, k, v, g, bx, w, u_down, u_up, S0, m0))
    T, DK = q.shape
    DV = v.shape[1]
    R = u_down.shape[0]
    o = np.zeros((T, DV))
    S_T = np.zeros((DV, DK))
    m_T = np.zeros(DV)
    rc = _load().carve_oracle_fwd_erase(
        T, DK, DV, R, int(L), int(erase), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
        _ptr(bx),
        _ptr(w), _ptr(u_down), _ptr(u_up), _ptr(S0), _ptr(m0), _ptr(o),
        _ptr(S_T), _ptr(m_T))
    if rc != 0:
        raise RuntimeError("carve_oracle_fwd failed with code %d" % rc)
    return o, S_T, m_T


def bwd_pair(q, k, v, g, bx, w, u_down, u_up, L, d_o, S0=None, m0=None,
             dS_T=None, dm_T=None, erase=0):
    """Reverse mode.  Returns a dict of fp64 gradients for one pair:
    dq, dk, dg, dbx [T, DK]; dv [T, DV]; dw [T]; du_down [R, DV];
    du_up [DK, R]; dS0 [DV, DK]; dm0 [DV]."""
    q, k, v, g, bx, w, u_down, u_up, S0, m0, d_o, dS_T, dm_T = map(
        _c64, (q, k, v, g, bx, w, u_down, u_up, S0, m0, d_o, dS_T, dm_T))
    T, DK = q.shape
    DV = v.shape[1]
    R = u_down.shape[0]
    out = dict(dq=np.zeros((T, DK)), dk=np.zeros((T, DK)),
               dv=np.zeros((T, DV)), dg=np.zeros((T, DK)),
               dbx=np.zeros((T, DK)), dw=np.zeros(T),
               du_down=np.zeros((R, DV)), du_up=np.zeros((DK, R)),
               dS0=np.zeros((DV, DK)), dm0=np.zeros(DV))
    rc = _load().carve_oracle_bwd_erase(
        T, DK, DV, R, int(L), int(erase), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
        _ptr(bx),
        _ptr(w), _ptr(u_down), _ptr(u_up), _ptr(S0), _ptr(m0), _ptr(d_o),
        _ptr(dS_T), _ptr(dm_T), _ptr(out["dq"]), _ptr(out["dk"]),
        _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["dbx"]), _ptr(out["dw"]),
        _ptr(out["du_down"]), _ptr(out["du_up"]), _ptr(out["dS0"]),
        _ptr(out["dm0"]))
    if rc != 0:
        raise RuntimeError("carve_oracle_bwd failed with code %d" % rc)
    return out


# ----------------------------------------------------------------------------
# batched helpers (library layouts)

def _np64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def pair_inputs(inp, b, h):
    """Extract one pair's fp64 arrays from batched inputs (dict with keys
    q k v g bx w u_down u_up and optional S0 m0)."""
    def sl(name):
        x = inp.get(name)
        if x is None:
            return None
        if name in ("q", "k", "v", "g", "bx"):
            x = x[b, :, h, :]
        elif name == "w":
            x = x[b, :, h]
        elif name in ("u_down", "u_up"):
            x = x[h]
        elif name in ("S0", "m0"):
            x = x[b, h]
        return np.ascontiguousarray(_np64(x))
    return {n: sl(n) for n in ("q", "k", "v", "g", "bx", "w", "u_down",
                               "u_up", "S0", "m0")}


def _threads(threads):
    if threads:
        return int(threads)
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def _activate(a, decay_scale):
    """decay_scale > 0: the pair's `g` holds raw decay logits; replace them
    by the log-decay the recurrence receives (oracle/activation.py).
    Returns the raw logits (or None)."""
    if not decay_scale:
        return None
    from .activation import decay_from_logits
    raw = a["g"]
    a["g"] = decay_from_logits(raw, decay_scale)
    return raw


def _normalise(a, qk_norm):
    """qk_norm: the pair's q and k are raw; replace them by their per-token
    L2 normalisations (oracle/normalize.py).  Returns the raw (q, k)."""
    if not qk_norm:
        return None
    from .normalize import l2_normalise
    raw = (a["q"], a["k"])
    a["q"], a["k"] = l2_normalise(a["q"]), l2_normalise(a["k"])
    return raw


def fwd_batch(inp, L, pairs=None, threads=None, decay_scale=0.0,
              qk_norm=False, erase=0):
    """Oracle forward over (b, h) pairs.  Returns {(b, h): (o, S_T, m_T)}.
    decay_scale > 0: inp["g"] holds raw decay logits a, and the recurrence
    runs on g = -decay_scale * softplus(a).  qk_norm: q and k are raw and
    the recurrence runs on their per-token L2 normalisations."""
    B, _, H, _ = tuple(inp["q"].shape)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(H)]

    def one(bh):
        a = pair_inputs(inp, *bh)
        _activate(a, decay_scale)
        _normalise(a, qk_norm)
        return bh, fwd_pair(a["q"], a["k"], a["v"], a["g"], a["bx"], a["w"],
                            a["u_down"], a["u_up"], L, a["S0"], a["m0"],
                            erase)

    with ThreadPoolExecutor(_threads(threads)) as ex:
        return dict(ex.map(one, pairs))


def bwd_batch(inp, L, d_o, dS_T=None, dm_T=None, pairs=None, threads=None,
              decay_scale=0.0, qk_norm=False, erase=0):
    """Oracle reverse pass over (b, h) pairs.  d_o [B, T, H, DV],
    dS_T [B, H, DV, DK] or None, dm_T [B, H, DV] or None.
    Returns {(b, h): grads dict} (per-pair du_down / du_up, not summed).
    decay_scale > 0: inp["g"] holds raw decay logits a, and "dg" is the
    gradient with respect to a (chain rule through the activation).
    qk_norm: q and k are raw; "dq", "dk" are with respect to the raw ones."""
    B, _, H, _ = tuple(inp["q"].shape)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(H)]

    def one(bh):
        b, h = bh
        a = pair_inputs(inp, b, h)
        raw = _activate(a, decay_scale)
        raw_qk = _normalise(a, qk_norm)
        do = np.ascontiguousarray(_np64(d_o[b, :, h, :]))
        dst = None if dS_T is None else np.ascontiguousarray(_np64(dS_T[b, h]))
        dmt = None if dm_T is None else np.ascontiguousarray(_np64(dm_T[b, h]))
        gr = bwd_pair(a["q"], a["k"], a["v"], a["g"], a["bx"], a["w"],
                      a["u_down"], a["u_up"], L, do, a["S0"], a["m0"], dst, dmt,
                      erase)
        if raw is not None:
            from .activation import decay_grad
            gr["dg"] = gr["dg"] * decay_grad(raw, decay_scale)
        if raw_qk is not None:
            from .normalize import l2_normalise_grad
            gr["dq"] = l2_normalise_grad(raw_qk[0], gr["dq"])
            gr["dk"] = l2_normalise_grad(raw_qk[1], gr["dk"])
        return bh, gr

    with ThreadPoolExecutor(_threads(threads)) as ex:
        return dict(ex.map(one, pairs))
