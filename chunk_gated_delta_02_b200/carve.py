"""ctypes binding of libcarve (include/carve.h).

Argument marshalling only: every step of the recurrence runs in the CUDA
kernels of libcarve.so.  Tensors must be CUDA, contiguous, in the layouts of
carve.h; outputs are allocated with torch on the inputs' device and the work
is enqueued on torch's current stream.  There is no CPU fallback: a missing
library or a CPU tensor raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcarve.so")

CARVE_BF16, CARVE_FP32 = 0, 1
_DTYPES = {torch.bfloat16: CARVE_BF16, torch.float32: CARVE_FP32}
STATUS = {0: "CARVE_OK", 1: "CARVE_ERR_INVALID_ARG", 2: "CARVE_ERR_UNSUPPORTED",
          3: "CARVE_ERR_WORKSPACE", 4: "CARVE_ERR_CUDA", 5: "CARVE_ERR_TIMEOUT"}

# Entry points declared in include/carve.h (the ABI test checks the list).
EXPORTS = ("carve_workspace_bytes", "carve_chunk_fwd", "carve_chunk_bwd",
           "carve_get_status", "carve_reset_status", "carve_status_str",
           "carve_fwd_path", "carve_chunk_fwd_noalloc", "carve_decode_step",
           "carve_chunk_fwd_varlen")


class Shape(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_int32)
                 for n in ("B", "T", "H", "DK", "DV", "R", "L", "dtype")]
                + [("decay_scale", ctypes.c_float), ("qk_l2norm", ctypes.c_int32),
                   ("erase_form", ctypes.c_int32)])


class CarveError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__("%s failed: %s" % (fn, STATUS.get(code, code)))
        self.code = code


_lib = None


def lib():
    """Load libcarve.so (built in-tree by chunk_gated_delta_02_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libcarve.so is not built (%s); run "
                "`python -m chunk_gated_delta_02_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        sp = ctypes.POINTER(Shape)
        L.carve_workspace_bytes.argtypes = [sp, i32]
        L.carve_workspace_bytes.restype = sz
        L.carve_chunk_fwd.argtypes = [sp] + [vp] * 13 + [vp, sz, i32, vp]
        L.carve_chunk_fwd.restype = i32
        L.carve_chunk_bwd.argtypes = ([sp] + [vp] * 11 + [vp, sz] + [vp] * 10
                                      + [vp])
        L.carve_chunk_bwd.restype = i32
        L.carve_get_status.argtypes = [vp, vp]
        L.carve_get_status.restype = i32
        L.carve_reset_status.argtypes = [vp, vp]
        L.carve_reset_status.restype = i32
        L.carve_status_str.argtypes = [i32]
        L.carve_status_str.restype = ctypes.c_char_p
        L.carve_fwd_path.argtypes = [sp]
        L.carve_fwd_path.restype = ctypes.c_char_p
        L.carve_decode_step.argtypes = [sp] + [vp] * 13 + [vp]
        L.carve_decode_step.restype = i32
        L.carve_chunk_fwd_varlen.argtypes = [sp] + [vp] * 15 + [sz, vp]
        L.carve_chunk_fwd_varlen.restype = i32
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def make_shape(B, T, H, DK, DV, R, L, dtype, decay_scale=0.0,
               qk_l2norm=False, erase_form=0):
    """decay_scale > 0: `g` holds raw decay logits a and the kernels use
    g = -decay_scale * softplus(a); the backward then returns dL/da.
    qk_l2norm: q and k are raw and the kernels normalise them per token.
    erase_form 1: the other key-axis erase S' (I - (b k) k^T)."""
    return Shape(B, T, H, DK, DV, R, L, _DTYPES[dtype] if isinstance(
        dtype, torch.dtype) else int(dtype), float(decay_scale),
        int(bool(qk_l2norm)), int(erase_form))


def workspace_bytes(shape, training):
    n = lib().carve_workspace_bytes(ctypes.byref(shape), int(bool(training)))
    if n == 0:
        raise CarveError("carve_workspace_bytes", 2)
    return n


def fwd_path(shape):
    r = lib().carve_fwd_path(ctypes.byref(shape))
    return None if r is None else r.decode()


def _check(t, name, dtype, shape, device):
    if t is None:
        raise ValueError("%s is required" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (no CPU path)" % name)
    if t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if t.dtype != dtype:
        raise ValueError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s"
                         % (name, tuple(t.shape), tuple(shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _dims(q, v, u_down):
    B, T, H, DK = q.shape
    DV = v.shape[-1]
    R = u_down.shape[1] if u_down is not None else 0
    return B, T, H, DK, DV, R


def chunk_fwd(q, k, v, g, bx, w, u_down, u_up, L, S0=None, m0=None,
              training=False, workspace=None, o=None, want_state=True,
              decay_scale=0.0, qk_l2norm=False, erase_form=0):
    """Forward pass.  Returns (o, S_T, m_T, workspace).

    q, k, g, bx [B, T, H, DK]; v [B, T, H, DV]; w [B, T, H]; u_down
    [H, R, DV]; u_up [H, DK, R] -- all bf16 or all fp32.  S0 [B, H, DV, DK]
    and m0 [B, H, DV] fp32 or None.  With training=True the returned
    workspace holds what chunk_bwd needs.  decay_scale > 0: g holds raw
    decay logits a, the log-decay is -decay_scale * softplus(a)."""
    dev = q.device
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError("dtype must be bfloat16 or float32")
    B, T, H, DK, DV, R = _dims(q, v, u_down)
    for t, n, s in ((q, "q", (B, T, H, DK)), (k, "k", (B, T, H, DK)),
                    (v, "v", (B, T, H, DV)), (g, "g", (B, T, H, DK)),
                    (bx, "bx", (B, T, H, DK)), (w, "w", (B, T, H)),
                    (u_down, "u_down", (H, R, DV)), (u_up, "u_up", (H, DK, R))):
        _check(t, n, dt, s, dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (B, H, DV, DK), dev)
    if m0 is not None:
        _check(m0, "m0", torch.float32, (B, H, DV), dev)
    shape = make_shape(B, T, H, DK, DV, R, L, dt, decay_scale, qk_l2norm,
                       erase_form)
    nbytes = workspace_bytes(shape, training)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        workspace[:256].zero_()
    if o is None:
        o = torch.empty((B, T, H, DV), dtype=dt, device=dev)
    S_T = m_T = None
    if want_state:
        S_T = torch.empty((B, H, DV, DK), dtype=torch.float32, device=dev)
        m_T = torch.empty((B, H, DV), dtype=torch.float32, device=dev)
    rc = lib().carve_chunk_fwd(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(bx),
        _ptr(w), _ptr(u_down), _ptr(u_up), _ptr(S0), _ptr(m0), _ptr(o),
        _ptr(S_T), _ptr(m_T), _ptr(workspace), ctypes.c_size_t(
            workspace.numel()), int(bool(training)), _stream(dev))
    if rc != 0:
        raise CarveError("carve_chunk_fwd", rc)
    return o, S_T, m_T, workspace


def chunk_fwd_varlen(q, k, v, g, bx, w, u_down, u_up, L, cu_seqlens, S0=None,
                     m0=None, workspace=None, o=None, want_state=True,
                     decay_scale=0.0, qk_l2norm=False, erase_form=0):
    """Forward (no training) over packed sequences of different lengths.
    Returns (o, S_T, m_T, workspace).

    q, k, g, bx [T, H, DK]; v [T, H, DV]; w [T, H] (bf16 or fp32); u_down
    [H, R, DV]; u_up [H, DK, R]; cu_seqlens [N + 1] int32 on the device
    (sequence n is tokens cu_seqlens[n] .. cu_seqlens[n + 1] - 1); S0
    [N, H, DV, DK], m0 [N, H, DV] fp32 or None.  S_T, m_T are per sequence."""
    dev = q.device
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError("dtype must be bfloat16 or float32")
    T, H, DK = q.shape
    DV = v.shape[-1]
    R = u_down.shape[1] if u_down is not None else 0
    N = cu_seqlens.numel() - 1
    if N < 1:
        raise ValueError("cu_seqlens needs at least two entries")
    for t, n, s in ((q, "q", (T, H, DK)), (k, "k", (T, H, DK)),
                    (v, "v", (T, H, DV)), (g, "g", (T, H, DK)),
                    (bx, "bx", (T, H, DK)), (w, "w", (T, H)),
                    (u_down, "u_down", (H, R, DV)), (u_up, "u_up", (H, DK, R))):
        _check(t, n, dt, s, dev)
    _check(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), dev)
    if S0 is not None:
        _check(S0, "S0", torch.float32, (N, H, DV, DK), dev)
    if m0 is not None:
        _check(m0, "m0", torch.float32, (N, H, DV), dev)
    shape = make_shape(N, T, H, DK, DV, R, L, dt, decay_scale, qk_l2norm,
                       erase_form)
    nbytes = workspace_bytes(shape, False)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        workspace[:256].zero_()
    if o is None:
        o = torch.zeros((T, H, DV), dtype=dt, device=dev)
    S_T = m_T = None
    if want_state:
        S_T = torch.empty((N, H, DV, DK), dtype=torch.float32, device=dev)
        m_T = torch.empty((N, H, DV), dtype=torch.float32, device=dev)
    rc = lib().carve_chunk_fwd_varlen(
        ctypes.byref(shape), _ptr(cu_seqlens), _ptr(q), _ptr(k), _ptr(v),
        _ptr(g), _ptr(bx), _ptr(w), _ptr(u_down), _ptr(u_up), _ptr(S0),
        _ptr(m0), _ptr(o), _ptr(S_T), _ptr(m_T), _ptr(workspace),
        ctypes.c_size_t(workspace.numel()), _stream(dev))
    if rc != 0:
        raise CarveError("carve_chunk_fwd_varlen", rc)
    return o, S_T, m_T, workspace


def chunk_bwd(q, k, v, g, bx, w, u_down, u_up, L, d_o, workspace, dS_T=None,
              dm_T=None, want_dS0=True, out=None, decay_scale=0.0,
              qk_l2norm=False, erase_form=0):
    """Backward pass after a training-mode chunk_fwd with the same inputs
    (and the same decay_scale; with decay_scale > 0, "dg" is dL/da of the
    raw decay logits).  Returns a dict: dq dk dg dbx [B, T, H, DK], dv
    [B, T, H, DV], dw [B, T, H] (input dtype); du_down [H, R, DV], du_up
    [H, DK, R], dS0 [B, H, DV, DK], dm0 [B, H, DV] (fp32)."""
    dev = q.device
    dt = q.dtype
    B, T, H, DK, DV, R = _dims(q, v, u_down)
    _check(d_o, "d_o", dt, (B, T, H, DV), dev)
    if dS_T is not None:
        _check(dS_T, "dS_T", torch.float32, (B, H, DV, DK), dev)
    if dm_T is not None:
        _check(dm_T, "dm_T", torch.float32, (B, H, DV), dev)
    shape = make_shape(B, T, H, DK, DV, R, L, dt, decay_scale, qk_l2norm,
                       erase_form)
    if out is None:
        e = lambda s, d=dt: torch.empty(s, dtype=d, device=dev)
        out = dict(dq=e((B, T, H, DK)), dk=e((B, T, H, DK)),
                   dv=e((B, T, H, DV)), dg=e((B, T, H, DK)),
                   dbx=e((B, T, H, DK)), dw=e((B, T, H)),
                   du_down=e((H, R, DV), torch.float32),
                   du_up=e((H, DK, R), torch.float32),
                   dS0=e((B, H, DV, DK), torch.float32) if want_dS0 else None,
                   dm0=e((B, H, DV), torch.float32) if want_dS0 else None)
    rc = lib().carve_chunk_bwd(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(bx),
        _ptr(w), _ptr(u_down), _ptr(u_up), _ptr(d_o), _ptr(dS_T),
        _ptr(dm_T), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
        _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]),
        _ptr(out["dbx"]), _ptr(out["dw"]), _ptr(out["du_down"]),
        _ptr(out["du_up"]), _ptr(out.get("dS0")), _ptr(out.get("dm0")),
        _stream(dev))
    if rc != 0:
        raise CarveError("carve_chunk_bwd", rc)
    return out


def decode_step(q, k, v, g, bx, w, u_down, u_up, L, pos, S, m, osum, o=None,
                decay_scale=0.0, qk_l2norm=False, erase_form=0):
    """One recurrent decode step (one new token per (sequence, head)).

    q, k, g, bx [B, H, DK]; v [B, H, DV]; w [B, H] (bf16 or fp32); u_down
    [H, R, DV], u_up [H, DK, R]; pos [B] int32 (tokens already processed,
    read only); S [B, H, DV, DK], m, osum [B, H, DV] fp32, updated in place.
    Returns o [B, H, DV]."""
    dev = q.device
    dt = q.dtype
    if dt not in _DTYPES:
        raise ValueError("dtype must be bfloat16 or float32")
    B, H, DK = q.shape
    DV = v.shape[-1]
    R = u_down.shape[1] if u_down is not None else 0
    for t, n, s in ((q, "q", (B, H, DK)), (k, "k", (B, H, DK)),
                    (v, "v", (B, H, DV)), (g, "g", (B, H, DK)),
                    (bx, "bx", (B, H, DK)), (w, "w", (B, H)),
                    (u_down, "u_down", (H, R, DV)), (u_up, "u_up", (H, DK, R))):
        _check(t, n, dt, s, dev)
    _check(pos, "pos", torch.int32, (B,), dev)
    _check(S, "S", torch.float32, (B, H, DV, DK), dev)
    _check(m, "m", torch.float32, (B, H, DV), dev)
    _check(osum, "osum", torch.float32, (B, H, DV), dev)
    if o is None:
        o = torch.empty((B, H, DV), dtype=dt, device=dev)
    shape = make_shape(B, 1, H, DK, DV, R, L, dt, decay_scale, qk_l2norm,
                       erase_form)
    rc = lib().carve_decode_step(
        ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(bx),
        _ptr(w), _ptr(u_down), _ptr(u_up), _ptr(pos), _ptr(S), _ptr(m),
        _ptr(osum), _ptr(o), _stream(dev))
    if rc != 0:
        raise CarveError("carve_decode_step", rc)
    return o


def get_status(workspace):
    """Synchronise the current stream and read the device status word."""
    return lib().carve_get_status(_ptr(workspace), _stream(workspace.device))


class CarveFunction(torch.autograd.Function):
    """Autograd wrapper: o, S_T, m_T = CarveFunction.apply(q, k, v, g, bx, w,
    u_down, u_up, S0, m0, L)."""

    @staticmethod
    def forward(ctx, q, k, v, g, bx, w, u_down, u_up, S0, m0, L,
                decay_scale=0.0):
        o, S_T, m_T, ws = chunk_fwd(q, k, v, g, bx, w, u_down, u_up, L, S0,
                                    m0, training=True, decay_scale=decay_scale)
        ctx.save_for_backward(q, k, v, g, bx, w, u_down, u_up, ws)
        ctx.L = L
        ctx.decay_scale = decay_scale
        ctx.has_S0, ctx.has_m0 = S0 is not None, m0 is not None
        return o, S_T, m_T

    @staticmethod
    def backward(ctx, d_o, dS_T, dm_T):
        q, k, v, g, bx, w, u_down, u_up, ws = ctx.saved_tensors
        d_o = torch.zeros_like(q[..., :1].expand(*q.shape[:3], v.shape[-1]))\
            if d_o is None else d_o.contiguous()
        gr = chunk_bwd(q, k, v, g, bx, w, u_down, u_up, ctx.L, d_o, ws,
                       None if dS_T is None else dS_T.contiguous(),
                       None if dm_T is None else dm_T.contiguous(),
                       decay_scale=ctx.decay_scale)
        return (gr["dq"], gr["dk"], gr["dv"], gr["dg"], gr["dbx"], gr["dw"],
                gr["du_down"].to(u_down.dtype), gr["du_up"].to(u_up.dtype),
                gr["dS0"] if ctx.has_S0 else None,
                gr["dm0"] if ctx.has_m0 else None, None, None)


def carve(q, k, v, g, bx, w, u_down, u_up, L, S0=None, m0=None,
          decay_scale=0.0):
    """Differentiable CARVE recurrent core; returns (o, S_T, m_T).
    decay_scale > 0: g holds raw decay logits (see chunk_fwd)."""
    return CarveFunction.apply(q, k, v, g, bx, w, u_down, u_up, S0, m0, L,
                               decay_scale)
