"""The C-ABI library loads and exports what include/carve.h declares, and its
host-side validation rejects bad calls before touching the GPU.

CPU only: every call below fails validation on the host, so no kernel is
ever launched (the pointers passed are never dereferenced).
"""
import ctypes
import os
import re

import pytest

from chunk_gated_delta_02_b200 import build as cbuild
from chunk_gated_delta_02_b200 import carve

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "carve.h")


@pytest.fixture(scope="module")
def lib():
    cbuild.build()
    return carve.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(carve_[a-z_]+)\s*\(", src)))


def test_header_declarations_are_exported(lib):
    names = declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), "missing export " + n
    assert sorted(carve.EXPORTS) == names


def shape(**kw):
    d = dict(B=2, T=128, H=3, DK=64, DV=64, R=8, L=64, dtype=0,
             decay_scale=0.0, qk_l2norm=0, erase_form=0)
    d.update(kw)
    return carve.Shape(*(d[n] for n in ("B", "T", "H", "DK", "DV", "R", "L",
                                        "dtype", "decay_scale", "qk_l2norm",
                                        "erase_form")))


def ws_bytes(lib, s, training):
    return lib.carve_workspace_bytes(ctypes.byref(s), training)


def test_workspace_bytes(lib):
    s = shape()
    inf, trn = ws_bytes(lib, s, 0), ws_bytes(lib, s, 1)
    assert inf > 256 and trn > inf
    # training adds the block-start states: (NB + 1) states per pair
    P, NB, DV, DK = 2 * 3, 128 // 64, 64, 64
    assert trn - inf >= P * (NB + 1) * DV * DK * 4
    for bad in (dict(DK=24), dict(DV=272), dict(L=96),
                dict(R=65), dict(B=0), dict(dtype=7), dict(L=0)):
        assert ws_bytes(lib, shape(**bad), 0) == 0, bad
    assert ws_bytes(lib, shape(T=0), 0) > 0
    # a short last chunk: the forward takes it, training does not
    assert ws_bytes(lib, shape(T=100), 0) > 0
    assert ws_bytes(lib, shape(T=100), 1) == 0


def test_decay_scale_validation(lib):
    # 0 (g is the log-decay) and any positive finite scale are accepted; a
    # negative, NaN or infinite scale is an invalid argument
    for ok in (0.0, 0.1, 5.0):
        assert ws_bytes(lib, shape(decay_scale=ok), 0) > 0, ok
    for bad in (-0.1, float("nan"), float("inf")):
        assert ws_bytes(lib, shape(decay_scale=bad), 0) == 0, bad
        assert call_fwd(lib, shape(decay_scale=bad), FAKE, 1 << 20) == 1, bad
    # the fused q / k normalisation is on or off
    assert ws_bytes(lib, shape(qk_l2norm=1), 1) > 0
    for bad in (2, -1):
        assert call_fwd(lib, shape(qk_l2norm=bad), FAKE, 1 << 20) == 1, bad
    # it runs (and trains) on the tensor-core kernels
    path = lambda **kw: lib.carve_fwd_path(ctypes.byref(shape(**kw))).decode()
    tc = dict(DK=128, DV=128, R=32, L=64, T=128, dtype=carve.CARVE_BF16)
    assert path(**dict(tc, qk_l2norm=1)) == "tc"
    # the other erase form runs on the generic kernels
    assert path(**dict(tc, erase_form=1)) == "generic"
    for bad in (2, -1):
        assert call_fwd(lib, shape(erase_form=bad), FAKE, 1 << 20) == 1, bad
    # the tensor-core backward normalises again from the raw rows: training
    # with the flag keeps the same workspace as without it
    n_tc = ws_bytes(lib, shape(**tc), 1)
    assert ws_bytes(lib, shape(**dict(tc, qk_l2norm=1)), 1) == n_tc


def test_status_strings_and_path(lib):
    for code, name in carve.STATUS.items():
        assert lib.carve_status_str(code).decode() == name
    assert lib.carve_fwd_path(ctypes.byref(shape())) is not None
    assert lib.carve_fwd_path(ctypes.byref(shape(DK=24))) is None
    # kernel family selection (host logic only): tensor cores for bf16,
    # DK = 128, R <= 32, DV = 128 or 256 and L a multiple of 64, or (forward
    # without training) L of 16, 32 or 48; generic otherwise
    path = lambda **kw: lib.carve_fwd_path(ctypes.byref(shape(**kw))).decode()
    tc = dict(DK=128, DV=128, R=32, L=64, T=128, dtype=carve.CARVE_BF16)
    assert path(**tc) == "tc"
    assert path(**dict(tc, DV=256)) == "tc"
    assert path(**dict(tc, L=128)) == "tc"
    for L in (16, 32):
        assert path(**dict(tc, L=L)) == "tc", L
        assert path(**dict(tc, L=L, DV=256)) == "tc", L
    assert path(**dict(tc, L=48, T=96)) == "tc"
    for other in (dict(DV=64), dict(DK=64), dict(L=8), dict(L=4), dict(R=48),
                  dict(dtype=carve.CARVE_FP32), dict(DV=192)):
        assert path(**dict(tc, **other)) == "generic", other
    # training with chunks shorter than 64 tokens stays on the generic
    # kernels: its workspace has the generic per-block checkpoints
    s32 = shape(**dict(tc, L=32))
    assert ws_bytes(lib, s32, 1) - ws_bytes(lib, s32, 0) >= \
        2 * 3 * (128 // 32 + 1) * 128 * 128 * 4
    # training on the tensor-core family adds the per-block records
    # (56 KiB per block and pair), one fp32 state per pair (the final one),
    # the chunk gate inputs and gradients, and the per-pair dU partials
    B, H, NB, NC, R = 2, 3, 128 // 64, 128 // 64, 32
    a256 = lambda x: (x + 255) // 256 * 256
    expect = (256 + a256(B * H * 128 * 128 * 4) + a256(B * H * NC * 128 * 4)
              + a256(B * H * NC * (128 + R) * 4)
              + a256(B * H * (R * 128 + 128 * R) * 4)
              + a256(B * H * NB * 57344) + a256(B * H * NC * (128 + R) * 4))
    assert ws_bytes(lib, shape(**tc), 1) == expect
    # the tensor-core inference forward needs the header only
    assert ws_bytes(lib, shape(**tc), 0) == 256


def test_workspace_follows_the_kernel_family(lib, monkeypatch):
    # the generic kernels keep the fp32 state at every block start and a
    # per-pair scratch, so the same shape needs more when they are selected
    tc = shape(DK=128, DV=128, R=32, L=64, T=128, dtype=carve.CARVE_BF16)
    n_tc = (ws_bytes(lib, tc, 0), ws_bytes(lib, tc, 1))
    monkeypatch.setenv("CARVE_FWD_PATH", "generic")
    assert lib.carve_fwd_path(ctypes.byref(tc)).decode() == "generic"
    n_ge = (ws_bytes(lib, tc, 0), ws_bytes(lib, tc, 1))
    B, H, NB = 2, 3, 2
    assert n_ge[1] - n_ge[0] >= B * H * (NB + 1) * 128 * 128 * 4
    assert n_ge[0] > n_tc[0]
    # a backward given a workspace sized for the tensor-core forward while
    # the generic backward is selected is refused on the host
    monkeypatch.delenv("CARVE_FWD_PATH")
    monkeypatch.setenv("CARVE_BWD_PATH", "generic")
    ins = [FAKE] * 8 + [FAKE, None, None]
    outs = [FAKE] * 8 + [None, None]
    rc = lib.carve_chunk_bwd(ctypes.byref(tc), *ins, FAKE,
                             ctypes.c_size_t(n_tc[1]), *outs, None)
    assert carve.STATUS[rc] == "CARVE_ERR_WORKSPACE"


FAKE = ctypes.c_void_p(1 << 20)          # aligned, never dereferenced
MIS = ctypes.c_void_p((1 << 20) + 4)     # misaligned


def call_fwd(lib, s, ws=None, nbytes=0, training=0, **over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, bx=FAKE, w=FAKE, ud=FAKE,
                uu=FAKE, S0=None, m0=None, o=FAKE, S_T=None, m_T=None)
    args.update(over)
    return lib.carve_chunk_fwd(
        ctypes.byref(s) if s is not None else None, args["q"], args["k"],
        args["v"], args["g"], args["bx"], args["w"], args["ud"], args["uu"],
        args["S0"], args["m0"], args["o"], args["S_T"], args["m_T"], ws,
        ctypes.c_size_t(nbytes), training, None)


def test_fwd_validation_returns_before_launch(lib):
    s = shape()
    need = ws_bytes(lib, s, 0)
    assert call_fwd(lib, None) == 1                       # no shape
    assert call_fwd(lib, shape(DK=24), FAKE, need) == 2   # unsupported
    assert call_fwd(lib, shape(T=100), FAKE, 1 << 30,
                    training=1) == 2                      # training, T % L != 0
    assert call_fwd(lib, s, FAKE, need, q=None) == 1      # null input
    assert call_fwd(lib, s, FAKE, need, v=MIS) == 1       # misaligned
    assert call_fwd(lib, s, FAKE, need, S_T=MIS) == 1     # misaligned output
    assert call_fwd(lib, s, None, need) == 3              # no workspace
    assert call_fwd(lib, s, FAKE, need - 1) == 3          # too small
    assert call_fwd(lib, s, MIS, need) == 3               # misaligned ws


def test_varlen_validation_returns_before_launch(lib):
    f = lib.carve_chunk_fwd_varlen
    f.argtypes = ([ctypes.POINTER(carve.Shape)] + [ctypes.c_void_p] * 15
                  + [ctypes.c_size_t, ctypes.c_void_p])
    f.restype = ctypes.c_int
    s = shape(T=100)  # any total length
    need = ws_bytes(lib, s, 0)

    def call(sh, cu=FAKE, ws=FAKE, nbytes=need, **over):
        a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, bx=FAKE, w=FAKE, ud=FAKE,
                 uu=FAKE, S0=None, m0=None, o=FAKE, S_T=None, m_T=None)
        a.update(over)
        return f(ctypes.byref(sh), cu, a["q"], a["k"], a["v"], a["g"],
                 a["bx"], a["w"], a["ud"], a["uu"], a["S0"], a["m0"], a["o"],
                 a["S_T"], a["m_T"], ws, nbytes, None)

    assert call(s, cu=None) == 1                          # no offsets
    assert call(s, cu=MIS) == 1                           # misaligned offsets
    assert call(shape(DK=24)) == 2
    assert call(s, q=None) == 1
    assert call(s, ws=None) == 3
    assert call(s, nbytes=need - 1) == 3


def test_bwd_validation_returns_before_launch(lib):
    s = shape()
    need = ws_bytes(lib, s, 1)
    base = [FAKE] * 8 + [FAKE, None, None]
    outs = [FAKE] * 8 + [None, None]

    def call(sh, ws, nbytes, ins=base, o=outs):
        return lib.carve_chunk_bwd(ctypes.byref(sh), *ins, ws,
                                   ctypes.c_size_t(nbytes), *o, None)

    assert call(shape(L=96), FAKE, need) == 2
    bad_in = list(base)
    bad_in[8] = None                                      # d_o missing
    assert call(s, FAKE, need, ins=bad_in) == 1
    bad_out = list(outs)
    bad_out[6] = None                                     # du_down missing
    assert call(s, FAKE, need, o=bad_out) == 1
    # inference-sized workspace is too small for the backward (checked
    # first, so that this call can never reach a launch)
    assert ws_bytes(lib, s, 0) < need
    assert call(s, FAKE, ws_bytes(lib, s, 0)) == 3


def call_noalloc(lib, s, **over):
    f = lib.carve_chunk_fwd_noalloc
    f.argtypes = [ctypes.POINTER(carve.Shape)] + [ctypes.c_void_p] * 14
    f.restype = ctypes.c_int
    args = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, bx=FAKE, w=FAKE, ud=FAKE,
                uu=FAKE, S0=None, m0=None, o=FAKE, S_T=None, m_T=None)
    args.update(over)
    return f(ctypes.byref(s) if s is not None else None, args["q"], args["k"],
             args["v"], args["g"], args["bx"], args["w"], args["ud"],
             args["uu"], args["S0"], args["m0"], args["o"], args["S_T"],
             args["m_T"], None)


def test_noalloc_validation_matches_the_workspace_entry_point(lib):
    # the allocation-free forward applies the same shape check and returns
    # the same codes as carve_chunk_fwd, all before any launch
    s = shape()
    need = ws_bytes(lib, s, 0)
    for bad in (dict(dtype=7), dict(B=0), dict(L=0), dict(DK=24),
                dict(R=65), dict(L=96)):
        want = call_fwd(lib, shape(**bad), FAKE, need)
        assert want in (1, 2), bad
        assert call_noalloc(lib, shape(**bad)) == want, bad
    assert call_noalloc(lib, None) == 1
    assert call_noalloc(lib, s, q=None) == 1
    assert call_noalloc(lib, s, v=MIS) == 1
    assert call_noalloc(lib, s, m_T=MIS) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 64, 1, 64, dtype=torch.bfloat16)
    u = torch.zeros(1, 4, 64, dtype=torch.bfloat16)
    uu = torch.zeros(1, 64, 4, dtype=torch.bfloat16)
    w = torch.zeros(1, 64, 1, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        carve.chunk_fwd(x, x, x, x, x, w, u, uu, 64)
