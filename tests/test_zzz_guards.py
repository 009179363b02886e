"""GPU: the kernels write only inside the tensors they are given.

Every output (and the workspace) is a view into a larger buffer whose
margins hold a sentinel bit pattern; after a training forward and the
backward the margins must be untouched.  Covers the tensor-core kernels
(bf16, dk = dv = 128) and the generic kernels (dk = dv = 64, bf16 and fp32).
"""
import math

import pytest
import torch

from chunk_gated_delta_02_b200 import carve

from _parity import grad_outputs, inputs, to_dev

pytestmark = pytest.mark.gpu

GUARD = 4096  # elements (or bytes, for the workspace) on each side
_BITS = {torch.bfloat16: (torch.int16, 0x7FC1),
         torch.float32: (torch.int32, 0x7FC00001),
         torch.uint8: (torch.uint8, 0xA5)}


def _guarded(shape, dtype):
    n = math.prod(shape)
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
    itype, pat = _BITS[dtype]
    buf.view(itype).fill_(pat)
    return buf, buf[GUARD:GUARD + n].view(shape)


def _margins_intact(buf, dtype):
    itype, pat = _BITS[dtype]
    bits = buf.view(itype)
    return bool((bits[:GUARD] == pat).all()) and bool((bits[-GUARD:] == pat).all())


CASES = [
    # B, H, T, DK, DV, R, L, dtype
    (1, 2, 128, 128, 128, 16, 64, torch.bfloat16),   # tensor-core kernels
    (1, 2, 128, 64, 64, 16, 64, torch.bfloat16),     # generic kernels
    (1, 2, 96, 64, 64, 8, 32, torch.float32),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[:7])) + ("bf16" if c[7] == torch.bfloat16 else "fp32"))
def test_outputs_and_workspace_stay_inside_their_tensors(case):
    B, H, T, DK, DV, R, L, dt = case
    cfg = dict(B=B, H=H, T=T, DK=DK, DV=DV, R=R, L=L)
    d = to_dev(inputs(cfg, 5, dt))
    gro = to_dev(grad_outputs(cfg, 6, dt))
    shape = carve.make_shape(B, T, H, DK, DV, R, L, dt)
    wbytes = carve.workspace_bytes(shape, True)
    assert wbytes > 0
    bufs = {}
    bufs["ws"], ws = _guarded((wbytes,), torch.uint8)
    ws[:256].zero_()  # the header (status word) starts at CARVE_OK
    bufs["o"], o = _guarded((B, T, H, DV), dt)
    carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                    d["u_down"], d["u_up"], L, d["S0"], d["m0"],
                    training=True, workspace=ws, o=o)
    shapes = dict(dq=((B, T, H, DK), dt), dk=((B, T, H, DK), dt),
                  dv=((B, T, H, DV), dt), dg=((B, T, H, DK), dt),
                  dbx=((B, T, H, DK), dt), dw=((B, T, H), dt),
                  du_down=((H, R, DV), torch.float32),
                  du_up=((H, DK, R), torch.float32),
                  dS0=((B, H, DV, DK), torch.float32),
                  dm0=((B, H, DV), torch.float32))
    out = {}
    for name, (shp, t) in shapes.items():
        bufs[name], out[name] = _guarded(shp, t)
    carve.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                    d["u_down"], d["u_up"], L, gro["d_o"], ws, out=out)
    torch.cuda.synchronize()
    assert carve.get_status(ws) == 0
    dtypes = dict({k: t for k, (_, t) in shapes.items()}, ws=torch.uint8, o=dt)
    bad = [k for k, b in bufs.items() if not _margins_intact(b, dtypes[k])]
    assert not bad, "writes outside the tensor: %s" % bad
    assert torch.isfinite(o).all()
    for name, t in out.items():
        assert torch.isfinite(t).all(), name
