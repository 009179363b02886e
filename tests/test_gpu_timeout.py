"""GPU: the bounded device-side waits of the tensor-core kernels give up,
report CARVE_ERR_TIMEOUT with the wait site, and leave the context usable.

No GPU fault is involved.  Two test-only environment knobs of libcarve make
one wait run out on purpose: CARVE_TEST_WAIT_CYCLES lowers the limit every
wait spins before it gives up (from about 1 s to about 0.5 ms here), and
CARVE_TEST_STALL_BLOCK=n makes CTA 0 send the commit of block n's first MMA
batch to a barrier that nobody waits on.  The MMAs themselves still run and
the aborting CTA waits for them (at the full limit) before it frees its
tensor memory and exits; every other wait of that CTA then returns at once.

After each stalled call the status word is reset, and the same process runs
the call again without the knobs and checks it against the fp64 oracle.
"""
import pytest
import torch

from chunk_gated_delta_02_b200 import carve

from _parity import (assert_within, bwd_errors, fwd_errors, grad_outputs,
                     inputs, to_dev)

pytestmark = pytest.mark.gpu

WAIT_CYCLES = str(1 << 20)
# wait sites recorded in the header's `where` word
WHERE_FWD_GRAM = 3     # forward: MMA 1 (S X^T and the Grams)
WHERE_FWD_PEER = 20    # forward, dv = 256: the partner CTA's half of U_down m
WHERE_BWD_GRAM = 13    # backward: S3 (the Grams)


def _where(ws):
    torch.cuda.synchronize()
    return int(ws[8:12].view(torch.int32).item())


def _stall(monkeypatch, block):
    monkeypatch.setenv("CARVE_TEST_WAIT_CYCLES", WAIT_CYCLES)
    monkeypatch.setenv("CARVE_TEST_STALL_BLOCK", str(block))


def _unstall(monkeypatch):
    monkeypatch.delenv("CARVE_TEST_WAIT_CYCLES", raising=False)
    monkeypatch.delenv("CARVE_TEST_STALL_BLOCK", raising=False)


def _case(DV, R=16, T=256, B=1, H=2, seed=51):
    cfg = dict(B=B, H=H, T=T, DK=128, DV=DV, R=R, L=64)
    inp = inputs(cfg, seed, torch.bfloat16)
    inp["u_down"] = (inp["u_down"].float() * 25).to(torch.bfloat16)
    inp["u_up"] = (inp["u_up"].float() * 25).to(torch.bfloat16)
    return cfg, inp


def _fwd(d, L, training, ws=None):
    return carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                           d["u_down"], d["u_up"], L, d["S0"], d["m0"],
                           training=training, workspace=ws)


@pytest.mark.parametrize("training", [False, True], ids=["infer", "train"])
@pytest.mark.parametrize("block", [0, 2])
def test_forward_wait_runs_out(monkeypatch, training, block):
    cfg, inp = _case(128)
    d = to_dev(inp)
    shape = carve.make_shape(1, cfg["T"], 2, 128, 128, cfg["R"], 64,
                             torch.bfloat16)
    assert carve.fwd_path(shape) == "tc"
    _stall(monkeypatch, block)
    _, _, _, ws = _fwd(d, 64, training)
    assert carve.STATUS[carve.get_status(ws)] == "CARVE_ERR_TIMEOUT"
    assert _where(ws) == WHERE_FWD_GRAM
    # the status word is sticky until reset; then the same process runs a
    # normal call that matches the oracle
    assert carve.STATUS[carve.get_status(ws)] == "CARVE_ERR_TIMEOUT"
    carve.lib().carve_reset_status(carve._ptr(ws), carve._stream(ws.device))
    assert carve.get_status(ws) == 0
    _unstall(monkeypatch)
    _fwd(d, 64, training, ws=ws)
    assert carve.get_status(ws) == 0
    assert_within(fwd_errors(inp, 64), 1e-2, "forward after a timeout")


def test_forward_dv256_partner_gives_up_too(monkeypatch):
    # CTA 0 of the first pair stalls in block 1; its partner CTA (the other
    # value half) then waits in vain for CTA 0's half of U_down m at the
    # next chunk, gives up as well, and both reach the cluster barrier at
    # exit
    cfg, inp = _case(256)
    d = to_dev(inp)
    _stall(monkeypatch, 1)
    _, _, _, ws = _fwd(d, 64, False)
    assert carve.STATUS[carve.get_status(ws)] == "CARVE_ERR_TIMEOUT"
    assert _where(ws) in (WHERE_FWD_GRAM, WHERE_FWD_PEER)
    carve.lib().carve_reset_status(carve._ptr(ws), carve._stream(ws.device))
    _unstall(monkeypatch)
    _fwd(d, 64, False, ws=ws)
    assert carve.get_status(ws) == 0
    assert_within(fwd_errors(inp, 64), 1e-2, "dv = 256 forward after a timeout")


@pytest.mark.parametrize("block", [3, 1])
def test_backward_wait_runs_out(monkeypatch, block):
    cfg, inp = _case(128)
    gro = grad_outputs(cfg, 52, torch.bfloat16)
    d = to_dev(inp)
    dd = to_dev(gro)
    _, _, _, ws = _fwd(d, 64, True)
    assert carve.get_status(ws) == 0
    _stall(monkeypatch, block)  # the backward visits blocks last to first
    carve.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                    d["u_down"], d["u_up"], 64, dd["d_o"], ws)
    assert carve.STATUS[carve.get_status(ws)] == "CARVE_ERR_TIMEOUT"
    assert _where(ws) == WHERE_BWD_GRAM
    carve.lib().carve_reset_status(carve._ptr(ws), carve._stream(ws.device))
    _unstall(monkeypatch)
    assert_within(bwd_errors(inp, 64, gro, du_heads=range(2)), 1e-2,
                  "backward after a timeout")
