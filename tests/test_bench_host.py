"""CPU checks of bench.py's measurement arithmetic.

The algorithmic work per token per head (the roofline numerator) is
checked against values worked out by hand from the chunk form's products
(K = dk, V = dv, L = chunk length, e = bytes per element):
forward 8LK + 8KV + 8LV FLOPs and e(4K + 2V + 1) bytes, backward
24LK + 18KV + 20LV FLOPs and e(8K + 3V + 2) bytes.  The DRAM-traffic lookup
must refuse figures taken on other kernel sources or another shape.
"""
import json
import os
import sys

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))

import bench  # noqa: E402


def test_work_per_token_head_at_the_layer_shape():
    # dk = dv = 128, L = 64, bf16: q k g b_x (4 x 256 B) + v (256 B) + w (2 B)
    # in, o (256 B) out
    assert bench.fwd_bytes(128, 128, 2) == 4 * 256 + 256 + 2 + 256
    assert bench.fwd_flops(64, 128, 128) == 262144
    assert bench.bwd_flops(64, 128, 128) == 655360
    # forward + backward bytes: e (12 K + 5 V + 3)
    assert bench.fwd_bytes(128, 128, 2) + bench.bwd_bytes(128, 128, 2) == 4358


def test_work_per_token_head_at_the_long_context_shape():
    assert bench.fwd_bytes(128, 256, 2) == 2050
    assert bench.fwd_flops(64, 128, 256) == 458752


def test_roofline_times_of_the_layer_shape():
    tokens_heads = 8 * 4096 * 16
    flops = bench.fwd_flops(64, 128, 128) * tokens_heads
    bytes_ = bench.fwd_bytes(128, 128, 2) * tokens_heads
    t_flop = flops / 1640.9e12
    t_hbm = bytes_ / 6441.9e9
    assert t_flop == pytest.approx(83.8e-6, rel=2e-3)
    # per-token bytes only: the per-(b, h) state writes (S_T, 4 K V bytes
    # per pair, 1% here) are left out, which makes the fraction conservative
    assert t_hbm == pytest.approx(125.2e-6, rel=2e-3)
    assert t_hbm > t_flop  # HBM-bound


def test_whole_job_throughput():
    assert bench.job_tokens_per_s(32768, 1, 1.0) == pytest.approx(32768e3)
    assert bench.job_tokens_per_s(32768, 8, 2.0) == pytest.approx(8 * 32768 / 2e-3)


def _traffic_file(tmp_path, sha):
    d = {"sources_sha1": sha, "kernels": {"bwd_tc": {
        "shape": {"DK": 128, "DV": 128, "L": 64, "R": 32},
        "dram_bytes_per_token_head": 3000.0}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "tc_traffic.json").write_text(json.dumps(d))


def test_traffic_lookup_scales_and_refuses_stale_or_other_shapes(tmp_path, monkeypatch):
    cfg = dict(DK=128, DV=128, L=64, R=32)
    monkeypatch.setattr(bench, "HERE", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_sources_sha1", lambda: "abc")
    _traffic_file(tmp_path, "abc")
    assert bench.measured_traffic("bwd_tc", cfg, 1000) == 3000.0 * 1000
    assert bench.measured_traffic("fwd_tc", cfg, 1000) is None
    assert bench.measured_traffic("bwd_tc", dict(cfg, L=128), 1000) is None
    monkeypatch.setattr(bench, "kernel_sources_sha1", lambda: "other")
    assert bench.measured_traffic("bwd_tc", cfg, 1000) is None


def test_committed_traffic_file_names_the_captured_kernels():
    d = json.load(open(os.path.join(os.path.dirname(HERE), "profiles",
                                    "tc_traffic.json")))
    assert len(d["sources_sha1"]) == 40
    for k in ("fwd_tc", "fwd_tc_train", "bwd_tc"):
        e = d["kernels"][k]
        assert e["dram_bytes"] == pytest.approx(
            e["dram_bytes_per_token_head"] * e["token_heads"])
