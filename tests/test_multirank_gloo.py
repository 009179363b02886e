"""World-size-2 CPU tests of the multi-rank path of bench.py (gloo backend).

The hot path shards into independent (sequence, head) pairs, so a run on N
GPUs is N independent batches with no data-path collective: the only
cross-rank steps are the barrier around the timed region and the max over
ranks of the measured time.  These tests run that host logic on two CPU
ranks: process-group setup, barrier, max over ranks, per-rank batches,
the whole-job throughput, and the reference arm printing on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)

TINY = dict(B=1, T=64, H=2, DK=16, DV=16, R=4, L=16)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank),
                      WORLD_SIZE=str(ws), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    w, r, _ = bench.dist_init("gloo")
    try:
        bench.barrier(w)
        # each rank reports its own time; all must see the slowest
        t_max = bench.max_over_ranks(10.0 * (r + 1), w)
        batch = bench.rank_batch(TINY, r, torch.float32)
        again = bench.rank_batch(TINY, r, torch.float32)
        digest = torch.tensor([float(batch["q"].double().sum()),
                               float(batch["d_o"].double().sum())],
                              dtype=torch.float64)
        gathered = [torch.zeros(2, dtype=torch.float64) for _ in range(w)]
        torch.distributed.all_gather(gathered, digest)
        res = {
            "ws": w, "rank": r, "t_max": t_max,
            "deterministic": all(torch.equal(batch[k], again[k]) for k in batch),
            "shapes": {k: list(v.shape) for k, v in batch.items()},
            "digests": [g.tolist() for g in gathered],
            "value": bench.job_tokens_per_s(1000, w, 4.0),
        }
        bench.barrier(w)
    finally:
        torch.distributed.destroy_process_group()
    with open(os.path.join(out_dir, "rank%d.json" % r), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks_barrier_max_and_independent_batches(tmp_path):
    ws = 2
    mp.start_processes(_rank_main, args=(ws, _free_port(), str(tmp_path)),
                       nprocs=ws, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(ws)]
    for r, d in enumerate(res):
        assert d["ws"] == ws and d["rank"] == r
        assert d["t_max"] == 20.0           # the slowest rank's time, on both
        assert d["deterministic"]
        assert d["shapes"]["q"] == [TINY["B"], TINY["T"], TINY["H"], TINY["DK"]]
        assert d["shapes"]["d_o"] == [TINY["B"], TINY["T"], TINY["H"], TINY["DV"]]
        assert d["value"] == pytest.approx(1000 * ws / 4e-3)
    # both ranks gathered the same digests; the two batches differ
    assert res[0]["digests"] == res[1]["digests"]
    assert res[0]["digests"][0] != res[0]["digests"][1]


def test_reference_arm_prints_once_under_torchrun():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--workload", "tiny",
           "--steps", "1", "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
