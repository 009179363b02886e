"""Benchmark of the CARVE chunk-parallel recurrent core on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--mode train|fwd|decode]
                    [--workload layer_1p3b|long_context|tiny] [--impl carve|reference]
                    [--chunk L] [--seq-len T] [--no-extras]

One step = one pass of the whole hot path over one batch: the training-mode
forward (chunk walk, gate, WY solve, state update, checkpoints) plus the
backward (reverse chunk walk and the U_b gradient reduction) -- or the
forward alone with --mode fwd, or the single-token decode step alone with
--mode decode (its own line: the `decode` entry below).  Inputs are synthetic (seeded, the
distributions of chunk_gated_delta_02_b200/inputs.py) and resident in HBM
when the timed region starts; they are larger than the 126 MB L2.

On one GPU the line also carries, timed the same way (CUDA events on the
launch stream, the same warm-up, clocks sampled throughout):
  fwd_infer     the 1.3B-layer inference forward, with its own roofline and
                oracle baseline
  sweep         that forward at chunk lengths 16, 32, 64, 128: tokens/s,
                roofline fraction, kernel family and the oracle error on one
                (sequence, head) pair per length
  decode        the decode step of all 128 (sequence, head) pairs: back to
                back in a CUDA graph over states evicted from L2, and single
                steps after an L2 flush
  long_context  the B=1, H=16, T=65536, dv=256 forward, with the bound its
                sequential chunk chain sets (--no-extras skips all three;
                --seq-len / --chunk change the main workload for profiling)

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of
the same shape (independent sequences, no data-path collective) -> weak
scaling; the time is the max over ranks.

Prints ONE JSON line on rank 0.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

from chunk_gated_delta_02_b200.inputs import (WORKLOADS, make_grad_outputs,  # noqa: E402
                                              make_inputs)

METRIC = "CARVE chunk fwd / fwd+bwd tokens/s on 1 B200; % of roofline"


def peaks():
    p = os.path.join(HERE, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d["bf16_tflops_sustained"]),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# Algorithmic work per token per head (K = DK, V = DV, e = element bytes):
# FLOPs are the chunk contractions at full L x L tiles; bytes are the
# compulsory tensor traffic (inputs read once, outputs written once).
def fwd_flops(L, K, V):
    return 8 * L * K + 8 * K * V + 8 * L * V


def bwd_flops(L, K, V):
    return 24 * L * K + 18 * K * V + 20 * L * V


def fwd_bytes(K, V, e):
    return e * (4 * K + 2 * V + 1)      # q k g bx v w in, o out


def bwd_bytes(K, V, e):
    return e * (8 * K + 3 * V + 2)      # q k g bx v w d_o in, 6 grads out


def roofline(flops, nbytes, pk, sustained=False):
    """Roofline time of one launch: the larger of its FLOPs over the dense
    bf16 tensor peak and its bytes over the HBM bandwidth (both measured).
    Returns (seconds, bound, peak, unit)."""
    peak_f = (pk["bf16_sus"] if sustained else pk["bf16"]) * 1e12
    t_f, t_b = flops / peak_f, nbytes / (pk["hbm"] * 1e9)
    if t_f > t_b:
        return t_f, "tensor", peak_f / 1e12, "TFLOP/s"
    return t_b, "hbm", pk["hbm"], "GB/s"


def roof_obj(name, flops, nbytes, ms, pk, traffic=None):
    """The `roofline` object of one kernel launch of `ms` milliseconds."""
    t, bound, peak, unit = roofline(flops, nbytes, pk)
    work = flops / 1e12 if bound == "tensor" else nbytes / 1e9
    achieved = work / (ms * 1e-3)
    return {"bound": bound, "kernel": name, "achieved": achieved,
            "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": traffic,
            "peak_src": pk["src"] + (" bf16_tflops" if bound == "tensor"
                                     else " hbm_gbs"),
            "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
            "roofline_ms": t * 1e3, "ms_per_launch": ms}


def kernel_sources_sha1():
    """Hash of the CUDA sources: DRAM counters taken on other sources are stale."""
    d = os.path.join(HERE, "chunk_gated_delta_02_b200", "csrc")
    h = hashlib.sha1()
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh")):
            h.update(f.encode())
            h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()


def measured_traffic(kernel, cfg, token_heads):
    """DRAM bytes (read + write) per launch of `kernel` at this shape, from
    the ncu capture summarised in profiles/tc_traffic.json (a smaller case of
    the same kernel, scaled by token-heads), or None when that capture was
    taken on other kernel sources or another shape family."""
    p = os.path.join(HERE, "profiles", "tc_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("sources_sha1") != kernel_sources_sha1():
        return None
    k = d.get("kernels", {}).get(kernel)
    if not k:
        return None
    for n in ("DK", "DV", "L", "R"):
        if k["shape"][n] != cfg[n]:
            return None
    return k["dram_bytes_per_token_head"] * token_heads


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.rows = []
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "200"] + self.sel,
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(", ") for r in out.strip().splitlines() if r.strip()]
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def dist_init(backend="nccl"):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE); the
    process group only carries the barrier and the max-over-ranks timing.
    backend="gloo" runs the same host logic on CPU ranks."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(
            backend, timeout=datetime.timedelta(seconds=120), **kw)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


def max_over_ranks(x, ws):
    """The slowest rank's time: every rank passes its own, all get the max."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_batch(cfg, rank, dtype):
    """This rank's own batch of the full shape (weak scaling: independent
    sequences, seeded by rank): inputs and the output gradient d_o."""
    inp = make_inputs(seed=1000 + rank, dtype=dtype, **cfg)
    gro = make_grad_outputs(seed=1000 + rank, dtype=dtype, **cfg)
    host = {k: v for k, v in inp.items() if v is not None}
    host["d_o"] = gro["d_o"]
    return host


def job_tokens_per_s(tokens_per_rank, ws, ms_per_step):
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * ws / (ms_per_step * 1e-3)


def host_cores():
    """(logical CPUs of the host, CPUs this process may run on)."""
    return os.cpu_count() or 1, len(os.sched_getaffinity(0))


def oracle_sample(cfg, mode, seed, threads=None):
    """Time the fp64 oracle on a bounded sample of the workload: `n` whole
    (sequence, head) pairs at the full sequence length, one thread per pair,
    n = every CPU this process may run on (at most B * H pairs).  Returns
    (seconds, pair_tokens, n_pairs, threads)."""
    from oracle import ref
    n = threads or host_cores()[1]
    n = max(1, min(n, cfg["B"] * cfg["H"]))
    inp = make_inputs(seed=seed, dtype=torch.bfloat16,
                      **dict(cfg, B=1, H=n))
    gro = make_grad_outputs(seed=seed, dtype=torch.bfloat16,
                            **dict(cfg, B=1, H=n))
    pairs = [(0, h) for h in range(n)]
    ref.fwd_batch(inp, cfg["L"], pairs=pairs[:1], threads=1)  # load/build
    t0 = time.perf_counter()
    if mode == "fwd":
        ref.fwd_batch(inp, cfg["L"], pairs=pairs, threads=n)
    else:
        ref.bwd_batch(inp, cfg["L"], gro["d_o"], pairs=pairs, threads=n)
    dt = time.perf_counter() - t0
    return dt, n * cfg["T"], n, n


def cpu_baseline_obj(cfg, mode, seed):
    secs, ptoks, npairs, thr = oracle_sample(cfg, mode, seed)
    ncpu, naff = host_cores()
    return {"value": ptoks / cfg["H"] / secs, "unit": "tokens/s",
            "cores": thr, "host_cpus": ncpu, "affinity_cpus": naff,
            "kind": "oracle",
            "sample": "%d (sequence, head) pairs x %d tokens, %s, fp64, one "
                      "thread per pair on %d of %d usable CPUs; tokens = "
                      "pair-tokens / H" % (
                          npairs, cfg["T"],
                          "fwd+bwd" if mode == "train" else "fwd", thr, naff)}


def run_reference(args, cfg, ws, rank):
    """The oracle as the reference arm (CPU, host cores)."""
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(cfg, args.mode, 100)
    secs, ptoks, npairs, thr = 0.0, 0, 0, 0
    for i in range(args.steps):
        s, p, npairs, thr = oracle_sample(cfg, args.mode, 200 + i)
        secs += s
        ptoks += p
    value = ptoks / cfg["H"] / secs
    sample = ("%d (sequence, head) pairs x %d tokens per step, %s, fp64; "
              "tokens = pair-tokens / H" % (npairs, cfg["T"],
                                            "fwd+bwd" if args.mode == "train"
                                            else "fwd"))
    line = {"impl": "reference", "metric": METRIC, "value": value,
            "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": config_dict(args, cfg),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": thr,
                             "host_cpus": host_cores()[0],
                             "affinity_cpus": host_cores()[1],
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s",
                    "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(args, cfg):
    name = args.workload if not args.seq_len else "%s(T=%d)" % (args.workload,
                                                               args.seq_len)
    if args.chunk:
        name += "(L=%d)" % args.chunk
    return {"workload": "%s %s" % (name,
                                   "fwd+bwd" if args.mode == "train" else "fwd"),
            "B": cfg["B"], "T": cfg["T"], "H": cfg["H"], "DK": cfg["DK"],
            "DV": cfg["DV"], "L": cfg["L"], "R": cfg["R"],
            "state": "fp32", "l2": "inputs larger than L2 (no flush needed)",
            "parallelism": "independent sequences per rank (dp%d)" % args.gpus}


def time_launches(fn, stream, warmup, iters):
    """Average milliseconds of fn() over `iters` back-to-back calls on
    `stream` (CUDA events around the batch, after `warmup` calls)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = (torch.cuda.Event(enable_timing=True) for _ in range(2))
    a.record(stream)
    for _ in range(iters):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def fwd_call(carve, d, L, training=False, ws=None, o=None):
    return carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                           d["u_down"], d["u_up"], L, d.get("S0"), None,
                           training=training, workspace=ws, o=o,
                           want_state=False)


def pair_error(carve, host, d, L, bh):
    """max|delta| / max|ref| of o and S_T on one (sequence, head) pair: the
    forward at chunk length L on the GPU against the fp64 oracle."""
    from oracle import ref
    import numpy as np
    o, S_T, _, _ = carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["bx"],
                                   d["w"], d["u_down"], d["u_up"], L,
                                   d.get("S0"), None)
    torch.cuda.synchronize()
    b, h = bh
    oo, SS, _ = ref.fwd_batch(host, L, pairs=[bh], threads=1)[bh]

    def rel(x, y):
        x = x.detach().double().cpu().numpy()
        return float(np.abs(x - y).max() / np.abs(y).max())
    return {"o": rel(o[b, :, h, :], oo), "S_T": rel(S_T[b, h], SS)}


def decode_bench(carve, d, cfg, it, warmup, pk, stream):
    """The decode step at the shape of `cfg` (one new token per (sequence,
    head), the fp32 state read and written once): back to back in a CUDA
    graph over cold states, and single steps after an L2 flush."""
    B, H, DK, DV = (cfg[n] for n in ("B", "H", "DK", "DV"))
    dev = d["q"].device
    L = cfg["L"]
    tok = {n: d[n][:, 0].contiguous() for n in ("q", "k", "v", "g", "bx", "w")}
    Sd = torch.randn((B, H, DV, DK), device=dev) * 0.1
    md = torch.zeros((B, H, DV), device=dev)
    od = torch.zeros((B, H, DV), device=dev)
    pos = torch.full((B,), 5, dtype=torch.int32, device=dev)
    outd = torch.empty((B, H, DV), dtype=d["q"].dtype, device=dev)
    step = lambda: carve.decode_step(tok["q"], tok["k"], tok["v"], tok["g"],
                                     tok["bx"], tok["w"], d["u_down"],
                                     d["u_up"], L, pos, Sd, md, od, o=outd)
    # the state (B H DV DK fp32 = 8 MiB here) fits in L2: write a buffer
    # larger than L2 between timed steps so that each reads S from HBM
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(it)]
    for _ in range(warmup):
        step()
    for e0, e1 in evs:
        flush.fill_(1)
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    msd = statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)
    del flush
    # back to back: steps over 20 separate states (160 MiB, more than L2),
    # each step reading a state the 19 before it evicted, captured in one
    # CUDA graph (as a serving loop would run them, without a Python call
    # per step); the average per step is the kernel's launch-to-launch time
    n_st = 20
    states = [torch.randn((B, H, DV, DK), device=dev) * 0.1 for _ in range(n_st)]
    bstep = lambda i: carve.decode_step(tok["q"], tok["k"], tok["v"], tok["g"],
                                        tok["bx"], tok["w"], d["u_down"],
                                        d["u_up"], L, pos, states[i % n_st],
                                        md, od, o=outd)
    n_b = 4 * n_st
    for i in range(n_st):
        bstep(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(n_b):
            bstep(i)
    for _ in range(2):
        graph.replay()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    reps = 3
    b0.record()
    for _ in range(reps):
        graph.replay()
    b1.record()
    torch.cuda.synchronize()
    msb = b0.elapsed_time(b1) / (reps * n_b)
    del graph, states
    pairs = B * H
    dec_bytes = pairs * (2 * DV * DK * 4 + 2 * (4 * DK + 2 * DV + 1)
                         + 4 * DV * 4)
    dec_flops = pairs * (6 * DV * DK + 2 * DV * DK)
    rdec = roof_obj("carve_decode_step", dec_flops, dec_bytes, msb, pk)
    return {
        "workload": "layer_1p3b decode step (B=8, H=16, dk=dv=128, r=32, "
                    "L=64; one token per sequence)",
        "ms": msb, "tokens_per_s": B / (msb * 1e-3), "roofline": rdec,
        "timing": "%d steps back to back in one CUDA graph over %d states "
                  "(%.0f MiB, above L2), average per step" % (
                      n_b, n_st, n_st * B * H * DV * DK * 4 / 2**20),
        "single_step_ms": msd,
        "single_step_timing": "median of %d single steps, L2 flushed before "
                              "each (includes the launch)" % it,
        "bytes_per_pair_step": dec_bytes / pairs}


def extras(carve, args, pk, host, d, stream, fwd_ms_train):
    """Inference forward, chunk-length sweep and long-context forward at
    their full sizes (one GPU), each timed like the main step."""
    cfg = WORKLOADS["layer_1p3b"]
    B, T, H, DK, DV, R = (cfg[n] for n in ("B", "T", "H", "DK", "DV", "R"))
    th = B * T * H
    it = max(5, args.steps)
    out = {}
    ws = None
    o = torch.empty_like(d["v"])

    # fwd_infer: config 1, training = 0
    L = cfg["L"]
    _, _, _, ws = fwd_call(carve, d, L, o=o)
    ms = time_launches(lambda: fwd_call(carve, d, L, ws=ws, o=o), stream,
                       args.warmup, it)
    assert carve.get_status(ws) == 0, "device status word set"
    ro = roof_obj("carve_chunk_fwd", fwd_flops(L, DK, DV) * th,
                  fwd_bytes(DK, DV, 2) * th, ms, pk,
                  measured_traffic("fwd_tc", dict(cfg, L=L), th))
    out["fwd_infer"] = {
        "workload": "layer_1p3b fwd (training = 0)", "ms": ms,
        "tokens_per_s": B * T / (ms * 1e-3), "roofline": ro,
        "kernel_path": carve.fwd_path(carve.make_shape(B, T, H, DK, DV, R, L,
                                                       torch.bfloat16)),
        "training_fwd_ms": fwd_ms_train,
        "cpu_baseline": (cpu_baseline_obj(cfg, "fwd", 7)
                         if not args.no_cpu_baseline else None)}

    # sweep: config 2, L in {16, 32, 64, 128}, forward only
    sweep = []
    for Ls in (16, 32, 64, 128):
        shape = carve.make_shape(B, T, H, DK, DV, R, Ls, torch.bfloat16)
        _, _, _, wsl = fwd_call(carve, d, Ls, o=o)
        n_it = it if carve.fwd_path(shape) == "tc" else 2
        msl = time_launches(lambda: fwd_call(carve, d, Ls, ws=wsl, o=o),
                            stream, 1 if n_it == 2 else args.warmup, n_it)
        assert carve.get_status(wsl) == 0, "device status word set"
        rl = roof_obj("carve_chunk_fwd", fwd_flops(Ls, DK, DV) * th,
                      fwd_bytes(DK, DV, 2) * th, msl, pk)
        err = (pair_error(carve, host, d, Ls, (B - 1, H - 1))
               if not args.no_cpu_baseline else None)
        sweep.append({"L": Ls, "ms": msl, "tokens_per_s": B * T / (msl * 1e-3),
                      "frac": rl["frac"], "bound": rl["bound"],
                      "roofline_ms": rl["roofline_ms"],
                      "kernel_path": carve.fwd_path(shape),
                      "timed_launches": n_it,
                      "oracle_error_pair": [B - 1, H - 1],
                      "oracle_error": err})
        del wsl
    out["sweep"] = sweep

    out["decode"] = decode_bench(carve, d, cfg, it, args.warmup, pk, stream)

    # long_context: config 3 (dv = 256, S0 != 0), forward
    lc = WORKLOADS["long_context"]
    hl = make_inputs(seed=3, dtype=torch.bfloat16, **lc)
    dl = {k: (v.to(d["q"].device) if v is not None else None)
          for k, v in hl.items()}
    Bl, Tl, Hl, DKl, DVl, Rl, Ll = (lc[n] for n in ("B", "T", "H", "DK", "DV",
                                                    "R", "L"))
    ol = torch.empty_like(dl["v"])
    _, _, _, wsc = fwd_call(carve, dl, Ll, o=ol)
    msc = time_launches(lambda: fwd_call(carve, dl, Ll, ws=wsc, o=ol), stream,
                        args.warmup, max(3, args.steps // 2))
    assert carve.get_status(wsc) == 0, "device status word set"
    thl = Bl * Tl * Hl
    rc = roof_obj("carve_chunk_fwd", fwd_flops(Ll, DKl, DVl) * thl,
                  fwd_bytes(DKl, DVl, 2) * thl + 2 * Bl * Hl * DVl * DKl * 4,
                  msc, pk)
    # the chunk chain: each (sequence, head) walks Tl / 64 blocks one after
    # another (the content gate of a chunk needs the previous chunk's
    # outputs), on 2 CTAs per pair (B * H * 2 = 32 of 148 SMs busy).  At the
    # per-block latency of the 1.3B-layer inference forward that chain takes:
    per_block_us = 1e3 * ms / (T // 64)
    chain_ms = per_block_us * (Tl // 64) * 1e-3
    out["long_context"] = {
        "workload": "long_context fwd (B=1, H=16, T=65536, dk=128, dv=256, "
                    "S0 ~ N(0, 0.01))",
        "ms": msc, "tokens_per_s": Bl * Tl / (msc * 1e-3), "roofline": rc,
        "kernel_path": carve.fwd_path(carve.make_shape(
            Bl, Tl, Hl, DKl, DVl, Rl, Ll, torch.bfloat16)),
        "chain_bound": {"blocks_per_pair": Tl // 64,
                        "per_block_us_at_layer_1p3b": per_block_us,
                        "chain_ms": chain_ms, "frac": chain_ms / msc,
                        "busy_sms": 2 * Bl * Hl, "sms": 148}}
    del dl, hl, ol, wsc
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--mode", choices=["train", "fwd", "decode"], default="train",
                    help="decode: the single-token decode step alone")
    ap.add_argument("--workload", default="layer_1p3b", choices=list(WORKLOADS))
    ap.add_argument("--impl", choices=["carve", "reference"], default="carve")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip fwd_infer, sweep and long_context")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override T (profiler captures of a smaller case)")
    ap.add_argument("--chunk", type=int, default=None,
                    help="override the chunk length L of the main workload")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "carve":
        ap.error("--warmup must be >= 3")
    cfg = dict(WORKLOADS[args.workload])
    if args.seq_len:
        cfg["T"] = args.seq_len
    if args.chunk:
        cfg["L"] = args.chunk
    ws, rank, local = dist_init() if args.impl == "carve" else (
        int(os.environ.get("WORLD_SIZE", "1")),
        int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        run_reference(args, cfg, ws, rank)
        return

    from chunk_gated_delta_02_b200 import carve
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dtype = torch.bfloat16
    if args.mode == "decode":
        # the decode step reads one token per sequence: inputs of 64 tokens
        host = rank_batch(dict(cfg, T=64), rank, dtype)
        dd = {k: v.to(dev) for k, v in host.items()}
        res = decode_bench(carve, dd, cfg, max(5, args.steps), args.warmup,
                           peaks(), torch.cuda.current_stream(dev))
        if rank == 0:
            print(json.dumps({
                "metric": "decode tokens/s (one new token per sequence)",
                "value": res["tokens_per_s"], "unit": "tokens/s", "n_gpus": ws,
                "mode": "decode", "higher_is_better": True, "data": "synthetic",
                "dtype": "bf16", "decode": res}), flush=True)
        return
    B, T, H, DK, DV, R, L = (cfg[n] for n in ("B", "T", "H", "DK", "DV", "R",
                                              "L"))
    host = rank_batch(cfg, rank, dtype)
    d = {k: v.to(dev) for k, v in host.items()}
    d.setdefault("S0", None)
    training = args.mode == "train"
    stream = torch.cuda.current_stream(dev)

    def fwd(ws_buf=None, o=None):
        return carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["bx"],
                               d["w"], d["u_down"], d["u_up"], L, d.get("S0"),
                               None, training=training, workspace=ws_buf, o=o)

    o, S_T, m_T, wsb = fwd()
    grads = None
    if training:
        grads = carve.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["bx"],
                                d["w"], d["u_down"], d["u_up"], L, d["d_o"],
                                wsb)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        carve.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                        d["u_down"], d["u_up"], L, d.get("S0"), None,
                        training=training, workspace=wsb, o=o,
                        want_state=False)
        if ev:
            ev[1].record(stream)
        if training:
            carve.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["bx"], d["w"],
                            d["u_down"], d["u_up"], L, d["d_o"], wsb,
                            out=grads)
        if ev:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert carve.get_status(wsb) == 0, "device status word set"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
           for _ in range(args.steps)]
    clocks = ClockSampler(dev) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    barrier(ws)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop() if clocks else None
    total_ms = t_start.elapsed_time(t_end)
    total_ms = max_over_ranks(total_ms, ws)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    bwd_ms = (sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
              if training else 0.0)
    assert carve.get_status(wsb) == 0, "device status word set"

    ms_step = total_ms / args.steps
    tokens = B * T
    value = job_tokens_per_s(tokens, ws, ms_step)

    # roofline of the dominant kernel (fwd or bwd): max(FLOPs / bf16 peak,
    # bytes / HBM bandwidth), both measured
    pk = peaks()
    e = 2
    th = B * T * H
    fwd_b = fwd_bytes(DK, DV, e) * th
    bwd_b = bwd_bytes(DK, DV, e) * th
    fwd_f = fwd_flops(L, DK, DV) * th
    bwd_f = bwd_flops(L, DK, DV) * th
    if training and bwd_ms >= fwd_ms:
        dom, dom_ms, dom_b, dom_f = "bwd", bwd_ms, bwd_b, bwd_f
    else:
        dom, dom_ms, dom_b, dom_f = "fwd", fwd_ms, fwd_b, fwd_f
    traffic = measured_traffic(dom + "_tc" + ("_train" if dom == "fwd" and
                                              training else ""), cfg, th)
    roof_t_fwd = roofline(fwd_f, fwd_b, pk)[0]
    roof_t_all = roofline(fwd_f + (bwd_f if training else 0),
                          fwd_b + (bwd_b if training else 0), pk)[0]
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded; inputs.py distributions)",
        "config": config_dict(args, cfg),
        "kernel_path": carve.fwd_path(carve.make_shape(B, T, H, DK, DV, R, L,
                                                       dtype)),
        "roofline": roof_obj("carve_chunk_" + dom, dom_f, dom_b, dom_ms, pk,
                             traffic),
        "step_roofline": {"roofline_ms": roof_t_all * 1e3,
                          "frac": roof_t_all * 1e3 / ms_step},
        "fwd": {"ms": fwd_ms, "tokens_per_s": tokens / (fwd_ms * 1e-3),
                "roofline_ms": roof_t_fwd * 1e3,
                "frac": roof_t_fwd * 1e3 / fwd_ms,
                "training": training},
        "bwd": {"ms": bwd_ms} if training else None,
        "workspace": {"bytes": int(wsb.numel()),
                      "bytes_per_token_head": wsb.numel() / th,
                      "training": training},
        # per step: the forward; the backward kernel and, with R > 0, the two
        # dU reduction kernels
        "gpu_launches": args.steps * ((2 + (2 if R > 0 else 0)) if training
                                      else 1),
    }

    # end to end through the public API: pinned host inputs -> device, step,
    # results -> pinned host, all inside the timed region.  Two device sets
    # of inputs and outputs: step i uses set i % 2, so step i's results copy
    # out while step i + 1's inputs copy in (PCIe is full duplex) and the
    # kernels run between them, each copy direction on its own stream.
    if not args.no_e2e:
        pin = {k: v.pin_memory() for k, v in host.items()}
        d_sets = [d, {k: (torch.empty_like(v) if v is not None else None)
                      for k, v in d.items()}]
        o_sets = [o, torch.empty_like(o)]
        g_sets = ([grads, {k: (torch.empty_like(v) if v is not None else None)
                           for k, v in grads.items()}]
                  if training else [None, None])
        outs_host = {"o": torch.empty(o.shape, dtype=o.dtype).pin_memory()}
        if training:
            for k, v in grads.items():
                if v is not None:
                    outs_host[k] = torch.empty(v.shape, dtype=v.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in pin.values())
        d2h = sum(v.numel() * v.element_size() for v in outs_host.values())
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)]
                                  for _ in range(3))
        count = [0]

        def e2e_step():
            i = count[0]
            count[0] += 1
            sset = i % 2
            ds, os_, gs = d_sets[sset], o_sets[sset], g_sets[sset]
            with torch.cuda.stream(s_in):
                if i >= 2:  # the kernels of step i - 2 have read this set
                    s_in.wait_event(ev_comp[sset])
                for k, v in pin.items():
                    ds[k].copy_(v, non_blocking=True)
                ev_in[sset].record(s_in)
            stream.wait_event(ev_in[sset])
            if i >= 2:  # step i - 2's results have left this set
                stream.wait_event(ev_out[sset])
            carve.chunk_fwd(ds["q"], ds["k"], ds["v"], ds["g"], ds["bx"],
                            ds["w"], ds["u_down"], ds["u_up"], L, ds.get("S0"),
                            None, training=training, workspace=wsb, o=os_,
                            want_state=False)
            if training:
                carve.chunk_bwd(ds["q"], ds["k"], ds["v"], ds["g"], ds["bx"],
                                ds["w"], ds["u_down"], ds["u_up"], L,
                                ds["d_o"], wsb, out=gs)
            ev_comp[sset].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[sset])
                outs_host["o"].copy_(os_, non_blocking=True)
                if training:
                    for k, v in gs.items():
                        if v is not None:
                            outs_host[k].copy_(v, non_blocking=True)
                ev_out[sset].record(s_out)
            return sset

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        a, b = (torch.cuda.Event(enable_timing=True) for _ in range(2))
        n_e2e = max(6, args.steps // 2)
        a.record(s_in)
        for _ in range(n_e2e):
            last = e2e_step()
        stream.wait_event(ev_out[last])
        b.record(stream)
        torch.cuda.synchronize()
        assert carve.get_status(wsb) == 0, "device status word set"
        e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, ws)
        line["e2e"] = {"value": job_tokens_per_s(tokens, ws, e2e_ms),
                       "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                       "pipelining": "double-buffered: step i's D2H overlaps "
                                     "step i+1's H2D (separate streams)"}

    line["clocks"] = clk
    if (ws == 1 and not args.no_extras and args.workload == "layer_1p3b"
            and not args.seq_len and not args.chunk):
        xclk = ClockSampler(dev)
        xclk.start()
        time.sleep(0.3)
        line.update(extras(carve, args, pk, host, d, stream,
                           fwd_ms if training else None))
        line["extras_clocks"] = xclk.stop()
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_obj(cfg, args.mode, 7)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
