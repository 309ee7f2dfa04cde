"""Benchmark of the MALA hot path on synthetic data (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mala|reference]

Workload (per GPU): long-context GQA prefill, batch 1, 32 query heads, 8 KV
heads, N = 32768, d = 128, 128 x 128 tiles, bf16, causal, heads in thirds
(diffuse / local / retrieval), tau = 0.2. One step = one pass of the hot path
over that batch: the MALA forward, then (when built) the MALA backward with
dO ~ N(0, 1). Inputs (~0.4 GB) are larger than the 126 MB L2.

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch
(independent problems, no data-path collective), time = max over ranks,
value = tokens of all ranks / that time ("weak" scaling).

--impl reference times the fp64 CPU oracle (the only reference this operator
has) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MALA fwd/bwd tokens/s at N=32k,d=128; executed TFLOP/s vs bf16 peak"
WORKLOAD = "gqa_32k"
TAU = 0.2
SEED = 42
TILE = 128


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def tile_flops(d: int = 128) -> float:
    """FLOPs of one 128 x 128 x d tile matmul (2 per multiply-add)."""
    return 2.0 * TILE * TILE * d


def run_mala(args):
    import torch
    import torch.distributed as dist
    from tile_skipping_causal_b200 import mala, synth

    world, rank, local = _dist_init()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    mala.load_library()

    w = synth.WORKLOADS[WORKLOAD]
    t = synth.make_prefill(w, SEED + rank, with_do=True, seqlen=args.seqlen)
    host = {n: x.pin_memory() for n, x in t.items()}
    q, k, v, do = (host[n].to(dev) for n in ("q", "k", "v", "do"))
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    nQB = nKB = N // TILE
    stream = torch.cuda.current_stream()
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    keep = torch.empty((B, Hq, nQB, mala.mask_words(nKB)), dtype=torch.int32, device=dev)
    stats = torch.zeros(4, dtype=torch.int64, device=dev)
    launches_per_step = 1

    def step(tau, st=None):
        mala.mala_fwd(q, k, v, tau, TILE, TILE, o=o, lse=lse, keep_mask=keep, stats=st)

    # one measured step for the executed-work counts
    stats.zero_()
    step(TAU, stats)
    mala.check_device_error()
    tested, kept, slots = (int(x) for x in stats.cpu().tolist()[:3])
    fwd_flops = tile_flops(d) * (tested + kept)

    for _ in range(args.warmup):
        step(TAU)
    torch.cuda.synchronize()

    # per-launch kernel time with events on the launching stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for s in range(args.steps):
            ev[s][0].record(stream)
            step(TAU)
            ev[s][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    elapsed = t0.elapsed_time(t1) / 1e3
    mala.check_device_error()
    fwd_times = [a.elapsed_time(b) / 1e3 for a, b in ev]
    if world > 1:
        tt = torch.tensor([elapsed], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        elapsed = float(tt.item())
    ms_per_step = elapsed / args.steps * 1e3
    tokens = B * N * world * args.steps
    value = tokens / elapsed

    if args.no_extras:
        if rank == 0:
            print(json.dumps({"profile_case": True, "seqlen": N, "ms_per_step": ms_per_step}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    # dense comparison: the same kernels at tau = 0
    stats.zero_()
    step(0.0, stats)
    d_tested, d_kept, _ = (int(x) for x in stats.cpu().tolist()[:3])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(max(1, args.steps // 2)):
        step(0.0)
    e1.record(stream)
    torch.cuda.synchronize()
    dense_s = e0.elapsed_time(e1) / 1e3 / max(1, args.steps // 2)

    # end to end through the public API with pinned host buffers
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    h2d = sum(host[n].numel() * host[n].element_size() for n in ("q", "k", "v"))
    d2h = o_h.numel() * o_h.element_size()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        qd = host["q"].to(dev, non_blocking=True)
        kd = host["k"].to(dev, non_blocking=True)
        vd = host["v"].to(dev, non_blocking=True)
        od, _, _ = mala.mala_fwd(qd, kd, vd, TAU, TILE, TILE, with_mask=False)
        o_h.copy_(od, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_s = e0.elapsed_time(e1) / 1e3

    peaks = _peaks()
    kern_s = statistics.mean(fwd_times)
    achieved = fwd_flops / kern_s / 1e12
    peak = peaks["bf16_tflops_sustained"]
    res = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic, seeded (gqa_32k recipe: diffuse / local / retrieval head thirds)",
        "config": {"workload": WORKLOAD, "batch": B, "heads_q": Hq, "heads_kv": Hkv, "seqlen": N,
                   "head_dim": d, "block_q": TILE, "block_k": TILE, "tau": TAU, "pass": "fwd",
                   "l2": "inputs (0.4 GB) larger than L2; no flush"},
        "fwd": {"ms": kern_s * 1e3, "tflops_executed": achieved, "tiles_tested": tested,
                "tiles_kept": kept, "kept_fraction": kept / tested,
                "slots_per_query": slots / (B * Hq * N)},
        "tau0": {"ms_per_step": dense_s * 1e3, "tokens_per_s": B * N * world / dense_s,
                 "tflops_executed": tile_flops(d) * (d_tested + d_kept) / dense_s / 1e12},
        "roofline": {"bound": "tensor", "kernel": "mala_fwd_tc_kernel<128>", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peaks['source']} bf16_tflops_sustained",
                     "traffic": None},
        "e2e": {"value": B * N * args.steps / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def _oracle_sample(budget_s: float):
    """Time the fp64 oracle on a seeded random sample of query blocks of the
    bench workload; returns (rows processed, seconds, blocks)."""
    import numpy as np
    from oracle import mala_oracle as orc
    from tile_skipping_causal_b200 import synth

    w = synth.WORKLOADS[WORKLOAD]
    t = synth.make_prefill(w, SEED)
    q, k, v = t["q"], t["k"], t["v"]
    N, G = w.seqlen, w.group
    rng = np.random.default_rng(0)
    rows = 0
    t0 = time.perf_counter()
    nb = 0
    while time.perf_counter() - t0 < budget_s:
        h = int(rng.integers(0, w.heads_q))
        i = int(rng.integers(0, N // TILE))
        Q = q[0, i * TILE:(i + 1) * TILE, h].double().numpy()
        K = k[0, :, h // G].double().numpy()
        V = v[0, :, h // G].double().numpy()
        st = orc.forward_block(Q, np.arange(i * TILE, (i + 1) * TILE), K, V, TILE, TAU,
                               orc.causal_tiles((i + 1) * TILE - 1, TILE, N // TILE))
        orc.finalize(st)
        rows += TILE
        nb += 1
    return rows, time.perf_counter() - t0, nb


def _threads():
    try:
        import threadpoolctl
        return max(i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()) or 1
    except Exception:
        return 1


def cpu_baseline(seconds: float = 15.0):
    rows, secs, nb = _oracle_sample(seconds)
    return {"value": rows / secs, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
            "sample": f"{nb} random query blocks (128 rows, all their causal key tiles) of the "
                      f"{WORKLOAD} workload at tau={TAU}, forward, fp64 numpy, {secs:.1f} s"}


def run_reference(args):
    world, rank, _ = _dist_init()
    if rank != 0:
        return
    per = []
    for _ in range(args.warmup):
        _oracle_sample(1.0)
    rows_total, secs_total = 0, 0.0
    for _ in range(args.steps):
        r, s, _ = _oracle_sample(args.cpu_seconds / max(args.steps, 1))
        rows_total += r
        secs_total += s
        per.append(s)
    value = rows_total / secs_total
    res = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs_total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic, seeded (gqa_32k recipe)",
        "config": {"workload": WORKLOAD, "batch": 1, "heads_q": 32, "heads_kv": 8, "seqlen": 32768,
                   "head_dim": 128, "block_q": TILE, "block_k": TILE, "tau": TAU, "pass": "fwd"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": _threads(), "kind": "oracle",
                         "sample": f"{args.steps} steps of random 128-row query blocks, "
                                   f"{secs_total:.1f} s total"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["mala", "reference"], default="mala")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="shrink N (same recipe); for profiling captures only")
    ap.add_argument("--no-extras", action="store_true",
                    help="time the step only (no tau=0, e2e, baseline); for profiling captures")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_mala(args)


if __name__ == "__main__":
    main()
