"""Benchmark of the MALA hot path on synthetic data (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mala|reference]

Workload (per GPU): long-context GQA prefill, batch 1, 32 query heads, 8 KV
heads, N = 32768, d = 128, 128 x 128 tiles, bf16, causal, heads in thirds
(diffuse / local / retrieval), tau = 0.2. One step = one pass of the hot path
over that batch: the MALA forward, then the MALA backward (mask replay)
with dO ~ N(0, 1). Inputs (~0.7 GB) are larger than the 126 MB L2.

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
# the workload's other tau, and a larger one at which this synthetic data
# skips tiles (the skipped work then shows up as time), beside the headline tau
TAU_SWEEP = (0.02, 64.0)
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


# DRAM bytes per launch from ncu (dram__bytes_read.sum + dram__bytes_write.sum)
# on the kernel versions in this tree. Backward: one full-size launch of this
# workload. Decode: one launch at N_k = 8192, scaled to N_k = 131072 by the
# key/value bytes (read once, so traffic grows with N_k; the split partials
# are the same at both sizes). Set an entry to None when its kernel changes.
NCU_TRAFFIC = {
    "mala_bwd_tc_kernel": 9_435_351_552 + 4_808_597_504,
    # decode, bf16 cache: the N_k = 8192 launch read 2,148,169,472 B (K and V
    # 2,147,483,648 B) and wrote 6,148,608 B; K and V grow 16x at 131072
    "mala_decode_split_kernel@131072": 16 * 2_147_483_648 + (2_148_169_472 - 2_147_483_648) + 6_148_608,
    # decode, e4m3 cache: the N_k = 8192 launch read 1,074,353,408 B (K and V
    # 1,073,741,824 B) and wrote 6,011,904 B; K and V grow 16x at 131072
    "mala_decode_split_kernel@131072/e4m3": 16 * 1_073_741_824 + (1_074_353_408 - 1_073_741_824) + 6_011_904,
}


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of ``x`` over all ranks (the slowest rank's time); the
    value itself when no process group is running."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """Units all ranks processed per second of the slowest rank (weak scaling:
    every rank processes its own units_per_rank)."""
    return units_per_rank * world / seconds


def workload_config(B: int, Hq: int, Hkv: int, N: int, d: int) -> dict:
    """The "config" object of both arms' JSON lines (the same workload)."""
    return {"workload": WORKLOAD, "batch": B, "heads_q": Hq, "heads_kv": Hkv, "seqlen": N,
            "head_dim": d, "block_q": TILE, "block_k": TILE, "tau": TAU, "pass": "fwd+bwd",
            "l2": "inputs (0.7 GB) larger than L2; no flush"}


def tile_flops(d: int = 128, bq: int = TILE, bk: int = TILE) -> float:
    """FLOPs of one bq x bk x d tile matmul (2 per multiply-add)."""
    return 2.0 * bq * bk * d


def tc_fracs(tflops: float, peaks) -> dict:
    """Fractions of the measured dense bf16 peak: the burst figure (cuBLAS
    timed alone, the headline denominator) and the sustained one (cuBLAS
    looped for seconds under the power cap)."""
    return {"frac_of_peak": tflops / peaks["bf16_tflops"],
            "frac_of_sustained": tflops / peaks["bf16_tflops_sustained"]}


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
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stats = torch.zeros(4, dtype=torch.int64, device=dev)
    bstats = torch.zeros(4, dtype=torch.int64, device=dev)
    # mala_fwd: 1 launch; mala_bwd: pre-pass, main kernel, dQ conversion
    launches_per_step = 4

    def step(tau, st=None, bst=None, ev_f=None, ev_b=None):
        if ev_f is not None:
            ev_f[0].record(stream)
        mala.mala_fwd(q, k, v, tau, TILE, TILE, o=o, lse=lse, keep_mask=keep, stats=st)
        if ev_f is not None:
            ev_f[1].record(stream)
            ev_b[0].record(stream)
        mala.mala_bwd(q, k, v, o, do, lse, tau, keep, dq=dq, dk=dk, dv=dv, stats=bst)
        if ev_b is not None:
            ev_b[1].record(stream)

    # one measured step for the executed-work counts
    stats.zero_()
    bstats.zero_()
    step(TAU, stats, bstats)
    mala.check_device_error()
    tested, kept, slots = (int(x) for x in stats.cpu().tolist()[:3])
    b_visit, b_kept, b_slots = (int(x) for x in bstats.cpu().tolist()[:3])
    fwd_flops = tile_flops(d) * (tested + kept)
    bwd_flops = tile_flops(d) * (b_visit + 4 * b_kept)

    for _ in range(args.warmup):
        step(TAU)
    torch.cuda.synchronize()

    # per-launch kernel times with events on the launching stream
    mk = lambda: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    evf = [mk() for _ in range(args.steps)]
    evb = [mk() for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for s_ in range(args.steps):
            step(TAU, ev_f=evf[s_], ev_b=evb[s_])
        t1.record(stream)
        torch.cuda.synchronize()
    elapsed = t0.elapsed_time(t1) / 1e3
    mala.check_device_error()
    fwd_times = [a.elapsed_time(b_) / 1e3 for a, b_ in evf]
    bwd_times = [a.elapsed_time(b_) / 1e3 for a, b_ in evb]
    elapsed = max_over_ranks(elapsed, dev)
    ms_per_step = elapsed / args.steps * 1e3
    value = whole_job_rate(B * N * args.steps, world, elapsed)

    if args.no_extras:
        if rank == 0:
            print(json.dumps({"profile_case": True, "seqlen": N, "ms_per_step": ms_per_step}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return

    # the workload's other tau (0.02): same kernels, same accounting
    sweep = []
    for tau_x in TAU_SWEEP:
        stats.zero_()
        bstats.zero_()
        step(tau_x, stats, bstats)
        x_tested, x_kept, _ = (int(x) for x in stats.cpu().tolist()[:3])
        xb_visit, xb_kept, _ = (int(x) for x in bstats.cpu().tolist()[:3])
        torch.cuda.synchronize()
        ex0, ex1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_x = max(1, args.steps // 2)
        ex0.record(stream)
        for _ in range(n_x):
            step(tau_x)
        ex1.record(stream)
        torch.cuda.synchronize()
        x_s = max_over_ranks(ex0.elapsed_time(ex1) / 1e3 / n_x, dev)
        x_flops = tile_flops(d) * (x_tested + x_kept + xb_visit + 4 * xb_kept)
        sweep.append({"tau": tau_x, "ms_per_step": x_s * 1e3, "tokens_per_s": whole_job_rate(B * N, world, x_s),
                      "fwd_tiles_kept": x_kept, "bwd_tiles_kept": xb_kept,
                      "tflops_executed": x_flops / x_s / 1e12, "fwd_kept_fraction": x_kept / x_tested,
                      "bwd_kept_fraction": xb_kept / max(xb_visit, 1)})

    # dense comparison: the same kernels at tau = 0
    stats.zero_()
    bstats.zero_()
    step(0.0, stats, bstats)
    d_tested, d_kept, _ = (int(x) for x in stats.cpu().tolist()[:3])
    db_visit, db_kept, _ = (int(x) for x in bstats.cpu().tolist()[:3])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_dense = max(1, args.steps // 2)
    e0.record(stream)
    for _ in range(n_dense):
        step(0.0)
    e1.record(stream)
    torch.cuda.synchronize()
    dense_s = max_over_ranks(e0.elapsed_time(e1) / 1e3 / n_dense, dev)
    dense = {"o": o.clone(), "lse": lse.clone(), "dq": dq.clone(), "dk": dk.clone(), "dv": dv.clone()}
    dense_flops = tile_flops(d) * (d_tested + d_kept + db_visit + 4 * db_kept)

    # end to end through the public API with pinned host buffers: every step
    # copies its inputs in (Q, K, V, dO) and its output and gradients out
    # (O, dQ, dK, dV). The copies run double-buffered on two side streams
    # (one per direction), so that step k+1's inputs and step k-1's results
    # cross PCIe while step k computes; every step's own copies stay inside
    # the timed region.
    names_in, names_out = ("q", "k", "v", "do"), ("o", "dq", "dk", "dv")
    ins_d = [{n: torch.empty_like(host[n], device=dev) for n in names_in} for _ in range(2)]
    outs_d = [{n: torch.empty_like(x) for n, x in zip(names_out, (o, dq, dk, dv))} for _ in range(2)]
    outs_h = [{n: torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for n, x in zip(names_out, (o, dq, dk, dv))}
              for _ in range(2)]
    lse_d = [torch.empty_like(lse) for _ in range(2)]
    keep_d = [torch.empty_like(keep) for _ in range(2)]
    h2d = sum(host[n].numel() * host[n].element_size() for n in names_in)
    d2h = sum(x.numel() * x.element_size() for x in outs_h[0].values())
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]

    def copy_in(kstep):
        b_ = kstep % 2
        s_in.wait_event(comp_done[b_])            # step k-2 has finished with this input set
        with torch.cuda.stream(s_in):
            for n_ in names_in:
                ins_d[b_][n_].copy_(host[n_], non_blocking=True)
        h2d_done[b_].record(s_in)

    torch.cuda.synchronize()
    e0.record(stream)
    copy_in(0)
    for ks in range(args.steps):
        b_ = ks % 2
        if ks + 1 < args.steps:
            copy_in(ks + 1)
        stream.wait_event(h2d_done[b_])
        stream.wait_event(d2h_done[b_])           # step k-2's results have left this output set
        ti, to = ins_d[b_], outs_d[b_]
        mala.mala_fwd(ti["q"], ti["k"], ti["v"], TAU, TILE, TILE, o=to["o"], lse=lse_d[b_], keep_mask=keep_d[b_])
        mala.mala_bwd(ti["q"], ti["k"], ti["v"], to["o"], ti["do"], lse_d[b_], TAU, keep_d[b_],
                      dq=to["dq"], dk=to["dk"], dv=to["dv"])
        comp_done[b_].record(stream)
        s_out.wait_event(comp_done[b_])
        with torch.cuda.stream(s_out):
            for n_ in names_out:
                outs_h[b_][n_].copy_(to[n_], non_blocking=True)
        d2h_done[b_].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    mala.check_device_error()
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, dev)
    del ins_d, outs_d, outs_h, lse_d, keep_d

    # fidelity against the dense (tau = 0) run on the same inputs: the
    # retained share of each row's softmax mass is exp(z_mala - z_dense), so
    # the omitted mass is 1 minus it; relative L2 errors of O and gradients
    step(TAU)
    torch.cuda.synchronize()
    omitted = (1.0 - torch.exp(lse.double() - dense["lse"].double())).clamp_min(0.0)
    rel = lambda a_, b_: float((a_.double() - b_.double()).norm() / b_.double().norm())
    fidelity = {"omitted_mass_mean": float(omitted.mean()), "omitted_mass_max": float(omitted.max()),
                "o_rel_l2": rel(o, dense["o"]), "dq_rel_l2": rel(dq, dense["dq"]),
                "dk_rel_l2": rel(dk, dense["dk"]), "dv_rel_l2": rel(dv, dense["dv"])}
    del dense

    peaks = _peaks()
    chunk = bench_chunk(args, q, k, v, stream, peaks)
    grp = None if args.no_extras else bench_group_fwd(args, q, k, v, stream, peaks)
    dec = None if args.no_decode else bench_decode(args, dev, stream, peaks)
    dec8 = None if args.no_decode else bench_decode(args, dev, stream, peaks, e4m3=True)
    cfgs = None if args.no_configs else bench_configs(args, dev, stream, peaks)
    kern_f = statistics.mean(fwd_times)
    kern_b = statistics.mean(bwd_times)
    ach_f = fwd_flops / kern_f / 1e12
    ach_b = bwd_flops / kern_b / 1e12
    peak = peaks["bf16_tflops"]
    dom = ("mala_bwd (pre + mala_bwd_tc_kernel + dQ conversion)", ach_b) if kern_b >= kern_f \
        else ("mala_fwd_tc_kernel<128>", ach_f)
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
        "data": "synthetic, seeded (gqa_32k recipe: diffuse / local / retrieval head thirds; dO ~ N(0,1))",
        "config": workload_config(B, Hq, Hkv, N, d),
        "tflops_executed": (fwd_flops + bwd_flops) / (elapsed / args.steps / world) / 1e12,
        "fwd": {"ms": kern_f * 1e3, "tflops_executed": ach_f, **tc_fracs(ach_f, peaks),
                "tiles_tested": tested, "tiles_kept": kept, "kept_fraction": kept / tested,
                "slots_per_query": slots / (B * Hq * N)},
        "bwd": {"ms": kern_b * 1e3, "tflops_executed": ach_b, **tc_fracs(ach_b, peaks),
                "tiles_visited": b_visit, "tiles_kept": b_kept, "kept_fraction": b_kept / max(b_visit, 1),
                "slots_per_query": b_slots / (B * Hq * N)},
        "tau0": {"ms_per_step": dense_s * 1e3, "tokens_per_s": whole_job_rate(B * N, world, dense_s),
                 "tflops_executed": dense_flops / dense_s / 1e12},
        "speedup_vs_tau0": {str(x["tau"]): dense_s * 1e3 / x["ms_per_step"] for x in sweep} |
                           {str(TAU): dense_s / (elapsed / args.steps)},
        "fidelity_vs_tau0": fidelity,
        "tau_sweep": sweep,
        "roofline": {"bound": "tensor", "kernel": dom[0], "achieved": dom[1],
                     "peak": peak, "unit": "TFLOP/s", "frac": dom[1] / peak,
                     "peak_source": f"{peaks['source']} bf16_tflops (burst)",
                     "frac_of_sustained": dom[1] / peaks["bf16_tflops_sustained"],
                     "traffic": (NCU_TRAFFIC.get("mala_bwd_tc_kernel")
                                 if kern_b >= kern_f and N == 32768 else None),
                     "traffic_note": "ncu DRAM bytes of the mala_bwd_tc_kernel launch (bytes per launch)"},
        "e2e": {"value": whole_job_rate(B * N * args.steps, world, e2e_s), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    res["chunked_prefill"] = chunk
    if grp is not None:
        res["fwd_group_vote"] = grp
    if dec is not None:
        res["decode"] = dec
        res["decode_e4m3"] = dec8
    if cfgs is not None:
        res["configs"] = cfgs
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def bench_chunk(args, q, k, v, stream, peaks, chunk: int = 4096):
    """Chunked prefill: the forward of the last ``chunk`` queries of the
    workload against all of its keys (bottom-right causal alignment, query q
    at position q + N_k - N_q), on the same inputs. Executed FLOPs as for
    the full forward: every tested tile pays QK^T, every retained one PV."""
    import torch
    from tile_skipping_causal_b200 import mala

    Nk = k.shape[1]
    chunk = min(chunk, Nk // 2)           # shorter runs (--seqlen) take half of their queries
    qc = q[:, Nk - chunk:]
    stats = torch.zeros(4, dtype=torch.int64, device=q.device)
    o, lse, keep = mala.mala_fwd(qc, k, v, TAU, TILE, TILE, stats=stats)
    mala.check_device_error()
    tested, kept = (int(x) for x in stats.cpu().tolist()[:2])
    for _ in range(max(3, args.warmup)):
        mala.mala_fwd(qc, k, v, TAU, TILE, TILE, o=o, lse=lse, keep_mask=keep)
    torch.cuda.synchronize()
    n = max(5, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        mala.mala_fwd(qc, k, v, TAU, TILE, TILE, o=o, lse=lse, keep_mask=keep)
    e1.record(stream)
    torch.cuda.synchronize()
    mala.check_device_error()
    t = e0.elapsed_time(e1) / 1e3 / n
    flops = tile_flops(q.shape[3]) * (tested + kept)
    return {"seqlen_q": chunk, "seqlen_k": Nk, "tau": TAU, "ms": t * 1e3,
            "tokens_per_s": q.shape[0] * chunk / t, "tiles_tested": tested, "tiles_kept": kept,
            "tflops_executed": flops / t / 1e12, **tc_fracs(flops / t / 1e12, peaks)}


def bench_group_fwd(args, q, k, v, stream, peaks, taus=(TAU, 64.0)):
    """The forward of the workload with group-joint voting (the query heads
    of a KV head decide together per tile), and per-head voting beside it, at
    each tau: device time per call, tiles tested / kept per head, executed
    FLOPs as for the step's forward."""
    import torch
    from tile_skipping_causal_b200 import mala

    B, N, Hq, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    out = {}
    for tau in taus:
        row = {}
        for mode in ("group", "per_head"):
            gv = mode == "group"
            stats = torch.zeros(4, dtype=torch.int64, device=q.device)
            keep = mala.mala_fwd(q, k, v, tau, TILE, TILE, o=o, lse=lse, stats=stats, group_vote=gv)[2]
            mala.check_device_error()
            tested, kept = (int(x) for x in stats.cpu().tolist()[:2])
            for _ in range(max(3, args.warmup)):
                mala.mala_fwd(q, k, v, tau, TILE, TILE, o=o, lse=lse, keep_mask=keep, group_vote=gv)
            torch.cuda.synchronize()
            n = max(5, args.steps // 2)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                mala.mala_fwd(q, k, v, tau, TILE, TILE, o=o, lse=lse, keep_mask=keep, group_vote=gv)
            e1.record(stream)
            torch.cuda.synchronize()
            mala.check_device_error()
            t = e0.elapsed_time(e1) / 1e3 / n
            flops = tile_flops(d) * (tested + kept)
            row[mode] = {"ms": t * 1e3, "tiles_tested": tested, "tiles_kept": kept,
                         "kept_fraction": kept / tested, "tflops_executed": flops / t / 1e12,
                         **tc_fracs(flops / t / 1e12, peaks)}
        out[str(tau)] = row
    return out


def bench_decode(args, dev, stream, peaks, seqlen_k: int = 131072, e4m3: bool = False,
                 with_group: bool = True):
    """Split-KV decode on the largest decode workload (batch 64, 32 query
    heads, 8 KV heads, d = 128, bf16 cache of seqlen_k keys, tau = 0.05).
    The 34 GB cache is drawn on the device with the decode recipe (sink key,
    16 needles per sequence); with e4m3 it is then quantised to e4m3 codes
    (scale 1, 17 GB). HBM roofline on the bytes actually read: every K tile
    plus the V tiles some head retained, plus the queries and the split
    partials written and read back."""
    import torch
    from tile_skipping_causal_b200 import mala, synth

    w = synth.decode_workload(seqlen_k if args.decode_seqlen is None or seqlen_k != 131072 else args.decode_seqlen)
    q = synth.make_decode_query(w, SEED).to(dev)
    k, v = synth.fill_decode_cache(w, SEED, q.cpu(), dev, slices=[])
    if e4m3:
        k = k.to(torch.float8_e4m3fn)
        v = v.to(torch.float8_e4m3fn)
        torch.cuda.empty_cache()
    esz = k.element_size()
    stats = torch.zeros(4, dtype=torch.int64, device=dev)
    o, lse, keep, P = mala.mala_decode(q, k, v, w.tau, 128, 0, stats=stats)
    mala.check_device_error()
    tested, vread, kept_heads = (int(x) for x in stats.cpu().tolist()[:3])
    out = torch.empty_like(q)
    l2 = torch.empty((w.batch, w.heads_q), dtype=torch.float32, device=dev)
    km = torch.empty_like(keep)
    workspace = torch.empty(w.batch * w.heads_q * P * 129 * 4 + 256, dtype=torch.uint8, device=dev)

    def call():
        mala.mala_decode(q, k, v, w.tau, 128, P, o=out, lse=l2, keep_mask=km, workspace=workspace)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    n = max(5, args.steps // 2)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    mala.check_device_error()
    t = e0.elapsed_time(e1) / 1e3 / n
    group = None
    if with_group and not e4m3:
        # group-joint voting (one decision per key tile for the query heads of
        # a KV head) on the same cache
        gstats = torch.zeros(4, dtype=torch.int64, device=dev)
        mala.mala_decode(q, k, v, w.tau, 128, P, o=out, lse=l2, keep_mask=km, workspace=workspace,
                         stats=gstats, group_vote=True)
        for _ in range(3):
            mala.mala_decode(q, k, v, w.tau, 128, P, o=out, lse=l2, keep_mask=km, workspace=workspace,
                             group_vote=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n):
            mala.mala_decode(q, k, v, w.tau, 128, P, o=out, lse=l2, keep_mask=km, workspace=workspace,
                             group_vote=True)
        e1.record(stream)
        torch.cuda.synchronize()
        mala.check_device_error()
        tg = e0.elapsed_time(e1) / 1e3 / n
        gt, gv = (int(x) for x in gstats.cpu().tolist()[:2])
        group = {"ms": tg * 1e3, "tokens_per_s": w.batch / tg, "v_tiles_read": gv, "v_read_fraction": gv / gt}
    d = w.head_dim
    kbytes = w.batch * w.heads_kv * w.seqlen_k * d * esz
    vbytes = vread * 128 * d * esz
    other = w.batch * w.heads_q * d * 2 * 2 + (w.batch * w.heads_q * P * (d + 1) * 4 * 2 if P > 1 else 0)
    total = kbytes + vbytes + other
    gbs = total / t / 1e9
    del k, v
    torch.cuda.empty_cache()
    return {"workload": w.name, "cache": "e4m3" if e4m3 else "bf16", "batch": w.batch, "heads_q": w.heads_q,
            "heads_kv": w.heads_kv,
            "seqlen_k": w.seqlen_k, "tau": w.tau, "splits": P, "ms": t * 1e3,
            "tokens_per_s": w.batch / t, "tiles_tested": tested, "v_tiles_read": vread,
            "v_read_fraction": vread / tested, "head_tiles_kept_fraction": kept_heads / (tested * w.group),
            "bytes_read_per_call": kbytes + vbytes + w.batch * w.heads_q * d * 2,
            "roofline": {"bound": "hbm", "kernel": "mala_decode_split_kernel", "achieved": gbs,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                         "peak_source": f"{peaks['source']} hbm_gbs",
                         "traffic": NCU_TRAFFIC.get(f"mala_decode_split_kernel@{w.seqlen_k}" + ("/e4m3" if e4m3 else "")),
                         "traffic_note": "ncu DRAM bytes per launch, N_k = 8192 capture scaled by N_k"},
            "group_vote": group}


L2_FLUSH_BYTES = 256 << 20          # twice the 126 MB L2


def _time_flushed(fn, n: int, stream, flush) -> float:
    """Mean device time of ``fn`` over n calls, each preceded (outside its
    own CUDA events) by a write of a buffer larger than L2, so that no call
    finds the previous call's inputs in L2."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs) / 1e3


def bench_configs(args, dev, stream, peaks) -> dict:
    """Every benchmark configuration of the operator at its own taus, each
    beside tau = 0 (FullAttn) on the same inputs and kernels: device time,
    tokens/s, executed TFLOP/s (every tested tile pays QK^T, every retained
    one PV; the backward pays the recomputed S^T per visited tile and four
    matmuls per retained one), kept-tile fractions and post-score key slots
    per query (the pages' cost measure). Each timed call starts with L2
    flushed. Decoding: the decode workload at every cache length with its
    HBM roofline (the largest length is the separate "decode" entry)."""
    import torch
    from tile_skipping_causal_b200 import mala, synth

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    n = max(5, args.steps // 2)
    out = {}

    def prefill(name, taus, backward):
        w = synth.WORKLOADS[name]
        t = {k_: x.to(dev) for k_, x in synth.make_prefill(w, SEED, with_do=backward).items()}
        q, k, v = t["q"], t["k"], t["v"]
        B, N, Hq, d = q.shape
        fp32 = w.dtype == "fp32"
        bq, bk = w.block_q, w.block_k
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
        nKB = -(-N // bk)
        keep = torch.empty((B, Hq, -(-N // bq), mala.mask_words(nKB)), dtype=torch.int32, device=dev)
        if backward:
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        rows = []
        for tau in (0.0,) + tuple(x for x in taus if x != 0.0):
            st = torch.zeros(4, dtype=torch.int64, device=dev)
            bst = torch.zeros(4, dtype=torch.int64, device=dev)
            mala.mala_fwd(q, k, v, tau, bq, bk, o=o, lse=lse, keep_mask=keep, stats=st)
            if backward:
                mala.mala_bwd(q, k, v, o, t["do"], lse, tau, keep, dq=dq, dk=dk, dv=dv, stats=bst)
            mala.check_device_error()
            tested, kept, slots = (int(x) for x in st.cpu().tolist()[:3])
            fwd = lambda: mala.mala_fwd(q, k, v, tau, bq, bk, o=o, lse=lse, keep_mask=keep)
            for _ in range(3):
                fwd()
            tf = _time_flushed(fwd, n, stream, flush)
            ff = tile_flops(d, bq, bk) * (tested + kept)
            row = {"tau": tau, "fwd_ms": tf * 1e3, "fwd_tflops_executed": ff / tf / 1e12,
                   "fwd_tiles_tested": tested, "fwd_tiles_kept": kept, "fwd_kept_fraction": kept / tested,
                   "fwd_slots_per_query": slots / (B * Hq * N)}
            if not fp32:
                row.update({"fwd_" + k_: x for k_, x in tc_fracs(ff / tf / 1e12, peaks).items()})
            total = tf
            if backward:
                bv, bkp, bsl = (int(x) for x in bst.cpu().tolist()[:3])
                bwd = lambda: mala.mala_bwd(q, k, v, o, t["do"], lse, tau, keep, dq=dq, dk=dk, dv=dv)
                for _ in range(3):
                    bwd()
                tb = _time_flushed(bwd, n, stream, flush)
                bf = tile_flops(d) * (bv + 4 * bkp)
                row.update({"bwd_ms": tb * 1e3, "bwd_tflops_executed": bf / tb / 1e12,
                            "bwd_tiles_visited": bv, "bwd_tiles_kept": bkp,
                            "bwd_kept_fraction": bkp / max(bv, 1), "bwd_slots_per_query": bsl / (B * Hq * N)})
                row.update({"bwd_" + k_: x for k_, x in tc_fracs(bf / tb / 1e12, peaks).items()})
                total += tb
            mala.check_device_error()
            row["tokens_per_s"] = B * N / total
            rows.append(row)
        dense_ms = rows[0]["fwd_ms"] + rows[0].get("bwd_ms", 0.0)
        for r in rows:
            r["speedup_vs_tau0"] = dense_ms / (r["fwd_ms"] + r.get("bwd_ms", 0.0))
        out[name] = {"batch": B, "heads_q": Hq, "heads_kv": k.shape[2], "seqlen": N, "head_dim": d,
                     "block_q": bq, "block_k": bk, "dtype": w.dtype,
                     "pass": "fwd+bwd" if backward else "fwd", "per_tau": rows}
        if fp32:
            out[name]["note"] = "fp32 CUDA-core path (64 x 64 tiles); inputs fit in L2, which is flushed"
        del t, q, k, v, o
        torch.cuda.empty_cache()

    prefill("toy_fp32_512", synth.WORKLOADS["toy_fp32_512"].taus, False)
    prefill("prefill_4k", synth.WORKLOADS["prefill_4k"].taus, False)
    prefill("train_8k", synth.WORKLOADS["train_8k"].taus, True)
    del flush
    torch.cuda.empty_cache()
    if not args.no_decode:
        out["decode_sweep"] = [bench_decode(args, dev, stream, peaks, seqlen_k=nk, with_group=False)
                               for nk in synth.DECODE_SEQLENS if nk != 131072]
    return out


_ORACLE_INPUTS = {}


def _oracle_sample(budget_s: float):
    """Time the fp64 oracle on a seeded random sample of query blocks of the
    bench workload: for each sampled (head, query block) the forward over all
    its causal key tiles and the backward work of the same tiles (its dQ rows
    and its share of dK/dV). Returns (rows processed, seconds, blocks)."""
    import numpy as np
    from oracle import mala_oracle as orc
    from tile_skipping_causal_b200 import synth

    w = synth.WORKLOADS[WORKLOAD]
    if "t" not in _ORACLE_INPUTS:
        _ORACLE_INPUTS["t"] = synth.make_prefill(w, SEED, with_do=True)
    t = _ORACLE_INPUTS["t"]
    q, k, v, do = t["q"], t["k"], t["v"], t["do"]
    N, G = w.seqlen, w.group
    nb_ = N // TILE
    rng = np.random.default_rng(0)
    rows = 0
    t0 = time.perf_counter()
    nb = 0
    while time.perf_counter() - t0 < budget_s:
        h = int(rng.integers(0, w.heads_q))
        i = int(rng.integers(0, nb_))
        q0, q1 = i * TILE, (i + 1) * TILE
        Qh = q[0, :, h].double().numpy()
        K = k[0, :, h // G].double().numpy()
        V = v[0, :, h // G].double().numpy()
        st = orc.forward_block(Qh[q0:q1], np.arange(q0, q1), K, V, TILE, TAU,
                               orc.causal_tiles(q1 - 1, TILE, nb_))
        Ob, zb = orc.finalize(st)
        O = np.zeros_like(Qh)
        z = np.zeros(N)
        O[q0:q1], z[q0:q1] = Ob, zb
        fm = np.zeros((nb_, nb_), dtype=bool)
        fm[i, :i + 1] = [st["keep"][j] for j in range(i + 1)]
        orc.backward_head(Qh, K, V, O, do[0, :, h].double().numpy(), z, TILE, TILE, TAU, fm,
                          qblocks=[i])
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
            "sample": f"{nb} random query blocks (128 rows, forward over all their causal key tiles "
                      f"and the backward of the same tiles) of the {WORKLOAD} workload at tau={TAU}, "
                      f"fp64 numpy, {secs:.1f} s"}


def _reference_config() -> dict:
    from tile_skipping_causal_b200 import synth
    w = synth.WORKLOADS[WORKLOAD]
    return workload_config(w.batch, w.heads_q, w.heads_kv, w.seqlen, w.head_dim)


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
        "config": _reference_config(),
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
    ap.add_argument("--no-decode", action="store_true", help="skip the decode measurement")
    ap.add_argument("--decode-seqlen", type=int, default=None,
                    help="decode cache length (default 131072); for profiling captures")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode measurement (profiling captures)")
    ap.add_argument("--decode-e4m3", action="store_true",
                    help="with --decode-only: an e4m3 cache instead of bf16")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration measurements (prefill_4k, train_8k, decode sweep, toy)")
    ap.add_argument("--configs-only", action="store_true",
                    help="run only the per-configuration measurements")
    ap.add_argument("--group-only", action="store_true",
                    help="run only the group-joint voting forward measurement")
    ap.add_argument("--no-extras", action="store_true",
                    help="time the step only (no tau=0, e2e, baseline); for profiling captures")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        run_reference(args)
    elif args.group_only:
        import torch
        from tile_skipping_causal_b200 import mala, synth
        mala.load_library()
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        t = synth.make_prefill(synth.WORKLOADS[WORKLOAD], SEED, seqlen=args.seqlen)
        q, k, v = (t[n].to(dev) for n in ("q", "k", "v"))
        print(json.dumps(bench_group_fwd(args, q, k, v, torch.cuda.current_stream(), _peaks())), flush=True)
    elif args.configs_only:
        import torch
        from tile_skipping_causal_b200 import mala
        mala.load_library()
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps(bench_configs(args, dev, torch.cuda.current_stream(), _peaks())), flush=True)
    elif args.decode_only:
        import torch
        from tile_skipping_causal_b200 import mala
        mala.load_library()
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps(bench_decode(args, dev, torch.cuda.current_stream(), _peaks(), e4m3=args.decode_e4m3)),
              flush=True)
    else:
        run_mala(args)


if __name__ == "__main__":
    main()
