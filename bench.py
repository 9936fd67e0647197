#!/usr/bin/env python
"""Benchmark: one LSA attention layer in prefill (index build + key selection +
exact sparse attention) on the 1,048,576-token workload, on N GPUs.

Each GPU processes its own independent layer instance (same recipe, seed
offset by rank): weak scaling with no data-path collective.  Timing: W
untimed warm-up steps, then K steps between CUDA events on the launching
stream, bracketed by barrier + synchronize, max over ranks.  Inputs stay
resident in HBM and are larger than L2 (Q alone is 4 GiB).

Prints ONE JSON line on rank 0.  `--impl reference` times the CPU oracle
instead (bounded sample, scaled to the whole layer).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
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

METRIC = "LSA prefill tokens/s per layer (index+select+attn) at 1M ctx; % of roofline"
UNIT = "tokens/s"
# The CPU oracle's bounded sample, the same for the bench's cpu_baseline and
# for every step of the reference arm: one Lloyd round timed on every 8th
# block, select + attention on 128 sampled queries.
CPU_SAMPLE_QUERIES = 128
CPU_LLOYD_STRIDE = 8


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill_1m")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=16,
                    help="query chunks of the end-to-end pipeline (each chunk's O goes down while the next computes)")
    ap.add_argument("--cpu-sample-queries", type=int, default=CPU_SAMPLE_QUERIES)
    ap.add_argument("--query-range", default=None,
                    help="START:COUNT - profiling case: full index, select+attention on that query range only")
    return ap.parse_args()


# ------------------------------------------------------------------ plumbing
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a host float over ranks (timing only; not a data-path exchange)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every interval_ms (200 ms
    by default; short timed regions ask for a shorter interval)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, interval_ms: int = 200):
        self.gpu = gpu_index
        self.interval_ms = interval_ms
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        """Start sampling and wait (3 s at most) for the first sample, so that
        the timed region that follows is covered from its start."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.interval_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t_end = time.time() + 3.0
        while not self.lines and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        loaded = [s for s, p in zip(sm, power) if p > 200] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_sha(fnames: str) -> str:
    """sha256[:16] of the kernel's source files ("a.cu+b.cuh": concatenated in that order)."""
    h = hashlib.sha256()
    for fname in fnames.split("+"):
        with open(os.path.join(ROOT, "hierarchical_latent_key_gemm_b200", "csrc", fname), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, src: str):
    """DRAM bytes per launch recorded from an ncu capture (profiles/traffic.txt),
    or None when absent or when the kernel source changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    sha = kernel_source_sha(src)
    with open(p) as f:
        for line in f:
            if line.startswith("#") or "|" not in line:
                continue
            parts = [x.strip() for x in line.split("|")]
            if len(parts) >= 5 and parts[0] == kernel and parts[1] == workload and parts[2] == src:
                return int(parts[4]) if parts[3] == sha else None
    return None


def run_config(w, world: int, seed: int) -> dict:
    """The workload description both arms print (the reference arm runs the
    same workload on the host cores of rank 0)."""
    from hierarchical_latent_key_gemm_b200.workloads import describe
    return {"workload": describe(w), "global_batch": w.batch * world, "seq_len": w.n_tokens,
            "parallelism": f"dp{world} (one independent layer instance per GPU)",
            "l2": "inputs larger than L2 (Q 4 GiB, K and V 0.5 GiB each); no flush needed", "seed": seed}


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    from hierarchical_latent_key_gemm_b200 import lsa
    from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, describe, input_bytes, make_inputs

    w = WORKLOADS[args.workload]
    lsa.lib()
    if w.decode_steps:
        return run_decode(args, w, rank, world, dev)
    seed = args.seed + 1000 * rank
    inp = make_inputs(w, seed=seed, device=dev)
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W"]
    N = w.n_tokens
    dt = lsa.LSA_BF16 if w.dtype == "bf16" else lsa.LSA_F32
    bp = lsa.make_build_params(w.batch, N, N, w.hkv, w.d, w.r, w.pool, dt, w.level_sizes, w.lloyd_iters,
                               w.grid_log2, w.sink, 0)
    sp = lsa.make_select_params(w.hq, w.beam, w.topk, w.sink, w.window)
    max_sel = w.max_sel
    q0, nq = 0, N
    if args.query_range:
        q0, nq = (int(x) for x in args.query_range.split(":"))
        Q = Q[:, q0:q0 + nq].contiguous()
        inp["Q"] = Q
        torch.cuda.empty_cache()
    idx = torch.empty((w.batch, nq, w.hkv, max_sel), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.batch, nq, w.hkv), dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    lse = torch.empty((w.batch, nq, w.hq), dtype=torch.float32, device=dev)

    def step(ev=None):
        if ev:
            ev[0].record()
        ix = lsa.lsa_build_index(bp, K, W)
        if ev:
            ev[1].record()
        lsa.lsa_select(ix, sp, Q, idx=idx, cnt=cnt, max_sel=max_sel, q_pos0=q0)
        if ev:
            ev[2].record()
        lsa.lsa_sparse_attn_banded(Q, K, V, idx, cnt, w.hkv, w.sink, w.window, q_pos0=q0, O=O, lse=lse)
        if ev:
            ev[3].record()
        return ix

    for _ in range(args.warmup):
        step().free()
    torch.cuda.synchronize()
    st = lsa.lsa_check(None)
    if st != lsa.LSA_OK:
        raise SystemExit(f"device error after warm-up: {lsa.strerror(st)}")

    clocks = ClockSampler(local)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    launches0 = lsa.lsa_launch_count()
    t0.record()
    for k in range(args.steps):
        step(evs[k]).free()
    t1.record()
    torch.cuda.synchronize()
    launches = lsa.lsa_launch_count() - launches0
    clk = clocks.stop()
    barrier(world)
    ms_local = t0.elapsed_time(t1)
    ms = max_over_ranks(ms_local, world, dev)
    ms_step = ms / args.steps
    value = world * N * w.batch / (ms_step / 1e3)

    build_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    select_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)

    peaks = measured_peaks()
    # Work counts for the rooflines, taken outside the timed region on the
    # same inputs: the tree nodes and candidate blocks select scored, and the
    # selection sizes.
    ix = lsa.lsa_build_index(bp, K, W)
    _, _, nodes, blocks = lsa.lsa_select_work(ix, sp, Q, idx=idx, cnt=cnt, max_sel=max_sel, q_pos0=q0)
    ix.free()
    torch.cuda.synchronize()
    sel_tokens = int(cnt.sum(dtype=torch.int64).item())
    stages = stage_rooflines(w, inp, bp, dev, peaks, build_ms, select_ms, attn_ms, nodes, blocks, sel_tokens,
                             q0, nq)
    sel = stages["select"]
    roofline = {"bound": "hbm", "kernel": ("select_kernel<64, tree> (select stage: query latents, dense-level scores, "
                                           "leaf tiles, select)"),
                "achieved": sel["achieved_GBps"], "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": sel["frac"],
                "traffic": recorded_traffic("select_kernel<64, tree>", w.name, "select.cu+select_common.cuh"),
                "algorithmic_bytes_per_launch": sel["algorithmic_bytes"], "peak_source": peaks["source"],
                "note": sel["formula"]}

    if args.query_range:
        # profiling case: report the stages only
        print(json.dumps({"profile_case": args.query_range, "stages": stages, "gpu_launches_per_step":
                          launches / args.steps}), flush=True)
        return
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, inp, bp, sp, idx, cnt, O, lse, dev, world)

    extra = None
    if not args.no_extra and rank == 0:
        extra = run_extra(w, inp, bp, sp, dev, select_ms, idx, cnt)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_estimate(w, inp, args.cpu_sample_queries)

    # the other workloads, one after another on the same GPU (the prefill
    # buffers freed first): per-layer and per-step figures
    others = None
    if not args.no_extra and rank == 0:
        del idx, cnt, O, lse, inp, Q, K, V
        torch.cuda.empty_cache()
        others = run_other_workloads(dev, peaks)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": run_config(w, world, args.seed),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk, "stages": stages, "extra": extra, "workloads": others,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_decode(args, w, rank, world, dev):
    """Decode workload as the bench line (see decode_measure)."""
    from hierarchical_latent_key_gemm_b200.workloads import describe
    r = decode_measure(w, dev, args.seed + 1000 * rank, args.warmup, world, not args.no_extra and rank == 0)
    if rank == 0:
        print(json.dumps({
            "metric": "LSA decode ms per step (append + select + attention, all sequences) at 10M context",
            "value": r["ms_per_step"], "unit": "ms/step", "n_gpus": world, "steps": r["steps"],
            "warmup": r["warmup"], "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": {"workload": describe(w)}, "build_ms": r["build_ms"],
            "index_device_bytes": r["index_device_bytes"], "gpu_launches": r["gpu_launches"],
            "status": r["status"], "clocks": r["clocks"], "extra": r["extra"]}), flush=True)


def decode_measure(w, dev, seed, warmup, world=1, extra=True):
    """Decode workload: build the index over every sequence's context (timed
    once), then time decode steps: append the new token's key, select for the
    new query, attend; one step covers all sequences of the batch."""
    import torch
    from hierarchical_latent_key_gemm_b200 import lsa
    from hierarchical_latent_key_gemm_b200.workloads import make_inputs
    inp = make_inputs(w, seed=seed, device=dev)
    K, V, Q, W = inp["K"], inp["V"], inp["Q"], inp["W"]
    N = w.n_tokens
    bp = lsa.make_build_params(w.batch, N, N + w.decode_steps, w.hkv, w.d, w.r, w.pool, lsa.LSA_BF16,
                               w.level_sizes, w.lloyd_iters, w.grid_log2, w.sink, w.decode_steps)
    sp = lsa.make_select_params(w.hq, w.beam, w.topk, w.sink, w.window)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lsa.lsa_build_index(bp, K, W).free()  # warm-up build
    torch.cuda.synchronize()
    e0.record()
    ix = lsa.lsa_build_index(bp, K, W)
    e1.record()
    torch.cuda.synchronize()
    build_ms = e0.elapsed_time(e1)
    qs = [Q[:, s:s + 1].contiguous() for s in range(w.decode_steps)]
    # decode through the public decode path: the append as a call, select +
    # attention replayed from the CUDA graph captured at set-up (pipeline.DecodeStep)
    from hierarchical_latent_key_gemm_b200.pipeline import DecodeStep
    c0 = lsa.lsa_launch_count()
    ds = DecodeStep(ix, sp, K, V, w.hq, w.max_sel)
    per_replay = (lsa.lsa_launch_count() - c0) // 2     # set-up ran select + attention eagerly once, then captured

    def step(s):
        ds.step(qs[s], N + s)

    warm = min(warmup, w.decode_steps // 4)
    for s in range(warm):
        step(s)
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank(), interval_ms=20)   # the timed region lasts ~20 ms
    clocks.start()
    launches0 = lsa.lsa_launch_count()
    e0.record()
    for s in range(warm, w.decode_steps):
        step(s)
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    n_timed = w.decode_steps - warm
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / n_timed
    # appends launch as calls; every replay runs the captured select + attention kernels
    launches = lsa.lsa_launch_count() - launches0 + n_timed * per_replay
    st = lsa.lsa_check(ix)
    info = ix.info()
    del ds
    ext = decode_extra(w, inp, ix, sp, dev) if extra else None
    ix.free()
    del inp, qs
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "steps": n_timed, "warmup": warm, "build_ms": build_ms,
            "index_device_bytes": int(info.device_bytes), "gpu_launches": launches, "status": lsa.strerror(st),
            "clocks": clk, "extra": ext}


def decode_extra(w, inp, ix, sp, dev):
    """Not timed in the headline: after the decode steps, every decode query
    (all steps x sequences, each at its own position; later appends hold only
    blocks past its causal bound, so its selection is the one it had) is
    selected at once by the tree and by the full-scan indexer over the whole
    10M-token context: their times for that batch, the tree's recall of the
    full scan's long-range picks on a sample, and needle hit rates."""
    import torch
    from hierarchical_latent_key_gemm_b200 import lsa
    N, S = w.n_tokens, w.decode_steps
    Q = inp["Q"]
    qpos = (N + torch.arange(S, device=dev, dtype=torch.int64))[None, :].repeat(w.batch, 1).contiguous()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = {}
    for name, fn in (("tree", lsa.lsa_select), ("fullscan", lsa.lsa_fullscan_select)):
        fn(ix, sp, Q, q_pos=qpos)       # warm-up
        torch.cuda.synchronize()
        e0.record()
        sel = fn(ix, sp, Q, q_pos=qpos)
        e1.record()
        torch.cuda.synchronize()
        out[name] = (e0.elapsed_time(e1), sel)
    (t_ms, (ti, tc)), (f_ms, (fi, fc)) = out["tree"], out["fullscan"]
    ti, tc, fi, fc = ti.cpu(), tc.cpu(), fi.cpu(), fc.cpu()
    hit = tot = 0
    for b in range(w.batch):
        for h in range(w.hkv):
            for s in range(0, S, 8):
                i = N + s
                lo = max(0, i - w.window + 1)
                base = set(range(min(w.sink, lo))) | set(range(lo, i + 1))
                f = set(fi[b, s, h, : fc[b, s, h]].tolist()) - base
                t = set(ti[b, s, h, : tc[b, s, h]].tolist()) - base
                tot += len(f)
                hit += len(f & t)
    needles = inp["needles"]
    nh_t = nh_f = 0
    for (b, h, p, qp) in needles:
        s = qp - N
        nh_t += int(p in set(ti[b, s, h, : tc[b, s, h]].tolist()))
        nh_f += int(p in set(fi[b, s, h, : fc[b, s, h]].tolist()))
    return {"queries": w.batch * S, "tree_select_ms": t_ms, "fullscan_select_ms": f_ms,
            "tree_vs_fullscan_speedup": f_ms / t_ms, "tree_recall_vs_fullscan_topk": hit / max(1, tot),
            "recall_sample": "every 8th decode step, all sequences",
            "needle_hit_rate_tree": nh_t / max(1, len(needles)),
            "needle_hit_rate_fullscan": nh_f / max(1, len(needles)), "needles": len(needles)}


def local_rank() -> int:
    return int(os.environ.get("LOCAL_RANK", "0"))


def run_e2e(args, w, inp, bp, sp, idx, cnt, O, lse, dev, world):
    """Same metric through the public API with HOST buffers: every step copies
    Q, K, V, W from pinned host memory and reads O back
    (hierarchical_latent_key_gemm_b200.pipeline.HostPrefill: K, W up, index
    build while V and then Q go up (Q in --e2e-chunks chunks), select + banded attention
    per chunk, each O chunk back while the next computes)."""
    import torch
    from hierarchical_latent_key_gemm_b200.pipeline import HostPrefill
    hQ = inp["Q"].cpu().pin_memory()
    hK = inp["K"].cpu().pin_memory()
    hV = inp["V"].cpu().pin_memory()
    hW = inp["W"].cpu().pin_memory()
    hO = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
    hp = HostPrefill(bp, sp, hQ, hK, hV, hW, hO, w.sink, w.window, chunks=args.e2e_chunks, device=dev)

    n = max(1, min(args.steps, 3))
    hp.run().free()
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(n):
        hp.run().free()
    t1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev) / n
    return {"value": world * w.n_tokens * w.batch / (ms / 1e3), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": hp.h2d_bytes, "d2h_bytes_per_step": hp.d2h_bytes,
            "pipeline": (f"3 streams; K, W up, then V during the build; Q up and O down in {args.e2e_chunks} chunks "
                         "overlapped with select + attention")}


def run_extra(w, inp, bp, sp, dev, select_ms, idx, cnt):
    """Not timed in the headline: full-scan indexer on a query sample (speedup
    and recall of the tree against exact full-scan top-K), needle hit-rates,
    index bytes."""
    import torch
    from hierarchical_latent_key_gemm_b200 import lsa
    Q, K = inp["Q"], inp["K"]
    N = w.n_tokens
    ix = lsa.lsa_build_index(bp, K, inp["W"])
    info = ix.info()
    # full-scan time: 8 runs of 4,096 consecutive queries, one in the middle
    # of every eighth of the sequence (the causal cost grows with the
    # position), timed in one call and scaled to all N queries
    runs = 8
    run_len = min(4096, max(1, N // (2 * runs)))
    tpos = torch.cat([torch.arange(run_len, device=dev) + (2 * j + 1) * N // (2 * runs) - run_len // 2
                      for j in range(runs)]).clamp_(0, N - 1).unique()
    tq = Q[:, tpos].contiguous()
    tqpos = tpos[None, :].repeat(w.batch, 1).contiguous()
    lsa.lsa_fullscan_select(ix, sp, tq, q_pos=tqpos)  # warm-up
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    lsa.lsa_fullscan_select(ix, sp, tq, q_pos=tqpos)
    e1.record()
    torch.cuda.synchronize()
    full_ms_sample = e0.elapsed_time(e1)
    full_ms_est = full_ms_sample * N / tpos.numel()
    del tq, tqpos
    # recall and needles: 2,048 queries spread over the sequence
    ns = 2048
    pos = torch.linspace(0, N - 1, ns, device=dev).round().to(torch.int64)
    pos = torch.unique(pos)
    qs = Q[:, pos].contiguous()
    qpos = pos[None, :].repeat(w.batch, 1).contiguous()
    fidx, fcnt = lsa.lsa_fullscan_select(ix, sp, qs, q_pos=qpos)
    tidx = idx[:, pos]
    tcnt = cnt[:, pos]

    def recall(sidx, scnt):
        """share of the exact full-scan long-range picks that a selection also made"""
        fi, fc, si, sc_ = fidx.cpu(), fcnt.cpu(), sidx.cpu(), scnt.cpu()
        hit = tot = 0
        for b in range(w.batch):
            for h in range(w.hkv):
                for k in range(pos.numel()):
                    i = int(pos[k])
                    lo = max(0, i - w.window + 1)
                    base = set(range(min(w.sink, lo))) | set(range(lo, i + 1))
                    f = set(fi[b, k, h, : fc[b, k, h]].tolist()) - base
                    t = set(si[b, k, h, : sc_[b, k, h]].tolist()) - base
                    tot += len(f)
                    hit += len(f & t)
        return hit / max(1, tot)

    tree_recall = recall(tidx, tcnt)
    needles = inp["needles"]
    nh_tree = nh_full = 0
    for (b, h, p, qp) in needles:
        row = idx[b, qp, h, : cnt[b, qp, h]]
        nh_tree += int((row == p).any().item())
    if needles:
        npos = torch.tensor([qp for (_, _, _, qp) in needles], device=dev)
        nq_ = Q[:, npos].contiguous()
        nqpos = npos[None, :].repeat(w.batch, 1).contiguous()
        nf, nfc = lsa.lsa_fullscan_select(ix, sp, nq_, q_pos=nqpos)
        for k, (b, h, p, qp) in enumerate(needles):
            nh_full += int((nf[b, k, h, : nfc[b, k, h]] == p).any().item())
    ix.free()
    # flat-vs-tree study: one level of the same leaf count, same beam, K, S, W
    flat = None
    if len(w.level_sizes) > 1:
        bpf = lsa.make_build_params(w.batch, N, N, w.hkv, w.d, w.r, w.pool,
                                    lsa.LSA_BF16 if w.dtype == "bf16" else lsa.LSA_F32, (w.level_sizes[-1],),
                                    w.lloyd_iters, w.grid_log2, w.sink, 0)
        e0.record()
        ixf = lsa.lsa_build_index(bpf, K, inp["W"])
        e1.record()
        torch.cuda.synchronize()
        flat_build_ms = e0.elapsed_time(e1)
        nfq = min(N, 131072)
        qf = Q[:, N - nfq:].contiguous()
        lsa.lsa_select(ixf, sp, qf, q_pos0=N - nfq)
        torch.cuda.synchronize()
        e0.record()
        lsa.lsa_select(ixf, sp, qf, q_pos0=N - nfq)
        e1.record()
        torch.cuda.synchronize()
        flat_ms_est = e0.elapsed_time(e1) * N / nfq
        fsi, fsc = lsa.lsa_select(ixf, sp, qs, q_pos=qpos)
        nh_flat = 0
        if needles:
            ff, ffc = lsa.lsa_select(ixf, sp, nq_, q_pos=nqpos)
            for k, (b, h, p, qp) in enumerate(needles):
                nh_flat += int((ff[b, k, h, : ffc[b, k, h]] == p).any().item())
        flat = {"leaves": w.level_sizes[-1], "build_ms": flat_build_ms,
                "select_ms_estimate": flat_ms_est, "select_sample_queries": nfq,
                "recall_vs_fullscan_topk": recall(fsi, fsc),
                "needle_hit_rate": nh_flat / max(1, len(needles))}
        ixf.free()
    # training-free PCA map (row f1): its time, and the tree's recall and needle
    # hits when the map replaces the seeded W (full scan in the same latent space)
    pca = None
    if w.d in (64, 128):
        e0.record()
        Wp, evp = lsa.lsa_pca_map(K, N, w.pool, w.r)
        e1.record()
        torch.cuda.synchronize()
        pca_ms = e0.elapsed_time(e1)
        ixp = lsa.lsa_build_index(bp, K, Wp)
        psi, psc = lsa.lsa_select(ixp, sp, qs, q_pos=qpos)
        pfi, pfc = lsa.lsa_fullscan_select(ixp, sp, qs, q_pos=qpos)
        nh_pca = 0
        if needles:
            pn, pnc = lsa.lsa_select(ixp, sp, nq_, q_pos=nqpos)
            for k, (b, h, p, qp) in enumerate(needles):
                nh_pca += int((pn[b, k, h, : pnc[b, k, h]] == p).any().item())
        fidx, fcnt = pfi, pfc          # recall() compares against this full scan
        pca = {"map_ms": pca_ms, "explained_top_r": float(evp.sum().item()),
               "tree_recall_vs_fullscan_topk": recall(psi, psc),
               "needle_hit_rate_tree": nh_pca / max(1, len(needles))}
        ixp.free()
    return {"fullscan_ms_estimate": full_ms_est, "fullscan_sample_queries": int(tpos.numel()),
            "fullscan_sample": f"{runs} runs of {run_len} consecutive queries, one in the middle of every "
                               f"eighth of the sequence, timed in one call, scaled to {N} queries",
            "pca_map": pca,
            "tree_select_ms": select_ms, "tree_vs_fullscan_speedup": full_ms_est / select_ms,
            "tree_recall_vs_fullscan_topk": tree_recall, "flat_vs_tree": flat,
            "needle_hit_rate_tree": nh_tree / max(1, len(needles)),
            "needle_hit_rate_fullscan": nh_full / max(1, len(needles)), "needles": len(needles),
            "index_device_bytes": int(info.device_bytes),
            "select_queries_per_s": N * w.batch * w.hkv / (select_ms / 1e3)}


# ------------------------------------------------------------------ stages
def time_ms(fn, reps: int = 3) -> float:
    """Median device time of fn() in ms (CUDA events on the current stream,
    one untimed call first)."""
    import torch
    fn()
    torch.cuda.synchronize()
    out = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1))
    return statistics.median(out)


def stage_rooflines(w, inp, bp, dev, peaks, build_ms, select_ms, attn_ms, nodes, blocks, sel_tokens, q0, nq):
    """Every stage against its roofline, on each stage's algorithmic work:
      a1 project + pool   HBM: K read (2 B per element) + latent keys written (r x 4 B per block)
      a5 query latent     HBM: Q read + latent queries written (r x 4 B per (query, KV head))
      a2 leaf k-means     tensor (bf16 dense peak): 2 x blocks x leaves x r flops per round
      select (a5-a8)      HBM: a5 + tree nodes scored x r x 2 B (a6) + candidate blocks scored
                          x r x 2 B (a7) + selected tokens x 4 B (a8)
      attention (a9)      tensor: |Sel| x d x 4 x G flops; also gathered K/V rows |Sel| x d x 2 x 2 B
    a1, a5 and a2 are timed alone here (their kernels, outside the step); select
    and attention are the step's own stage times."""
    import torch
    from hierarchical_latent_key_gemm_b200 import lsa
    K, Q, W = inp["K"], inp["Q"], inp["W"]
    if q0 or nq != Q.shape[1]:
        Q = Q[:, q0:q0 + nq].contiguous()
    N, P, r, d, G = w.n_tokens, w.pool, w.r, w.d, w.group
    units = w.batch * w.hkv
    nb = N // P
    L = w.level_sizes[-1]
    hbm, tf, tfs = peaks["hbm_gbs"], peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
    es = 2 if w.dtype == "bf16" else 4
    Kl = torch.empty((units, nb, r), dtype=torch.float32, device=dev)
    t_a1 = time_ms(lambda: lsa.lsa_project_pool(K, W, N, P, Kl=Kl))
    a1 = w.batch * N * w.hkv * d * es + units * nb * r * 4
    qbar = torch.empty((w.batch, nq, w.hkv, r), dtype=torch.float32, device=dev)
    t_a5 = time_ms(lambda: lsa.lsa_query_latent(Q, W, w.hkv, qbar=qbar))
    a5 = Q.numel() * es + qbar.numel() * 4
    t_a2 = time_ms(lambda: lsa.lsa_kmeans(Kl, L, w.lloyd_iters), reps=2)
    a2 = 2 * nb * L * r * w.lloyd_iters * units
    del Kl, qbar
    torch.cuda.empty_cache()
    a6, a7, a8 = nodes * r * 2, blocks * r * 2, sel_tokens * 4
    sel_bytes = a5 + a6 + a7 + a8
    sel_gbs = sel_bytes / (select_ms / 1e3) / 1e9
    attn_flops = sel_tokens * d * 4 * G
    attn_bytes = sel_tokens * d * 2 * 2
    attn_tf = attn_flops / (attn_ms / 1e3) / 1e12
    # the projections also do d x r fused multiply-adds per mean row on CUDA cores: their fp32 rate
    # against the peak from unit counts and clock (SMs x 128 FP32 lanes x 2 flops x 1.965 GHz)
    fp32_peak = torch.cuda.get_device_properties(dev).multi_processor_count * 128 * 2 * 1.965e9 / 1e12
    a1_fl = units * nb * d * r * 2
    a5_fl = w.batch * nq * w.hkv * d * r * 2

    def alu(fl, ms):
        return {"flops": fl, "achieved_TFLOPs": fl / (ms / 1e3) / 1e12, "peak_TFLOPs": fp32_peak,
                "frac": fl / (ms / 1e3) / 1e12 / fp32_peak,
                "note": "fp32 FMA work of the projection of the mean rows; peak from SM count x 128 lanes x "
                        "2 flops x 1.965 GHz"}
    return {
        "build": {"ms": build_ms, "note": "a1 + a2 + upper levels + bucket layout, in the step"},
        "a1_project_pool": {"ms": t_a1, "bytes": a1, "achieved_GBps": a1 / (t_a1 / 1e3) / 1e9, "peak_GBps": hbm,
                            "frac": a1 / (t_a1 / 1e3) / 1e9 / hbm, "bound": "hbm", "alu": alu(a1_fl, t_a1)},
        "a5_query_latent": {"ms": t_a5, "bytes": a5, "achieved_GBps": a5 / (t_a5 / 1e3) / 1e9, "peak_GBps": hbm,
                            "frac": a5 / (t_a5 / 1e3) / 1e9 / hbm, "bound": "hbm", "alu": alu(a5_fl, t_a5)},
        "a2_leaf_kmeans": {"ms": t_a2, "flops": a2, "rounds": w.lloyd_iters,
                           "achieved_TFLOPs": a2 / (t_a2 / 1e3) / 1e12, "peak_TFLOPs": tf,
                           "frac": a2 / (t_a2 / 1e3) / 1e12 / tf, "bound": "tensor",
                           "note": "whole leaf k-means (assign on tensor cores + update + grouping) against the "
                                   "assign's dense flops; bf16 burst peak"},
        "select": {"ms": select_ms, "queries_per_s": nq * w.batch * w.hkv / (select_ms / 1e3),
                   "tree_nodes_scored": nodes, "candidate_blocks_scored": blocks, "selected_tokens": sel_tokens,
                   "bytes": {"a5_query_latent": a5, "a6_nodes": a6, "a7_blocks": a7, "a8_selection": a8},
                   "algorithmic_bytes": sel_bytes, "achieved_GBps": sel_gbs, "peak_GBps": hbm,
                   "frac": sel_gbs / hbm, "bound": "hbm",
                   "formula": ("(Q bytes + latent queries r x 4 B + tree nodes scored x r x 2 B + candidate "
                               "blocks scored x r x 2 B + selected tokens x 4 B) / select-stage time; the "
                               "latents stay L2-resident, so DRAM carries far fewer bytes (traffic)")},
        "attention": {"ms": attn_ms, "tokens_per_s": nq * w.batch / (attn_ms / 1e3), "selected_rows": sel_tokens,
                      "flops": attn_flops, "achieved_TFLOPs": attn_tf, "peak_TFLOPs": tfs,
                      "frac": attn_tf / tfs, "bound": "tensor",
                      "gathered_bytes": attn_bytes, "gathered_GBps": attn_bytes / (attn_ms / 1e3) / 1e9,
                      "gathered_frac_of_hbm": attn_bytes / (attn_ms / 1e3) / 1e9 / hbm,
                      "note": ("flops = |Sel| x d x 4 x G (QK and PV); bf16 sustained peak (timed inside the "
                               "step); gathered bytes = |Sel| x d x 2 B x 2 (K and V rows), mostly served by L2 "
                               "because neighbouring queries share rows, so they can exceed the HBM rate")},
    }


def _sampled_positions(w, count: int):
    import torch
    pos = torch.linspace(0, w.n_tokens - 1, count).round().to(torch.int64)
    return torch.unique(pos)


def _long_range(row, i, w):
    lo = max(0, i - w.window + 1)
    base = set(range(min(w.sink, lo))) | set(range(lo, i + 1))
    return set(row) - base


def recall_of(w, pos, fidx, fcnt, sidx, scnt) -> float:
    """Share of the exact full-scan long-range picks that a selection also made
    (rows at positions pos, every sequence and KV head)."""
    fi, fc, si, sc = fidx.cpu(), fcnt.cpu(), sidx.cpu(), scnt.cpu()
    hit = tot = 0
    for b in range(w.batch):
        for h in range(w.hkv):
            for k in range(pos.numel()):
                i = int(pos[k])
                f = _long_range(fi[b, k, h, : fc[b, k, h]].tolist(), i, w)
                t = _long_range(si[b, k, h, : sc[b, k, h]].tolist(), i, w)
                tot += len(f)
                hit += len(f & t)
    return hit / max(1, tot)


def recall_study(w, inp, dev, pool=None, sample: int = 2048) -> dict:
    """Tree selection against the exact full-scan top-K on the same data (one
    build, sampled queries, every KV head), and the planted needles' hit
    rates; `pool` overrides the workload's block size (same K, Q, W)."""
    import torch
    from hierarchical_latent_key_gemm_b200 import lsa
    P = pool or w.pool
    dt = lsa.LSA_BF16 if w.dtype == "bf16" else lsa.LSA_F32
    bp = lsa.make_build_params(w.batch, w.n_tokens, w.n_tokens, w.hkv, w.d, w.r, P, dt, w.level_sizes,
                               w.lloyd_iters, w.grid_log2, w.sink, 0)
    sp = lsa.make_select_params(w.hq, w.beam, w.topk, w.sink, w.window)
    ix = lsa.lsa_build_index(bp, inp["K"], inp["W"])
    pos = _sampled_positions(w, sample).to(dev)
    qs = inp["Q"][:, pos].contiguous()
    qpos = pos[None, :].repeat(w.batch, 1).contiguous()
    ti, tc = lsa.lsa_select(ix, sp, qs, q_pos=qpos)
    fi, fc = lsa.lsa_fullscan_select(ix, sp, qs, q_pos=qpos)
    rec = recall_of(w, pos.cpu(), fi, fc, ti, tc)
    needles = inp["needles"]
    nh_t = nh_f = 0
    if needles:
        npos = torch.tensor([qp for (_, _, _, qp) in needles], device=dev)
        nq_ = inp["Q"][:, npos].contiguous()
        nqpos = npos[None, :].repeat(w.batch, 1).contiguous()
        a, ac = lsa.lsa_select(ix, sp, nq_, q_pos=nqpos)
        f, fcn = lsa.lsa_fullscan_select(ix, sp, nq_, q_pos=nqpos)
        for k, (b, h, p, qp) in enumerate(needles):
            nh_t += int((a[b, k, h, : ac[b, k, h]] == p).any().item())
            nh_f += int((f[b, k, h, : fcn[b, k, h]] == p).any().item())
    ix.free()
    return {"pool": P, "sample_queries": int(pos.numel()), "tree_recall_vs_fullscan_topk": rec,
            "needle_hit_rate_tree": nh_t / max(1, len(needles)),
            "needle_hit_rate_fullscan": nh_f / max(1, len(needles)), "needles": len(needles)}


def layer_measure(w, dev, steps: int = 3, warmup: int = 2, seed: int = 0, inp=None) -> dict:
    """One prefill layer of workload w (build + select for every query +
    banded attention), stage times by CUDA events, mean over `steps`."""
    import torch
    from hierarchical_latent_key_gemm_b200 import lsa
    from hierarchical_latent_key_gemm_b200.workloads import describe, make_inputs
    if inp is None:
        inp = make_inputs(w, seed=seed, device=dev)
    Q, K, V, W = inp["Q"], inp["K"], inp["V"], inp["W"]
    N = w.n_tokens
    dt = lsa.LSA_BF16 if w.dtype == "bf16" else lsa.LSA_F32
    bp = lsa.make_build_params(w.batch, N, N, w.hkv, w.d, w.r, w.pool, dt, w.level_sizes, w.lloyd_iters,
                               w.grid_log2, w.sink, 0)
    sp = lsa.make_select_params(w.hq, w.beam, w.topk, w.sink, w.window)
    idx = torch.empty((w.batch, N, w.hkv, w.max_sel), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.batch, N, w.hkv), dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    lse = torch.empty((w.batch, N, w.hq), dtype=torch.float32, device=dev)

    def step(ev=None):
        if ev:
            ev[0].record()
        ix = lsa.lsa_build_index(bp, K, W)
        if ev:
            ev[1].record()
        lsa.lsa_select(ix, sp, Q, idx=idx, cnt=cnt, max_sel=w.max_sel)
        if ev:
            ev[2].record()
        lsa.lsa_sparse_attn_banded(Q, K, V, idx, cnt, w.hkv, w.sink, w.window, O=O, lse=lse)
        if ev:
            ev[3].record()
        return ix

    for _ in range(warmup):
        step().free()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for k in range(steps):
        step(evs[k]).free()
    torch.cuda.synchronize()
    st = lsa.lsa_check(None)
    b_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    s_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    a_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    layer = statistics.mean(e[0].elapsed_time(e[3]) for e in evs)
    del idx, cnt, O, lse
    return {"workload": describe(w), "layer_ms": layer, "tokens_per_s": N * w.batch / (layer / 1e3),
            "build_ms": b_ms, "select_ms": s_ms, "select_queries_per_s": N * w.batch * w.hkv / (s_ms / 1e3),
            "attn_ms": a_ms, "attn_tokens_per_s": N * w.batch / (a_ms / 1e3), "steps": steps, "warmup": warmup,
            "status": lsa.strerror(st)}


def run_other_workloads(dev, peaks) -> dict:
    """The other four workloads, measured after the headline one on the same
    GPU: per-layer prefill figures (and, for gqa_128k, the tree's recall and
    needle hits with the configured pooling and without pooling), and the
    decode step at 10M tokens x 4 sequences."""
    import torch
    from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, make_inputs
    out = {}
    for name in ("flat_4k_f32", "int_exact_16k", "gqa_128k"):
        w = WORKLOADS[name]
        inp = make_inputs(w, seed=0, device=dev)
        out[name] = layer_measure(w, dev, inp=inp)
        if name == "gqa_128k":
            out[name]["recall"] = [recall_study(w, inp, dev), recall_study(w, inp, dev, pool=1)]
        del inp
        torch.cuda.empty_cache()
    w = WORKLOADS["decode_10m_x4"]
    r = decode_measure(w, dev, 0, 3, 1, True)
    r.pop("clocks", None)
    out[w.name] = r
    return out


# ------------------------------------------------------------------ CPU oracle
def cpu_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 0) for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_oracle_estimate(w, inp, sample_queries: int, lloyd_stride: int = CPU_LLOYD_STRIDE) -> dict:
    """Time the oracle, as it stands, on a bounded sample of the workload and
    scale to one whole layer: latents of every block; one Lloyd round of one
    KV head over every lloyd_stride-th block against all leaf centroids
    (x lloyd_stride x rounds x heads: assignment cost is linear in the
    points); the upper tree levels in full; select + attention on sampled
    queries (x all queries x heads)."""
    import numpy as np
    import oracle as O
    K = inp["K"]
    Q = inp["Q"]
    V = inp["V"]
    Wm = inp["W"].double().cpu().numpy()
    N, G = w.n_tokens, w.group
    t_start = time.perf_counter()
    # latents (all heads)
    t = time.perf_counter()
    Kls = []
    Kh = []
    for h in range(w.hkv):
        kh = K[0, :N, h].float().cpu().numpy().astype(np.float64)
        Kh.append(kh)
        Kls.append(O.project_pool(kh, Wm, w.pool))
    t_lat = time.perf_counter() - t
    # one Lloyd round of head 0 on a strided sample of the blocks
    C0 = O.kmeans_init(Kls[0], w.level_sizes[-1])
    Xs = Kls[0][::lloyd_stride]
    t = time.perf_counter()
    lab_s, _ = O.kmeans_assign(Xs, C0)
    O.kmeans_update(Xs, lab_s, C0, w.grid_log2)
    t_round = (time.perf_counter() - t) * (Kls[0].shape[0] / Xs.shape[0])
    # the tree the query sample runs on: every block takes the label of its
    # stride group's sampled block (same bucket sizes as a real round, at no
    # extra assignment cost; not timed)
    lab = np.repeat(lab_s, lloyd_stride)[: Kls[0].shape[0]]
    C1 = O.kmeans_update(Kls[0], lab, C0, w.grid_log2)
    # upper levels in full, on the leaf centroids of that round
    t = time.perf_counter()
    cents = [None] * len(w.level_sizes)
    parents = [None] * len(w.level_sizes)
    cents[-1] = C1
    pts = C1
    for l in range(len(w.level_sizes) - 2, -1, -1):
        r = O.kmeans(pts, w.level_sizes[l], w.lloyd_iters, w.grid_log2)
        parents[l + 1] = r.labels
        cents[l] = r.centroids
        pts = r.centroids
    t_upper = time.perf_counter() - t
    tree = O.Tree(w.pool, w.sink, list(w.level_sizes), cents, parents, lab, [[]] * len(w.level_sizes)).finish()
    # select + attention on sampled queries
    rng = np.random.default_rng(0)
    rows = np.sort(rng.integers(w.sink + w.window + w.pool, N, sample_queries))
    Vh = V[0, :N, 0].float().cpu().numpy().astype(np.float64)
    t = time.perf_counter()
    for i in rows:
        q = Q[0, int(i), 0:G].float().cpu().numpy().astype(np.float64)
        qb = O.query_latent(q[None], Wm)[0]
        blk = O.select_blocks(tree, Kls[0], qb, int(i), w.beam, w.topk, w.window)
        sel = O.selection_tokens(blk, int(i), w.sink, w.window, w.pool)
        O.sparse_attention(q, Kh[0], Vh, sel)
    t_query = (time.perf_counter() - t) / len(rows)
    est = t_lat + t_round * w.lloyd_iters * w.hkv + t_upper * w.hkv + t_query * N * w.hkv * w.batch
    wall = time.perf_counter() - t_start
    return {"value": N * w.batch / est, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": (f"numpy fp64 oracle: latents of all {w.hkv} KV heads in full ({t_lat:.1f} s); one full-size "
                       f"Lloyd round of one KV head, timed on every {lloyd_stride}th block and scaled "
                       f"({t_round:.1f} s) x {w.lloyd_iters} rounds x {w.hkv} heads; "
                       f"upper levels in full ({t_upper:.1f} s) x {w.hkv}; select+attention on {len(rows)} "
                       f"sampled queries over a tree whose leaves take the sampled labels "
                       f"({t_query * 1e3:.1f} ms each) x {N} queries x {w.hkv} heads; "
                       f"estimated layer time {est:.0f} s from {wall:.0f} s of CPU work"),
            "estimated_layer_s": est}


def run_reference(args):
    import torch
    rank, world, local = dist_env()
    if rank != 0:
        return
    from hierarchical_latent_key_gemm_b200.workloads import WORKLOADS, describe, make_inputs
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    inp = make_inputs(w, seed=args.seed, device=dev)
    vals = []
    cpu = None
    for k in range(args.warmup + args.steps):
        r = cpu_oracle_estimate(w, inp, args.cpu_sample_queries)
        if k >= args.warmup:
            vals.append(r["value"])
            cpu = r
    value = statistics.mean(vals)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * w.n_tokens / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": run_config(w, world, args.seed),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu["cores"], "kind": "oracle",
                             "sample": cpu["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
