#!/usr/bin/env python
"""Benchmark: KV tokens compressed per second at the Llama-3.1-8B shape (64k context,
20 % kept), plus decode attention over the compressed cache in GB/s.

One step = the whole hot path over one sequence of synthetic inputs resident in
HBM: top-256 entropy of every logits row, representation change of every
(layer, token), window attention + InfoKV score of every (layer, KV head) row,
per-layer top-k selection, compaction of the kept K/V, and one decode-attention
step (all layers) over the compressed cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); every rank compresses its own
independent sequence (weak scaling, no collective on the data path); the time
is the max over ranks of device-timed CUDA events.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV tokens compressed/s (8B shape, 64k, 20% kept); decode-attn GB/s vs HBM peak"


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs: NVML every
    2 ms from a thread, so that a region of a few tens of milliseconds still gets dozens of
    samples; nvidia-smi every 200 ms when NVML is not importable.  Reads only."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.out = None
        self.thread = None
        self.samples = []

    def _nvml_loop(self, nv, h, masks):
        while not self.halt.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                break
            self.samples.append((mhz, {nm for nm, m in masks if r & m}))
            self.halt.wait(0.002)

    def start(self):
        self.samples = []
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            masks = [(nm, getattr(nv, "nvmlClocksEventReason" + key)) for nm, key in
                     zip(self.NAMES, ("HwSlowdown", "HwThermalSlowdown", "SwThermalSlowdown", "SwPowerCap"))]
            self.halt = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h, masks), daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        self.out = tempfile.TemporaryFile(mode="w+")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)          # its first sample takes a moment
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.halt.set()
            self.thread.join(timeout=5)
            if not self.samples:
                return None
            reasons = set().union(*(r for _, r in self.samples))
            return {"sm_mhz": statistics.median(float(m) for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml, 2 ms"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.count(",") >= 6]
        sm, mx, reasons = [], 0.0, set()
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx = max(mx, float(r[1]))
            except ValueError:
                continue
            for nm, v in zip(self.NAMES, r[3:7]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, 200 ms"}


def profiled_traffic(kernel: str, units: int):
    """DRAM bytes per launch of `kernel` from the ncu record under profiles/, scaled by the
    units one launch processes; None when no record exists or the kernel's sources have
    changed since the counters were taken (the record keeps their sha256)."""
    root = os.path.dirname(os.path.abspath(__file__))
    pat = re.compile(r"^traffic-record: (\w+) ([0-9.]+) bytes per \w+, sources (\S+) sha256 ([0-9a-f]+)$")
    for f in sorted(glob.glob(os.path.join(root, "profiles", "*.md"))):
        for line in open(f):
            mt = pat.match(line.strip())
            if not mt or mt.group(1) != kernel:
                continue
            h = hashlib.sha256()
            try:
                for src in mt.group(3).split(","):
                    h.update(open(os.path.join(root, src), "rb").read())
            except OSError:
                return None
            return float(mt.group(2)) * units if h.hexdigest() == mt.group(4) else None
    return None


# ----------------------------------------------------------------------------- CPU oracle timing
#
# The fp64 oracle of the compression step, timed on every host core the process may use:
# one spawned worker process per core (one BLAS thread each).  Phase 1 computes the
# top-k entropy of row chunks and the representation change of each layer; phase 2
# (which needs every H and its layer's D) the window attention, InfoKV combination and
# top-k selection of each (layer, KV head) row.  Every worker draws its own units'
# synthetic inputs (same shapes and distributions as the GPU workload, per-unit seeds)
# before the timed region; a barrier starts each phase, and a phase's time runs from the
# first worker's start to the last worker's end.


def _oracle_unit_inputs(wl, n, unit, seed):
    """Synthetic inputs of one oracle unit (fp64 numpy), drawn on the CPU by synth."""
    import numpy as np
    from long_context_kv_obs_b200 import synth
    kind = unit[0]
    f = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    if kind == "H":
        _, r0, r1 = unit
        return f(synth.gen_logits(r1 - r0, wl.vocab, wl.dtype, seed * 7919 + r0, "cpu", wl.dominant_rows))
    if kind == "D":
        return f(synth.gen_hidden(2, n, wl.hidden, wl.dtype, seed * 7919 + unit[1], "cpu"))
    _, l = unit
    one = synth.gen_prefill(wl.scaled(n_layers=1, n=n), seed * 7919 + 100_000 + l, "cpu",
                            with_logits=False, with_hidden=False)
    return f(one.Qw[0]), f(one.K[0])


def _oracle_worker(rank, nproc, wl, n, seed, steps, barrier, q_in, q_out):
    import numpy as np
    from threadpoolctl import threadpool_limits
    from oracle import infokv as ik

    L, Hkv, G = wl.n_layers, wl.n_kv_heads, wl.group
    nch = max(nproc, L)
    bounds = [(n * c // nch, n * (c + 1) // nch) for c in range(nch)]
    units1 = [("H", r0, r1) for (r0, r1) in bounds if r1 > r0] + [("D", l) for l in range(L)]
    mine1 = units1[rank::nproc]
    mine2 = [("W", l) for l in range(L)][rank::nproc]
    with threadpool_limits(1):
        data = {u: _oracle_unit_inputs(wl, n, u, seed) for u in mine1 + mine2}
        k = ik.uniform_budgets(n, wl.rho, 1, wl.w)[0]
        for _ in range(steps):
            barrier.wait()
            t0 = time.perf_counter()
            res = {}
            for u in mine1:
                if u[0] == "H":
                    res[u] = ik.topk_entropy(data[u], wl.topk)
                else:
                    hid = data[u]
                    res[u] = ik.repr_change(hid[0], hid[1], wl.tau)
            t1 = time.perf_counter()
            q_out.put((rank, 1, t0, t1, res))
            H, Drows = q_in.get()
            barrier.wait()
            t2 = time.perf_counter()
            for u in mine2:
                Qw, K = data[u]
                _, P, _ = ik.entropy_scores(Drows[u[1]], H)
                S = np.stack([ik.combine(ik.window_attention(Qw[g * G:(g + 1) * G], K[g]), P, wl.alpha)
                              for g in range(Hkv)])
                if wl.sel_mode == "gqa_union":
                    ik.select_topk(ik.union_max(S), k, wl.w)
                else:
                    for g in range(Hkv):
                        ik.select_topk(S[g], k, wl.w)
            t3 = time.perf_counter()
            q_out.put((rank, 2, t2, t3, None))


def oracle_parallel_times(wl, n: int, steps: int, seed: int = 0, cores: int = 0):
    """Seconds per step of the fp64 oracle's compression step (entropy, representation
    change, window attention, combination, selection) on n tokens of workload wl, on
    `cores` worker processes (default: every core of this process's affinity set).
    Returns (list of step times, cores used)."""
    import multiprocessing as mp
    import numpy as np
    cores = cores or len(os.sched_getaffinity(0))
    L = wl.n_layers
    nproc = max(1, min(cores, max(L, 1) * 8))
    ctx = mp.get_context("spawn")           # never fork a process that has touched CUDA
    barrier = ctx.Barrier(nproc)
    q_out = ctx.Queue()
    q_in = [ctx.Queue() for _ in range(nproc)]
    procs = [ctx.Process(target=_oracle_worker, args=(r, nproc, wl, n, seed, steps, barrier, q_in[r], q_out),
                         daemon=True) for r in range(nproc)]
    for p in procs:
        p.start()
    times = []
    try:
        for _ in range(steps):
            H = np.zeros(n)
            D = np.zeros((L, n))
            t0, t1 = [], []
            for _ in range(nproc):
                _, ph, a, b, res = q_out.get(timeout=1800)
                t0.append(a)
                t1.append(b)
                for u, v in res.items():
                    if u[0] == "H":
                        H[u[1]:u[2]] = v
                    else:
                        D[u[1]] = v
            for r in range(nproc):
                q_in[r].put((H, D))
            t2, t3 = [], []
            for _ in range(nproc):
                _, ph, a, b, _ = q_out.get(timeout=1800)
                t2.append(a)
                t3.append(b)
            times.append((max(t1) - min(t0)) + (max(t3) - min(t2)))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.terminate()
    return times, nproc


def run_reference(args, wl, rank, world):
    """The oracle as the reference arm: rank 0 times it on every host core, one bounded
    sample of the workload per step."""
    if rank != 0:
        return
    n_sample = args.cpu_tokens
    times, cores = oracle_parallel_times(wl, n_sample, args.warmup + args.steps, seed=2)
    t = sum(times[args.warmup:])
    value = args.steps * n_sample / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(wl, world),
            "cpu_baseline": {"kind": "oracle", "cores": cores, "value": value, "unit": "tokens/s",
                             "sample": f"{wl.name} shape with n={n_sample} tokens per step "
                                       f"(fp64 oracle, {cores} worker processes, one BLAS thread each)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def bench_config(wl, world):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": wl.name, "n": wl.n, "layers": wl.n_layers, "q_heads": wl.n_q_heads,
            "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "vocab": wl.vocab, "hidden": wl.hidden,
            "kept": wl.rho, "window": wl.W, "recent": wl.w, "select": wl.sel_mode,
            "l2": "inputs larger than L2 (no flush needed)",
            "parallelism": f"dp{world} (independent sequences)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the merge / probe / recompress rows")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--n", type=int, default=0, help="override the context length (profiling runs)")
    ap.add_argument("--layers", type=int, default=0, help="override the layer count (profiling runs)")
    ap.add_argument("--cpu-tokens", type=int, default=8192,
                    help="tokens of the bounded sample the CPU oracle compresses per step")
    ap.add_argument("--lmhead-only", type=int, default=0, metavar="N",
                    help="time only kvc_lmhead_entropy at the 8B shape with N positions, print its row")
    ap.add_argument("--rows-only", default="", metavar="GROUPS",
                    help="run only these row groups (comma-separated: " + ", ".join(ROW_GROUPS) +
                    ") and print them, without the headline step")
    args = ap.parse_args()
    if args.rows_only:
        import torch
        only = set(args.rows_only.split(","))
        bad = only - set(ROW_GROUPS)
        if bad:
            ap.error(f"unknown row groups {sorted(bad)}")
        torch.cuda.set_device(0)
        hbm, _, _ = measured_peaks()
        print(json.dumps(measure_rows(torch, torch.device("cuda", 0), hbm, only=only)))
        return
    if args.lmhead_only:
        import torch
        from long_context_kv_obs_b200 import binding as B
        from long_context_kv_obs_b200 import synth
        torch.cuda.set_device(0)
        print(json.dumps(lmhead_entropy_row(torch, B, synth, torch.device("cuda", 0), n=args.lmhead_only)))
        return

    from long_context_kv_obs_b200 import dist as kdist
    rank, world, local_rank = kdist.rank_env()

    from long_context_kv_obs_b200 import synth
    wl = synth.WORKLOADS[args.config]
    if args.n:
        wl = wl.scaled(n=args.n)
    if args.layers:
        wl = wl.scaled(n_layers=args.layers)
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from long_context_kv_obs_b200 import binding as B

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=600), device_id=dev)

    L, Hq, Hkv, d, n, W = wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n, wl.W
    m = B.model(L, Hq, Hkv, d)
    inp = synth.gen_prefill(wl, seed=kdist.sequence_seed(1000, rank), device=dev)
    f32, i32 = torch.float32, torch.int32
    H = torch.empty(n, dtype=f32, device=dev)
    D = torch.empty(L, n, dtype=f32, device=dev)
    S = torch.empty(L, Hkv, n, dtype=f32, device=dev)
    Eb = torch.empty(L, dtype=f32, device=dev)
    kcap = wl.k_uniform
    k = torch.empty(L, dtype=i32, device=dev)
    idx = torch.empty(L, Hkv, kcap, dtype=i32, device=dev)
    Kc = torch.empty(L, Hkv, kcap, d, dtype=wl.dtype, device=dev)
    Vc = torch.empty_like(Kc)
    q = torch.randn(1, L, Hq, d, device=dev).to(wl.dtype)
    o = torch.empty(1, L, Hq, d, dtype=f32, device=dev)
    lens = torch.full((1, L), kcap, dtype=i32, device=dev)
    ws = {}

    def stages(inputs):
        logits, hidden, Qw, K, V = inputs
        return [
            ("entropy", lambda: ws.__setitem__("h", B.kvc_score(
                m, mode=B.SCORE_INFOKV, n=n, W=0, Qw=Qw, K=K, S=None, logits=logits, H_out=H,
                topk=wl.topk, workspace=ws.get("h")))),
            ("repr", lambda: ws.__setitem__("d", B.kvc_score(
                m, mode=B.SCORE_INFOKV, n=n, W=0, Qw=Qw, K=K, S=None, hidden=hidden, D_out=D,
                tau=wl.tau, workspace=ws.get("d")))),
            ("window_score", lambda: ws.__setitem__("s", B.kvc_score(
                m, mode=B.SCORE_INFOKV, n=n, W=W, Qw=Qw, K=K, S=S, H_in=H, H_strides=(0, 0), D_in=D,
                D_strides=(n, 0), alpha=wl.alpha, tau=wl.tau, Ebar=Eb, workspace=ws.get("s")))),
            ("select", lambda: ws.__setitem__("x", B.kvc_select(
                m, n=n, w=wl.w, S=S, k_out=k, idx=idx, budget_mode=B.BUDGET_UNIFORM, rho=wl.rho,
                workspace=ws.get("x")))),
            ("compact", lambda: B.kvc_compact(m, n=n, idx=idx, k=k, src_K=K, dst_K=Kc, src_V=V,
                                              dst_V=Vc)),
            ("decode", lambda: ws.__setitem__("o", B.kvc_decode_attn(
                m, q=q, K=Kc[None], V=Vc[None], lens=lens, max_len=kcap, o=o,
                workspace=ws.get("o")))),
        ]

    dev_inputs = (inp.logits, inp.hidden, inp.Qw, inp.K, inp.V)
    st = stages(dev_inputs)
    names = [s[0] for s in st]

    def run_step(events=None):
        for j, (_, fn) in enumerate(st):
            if events is not None:
                events[j].record()
            fn()
        if events is not None:
            events[len(st)].record()

    for _ in range(max(3, args.warmup)):
        run_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    K_ = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(st) + 1)] for _ in range(K_)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    sampler.start()
    launches0 = B.kvc_launch_count()
    t0.record()
    for i in range(K_):
        run_step(ev[i])
    t1.record()
    launches = B.kvc_launch_count() - launches0
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    ms = kdist.max_over_ranks(t0.elapsed_time(t1), dist, dev)
    stage_ms = {nm: sum(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K_)) / K_
                for j, nm in enumerate(names)}

    hbm, bf16_tf, peak_kind = measured_peaks()
    es = 2 if wl.dtype == torch.bfloat16 else 4
    kk = k.cpu()
    kept_total = int(kk.sum()) * Hkv
    alg_bytes = {
        "entropy": n * wl.vocab * es,
        "repr": L * n * wl.hidden * es,
        "window_score": L * Hkv * n * d * es,
        "compact": 2 * 2 * kept_total * d * es,
        "decode": 2 * kept_total * d * es,
    }
    dominant = max(("entropy", "repr"), key=lambda s: stage_ms[s])
    ach = alg_bytes[dominant] / (stage_ms[dominant] * 1e-3) / 1e9
    decode_gbs = alg_bytes["decode"] / (stage_ms["decode"] * 1e-3) / 1e9
    value = kdist.weak_throughput(world, n, K_, ms)
    # the compression step as a whole: its algorithmic bytes over the summed stage times
    comp_stages = ("entropy", "repr", "window_score", "select", "compact")
    comp_ms = sum(stage_ms[s_] for s_ in comp_stages)
    comp_bytes = sum(alg_bytes[s_] for s_ in comp_stages if s_ in alg_bytes)
    comp_gbs = comp_bytes / (comp_ms * 1e-3) / 1e9
    compression = {"stages": list(comp_stages), "ms": comp_ms, "bytes": comp_bytes, "gbs": comp_gbs,
                   "tokens_per_s": n / (comp_ms * 1e-3), "frac": comp_gbs / hbm, "peak": hbm,
                   "peak_kind": peak_kind, "frac_of_8tbs": comp_gbs / 8000.0}

    # ---------------------------------------------------------------- adaptive budgets, same inputs
    adaptive = None
    if rank == 0 and not args.no_rows and not (args.n or args.layers):
        adaptive = run_adaptive(torch, B, m, wl, inp, H, D, S, Eb, ws, K_, hbm)

    # ---------------------------------------------------------------- end to end through host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, torch, dev, inp, stages, names, n, world, dist, idx, k, kdist)

    cpu = None
    rows = None
    if rank == 0 and not args.no_rows and not (args.n or args.layers):
        del inp, st
        dev_inputs = None
        torch.cuda.empty_cache()
        rows = measure_rows(torch, dev, hbm, cpu_rows=not args.no_cpu and world == 1,
                            cpu_tokens=args.cpu_tokens)

    if rank == 0 and world == 1 and not args.no_cpu:
        n_sample = args.cpu_tokens
        times, cores = oracle_parallel_times(wl, n_sample, 1, seed=1)
        cpu = {"value": n_sample / times[0], "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{wl.name} shape (L={L}, Hq={Hq}, Hkv={Hkv}, vocab={wl.vocab}, "
                         f"hidden={wl.hidden}) with n={n_sample} tokens: fp64 oracle of entropy, "
                         f"representation change, window attention, combination and selection on "
                         f"{cores} worker processes (one BLAS thread each), {times[0]:.2f} s wall"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K_, "warmup": max(3, args.warmup), "ms_per_step": ms / K_,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": bench_config(wl, world),
            "roofline": {"bound": "hbm", "kernel": dominant, "achieved": ach, "peak": hbm,
                         "unit": "GB/s", "frac": ach / hbm,
                         "traffic": profiled_traffic(dominant, n if dominant == "entropy" else L * n),
                         "peak_kind": peak_kind},
            "compression": compression,
            "decode_attn": {"gbs": decode_gbs, "frac": decode_gbs / hbm, "ms": stage_ms["decode"],
                            "bytes": alg_bytes["decode"]},
            "stage_ms": stage_ms,
            "stage_gbs": {s_: alg_bytes[s_] / (stage_ms[s_] * 1e-3) / 1e9 for s_ in alg_bytes},
            "window_alu": window_alu(wl, stage_ms["window_score"], clocks),
            "gpu_launches": launches,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "adaptive": adaptive,
            "rows": rows,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


MUFU_EX2_PER_CLK_SM = 16   # ex2 results per clock per SM (sm_100a's MUFU; 15.9 measured)


def window_alu(wl, ms, clocks):
    """The window stage against its exponential roofline: both passes take one exp2 per
    (window row, key) of every (layer, KV head) row, 2 G W n L Hkv in all, and the MUFU
    gives MUFU_EX2_PER_CLK_SM of them per clock per SM (peak at the max SM clock)."""
    import torch
    exps = 2.0 * wl.group * wl.W * wl.n * wl.n_layers * wl.n_kv_heads
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    mhz = (clocks or {}).get("sm_max_mhz") or 1965.0
    peak = MUFU_EX2_PER_CLK_SM * sms * mhz * 1e6
    ach = exps / (ms * 1e-3)
    return {"bound": "alu", "unit": "exp2/s", "exps": exps, "achieved": ach, "peak": peak, "frac": ach / peak,
            "peak_kind": f"{MUFU_EX2_PER_CLK_SM} per clock per SM x {sms} SMs x {mhz:.0f} MHz"}


def run_adaptive(torch, B, m, wl, inp, H, D, S, Eb, ws, steps, hbm):
    """The same compression step with adaptive budgets k_l proportional to E-bar^(l) (same
    total B = L * floor(rho n)): score, adaptive select, compact; CUDA events per stage."""
    L, Hkv, d, n = wl.n_layers, wl.n_kv_heads, wl.head_dim, wl.n
    dev = inp.K.device
    ku = wl.k_uniform
    kcap = min(n, 2 * ku)
    k2 = torch.empty(L, dtype=torch.int32, device=dev)
    idx2 = torch.empty(L, Hkv, kcap, dtype=torch.int32, device=dev)
    Kc2 = torch.empty(L, Hkv, kcap, d, dtype=wl.dtype, device=dev)
    Vc2 = torch.empty_like(Kc2)
    wsa = {}

    def step():
        ws["h"] = B.kvc_score(m, mode=B.SCORE_INFOKV, n=n, W=0, Qw=inp.Qw, K=inp.K, S=None, logits=inp.logits,
                              H_out=H, topk=wl.topk, workspace=ws.get("h"))
        ws["d"] = B.kvc_score(m, mode=B.SCORE_INFOKV, n=n, W=0, Qw=inp.Qw, K=inp.K, S=None, hidden=inp.hidden,
                              D_out=D, tau=wl.tau, workspace=ws.get("d"))
        ws["s"] = B.kvc_score(m, mode=B.SCORE_INFOKV, n=n, W=wl.W, Qw=inp.Qw, K=inp.K, S=S, H_in=H,
                              H_strides=(0, 0), D_in=D, D_strides=(n, 0), alpha=wl.alpha, tau=wl.tau,
                              Ebar=Eb, workspace=ws.get("s"))
        wsa["x"] = B.kvc_select(m, n=n, w=wl.w, S=S, k_out=k2, idx=idx2, budget_mode=B.BUDGET_ADAPTIVE,
                                B_total=L * ku, Ebar=Eb, workspace=wsa.get("x"))
        B.kvc_compact(m, n=n, idx=idx2, k=k2, src_K=inp.K, dst_K=Kc2, src_V=inp.V, dst_V=Vc2)

    ms = _time_ms(torch, step, reps=steps)
    kl = k2.cpu()
    es = 2
    nbytes = n * wl.vocab * es + L * n * wl.hidden * es + L * Hkv * n * d * es + 2 * 2 * int(kl.sum()) * Hkv * d * es
    return {"workload": wl.name + "-adaptive", "ms": ms, "tokens_per_s": n / (ms * 1e-3),
            "B_total": L * ku, "k_min": int(kl.min()), "k_max": int(kl.max()), "bytes": nbytes,
            "gbs": nbytes / ms / 1e6, "frac": nbytes / ms / 1e6 / hbm}


def _time_ms(torch, fn, reps: int = 5) -> float:
    """Mean device time of fn() over reps calls, after one untimed call."""
    fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


ROW_GROUPS = ("lmhead", "config1", "selkv", "recompress", "decode_time_run", "decode_time_sparse",
              "recas_controller")


def measure_rows(torch, dev, hbm, cpu_rows: bool = False, cpu_tokens: int = 8192, only=None):
    """The rows of the path outside the headline step, each on its own workload and timed
    with CUDA events on the current stream:
      * config1_compression - score, select (GQA union) and compact at the Llama-3.2-3B
        16k shape, 40 % kept;
      * merge, rope_reposition, decode_bias, decode_probe - the SelKV 100k workload;
      * decode_loop - 256 decode steps with one K/V row appended per step, over the
        merged 100k cache and over the full one (their time ratio);
      * recompress - one decode-time recompression at the largest cache of the batch-8
        Qwen-7B-shaped workload;
      * decode_time_run - that workload run in full: 32768 generated tokens per sequence,
        recompression every 1024, the RECAS probe every 64 steps;
      * lmhead_entropy - H from the LM head's input at the 8B 64k shape, the logits never
        written (tensor-bound)."""
    from long_context_kv_obs_b200 import binding as B
    from long_context_kv_obs_b200 import pipeline, synth
    out = {}
    f32, i32 = torch.float32, torch.int32

    def want(group):
        return only is None or group in only

    if want("config1"):
        config1_rows(torch, B, pipeline, synth, dev, hbm, out, cpu_rows, cpu_tokens)
    if want("selkv"):
        selkv_rows(torch, B, pipeline, synth, dev, hbm, out)
    if want("recompress"):
        out["recompress"] = recompress_row(torch, B, pipeline, synth, dev, hbm)
    if want("decode_time_run"):
        out["decode_time_run"] = decode_time_run_row(torch, B, pipeline, synth, synth.WORKLOADS[4], dev, hbm)
    if want("decode_time_sparse"):
        out["decode_time_sparse"] = decode_time_sparse_row(torch, B, pipeline, synth, synth.WORKLOADS[4], dev, hbm)
    if want("recas_controller"):
        out["recas_controller"] = recas_controller_row(torch, B, pipeline, synth, synth.WORKLOADS[4], dev)
    # ---- InfoKV's H from the LM head's input (8B shape, 64k positions), last: seconds of
    # tensor work at the power cap leave the clocks low for the HBM-bound rows after it
    if want("lmhead"):
        out["lmhead_entropy"] = lmhead_entropy_row(torch, B, synth, dev)
    return out


def config1_rows(torch, B, pipeline, synth, dev, hbm, out, cpu_rows, cpu_tokens):
    """Score, select (GQA union) and compact at the Llama-3.2-3B 16k shape, 40 % kept."""

    # ---- Llama-3.2-3B 16k, 40 % kept, GQA union: the compression step
    wl = synth.WORKLOADS[1]
    inp = synth.gen_prefill(wl, seed=1001, device=dev)
    pc = pipeline.PrefillCompressor(wl, inp)
    ms = _time_ms(torch, pc.run)
    L, Hkv, d, n = wl.n_layers, wl.n_kv_heads, wl.head_dim, wl.n
    kept = int(pc.k.sum()) * Hkv
    nbytes = n * wl.vocab * 2 + L * n * wl.hidden * 2 + L * Hkv * n * d * 2 + 2 * 2 * kept * d * 2
    out["config1_compression"] = {"workload": wl.name, "ms": ms, "tokens_per_s": n / (ms * 1e-3),
                                  "bytes": nbytes, "gbs": nbytes / ms / 1e6, "frac": nbytes / ms / 1e6 / hbm}
    del pc, inp
    torch.cuda.empty_cache()
    if cpu_rows:
        n1 = min(wl.n, max(1024, cpu_tokens // 2))
        times, cores = oracle_parallel_times(wl, n1, 1, seed=1)
        out["config1_compression"]["cpu_baseline"] = {
            "value": n1 / times[0], "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{wl.name} shape with n={n1} tokens (fp64 oracle, {cores} worker processes)"}


def selkv_rows(torch, B, pipeline, synth, dev, hbm, out):
    """The SelKV 100k workload: merge, RoPE re-positioning, decode with the log R bias, the
    RECAS probe over the full history, and the 256-step decode loop."""
    i32 = torch.int32
    # ---- SelKV 100k: prefill scores (VATP, union), selection, merge
    wl = synth.WORKLOADS[3]
    L, Hq, Hkv, d, n = wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n
    inp = synth.gen_prefill(wl, seed=3000, device=dev, with_logits=False, with_hidden=False)
    pc = pipeline.PrefillCompressor(wl, inp, merge=True)
    pc.score()
    pc.select()
    pc.compact()
    kept = int(pc.k.sum()) * Hkv
    ms = _time_ms(torch, pc.do_merge)
    nbytes = L * Hkv * n * (d * 2 + 4) + kept * (d * 2 + 4)      # V and A read, V' and R written
    out["merge"] = {"workload": wl.name, "ms": ms, "gbs": nbytes / ms / 1e6, "frac": nbytes / ms / 1e6 / hbm,
                    "bytes": nbytes}

    # SelKV RoPE re-positioning of the kept keys (into a second buffer: the cache stays as it is)
    Kr = torch.empty_like(pc.Kc)
    ms = _time_ms(torch, lambda: B.kvc_rope_reposition(pc.m, K=pc.Kc, pos=pc.idx, k=pc.k,
                                                       base=wl.rope_base, K_dst=Kr))
    nbytes = kept * (2 * d * 2 + 4)                                   # K row read and written, position read
    out["rope_reposition"] = {"workload": wl.name, "ms": ms, "gbs": nbytes / ms / 1e6,
                              "frac": nbytes / ms / 1e6 / hbm, "bytes": nbytes}
    del Kr

    # decode step over the merged cache with the alpha_c log R bias
    kc = int(pc.k.max())
    q = synth.gen_decode_queries(wl.scaled(batch=1), seed=3001, step=0, device=dev)
    lens = pc.k.view(1, L).contiguous()
    att = pipeline.DecodeAttention(pc.m, 1, L, Hq, d, dev, probe=True, Hkv=Hkv)
    ms = _time_ms(torch, lambda: att(q, pc.Kc[None], pc.Vc[None], lens, kc, R=pc.R[None],
                                     alpha_c=wl.alpha_c))
    nbytes = kept * (2 * d * 2 + 4)
    out["decode_bias"] = {"workload": wl.name, "ms": ms, "gbs": nbytes / ms / 1e6,
                          "frac": nbytes / ms / 1e6 / hbm, "bytes": nbytes}

    # RECAS probe: the same step against the full cache, with the kept-position bits
    nwords = (n + 31) // 32
    acc = torch.zeros(L, Hkv, nwords, dtype=torch.int64, device=dev)
    for l in range(L):
        kl = int(pc.k[l])
        p64 = pc.idx[l, :, :kl].to(torch.int64)
        acc[l].scatter_add_(-1, p64 // 32, torch.ones_like(p64) << (p64 % 32))
    bits = torch.where(acc >= 2 ** 31, acc - 2 ** 32, acc).to(i32)[None].contiguous()
    lens_full = torch.full((1, L), n, dtype=i32, device=dev)
    full = (inp.K[None], inp.V[None], lens_full, n, bits)
    ms = _time_ms(torch, lambda: att(q, pc.Kc[None], pc.Vc[None], lens, kc, full=full))
    nbytes = kept * 2 * d * 2 + L * Hkv * n * 2 * d * 2
    out["decode_probe"] = {"workload": wl.name, "ms": ms, "gbs": nbytes / ms / 1e6,
                           "frac": nbytes / ms / 1e6 / hbm, "bytes": nbytes}
    del full, acc, bits
    out["decode_loop"] = decode_loop_row(torch, B, pipeline, synth, wl, pc, inp, dev, hbm)
    del pc, inp, att
    torch.cuda.empty_cache()


def recompress_row(torch, B, pipeline, synth, dev, hbm):
    """One decode-time recompression of the batch-8 Qwen-7B-shaped workload at its largest
    cache (t = n0 + 32 periods).  The cache's last W rows come from W decode steps (append,
    then attention over the cache), so the window queries' log-sum-exp ring is filled as in
    a run and the recompression takes the rows' softmax statistics from it (one pass over
    K); the same call recomputing them (two passes) is timed beside it."""
    i32 = torch.int32
    wl = synth.WORKLOADS[4]
    Bn, L, Hq, Hkv, d, n0, W = wl.batch, wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n, wl.W
    g = torch.Generator(device=dev).manual_seed(4000)
    Kp = torch.randn(Bn, L, Hkv, n0, d, device=dev, generator=g).to(wl.dtype)
    Vp = torch.randn(Bn, L, Hkv, n0, d, device=dev, generator=g).to(wl.dtype)
    Hp = torch.rand(Bn, n0, device=dev, generator=g) * 4
    Dp = torch.rand(Bn, L, n0, device=dev, generator=g) + 1.0
    dc = pipeline.DecodeTimeCompressor(wl, Kp, Vp, Hp, Dp)
    t = n0 + (wl.gen_tokens // wl.period) * wl.period
    ln = math.floor(wl.rho * (t - wl.period)) + wl.period     # cache length when it is due
    ln = min(ln, dc.cap)
    c = dc.cur
    m0 = ln - W                                               # rows before the window's steps
    dc.K[c, :, :, :, :m0] = torch.randn(Bn, L, Hkv, m0, d, device=dev, generator=g).to(wl.dtype)
    dc.V[c, :, :, :, :m0] = torch.randn(Bn, L, Hkv, m0, d, device=dev, generator=g).to(wl.dtype)
    dc.pos[c, :, :, :, :m0] = torch.sort(torch.randperm(t - W, device=dev, generator=g)[:m0])[0].to(i32)
    dc.Hs[c, :, :, :, :m0] = torch.rand(Bn, L, Hkv, m0, device=dev, generator=g) * 4
    dc.Ds[c, :, :, :, :m0] = torch.rand(Bn, L, Hkv, m0, device=dev, generator=g) + 1.0
    dc.len, dc.t, dc.generated = m0, t - W, 0
    dc.lens.fill_(m0)
    for s in range(W):
        q = synth.gen_decode_queries(wl, 4001, s, dev)
        k, v = synth.gen_decode_kv(wl, 4001, s, dev)
        dc.append(k, v, torch.rand(Bn, device=dev, generator=g) * 4,
                  torch.rand(Bn, L, device=dev, generator=g) + 1.0, q)
        dc.attend(q)
    assert dc.len == ln and dc.t == t and dc.lse_streak >= W

    def one(one_pass):
        def call():
            dc.cur, dc.len, dc.t = c, ln, t
            dc.lens.fill_(ln)
            dc.lse_streak = W if one_pass else 0
            dc.recompress()
        return call

    ms = _time_ms(torch, one(True))
    ms2 = _time_ms(torch, one(False))
    keep = max(min(wl.w, ln), min(ln, math.floor(wl.rho * t)))
    nbytes = Bn * L * Hkv * (ln * d * 2 + 2 * 2 * keep * d * 2)   # K scored, K and V kept rows moved
    # the window score takes one exp2 per (window row, cached key) and pass: the floor of the
    # step is that at the exp2 peak plus the bytes at the copy peak
    exps = 1.0 * wl.group * W * ln * Bn * L * Hkv
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    exp_peak = MUFU_EX2_PER_CLK_SM * sms * 1965e6
    floor_ms = exps / exp_peak * 1e3 + nbytes / hbm / 1e6
    row = {"workload": wl.name, "ms": ms, "tokens_per_s": Bn * ln / ms * 1e3,
           "cache_len": ln, "kept": keep, "gbs": nbytes / ms / 1e6,
           "frac": nbytes / ms / 1e6 / hbm, "bytes": nbytes,
           "window_stats": "log-sum-exp of each window query's own decode step (one pass over K)",
           "exps": exps, "floor_ms": floor_ms, "frac_of_floor": floor_ms / ms,
           "floor": "window exp2 at the MUFU peak plus the bytes at the copy peak",
           "two_pass": {"ms": ms2, "frac": nbytes / ms2 / 1e6 / hbm,
                        "floor_ms": 2 * exps / exp_peak * 1e3 + nbytes / hbm / 1e6}}
    del dc, Kp, Vp, Hp, Dp
    torch.cuda.empty_cache()
    return row


def lmhead_entropy_row(torch, B, synth, dev, reps: int = 3, n: int = 0):
    """H from the LM head's input at the 8B shape, 64k positions (Dh 4096, vocab 128256):
    kvc_lmhead_entropy (tcgen05 GEMM with the top-k epilogue, the logits never written),
    timed with CUDA events, against the roofline of its 2 n Dh V flops.  For context, the
    unfused pair it replaces: a library GEMM writing the bf16 logits, then the logits-row
    entropy kernel on them (kvc_score, signals only)."""
    wl = synth.WORKLOADS[2]
    n, Dh, V = n or wl.n, wl.hidden, wl.vocab
    x, W = synth.gen_lmhead(n, Dh, V, seed=2002, device=dev)
    H = torch.empty(n, device=dev)
    ws = B.kvc_lmhead_entropy(x=x, W=W, H=H)
    ms = _time_ms(torch, lambda: B.kvc_lmhead_entropy(x=x, W=W, H=H, workspace=ws), reps)
    flops = 2.0 * n * Dh * V
    _, peak, kind = measured_peaks()
    sustained = 1400.0
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pp):
        with open(pp) as f:
            sustained = float(json.load(f).get("bf16_tflops_sustained", sustained))
    tf = flops / ms / 1e9
    row = {"workload": wl.name + "-lmhead", "n": n, "Dh": Dh, "vocab": V, "k": 256, "ms": ms,
           "tokens_per_s": n / (ms * 1e-3), "flops": flops, "tflops": tf,
           "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                        "peak_kind": kind, "frac_of_sustained": tf / sustained},
           "workspace_bytes": ws.numel(), "logits_bytes_avoided": 2 * n * V * 2}
    del ws
    torch.cuda.empty_cache()
    m1 = B.model(1, 1, 1, 128)
    logits = torch.empty(n, V, dtype=torch.bfloat16, device=dev)
    Hz = torch.empty(n, device=dev)
    Qd = torch.zeros(1, 128, dtype=torch.bfloat16, device=dev)
    Kd = torch.zeros(1, 1, n, 128, dtype=torch.bfloat16, device=dev)
    wsz = {}

    def unfused():
        torch.matmul(x, W.t(), out=logits)
        wsz["s"] = B.kvc_score(m1, mode=B.SCORE_INFOKV, n=n, W=0, Qw=Qd, K=Kd, S=None, logits=logits, H_out=Hz,
                               workspace=wsz.get("s"))

    row["unfused_ms"] = _time_ms(torch, unfused, reps)
    row["unfused"] = "library GEMM to bf16 logits [n][V], then the logits-row entropy kernel"
    row["max_abs_diff_vs_unfused"] = float((H - Hz).abs().max())
    del logits, x, W, Kd
    torch.cuda.empty_cache()
    return row


def decode_loop_row(torch, B, pipeline, synth, wl, pc, inp, dev, hbm, steps: int = 256):
    """256 decode steps at batch 1, one random K/V row appended per step (R = 1 for it):
    over the merged cache (alpha_c log R bias) and over the full 100k cache (no bias).
    Each loop is timed whole (appends included) with CUDA events; its bytes are the K and
    V rows (and R) every step reads."""
    L, Hq, Hkv, d, n = wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n
    kc = int(pc.k.max())
    cap_c, cap_f = kc + steps, n + steps
    Kc = torch.empty(1, L, Hkv, cap_c, d, dtype=wl.dtype, device=dev)
    Vc = torch.empty_like(Kc)
    Kc[0, :, :, :kc] = pc.Kc[:, :, :kc]
    Vc[0, :, :, :kc] = pc.Vc[:, :, :kc]
    Rc = torch.ones(1, L, Hkv, cap_c, dtype=torch.float32, device=dev)
    Rc[0, :, :, :kc] = pc.R[:, :, :kc]
    Kf = torch.empty(1, L, Hkv, cap_f, d, dtype=wl.dtype, device=dev)
    Vf = torch.empty_like(Kf)
    Kf[0, :, :, :n] = inp.K
    Vf[0, :, :, :n] = inp.V
    w1 = wl.scaled(batch=1)
    qs = [synth.gen_decode_queries(w1, 3100, s_, dev) for s_ in range(steps)]
    kvs = [synth.gen_decode_kv(w1, 3100, s_, dev) for s_ in range(steps)]
    att = pipeline.DecodeAttention(pc.m, 1, L, Hq, d, dev)
    res = {}
    for name, K, V, R, base in (("compressed", Kc, Vc, Rc, pc.k.view(1, L)), ("full", Kf, Vf, None, None)):
        lens = (base.clone() if base is not None else torch.full((1, L), n, dtype=torch.int32, device=dev))
        l0 = kc if base is not None else n
        lens0 = lens.clone()
        att(qs[0], K, V, lens, l0 + steps, R=R, alpha_c=wl.alpha_c)       # workspace at its largest

        def loop():
            lens.copy_(lens0)
            for s_ in range(steps):
                B.kvc_append(pc.m, k=kvs[s_][0], v=kvs[s_][1], K=K, V=V, lens=lens, pos=n + s_,
                             side_R=R)
                att(qs[s_], K, V, lens, l0 + s_ + 1, R=R, alpha_c=wl.alpha_c)

        loop()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        loop()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
        rows = L * Hkv * (l0 + (steps + 1) / 2)             # mean cache rows read per step
        nbytes = rows * (2 * d * 2 + (4 if R is not None else 0))
        res[name] = {"ms_per_step": ms, "mean_cache_tokens": l0 + (steps + 1) / 2,
                     "gbs": nbytes / ms / 1e6, "frac": nbytes / ms / 1e6 / hbm}
    return {"workload": wl.name, "steps": steps, **res,
            "full_over_compressed": res["full"]["ms_per_step"] / res["compressed"]["ms_per_step"]}


def decode_time_sparse_row(torch, B, pipeline, synth, wl, dev, hbm, steps: int = 4096, pool: int = 64,
                           sparse=(0.293, 0.5, 0.5)):
    """RECAS dynamic sparse decode on the decode-time workload: a stated slice of the run (the
    first `steps` generated tokens of the batch of 8, recompression every 1024), every step
    decoded over the top ceil(kappa n) tokens of each row (kappa 0.293, the active share the
    RECAS page reports).  Per-step sparse decode timed with CUDA events; its algorithmic
    bytes are every cached key row (the query-key score), the active value rows, and the
    position and history of every cached token."""
    Bn, L, Hq, Hkv, d, n0 = wl.batch, wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n
    wl = wl.scaled(gen_tokens=steps)
    m = B.model(L, Hq, Hkv, d)
    g = torch.Generator(device=dev).manual_seed(4200)
    Kp = torch.randn(Bn, L, Hkv, n0, d, device=dev, generator=g).to(wl.dtype)
    Vp = torch.randn(Bn, L, Hkv, n0, d, device=dev, generator=g).to(wl.dtype)
    dc = pipeline.DecodeTimeCompressor(wl, Kp, Vp, torch.rand(Bn, n0, device=dev, generator=g) * 4,
                                       torch.rand(Bn, L, n0, device=dev, generator=g) + 1, sparse=sparse)
    del Kp, Vp
    ins = []
    for s_ in range(pool):
        q = synth.gen_decode_queries(wl, 4201, s_, dev)
        k, v = synth.gen_decode_kv(wl, 4201, s_, dev)
        ins.append((q, k, v))
    Hn = torch.rand(Bn, device=dev, generator=g) * 4
    Dn = torch.rand(Bn, L, device=dev, generator=g) + 1
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(1024)]
    dc.attend_sparse(ins[0][0])
    torch.cuda.synchronize()
    dense_bytes = sp_bytes = sp_ms = 0.0
    kappa = sparse[0]
    for s_ in range(steps):
        q, k, v = ins[s_ % pool]
        dc.append(k, v, Hn, Dn, q)
        e = ev[s_ % 1024]
        e[0].record()
        dc.attend_sparse(q)
        e[1].record()
        n = dc.len
        kt = min(n, max(1, math.ceil(kappa * n - 1e-12)))
        rows = Bn * L * Hkv
        sp_bytes += rows * (n * (d * 2 + 4 + 2 * 4) + kt * d * 2)
        dense_bytes += rows * n * 2 * d * 2
        if dc.due():
            dc.recompress()
        if s_ % 1024 == 1023:
            torch.cuda.synchronize()
            sp_ms += sum(x.elapsed_time(y) for x, y in ev)
    torch.cuda.synchronize()
    res = {"workload": wl.name, "slice_steps": steps, "kappa": kappa, "a_tr": sparse[1], "b_hi": sparse[2],
           "sparse_ms_per_step": sp_ms / steps, "gbs": sp_bytes / sp_ms / 1e6, "frac": sp_bytes / sp_ms / 1e6 / hbm,
           "bytes_vs_dense": sp_bytes / dense_bytes}
    del dc, ins
    torch.cuda.empty_cache()
    return res


def recas_controller_row(torch, B, pipeline, synth, wl, dev, steps: int = 2048, probe_every: int = 64,
                         pool: int = 64, eps: float = 0.5, alpha: float = 0.1):
    """The RECAS calibrated estimator and adaptive budget on a stated slice of the decode-time
    workload (the first `steps` generated tokens of the batch of 8): the exact dropped mass at
    a probe every 64 steps recalibrates the estimate; each recompression keeps the budget the
    controller derives for eps.  Reported: the budgets against floor(rho t), and the coverage
    of the upper bound - the share of probe measurements delta_h at or below the bound
    delta_bar of their row computed before that probe (the page's 1 - alpha target)."""
    Bn, L, Hq, Hkv, d, n0 = wl.batch, wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n
    wl = wl.scaled(gen_tokens=steps)
    G = Hq // Hkv
    g = torch.Generator(device=dev).manual_seed(4300)
    Kp = torch.randn(Bn, L, Hkv, n0, d, device=dev, generator=g).to(wl.dtype)
    Vp = torch.randn(Bn, L, Hkv, n0, d, device=dev, generator=g).to(wl.dtype)
    dc = pipeline.DecodeTimeCompressor(wl, Kp, Vp, torch.rand(Bn, n0, device=dev, generator=g) * 4,
                                       torch.rand(Bn, L, n0, device=dev, generator=g) + 1, probe=True,
                                       recas_eps=eps, recas_alpha=alpha)
    del Kp, Vp
    ins = [(synth.gen_decode_queries(wl, 4301, s_, dev),) + synth.gen_decode_kv(wl, 4301, s_, dev)
           for s_ in range(pool)]
    Hn = torch.rand(Bn, device=dev, generator=g) * 4
    Dn = torch.rand(Bn, L, device=dev, generator=g) + 1
    hits = torch.zeros((), device=dev)
    total = 0
    budgets = []
    for s_ in range(steps):
        q, k, v = ins[s_ % pool]
        dc.append(k, v, Hn, Dn, q)
        probe = s_ % probe_every == probe_every - 1
        dc.attend(q, probe=probe)
        if probe:
            if s_ >= 3 * probe_every:          # from the third probe on (the bound is +inf before any)
                bar = dc.delta_bar.repeat_interleave(G, dim=2)    # the bound before this probe
                hits += (dc.attn.delta <= bar).sum()
                total += dc.attn.delta.numel()
            dc.calibrate()
        if dc.due():
            t = dc.t
            keep = dc.recompress()
            budgets.append({"t": t, "floor_rho_t": math.floor(wl.rho * t), "budget": keep})
    torch.cuda.synchronize()
    st = B.recas_fields(dc.recas_state)
    res = {"workload": wl.name, "slice_steps": steps, "probe_every": probe_every, "eps": eps, "alpha": alpha,
           "budgets": budgets, "coverage": float(hits.item()) / max(1, total), "probe_measurements": total,
           "c_mean": float(st["c"].mean()), "q_mean": float(st["q"].mean())}
    del dc, ins
    torch.cuda.empty_cache()
    return res


def decode_time_run_row(torch, B, pipeline, synth, wl, dev, hbm, probe_every: int = 64, pool: int = 64):
    """The decode-time compression workload in full: batch of 8, 2048-token prompts, 32768
    generated tokens each.  Every step: H / D of the new token from its logits row and
    hidden states (kvc_score), append (kvc_append), decode over the compressed cache;
    every 64 steps the RECAS probe over the full history; every 1024 steps kvc_recompress
    to floor(rho t).  Per-step inputs cycle through a pool of 64 drawn steps.  Decode
    kernels are timed per step with CUDA events; the whole loop is timed too."""
    Bn, L, Hq, Hkv, d, n0 = wl.batch, wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n
    m = B.model(L, Hq, Hkv, d)
    Kp, Vp, Lp, Hp = synth.gen_prompt_batch(wl, 4100, device=dev)
    H0 = torch.empty(Bn, n0, device=dev)
    D0 = torch.empty(Bn, L, n0, device=dev)
    for b in range(Bn):
        B.kvc_score(m, mode=B.SCORE_INFOKV, n=n0, W=0, Qw=Kp[b, 0, 0], K=Kp[b], S=None, logits=Lp[b],
                    hidden=Hp[b], H_out=H0[b], D_out=D0[b])
    del Lp, Hp
    dc = pipeline.DecodeTimeCompressor(wl, Kp, Vp, H0, D0, probe=True)
    del Kp, Vp
    ins = []
    for s_ in range(pool):
        q = synth.gen_decode_queries(wl, 4101, s_, dev)
        k, v = synth.gen_decode_kv(wl, 4101, s_, dev)
        lg, hid = synth.gen_decode_signals(wl, 4101, s_, dev)
        ins.append((q, k, v, lg, hid.transpose(0, 1).contiguous()))
    Hn = torch.empty(Bn, device=dev)
    Dn = torch.empty(L, Bn, device=dev)
    nprobe = wl.gen_tokens // probe_every
    pr_delta = torch.zeros(nprobe, Bn, L, Hq, device=dev)
    pr_err = torch.zeros_like(pr_delta)
    pr_bound = torch.zeros_like(pr_delta)
    # events on the stream: around every decode, and around the signals and the append of every
    # SAMPLE-th step (two more records every step cost enough host time to slow the loop)
    SAMPLE = 16
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for _ in range(1024)]
    dec_ms, sig_ms, app_ms, nsamp, dec_bytes, re_ms, cache_sum = 0.0, 0.0, 0.0, 0, 0.0, [], 0
    re_ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    wsd = {}
    # the largest decode workspaces first (max_len is only a bound), so no step allocates
    T = n0 + wl.gen_tokens
    dc.attn(ins[0][0], dc.K[dc.cur], dc.V[dc.cur], dc.lens, dc.cap)
    dc.attn(ins[0][0], dc.K[dc.cur], dc.V[dc.cur], dc.lens, dc.cap, full=(dc.Kf, dc.Vf, dc.lens_full, T, dc.bits))
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = B.kvc_launch_count()
    a0.record()
    pi = 0
    for s_ in range(wl.gen_tokens):
        q, k, v, lg, hid = ins[s_ % pool]
        e = ev[s_ % 1024]
        sampled = s_ % SAMPLE == 0
        if sampled:
            e[0].record()
        wsd["s"] = B.kvc_score(m, mode=B.SCORE_INFOKV, n=Bn, W=0, Qw=q, K=k[None], S=None, logits=lg,
                               hidden=hid, H_out=Hn, D_out=Dn, workspace=wsd.get("s"))
        if sampled:
            e[1].record()
        dc.append(k, v, Hn, Dn.t(), q)
        probe = s_ % probe_every == probe_every - 1
        e[2].record()
        dc.attend(q, probe=probe)
        e[3].record()
        cache_sum += dc.len
        dec_bytes += Bn * L * Hkv * dc.len * 2 * d * 2
        if probe:
            pr_delta[pi].copy_(dc.attn.delta)
            pr_err[pi].copy_(dc.attn.err)
            pr_bound[pi].copy_(dc.attn.bound)
            pi += 1
            dec_bytes += Bn * L * Hkv * dc.t * 2 * d * 2        # the probe's full-history pass
        if dc.due():
            re_ev[0].record()
            dc.recompress()
            re_ev[1].record()
            re_ev[1].synchronize()
            re_ms.append(re_ev[0].elapsed_time(re_ev[1]))
        if s_ % 1024 == 1023:
            torch.cuda.synchronize()
            dec_ms += sum(x[2].elapsed_time(x[3]) for x in ev)
            sig_ms += sum(x[0].elapsed_time(x[1]) for x in ev[::SAMPLE])
            app_ms += sum(x[1].elapsed_time(x[2]) for x in ev[::SAMPLE])
            nsamp += len(ev[::SAMPLE])
    a1.record()
    torch.cuda.synchronize()
    launches = B.kvc_launch_count() - launches0
    total_ms = a0.elapsed_time(a1)
    steps = wl.gen_tokens
    ok = (pr_err[:pi] <= pr_bound[:pi] + 1e-5).float().mean().item()
    res = {"workload": wl.name, "steps": steps, "batch": Bn, "loop_ms_per_step": total_ms / steps,
           "decode_ms_per_step": dec_ms / steps, "signals_ms_per_step": sig_ms / max(1, nsamp),
           "append_ms_per_step": app_ms / max(1, nsamp), "phase_sample": f"signals and append timed on every {SAMPLE}th step",
           "decode_gbs": dec_bytes / dec_ms / 1e6,
           "decode_frac": dec_bytes / dec_ms / 1e6 / hbm, "mean_cache_tokens": cache_sum / steps,
           "recompressions": len(re_ms), "recompress_ms_mean": sum(re_ms) / max(1, len(re_ms)),
           "probes": pi, "probe_every": probe_every,
           "delta_mean": pr_delta[:pi].mean().item(), "delta_max": pr_delta[:pi].max().item(),
           "bound_mean": pr_bound[:pi].mean().item(), "bound_max": pr_bound[:pi].max().item(),
           "err_mean": pr_err[:pi].mean().item(), "err_max": pr_err[:pi].max().item(),
           "err_within_bound": ok, "kvc_launches": launches,
           "note": "decode time and bytes include the probe steps' full-history pass"}
    del dc, ins
    torch.cuda.empty_cache()
    return res


def run_e2e(args, torch, dev, inp, stages, names, n, world, dist, idx, k, kdist):
    """Same metric through the public API with inputs in pinned host memory (copied every step)."""
    tensors = [inp.logits, inp.hidden, inp.Qw, inp.K, inp.V]
    nbytes = sum(t.numel() * t.element_size() for t in tensors)
    try:
        with open("/proc/meminfo") as f:
            avail = next(int(l.split()[1]) * 1024 for l in f if l.startswith("MemAvailable"))
    except Exception:
        avail = 0
    # every rank must take the same branch: the timed region below has barriers
    if not kdist.all_ranks_agree(avail >= 1.25 * nbytes, dist, dev):
        return {"value": None, "unit": "tokens/s",
                "skipped": f"host RAM {avail / 1e9:.0f} GB < 1.25 x {nbytes / 1e9:.0f} GB of inputs on some rank"}
    host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in tensors]
    for h, t in zip(host, tensors):
        h.copy_(t)
    dev_bufs = tensors  # reuse the device buffers as the destination of every step's copy
    idx_h = torch.empty(idx.shape, dtype=idx.dtype, pin_memory=True)
    k_h = torch.empty(k.shape, dtype=k.dtype, pin_memory=True)
    st = stages(tuple(dev_bufs))

    def step():
        for h, dbuf in zip(host, dev_bufs):
            dbuf.copy_(h, non_blocking=True)
        for _, fn in st:
            fn()
        idx_h.copy_(idx, non_blocking=True)
        k_h.copy_(k, non_blocking=True)

    step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.e2e_steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = kdist.max_over_ranks(a.elapsed_time(b), dist, dev)
    return {"value": kdist.weak_throughput(world, n, args.e2e_steps, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": nbytes,
            "d2h_bytes_per_step": idx.numel() * 4 + k.numel() * 4}


if __name__ == "__main__":
    main()
