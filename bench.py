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
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.out = None

    def start(self):
        self.out = tempfile.TemporaryFile(mode="w+")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
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
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx = max(mx, float(r[1]))
            except ValueError:
                continue
            for nm, v in zip(names, r[3:7]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


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


def oracle_sample_time(wl, n_sample: int, seed: int = 0):
    """Time the fp64 oracle (one host thread) compressing a config-shaped sequence of n_sample tokens."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    from long_context_kv_obs_b200 import synth
    from oracle import infokv as ik
    from oracle import pipeline as op

    sw = wl.scaled(n=n_sample)
    inp = synth.gen_prefill(sw, seed=seed, device="cpu")
    f = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    logits, hidden, Qw, K = f(inp.logits), f(inp.hidden), f(inp.Qw), f(inp.K)
    with threadpool_limits(1):
        t0 = time.perf_counter()
        ref = op.prefill_scores(logits, hidden, Qw, K, G=sw.group, alpha=sw.alpha, tau=sw.tau,
                                topk=sw.topk)
        budgets = ik.uniform_budgets(sw.n, sw.rho, sw.n_layers, sw.w)
        op.prefill_select(ref["S"], budgets, sw.w, sw.sel_mode)
        dt = time.perf_counter() - t0
    return dt


def run_reference(args, wl, rank, world):
    """The oracle as the reference arm: rank 0 times it on bounded samples of the workload."""
    if rank != 0:
        return
    n_sample = 1024
    for _ in range(args.warmup):
        oracle_sample_time(wl, n_sample, seed=1)
    times = [oracle_sample_time(wl, n_sample, seed=2 + i) for i in range(args.steps)]
    t = sum(times)
    value = args.steps * n_sample / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "sample_tokens": n_sample},
            "cpu_baseline": {"kind": "oracle", "cores": 1, "value": value, "unit": "tokens/s",
                             "sample": f"{wl.name} shape with n={n_sample} tokens per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


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
    args = ap.parse_args()

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
    time.sleep(0.3)
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

    # ---------------------------------------------------------------- end to end through host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, torch, dev, inp, stages, names, n, world, dist, idx, k, kdist)

    cpu = None
    rows = None
    if rank == 0 and not args.no_rows and not (args.n or args.layers):
        rows = measure_rows(torch, dev, hbm)

    if rank == 0 and world == 1 and not args.no_cpu:
        n_sample = 2048
        t = oracle_sample_time(wl, n_sample)
        cpu = {"value": n_sample / t, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{wl.name} shape (L={L}, Hq={Hq}, Hkv={Hkv}, vocab={wl.vocab}, "
                         f"hidden={wl.hidden}) with n={n_sample} tokens, fp64, one thread"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K_, "warmup": max(3, args.warmup), "ms_per_step": ms / K_,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.name, "n": n, "layers": L, "q_heads": Hq, "kv_heads": Hkv,
                       "head_dim": d, "vocab": wl.vocab, "hidden": wl.hidden, "kept": wl.rho,
                       "window": W, "recent": wl.w, "select": wl.sel_mode,
                       "l2": "inputs larger than L2 (no flush needed)",
                       "parallelism": f"dp{world} (independent sequences)"},
            "roofline": {"bound": "hbm", "kernel": dominant, "achieved": ach, "peak": hbm,
                         "unit": "GB/s", "frac": ach / hbm,
                         "traffic": profiled_traffic(dominant, n if dominant == "entropy" else L * n),
                         "peak_kind": peak_kind},
            "decode_attn": {"gbs": decode_gbs, "frac": decode_gbs / hbm, "ms": stage_ms["decode"],
                            "bytes": alg_bytes["decode"]},
            "stage_ms": stage_ms,
            "stage_gbs": {s: alg_bytes[s] / (stage_ms[s] * 1e-3) / 1e9 for s in alg_bytes},
            "gpu_launches": launches,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "rows": rows,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


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


def measure_rows(torch, dev, hbm):
    """The rows of the path outside the compression step, each on its own workload and
    timed alone (CUDA events on the current stream): SelKV merge, decode with the log R
    bias over the merged cache and the RECAS probe (100k SelKV workload), and one
    decode-time recompression (batch-8 decode workload, largest cache); the SelKV RoPE
    re-positioning of the kept keys on the 100k workload."""
    from long_context_kv_obs_b200 import binding as B
    from long_context_kv_obs_b200 import pipeline, synth
    out = {}
    f32, i32 = torch.float32, torch.int32

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
    del pc, inp, att, full, acc, bits
    torch.cuda.empty_cache()

    # ---- decode-time recompression, batch 8, at the largest cache (t = n0 + 32 periods)
    wl = synth.WORKLOADS[4]
    Bn, L, Hq, Hkv, d, n0 = wl.batch, wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n
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
    dc.K[c, :, :, :, :ln] = torch.randn(Bn, L, Hkv, ln, d, device=dev, generator=g).to(wl.dtype)
    dc.V[c, :, :, :, :ln] = torch.randn(Bn, L, Hkv, ln, d, device=dev, generator=g).to(wl.dtype)
    dc.pos[c, :, :, :, :ln] = torch.sort(torch.randperm(t, device=dev, generator=g)[:ln])[0].to(i32)
    dc.Hs[c, :, :, :, :ln] = torch.rand(Bn, L, Hkv, ln, device=dev, generator=g) * 4
    dc.Ds[c, :, :, :, :ln] = torch.rand(Bn, L, Hkv, ln, device=dev, generator=g) + 1.0
    dc.Qring.copy_(torch.randn(dc.Qring.shape, device=dev, generator=g).to(wl.dtype))
    dc.qpos.copy_(torch.arange(t - wl.W, t, dtype=i32, device=dev).expand(Bn, wl.W))

    def one():
        dc.cur, dc.len, dc.t = c, ln, t
        dc.lens.fill_(ln)
        dc.recompress()

    ms = _time_ms(torch, one)
    keep = max(min(wl.w, ln), min(ln, math.floor(wl.rho * t)))
    nbytes = Bn * L * Hkv * (ln * d * 2 + 2 * 2 * keep * d * 2)   # K scored, K and V kept rows moved
    out["recompress"] = {"workload": wl.name, "ms": ms, "tokens_per_s": Bn * ln / ms * 1e3,
                         "cache_len": ln, "kept": keep, "gbs": nbytes / ms / 1e6,
                         "frac": nbytes / ms / 1e6 / hbm, "bytes": nbytes}
    return out


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
