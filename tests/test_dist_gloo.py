"""The multi-process path on CPU: two gloo ranks exercise the plumbing the multi-GPU
benchmark uses (rank environment, per-rank sequences, max-over-ranks timing, agreement
on optional measurements, weak-scaling throughput).  No GPU: the compression itself is
per-sequence and is covered by the single-GPU parity tests."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_kv_obs_b200 import dist as D
from long_context_kv_obs_b200 import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, local = D.rank_env()
    dist.init_process_group("gloo", rank=r, world_size=w)
    try:
        dev = torch.device("cpu")
        # each rank compresses its own synthetic sequence
        wl = synth.WORKLOADS[0].scaled(n=128)
        inp = synth.gen_prefill(wl, seed=D.sequence_seed(1000, r), device="cpu", with_hidden=False)
        digest = torch.tensor([float(inp.logits.double().sum()), float(inp.K.double().sum())])
        gathered = [torch.zeros(2, dtype=torch.float64) for _ in range(w)]
        dist.all_gather(gathered, digest.double())
        # timing: the job's time is the slowest rank's
        ms = 10.0 + 5.0 * r
        job_ms = D.max_over_ranks(ms, dist, dev)
        # an optional measurement runs on every rank or on none
        agree_some = D.all_ranks_agree(r == 0, dist, dev)
        agree_all = D.all_ranks_agree(True, dist, dev)
        value = D.weak_throughput(w, wl.n, 3, job_ms)
        out[r] = (r, w, local, job_ms, agree_some, agree_all, value,
                  [g.tolist() for g in gathered])
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_plumbing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 0], codes
    assert sorted(res) == [0, 1]
    for r in range(world):
        rr, w, local, job_ms, some, allv, value, gathered = res[r]
        assert (rr, w, local) == (r, world, r)
        assert job_ms == 15.0                       # max over ranks, same on every rank
        assert some is False and allv is True       # one dissenting rank vetoes everywhere
        assert value == pytest.approx(world * 128 * 3 / 15e-3)
        # the ranks hold different sequences
        assert gathered[0] != gathered[1]
    assert res[0][7] == res[1][7]


def test_rank_env_parsing_and_single_process_fallbacks():
    assert D.rank_env({}) == (0, 1, 0)
    assert D.rank_env({"RANK": "3", "WORLD_SIZE": "8", "LOCAL_RANK": "3"}) == (3, 8, 3)
    with pytest.raises(ValueError):
        D.rank_env({"RANK": "8", "WORLD_SIZE": "8"})
    assert not dist.is_initialized()
    assert D.max_over_ranks(4.5, dist, None) == 4.5
    assert D.all_ranks_agree(False, dist, None) is False
    assert D.sequence_seed(1000, 0) != D.sequence_seed(1000, 1)
    with pytest.raises(ValueError):
        D.weak_throughput(1, 10, 1, 0.0)
    assert D.weak_throughput(4, 65536, 5, 10.0) == pytest.approx(4 * 65536 * 5 / 0.01)
