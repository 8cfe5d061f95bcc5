"""GPU: a bounded device-side wait that runs out reports KVC_ERR_TIMEOUT, and the context
stays usable.

The single-launch window kernel waits (bounded) for the row constants another CTA publishes
once a slice's pass 1 is merged.  With one (layer, KV head) slice of 64 chunks, 64 CTAs
take the pass-1 chunks and the next 64 take the pass-2 chunks at once, so those wait for
the whole of pass 1 - several microseconds.  A limit of 1 us makes that wait run out: the
kernel records the timeout, drains the copies and MMAs it issued, frees its tensor memory
and returns.  A following call with the default limit must succeed and match the oracle."""
import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from long_context_kv_obs_b200 import synth
from oracle import pipeline as op
from tests.helpers import assert_close_rel, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_window_wait_runs_out_and_the_next_call_is_correct():
    wl = synth.WORKLOADS[2].scaled(n_layers=1, n_q_heads=4, n_kv_heads=1, n=65536)
    inp = synth.gen_prefill(wl, seed=13, device=DEV, with_logits=False, with_hidden=False)
    m = B.model(1, 4, 1, 128)
    S = torch.empty(1, 1, wl.n, device=DEV)
    B.kvc_check_status()                                   # start from a clean status word
    kw = dict(mode=B.SCORE_ATTN, n=wl.n, W=wl.W, Qw=inp.Qw, K=inp.K, S=S)
    ws = B.kvc_score(m, wait_limit_ns=1000, **kw)
    with pytest.raises(B.KvcError) as ei:
        B.kvc_check_status()
    assert ei.value.status == 5                            # KVC_ERR_TIMEOUT
    B.kvc_score(m, workspace=ws, **kw)                     # default limit, same workspace
    assert B.kvc_check_status() == 0
    ref = op.prefill_scores(None, None, np64(inp.Qw), np64(inp.K), G=4, mode="attn")
    assert_close_rel(np64(S), ref["S"], rtol=1e-4, atol=1e-12, what="S")
