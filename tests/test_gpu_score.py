"""GPU parity: observation-window attention A and the combined score S (all score modes)."""
import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from long_context_kv_obs_b200 import synth
from oracle import infokv as ik
from oracle import pipeline as op
from tests.helpers import assert_close_rel, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_score(wl, inp, mode):
    L, Hq, Hkv, d, n = wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n
    m = B.model(L, Hq, Hkv, d)
    S = torch.empty(L, Hkv, n, device=DEV)
    A = torch.empty(L, Hkv, n, device=DEV)
    H = torch.empty(n, device=DEV)
    D = torch.empty(L, n, device=DEV)
    Eb = torch.empty(L, device=DEV)
    kw = dict(mode=mode, n=n, W=wl.W, Qw=inp.Qw, K=inp.K, S=S, A=A, alpha=wl.alpha, tau=wl.tau,
              topk=wl.topk)
    if mode == B.SCORE_INFOKV:
        kw.update(logits=inp.logits, hidden=inp.hidden, H_out=H, D_out=D, Ebar=Eb)
    elif mode == B.SCORE_VATP:
        kw.update(V=inp.V)
    B.kvc_score(m, **kw)
    torch.cuda.synchronize()
    return dict(S=S, A=A, H=H, D=D, Ebar=Eb)


def oracle_scores(wl, inp, mode):
    name = {B.SCORE_INFOKV: "infokv", B.SCORE_VATP: "vatp", B.SCORE_ATTN: "attn"}[mode]
    return op.prefill_scores(np64(inp.logits) if inp.logits is not None else None,
                             np64(inp.hidden) if inp.hidden is not None else None,
                             np64(inp.Qw), np64(inp.K), np64(inp.V), G=wl.group, alpha=wl.alpha,
                             tau=wl.tau, topk=wl.topk, mode=name)


SMALL = [
    synth.WORKLOADS[0],                                                     # fp32, d=64, G=2
    synth.WORKLOADS[2].scaled(n_layers=2, n=3000, vocab=5000, hidden=512),  # bf16, d=128, G*W=128
    synth.WORKLOADS[1].scaled(n_layers=2, n=1500, vocab=3001, hidden=256),  # bf16, G*W=96
    synth.WORKLOADS[4].scaled(n_layers=2, n=2100, vocab=4000, hidden=512, batch=1),  # G*W=224
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_infokv_score_matches_oracle(wl):
    inp = synth.gen_prefill(wl, seed=11, device=DEV)
    got = run_score(wl, inp, B.SCORE_INFOKV)
    ref = oracle_scores(wl, inp, B.SCORE_INFOKV)
    assert_close_rel(np64(got["H"]), ref["H"], rtol=1e-4, atol=1e-5, what="H")
    assert_close_rel(np64(got["D"]), ref["D"], rtol=0, atol=2e-5, what="D")
    assert_close_rel(np64(got["Ebar"]), ref["Ebar"], rtol=1e-4, what="Ebar")
    assert_close_rel(np64(got["A"]), ref["A"], rtol=1e-4, atol=1e-12, what="A")
    assert_close_rel(np64(got["S"]), ref["S"], rtol=1e-4, atol=1e-12, what="S")
    # S is a convex mix of two distributions: every row sums to 1
    np.testing.assert_allclose(np64(got["S"]).sum(-1), 1.0, atol=1e-4)


@pytest.mark.parametrize("wl", SMALL[:2], ids=lambda w: w.name)
@pytest.mark.parametrize("mode", [B.SCORE_VATP, B.SCORE_ATTN])
def test_vatp_and_attention_scores_match_oracle(wl, mode):
    inp = synth.gen_prefill(wl, seed=12, device=DEV, with_logits=False, with_hidden=False)
    got = run_score(wl, inp, mode)
    ref = oracle_scores(wl, inp, mode)
    assert_close_rel(np64(got["A"]), ref["A"], rtol=1e-4, atol=1e-12, what="A")
    assert_close_rel(np64(got["S"]), ref["S"], rtol=1e-4, atol=1e-12, what="S")


def test_window_with_positions_and_window_queries_of_another_order():
    """Keys with arbitrary ascending positions and window queries at given positions."""
    wl = synth.WORKLOADS[2].scaled(n_layers=1, n=777)
    L, Hq, Hkv, d, n, W = 1, 32, 8, 128, 777, 32
    g = torch.Generator(device=DEV).manual_seed(5)
    K = torch.randn(L, Hkv, n, d, device=DEV, generator=g).to(torch.bfloat16)
    Qw = torch.randn(L, Hq, W, d, device=DEV, generator=g).to(torch.bfloat16)
    kpos = torch.sort(torch.randperm(5000, device=DEV, generator=g)[:n])[0].to(torch.int32)
    kpos_full = kpos.repeat(L, Hkv, 1).contiguous()
    qpos = kpos[-W:].flip(0).contiguous()            # the last W keys, queries in reverse order
    m = B.model(L, Hq, Hkv, d)
    S = torch.empty(L, Hkv, n, device=DEV)
    A = torch.empty(L, Hkv, n, device=DEV)
    B.kvc_score(m, mode=B.SCORE_ATTN, n=n, W=W, Qw=Qw, K=K, S=S, A=A, qpos=qpos, kpos=kpos_full,
                kpos_strides=(Hkv * n, n))
    torch.cuda.synchronize()
    for gg in range(Hkv):
        ref = ik.window_attention(np64(Qw[0, gg * 4:(gg + 1) * 4]), np64(K[0, gg]), qpos=np64(qpos),
                                  kpos=np64(kpos))
        assert_close_rel(np64(A[0, gg]), ref, rtol=1e-4, atol=1e-12, what=f"A head {gg}")


def _window_A(L, Hq, Hkv, n, W, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    K = torch.randn(L, Hkv, n, 128, device=DEV, generator=g).to(torch.bfloat16)
    Qw = (torch.randn(L, Hq, W, 128, device=DEV, generator=g) * 1.5).to(torch.bfloat16)
    m = B.model(L, Hq, Hkv, 128)
    S = torch.empty(L, Hkv, n, device=DEV)
    A = torch.empty(L, Hkv, n, device=DEV)
    B.kvc_score(m, mode=B.SCORE_ATTN, n=n, W=W, Qw=Qw, K=K, S=S, A=A)
    torch.cuda.synchronize()
    return Qw, K, A, S


@pytest.mark.parametrize("L,Hq,Hkv,n,W", [
    (1, 4, 1, 300, 32),      # one slice
    (1, 8, 2, 5000, 32),     # fewer slices than the pass-1 / pass-2 lag, ragged last item
    (2, 32, 8, 100, 32),     # less than one 128-key tile
    (3, 16, 8, 4097, 16),    # G*W = 32, one key past a work-item edge
    (1, 64, 8, 2048, 16),    # G*W = 128, exactly one work item
    (2, 28, 4, 3000, 32),    # G*W = 224: two M tiles, pass-2 columns split 7 / 7 chunks
    (1, 9, 1, 1500, 16),     # G*W = 144: pass-2 columns split 5 / 4 chunks
    (1, 16, 1, 777, 16),     # G*W = 256: both M tiles full
])
def test_window_attention_slice_layouts(L, Hq, Hkv, n, W):
    Qw, K, A, S = _window_A(L, Hq, Hkv, n, W, seed=L * 1000 + n)
    G = Hq // Hkv
    np.testing.assert_array_equal(np64(S), np64(A))
    for l in range(L):
        for gg in range(Hkv):
            ref = ik.window_attention(np64(Qw[l, gg * G:(gg + 1) * G]), np64(K[l, gg]))
            assert_close_rel(np64(A[l, gg]), ref, rtol=1e-4, atol=1e-12, what=f"A ({l}, {gg})")


def test_window_attention_full_size_sampled():
    """32 layers x 8 KV heads x 65536 keys, G*W = 128 (the 8B-shape prefill): every
    slice's A sums to 1 (mean of softmax rows) and sampled slices match the oracle."""
    L, Hq, Hkv, n, W = 32, 32, 8, 65536, 32
    Qw, K, A, _ = _window_A(L, Hq, Hkv, n, W, seed=77)
    sums = np64(A.sum(-1, dtype=torch.float64))
    np.testing.assert_allclose(sums, 1.0, atol=1e-4)
    for l, gg in [(0, 0), (17, 5), (31, 7)]:
        ref = ik.window_attention(np64(Qw[l, gg * 4:(gg + 1) * 4]), np64(K[l, gg]))
        assert_close_rel(np64(A[l, gg]), ref, rtol=1e-4, atol=1e-12, what=f"A ({l}, {gg})")


def test_window_beside_signals_equals_sequential():
    """kvc_score's two schedules - the window pass on a share of the SMs beside the entropy
    and representation scans, or the stages in sequence - give the same A bit for bit (the
    partials merge in a fixed order whatever the grid) and the same S up to the rounding of
    where the combination is formed; both match the oracle."""
    wl = synth.WORKLOADS[1].scaled(n_layers=3, n=4500, vocab=3001, hidden=256)
    inp = synth.gen_prefill(wl, seed=17, device=DEV)
    L, Hq, Hkv, d, n = wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n
    m = B.model(L, Hq, Hkv, d)
    res = {}
    for split in (-1, 8, 37, 10000):
        S = torch.empty(L, Hkv, n, device=DEV)
        A = torch.empty(L, Hkv, n, device=DEV)
        B.kvc_score(m, mode=B.SCORE_INFOKV, n=n, W=wl.W, Qw=inp.Qw, K=inp.K, S=S, A=A, logits=inp.logits,
                    hidden=inp.hidden, H_out=torch.empty(n, device=DEV), D_out=torch.empty(L, n, device=DEV),
                    alpha=wl.alpha, tau=wl.tau, topk=wl.topk, window_sms=split)
        torch.cuda.synchronize()
        res[split] = (S, A)
    assert B.kvc_check_status() == 0
    for split in (8, 37, 10000):
        assert torch.equal(res[split][1], res[-1][1])
        assert_close_rel(np64(res[split][0]), np64(res[-1][0]), rtol=1e-6, atol=1e-12, what="S")
    ref = oracle_scores(wl, inp, B.SCORE_INFOKV)
    assert_close_rel(np64(res[37][0]), ref["S"], rtol=1e-4, atol=1e-12, what="S")
