"""GPU parity: RECAS dynamic sparse decode (kvc_sparse_decode) against the fp64 oracle
(oracle/recas.py sparse_decode_step), one step on random rows and a decode-time run with
appends and recompressions against the oracle replay.

Tolerances: the active set is an integer set chosen from fp32 sparse scores, so it must
equal the oracle's except for positions whose oracle score lies within 1e-5 relative of
the K_t-th largest (the tie zone); rows whose sets are equal are compared value by
value: outputs within 2e-3 (fp32 outputs), the attention history within 1e-5."""
import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from long_context_kv_obs_b200 import synth
from long_context_kv_obs_b200.pipeline import DecodeTimeCompressor
from oracle import infokv as ik
from oracle import pipeline as op
from oracle import recas
from tests.helpers import OUT_ATOL, kept_sets_agree, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _zone(sigma, kt):
    """Positions whose score lies within 1e-5 relative of the kt-th largest."""
    thr = np.sort(sigma)[::-1][kt - 1]
    return np.flatnonzero(np.abs(sigma - thr) <= 1e-5 * abs(thr))


@pytest.mark.parametrize("Hq,Hkv,kappa,ab", [(8, 2, 0.3, (0.6, 0.4)), (28, 4, 0.05, (0.5, 0.5)),
                                             (8, 2, 1.0, (1.0, 0.0)), (16, 2, 0.5, (0.0, 1.0))])
def test_sparse_step_matches_oracle(Hq, Hkv, kappa, ab):
    Bn, L, d, cap, n0, t_cur = 2, 2, 128, 700, 1500, 2000
    G = Hq // Hkv
    m = B.model(L, Hq, Hkv, d)
    g = torch.Generator(device=DEV).manual_seed(Hq * 7 + Hkv)
    K = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(torch.bfloat16)
    V = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(torch.bfloat16)
    K[..., 0, :] *= 4
    q = torch.randn(Bn, L, Hq, d, device=DEV, generator=g).to(torch.bfloat16)
    lens = torch.tensor([[700, 1], [333, 512]], dtype=torch.int32, device=DEV)
    rng = np.random.default_rng(Hq + Hkv)
    pos = np.zeros((Bn, L, Hkv, cap), np.int32)
    for b in range(Bn):
        for l in range(L):
            for h in range(Hkv):
                pos[b, l, h] = np.sort(rng.choice(t_cur, cap, replace=False))
    acc = (rng.random((Bn, L, Hkv, cap)) * 3).astype(np.float32)
    pos_t, acc_t = torch.from_numpy(pos).to(DEV), torch.from_numpy(acc).to(DEV)
    o = torch.empty(Bn, L, Hq, d, device=DEV)
    active = torch.full((Bn, L, Hkv, cap), -1, dtype=torch.int32, device=DEV)
    n_act = torch.empty(Bn, L, Hkv, dtype=torch.int32, device=DEV)
    B.kvc_sparse_decode(m, q=q, K=K, V=V, lens=lens, max_len=cap, pos=pos_t, acc=acc_t, t_cur=t_cur, n_prompt=n0,
                        kappa=kappa, a_tr=ab[0], b_hi=ab[1], o=o, active=active, n_active=n_act)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    Kn, Vn, qn, on = np64(K), np64(V), np64(q), np64(o)
    act, na, accg = active.cpu().numpy(), n_act.cpu().numpy(), acc_t.cpu().numpy()
    equal_rows = 0
    for b in range(Bn):
        for l in range(L):
            n = int(lens[b, l])
            for h in range(Hkv):
                cnt = recas.cached_steps(pos[b, l, h, :n], t_cur, n0)
                ro, ract, racc, sig = recas.sparse_decode_step(qn[b, l, h * G:(h + 1) * G], Kn[b, l, h, :n],
                                                               Vn[b, l, h, :n], acc[b, l, h, :n], cnt, kappa, *ab)
                kt = recas.sparse_active_count(n, kappa)
                assert na[b, l, h] == kt
                got = act[b, l, h, :kt]
                assert np.all(np.diff(got) > 0)
                ok, msg = kept_sets_agree(got, ract, _zone(sig, kt))
                assert ok, f"row {(b, l, h)}: {msg}"
                if set(got.tolist()) != set(ract.tolist()):
                    continue
                equal_rows += 1
                np.testing.assert_allclose(on[b, l, h * G:(h + 1) * G], ro, atol=OUT_ATOL, rtol=0)
                np.testing.assert_allclose(accg[b, l, h, :n], racc, atol=1e-5, rtol=0)
                np.testing.assert_array_equal(accg[b, l, h, n:], acc[b, l, h, n:])     # rows past len untouched
    assert equal_rows >= Bn * L * Hkv - 1


def test_decode_time_run_with_sparse_decode_matches_oracle_replay():
    """Scaled decode-time workload, every step decoded sparsely (kappa 0.3, a = b = 0.5), with
    appends and two recompressions: the history travels with its tokens."""
    wl = synth.WORKLOADS[4].scaled(n_layers=2, n=256, vocab=3000, hidden=512, batch=2, gen_tokens=128,
                                   period=64)
    seed, sparse = 53, (0.3, 0.5, 0.5)
    Kp, Vp, Lp, Hp = synth.gen_prompt_batch(wl, seed, device=DEV)
    m = B.model(wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim)
    Bn, L, n0, Hkv, G = wl.batch, wl.n_layers, wl.n, wl.n_kv_heads, wl.group
    H0 = torch.empty(Bn, n0, device=DEV)
    D0 = torch.empty(Bn, L, n0, device=DEV)
    for b in range(Bn):
        B.kvc_score(m, mode=B.SCORE_INFOKV, n=n0, W=0, Qw=Kp[b, 0, 0], K=Kp[b], S=None, logits=Lp[b],
                    hidden=Hp[b], H_out=H0[b], D_out=D0[b])
    dc = DecodeTimeCompressor(wl, Kp, Vp, H0, D0, sparse=sparse)
    reps = []
    for b in range(Bn):
        hb = np64(Hp[b])
        Dref = np.stack([ik.repr_change(hb[l], hb[L - 1], wl.tau) for l in range(L)])
        reps.append(op.DecodeCompressionReplay(np64(Kp[b]), np64(Vp[b]), ik.topk_entropy(np64(Lp[b]), wl.topk),
                                               Dref, n_q_heads=wl.n_q_heads, W=wl.W, w=wl.w, rho=wl.rho,
                                               alpha=wl.alpha, tau=wl.tau, period=wl.period))
    live = np.ones((Bn, L, Hkv), bool)
    Hn = torch.empty(Bn, device=DEV)
    Dn = torch.empty(L, Bn, device=DEV)
    for step in range(wl.gen_tokens):
        q = synth.gen_decode_queries(wl, seed, step, DEV)
        k, v = synth.gen_decode_kv(wl, seed, step, DEV)
        lg, hid = synth.gen_decode_signals(wl, seed, step, DEV)
        B.kvc_score(m, mode=B.SCORE_INFOKV, n=Bn, W=0, Qw=q, K=k[None], S=None, logits=lg,
                    hidden=hid.transpose(0, 1).contiguous(), H_out=Hn, D_out=Dn)
        dc.append(k, v, Hn, Dn.t(), q)
        o = dc.attend_sparse(q)
        torch.cuda.synchronize()
        on, Ug, pos = np64(o), dc.U[dc.cur].cpu().numpy(), dc.pos[dc.cur].cpu().numpy()
        for b in range(Bn):
            ro, _ = reps[b].step(np64(q[b]), np64(k[b]), np64(v[b]), np64(lg[b]), np64(hid[b]), topk=wl.topk,
                                 sparse=sparse)
            for l in range(L):
                for h in range(Hkv):
                    if not live[b, l, h]:
                        continue
                    n = dc.len
                    np.testing.assert_array_equal(pos[b, l, h, :n], reps[b].pos[l][h])
                    # o agrees while the active sets have (the history of a row, which decides the
                    # next set, is compared too); a tie-zone difference ends the row's comparison
                    if np.abs(on[b, l, h * G:(h + 1) * G] - ro[l, h * G:(h + 1) * G]).max() > OUT_ATOL or \
                            np.abs(Ug[b, l, h, :n] - reps[b].U[l][h]).max() > 1e-5:
                        live[b, l, h] = False
        if dc.due():
            keep = dc.recompress()
            torch.cuda.synchronize()
            pos = dc.pos[dc.cur].cpu().numpy()
            for b in range(Bn):
                info = reps[b].recompress()
                for l in range(L):
                    for h in range(Hkv):
                        if not live[b, l, h]:
                            continue
                        S, before = info[(l, h)]
                        ok, msg = kept_sets_agree(pos[b, l, h, :keep], reps[b].pos[l][h],
                                                  before[ik.tie_zone(S, keep, wl.w)])
                        assert ok, msg
                        if set(pos[b, l, h, :keep].tolist()) != set(reps[b].pos[l][h].tolist()):
                            live[b, l, h] = False
    assert live.mean() >= 0.75, live
    assert B.kvc_check_status() == 0
