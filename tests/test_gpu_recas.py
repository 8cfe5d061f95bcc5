"""GPU parity: RECAS calibrated dropped-mass estimator and adaptive budget controller
([RECAS] 2.B) against the fp64 oracle (oracle/recas.py), and the decode-time workload
run with the controller against the oracle replay.

Tolerances: the calibration works in fp64 on both sides from the same fp32 inputs, so
c, q and the sums agree to 1e-12 relative (only the summation order differs).  The
controller's need is an integer decided in fp64 on both sides; where the two differ the
decision must sit on the bound (within 1e-9 of eps).  In the end-to-end run the GPU's
probe deltas and window attention carry their own rounding (delta within the bound
tests.helpers.delta_rel_bound derives, A within 1e-4), so the GPU budget must lie
between the oracle's budgets at eps (1 + 1e-2) and eps (1 - 1e-2)."""
import math

import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from long_context_kv_obs_b200 import synth
from long_context_kv_obs_b200.pipeline import DecodeTimeCompressor
from oracle import infokv as ik
from oracle import pipeline as op
from oracle import recas
from tests.helpers import kept_sets_agree, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _probe_stream(rng, Bn, L, Hq, Hkv, steps):
    """Synthetic probe data: x per row, delta per query head ~ c* x (1 + noise), fp32."""
    out = []
    for _ in range(steps):
        x = rng.uniform(0.0, 0.3, size=(Bn, L, Hkv)).astype(np.float32)
        c = rng.uniform(0.5, 2.0, size=(Bn, L, 1, 1)).astype(np.float32)
        d = (np.repeat(x[..., None], Hq // Hkv, axis=-1) * c * (1 + 0.4 * rng.standard_normal((Bn, L, Hkv, Hq // Hkv)))
             ).reshape(Bn, L, Hq).clip(0, 1).astype(np.float32)
        out.append((d, x))
    return out


def _oracle_cals(stream, Bn, L, G, alpha):
    cals = [[recas.DroppedMassCalibrator(alpha=alpha) for _ in range(L)] for _ in range(Bn)]
    for d, x in stream:
        for b in range(Bn):
            for l in range(L):
                cals[b][l].observe(d[b, l].astype(np.float64), x[b, l].astype(np.float64), G)
    return cals


@pytest.mark.parametrize("Hq,Hkv,steps,alpha", [(8, 2, 40, 0.1), (28, 4, 3, 0.2), (32, 8, 12, 0.05)])
def test_calibrate_matches_oracle(Hq, Hkv, steps, alpha):
    Bn, L = 2, 3
    m = B.model(L, Hq, Hkv, 128)
    rng = np.random.default_rng(Hq * 100 + steps)
    stream = _probe_stream(rng, Bn, L, Hq, Hkv, steps)
    st = B.recas_state(Bn, L, DEV)
    dh = torch.empty(Bn, L, Hkv, device=DEV)
    db = torch.empty(Bn, L, Hkv, device=DEV)
    cals = [[recas.DroppedMassCalibrator(alpha=alpha) for _ in range(L)] for _ in range(Bn)]
    for j, (d, x) in enumerate(stream):
        B.kvc_recas_calibrate(m, delta=torch.from_numpy(d).to(DEV), x=torch.from_numpy(x).to(DEV), state=st,
                              alpha=alpha, delta_hat=dh, delta_bar=db)
        f = B.recas_fields(st)
        for b in range(Bn):
            for l in range(L):
                cal = cals[b][l]
                cal.observe(d[b, l].astype(np.float64), x[b, l].astype(np.float64), Hq // Hkv)
                assert float(f["c"][b, l]) == pytest.approx(cal.c, rel=1e-12)
                assert int(f["count"][b, l]) == (j + 1) * Hq
                q = float(f["q"][b, l])
                if math.isinf(cal.q):
                    assert math.isinf(q)
                else:
                    assert q == pytest.approx(cal.q, rel=1e-12, abs=1e-15)
                ring = np.sort(f["ring"][b, l].numpy()[:min(int(f["count"][b, l]), B.RECAS_RING)])
                np.testing.assert_allclose(ring, np.sort(cal.res), rtol=1e-12, atol=1e-15)
                want_h, want_b = cal.estimate(x[b, l].astype(np.float64))
                np.testing.assert_allclose(np64(dh[b, l]), want_h, rtol=1e-6, atol=1e-9)
                got_b = np64(db[b, l])
                if math.isinf(cal.q):
                    assert np.all(np.isinf(got_b))
                else:
                    np.testing.assert_allclose(got_b, want_b, rtol=1e-6, atol=1e-9)
    assert B.kvc_check_status() == 0


def _check_need(got, S, A, w, k0, c, q, eps):
    want = recas.controller_need(S, A, w, k0, c, q, eps)
    if got == want:
        return
    ks, x = recas.dropped_share_curve(S, A, w)
    f = dict(zip(ks.tolist(), (c * x + q).tolist()))
    assert f[got] <= eps + 1e-9, (got, want)
    assert got == max(k0, min(w, len(S))) or f[got - 1] > eps - 1e-9, (got, want)


@pytest.mark.parametrize("n,w,union", [(1, 0, False), (37, 8, False), (600, 32, True), (5248, 32, False),
                                       (16384, 64, False), (300, 300, False), (4097, 1, True)])
def test_control_matches_oracle(n, w, union):
    Bn, L, Hq, Hkv = 2, 2, 8, 2
    G = Hq // Hkv
    m = B.model(L, Hq, Hkv, 128)
    rng = np.random.default_rng(n + w)
    stream = _probe_stream(rng, Bn, L, Hq, Hkv, 6)
    st = B.recas_state(Bn, L, DEV)
    for d, x in stream:
        B.kvc_recas_calibrate(m, delta=torch.from_numpy(d).to(DEV), x=torch.from_numpy(x).to(DEV), state=st,
                              alpha=0.1)
    cals = _oracle_cals(stream, Bn, L, G, 0.1)
    S = (np.round(rng.random((Bn, L, Hkv, n)) * 50) / 50).astype(np.float32)       # many ties
    A = (rng.random((Bn, L, Hkv, n)) ** 4 * (rng.random((Bn, L, Hkv, n)) < 0.9)).astype(np.float32)
    A /= A.sum(axis=-1, keepdims=True) + 1e-30
    pad = 5                                                                          # row stride > n
    St = torch.zeros(Bn, L, Hkv, n + pad, device=DEV)
    At = torch.zeros(Bn, L, Hkv, n + pad, device=DEV)
    St[..., :n] = torch.from_numpy(S)
    At[..., :n] = torch.from_numpy(A)
    for k0, eps in ((min(w, n), 0.3), (n // 3, 0.2), (n, 0.5), (n // 2, 0.0)):
        need = torch.empty(Bn, L, Hkv, dtype=torch.int32, device=DEV)
        budget = torch.zeros(1, dtype=torch.int32, device=DEV)
        B.kvc_recas_control(m, S=St, A=At, n=n, w=w, k0=k0, state=st, eps=eps, need=need, budget=budget,
                            sel_mode=B.SEL_GQA_UNION if union else B.SEL_PER_KV_HEAD)
        got = need.cpu().numpy()
        for b in range(Bn):
            for l in range(L):
                cal = cals[b][l]
                Sl = ik.union_max(S[b, l].astype(np.float64)) if union else None
                for g in range(Hkv):
                    row_S = Sl if union else S[b, l, g].astype(np.float64)
                    _check_need(int(got[b, l, g]), row_S, A[b, l, g].astype(np.float64), w, k0, cal.c, cal.q, eps)
        assert int(budget) == int(got.max())
        kmax = max(1, n // 2)
        B.kvc_recas_control(m, S=St, A=At, n=n, w=w, k0=k0, state=st, eps=eps, need=need, budget=budget,
                            k_max=kmax, sel_mode=B.SEL_GQA_UNION if union else B.SEL_PER_KV_HEAD)
        assert int(budget) == min(int(got.max()), kmax)
    assert B.kvc_check_status() == 0


def test_control_refuses_rows_longer_than_16384():
    m = B.model(1, 2, 1, 128)
    St = torch.zeros(1, 1, 1, 16385, device=DEV)
    need = torch.empty(1, 1, 1, dtype=torch.int32, device=DEV)
    with pytest.raises(B.KvcError) as ei:
        B.kvc_recas_control(m, S=St, A=St, n=16385, w=0, k0=0, state=B.recas_state(1, 1, DEV), eps=0.1,
                            need=need)
    assert ei.value.status == 2


def test_decode_time_compression_with_recas_budget_matches_oracle_replay():
    """Scaled decode-time workload with the controller on: probe (and calibration) every 16
    steps, recompression every 64 with the budget from the calibrated bound."""
    wl = synth.WORKLOADS[4].scaled(n_layers=2, n=256, vocab=3000, hidden=512, batch=2, gen_tokens=192,
                                   period=64)
    seed, eps, alpha, every = 37, 0.35, 0.1, 16
    Kp, Vp, Lp, Hp = synth.gen_prompt_batch(wl, seed, device=DEV)
    m = B.model(wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim)
    Bn, L, n0, Hkv, G = wl.batch, wl.n_layers, wl.n, wl.n_kv_heads, wl.group
    H0 = torch.empty(Bn, n0, device=DEV)
    D0 = torch.empty(Bn, L, n0, device=DEV)
    for b in range(Bn):
        B.kvc_score(m, mode=B.SCORE_INFOKV, n=n0, W=0, Qw=Kp[b, 0, 0], K=Kp[b], S=None, logits=Lp[b],
                    hidden=Hp[b], H_out=H0[b], D_out=D0[b])
    dc = DecodeTimeCompressor(wl, Kp, Vp, H0, D0, probe=True, recas_eps=eps, recas_alpha=alpha)
    k_max = dc.cap - wl.period
    reps, cals = [], []
    for b in range(Bn):
        hb = np64(Hp[b])
        Dref = np.stack([ik.repr_change(hb[l], hb[L - 1], wl.tau) for l in range(L)])
        reps.append(op.DecodeCompressionReplay(np64(Kp[b]), np64(Vp[b]), ik.topk_entropy(np64(Lp[b]), wl.topk),
                                               Dref, n_q_heads=wl.n_q_heads, W=wl.W, w=wl.w, rho=wl.rho,
                                               alpha=wl.alpha, tau=wl.tau, period=wl.period))
        reps[b].x = {(l, g): 0.0 for l in range(L) for g in range(Hkv)}
        cals.append([recas.DroppedMassCalibrator(alpha=alpha) for _ in range(L)])
    same = True                      # GPU and oracle budgets agree so far
    live = np.ones((Bn, L, Hkv), bool)
    Hn = torch.empty(Bn, device=DEV)
    Dn = torch.empty(L, Bn, device=DEV)
    grown = 0
    for step in range(wl.gen_tokens):
        q = synth.gen_decode_queries(wl, seed, step, DEV)
        k, v = synth.gen_decode_kv(wl, seed, step, DEV)
        lg, hid = synth.gen_decode_signals(wl, seed, step, DEV)
        B.kvc_score(m, mode=B.SCORE_INFOKV, n=Bn, W=0, Qw=q, K=k[None], S=None, logits=lg,
                    hidden=hid.transpose(0, 1).contiguous(), H_out=Hn, D_out=Dn)
        dc.append(k, v, Hn, Dn.t(), q)
        probe = step % every == every - 1
        dc.attend(q, probe=probe)
        if probe:
            dc.calibrate()
        for b in range(Bn):
            _, pr = reps[b].step(np64(q[b]), np64(k[b]), np64(v[b]), np64(lg[b]), np64(hid[b]), topk=wl.topk,
                                 probe=probe)
            if probe:
                for l in range(L):
                    delta = np.concatenate([pr[(l, g)]["delta"] for g in range(Hkv)])
                    cals[b][l].observe(delta, np.array([reps[b].x[(l, g)] for g in range(Hkv)]), G)
        if probe and same and live.all():
            f = B.recas_fields(dc.recas_state)
            for b in range(Bn):
                for l in range(L):
                    assert float(f["c"][b, l]) == pytest.approx(cals[b][l].c, rel=2e-3)
        if dc.due():
            keep = dc.recompress()
            torch.cuda.synchronize()
            scores = [reps[b].scores() for b in range(Bn)]

            def oracle_budget(e):
                k0 = min(reps[0].K[0][0].shape[0], max(min(wl.w, reps[0].t), math.floor(wl.rho * reps[0].t)))
                need = max(max(reps[b].recas_needs(scores[b], e, cals[b]).values()) for b in range(Bn))
                return max(k0, min(need, k_max))

            want = oracle_budget(eps)
            assert oracle_budget(eps * 1.01) <= keep <= oracle_budget(eps * 0.99), (keep, want)
            grown += keep > math.floor(wl.rho * dc.t)
            pos = dc.pos[dc.cur].cpu().numpy()
            xg = np64(dc.recas_x)
            for b in range(Bn):
                info = reps[b].recompress(budget=keep, scores=scores[b])
                for l in range(L):
                    for g in range(Hkv):
                        if not (same and live[b, l, g]):
                            continue
                        S, before = info[(l, g)]
                        zone = before[ik.tie_zone(S, keep, wl.w)]
                        ok, msg = kept_sets_agree(pos[b, l, g, :keep], reps[b].pos[l][g], zone)
                        assert ok, f"seq {b} layer {l} head {g}: {msg}"
                        if set(pos[b, l, g, :keep].tolist()) != set(reps[b].pos[l][g].tolist()):
                            live[b, l, g] = False
                            continue
                        assert abs(xg[b, l, g] - reps[b].x[(l, g)]) <= 2e-4
            same = same and keep == want
    assert grown >= 1                 # the controller did grow a budget in this run
    assert B.kvc_check_status() == 0
