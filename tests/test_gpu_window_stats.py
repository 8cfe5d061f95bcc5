"""GPU parity: window-row softmax statistics taken from the rows' own decode steps.

kvc_decode_attn can write each step's log-sum-exp into one slot of a [B][L][Hq][W] ring
(lse_stride = W).  kvc_recompress given that ring (win_lse) forms A_i of [InfoKV]
Methodology in one pass from exp(q k_i * scale - lse) instead of recomputing each window
row's max and sum over the cache.  The identity behind it: a window row sees the cache rows
at or before its position, and every one of them was in the cache when its decode step ran
([InfoKV] Technical details: compression runs periodically during decoding; the window is
shorter than the period), so that step's log-sum-exp is the row's.

Tolerances.  A logit is an fp32 sum of d exact bf16 products: within gamma_d * sum|q k| of
the exact one (gamma_m = m u / (1 - m u), u = 2^-24), times the scale; the log-sum-exp moves
by at most the largest logit error, plus the fp32 exp / log rounding of the merge (2e-6
relative, 1e-6 absolute).  Kept sets follow the shared rule: equal to the fp64 oracle's but
for positions within 1e-5 relative of the k-th score.
"""
import math

import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from long_context_kv_obs_b200 import synth
from long_context_kv_obs_b200.pipeline import DecodeTimeCompressor
from oracle import infokv as ik
from tests.helpers import kept_sets_agree, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"
U = 2.0 ** -24


def test_decode_lse_into_a_ring_slot():
    """lse_stride = W writes the contiguous lse's values into slot 5 of the ring and nothing
    else, and they are the fp64 log-sum-exp of the scaled logits within the derived bound."""
    Bn, L, Hq, Hkv, d, W, n = 2, 3, 8, 2, 128, 32, 700
    G = Hq // Hkv
    m = B.model(L, Hq, Hkv, d)
    g = torch.Generator(device=DEV).manual_seed(7)
    K = torch.randn(Bn, L, Hkv, n, d, device=DEV, generator=g).to(torch.bfloat16)
    V = torch.randn(Bn, L, Hkv, n, d, device=DEV, generator=g).to(torch.bfloat16)
    q = torch.randn(Bn, L, Hq, d, device=DEV, generator=g).to(torch.bfloat16)
    lens = torch.tensor([[n, n - 37, 1], [n - 1, 256, n]], dtype=torch.int32, device=DEV)
    o = torch.empty(Bn, L, Hq, d, device=DEV)
    lse = torch.empty(Bn, L, Hq, device=DEV)
    ring = torch.full((Bn, L, Hq, W), float("nan"), device=DEV)
    B.kvc_decode_attn(m, q=q, K=K, V=V, lens=lens, max_len=n, o=o, lse=lse)
    B.kvc_decode_attn(m, q=q, K=K, V=V, lens=lens, max_len=n, o=o, lse=ring[:, :, :, 5])
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    assert torch.equal(ring[:, :, :, 5], lse)
    assert torch.isnan(ring[:, :, :, :5]).all() and torch.isnan(ring[:, :, :, 6:]).all()
    qn, Kn, ln = np64(q), np64(K), lens.cpu().numpy()
    scale = 1.0 / math.sqrt(d)
    gamma = d * U / (1 - d * U)
    got = np64(lse)
    for b in range(Bn):
        for l in range(L):
            rows = Kn[b, l, :, :ln[b, l]]
            for h in range(Hq):
                s = rows[h // G] @ qn[b, l, h] * scale
                mx = s.max()
                ref = mx + math.log(np.exp(s - mx).sum())
                tol = gamma * scale * (np.abs(rows[h // G]) @ np.abs(qn[b, l, h])).max() + 2e-6 * abs(ref) + 1e-6
                assert abs(got[b, l, h] - ref) <= tol, (b, l, h, got[b, l, h], ref, tol)


def test_sparse_decode_lse_is_over_the_whole_cache():
    """kvc_sparse_decode's lse (into a ring slot) is each head's log-sum-exp over every cached
    key, not only the active set: the dense decode's within twice the logit bound."""
    Bn, L, Hq, Hkv, d, W, cap, t_cur = 2, 2, 28, 4, 128, 32, 700, 2000
    G = Hq // Hkv
    m = B.model(L, Hq, Hkv, d)
    g = torch.Generator(device=DEV).manual_seed(17)
    K = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(torch.bfloat16)
    V = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(torch.bfloat16)
    q = torch.randn(Bn, L, Hq, d, device=DEV, generator=g).to(torch.bfloat16)
    lens = torch.tensor([[700, 1], [333, 512]], dtype=torch.int32, device=DEV)
    pos = torch.sort(torch.rand(Bn, L, Hkv, cap, device=DEV, generator=g) * t_cur, dim=-1)[0].to(torch.int32)
    acc = torch.rand(Bn, L, Hkv, cap, device=DEV, generator=g) * 3
    o = torch.empty(Bn, L, Hq, d, device=DEV)
    ring = torch.full((Bn, L, Hq, W), float("nan"), device=DEV)
    B.kvc_sparse_decode(m, q=q, K=K, V=V, lens=lens, max_len=cap, pos=pos, acc=acc, t_cur=t_cur, n_prompt=1500,
                        kappa=0.1, a_tr=0.5, b_hi=0.5, o=o, lse=ring[:, :, :, 3])
    dense = torch.empty(Bn, L, Hq, device=DEV)
    B.kvc_decode_attn(m, q=q, K=K, V=V, lens=lens, max_len=cap, o=torch.empty_like(o), lse=dense)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    assert torch.isnan(ring[:, :, :, :3]).all() and torch.isnan(ring[:, :, :, 4:]).all()
    got, ref = np64(ring[:, :, :, 3]), np64(dense)
    qn, Kn, ln = np64(q), np64(K), lens.cpu().numpy()
    scale = 1.0 / math.sqrt(d)
    gamma = d * U / (1 - d * U)
    for b in range(Bn):
        for l in range(L):
            rows = Kn[b, l, :, :ln[b, l]]
            for h in range(Hq):
                tol = 2 * (gamma * scale * (np.abs(rows[h // G]) @ np.abs(qn[b, l, h])).max()
                           + 2e-6 * abs(ref[b, l, h]) + 1e-6)
                assert abs(got[b, l, h] - ref[b, l, h]) <= tol, (b, l, h, got[b, l, h], ref[b, l, h], tol)


def _oracle_kept(dc, c, len_, t, keep, wl):
    """The fp64 oracle's kept positions and tie zone of every (sequence, layer, KV head) row
    of the decode-time cache c: window attention with the ring's queries at their positions,
    Softmax(D * H), the InfoKV mix, top-k with the recent window."""
    G, Hkv = wl.group, wl.n_kv_heads
    K, pos = np64(dc.K[c]), dc.pos[c].cpu().numpy()
    H, D = np64(dc.Hs[c]), np64(dc.Ds[c])
    Q, qpos = np64(dc.Qring), dc.qpos.cpu().numpy()
    out = {}
    for b in range(wl.batch):
        for l in range(wl.n_layers):
            S = {}
            for g in range(Hkv):
                A = ik.window_attention(Q[b, l, g * G:(g + 1) * G], K[b, l, g, :len_], qpos=qpos[b],
                                        kpos=pos[b, l, g, :len_])
                _, P, _ = ik.entropy_scores(D[b, l, g, :len_], H[b, l, g, :len_])
                S[g] = ik.combine(A, P, wl.alpha)
            for g in range(Hkv):
                Sg = ik.union_max(np.stack([S[j] for j in range(Hkv)])) if wl.sel_mode == "gqa_union" else S[g]
                p = pos[b, l, g, :len_]
                out[(b, l, g)] = (p[ik.select_topk(Sg, keep, wl.w)], p[ik.tie_zone(Sg, keep, wl.w)])
    return out


def test_recompress_with_window_stats_from_the_decode_steps():
    """After W+ decode steps through attend(), kvc_recompress with the decode steps' ring
    (one pass) and without it (both passes) keep the fp64 oracle's sets."""
    wl = synth.WORKLOADS[4].scaled(n_layers=2, n=1024, batch=2, gen_tokens=512, period=1024)
    seed = 53
    Bn, L, Hkv, d, n0 = wl.batch, wl.n_layers, wl.n_kv_heads, wl.head_dim, wl.n
    g = torch.Generator(device=DEV).manual_seed(seed)
    Kp = torch.randn(Bn, L, Hkv, n0, d, device=DEV, generator=g).to(wl.dtype)
    Vp = torch.randn(Bn, L, Hkv, n0, d, device=DEV, generator=g).to(wl.dtype)
    H0 = torch.rand(Bn, n0, device=DEV, generator=g) * 4
    D0 = torch.rand(Bn, L, n0, device=DEV, generator=g) + 1.0
    dc = DecodeTimeCompressor(wl, Kp, Vp, H0, D0)
    for step in range(wl.W + 16):
        q = synth.gen_decode_queries(wl, seed, step, DEV)
        k, v = synth.gen_decode_kv(wl, seed, step, DEV)
        Hn = torch.rand(Bn, device=DEV, generator=g) * 4
        Dn = torch.rand(Bn, L, device=DEV, generator=g) + 1.0
        dc.append(k, v, Hn, Dn, q)
        dc.attend(q)
    assert dc.lse_streak >= wl.W
    c, len_, t = dc.cur, dc.len, dc.t
    keep = max(min(wl.w, len_), math.floor(wl.rho * t))
    ref = _oracle_kept(dc, c, len_, t, keep, wl)
    results = {}
    for one_pass in (True, False):
        kw = dc._recompress_kw(len_, t)
        kw["win_lse"] = dc.lse_ring if one_pass else None
        B.kvc_recompress(dc.m, workspace=dc.ws_re, **kw)
        torch.cuda.synchronize()
        assert B.kvc_check_status() == 0
        results[one_pass] = dc.pos[1 - c][..., :keep].cpu().numpy().copy()
    same = 0
    for (b, l, gg), (want, zone) in ref.items():
        for one_pass, got in results.items():
            ok, msg = kept_sets_agree(got[b, l, gg], want, zone)
            assert ok, f"one_pass={one_pass} seq {b} layer {l} head {gg}: {msg}"
        same += np.array_equal(results[True][b, l, gg], results[False][b, l, gg])
    assert same >= 0.9 * len(ref)


def test_recompress_window_stats_batched_equals_per_sequence_path():
    """With the decode steps' ring, the batched call (sequences folded into the layers) and
    the per-sequence path taken for batch-strided caches give bit-identical results."""
    wl = synth.WORKLOADS[4].scaled(n_layers=2, n=512, batch=2, gen_tokens=512, period=1024)
    seed = 61
    Bn, L, Hkv, d, n0 = wl.batch, wl.n_layers, wl.n_kv_heads, wl.head_dim, wl.n
    g = torch.Generator(device=DEV).manual_seed(seed)
    Kp = torch.randn(Bn, L, Hkv, n0, d, device=DEV, generator=g).to(wl.dtype)
    Vp = torch.randn(Bn, L, Hkv, n0, d, device=DEV, generator=g).to(wl.dtype)
    dc = DecodeTimeCompressor(wl, Kp, Vp, torch.rand(Bn, n0, device=DEV, generator=g) * 4,
                              torch.rand(Bn, L, n0, device=DEV, generator=g) + 1.0)
    for step in range(wl.W + 3):
        q = synth.gen_decode_queries(wl, seed, step, DEV)
        k, v = synth.gen_decode_kv(wl, seed, step, DEV)
        dc.append(k, v, torch.rand(Bn, device=DEV, generator=g) * 4, torch.rand(Bn, L, device=DEV, generator=g) + 1.0, q)
        dc.attend(q)
    c, n, len_, t = dc.cur, 1 - dc.cur, dc.len, dc.t
    keep = max(min(wl.w, len_), math.floor(wl.rho * t))
    kw = dc._recompress_kw(len_, t)
    assert kw["win_lse"] is not None
    B.kvc_recompress(dc.m, workspace=dc.ws_re, **kw)
    torch.cuda.synchronize()
    batched = [x[..., :keep, :].clone() if x.dim() == 5 else x[..., :keep].clone()
               for x in (dc.K[n], dc.V[n], dc.pos[n], dc.Hs[n], dc.Ds[n])]
    cap = dc.K.shape[-2]
    Kbig = torch.zeros(Bn, 2 * L, Hkv, cap, d, dtype=wl.dtype, device=DEV)
    Vbig = torch.zeros_like(Kbig)
    Kbig[:, :L] = dc.K[c]
    Vbig[:, :L] = dc.V[c]
    for x in (dc.K[n], dc.V[n], dc.pos[n], dc.Hs[n], dc.Ds[n]):
        x.zero_()
    kw = dc._recompress_kw(len_, t)
    kw["K"], kw["V"] = Kbig[:, :L], Vbig[:, :L]
    B.kvc_recompress(dc.m, workspace=dc.ws_re, **kw)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    strided = [x[..., :keep, :] if x.dim() == 5 else x[..., :keep]
               for x in (dc.K[n], dc.V[n], dc.pos[n], dc.Hs[n], dc.Ds[n])]
    for a_, b_ in zip(batched, strided):
        assert torch.equal(a_, b_)
