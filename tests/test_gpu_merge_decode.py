"""GPU parity: SelKV merge (V', R), compensated decode attention and the RECAS probe."""
import math

import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from long_context_kv_obs_b200 import synth
from oracle import infokv as ik
from oracle import recas, selkv
from tests.helpers import OUT_ATOL, assert_close_rel, bf16_rne, bf16_ulp, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _kept_sets(L, Hkv, n, k, w, seed, union):
    g = torch.Generator(device=DEV).manual_seed(seed)
    S = (torch.rand(L, Hkv, n, device=DEV, generator=g) ** 4).cpu().numpy().astype(np.float64)
    idx = np.zeros((L, Hkv, k), np.int32)
    for l in range(L):
        if union:
            keep = ik.select_topk(ik.union_max(S[l]), k, w)
            idx[l] = keep[None]
        else:
            for gg in range(Hkv):
                idx[l, gg] = ik.select_topk(S[l, gg], k, w)
    return idx


@pytest.mark.parametrize("n,bucket,k,dt,union", [(3000, 512, 750, torch.bfloat16, True),
                                                 (2048, 512, 100, torch.bfloat16, False),
                                                 (1111, 128, 400, torch.float32, False),
                                                 (600, 512, 40, torch.bfloat16, True)])
def test_merge_matches_oracle(n, bucket, k, dt, union):
    L, Hkv, d = 2, 4, 128
    wl = synth.WORKLOADS[3].scaled(n_layers=L, n_kv_heads=Hkv, n_q_heads=4 * Hkv, n=n, bucket=bucket)
    inp = synth.gen_prefill(wl, seed=n, device=DEV, with_logits=False, with_hidden=False)
    V = inp.V.to(dt)
    g = torch.Generator(device=DEV).manual_seed(n)
    A = (torch.rand(L, Hkv, n, device=DEV, generator=g) ** 3 * 1e-3).contiguous()
    A[:, :, inp.anchors] *= 50.0
    idx = torch.from_numpy(_kept_sets(L, Hkv, n, k, 32, n, union)).to(DEV)
    kk = torch.full((L,), k, dtype=torch.int32, device=DEV)
    Vm = torch.empty(L, Hkv, k, d, dtype=dt, device=DEV)
    Vf = torch.empty(L, Hkv, k, d, device=DEV)
    R = torch.empty(L, Hkv, k, device=DEV)
    B.kvc_merge(B.model(L, 4 * Hkv, Hkv, d), n=n, V=V, A=A, idx=idx, k=kk, dst_V=Vm, R=R,
                bucket=bucket, dst_V_f32=Vf)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    Vn, An, ix = np64(V), np64(A), idx.cpu().numpy()
    for l in range(L):
        for gg in range(Hkv):
            Vp, Rr = selkv.merge(Vn[l, gg], An[l, gg], ix[l, gg], bucket)
            np.testing.assert_allclose(np64(Vf[l, gg]), Vp, atol=OUT_ATOL, rtol=0)
            assert_close_rel(np64(R[l, gg]), Rr, rtol=1e-4, what="R")
            got = np64(Vm[l, gg])
            if dt == torch.bfloat16:
                assert np.all(np.abs(got - bf16_rne(Vp)) <= bf16_ulp(Vp) * 1.0001)
            else:
                np.testing.assert_allclose(got, Vp, atol=OUT_ATOL, rtol=0)
            # slots that merged nothing keep the value bit-for-bit and R = 1
            plain = np.flatnonzero(Rr == 1.0)
            if dt == torch.bfloat16:
                np.testing.assert_array_equal(got[plain], Vn[l, gg][ix[l, gg][plain]])
            else:
                np.testing.assert_allclose(got[plain], Vn[l, gg][ix[l, gg][plain]], rtol=1e-6, atol=0)


def _decode_case(Bn, L, Hq, Hkv, d, lens, dt, seed, with_R):
    g = torch.Generator(device=DEV).manual_seed(seed)
    cap = int(max(lens)) + 5
    K = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g)
    K[..., 0, :] *= 4.0
    V = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g)
    q = torch.randn(Bn, L, Hq, d, device=DEV, generator=g)
    R = (1.0 + 3.0 * torch.rand(Bn, L, Hkv, cap, device=DEV, generator=g) ** 4) if with_R else None
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV).view(Bn, L)
    return K.to(dt), V.to(dt), q.to(dt), R, lens_t


@pytest.mark.parametrize("Bn,L,Hq,Hkv,d,dt", [(1, 2, 32, 8, 128, torch.bfloat16),
                                              (2, 3, 28, 4, 128, torch.bfloat16),
                                              (1, 2, 24, 8, 128, torch.float32),
                                              (2, 2, 4, 2, 64, torch.float32)])
def test_decode_with_bias_matches_oracle(Bn, L, Hq, Hkv, d, dt):
    rng = np.random.default_rng(Hq)
    lens = rng.integers(1, 2500, size=Bn * L)
    lens[0] = 1
    K, V, q, R, lens_t = _decode_case(Bn, L, Hq, Hkv, d, lens, dt, seed=Hq, with_R=True)
    o = torch.empty(Bn, L, Hq, d, device=DEV)
    lse = torch.empty(Bn, L, Hq, device=DEV)
    B.kvc_decode_attn(B.model(L, Hq, Hkv, d), q=q, K=K, V=V, lens=lens_t, max_len=int(lens.max()),
                      o=o, R=R, alpha_c=1.0, lse=lse)
    torch.cuda.synchronize()
    G = Hq // Hkv
    Kn, Vn, qn, Rn, on = np64(K), np64(V), np64(q), np64(R), np64(o)
    for b in range(Bn):
        for l in range(L):
            m_ = int(lens[b * L + l])
            for gg in range(Hkv):
                want = selkv.decode_attention(qn[b, l, gg * G:(gg + 1) * G], Kn[b, l, gg, :m_],
                                              Vn[b, l, gg, :m_], Rn[b, l, gg, :m_], 1.0)
                np.testing.assert_allclose(on[b, l, gg * G:(gg + 1) * G], want, atol=OUT_ATOL, rtol=0)
                s = qn[b, l, gg * G:(gg + 1) * G] @ Kn[b, l, gg, :m_].T / math.sqrt(d) + np.log(Rn[b, l, gg, :m_])
                mx = s.max(-1)
                ref_lse = mx + np.log(np.exp(s - mx[:, None]).sum(-1))
                assert_close_rel(np64(lse[b, l, gg * G:(gg + 1) * G]), ref_lse, rtol=1e-5, atol=1e-4, what="lse")


def test_decode_unit_ratio_equals_unbiased():
    Bn, L, Hq, Hkv, d = 1, 2, 32, 8, 128
    lens = [3000, 17]
    K, V, q, _, lens_t = _decode_case(Bn, L, Hq, Hkv, d, lens, torch.bfloat16, seed=3, with_R=False)
    m = B.model(L, Hq, Hkv, d)
    o1 = torch.empty(Bn, L, Hq, d, device=DEV)
    o2 = torch.empty_like(o1)
    B.kvc_decode_attn(m, q=q, K=K, V=V, lens=lens_t, max_len=3000, o=o1)
    R1 = torch.ones(Bn, L, Hkv, K.shape[3], device=DEV)
    B.kvc_decode_attn(m, q=q, K=K, V=V, lens=lens_t, max_len=3000, o=o2, R=R1, alpha_c=1.0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)          # log 1 = 0 exactly


@pytest.mark.parametrize("Bn,L,Hq,Hkv,T", [(2, 2, 28, 4, 2600), (1, 1, 32, 8, 300)])
def test_probe_matches_oracle_and_bound_holds(Bn, L, Hq, Hkv, T):
    d = 128
    lens = np.full(Bn * L, T)
    K, V, q, _, lens_t = _decode_case(Bn, L, Hq, Hkv, d, lens, torch.bfloat16, seed=T, with_R=False)
    g = torch.Generator(device="cpu").manual_seed(T)
    kept = torch.rand(Bn, L, Hkv, T, generator=g) < 0.3
    kept[..., -32:] = True
    words = (T + 31) // 32
    bits = np.zeros((Bn, L, Hkv, words), np.int64)
    kn = kept.numpy()
    for i in range(T):
        bits[..., i // 32] |= kn[..., i].astype(np.int64) << (i % 32)
    bits = np.where(bits >= 2 ** 31, bits - 2 ** 32, bits).astype(np.int32)
    bits_t = torch.from_numpy(bits).to(DEV)
    m = B.model(L, Hq, Hkv, d)
    shp = (Bn, L, Hq)
    delta, err, bound = (torch.empty(shp, device=DEV) for _ in range(3))
    vmax = torch.empty(Bn, L, Hkv, device=DEV)
    o = torch.empty(Bn, L, Hq, d, device=DEV)
    o_full, o_kept = torch.empty_like(o), torch.empty_like(o)
    B.kvc_decode_attn(m, q=q, K=K, V=V, lens=lens_t, max_len=T, o=o, K_full=K, V_full=V,
                      lens_full=lens_t, max_len_full=T, kept_bits=bits_t, delta=delta, vmax=vmax,
                      err=err, bound=bound, o_full=o_full, o_kept=o_kept)
    torch.cuda.synchronize()
    G = Hq // Hkv
    Kn, Vn, qn = np64(K), np64(V), np64(q)
    for b in range(Bn):
        for l in range(L):
            for gg in range(Hkv):
                r = recas.dropped_mass_probe(qn[b, l, gg * G:(gg + 1) * G], Kn[b, l, gg, :T],
                                             Vn[b, l, gg, :T], kn[b, l, gg])
                sl = slice(gg * G, (gg + 1) * G)
                assert_close_rel(np64(delta[b, l, sl]), r["delta"], rtol=1e-4, atol=1e-7, what="delta")
                assert abs(float(vmax[b, l, gg]) - r["vmax"]) <= 1e-5 * r["vmax"]
                np.testing.assert_allclose(np64(o_full[b, l, sl]), r["o_full"], atol=OUT_ATOL, rtol=0)
                np.testing.assert_allclose(np64(o_kept[b, l, sl]), r["o_kept"], atol=OUT_ATOL, rtol=0)
                np.testing.assert_allclose(np64(err[b, l, sl]), r["err"], atol=OUT_ATOL, rtol=0)
                assert np.all(np64(err[b, l, sl]) <= np64(bound[b, l, sl]) * (1 + 1e-4) + 1e-6)
    # the full-cache pass equals plain decode over the full cache
    np.testing.assert_allclose(np64(o_full), np64(o), atol=1e-5, rtol=0)


def test_decode_strided_rows_matches_oracle():
    """K and V interleaved in one [.., 2d] tensor: rows 512 bytes apart (per-row copies)."""
    Bn, L, Hq, Hkv, d = 1, 2, 32, 8, 128
    lens = [1500, 77]
    g = torch.Generator(device=DEV).manual_seed(21)
    KV = torch.randn(Bn, L, Hkv, 1600, 2 * d, device=DEV, generator=g).to(torch.bfloat16)
    K, V = KV[..., :d], KV[..., d:]
    q = torch.randn(Bn, L, Hq, d, device=DEV, generator=g).to(torch.bfloat16)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV).view(Bn, L)
    o = torch.empty(Bn, L, Hq, d, device=DEV)
    B.kvc_decode_attn(B.model(L, Hq, Hkv, d), q=q, K=K, V=V, lens=lens_t, max_len=1500, o=o)
    torch.cuda.synchronize()
    G = Hq // Hkv
    Kn, Vn, qn, on = np64(K), np64(V), np64(q), np64(o)
    for l in range(L):
        for gg in range(Hkv):
            want = selkv.decode_attention(qn[0, l, gg * G:(gg + 1) * G], Kn[0, l, gg, :lens[l]],
                                          Vn[0, l, gg, :lens[l]])
            np.testing.assert_allclose(on[0, l, gg * G:(gg + 1) * G], want, atol=OUT_ATOL, rtol=0)


def test_decode_full_size_sampled():
    """8B shape after 20 % compression: 32 layers x 8 KV heads x 13107 kept keys, G = 4,
    the launch the benchmark times; sampled (layer, head) rows against the oracle."""
    Bn, L, Hq, Hkv, d, n = 1, 32, 32, 8, 128, 13107
    g = torch.Generator(device=DEV).manual_seed(8)
    K = torch.randn(Bn, L, Hkv, n, d, device=DEV, generator=g).to(torch.bfloat16)
    V = torch.randn(Bn, L, Hkv, n, d, device=DEV, generator=g).to(torch.bfloat16)
    q = (torch.randn(Bn, L, Hq, d, device=DEV, generator=g) * 2).to(torch.bfloat16)
    lens_t = torch.full((Bn, L), n, dtype=torch.int32, device=DEV)
    o = torch.empty(Bn, L, Hq, d, device=DEV)
    B.kvc_decode_attn(B.model(L, Hq, Hkv, d), q=q, K=K, V=V, lens=lens_t, max_len=n, o=o)
    torch.cuda.synchronize()
    assert torch.isfinite(o).all()
    G = Hq // Hkv
    for l, gg in [(0, 0), (13, 6), (31, 7)]:
        want = selkv.decode_attention(np64(q[0, l, gg * G:(gg + 1) * G]), np64(K[0, l, gg]), np64(V[0, l, gg]))
        np.testing.assert_allclose(np64(o[0, l, gg * G:(gg + 1) * G]), want, atol=OUT_ATOL, rtol=0)


def test_decode_fp32_query_bf16_cache_matches_oracle():
    """fp32 queries over a bf16 cache (the bulk-copy CUDA-core kernel), with the log R bias."""
    Bn, L, Hq, Hkv, d = 2, 2, 32, 8, 128
    lens = [2200, 1, 640, 1500]
    K, V, _, R, lens_t = _decode_case(Bn, L, Hq, Hkv, d, lens, torch.bfloat16, seed=9, with_R=True)
    q = torch.randn(Bn, L, Hq, d, device=DEV, generator=torch.Generator(device=DEV).manual_seed(10))
    o = torch.empty(Bn, L, Hq, d, device=DEV)
    B.kvc_decode_attn(B.model(L, Hq, Hkv, d), q=q, K=K, V=V, lens=lens_t, max_len=max(lens), o=o, R=R,
                      alpha_c=1.0)
    torch.cuda.synchronize()
    G = Hq // Hkv
    Kn, Vn, qn, Rn, on = np64(K), np64(V), np64(q), np64(R), np64(o)
    for b in range(Bn):
        for l in range(L):
            m_ = lens[b * L + l]
            for gg in range(Hkv):
                want = selkv.decode_attention(qn[b, l, gg * G:(gg + 1) * G], Kn[b, l, gg, :m_],
                                              Vn[b, l, gg, :m_], Rn[b, l, gg, :m_], 1.0)
                np.testing.assert_allclose(on[b, l, gg * G:(gg + 1) * G], want, atol=OUT_ATOL, rtol=0)


def test_probe_long_history_sampled():
    """RECAS probe over a 100k-token history (2 layers of the 8B shape, a quarter of the
    positions kept) in the persistent tensor-core launch; sampled heads against the oracle."""
    Bn, L, Hq, Hkv, d, T = 1, 2, 32, 8, 128, 100000
    g = torch.Generator(device=DEV).manual_seed(31)
    K = torch.randn(Bn, L, Hkv, T, d, device=DEV, generator=g).to(torch.bfloat16)
    V = torch.randn(Bn, L, Hkv, T, d, device=DEV, generator=g).to(torch.bfloat16)
    q = (torch.randn(Bn, L, Hq, d, device=DEV, generator=g) * 2).to(torch.bfloat16)
    kept = torch.rand(Bn, L, Hkv, T, device=DEV, generator=g) < 0.25
    kept[..., -32:] = True
    words = (T + 31) // 32
    pad = torch.zeros(Bn, L, Hkv, words * 32, dtype=torch.int64, device=DEV)
    pad[..., :T] = kept.to(torch.int64)
    bits = (pad.view(Bn, L, Hkv, words, 32) << torch.arange(32, device=DEV)).sum(-1)
    bits = torch.where(bits >= 2 ** 31, bits - 2 ** 32, bits).to(torch.int32).contiguous()
    lens_t = torch.full((Bn, L), T, dtype=torch.int32, device=DEV)
    shp = (Bn, L, Hq)
    delta, err, bound = (torch.empty(shp, device=DEV) for _ in range(3))
    vmax = torch.empty(Bn, L, Hkv, device=DEV)
    o = torch.empty(Bn, L, Hq, d, device=DEV)
    o_full, o_kept = torch.empty_like(o), torch.empty_like(o)
    B.kvc_decode_attn(B.model(L, Hq, Hkv, d), q=q, K=K, V=V, lens=lens_t, max_len=T, o=o, K_full=K,
                      V_full=V, lens_full=lens_t, max_len_full=T, kept_bits=bits, delta=delta,
                      vmax=vmax, err=err, bound=bound, o_full=o_full, o_kept=o_kept)
    torch.cuda.synchronize()
    G = Hq // Hkv
    for l, gg in [(0, 0), (1, 5)]:
        r = recas.dropped_mass_probe(np64(q[0, l, gg * G:(gg + 1) * G]), np64(K[0, l, gg]), np64(V[0, l, gg]),
                                     kept[0, l, gg].cpu().numpy())
        sl = slice(gg * G, (gg + 1) * G)
        assert_close_rel(np64(delta[0, l, sl]), r["delta"], rtol=1e-4, atol=1e-7, what="delta")
        assert abs(float(vmax[0, l, gg]) - r["vmax"]) <= 1e-5 * r["vmax"]
        np.testing.assert_allclose(np64(o_full[0, l, sl]), r["o_full"], atol=OUT_ATOL, rtol=0)
        np.testing.assert_allclose(np64(o_kept[0, l, sl]), r["o_kept"], atol=OUT_ATOL, rtol=0)
        assert np.all(np64(err[0, l, sl]) <= np64(bound[0, l, sl]) * (1 + 1e-4) + 1e-6)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float32])
def test_merge_edge_branches(dt):
    """Planted cases, each compared with the oracle:
      bucket 0: both kept tokens have A = 0 - the target (lower position) has zero attention,
                so nothing merges (V' = v, R = 1) and the status word says so (not an error);
      bucket 1: every evicted value is -v_target - gate 0 drops them all (V' = v, R = 1 exactly);
      bucket 2: no kept token - its evicted tokens are dropped, nothing is written for it;
      bucket 3: the only kept token is the target - an ordinary gated merge."""
    L, Hkv, d, n, bucket = 1, 2, 128, 2048, 512
    g = torch.Generator(device=DEV).manual_seed(11)
    V = torch.randn(L, Hkv, n, d, device=DEV, generator=g)
    A = torch.rand(L, Hkv, n, device=DEV, generator=g) * 1e-3 + 1e-5
    kept = np.array([5, 100, 600, 1600], np.int32)
    A[:, :, 5] = 0.0
    A[:, :, 100] = 0.0
    for j in range(512, 1024):
        if j != 600:
            V[:, :, j] = -V[:, :, 600]
    V = V.to(dt)
    k = len(kept)
    idx = torch.from_numpy(np.broadcast_to(kept, (L, Hkv, k)).copy()).to(DEV)
    kk = torch.full((L,), k, dtype=torch.int32, device=DEV)
    Vm = torch.full((L, Hkv, k, d), 7.0, dtype=dt, device=DEV)
    Vf = torch.empty(L, Hkv, k, d, device=DEV)
    R = torch.empty(L, Hkv, k, device=DEV)
    B.kvc_merge(B.model(L, 4 * Hkv, Hkv, d), n=n, V=V, A=A, idx=idx, k=kk, dst_V=Vm, R=R, bucket=bucket,
                dst_V_f32=Vf)
    code = B.kvc_check_status()                      # zero attention is reported, not an error
    assert code & 4
    Vn, An = np64(V), np64(A)
    for gg in range(Hkv):
        Vp, Rr = selkv.merge(Vn[0, gg], An[0, gg], kept, bucket)
        got_f, got_b, got_R = np64(Vf[0, gg]), np64(Vm[0, gg]), np64(R[0, gg])
        # buckets 0 and 1: bit-exact copies and R = 1 exactly
        for j in (0, 1, 2):
            assert np.array_equal(got_b[j], Vn[0, gg, kept[j]]) and got_R[j] == 1.0
            assert np.array_equal(got_f[j], Vn[0, gg, kept[j]])
        np.testing.assert_array_equal(Vp[:3], Vn[0, gg, kept[:3]])
        # bucket 3: the merge itself
        assert Rr[3] > 1.0
        np.testing.assert_allclose(got_f[3], Vp[3], atol=OUT_ATOL, rtol=0)
        assert_close_rel(got_R[3:], Rr[3:], rtol=1e-4, what="R")
        if dt == torch.bfloat16:
            assert np.all(np.abs(got_b[3] - bf16_rne(Vp[3])) <= bf16_ulp(Vp[3]))
