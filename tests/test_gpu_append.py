"""GPU: kvc_append (one generated token into every cache row) and the kept-position bits
kvc_recompress rebuilds, against their plain definitions written with torch indexing."""
import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from long_context_kv_obs_b200 import synth
from long_context_kv_obs_b200.pipeline import DecodeTimeCompressor

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits_of(words: torch.Tensor) -> np.ndarray:
    """[.., words] int32 -> [.., 32 * words] bool (bit p of word p // 32)."""
    w = words.cpu().numpy().astype(np.int64) & 0xFFFFFFFF
    return ((w[..., :, None] >> np.arange(32)) & 1).astype(bool).reshape(*w.shape[:-1], -1)


@pytest.mark.parametrize("dt,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_append_writes_every_row_and_side_array(dt, d):
    Bn, L, Hq, Hkv, cap, W = 2, 3, 8, 2, 11, 4
    m = B.model(L, Hq, Hkv, d)
    g = torch.Generator(device=DEV).manual_seed(7)
    K = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(dt)
    V = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(dt)
    lens = torch.randint(0, cap, (Bn, L), device=DEV, generator=g, dtype=torch.int32)
    lens[1, 2] = cap                                   # a full row: refused on the device
    pos_s = torch.randint(0, 1000, (Bn, L, Hkv, cap), device=DEV, generator=g, dtype=torch.int32)
    H_s = torch.rand(Bn, L, Hkv, cap, device=DEV, generator=g)
    D_s = torch.rand(Bn, L, Hkv, cap, device=DEV, generator=g)
    R_s = torch.rand(Bn, L, Hkv, cap, device=DEV, generator=g) + 2
    bits = torch.randint(-2 ** 31, 2 ** 31 - 1, (Bn, L, Hkv, 40), device=DEV, generator=g, dtype=torch.int32)
    k = torch.randn(Bn, L, Hkv, d, device=DEV, generator=g).to(dt)
    v = torch.randn(Bn, L, Hkv, d, device=DEV, generator=g).to(dt)
    q = torch.randn(Bn, L, Hq, d, device=DEV, generator=g).to(dt)
    Qring = torch.randn(Bn, L, Hq, W, d, device=DEV, generator=g).to(dt)
    qpos = torch.zeros(Bn, W, device=DEV, dtype=torch.int32)
    H_new = torch.rand(Bn, device=DEV, generator=g)
    D_lb = torch.rand(L, Bn, device=DEV, generator=g)     # [L][B]: D_new passed transposed
    pos, slot = 1234, 2
    before = [x.clone() for x in (K, V, lens, pos_s, H_s, D_s, R_s, bits, Qring)]
    B.kvc_append(m, k=k, v=v, K=K, V=V, lens=lens, pos=pos, side_pos=pos_s, side_H=H_s, side_D=D_s,
                 side_R=R_s, H_new=H_new, D_new=D_lb.t(), kept_bits=bits, q=q, Qring=Qring, qpos=qpos,
                 slot=slot)
    with pytest.raises(B.KvcError) as ei:
        B.kvc_check_status()
    assert ei.value.status == 6                       # KVC_ERR_DEVICE: the full row
    K0, V0, l0, p0, H0, D0, R0, b0, Q0 = before
    eK, eV, ep, eH, eD, eR, eb = K0.clone(), V0.clone(), p0.clone(), H0.clone(), D0.clone(), R0.clone(), b0.clone()
    el = l0.clone()
    eQ = Q0.clone()
    for b in range(Bn):
        for l in range(L):
            i = int(l0[b, l])
            if i >= cap:
                continue                               # nothing written, length unchanged
            eK[b, l, :, i] = k[b, l]
            eV[b, l, :, i] = v[b, l]
            ep[b, l, :, i] = pos
            eH[b, l, :, i] = H_new[b]
            eD[b, l, :, i] = D_lb[l, b]
            eR[b, l, :, i] = 1.0
            el[b, l] = i + 1
            eQ[b, l, :, slot] = q[b, l]
            word = eb[b, l, :, pos // 32].to(torch.int64) | (1 << (pos % 32))
            eb[b, l, :, pos // 32] = torch.where(word >= 2 ** 31, word - 2 ** 32, word).to(torch.int32)
    for got, want in ((K, eK), (V, eV), (lens, el), (pos_s, ep), (H_s, eH), (D_s, eD), (R_s, eR), (bits, eb),
                      (Qring, eQ)):
        assert torch.equal(got, want)
    assert torch.equal(qpos[:, slot], torch.full((Bn,), pos, device=DEV, dtype=torch.int32))
    assert torch.equal(qpos[:, :slot], torch.zeros(Bn, slot, device=DEV, dtype=torch.int32))


def test_append_second_cache_in_the_same_launch():
    """The full history the probe reads, appended in the same launch (K2, V2, lens2), equals a
    second kvc_append into it; a second cache at capacity leaves both caches unwritten."""
    Bn, L, Hq, Hkv, d, cap, cap2 = 3, 2, 8, 2, 128, 9, 17
    m = B.model(L, Hq, Hkv, d)
    g = torch.Generator(device=DEV).manual_seed(11)
    dt = torch.bfloat16
    K = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(dt)
    V = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(dt)
    Kf = torch.randn(Bn, L, Hkv, cap2, d, device=DEV, generator=g).to(dt)
    Vf = torch.randn(Bn, L, Hkv, cap2, d, device=DEV, generator=g).to(dt)
    lens = torch.randint(0, cap, (Bn, L), device=DEV, generator=g, dtype=torch.int32)
    lens2 = torch.randint(0, cap2, (Bn, L), device=DEV, generator=g, dtype=torch.int32)
    k = torch.randn(Bn, L, Hkv, d, device=DEV, generator=g).to(dt)
    v = torch.randn(Bn, L, Hkv, d, device=DEV, generator=g).to(dt)
    ref = [x.clone() for x in (K, V, Kf, Vf, lens, lens2)]
    B.kvc_append(m, k=k, v=v, K=ref[0], V=ref[1], lens=ref[4], pos=40)
    B.kvc_append(m, k=k, v=v, K=ref[2], V=ref[3], lens=ref[5], pos=40)
    n0 = B.kvc_launch_count()
    B.kvc_append(m, k=k, v=v, K=K, V=V, lens=lens, pos=40, K2=Kf, V2=Vf, lens2=lens2)
    assert B.kvc_launch_count() - n0 == 1
    assert B.kvc_check_status() == 0
    for got, want in zip((K, V, Kf, Vf, lens, lens2), ref):
        assert torch.equal(got, want)
    # one (sequence, layer) of the second cache full: neither cache of it is written
    lens2[1, 0] = cap2
    before = [x.clone() for x in (K, V, Kf, Vf, lens, lens2)]
    B.kvc_append(m, k=k, v=v, K=K, V=V, lens=lens, pos=41, K2=Kf, V2=Vf, lens2=lens2)
    with pytest.raises(B.KvcError) as ei:
        B.kvc_check_status()
    assert ei.value.status == 6                       # KVC_ERR_DEVICE: the full row
    K0, V0, Kf0, Vf0, l0, l20 = before
    assert torch.equal(K[1, 0], K0[1, 0]) and torch.equal(V[1, 0], V0[1, 0])
    assert torch.equal(Kf[1, 0], Kf0[1, 0]) and torch.equal(Vf[1, 0], Vf0[1, 0])
    assert int(lens[1, 0]) == int(l0[1, 0]) and int(lens2[1, 0]) == cap2
    others = torch.ones(Bn, L, dtype=torch.bool, device=DEV)
    others[1, 0] = False
    assert torch.equal(lens[others], l0[others] + 1) and torch.equal(lens2[others], l20[others] + 1)


def test_append_validation():
    m = B.model(2, 4, 2, 128)
    K = torch.zeros(1, 2, 2, 8, 128, device=DEV, dtype=torch.bfloat16)
    k = torch.zeros(1, 2, 2, 128, device=DEV, dtype=torch.bfloat16)
    lens = torch.zeros(1, 2, device=DEV, dtype=torch.int32)
    bits = torch.zeros(1, 2, 2, 2, device=DEV, dtype=torch.int32)
    with pytest.raises(B.KvcError):            # position past the bit words
        B.kvc_append(m, k=k, v=k, K=K, V=K.clone(), lens=lens, pos=64, kept_bits=bits)
    with pytest.raises(B.KvcError):            # ring slot outside [0, W)
        B.kvc_append(m, k=k, v=k, K=K, V=K.clone(), lens=lens, pos=3, q=torch.zeros(1, 2, 4, 128, device=DEV,
                     dtype=torch.bfloat16), Qring=torch.zeros(1, 2, 4, 2, 128, device=DEV, dtype=torch.bfloat16),
                     qpos=torch.zeros(1, 2, device=DEV, dtype=torch.int32), slot=2)
    assert int(lens.sum()) == 0


def test_decode_time_bookkeeping_runs_only_library_kernels():
    """Append, decode (with the probe) and recompression of the decode-time workload launch
    only libkvc kernels: the kernels a CUDA profiler sees are the library's, as many as its
    own launch count; the kept bits after a recompression are exactly the kept positions."""
    wl = synth.WORKLOADS[4].scaled(n_layers=2, n=200, batch=2, gen_tokens=80, period=40, W=8, w=8)
    Bn, L, n0 = wl.batch, wl.n_layers, wl.n
    g = torch.Generator(device=DEV).manual_seed(3)
    Kp = torch.randn(Bn, L, wl.n_kv_heads, n0, wl.head_dim, device=DEV, generator=g).to(wl.dtype)
    Vp = torch.randn(Bn, L, wl.n_kv_heads, n0, wl.head_dim, device=DEV, generator=g).to(wl.dtype)
    dc = DecodeTimeCompressor(wl, Kp, Vp, torch.rand(Bn, n0, device=DEV) * 4,
                              torch.rand(Bn, L, n0, device=DEV) + 1, probe=True)
    steps = []
    for s in range(wl.period):
        q = synth.gen_decode_queries(wl, 5, s, DEV)
        k, v = synth.gen_decode_kv(wl, 5, s, DEV)
        steps.append((q, k, v, torch.rand(Bn, device=DEV), torch.rand(Bn, L, device=DEV) + 1))
    torch.cuda.synchronize()
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        n0_launch = B.kvc_launch_count()
        for (q, k, v, Hn, Dn) in steps:
            dc.append(k, v, Hn, Dn, q)
            dc.attend(q, probe=True)
        assert dc.due()
        keep = dc.recompress()
        torch.cuda.synchronize()
        launched = B.kvc_launch_count() - n0_launch
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA
             and "memset" not in e.name.lower() and "memcpy" not in e.name.lower()]
    assert names and all("kvc::" in nm for nm in names), sorted(set(nm for nm in names if "kvc::" not in nm))
    assert len(names) == launched
    assert B.kvc_check_status() == 0
    # kept bits: exactly the positions the compressed cache holds
    pos = dc.pos[dc.cur, :, :, :, :keep].cpu().numpy()
    got = _bits_of(dc.bits)
    want = np.zeros_like(got)
    for b in range(Bn):
        for l in range(L):
            for h in range(wl.n_kv_heads):
                want[b, l, h, pos[b, l, h]] = True
    assert np.array_equal(got, want)
    assert int(dc.lens.min()) == keep == int(dc.lens.max())
