"""GPU parity: SelKV RoPE re-positioning of the kept keys against the fp64 oracle.

Tolerance, from the arithmetic: the kernel reduces each angle modulo pi/2 in
fp64 and turns the pair in fp32, with sine and cosine of the reduced angle from
their Taylor series (truncation below 1e-7).  Rounding the reduced angle to fp32
and the series together leave an angle error below 2e-7 rad, so an output may
differ from the fp64 value by 4e-7 * (|x_i| + |x_{i+d/2}|) of its input pair,
plus one bf16 ulp where the result is stored as bf16.
"""
import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from oracle import selkv
from tests.helpers import bf16_ulp, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _positions(L, Hkv, k_cap, n, seed):
    """Ascending distinct positions < n per (l, g), like the kept lists of a selection."""
    rng = np.random.default_rng(seed)
    pos = np.zeros((L, Hkv, k_cap), np.int32)
    for l in range(L):
        for g in range(Hkv):
            pos[l, g] = np.sort(rng.choice(n, size=k_cap, replace=False))
    return pos


def _limit(x, dt):
    """Per-element tolerance of the turned pair (see the module docstring)."""
    h = x.shape[-1] // 2
    pair = np.abs(x[..., :h]) + np.abs(x[..., h:])
    lim = 4e-7 * np.concatenate([pair, pair], axis=-1) + 1e-30
    return lim


def _check_rows(got, x, old, new, base, dt, what):
    ref = selkv.rope_reposition(x, old, new, base)
    lim = _limit(x, dt)
    if dt == torch.bfloat16:
        lim = lim + bf16_ulp(ref)
    err = np.abs(got - ref)
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside; worst at {i}: "
                             f"gpu={got[i]!r} ref={ref[i]!r} lim={lim[i]!r}")


@pytest.mark.parametrize("L,Hkv,d,k_cap,dt,in_place,base", [
    (3, 2, 128, 300, torch.bfloat16, False, 10000.0),   # ragged k: full, 17 rows, none
    (2, 4, 64, 129, torch.float32, True, 500000.0),     # d 64, fp32, in place
    (2, 1, 64, 77, torch.bfloat16, True, 10000.0),      # d 64 bf16: four lanes a row
    (1, 3, 128, 1000, torch.float32, False, 1000000.0),  # d 128 fp32: sixteen lanes a row
])
def test_rope_reposition_matches_oracle(L, Hkv, d, k_cap, dt, in_place, base):
    n = 100000
    g = torch.Generator(device=DEV).manual_seed(L * 100 + d + k_cap)
    K = (torch.randn(L, Hkv, k_cap, d, device=DEV, generator=g) * 2).to(dt)
    x = np64(K)
    pos_np = _positions(L, Hkv, k_cap, n, seed=k_cap)
    pos = torch.from_numpy(pos_np).to(DEV)
    kl = [k_cap, 17, 0][:L] if L == 3 else [k_cap] * (L - 1) + [k_cap // 2]
    k = torch.tensor(kl, dtype=torch.int32, device=DEV)
    new0 = 5
    pos_dst = torch.full_like(pos, -7)
    K_dst = None if in_place else torch.full_like(K, 3.0)
    B.kvc_rope_reposition(B.model(L, Hkv, Hkv, d), K=K, pos=pos, k=k, base=base, new0=new0,
                          K_dst=K_dst, pos_dst=pos_dst)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    out = np64(K if in_place else K_dst)
    pd = pos_dst.cpu().numpy()
    for l in range(L):
        kk = kl[l]
        new = new0 + np.arange(kk)
        for gg in range(Hkv):
            _check_rows(out[l, gg, :kk], x[l, gg, :kk], pos_np[l, gg, :kk], new, base, dt, f"({l},{gg})")
            np.testing.assert_array_equal(pd[l, gg, :kk], new)
            assert np.all(pd[l, gg, kk:] == -7)
            # rows past k_l are not touched
            rest = x[l, gg, kk:] if in_place else np.full_like(x[l, gg, kk:], 3.0)
            np.testing.assert_array_equal(out[l, gg, kk:], rest)


def test_rope_already_contiguous_is_identity_and_in_place_positions():
    """Keys already at new0 + j come back bit for bit; positions updated in place."""
    L, Hkv, d, k_cap = 2, 2, 128, 500
    g = torch.Generator(device=DEV).manual_seed(5)
    K = torch.randn(L, Hkv, k_cap, d, device=DEV, generator=g).to(torch.bfloat16)
    K0 = K.clone()
    pos = (torch.arange(k_cap, dtype=torch.int32, device=DEV) + 11).expand(L, Hkv, k_cap).contiguous()
    k = torch.full((L,), k_cap, dtype=torch.int32, device=DEV)
    B.kvc_rope_reposition(B.model(L, Hkv, Hkv, d), K=K, pos=pos, k=k, base=10000.0, new0=11, pos_dst=pos)
    torch.cuda.synchronize()
    assert torch.equal(K, K0)
    # shifting every key by -11 then, in place, the positions
    B.kvc_rope_reposition(B.model(L, Hkv, Hkv, d), K=K, pos=pos, k=k, base=10000.0, new0=0, pos_dst=pos)
    torch.cuda.synchronize()
    assert torch.equal(pos[0, 0], torch.arange(k_cap, dtype=torch.int32, device=DEV))
    _check_rows(np64(K)[1, 1], np64(K0)[1, 1], np.arange(k_cap) + 11, np.arange(k_cap), 10000.0,
                torch.bfloat16, "shift by -11")


def test_rope_strided_rows_and_composition():
    """Rows inside a wider buffer (s_tok > d) and into a second buffer; turning A -> B -> C
    agrees with A -> C."""
    L, Hkv, d, k_cap, base = 2, 2, 128, 260, 500000.0
    g = torch.Generator(device=DEV).manual_seed(9)
    big = torch.randn(L, Hkv, k_cap, 192, device=DEV, generator=g)
    big0 = big.clone()
    K = big[..., :128]
    x = np64(K)
    pos_np = _positions(L, Hkv, k_cap, 60000, seed=9)
    pos = torch.from_numpy(pos_np).to(DEV)
    k = torch.full((L,), k_cap, dtype=torch.int32, device=DEV)
    m = B.model(L, Hkv, Hkv, d)
    mid = torch.empty(L, Hkv, k_cap, d, device=DEV)
    B.kvc_rope_reposition(m, K=K, pos=pos, k=k, base=base, new0=40000, K_dst=mid)
    mid_pos = (torch.arange(k_cap, dtype=torch.int32, device=DEV) + 40000).expand(L, Hkv, k_cap).contiguous()
    two = torch.empty_like(mid)
    B.kvc_rope_reposition(m, K=mid, pos=mid_pos, k=k, base=base, new0=3, K_dst=two)
    one = torch.empty_like(mid)
    B.kvc_rope_reposition(m, K=K, pos=pos, k=k, base=base, new0=3, K_dst=one)
    torch.cuda.synchronize()
    assert torch.equal(big, big0)                     # the source is only read
    for l in range(L):
        for gg in range(Hkv):
            _check_rows(np64(one)[l, gg], x[l, gg], pos_np[l, gg], 3 + np.arange(k_cap), base,
                        torch.float32, f"one ({l},{gg})")
    lim = 2 * _limit(x, torch.float32)
    assert np.all(np.abs(np64(two) - np64(one)) <= lim + 1e-6)


def test_rope_full_size_sampled():
    """The SelKV 100k shape: 32 layers x 8 KV heads x 25000 kept keys (bf16, in place).
    Sampled rows match the oracle; every pair keeps its norm to bf16 rounding."""
    L, Hkv, d, k_cap, n = 32, 8, 128, 25000, 100000
    g = torch.Generator(device=DEV).manual_seed(100)
    K = torch.randn(L, Hkv, k_cap, d, device=DEV, generator=g).to(torch.bfloat16)
    K0 = K.clone()
    pos = torch.sort(torch.randint(0, n, (L, Hkv, k_cap), device=DEV, generator=g,
                                   dtype=torch.int32), dim=-1)[0].contiguous()
    k = torch.full((L,), k_cap, dtype=torch.int32, device=DEV)
    B.kvc_rope_reposition(B.model(L, 4 * Hkv, Hkv, d), K=K, pos=pos, k=k, base=500000.0)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    rng = np.random.default_rng(7)
    for _ in range(64):
        l, gg, j = int(rng.integers(L)), int(rng.integers(Hkv)), int(rng.integers(k_cap))
        _check_rows(np64(K[l, gg, j]), np64(K0[l, gg, j]), int(pos[l, gg, j]), j, 500000.0,
                    torch.bfloat16, f"row ({l},{gg},{j})")
    # norm of every pair, over all 6.4 M rows: |y|^2 = |x|^2 up to the bf16 rounding of y
    y, x0 = K.float(), K0.float()
    ny = y[..., :64] ** 2 + y[..., 64:] ** 2
    nx = x0[..., :64] ** 2 + x0[..., 64:] ** 2
    assert torch.all((ny - nx).abs() <= nx * 2 ** -6 + 1e-30)


def test_prefill_compressor_reposition_step():
    """SelKV step 6 through the pipeline: after score / select / compact, the compacted keys
    are re-embedded in place at new0 + j from the positions their kept lists hold."""
    from long_context_kv_obs_b200 import synth
    from long_context_kv_obs_b200.pipeline import PrefillCompressor
    wl = synth.WORKLOADS[3].scaled(n_layers=2, n=3000, vocab=1000, hidden=256)
    inp = synth.gen_prefill(wl, seed=31, device=DEV, with_logits=False, with_hidden=False)
    pc = PrefillCompressor(wl, inp)
    pc.run()
    torch.cuda.synchronize()
    K0 = np64(pc.Kc)
    pos_out = torch.full_like(pc.idx, -1)
    pc.reposition(new0=100, pos_dst=pos_out)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    idx, k, got, pout = pc.idx.cpu().numpy(), pc.k.cpu().numpy(), np64(pc.Kc), pos_out.cpu().numpy()
    for l in range(wl.n_layers):
        kl = int(k[l])
        for gg in range(wl.n_kv_heads):
            _check_rows(got[l, gg, :kl], K0[l, gg, :kl], idx[l, gg, :kl], 100 + np.arange(kl),
                        wl.rope_base, wl.dtype, f"({l},{gg})")
            np.testing.assert_array_equal(pout[l, gg, :kl], 100 + np.arange(kl))
