"""GPU parity: budgets, top-k selection (exact on identical fp32 scores) and compaction (bit-exact)."""
import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from oracle import infokv as ik
from tests.helpers import np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def synthetic_scores(L, Hkv, n, seed, ties=False):
    g = torch.Generator(device=DEV).manual_seed(seed)
    S = torch.rand(L, Hkv, n, device=DEV, generator=g) ** 3 * 1e-3
    if ties:
        S = torch.round(S * 2e4) / 2e4          # many exactly equal scores
    return S.contiguous()


def gpu_select(L, Hq, Hkv, n, w, S, budget="uniform", rho=0.25, k_in=None, B_total=0, Ebar=None,
               union=False, k_cap=None):
    m = B.model(L, Hq, Hkv, 128)
    k = torch.empty(L, dtype=torch.int32, device=DEV)
    k_cap = k_cap or n
    idx = torch.full((L, Hkv, k_cap), -7, dtype=torch.int32, device=DEV)
    mode = {"uniform": B.BUDGET_UNIFORM, "explicit": B.BUDGET_EXPLICIT, "adaptive": B.BUDGET_ADAPTIVE}[budget]
    B.kvc_select(m, n=n, w=w, S=S, k_out=k, idx=idx, sel_mode=B.SEL_GQA_UNION if union else B.SEL_PER_KV_HEAD,
                 budget_mode=mode, rho=rho, k_in=k_in, B_total=B_total, Ebar=Ebar)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    return k.cpu().numpy(), idx.cpu().numpy()


@pytest.mark.parametrize("n,w,rho,ties", [(512, 16, 0.25, False), (3000, 32, 0.4, True),
                                          (65536, 64, 0.2, False), (100000, 32, 0.25, True),
                                          (40, 64, 0.5, False), (1000, 0, 0.0, False),
                                          (1000, 10, 1.0, True)])
def test_select_per_head_is_exact(n, w, rho, ties):
    L, Hkv = 2, 3
    S = synthetic_scores(L, Hkv, n, seed=n + w, ties=ties)
    k, idx = gpu_select(L, 6, Hkv, n, w, S, rho=rho)
    kref = ik.uniform_budgets(n, rho, L, w)
    np.testing.assert_array_equal(k, kref)
    Sn = np64(S)
    for l in range(L):
        for g in range(Hkv):
            want = ik.select_topk(Sn[l, g], int(kref[l]), w)
            np.testing.assert_array_equal(idx[l, g, :len(want)], want)


def test_select_union_is_exact_and_shared_by_heads():
    L, Hkv, n, w = 3, 8, 16384, 32
    S = synthetic_scores(L, Hkv, n, seed=3)
    k, idx = gpu_select(L, 24, Hkv, n, w, S, rho=0.4, union=True)
    Sn = np64(S)
    for l in range(L):
        want = ik.select_topk(ik.union_max(Sn[l]), int(k[l]), w)
        for g in range(Hkv):
            np.testing.assert_array_equal(idx[l, g, :len(want)], want)


def test_adaptive_and_explicit_budgets():
    L, Hkv, n, w = 32, 2, 4096, 64
    S = synthetic_scores(L, Hkv, n, seed=9)
    g = torch.Generator(device=DEV).manual_seed(1)
    Ebar = (torch.rand(L, device=DEV, generator=g) * 2 + 0.5).contiguous()
    Btot = L * 819
    k, idx = gpu_select(L, 4, Hkv, n, w, S, budget="adaptive", B_total=Btot, Ebar=Ebar)
    kref = ik.adaptive_budgets(np64(Ebar), Btot, w, n)
    assert k.sum() == Btot
    # identical fp32 E-bar on both sides: identical integer decisions
    np.testing.assert_array_equal(k, kref)
    Sn = np64(S)
    for l in range(L):
        for gg in range(Hkv):
            np.testing.assert_array_equal(idx[l, gg, :k[l]], ik.select_topk(Sn[l, gg], int(k[l]), w))
    # skewed shares with both bounds active
    Ebar2 = torch.tensor([1e-4] * 4 + [1.0] * 27 + [500.0], device=DEV)
    Btot2 = 32 * 600
    k2, _ = gpu_select(L, 4, Hkv, n, w, S, budget="adaptive", B_total=Btot2, Ebar=Ebar2)
    np.testing.assert_array_equal(k2, ik.adaptive_budgets(np64(Ebar2), Btot2, w, n))
    kin = torch.arange(L, dtype=torch.int32, device=DEV) * 150
    k3, idx3 = gpu_select(L, 4, Hkv, n, w, S, budget="explicit", k_in=kin)
    np.testing.assert_array_equal(k3, np.clip(np64(kin), w, n))


def test_compaction_is_bit_exact_with_side_arrays():
    L, Hkv, n, d, kc = 3, 4, 5000, 128, 1300
    g = torch.Generator(device=DEV).manual_seed(2)
    for dt in (torch.bfloat16, torch.float32):
        K = torch.randn(L, Hkv, n, d, device=DEV, generator=g).to(dt)
        V = torch.randn(L, Hkv, n, d, device=DEV, generator=g).to(dt)
        pos = (torch.arange(n, device=DEV, dtype=torch.int32) * 3 + 11).repeat(L, Hkv, 1).contiguous()
        Hs = torch.rand(n, device=DEV, generator=g)
        Ds = torch.rand(L, n, device=DEV, generator=g)
        idx = torch.stack([torch.sort(torch.randperm(n, device=DEV, generator=g)[:kc])[0]
                           for _ in range(L * Hkv)]).view(L, Hkv, kc).to(torch.int32)
        k = torch.tensor([kc, kc - 7, 1], dtype=torch.int32, device=DEV)
        Kc = torch.zeros(L, Hkv, kc, d, dtype=dt, device=DEV)
        Vc = torch.zeros_like(Kc)
        pc = torch.full((L, Hkv, kc), -1, dtype=torch.int32, device=DEV)
        hc = torch.zeros(L, Hkv, kc, device=DEV)
        dc = torch.zeros(L, Hkv, kc, device=DEV)
        m = B.model(L, Hkv, Hkv, d)
        B.kvc_compact(m, n=n, idx=idx, k=k, src_K=K, src_V=V, dst_K=Kc, dst_V=Vc, src_pos=pos,
                      pos_strides=(Hkv * n, n), dst_pos=pc, src_H=Hs, H_strides=(0, 0), dst_H=hc,
                      src_D=Ds, D_strides=(n, 0), dst_D=dc)
        torch.cuda.synchronize()
        for l in range(L):
            kl = int(k[l])
            for gg in range(Hkv):
                ii = idx[l, gg, :kl].long()
                assert torch.equal(Kc[l, gg, :kl], K[l, gg, ii])
                assert torch.equal(Vc[l, gg, :kl], V[l, gg, ii])
                assert torch.equal(pc[l, gg, :kl], pos[l, gg, ii])
                assert torch.equal(hc[l, gg, :kl], Hs[ii])
                assert torch.equal(dc[l, gg, :kl], Ds[l, ii])
                assert torch.all(Kc[l, gg, kl:] == 0)        # rows past k_l untouched
    # identity compaction (k = n)
    idx = torch.arange(n, dtype=torch.int32, device=DEV).repeat(L, Hkv, 1).contiguous()
    k = torch.full((L,), n, dtype=torch.int32, device=DEV)
    Kc = torch.empty_like(K)
    B.kvc_compact(m, n=n, idx=idx, k=k, src_K=K, dst_K=Kc)
    torch.cuda.synchronize()
    assert torch.equal(Kc, K)


def test_compaction_flags_out_of_range_indices():
    L, Hkv, n, d = 1, 1, 64, 128
    K = torch.randn(L, Hkv, n, d, device=DEV).to(torch.bfloat16)
    idx = torch.tensor([[[0, 5, 70, 3]]], dtype=torch.int32, device=DEV)   # 70 >= n
    k = torch.tensor([4], dtype=torch.int32, device=DEV)
    Kc = torch.zeros(L, Hkv, 4, d, dtype=torch.bfloat16, device=DEV)
    B.kvc_compact(B.model(1, 1, 1, d), n=n, idx=idx, k=k, src_K=K, dst_K=Kc)
    with pytest.raises(B.KvcError) as e:
        B.kvc_check_status()
    assert e.value.status == 6
    assert torch.equal(Kc[0, 0, 1], K[0, 0, 5]) and torch.all(Kc[0, 0, 2] == 0)
    assert B.kvc_check_status() == 0                    # the word was cleared
