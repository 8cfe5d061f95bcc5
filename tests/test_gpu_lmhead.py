"""GPU parity: top-k entropy from the LM head's input (kvc_lmhead_entropy) against the
fp64 oracle (oracle/infokv.py lmhead_topk_entropy).

Tolerance, derived per row.  The GPU logits are fp32 sums of exact bf16 products, so
each is within dz = gamma_Dh * max_v sum_d |x_d W_vd| of the exact one (gamma_m = m u /
(1 - m u), u = 2^-24).  For a fixed top-k set, dH = -sum_i p_i (dz_i - sum_j p_j dz_j)
log p_i, so |dH| <= 2 max|dz| H.  The GPU's top-k set can differ from the exact one only
by values within 2 dz of the k-th largest, the same as moving each of those by at most
2 dz more: with |dz_i| <= 3 dz, |dH| <= 6 dz H.  The fp32 exponentials and logarithm of
the entropy itself add at most 1e-4 H + 1e-5, the bound the logits-row kernel's tests
use.  Bound: |H_gpu - H| <= 6 dz H + 1e-4 H + 1e-5.
"""
import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from long_context_kv_obs_b200 import synth
from oracle import infokv as ik
from tests.helpers import np64

pytestmark = pytest.mark.gpu
DEV = "cuda"
U = 2.0 ** -24


def _bound(x, W, H):
    """Per-row tolerance of the module docstring; x [n][Dh], W [V][Dh] float64."""
    Dh = x.shape[1]
    gamma = Dh * U / (1 - Dh * U)
    dz = gamma * (np.abs(x) @ np.abs(W).T).max(axis=1)
    return 6 * dz * H + 1e-4 * H + 1e-5


def _check(x_t, W_t, H_t, k, rows=None):
    x, W = np64(x_t), np64(W_t)
    if rows is not None:
        x = x[rows]
    ref = ik.lmhead_topk_entropy(x, W, k)
    got = np64(H_t) if rows is None else np64(H_t)[rows]
    tol = _bound(x, W, ref)
    err = np.abs(got - ref)
    assert np.all(err <= tol), f"max err {err.max():.3e} at row {err.argmax()}, tol there {tol[err.argmax()]:.3e}"
    return err


@pytest.mark.parametrize("n,Dh,V,k", [
    (300, 512, 5000, 256),        # ragged M and N tiles, 8 K slices
    (129, 136, 3001, 100),        # Dh past a 64-wide slice, k < 256
    (64, 256, 200, 256),          # fewer logits than k: the whole row
    (1000, 1024, 32768, 256),     # several vocabulary segments
    (1, 64, 1, 256),              # one row, one logit: H = 0
])
def test_lmhead_entropy_matches_oracle(n, Dh, V, k):
    x, W = synth.gen_lmhead(n, Dh, V, seed=n + V, device=DEV)
    H = torch.full((n,), float("nan"), device=DEV)
    B.kvc_lmhead_entropy(x=x, W=W, H=H, k=k)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    _check(x, W, H, k)


def test_lmhead_entropy_ties_and_strided_rows():
    """W rows repeat (many equal logits at the k-th value); x is a view with a wider row stride."""
    n, Dh, V = 257, 320, 4000
    x_wide, W0 = synth.gen_lmhead(n, Dh + 64, 50, seed=5, device=DEV)
    x = x_wide[:, :Dh]
    W = W0[torch.arange(V, device=DEV) % 50, :Dh].contiguous()
    H = torch.empty(n, device=DEV)
    B.kvc_lmhead_entropy(x=x, W=W, H=H, k=256)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    _check(x, W, H, 256)


def test_lmhead_entropy_agrees_with_the_logits_row_kernel():
    """The same H through kvc_score's entropy pass over logits materialised by the oracle's
    own fp64 product (rounded to fp32): both kernels see the same top-k sets up to ties."""
    n, Dh, V = 200, 256, 9000
    x, W = synth.gen_lmhead(n, Dh, V, seed=11, device=DEV)
    H = torch.empty(n, device=DEV)
    B.kvc_lmhead_entropy(x=x, W=W, H=H, k=256)
    z = torch.from_numpy(np64(x) @ np64(W).T).to(DEV, torch.float32)
    m = B.model(1, 1, 1, 128)
    Hz = torch.empty(n, device=DEV)
    B.kvc_score(m, mode=B.SCORE_INFOKV, n=n, W=0, Qw=torch.zeros(1, 128, dtype=torch.bfloat16, device=DEV),
                K=torch.zeros(1, 1, n, 128, dtype=torch.bfloat16, device=DEV), S=None, logits=z, H_out=Hz)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    tol = _bound(np64(x), np64(W), np64(Hz))
    assert np.all(np.abs(np64(H) - np64(Hz)) <= tol)


def test_lmhead_entropy_full_size_sampled():
    """The 8B shape at 64k positions (Dh 4096, vocab 128256), as the bench runs it; 12 rows
    compared with the oracle, the rest checked to lie in [0, ln 256]."""
    n, Dh, V = 65536, 4096, 128256
    x, W = synth.gen_lmhead(n, Dh, V, seed=3, device=DEV)
    H = torch.full((n,), float("nan"), device=DEV)
    ws = B.kvc_lmhead_entropy(x=x, W=W, H=H, k=256)
    torch.cuda.synchronize()
    assert B.kvc_check_status() == 0
    Hn = np64(H)
    assert np.all(np.isfinite(Hn)) and np.all(Hn >= 0) and np.all(Hn <= np.log(256) + 1e-5)
    rows = np.array([0, 1, 127, 128, 4095, 20000, 32767, 40000, 50001, 65407, 65408, n - 1])
    xs = np64(x[torch.from_numpy(rows).to(DEV)])
    Wc = W.cpu()
    zs, absW = [], np.zeros(len(rows))
    for v0 in range(0, V, 16384):                 # the sampled rows' fp64 logits, in vocabulary chunks
        Wk = Wc[v0:v0 + 16384].float().numpy().astype(np.float64)
        zs.append(xs @ Wk.T)
        absW = np.maximum(absW, (np.abs(xs) @ np.abs(Wk).T).max(axis=1))
    Href = ik.topk_entropy(np.concatenate(zs, axis=1), 256)
    gamma = Dh * U / (1 - Dh * U)
    tol = 6 * gamma * absW * Href + 1e-4 * Href + 1e-5
    assert np.all(np.abs(Hn[rows] - Href) <= tol), (Hn[rows] - Href, tol)
    del ws
