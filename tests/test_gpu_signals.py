"""GPU parity: top-k entropy (H), representation change (D) and their softmax statistics."""
import math

import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from long_context_kv_obs_b200 import synth
from oracle import infokv as ik
from tests.helpers import assert_close_rel, np64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gpu_entropy(logits: torch.Tensor, k: int, row_stride=None):
    """H via kvc_score's entropy stage (ATTN-free: a minimal InfoKV score call)."""
    n = logits.shape[0]
    L, Hq, Hkv, d, W = 1, 1, 1, 64, 1
    m = B.model(L, Hq, Hkv, d)
    K = torch.randn(L, Hkv, n, d, device=DEV)
    Qw = torch.randn(L, Hq, W, d, device=DEV)
    S = torch.empty(L, Hkv, n, device=DEV)
    H = torch.empty(n, device=DEV)
    D_in = torch.ones(L, n, device=DEV)
    B.kvc_score(m, mode=B.SCORE_INFOKV, n=n, W=W, Qw=Qw, K=K, S=S, logits=logits, D_in=D_in,
                D_strides=(n, 0), topk=k, H_out=H)
    torch.cuda.synchronize()
    return H


# Up to 512 rows of a long vocabulary take the split-row kernels (chunks spread over the
# GPU, then a merge per row); 600 rows take the row-per-warp kernel.
@pytest.mark.parametrize("dtype,V,k,rows", [(torch.bfloat16, 128256, 256, 96), (torch.float32, 1000, 256, 96),
                                            (torch.bfloat16, 152064, 256, 96), (torch.float32, 200, 256, 96),
                                            (torch.bfloat16, 3000, 64, 96), (torch.float32, 5000, 1024, 96),
                                            (torch.bfloat16, 152064, 256, 600), (torch.float32, 50000, 1024, 600),
                                            (torch.bfloat16, 152064, 256, 8), (torch.bfloat16, 152064, 1024, 1), (torch.bfloat16, 152064, 512, 3),
                                            (torch.float32, 128256, 256, 512), (torch.bfloat16, 16384, 1, 33)])
def test_entropy_matches_oracle(dtype, V, k, rows):
    logits = synth.gen_logits(rows, V, dtype, seed=7, device=DEV, dominant=True)
    H = gpu_entropy(logits, k)
    ref = ik.topk_entropy(np64(logits), k)
    assert_close_rel(np64(H), ref, rtol=1e-4, atol=1e-5, what="H")


def test_entropy_adversarial_rows():
    V = 20000
    rows = []
    rows.append(torch.arange(V, dtype=torch.float32) * 1e-3)                  # ascending: prune every step
    rows.append(-torch.arange(V, dtype=torch.float32) * 1e-3)                 # descending
    rows.append(torch.full((V,), 2.5))                                        # all equal: H = ln 256
    r = torch.zeros(V); r[::7] = 1.0                                          # heavy ties at the threshold
    rows.append(r)
    r = torch.randn(V) * 0.01; r[123] = 40.0                                  # one dominant logit
    rows.append(r)
    r = torch.full((V,), -1e30); r[:10] = torch.arange(10.0)                  # fewer than k distinct big values
    rows.append(r)
    r = torch.full((V,), float("-inf")); r[5000:5100] = torch.randn(100)      # masked: 100 finite logits
    rows.append(r)
    rows.append(torch.full((V,), float("-inf")))                              # every logit masked: H = 0
    x = torch.stack(rows).to(DEV)
    for reps in (1, 100):   # split-row kernels, then the row-per-warp kernel
        for dt in (torch.float32, torch.bfloat16):
            xd = x.repeat(reps, 1).to(dt)
            H = gpu_entropy(xd, 256)
            ref = ik.topk_entropy(np64(xd), 256)
            assert_close_rel(np64(H), ref, rtol=1e-4, atol=2e-5, what=f"H adversarial {dt} x{reps}")
            assert abs(float(H[2]) - math.log(256)) < 1e-4
            assert float(H[7]) == 0.0


@pytest.mark.parametrize("dtype,V", [(torch.bfloat16, 100003), (torch.float32, 70001), (torch.bfloat16, 8193)])
def test_entropy_split_rows_with_a_ragged_end(dtype, V):
    """Split-row path on rows whose length is no multiple of the 16-byte vector: a padded
    pitch keeps the rows aligned, the last values of each row go through scalar loads, and
    the pitch's padding (set to a huge logit here) must not be read."""
    rows = 8
    pitch = (V + 63) // 64 * 64
    big = torch.full((rows, pitch), 1e4, device=DEV, dtype=dtype)
    big[:, :V] = synth.gen_logits(rows, V, dtype, seed=11, device=DEV, dominant=True)
    big[3, V - 1] = 60.0                 # the largest logit is the last value of a row
    view = big[:, :V]
    H = gpu_entropy(view, 256)
    assert_close_rel(np64(H), ik.topk_entropy(np64(view), 256), rtol=1e-4, atol=1e-5, what="H")


def test_entropy_unaligned_rows_take_the_scalar_path():
    V, rows = 1003, 40                                 # 1003 * 2 bytes: rows not 16-byte aligned
    logits = synth.gen_logits(rows, V, torch.bfloat16, seed=3, device=DEV, dominant=True)
    H = gpu_entropy(logits, 256)
    assert_close_rel(np64(H), ik.topk_entropy(np64(logits), 256), rtol=1e-4, atol=1e-5, what="H")
    # strided view: a padded row pitch
    big = synth.gen_logits(rows, 1024, torch.float32, seed=4, device=DEV, dominant=False)
    view = big[:, :1000]
    H = gpu_entropy(view, 256)
    assert_close_rel(np64(H), ik.topk_entropy(np64(view), 256), rtol=1e-4, atol=1e-5, what="H")


@pytest.mark.parametrize("dtype,Dh,L,n", [(torch.float32, 256, 2, 512), (torch.bfloat16, 3072, 3, 700),
                                          (torch.bfloat16, 4096, 4, 333), (torch.bfloat16, 3584, 2, 100),
                                          (torch.bfloat16, 3584, 28, 8), (torch.float32, 2048, 5, 1),
                                          (torch.float32, 2048, 3, 7000)])
def test_repr_change_matches_oracle(dtype, Dh, L, n):
    hidden = synth.gen_hidden(L, n, Dh, dtype, seed=5, device=DEV)
    m = B.model(L, 2, 1, 64)
    K = torch.randn(L, 1, n, 64, device=DEV)
    Qw = torch.randn(L, 2, 1, 64, device=DEV)
    S = torch.empty(L, 1, n, device=DEV)
    D = torch.empty(L, n, device=DEV)
    Eb = torch.empty(L, device=DEV)
    H_in = torch.rand(n, device=DEV) * 5
    B.kvc_score(m, mode=B.SCORE_INFOKV, n=n, W=1, Qw=Qw, K=K, S=S, hidden=hidden, H_in=H_in,
                D_out=D, Ebar=Eb, tau=1.0)
    torch.cuda.synchronize()
    h = np64(hidden)
    ref = np.stack([ik.repr_change(h[l], h[L - 1], 1.0) for l in range(L)])
    assert_close_rel(np64(D), ref, rtol=0, atol=2e-5, what="D")
    E, P, Ebar = ik.entropy_scores(ref, np64(H_in)[None, :])
    assert_close_rel(np64(Eb), Ebar, rtol=1e-4, atol=1e-6, what="Ebar")


def test_repr_change_few_tokens_is_bit_identical_to_many():
    """A decode step's few tokens take the (token, layer) warp mapping; the same tokens in a
    long prefill take the warp-per-token kernel.  Both keep the same per-lane order of
    products and the same reduction tree, so D agrees bit for bit."""
    L, n, Dh = 6, 4096, 3584
    hidden = synth.gen_hidden(L, n, Dh, torch.bfloat16, seed=9, device=DEV)
    m = B.model(L, 1, 1, 64)

    def D_of(h):
        nn = h.shape[1]
        D = torch.empty(L, nn, device=DEV)
        H = torch.empty(nn, device=DEV)
        lg = torch.zeros(nn, 512, device=DEV)
        Qw = torch.zeros(L, 1, 1, 64, device=DEV)       # no window attention in a signals-only call
        B.kvc_score(m, mode=B.SCORE_INFOKV, n=nn, W=0, Qw=Qw, K=Qw, S=None, logits=lg, hidden=h,
                    H_out=H, D_out=D)
        torch.cuda.synchronize()
        return D

    D_big = D_of(hidden)
    D_few = D_of(hidden[:, :8].contiguous())
    assert torch.equal(D_few, D_big[:, :8])


@pytest.mark.parametrize("case", range(8))
def test_entropy_split_rows_random_shapes_with_ties(case):
    """Seeded shapes through the split-row kernels (few rows, long vocabularies), with the
    logits quantised to quarter steps so that many values tie at every chunk's and every
    row's k-th largest; one row is mostly masked.  Rows sit at a padded pitch."""
    rng = np.random.default_rng(1000 + case)
    rows = int(rng.choice([1, 2, 17, 100, 512]))
    V = int(rng.choice([8200, 33333, 131072, 200000]))
    k = int(rng.choice([1, 7, 256, 1000]))
    dtype = [torch.bfloat16, torch.float32][case % 2]
    pitch = (V + 15) // 16 * 16
    x = torch.randn(rows, pitch, generator=torch.Generator().manual_seed(case)) * 3.0
    x = torch.round(x * 4.0) / 4.0
    x[0, : V // 2] = float("-inf")
    big = x.to(dtype).to(DEV)
    view = big[:, :V]
    H = gpu_entropy(view, k)
    assert_close_rel(np64(H), ik.topk_entropy(np64(view), k), rtol=1e-4, atol=2e-5,
                     what=f"H rows={rows} V={V} k={k} {dtype}")
