"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test ties one oracle step to something other than the oracle itself:
a closed form, a value derived by hand (tests/golden), an invariant the
page states, a library routine computing the same quantity another way, or
brute force on tiny inputs.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

from oracle import infokv as ik
from oracle import pipeline, recas, selkv

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------- O1 entropy

def test_entropy_golden_hand_example():
    g = gold("entropy_small.json")
    assert ik.topk_entropy(np.array(g["logits"]), g["k"]) == pytest.approx(g["H"], rel=1e-14)


def test_entropy_equal_topk_is_log_k():
    rng = np.random.default_rng(0)
    z = rng.normal(size=1000) - 50.0
    z[rng.choice(1000, 256, replace=False)] = 5.0
    assert ik.topk_entropy(z, 256) == pytest.approx(math.log(256), rel=1e-12)


def test_entropy_dominant_logit_goes_to_zero():
    rng = np.random.default_rng(1)
    z = rng.normal(size=4000)
    z[17] = 60.0
    assert 0.0 <= ik.topk_entropy(z, 256) < 1e-20


def test_entropy_k_at_least_vocab_is_shannon_entropy():
    rng = np.random.default_rng(2)
    z = rng.normal(scale=2.0, size=(5, 200))
    for row in z:
        want = scipy.stats.entropy(scipy.special.softmax(row))
        assert ik.topk_entropy(row, 256) == pytest.approx(want, rel=1e-12)
        assert ik.topk_entropy(row, 200) == pytest.approx(want, rel=1e-12)


def test_entropy_matches_full_sort_and_library_entropy():
    rng = np.random.default_rng(3)
    z = rng.normal(scale=3.0, size=(20, 3000))
    z[:, 5] = z[:, 9]        # ties in the row do not matter
    H = ik.topk_entropy(z, 256)
    for r in range(z.shape[0]):
        top = np.sort(z[r])[::-1][:256]
        assert H[r] == pytest.approx(scipy.stats.entropy(scipy.special.softmax(top)), rel=1e-12)


def test_entropy_shift_and_permutation_invariant():
    rng = np.random.default_rng(4)
    z = rng.normal(size=1000)
    h = ik.topk_entropy(z, 256)
    assert ik.topk_entropy(z + 123.0, 256) == pytest.approx(h, rel=1e-12)
    assert ik.topk_entropy(rng.permutation(z), 256) == pytest.approx(h, rel=1e-14)


# --------------------------------------------------------------------------- O1' entropy from the LM head

def test_lmhead_entropy_one_hot_input_reads_one_weight_column():
    """x = e_j makes the logits column j of W: 256 equal top logits give ln 256."""
    rng = np.random.default_rng(40)
    V, Dh, j = 3000, 48, 17
    W = rng.normal(size=(V, Dh))
    W[:, j] = -50.0 + rng.normal(size=V)
    W[rng.choice(V, 256, replace=False), j] = 5.0
    x = np.zeros((2, Dh))
    x[0, j] = 1.0
    x[1, (j + 1) % Dh] = 1.0                       # another column: not ln 256
    H = ik.lmhead_topk_entropy(x, W, 256)
    assert H[0] == pytest.approx(math.log(256), rel=1e-12)
    assert abs(H[1] - math.log(256)) > 1e-3


def test_lmhead_entropy_geometric_top_k_closed_form():
    """Logits c*w_v with w_v = -v ln2 / c for v < 256 (the rest far below): the top-256
    distribution is p_v = 2^-v / Z, whose entropy is ln Z + ln2 E[v] in closed form."""
    V, Dh, c, N = 1000, 8, 3.0, 256
    W = np.full((V, Dh), 0.0)
    W[:, 2] = -1e3
    v = np.arange(N)
    W[v * 3 + 1, 2] = -v * math.log(2.0) / c      # spread over the vocabulary
    x = np.zeros((1, Dh))
    x[0, 2] = c
    r = 0.5
    Z = (1 - r ** N) / (1 - r)
    Ev = r * (1 - N * r ** (N - 1) + (N - 1) * r ** N) / (1 - r) ** 2 / Z
    want = math.log(Z) + math.log(2.0) * Ev
    assert ik.lmhead_topk_entropy(x, W, 256)[0] == pytest.approx(want, rel=1e-12)


def test_lmhead_entropy_brute_force_tiny():
    """Dot products and the entropy written out by loops on a tiny case (k < V and k > V)."""
    rng = np.random.default_rng(41)
    n, Dh, V = 3, 5, 7
    x = rng.normal(size=(n, Dh))
    W = rng.normal(size=(V, Dh))
    for k in (4, 9):
        got = ik.lmhead_topk_entropy(x, W, k)
        for i in range(n):
            z = [math.fsum(x[i, d] * W[v, d] for d in range(Dh)) for v in range(V)]
            top = sorted(z, reverse=True)[:min(k, V)]
            e = [math.exp(t - top[0]) for t in top]
            Zs = math.fsum(e)
            want = -math.fsum((q / Zs) * math.log(q / Zs) for q in e)
            assert got[i] == pytest.approx(want, rel=1e-12)


# --------------------------------------------------------------------------- O2 representation change

def test_repr_golden_hand_example():
    g = gold("repr_small.json")
    assert ik.repr_change(g["h_l"], g["h_L"], g["tau"]) == pytest.approx(g["D"], rel=1e-14)


def test_repr_special_cases():
    rng = np.random.default_rng(5)
    h = rng.normal(size=(4, 64))
    tau = 1.0
    np.testing.assert_allclose(ik.repr_change(h, h, tau), tau, atol=1e-14)          # final layer: D = tau
    np.testing.assert_allclose(ik.repr_change(-h, h, tau), 2.0 + tau, atol=1e-14)   # anti-parallel
    e0 = np.zeros(64); e0[0] = 3.0
    e1 = np.zeros(64); e1[1] = -2.0
    assert ik.repr_change(e0, e1, tau) == pytest.approx(1.0 + tau, abs=1e-15)       # orthogonal
    assert ik.repr_change(np.zeros(64), e1, tau) == pytest.approx(1.0 + tau)         # zero vector
    np.testing.assert_allclose(ik.repr_change(7.5 * h[0], h[1], 0.0),
                               ik.repr_change(h[0], 0.1 * h[1], 0.0), rtol=1e-13)  # scale invariant


def test_repr_matches_torch_cosine_similarity():
    rng = np.random.default_rng(6)
    a = rng.normal(size=(10, 300))
    b = rng.normal(size=(10, 300))
    cos = torch.nn.functional.cosine_similarity(torch.from_numpy(a), torch.from_numpy(b), dim=-1).numpy()
    np.testing.assert_allclose(ik.repr_change(a, b, 1.0), 2.0 - cos, rtol=1e-13)


# --------------------------------------------------------------------------- O3 entropy score softmax

def test_entropy_softmax_properties():
    rng = np.random.default_rng(7)
    D = 1.0 + 2.0 * rng.random((3, 500))
    H = rng.random(500) * 5.0
    E, P, Ebar = ik.entropy_scores(D, H[None, :])
    np.testing.assert_allclose(E, D * H[None, :], rtol=0, atol=0)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
    np.testing.assert_allclose(Ebar, E.mean(axis=1), rtol=1e-15)
    np.testing.assert_allclose(P, scipy.special.softmax(E, axis=1), rtol=1e-12)
    _, Pc, _ = ik.entropy_scores(np.ones((1, 40)), 2.5 * np.ones(40))
    np.testing.assert_allclose(Pc, 1.0 / 40, rtol=1e-14)


# --------------------------------------------------------------------------- O4/O5 window attention, combination

def _sdpa_weights(q, K, qpos, kpos, scale):
    """Attention weights via torch SDPA with V = identity (library reference)."""
    n = K.shape[0]
    mask = torch.from_numpy(kpos[None, :] <= qpos[:, None])
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.eye(n, dtype=torch.float64)[None],
        attn_mask=mask[None], scale=scale)
    return out[0].numpy()


@pytest.mark.parametrize("G,W,n,d", [(1, 1, 7, 4), (4, 16, 512, 64), (3, 8, 100, 16)])
def test_window_attention_matches_sdpa(G, W, n, d):
    rng = np.random.default_rng(8)
    Q = rng.normal(size=(G, W, d))
    K = rng.normal(size=(n, d))
    K[0] *= 4.0
    A = ik.window_attention(Q, K)
    qpos, kpos = np.arange(n - W, n), np.arange(n)
    want = np.zeros(n)
    for h in range(G):
        want += _sdpa_weights(Q[h], K, qpos, kpos, 1.0 / math.sqrt(d)).sum(axis=0)
    np.testing.assert_allclose(A, want / (G * W), rtol=1e-11, atol=1e-300)
    assert A.sum() == pytest.approx(1.0, abs=1e-13)


def test_window_attention_causal_and_positions():
    rng = np.random.default_rng(9)
    Q = rng.normal(size=(2, 4, 8))
    K = rng.normal(size=(20, 8))
    kpos = np.array(sorted(rng.choice(1000, 20, replace=False)))
    qpos = np.array([kpos[10], kpos[12], kpos[15], kpos[16]])
    A = ik.window_attention(Q, K, qpos=qpos, kpos=kpos)
    assert np.all(A[17:] == 0.0)          # later than every query: never attended
    assert np.all(A[:17] > 0.0)
    assert A.sum() == pytest.approx(1.0, abs=1e-14)
    np.testing.assert_array_equal(ik.window_attention(Q, K, qpos=qpos + 5000, kpos=kpos + 5000), A)
    A1 = ik.window_attention(Q[:, :1], K, qpos=np.array([kpos[5]]), kpos=kpos)
    want = np.zeros(20)
    for h in range(2):
        want[:6] += scipy.special.softmax(Q[h, 0] @ K[:6].T / math.sqrt(8)) / 2
    np.testing.assert_allclose(A1, want, rtol=1e-13, atol=0)


def test_combine_is_convex_mix():
    rng = np.random.default_rng(10)
    A = scipy.special.softmax(rng.normal(size=300))
    P = scipy.special.softmax(rng.normal(size=300))
    S = ik.combine(A, P, 0.9)
    assert S.sum() == pytest.approx(1.0, abs=1e-14)
    assert np.all(S >= np.minimum(A, P) - 1e-18) and np.all(S <= np.maximum(A, P) + 1e-18)
    np.testing.assert_array_equal(ik.combine(A, P, 1.0), A)
    np.testing.assert_array_equal(ik.combine(A, P, 0.0), P)


def test_vatp_and_union():
    A = np.array([[0.5, 0.25, 0.25], [0.1, 0.6, 0.3]])
    V = np.zeros((2, 3, 4))
    V[0, :, 0] = [3.0, 4.0, 0.0]
    V[1, :, 1] = [1.0, -2.0, 2.0]
    np.testing.assert_allclose(ik.vatp(A, V), [[1.5, 1.0, 0.0], [0.1, 1.2, 0.6]])
    np.testing.assert_array_equal(ik.union_max(A), [0.5, 0.6, 0.3])


# --------------------------------------------------------------------------- O6 budgets

def test_budgets_golden_cases():
    for c in gold("budget_small.json")["cases"]:
        k = ik.adaptive_budgets(c["Ebar"], c["B"], c["w"], c["n"])
        np.testing.assert_array_equal(k, c["k"])


def test_budgets_sum_to_B_and_equal_shares_are_uniform():
    rng = np.random.default_rng(11)
    for _ in range(200):
        L = int(rng.integers(1, 40))
        n = int(rng.integers(8, 5000))
        w = int(rng.integers(0, 64))
        lo = min(w, n)
        B = int(rng.integers(L * lo, L * n + 1))
        Ebar = rng.random(L) ** 3 * rng.choice([1e-3, 1.0, 50.0])
        k = ik.adaptive_budgets(Ebar, B, w, n)
        assert k.sum() == B
        assert np.all(k >= lo) and np.all(k <= n)
    n, rho, L = 65536, 0.2, 32
    ku = ik.uniform_budgets(n, rho, L, 64)
    assert np.all(ku == 13107)
    ka = ik.adaptive_budgets(np.full(L, 3.7), int(ku.sum()), 64, n)
    np.testing.assert_array_equal(ka, ku)


def test_budget_proportional_when_unclamped():
    Ebar = np.array([1.0, 2.0, 5.0, 2.0])
    k = ik.adaptive_budgets(Ebar, 1000, 10, 10_000)
    np.testing.assert_array_equal(k, [100, 200, 500, 200])


# --------------------------------------------------------------------------- O7/O8 selection and compaction

def _brute_force_keep(S, k, w):
    """Exhaustive: best-sum subset of the non-window positions, lexicographically lowest among equals."""
    n = len(S)
    cand = range(n - w)
    best, best_key = None, None
    for sub in itertools.combinations(cand, k - w):
        key = (-sum(S[i] for i in sub), sorted(sub))
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return sorted(list(best) + list(range(n - w, n)))


def test_select_brute_force_tiny():
    rng = np.random.default_rng(12)
    for _ in range(60):
        n = int(rng.integers(3, 11))
        w = int(rng.integers(0, 3))
        k = int(rng.integers(w, n + 1))
        S = rng.integers(0, 4, size=n).astype(float)   # many exact ties
        got = ik.select_topk(S, k, w)
        assert list(got) == _brute_force_keep(list(S), k, w)


def test_select_window_always_kept_and_sorted():
    rng = np.random.default_rng(13)
    S = rng.random(1000)
    S[-16:] = 0.0
    got = ik.select_topk(S, 128, 16)
    assert len(got) == 128 and np.all(np.diff(got) > 0)
    assert set(range(984, 1000)) <= set(got)
    np.testing.assert_array_equal(ik.select_topk(S, 1000, 16), np.arange(1000))


def test_prefill_select_ranks_by_own_or_union_score():
    """Per KV head: each head keeps its own top scores.  GQA union: every head keeps one set,
    ranked by the max over heads.  Checked as properties: the recent window is kept, and
    every other kept position scores at least as high as every dropped one."""
    rng = np.random.default_rng(26)
    L, Hkv, n, w = 2, 3, 40, 4
    S = rng.random((L, Hkv, n))
    S[1, 2, :10] += 5.0                           # head 2 of layer 1 alone rates the first tokens
    budgets = np.array([12, 15])
    for mode in ("per_kv_head", "gqa_union"):
        idx = pipeline.prefill_select(S, budgets, w, mode)
        for l in range(L):
            for g in range(Hkv):
                keep = np.asarray(idx[l][g])
                assert len(keep) == budgets[l] and np.all(np.diff(keep) > 0)
                assert set(range(n - w, n)) <= set(keep.tolist())
                score = S[l].max(axis=0) if mode == "gqa_union" else S[l, g]
                rest = np.setdiff1d(np.arange(n - w), keep)
                kept_old = np.setdiff1d(keep, np.arange(n - w, n))
                assert score[kept_old].min() >= score[rest].max()
                if mode == "gqa_union":
                    np.testing.assert_array_equal(keep, idx[l][0])
        if mode == "gqa_union":
            assert set(range(10)) <= set(np.asarray(idx[1][0]).tolist())   # head 2's choice wins


def test_compact_identity_and_gather():
    X = np.arange(40.0).reshape(10, 4)
    np.testing.assert_array_equal(ik.compact(X, np.arange(10)), X)
    np.testing.assert_array_equal(ik.compact(X, [1, 7]), X[[1, 7]])


# --------------------------------------------------------------------------- O9 merge

def test_merge_golden_hand_example():
    g = gold("merge_small.json")
    Vp, R = selkv.merge(np.array(g["V"]), np.array(g["A"]), np.array(g["kept"]), g["bucket"])
    np.testing.assert_allclose(Vp, g["V_merged"], rtol=1e-14)
    np.testing.assert_allclose(R, g["R"], rtol=1e-14)


def test_merge_gate_zero_is_a_drop():
    rng = np.random.default_rng(14)
    d = 16
    vt = rng.normal(size=d)
    ortho = rng.normal(size=d)
    ortho -= ortho @ vt / (vt @ vt) * vt
    V = np.stack([vt, -2.0 * vt, ortho, -vt + 0.0])
    A = np.array([0.4, 0.3, 0.2, 0.1])
    Vp, R = selkv.merge(V, A, np.array([0]), 512)
    np.testing.assert_allclose(Vp[0], vt, rtol=1e-12, atol=1e-12)
    assert R[0] == pytest.approx(1.0, abs=1e-12)


def test_merge_gate_one_closed_form_and_routing():
    d = 8
    rng = np.random.default_rng(15)
    v0, v2 = rng.normal(size=d), rng.normal(size=d)
    V = np.stack([v0, 2.5 * v2, v2, rng.normal(size=d)])
    A = np.array([0.1, 0.2, 0.5, 0.2])
    # kept {0, 2}: bucket target is position 2 (higher A); evicted 1 has g = 1 toward it
    Vp, R = selkv.merge(V[:3], A[:3], np.array([0, 2]), 512)
    want = (0.5 * v2 + 0.2 * 2.5 * v2) / (0.5 + 0.2)
    np.testing.assert_allclose(Vp[1], want, rtol=1e-13)
    assert R[1] == pytest.approx(0.7 / 0.5, rel=1e-14)
    np.testing.assert_array_equal(Vp[0], v0)
    assert R[0] == 1.0


def test_merge_bucket_without_kept_changes_nothing_and_buckets_are_separate():
    rng = np.random.default_rng(16)
    V = rng.normal(size=(12, 4))
    A = rng.random(12)
    kept = np.array([1, 2])              # bucket size 4: buckets 1 and 2 hold no kept token
    Vp, R = selkv.merge(V, A, kept, 4)
    Vp_alone, R_alone = selkv.merge(V[:4], A[:4], kept, 4)
    np.testing.assert_array_equal(Vp, Vp_alone)
    np.testing.assert_array_equal(R, R_alone)


# --------------------------------------------------------------------------- O10 decode with attention compensation

def test_decode_unbiased_matches_sdpa():
    rng = np.random.default_rng(17)
    q = rng.normal(size=(4, 64))
    K = rng.normal(size=(300, 64))
    V = rng.normal(size=(300, 64))
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0].numpy()
    np.testing.assert_allclose(selkv.decode_attention(q, K, V), want, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(selkv.decode_attention(q, K, V, np.ones(300), 1.0), want, rtol=1e-12, atol=1e-14)


def test_decode_bias_equals_duplicated_tokens():
    """A slot standing for m identical tokens with R = m (alpha_c = 1) attends exactly like m copies."""
    rng = np.random.default_rng(18)
    q = rng.normal(size=(3, 32))
    K = rng.normal(size=(50, 32))
    V = rng.normal(size=(50, 32))
    m = 5
    Kdup = np.vstack([K, np.repeat(K[7:8], m - 1, axis=0)])
    Vdup = np.vstack([V, np.repeat(V[7:8], m - 1, axis=0)])
    R = np.ones(50)
    R[7] = m
    np.testing.assert_allclose(selkv.decode_attention(q, K, V, R, 1.0),
                               selkv.decode_attention(q, Kdup, Vdup), rtol=1e-12, atol=1e-14)
    # R > 1 raises the slot's share (sign of the bias)
    base = selkv.decode_attention(q[:1], K[7:9], np.eye(2, 32)[:2])
    up = selkv.decode_attention(q[:1], K[7:9], np.eye(2, 32)[:2], np.array([2.0, 1.0]), 1.0)
    assert up[0, 0] > base[0, 0]


# --------------------------------------------------------------------------- f3 RoPE re-positioning

def test_rope_frequencies_closed_form():
    """theta_i = base^(-2i/d): base 100, d 4 -> (1, 1/10); base 10^4, d 8 -> 10^-i."""
    np.testing.assert_allclose(selkv.rope_inv_freq(4, 100.0), [1.0, 0.1], rtol=1e-15)
    np.testing.assert_allclose(selkv.rope_inv_freq(8, 1.0e4), [1.0, 0.1, 0.01, 0.001], rtol=1e-15)


def test_rope_single_pair_is_a_plane_rotation():
    """d = 2 (theta_0 = 1): (1, 0) moved by s turns to (cos s, sin s); (0, 1) to (-sin s, cos s)."""
    for s in (1, 2, 7, -3, 100000):
        got = selkv.rope_reposition(np.eye(2), [0, 0], [s, s], 10000.0)
        np.testing.assert_allclose(got, [[math.cos(s), math.sin(s)], [-math.sin(s), math.cos(s)]],
                                   rtol=0, atol=1e-12)


def test_rope_reposition_equals_embedding_at_the_new_position():
    """RoFormer's form: the pair (x_i, x_{i+d/2}) as one complex number times e^{i p theta_i}.
    A key embedded at p and re-positioned to p' equals the key embedded at p' directly."""
    theta = np.array([1.0, 0.1, 0.01, 0.001])          # d = 8, base 10^4 (hand values)

    def embed(x, p):
        z = (x[..., :4] + 1j * x[..., 4:]) * np.exp(1j * np.asarray(p, np.float64)[..., None] * theta)
        return np.concatenate([z.real, z.imag], axis=-1)

    rng = np.random.default_rng(23)
    x = rng.normal(size=(40, 8))
    old = rng.integers(0, 100000, size=40)
    new = np.arange(40) + 17
    got = selkv.rope_reposition(embed(x, old), old, new, 1.0e4)
    np.testing.assert_allclose(got, embed(x, new), rtol=0, atol=1e-9)


def test_rope_scores_depend_on_position_differences_only():
    """Shifting a query and a key by the same amount leaves q.k unchanged; shifts compose;
    norms are kept."""
    rng = np.random.default_rng(24)
    q, k = rng.normal(size=(2, 128))
    base = 5.0e5
    P, p, sft = 70000, 1234, 4321
    qP = selkv.rope_reposition(q, 0, P, base)
    kp = selkv.rope_reposition(k, 0, p, base)
    qs = selkv.rope_reposition(qP, P, P + sft, base)
    ks = selkv.rope_reposition(kp, p, p + sft, base)
    assert float(qs @ ks) == pytest.approx(float(qP @ kp), rel=1e-9, abs=1e-9)
    two = selkv.rope_reposition(selkv.rope_reposition(kp, p, 5, base), 5, 999, base)
    np.testing.assert_allclose(two, selkv.rope_reposition(kp, p, 999, base), rtol=0, atol=1e-9)
    assert np.linalg.norm(ks) == pytest.approx(np.linalg.norm(k), rel=1e-12)
    np.testing.assert_array_equal(selkv.rope_reposition(kp, p, p, base), kp)


# --------------------------------------------------------------------------- O11 RECAS bound

def test_bound_holds_and_is_tight():
    rng = np.random.default_rng(19)
    for _ in range(50):
        t = int(rng.integers(2, 400))
        q = rng.normal(size=(3, 16)) * rng.uniform(0.1, 3)
        K = rng.normal(size=(t, 16))
        V = rng.normal(size=(t, 16)) * rng.uniform(0.1, 5)
        kept = rng.random(t) < rng.uniform(0.05, 1.0)
        kept[-1] = True
        r = recas.dropped_mass_probe(q, K, V, kept)
        assert np.all(r["err"] <= r["bound"] * (1 + 1e-12) + 1e-15)
        assert np.all((r["delta"] >= 0) & (r["delta"] <= 1))
    # nothing evicted: delta = 0 and o = o'
    r = recas.dropped_mass_probe(q, K, V, np.ones(t, bool))
    assert np.all(r["delta"] == 0) and np.allclose(r["o_full"], r["o_kept"], atol=1e-14)
    # two tokens, opposite values of norm V_max: the bound is attained
    v = np.array([[3.0, 4.0], [-3.0, -4.0]])
    r = recas.dropped_mass_probe(np.array([[0.3, -0.2]]), np.array([[1.0, 0.0], [0.0, 1.0]]), v,
                                 np.array([True, False]))
    assert r["err"][0] == pytest.approx(r["bound"][0], rel=1e-12)


def test_probe_quantities_match_library_attention():
    """delta, o and o' against torch's scaled-dot-product attention (full history, and the
    kept positions only); V_max against a direct norm; the identity o - o' from the reading."""
    rng = np.random.default_rng(25)
    G, t, d = 4, 300, 64
    q = rng.normal(size=(G, d))
    K = rng.normal(size=(t, d))
    V = rng.normal(size=(t, d)) * rng.uniform(0.5, 3.0, size=(t, 1))
    kept = rng.random(t) < 0.3
    kept[-1] = True
    r = recas.dropped_mass_probe(q, K, V, kept)
    qt, Kt, Vt = (torch.from_numpy(x)[None] for x in (q, K, V))
    o_full = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)[0].numpy()
    o_kept = torch.nn.functional.scaled_dot_product_attention(qt, Kt[:, kept], Vt[:, kept])[0].numpy()
    np.testing.assert_allclose(r["o_full"], o_full, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r["o_kept"], o_kept, rtol=1e-10, atol=1e-12)
    # delta: attention of a one-hot value on every evicted position at once
    ind = torch.from_numpy((~kept).astype(np.float64))[None, :, None]
    delta = torch.nn.functional.scaled_dot_product_attention(qt, Kt, ind)[0, :, 0].numpy()
    np.testing.assert_allclose(r["delta"], delta, rtol=1e-10, atol=1e-14)
    assert r["vmax"] == pytest.approx(max(math.hypot(*row) for row in V), rel=1e-12)
    # o - o' = sum_ev p v - delta / (1 - delta) * sum_kept p v  (the decomposition behind the bound)
    s = q @ K.T / math.sqrt(d)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    dd = r["delta"][:, None]
    diff = p[:, ~kept] @ V[~kept] - dd / (1 - dd) * (p[:, kept] @ V[kept])
    np.testing.assert_allclose(r["o_full"] - r["o_kept"], diff, rtol=1e-9, atol=1e-12)


# --------------------------------------------------------------------------- O12 recompression schedule

def test_recompression_lengths_follow_floor_rho_t():
    rng = np.random.default_rng(20)
    L, Hkv, Hq, d, n0, Dh, V = 1, 1, 2, 8, 24, 16, 50
    period, rho = 16, 0.125
    K = rng.normal(size=(L, Hkv, n0, d))
    Vv = rng.normal(size=(L, Hkv, n0, d))
    H = rng.random(n0)
    D = 1.0 + rng.random((L, n0))
    rp = pipeline.DecodeCompressionReplay(K, Vv, H, D, n_q_heads=Hq, W=4, w=4, rho=rho,
                                          alpha=0.9, tau=1.0, period=period)
    lengths = []
    for j in range(4 * period):
        rp.step(rng.normal(size=(L, Hq, d)), rng.normal(size=(L, Hkv, d)), rng.normal(size=(L, Hkv, d)),
                rng.normal(size=V), rng.normal(size=(L, Dh)), topk=8)
        if rp.due():
            rp.recompress()
            lengths.append(rp.K[0][0].shape[0])
    # t = 24 + 16 j at the j-th compression; kept = floor(t / 8)
    assert lengths == [5, 7, 9, 11]
    assert np.all(np.diff(rp.pos[0][0]) > 0)


def test_replay_cache_is_the_kept_history_and_decode_attends_to_it():
    """Decode-time replay: after each compression every cached row (K, V, H, D) is the one
    inserted at its position; decode attends over exactly the cached rows and the probe
    over the whole history (both against torch attention); the window-query ring holds the
    last W positions."""
    rng = np.random.default_rng(27)
    L, Hkv, Hq, d, n0, Dh, Vocab, W = 2, 2, 4, 8, 20, 8, 40, 4
    period, rho = 8, 0.4
    K = rng.normal(size=(L, Hkv, n0, d))
    Vv = rng.normal(size=(L, Hkv, n0, d))
    H0 = rng.random(n0)
    D0 = 1.0 + rng.random((L, n0))
    rp = pipeline.DecodeCompressionReplay(K, Vv, H0, D0, n_q_heads=Hq, W=W, w=3, rho=rho,
                                          alpha=0.9, tau=1.0, period=period)
    Hs = {i: H0[i] for i in range(n0)}                  # H of every position as inserted
    Ds = {(l, i): D0[l, i] for l in range(L) for i in range(n0)}
    for j in range(3 * period):
        q = rng.normal(size=(L, Hq, d))
        logits = rng.normal(size=Vocab) * 2
        hid = rng.normal(size=(L, Dh))
        pos = rp.t
        o, probes = rp.step(q, rng.normal(size=(L, Hkv, d)), rng.normal(size=(L, Hkv, d)), logits, hid,
                            topk=8, probe=True)
        Hs[pos] = float(ik.topk_entropy(logits, 8))
        for l in range(L):
            Ds[(l, pos)] = float(ik.repr_change(hid[l], hid[L - 1], 1.0))
        for l in range(L):
            for g in range(Hkv):
                qt = torch.from_numpy(q[l, g * 2:(g + 1) * 2])[None]
                kc = torch.from_numpy(rp.K[l][g])[None]
                vc = torch.from_numpy(rp.V[l][g])[None]
                want = torch.nn.functional.scaled_dot_product_attention(qt, kc, vc)[0].numpy()
                np.testing.assert_allclose(o[l, g * 2:(g + 1) * 2], want, rtol=1e-10, atol=1e-12)
                kf = torch.from_numpy(rp.Kfull[l][g])[None]
                vf = torch.from_numpy(rp.Vfull[l][g])[None]
                full = torch.nn.functional.scaled_dot_product_attention(qt, kf, vf)[0].numpy()
                np.testing.assert_allclose(probes[(l, g)]["o_full"], full, rtol=1e-10, atol=1e-12)
                np.testing.assert_allclose(probes[(l, g)]["o_kept"], want, rtol=1e-10, atol=1e-12)
        assert [pp for _, pp in rp.qring] == list(range(max(n0, rp.t - W), rp.t))
        if rp.due():
            rp.recompress()
            for l in range(L):
                for g in range(Hkv):
                    ps = rp.pos[l][g]
                    np.testing.assert_array_equal(rp.K[l][g], rp.Kfull[l][g][ps])
                    np.testing.assert_array_equal(rp.V[l][g], rp.Vfull[l][g][ps])
                    np.testing.assert_array_equal(rp.H[l][g], [Hs[int(i)] for i in ps])
                    np.testing.assert_array_equal(rp.D[l][g], [Ds[(l, int(i))] for i in ps])
                    assert set(range(rp.t - 3, rp.t)) <= set(ps.tolist())      # recent window w = 3


# --------------------------------------------------------------------------- prefill composition and the tie zone

def _sdpa_group_weights(Qw_l, K_l, scale):
    """Window attention weights of every query head through torch SDPA with enable_gqa,
    so that torch's grouping convention (query head h reads KV head h // G), not the
    oracle's, decides which KV head each query head uses.  The values are the identity
    plus one indicator column per KV head: out[h, r, :n] are the weights of window row r
    of head h, out[h, r, n + g] is 1 exactly when head h read KV head g.
    Returns A [Hkv][n] = mean over the rows of the query heads that read each KV head."""
    Hq, W, d = Qw_l.shape
    Hkv, n, _ = K_l.shape
    val = np.zeros((Hkv, n, n + Hkv))
    for g in range(Hkv):
        val[g, :, :n] = np.eye(n)
        val[g, :, n + g] = 1.0
    qpos, kpos = np.arange(n - W, n), np.arange(n)
    mask = torch.from_numpy(kpos[None, :] <= qpos[:, None])
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Qw_l)[None], torch.from_numpy(K_l)[None], torch.from_numpy(val)[None],
        attn_mask=mask[None, None], scale=scale, enable_gqa=True)[0].numpy()
    A = np.einsum("hrn,hrg->gn", out[:, :, :n], out[:, :, n:])
    rows = out[:, :, n:].sum(axis=(0, 1))              # rows that read each KV head
    return A / rows[:, None]


def _prefill_case(L=2, Hq=4, Hkv=2, n=24, W=3, d=8, Dh=16, V=40, seed=28):
    rng = np.random.default_rng(seed)
    Qw = rng.normal(size=(L, Hq, W, d)) * rng.uniform(0.5, 3.0, size=(L, Hq, 1, 1))   # heads differ
    K = rng.normal(size=(L, Hkv, n, d))
    K[:, :, 0] *= 4.0
    Vv = rng.normal(size=(L, Hkv, n, d)) * rng.uniform(0.3, 3.0, size=(L, Hkv, n, 1))
    logits = rng.normal(size=(n, V)) * rng.uniform(0.5, 4.0, size=(n, 1))
    hidden = rng.normal(size=(L, n, Dh))
    return Qw, K, Vv, logits, hidden


def test_prefill_window_attention_follows_library_gqa_grouping():
    """A[l, g] is the mean window attention of exactly the query heads that torch's GQA
    convention assigns to KV head g (contiguous groups of G heads)."""
    Qw, K, Vv, logits, hidden = _prefill_case()
    L, Hq, W, d = Qw.shape
    Hkv = K.shape[1]
    out = pipeline.prefill_scores(None, None, Qw, K, G=Hq // Hkv, mode="attn")
    for l in range(L):
        want = _sdpa_group_weights(Qw[l], K[l], 1.0 / math.sqrt(d))
        np.testing.assert_allclose(out["A"][l], want, rtol=1e-11, atol=1e-300)
    np.testing.assert_array_equal(out["S"], out["A"])                   # attention-only mode


def test_prefill_infokv_composition_from_library_routines():
    """S = alpha A + (1 - alpha) Softmax(D H) per layer, with H from scipy's entropy of the
    renormalised top-k, D from torch's cosine similarity against the LAST stored layer,
    and the softmax from scipy - the same P for every KV head of a layer.  L == Hkv so a
    softmax broadcast along the wrong axis would still have the right shape."""
    Qw, K, Vv, logits, hidden = _prefill_case()
    L, Hq, W, d = Qw.shape
    Hkv = K.shape[1]
    topk, alpha, tau = 8, 0.9, 1.0
    out = pipeline.prefill_scores(logits, hidden, Qw, K, G=Hq // Hkv, alpha=alpha, tau=tau, topk=topk)
    H = np.array([scipy.stats.entropy(scipy.special.softmax(np.sort(r)[::-1][:topk])) for r in logits])
    hL = torch.from_numpy(hidden[L - 1])
    D = np.stack([2.0 - torch.nn.functional.cosine_similarity(torch.from_numpy(hidden[l]), hL, dim=-1).numpy()
                  for l in range(L)])
    P = scipy.special.softmax(D * H[None, :], axis=1)
    np.testing.assert_allclose(out["H"], H, rtol=1e-12)
    np.testing.assert_allclose(out["D"], D, rtol=1e-12)
    np.testing.assert_allclose(out["D"][L - 1], tau, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out["P"], P, rtol=1e-11)
    np.testing.assert_allclose(out["Ebar"], (D * H[None, :]).mean(axis=1), rtol=1e-12)
    for l in range(L):
        A = _sdpa_group_weights(Qw[l], K[l], 1.0 / math.sqrt(d))
        for g in range(Hkv):
            np.testing.assert_allclose(out["S"][l, g], alpha * A[g] + (1 - alpha) * P[l], rtol=1e-11)


def test_prefill_representation_change_is_against_the_last_layer():
    """Layer 0 = -h^(L), layer 1 orthogonal to h^(L), layer 2 = h^(L): D = (2 + tau, 1 + tau, tau)."""
    rng = np.random.default_rng(29)
    n, Dh, tau = 6, 8, 1.0
    hL = rng.normal(size=(n, Dh))
    ortho = rng.normal(size=(n, Dh))
    ortho -= (ortho * hL).sum(axis=1, keepdims=True) / (hL * hL).sum(axis=1, keepdims=True) * hL
    hidden = np.stack([-hL, ortho, hL])
    K = rng.normal(size=(3, 1, n, 4))
    Qw = rng.normal(size=(3, 1, 2, 4))
    out = pipeline.prefill_scores(rng.normal(size=(n, 10)), hidden, Qw, K, G=1, tau=tau, topk=4)
    np.testing.assert_allclose(out["D"], np.array([[2 + tau] * n, [1 + tau] * n, [tau] * n]), atol=1e-13)


def test_prefill_vatp_mode_is_attention_times_value_norm():
    Qw, K, Vv, logits, hidden = _prefill_case()
    L, Hq, W, d = Qw.shape
    Hkv = K.shape[1]
    out = pipeline.prefill_scores(None, None, Qw, K, Vv, G=Hq // Hkv, mode="vatp")
    for l in range(L):
        A = _sdpa_group_weights(Qw[l], K[l], 1.0 / math.sqrt(d))
        np.testing.assert_allclose(out["S"][l], A * np.linalg.norm(Vv[l], axis=-1), rtol=1e-11)


def test_tie_zone_hand_example():
    """n = 12, w = 2, k = 6: the window (positions 10, 11) is kept, 4 of positions 0..9 are
    chosen.  Candidate scores sorted: 1.0, 0.9, 0.8, then the 4th largest 0.5000025 (the
    threshold), 0.5, 0.5, 0.49999, 0.2, ...  Within 1e-5 relative of 0.5000025 (|diff| <=
    5.000025e-6): 0.5000025 itself and both 0.5 (diff 2.5e-6); not 0.49999 (diff 1.25e-5).
    Window position 10 carries the threshold's value too but is not a candidate."""
    S = np.array([0.5, 0.9, 0.2, 0.5000025, 1.0, 0.49999, 0.5, 0.8, 0.1, 0.3, 0.5000025, 7.0])
    np.testing.assert_array_equal(ik.tie_zone(S, 6, 2), [0, 3, 6])
    np.testing.assert_array_equal(ik.select_topk(S, 6, 2), [1, 3, 4, 7, 10, 11])
    assert ik.tie_zone(S, 12, 2).size == 0 and ik.tie_zone(S, 2, 2).size == 0    # nothing to choose
    # threshold 0.8 (k = 5): only 0.8 itself lies within 8e-6 of it
    np.testing.assert_array_equal(ik.tie_zone(S, 5, 2), [7])


def test_tie_zone_covers_every_swap_under_small_perturbations():
    """Scores perturbed by at most 4e-6 relative can change the kept set only on positions
    within 2 * 4e-6 / (1 - 4e-6) < 1e-5 relative of the k-th threshold: every swap lies in
    the zone."""
    rng = np.random.default_rng(30)
    for _ in range(300):
        n = int(rng.integers(8, 200))
        w = int(rng.integers(0, 6))
        k = int(rng.integers(w + 1, n))
        levels = rng.random(int(rng.integers(2, 6))) + 0.1
        S = levels[rng.integers(0, levels.size, size=n)] * (1 + rng.uniform(-3e-6, 3e-6, size=n))
        Sp = S * (1 + rng.uniform(-4e-6, 4e-6, size=n))
        diff = set(ik.select_topk(S, k, w).tolist()) ^ set(ik.select_topk(Sp, k, w).tolist())
        assert diff <= set(ik.tie_zone(S, k, w).tolist())


# --------------------------------------------------------------------------- RECAS calibrated estimator and controller

def test_conformal_quantile_rank_by_hand():
    """m = 5 residuals {1..5}: alpha 0.2 -> rank ceil(6 * 0.8) = 5 -> 5; alpha 0.5 -> rank 3
    -> 3; alpha 0.1 -> rank ceil(5.4) = 6 > 5 -> +inf; m = 9, alpha 0.1 -> rank 9 exactly."""
    r = [5.0, 1.0, 4.0, 2.0, 3.0]
    assert recas.conformal_quantile(r, 0.2) == 5.0
    assert recas.conformal_quantile(r, 0.5) == 3.0
    assert recas.conformal_quantile(r, 0.1) == math.inf
    assert recas.conformal_quantile(list(range(9, 0, -1)), 0.1) == 9.0
    assert recas.conformal_quantile([], 0.1) == math.inf


def test_conformal_quantile_coverage():
    """Split-conformal guarantee for exchangeable residuals: a new residual lies at or
    below the quantile of m earlier ones with probability in [1 - alpha, 1 - alpha + 1/(m+1)]."""
    rng = np.random.default_rng(31)
    for alpha, m in ((0.1, 49), (0.2, 20), (0.05, 99)):
        trials = 20000
        hits = 0
        for _ in range(trials):
            r = rng.standard_t(3, size=m + 1)
            hits += r[-1] <= recas.conformal_quantile(r[:-1], alpha)
        cov = hits / trials
        sd = math.sqrt(alpha * (1 - alpha) / trials)
        assert 1 - alpha - 4 * sd <= cov <= 1 - alpha + 1 / (m + 1) + 4 * sd, (alpha, m, cov)


def test_calibrator_ratio_and_out_of_sample_residuals_by_hand():
    """G = 2, Hkv = 2.  Probe 1: delta = (0.2, 0.2, 0.3, 0.3), x = (0.1, 0.15): residuals
    against c = 1: (0.1, 0.1, 0.15, 0.15); then c = 1.0 / 0.5 = 2.  Probe 2 exactly
    proportional to x with c = 2: residuals 0; c stays 2."""
    cal = recas.DroppedMassCalibrator(alpha=0.5)
    assert cal.c == 1.0 and cal.q == math.inf
    cal.observe([0.2, 0.2, 0.3, 0.3], [0.1, 0.15], G=2)
    np.testing.assert_allclose(cal.res, [0.1, 0.1, 0.15, 0.15], atol=1e-15)
    assert cal.c == pytest.approx(2.0, rel=1e-15)
    cal.observe([0.1, 0.1, 0.08, 0.08], [0.05, 0.04], G=2)
    np.testing.assert_allclose(cal.res[4:], 0.0, atol=1e-16)
    assert cal.c == pytest.approx(2.0, rel=1e-15)
    # ring of 8: the quantile at alpha 0.5 is the rank-5 residual of the 8 = 0.1
    assert cal.q == pytest.approx(0.1)
    dh, db = cal.estimate([0.1, 0.02])
    np.testing.assert_allclose(dh, [0.2, 0.04])
    np.testing.assert_allclose(db, [0.3, 0.14])


def test_upper_bound_covers_delta_on_synthetic_traces():
    """Probe traces delta = c* x (1 + noise): the bound computed before each probe covers
    that probe's delta at least at the stated level (1 - alpha), minus sampling slack."""
    rng = np.random.default_rng(32)
    alpha, G, Hkv = 0.1, 4, 2
    for c_true in (0.3, 1.0, 3.0):
        cal = recas.DroppedMassCalibrator(alpha=alpha)
        covered = total = 0
        for j in range(400):
            x = rng.uniform(0.01, 0.2, size=Hkv)
            delta = np.repeat(c_true * x, G) * (1 + 0.3 * rng.standard_normal(G * Hkv))
            if j >= 20:
                _, bar = cal.estimate(x)
                covered += int((delta <= np.repeat(bar, G)).sum())
                total += G * Hkv
            cal.observe(delta, x, G)
        assert covered / total >= 1 - alpha - 0.03, (c_true, covered / total)
        assert cal.c == pytest.approx(c_true, rel=0.05)


def _brute_need(S, A, w, k0, c, q, eps):
    n = len(S)
    for k in range(max(k0, min(w, n)), n + 1):
        keep = ik.select_topk(S, k, w)
        if c * recas.dropped_share(A, keep) + q <= eps:
            return k
    return n


def test_controller_need_brute_force_and_special_cases():
    rng = np.random.default_rng(33)
    for _ in range(300):
        n = int(rng.integers(2, 30))
        w = int(rng.integers(0, 4))
        S = rng.integers(0, 5, size=n).astype(float)          # ties
        A = rng.random(n) * (rng.random(n) < 0.8)
        k0 = int(rng.integers(min(w, n), n + 1))
        c, q, eps = rng.uniform(0.5, 2), rng.uniform(-0.05, 0.1), rng.uniform(0, 0.6)
        assert recas.controller_need(S, A, w, k0, c, q, eps) == _brute_need(S, A, w, k0, c, q, eps)
    S, A = rng.random(50), rng.random(50)
    assert recas.controller_need(S, A, 4, 10, 1.0, 0.0, 1.0) == 10          # bound already met at k0
    assert recas.controller_need(S, A, 4, 10, 1.0, 0.2, 0.1) == 50          # q > eps: keep the row
    ks, x = recas.dropped_share_curve(S, A, 4)
    assert x[-1] == pytest.approx(0.0, abs=1e-15) and np.all(np.diff(x) <= 1e-15)


def test_controller_need_monotone_in_eps():
    rng = np.random.default_rng(34)
    for _ in range(50):
        n = int(rng.integers(20, 200))
        S, A = rng.random(n), rng.random(n) ** 3
        k0 = int(rng.integers(4, n))
        needs = [recas.controller_need(S, A, 4, k0, 1.3, 0.01, e) for e in np.linspace(0, 1, 41)]
        assert all(a >= b for a, b in zip(needs, needs[1:]))


# --------------------------------------------------------------------------- RECAS dynamic sparse decode

def _sdpa_probs(q, K):
    """Attention weights of rows q [G][d] over keys K [n][d] via torch SDPA with V = I."""
    n = K.shape[0]
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.eye(n, dtype=torch.float64)[None])[0].numpy()


def test_sparse_active_count_by_hand():
    assert recas.sparse_active_count(10, 0.3) == 3          # 0.3 * 10 rounds to 3 + 2^-51 in binary
    assert recas.sparse_active_count(10, 0.31) == 4
    assert recas.sparse_active_count(7, 0.0) == 1
    assert recas.sparse_active_count(5, 1.0) == 5
    assert recas.sparse_active_count(2808, 0.293) == 823


def test_cached_steps_by_hand():
    """Prompt of 100: after the 5th generated token (t = 105) a prompt token has been cached
    for the 5 steps, the first generated token (position 100) for 5, this step's token
    (position 104) for 1."""
    np.testing.assert_array_equal(recas.cached_steps([0, 99, 100, 102, 104], 105, 100), [5, 5, 5, 3, 1])


def test_sparse_decode_full_activity_is_dense_attention():
    """kappa = 1: every token is active, the output is plain attention (torch SDPA) and each
    token's accumulator grows by its attention averaged over the heads."""
    rng = np.random.default_rng(41)
    q, K, V = rng.normal(size=(4, 32)), rng.normal(size=(50, 32)), rng.normal(size=(50, 32))
    acc, cnt = rng.random(50), rng.integers(1, 9, size=50).astype(float)
    o, active, acc2, _ = recas.sparse_decode_step(q, K, V, acc, cnt, 1.0, 0.6, 0.4)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0].numpy()
    np.testing.assert_allclose(o, want, rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(active, np.arange(50))
    np.testing.assert_allclose(acc2 - acc, _sdpa_probs(q, K).mean(axis=0), rtol=1e-12, atol=1e-16)


def test_sparse_decode_selection_and_output_against_library():
    """sigma = a tr + b hi with tr the head-mean of torch SDPA weights and hi = acc / cnt; the
    active set is the top ceil(kappa n) by sigma (ties to the lower position); the output
    is SDPA over the active rows; the accumulators gain exactly 1 in total."""
    rng = np.random.default_rng(42)
    for _ in range(40):
        n, G, d = int(rng.integers(1, 60)), int(rng.integers(1, 5)), 16
        q, K, V = rng.normal(size=(G, d)), rng.normal(size=(n, d)), rng.normal(size=(n, d))
        acc = np.round(rng.random(n) * 4) / 4                   # ties in hi
        cnt = rng.integers(1, 5, size=n).astype(float)
        kappa, a, b = rng.uniform(0, 1), rng.uniform(0, 1), rng.uniform(0, 1)
        o, active, acc2, sigma = recas.sparse_decode_step(q, K, V, acc, cnt, kappa, a, b)
        tr = _sdpa_probs(q, K).mean(axis=0)
        np.testing.assert_allclose(sigma, a * tr + b * acc / cnt, rtol=1e-12, atol=1e-15)
        kt = recas.sparse_active_count(n, kappa)
        order = sorted(range(n), key=lambda i: (-sigma[i], i))
        np.testing.assert_array_equal(active, sorted(order[:kt]))
        want = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None], torch.from_numpy(K[active])[None], torch.from_numpy(V[active])[None])[0].numpy()
        np.testing.assert_allclose(o, want, rtol=1e-11, atol=1e-13)
        assert acc2.sum() - acc.sum() == pytest.approx(1.0, abs=1e-12)
        np.testing.assert_array_equal(acc2[np.setdiff1d(np.arange(n), active)],
                                      acc[np.setdiff1d(np.arange(n), active)])


def test_sparse_decode_history_term_by_hand():
    """a = 0: the active set is the tokens with the largest mean attention per cached step:
    acc / cnt = (0.9/3, 0.5/1, 0.2/1, 0.6/2) = (0.3, 0.5, 0.2, 0.3) -> top 2: positions 1, 0
    (0 wins the tie with 3)."""
    rng = np.random.default_rng(43)
    q, K, V = rng.normal(size=(2, 8)), rng.normal(size=(4, 8)), rng.normal(size=(4, 8))
    _, active, _, _ = recas.sparse_decode_step(q, K, V, [0.9, 0.5, 0.2, 0.6], [3, 1, 1, 2], 0.5, 0.0, 1.0)
    np.testing.assert_array_equal(active, [0, 1])
