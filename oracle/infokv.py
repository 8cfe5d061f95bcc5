"""InfoKV token scoring, budgets and selection restated in fp64 (test infrastructure only).

Page: [InfoKV] "긴 추론을 위한 정보 인지형 KV 캐시 압축(InfoKV)" (aitrends.kr).

Readings of points the page leaves open (each one is listed with its reason
in the design notes of the repository):
  R1  top-k restricted entropy: the k largest logits are renormalised to a
      distribution of their own; natural logarithm.
  R2  the distribution of token i is the logits row produced at position i.
  R3  A^(l) is computed from layer l's own window queries and keys.
  R4  causal by position, scale 1/sqrt(d), no pooling, query head h belongs
      to KV group h // G, A averaged over the G*W rows of the group.
  R5  Softmax(E^(l)) runs over every cached token of the row, temperature 1.
  R6  D = 1 - cos + tau with tau = 1; cos := 0 when either vector is zero.
  R7  E-bar^(l) is the mean of E^(l) over the row's tokens.
  R8  the budget k_l includes the recent window.
  R9  adaptive budgets: the proportional share clamped to [w, n] with the
      scale chosen so the shares sum to B, then largest remainder (ties to
      the lower layer), so they sum to B exactly.
  R11 ties in the top-k go to the lower position; index lists ascend.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "topk_entropy", "lmhead_topk_entropy", "repr_change", "entropy_scores", "window_attention",
    "combine", "vatp", "union_max", "uniform_budgets", "adaptive_budgets",
    "select_topk", "tie_zone", "compact",
]


def topk_entropy(logits, k: int = 256) -> np.ndarray:
    """O1  H_i: entropy of token i's final-layer predictive distribution over its top k entries.

    [InfoKV] Methodology (second signal: top-k restricted entropy of the
    final layer's predictive distribution) and Glossary entry "Top-k
    restricted entropy"; k = 256 per Key contributions / Methodology.

    logits: [..., V] -> H: [...].  Only the multiset of the k largest values
    matters, so ties at the k-th value do not change the result.
    """
    z = np.asarray(logits, dtype=np.float64)
    V = z.shape[-1]
    kk = min(int(k), V)
    top = np.partition(z, V - kk, axis=-1)[..., V - kk:]
    top = top - top.max(axis=-1, keepdims=True)
    e = np.exp(top)
    q = e / e.sum(axis=-1, keepdims=True)
    safe = np.where(q > 0.0, q, 1.0)
    return -np.where(q > 0.0, q * np.log(safe), 0.0).sum(axis=-1)


def lmhead_topk_entropy(x, W, k: int = 256) -> np.ndarray:
    """O1' H_i from the LM head's input instead of its logits: z_i = W x_i, then O1.

    [InfoKV] Methodology (H_i is taken from the final layer's predictive
    distribution).  The distribution of position i is softmax(W x_i), x_i the
    LM head's input at position i (the final hidden state after the model's
    last normalisation) and W the [V][Dh] output projection; only its k largest
    logits enter H (O1), so the full row need not be kept.

    x: [n, Dh], W: [V, Dh] -> H: [n].
    """
    xx = np.asarray(x, dtype=np.float64)
    ww = np.asarray(W, dtype=np.float64)
    return topk_entropy(xx @ ww.T, k)


def repr_change(h_l, h_L, tau: float = 1.0) -> np.ndarray:
    """O2  D_i^(l) = 1 - cos(h_i^(l), h_i^(L)) + tau.

    [InfoKV] Methodology (cosine distance between layer l's and the final
    layer's hidden states) and Technical details (a bias tau keeps the final
    layer's score from vanishing; tau = 1).

    h_l, h_L: [..., Dh] -> D: [...].
    """
    a = np.asarray(h_l, dtype=np.float64)
    b = np.asarray(h_L, dtype=np.float64)
    dot = (a * b).sum(axis=-1)
    den = np.sqrt((a * a).sum(axis=-1)) * np.sqrt((b * b).sum(axis=-1))
    cos = np.where(den > 0.0, dot / np.where(den > 0.0, den, 1.0), 0.0)
    return 1.0 - cos + tau


def entropy_scores(D, H):
    """O3  E^(l) = D^(l) * H, its Softmax over the row's tokens, and its mean E-bar^(l).

    [InfoKV] Methodology (layer entropy score E_i^(l) = D_i^(l) * H_i,
    Softmax-normalised within the layer) and Technical details (Softmax
    normalises over the tokens of the layer).

    D: [..., n], H broadcastable to it -> (E, P, Ebar) with P summing to 1
    over the last axis.
    """
    E = np.asarray(D, dtype=np.float64) * np.asarray(H, dtype=np.float64)
    m = E.max(axis=-1, keepdims=True)
    e = np.exp(E - m)
    P = e / e.sum(axis=-1, keepdims=True)
    return E, P, E.mean(axis=-1)


def window_attention(Qg, K, qpos=None, kpos=None, scale=None) -> np.ndarray:
    """O4  A_i: observation-window attention of one KV head.

    [InfoKV] Methodology (window attention weights averaged to A_i^(l)) and
    Technical details (A_i^(l) from the query-key interaction inside the
    observation window of layer l).

    Qg:   [G][W][d] window queries of the G query heads sharing this KV head
    K:    [n][d] keys
    qpos: [W] query positions (default n-W .. n-1); kpos: [n] key positions
          (default 0 .. n-1).  Key i is visible to query r iff kpos[i] <= qpos[r].
    Returns A: [n], the mean over the G*W rows of each row's softmax.
    """
    Qg = np.asarray(Qg, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    G, W, d = Qg.shape
    n = K.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    kpos = np.arange(n) if kpos is None else np.asarray(kpos)
    qpos = np.arange(n - W, n) if qpos is None else np.asarray(qpos)
    hidden = kpos[None, :] > qpos[:, None]
    A = np.zeros(n)
    for h in range(G):
        s = (Qg[h] @ K.T) * scale
        s = np.where(hidden, -np.inf, s)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        A += p.sum(axis=0)
    return A / (G * W)


def combine(A, P, alpha: float = 0.9) -> np.ndarray:
    """O5  S^(l) = alpha * A^(l) + (1 - alpha) * Softmax(E^(l)).

    [InfoKV] Methodology (weighted sum of attention and entropy score) and
    Technical details (alpha = 0.9).
    """
    return alpha * np.asarray(A, np.float64) + (1.0 - alpha) * np.asarray(P, np.float64)


def vatp(A, V) -> np.ndarray:
    """SelKV importance: attention times value norm.

    [SelKV] Pipeline overview, step 1 (importance = attention weight x value
    vector magnitude).  A: [..., n], V: [..., n, d].
    """
    V = np.asarray(V, np.float64)
    return np.asarray(A, np.float64) * np.sqrt((V * V).sum(axis=-1))


def union_max(S) -> np.ndarray:
    """GQA union score: a token is ranked by its best KV head, S-hat_i = max_g S_{g,i}.

    [SelKV] Pipeline overview, step 2 (selection per head for MHA, through
    the union for GQA).  S: [Hkv][n] -> [n].
    """
    return np.asarray(S, np.float64).max(axis=0)


def uniform_budgets(n: int, rho: float, L: int, w: int) -> np.ndarray:
    """O6a  uniform per-layer budget k_l = floor(rho * n), clamped to [min(w, n), n].

    [InfoKV] Technical details and Hyper-parameters paragraph (uniform layer
    budget is the default).
    """
    k = int(np.floor(float(rho) * float(n)))
    k = min(n, max(min(w, n), k))
    return np.full(L, k, dtype=np.int64)


def adaptive_budgets(Ebar, B: int, w: int, n: int) -> np.ndarray:
    """O6b  adaptive budgets k_l = (E-bar^(l) / sum_m E-bar^(m)) * B, as integers summing to B.

    [InfoKV] Methodology and Technical details (k_l proportional to the
    layer's cumulative entropy share) and Glossary entry "Adaptive budget
    allocation".  Reading R9: every layer keeps at least its recent window
    and at most its n tokens, so the share is clamped -
    x_l = clamp(lambda * E-bar^(l), min(w, n), n) with lambda the scale for
    which sum_l x_l = B (clamped proportional share; without active bounds
    this is exactly the page's formula).  Integers: floor, then one extra
    token to the layers with the largest fractional parts (ties to the lower
    layer), never past n.
    """
    E = np.asarray(Ebar, dtype=np.float64)
    L = E.shape[0]
    lo, hi = min(w, n), n
    if not (E > 0).any():
        E = np.ones(L)                    # no entropy anywhere: equal shares
    if not (L * lo <= B <= L * hi):
        raise ValueError("total budget outside [L*min(w,n), L*n]")

    def f(lam):
        return np.clip(lam * E, lo, hi).sum()

    # f is continuous, piecewise linear and non-decreasing in lambda; its
    # breakpoints are where a layer leaves the lower bound or hits the upper.
    bps = [0.0] + [lo / e for e in E if e > 0] + [hi / e for e in E if e > 0]
    b0 = max(b for b in bps if f(b) <= B)
    above = [b for b in bps if b > b0]
    mid = 0.5 * (b0 + min(above)) if above else 2.0 * b0 + 1.0
    # on (b0, next breakpoint) the free layers are the ones strictly inside the bounds
    slope = sum(e for e in E if lo < mid * e < hi)
    lam = b0 if slope == 0.0 else b0 + (B - f(b0)) / slope
    x = np.clip(lam * E, lo, hi)
    k = np.floor(x).astype(np.int64)
    frac = x - k
    extra = B - int(k.sum())
    order = sorted((l for l in range(L) if k[l] < hi), key=lambda l: (-frac[l], l))
    for l in order[:max(extra, 0)]:
        k[l] += 1
    return k


def select_topk(S, k: int, w: int) -> np.ndarray:
    """O7  kept positions of one row: the last w positions plus the top (k - w) of the rest.

    [InfoKV] Technical details (keep the top k_l tokens of each layer) and
    [SelKV] Pipeline overview step 2 (top tokens together with a recent
    window).  Ties go to the lower position (R11); the result ascends.
    """
    S = np.asarray(S, dtype=np.float64)
    n = S.shape[0]
    w_ = min(w, n)
    k_ = min(k, n)
    if k_ < w_:
        raise ValueError("budget smaller than the recent window")
    cand = np.arange(n - w_)
    order = np.lexsort((cand, -S[: n - w_]))
    chosen = cand[order[: k_ - w_]]
    return np.sort(np.concatenate([chosen, np.arange(n - w_, n)]))


def tie_zone(S, k: int, w: int, rel: float = 1e-5) -> np.ndarray:
    """Positions whose score lies within rel (relative) of the k-th threshold of select_topk.

    Test helper: kept sets may legitimately differ only on these positions.
    """
    S = np.asarray(S, dtype=np.float64)
    n = S.shape[0]
    w_ = min(w, n)
    k_ = min(k, n)
    m = k_ - w_
    if m <= 0 or m >= n - w_:
        return np.zeros(0, dtype=np.int64)
    cand = S[: n - w_]
    thr = np.sort(cand)[::-1][m - 1]
    return np.flatnonzero(np.abs(cand - thr) <= rel * abs(thr))


def compact(X, idx) -> np.ndarray:
    """O8  compaction: row j of the result is row idx[j] of X (X: [n, ...])."""
    return np.asarray(X)[np.asarray(idx)]
