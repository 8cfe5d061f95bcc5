"""RECAS dropped attention mass and its output-error bound (fp64, test infrastructure only).

Page: [RECAS] "기술 요약: 긴 문맥 LLM을 위한 추론 인지적 오차 경계 KV-캐시 압축
및 희소 어텐션" (gist.science), section 2.B "error-bounded adaptive KV-cache
compression".

Reading R16: p is the full-history attention of the same query with no
bias; delta_t is the sum of p over evicted tokens; V_max is the largest value
norm of the full history of that KV head; the compressed output o' is plain
attention renormalised over the kept tokens.  Then
    o - o' = sum_ev p_i v_i - delta/(1-delta) * sum_kept p_i v_i,
and both terms have norm <= delta * V_max, which is the page's bound
||o - o'||_2 <= 2 * V_max * delta.
"""
from __future__ import annotations

import numpy as np

__all__ = ["dropped_mass_probe"]


def dropped_mass_probe(q, K, V, kept_mask, scale=None):
    """O11  delta, V_max, o (full), o' (kept only), ||o - o'||_2 and 2 * V_max * delta per query row.

    q: [G][d]; K, V: [t][d] full history; kept_mask: [t] bool.
    Returns a dict of arrays, one entry per query row (o and o' are [G][d]).
    """
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    kept = np.asarray(kept_mask, dtype=bool)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    s = (q @ K.T) * scale
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    p = e / e.sum(axis=-1, keepdims=True)
    delta = p[:, ~kept].sum(axis=-1)
    o_full = p @ V
    ek = e[:, kept]
    o_kept = (ek / ek.sum(axis=-1, keepdims=True)) @ V[kept]
    vmax = float(np.sqrt((V * V).sum(axis=-1)).max()) if V.shape[0] else 0.0
    err = np.sqrt(((o_full - o_kept) ** 2).sum(axis=-1))
    return {"delta": delta, "vmax": vmax, "o_full": o_full, "o_kept": o_kept,
            "err": err, "bound": 2.0 * vmax * delta}


# --------------------------------------------------------------------------- calibrated estimator
#
# [RECAS] 2.B "calibrated estimator": after eviction the exact full-cache attention is
# gone, so the dropped mass is estimated from a normalised predictor and recalibrated at
# periodic full-attention probe steps; a conservative upper estimate comes from the
# empirical (1 - alpha)-quantile of the residuals.  "adaptive controller": when that
# upper estimate threatens the error target eps_t, the cache budget grows, keeping
# tokens in utility order, until the bound holds.
#
# Readings (the page names the parts, not their formulas):
#   R24 normalised predictor: for a (layer, KV head) row compressed with window
#       attention A (normalised over the row's cached tokens), x = share of A on the
#       tokens the compression drops, x = 1 - sum_kept A / sum_all A.  It stays fixed
#       until the row's next compression.
#   R25 calibration, per (sequence, layer): at a probe step the exact delta of every
#       query head h is known.  Residuals r_h = delta_h - c * x_{g(h)} use the ratio
#       estimate c from the probes before this one (out of sample; c = 1 before any
#       probe); they join a ring of the last M residuals; then c = sum delta / sum x over
#       every probe so far.  q = the ceil((m + 1)(1 - alpha))-th smallest of the m
#       residuals in the ring (the split-conformal quantile; +inf when that rank exceeds
#       m).  Estimate delta_hat = c x, upper bound delta_bar = c x + q.
#   R26 controller: the utility order is the compression score S the selection ranks
#       by (the RECAS stage term gi is out of scope).  A row needs the smallest budget
#       k >= k0 = floor(rho t) whose kept set (recent window plus top k - w by S) leaves
#       x(k) with c x(k) + q <= eps; none up to the row's length: the whole row.  The
#       batch keeps B_t = the largest need over every row of every sequence, so the
#       caches stay rectangular.

RING = 256


def dropped_share(A, kept):
    """R24  x = 1 - sum over kept of A / sum of A (A >= 0, one row)."""
    A = np.asarray(A, np.float64)
    tot = A.sum()
    if tot <= 0.0:
        return 0.0
    return 1.0 - A[np.asarray(kept, dtype=np.int64)].sum() / tot


def conformal_quantile(residuals, alpha: float) -> float:
    """R25  the ceil((m + 1)(1 - alpha))-th smallest of m residuals; +inf if m is too small.

    The rank is taken 1e-12 below the product so that a product that is an integer in
    exact arithmetic (e.g. 10 * 0.9) is not pushed up by the binary rounding of 1 - alpha."""
    r = np.sort(np.asarray(residuals, np.float64))
    m = r.shape[0]
    rank = int(np.ceil((m + 1) * (1.0 - alpha) - 1e-12))
    if rank < 1:
        rank = 1
    return float(r[rank - 1]) if rank <= m else float("inf")


class DroppedMassCalibrator:
    """R25  ratio calibration of the predictor and the residual quantile of one (sequence, layer)."""

    def __init__(self, alpha: float = 0.1, ring: int = RING):
        self.alpha = alpha
        self.ring = ring
        self.res = []          # last `ring` residuals, oldest first
        self.sum_delta = 0.0
        self.sum_x = 0.0

    @property
    def c(self) -> float:
        return self.sum_delta / self.sum_x if self.sum_x > 0.0 else 1.0

    @property
    def q(self) -> float:
        return conformal_quantile(self.res, self.alpha)

    def observe(self, delta, x, G: int):
        """One probe step: delta [Hq] exact dropped mass per query head, x [Hkv] predictors."""
        delta = np.asarray(delta, np.float64)
        xh = np.repeat(np.asarray(x, np.float64), G)          # query head h reads KV head h // G
        c = self.c
        self.res.extend((delta - c * xh).tolist())
        self.res = self.res[-self.ring:]
        self.sum_delta += float(delta.sum())
        self.sum_x += float(xh.sum())

    def estimate(self, x):
        """(delta_hat, delta_bar) for predictors x."""
        x = np.asarray(x, np.float64)
        return self.c * x, self.c * x + self.q


def dropped_share_curve(S, A, w: int):
    """x(k) for every budget k = min(w, n) .. n of one row: the kept set is the recent
    window plus the top k - w by S (ties to the lower position), as in selection."""
    S = np.asarray(S, np.float64)
    A = np.asarray(A, np.float64)
    n = S.shape[0]
    w_ = min(w, n)
    tot = A.sum()
    cand = np.arange(n - w_)
    order = cand[np.lexsort((cand, -S[: n - w_]))]
    kept_mass = A[n - w_:].sum() + np.concatenate([[0.0], np.cumsum(A[order])])
    x = 1.0 - kept_mass / tot if tot > 0 else np.zeros(n - w_ + 1)
    return np.arange(w_, n + 1), x


def controller_need(S, A, w: int, k0: int, c: float, q: float, eps: float) -> int:
    """R26  the smallest k >= k0 whose kept set has c x(k) + q <= eps (the row's length if none)."""
    ks, x = dropped_share_curve(S, A, w)
    ok = (ks >= k0) & (c * x + q <= eps)
    return int(ks[ok][0]) if ok.any() else int(ks[-1])


# --------------------------------------------------------------------------- dynamic sparse decode
#
# [RECAS] 2.C "dynamic sparse decoding attention": inside the retained cache C_t a
# query-aware selector limits the interactions of each step.  The sparse score combines
# the immediate query-key compatibility with the utility score; the top K_t form the
# active set S_t; tokens outside S_t stay in C_t for later steps.  2.A: the utility
# u_i = alpha_t tr_i + beta_t hi_i + gamma_t gi (tr the query-key compatibility, hi the
# normalised attention accumulated over earlier steps, gi the reasoning-stage term).
# 2.D: active attention cost O(kappa_t rho_t N d), kappa_t the active ratio.
#
# Readings:
#   R27 per (sequence, layer, KV head) row: tr_i = attention of cached token i under the
#       current query, averaged over the G query heads of the KV head (softmax over the
#       retained cache, scale 1/sqrt(d)); hi_i = acc_i / cnt_i, acc_i the attention the
#       token received (mean over the heads, from the sparse attention actually
#       computed; 0 at a step where it was inactive) summed over the steps it has been
#       cached, cnt_i the number of those steps (this one included); sigma_i = a_tr tr_i
#       + b_hi hi_i.  gi needs the model's reasoning-stage signal: out of scope.
#   R28 K_t = ceil(kappa n) (at least 1, at most n) for a row of n cached tokens; S_t = the
#       top K_t by sigma, ties to the lower position.
#   R29 the output is attention renormalised over S_t (each head of the group, scale
#       1/sqrt(d)); acc_i += the mean over the heads of that attention, for i in S_t.


def sparse_active_count(n: int, kappa: float) -> int:
    """R28  K_t = ceil(kappa n), clamped to [1, n] (n >= 1)."""
    k = int(np.ceil(kappa * n - 1e-12))
    return min(n, max(1, k))


def sparse_decode_step(q, K, V, acc, cnt, kappa: float, a_tr: float, b_hi: float, scale=None):
    """R27-R29  one step of dynamic sparse decoding over one row of the retained cache.

    q [G][d]; K, V [n][d]; acc [n] accumulated attention; cnt [n] steps cached (>= 1).
    Returns (o [G][d], ascending active positions, new acc, sigma)."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    acc = np.asarray(acc, np.float64)
    cnt = np.asarray(cnt, np.float64)
    n, d = K.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    s = (q @ K.T) * scale                                 # [G][n]
    e = np.exp(s - s.max(axis=1, keepdims=True))
    tr = (e / e.sum(axis=1, keepdims=True)).mean(axis=0)
    sigma = a_tr * tr + b_hi * (acc / cnt)
    kt = sparse_active_count(n, kappa)
    idx = np.arange(n)
    active = np.sort(idx[np.lexsort((idx, -sigma))][:kt])
    sa = s[:, active]
    ea = np.exp(sa - sa.max(axis=1, keepdims=True))
    pa = ea / ea.sum(axis=1, keepdims=True)              # [G][K_t]
    o = pa @ V[active]
    acc_new = acc.copy()
    acc_new[active] += pa.mean(axis=0)
    return o, active, acc_new, sigma


def cached_steps(pos, t_cur: int, n_prompt: int):
    """R27  cnt_i: decode steps token i has been cached, this one included, when the
    sequence is t_cur long: t_cur - max(pos_i, n_prompt)."""
    return t_cur - np.maximum(np.asarray(pos), n_prompt)
