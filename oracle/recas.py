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
