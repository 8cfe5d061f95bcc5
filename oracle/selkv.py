"""SelKV routing, soft-cosine-gated merging, attention ratio and compensated decode (fp64, test infrastructure only).

Page: [SelKV] "SelKV: Selective KV Cache Merging with Per-Token Merge-or-Drop
and Attention Compensation" (gist.science).

Readings (listed with reasons in the design notes):
  R12 the routing target of an evicted token is the kept token of its
      positional bucket (floor(pos / bucket)) with the highest prefill window
      attention of that KV head; ties go to the lower position.  A bucket
      with no kept token drops its evicted tokens.
  R13 merge weights are the same prefill attention; only values are merged,
      keys stay; gates use the kept token's original value, so the result
      does not depend on the order of the evicted tokens.
  R14 R_{g,t} = (A_t + sum_j g_j A_j) / A_t per KV head; an unmerged slot
      has R = 1 exactly.
  R15 decode output is fp32/fp64; appended tokens carry R = 1.
  R23 RoPE re-positioning: keys carry the rotary embedding of their original
      positions; re-embedding at position p' rotates every dimension pair
      (i, i + d/2) by (p' - p) * base^(-2i/d), i < d/2 (the half-split pairing
      of the Llama / Qwen shapes used here; base given by the caller, no
      frequency scaling).  The kept slot j gets position new0 + j.
"""
from __future__ import annotations

import numpy as np

__all__ = ["merge", "soft_gate", "decode_attention", "rope_inv_freq", "rope_reposition"]


def soft_gate(v_evicted, v_kept) -> np.ndarray:
    """g = max(cos(v_evicted, v_kept), 0).

    [SelKV] Methodology, Core component 1 "soft cosine gate": g ~ 1 merges
    fully, g = 0 (orthogonal or opposed values) drops the token, values in
    between merge partially.  A zero-norm vector has cos := 0.
    """
    a = np.asarray(v_evicted, np.float64)
    b = np.asarray(v_kept, np.float64)
    dot = a @ b if a.ndim == 2 else float(a @ b)
    den = np.sqrt((a * a).sum(axis=-1)) * np.sqrt((b * b).sum())
    cos = np.where(den > 0.0, dot / np.where(den > 0.0, den, 1.0), 0.0)
    return np.maximum(cos, 0.0)


def merge(V, A, kept, bucket: int = 512):
    """O9  route every evicted token to its bucket's kept token, gate, merge values, and form R.

    [SelKV] Pipeline overview steps 3-5 (route evicted tokens inside
    positional buckets by prefill attention; soft-gated merge; attention
    compensation) and Methodology, Core components 1-2 (gated
    attention-weighted average of the kept value and the evicted
    contributions; R_{h,i} = attention mass the merged slot should receive
    relative to its original).

    V:    [n][d] values of one KV head (original positions 0..n-1)
    A:    [n] prefill window attention of that KV head
    kept: [k] ascending kept positions
    Returns (V' [k][d], R [k]):
        V'_t = (A_t v_t + sum_j g_j A_j v_j) / (A_t + sum_j g_j A_j)
        R_t  = (A_t + sum_j g_j A_j) / A_t
    for each bucket's target t; every other kept slot keeps v and R = 1.
    """
    V = np.asarray(V, np.float64)
    A = np.asarray(A, np.float64)
    kept = np.asarray(kept, dtype=np.int64)
    n = A.shape[0]
    is_kept = np.zeros(n, dtype=bool)
    is_kept[kept] = True
    slot = np.full(n, -1, dtype=np.int64)
    slot[kept] = np.arange(kept.shape[0])
    Vp = V[kept].copy()
    R = np.ones(kept.shape[0])
    for lo in range(0, n, bucket):
        hi = min(n, lo + bucket)
        kb = kept[(kept >= lo) & (kept < hi)]
        if kb.shape[0] == 0:
            continue                      # nothing to merge into: evicted tokens are dropped
        t = int(kb[np.argmax(A[kb])])     # first maximum is the lowest position
        if A[t] <= 0.0:
            continue
        ev = np.arange(lo, hi)[~is_kept[lo:hi]]
        if ev.shape[0] == 0:
            continue
        g = soft_gate(V[ev], V[t])
        wj = g * A[ev]
        den = A[t] + wj.sum()
        Vp[slot[t]] = (A[t] * V[t] + (wj[:, None] * V[ev]).sum(axis=0)) / den
        R[slot[t]] = den / A[t]
    return Vp, R


def decode_attention(q, K, V, R=None, alpha_c: float = 1.0, scale=None) -> np.ndarray:
    """O10  o = softmax(q k_i^T * scale + alpha_c * log R_i) V'.

    [SelKV] Methodology, Core component 2 "attention compensation": at decode
    time the bias alpha * log(R_i) is added to the attention logits of every
    cached slot so a merged slot receives attention in proportion to what it
    now represents.  q: [G][d], K, V: [m][d], R: [m] or None (no bias).
    """
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    s = (q @ K.T) * scale
    if R is not None:
        s = s + alpha_c * np.log(np.asarray(R, np.float64))[None, :]
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    return p @ V


def rope_inv_freq(d: int, base: float) -> np.ndarray:
    """Rotary frequencies theta_i = base^(-2i/d), i = 0 .. d/2 - 1 (fp64)."""
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def rope_reposition(K, old_pos, new_pos, base: float) -> np.ndarray:
    """Keys rotated at old_pos, re-embedded at new_pos.

    [SelKV] Pipeline overview, step 6 "RoPE re-positioning": the kept keys are
    re-embedded at contiguous positions (the pages switch the step off for
    long-context evaluation).  A rotary embedding at position p turns the pair
    (x_i, x_{i+d/2}) by the angle p * theta_i; moving a key from p to p' is
    one more turn by (p' - p) * theta_i (R23).

    K: [..., d]; old_pos, new_pos: integer arrays of K's leading shape.
    """
    K = np.asarray(K, np.float64)
    d = K.shape[-1]
    h = d // 2
    shift = np.asarray(new_pos, np.float64) - np.asarray(old_pos, np.float64)
    ang = shift[..., None] * rope_inv_freq(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = K[..., :h], K[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)
