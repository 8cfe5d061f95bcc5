"""Shared test helpers: exact host copies of device tensors and the comparison rules.

Comparison rules (restated from the tolerances the workload fixes):
* floating-point scores and signals: |gpu - oracle| <= 1e-4 * |oracle| + atol;
* kept index sets: identical except for positions whose oracle score lies
  within 1e-5 relative of the k-th threshold (tie zone);
* compaction: bit-exact given the indices;
* merged values and decode outputs: 2e-3 max-abs (fp32 outputs);
  merged bf16 cache values within one bf16 ulp of round-to-nearest(oracle).
"""
import numpy as np
import torch

SCORE_RTOL = 1e-4
TIE_REL = 1e-5
OUT_ATOL = 2e-3


def np64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a device/host tensor (bf16 and fp32 embed exactly)."""
    return t.detach().to("cpu", torch.float32).numpy().astype(np.float64) if t.is_floating_point() \
        else t.detach().cpu().numpy()


def assert_close_rel(gpu, ref, rtol=SCORE_RTOL, atol=0.0, what=""):
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    err = np.abs(g - r)
    lim = rtol * np.abs(r) + atol
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside rtol={rtol} atol={atol}; "
                             f"worst at {i}: gpu={g[i]!r} ref={r[i]!r}")


def kept_sets_agree(gpu_idx, ref_idx, zone):
    """True when the two kept sets differ only on tie-zone positions (and are equal in size)."""
    g = set(int(x) for x in gpu_idx)
    r = set(int(x) for x in ref_idx)
    if len(g) != len(r):
        return False, f"sizes {len(g)} vs {len(r)}"
    diff = g ^ r
    zs = set(int(x) for x in zone)
    outside = diff - zs
    if outside:
        return False, f"{len(outside)} differing positions outside the tie zone: {sorted(outside)[:10]}"
    return True, f"{len(diff)} tie-zone swaps"


def bf16_rne(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(x, np.float64))
    a = np.where(a > 0, a, 1e-38)
    e = np.floor(np.log2(a))
    return 2.0 ** (e - 7)


# --------------------------------------------------------------------------- derived bounds
#
# Two GPU results depend on other GPU results that are themselves only within a
# tolerance of the oracle's: the end-to-end merged values (through the GPU's window
# attention A) and the RECAS dropped mass delta (through fp32 logits).  Their test
# tolerances are derived here from that input error and the fp32 arithmetic, instead
# of being set by hand.

U32 = 2.0 ** -24          # fp32 unit roundoff (round to nearest)


def merge_value_bound(V, kept, bucket, Vp_ref, eps_A=SCORE_RTOL):
    """Per-element bound on |V'_gpu - V'_oracle| for the merged values of one (layer, KV head).

    V' is a weighted mean of value rows: V'_t = sum_i w_i v_i / sum_i w_i with
    w = (A_t, g_j A_j).  When every weight carries a relative error of at most e,
    the mean moves by at most e / (1 - e) * max_i |v_i - V'_t| (per component),
    the max taken over the rows in the mean; here over every row of t's bucket,
    a superset.  The gate g is an fp32 cosine of two d-vectors: e gets d * u more.
    The fp32 sums of up to one bucket of terms add gamma_m * (max|v| + |V'|) with
    gamma_m = m u / (1 - m u).

    V [n][d], kept [k] ascending positions, Vp_ref [k][d] -> bound [k][d].
    """
    V = np.asarray(V, np.float64)
    kept = np.asarray(kept)
    Vp_ref = np.asarray(Vp_ref, np.float64)
    n, d = V.shape
    e = eps_A + d * U32
    gm = (bucket + 1) * U32 / (1 - (bucket + 1) * U32)
    out = np.zeros_like(Vp_ref)
    for j, t in enumerate(kept):
        lo = (int(t) // bucket) * bucket
        rows = V[lo:min(n, lo + bucket)]
        spread = np.abs(rows - Vp_ref[j][None, :]).max(axis=0)
        vmax = np.abs(rows).max(axis=0)
        out[j] = e / (1 - e) * spread + gm * (vmax + np.abs(Vp_ref[j])) + 4 * U32 * np.abs(Vp_ref[j])
    return out


def ratio_bound(R_ref, eps_A=SCORE_RTOL):
    """Bound on |R_gpu - R_oracle|: R = 1 + sum_j g_j A_j / A_t; with every A within e
    relative, the ratio term moves by at most 2 e / (1 - e) of itself, plus fp32
    rounding of the sum and the division."""
    R_ref = np.asarray(R_ref, np.float64)
    e = eps_A + 128 * U32
    return (R_ref - 1.0) * 2 * e / (1 - e) + 520 * U32 * R_ref


def delta_rel_bound(q, K, scale, n_terms):
    """Relative bound on the GPU's dropped attention mass for query rows q [G][d] over
    keys K [t][d] (the exact bf16 inputs).

    Each logit s_i = scale * sum_j q_j k_ij is an fp32 dot product: |ds_i| <= D_i with
    D_i = gamma_d * scale * sum_j |q_j k_ij| (gamma_d for d terms, with the unit
    roundoff doubled to cover tensor-core accumulation that truncates).  delta is a
    ratio of sums of exp(s_i), so it moves by a factor within exp(+-2 max_i D_i).  The
    exponentials (ex2.approx, relative 2^-22) and the fp32 sums of n_terms terms add
    2^-21 + 2 gamma_{n_terms}.  Returns one bound per query row."""
    q = np.asarray(q, np.float64)
    K = np.asarray(K, np.float64)
    d = q.shape[-1]
    u2 = 2 * U32
    gd = d * u2 / (1 - d * u2)
    Dmax = gd * scale * (np.abs(q) @ np.abs(K).T).max(axis=-1)
    gt = n_terms * U32 / (1 - n_terms * U32)
    return np.expm1(2 * Dmax) + 2.0 ** -21 + 2 * gt
