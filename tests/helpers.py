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
