"""Planted mistakes: the pins must catch every plausible slip in the oracle.

Each mutant edits one line of an oracle module's source on the CPU - a dropped term,
a flipped sign, an off-by-one, a swapped operand or axis, a wrong tie rule, a missing
clamp - and the pins of test_oracle_pins.py run against the edited module in this
process.  At least one pin must fail; the module is restored afterwards.  This is how
the pins are known to hold the oracle to the pages rather than to itself.
"""
import importlib
import itertools

import pytest

from tests import test_oracle_pins as pins

MODULES = {"infokv": "oracle.infokv", "selkv": "oracle.selkv", "recas": "oracle.recas",
           "pipeline": "oracle.pipeline"}

# (module, original line, planted line, what the mistake is)
MUTANTS = [
    ("infokv", "kk = min(int(k), V)", "kk = min(int(k) - 1, V)", "top-k one short"),
    ("infokv", "top = np.partition(z, V - kk, axis=-1)[..., V - kk:]", "top = z",
     "entropy over the whole vocabulary"),
    ("infokv", "return -np.where(q > 0.0, q * np.log(safe), 0.0).sum(axis=-1)",
     "return np.where(q > 0.0, q * np.log(safe), 0.0).sum(axis=-1)", "entropy sign"),
    ("infokv", "return topk_entropy(xx @ ww.T, k)", "return topk_entropy(xx @ ww[:, ::-1].T, k)",
     "LM-head input dimensions paired with the wrong weight columns"),
    ("infokv", "return topk_entropy(xx @ ww.T, k)", "return topk_entropy(xx @ ww.T / np.sqrt(ww.shape[1]), k)",
     "LM-head logits scaled by 1/sqrt(Dh)"),
    ("infokv", "return topk_entropy(xx @ ww.T, k)", "return topk_entropy(np.abs(xx) @ ww.T, k)",
     "LM-head input taken by magnitude"),
    ("infokv", "    return 1.0 - cos + tau\n", "    return 1.0 - cos\n", "tau dropped"),
    ("infokv", "    return 1.0 - cos + tau\n", "    return 1.0 + cos + tau\n", "cosine sign"),
    ("infokv", "E = np.asarray(D, dtype=np.float64) * np.asarray(H, dtype=np.float64)",
     "E = np.asarray(D, dtype=np.float64) + np.asarray(H, dtype=np.float64)", "E as D + H"),
    ("infokv", "    return E, P, E.mean(axis=-1)", "    return E, P, E.sum(axis=-1)", "E-bar as a sum"),
    ("infokv", "hidden = kpos[None, :] > qpos[:, None]", "hidden = kpos[None, :] >= qpos[:, None]",
     "causal mask hides the query's own position"),
    ("infokv", "hidden = kpos[None, :] > qpos[:, None]", "hidden = kpos[None, :] < 0", "no causal mask"),
    ("infokv", "scale = 1.0 / np.sqrt(d)", "scale = 1.0 / d", "logit scale 1/d"),
    ("infokv", "    return A / (G * W)", "    return A / W", "window mean over W rows only"),
    ("infokv", "return alpha * np.asarray(A, np.float64) + (1.0 - alpha) * np.asarray(P, np.float64)",
     "return (1.0 - alpha) * np.asarray(A, np.float64) + alpha * np.asarray(P, np.float64)",
     "alpha and 1 - alpha swapped"),
    ("infokv", "return np.asarray(A, np.float64) * np.sqrt((V * V).sum(axis=-1))",
     "return np.asarray(A, np.float64) * (V * V).sum(axis=-1)", "squared value norm in VATP"),
    ("infokv", "return np.asarray(S, np.float64).max(axis=0)", "return np.asarray(S, np.float64).mean(axis=0)",
     "GQA union by mean"),
    ("infokv", "k = int(np.floor(float(rho) * float(n)))", "k = int(np.ceil(float(rho) * float(n)))",
     "uniform budget rounded up"),
    ("infokv", "key=lambda l: (-frac[l], l))", "key=lambda l: (-frac[l], -l))",
     "largest-remainder ties to the higher layer"),
    ("infokv", "x = np.clip(lam * E, lo, hi)", "x = lam * E", "adaptive budget clamp dropped"),
    ("infokv", "order = np.lexsort((cand, -S[: n - w_]))", "order = np.lexsort((-cand, -S[: n - w_]))",
     "selection ties to the higher position"),
    ("infokv", "return np.sort(np.concatenate([chosen, np.arange(n - w_, n)]))",
     "return np.sort(np.concatenate([chosen, np.arange(n - w_ - 1, n - 1)]))", "recent window off by one"),
    ("infokv", "return np.asarray(X)[np.asarray(idx)]", "return np.asarray(X)[np.asarray(idx)[::-1]]",
     "compaction order reversed"),
    ("selkv", "return np.maximum(cos, 0.0)", "return cos", "gate not clamped at 0"),
    ("selkv", "return np.maximum(cos, 0.0)", "return np.abs(cos)", "gate by |cos|"),
    ("selkv", "t = int(kb[np.argmax(A[kb])])", "t = int(kb[np.argmin(A[kb])])",
     "routing to the least-attended kept token"),
    ("selkv", "R[slot[t]] = den / A[t]", "R[slot[t]] = A[t] / den", "attention ratio inverted"),
    ("selkv", "wj = g * A[ev]", "wj = g", "merge weight without attention"),
    ("selkv", "s = s + alpha_c * np.log(np.asarray(R, np.float64))[None, :]",
     "s = s - alpha_c * np.log(np.asarray(R, np.float64))[None, :]", "decode bias sign"),
    ("recas", "delta = p[:, ~kept].sum(axis=-1)", "delta = p[:, kept].sum(axis=-1)", "kept mass taken as delta"),
    ("recas", '"bound": 2.0 * vmax * delta}', '"bound": vmax * delta}', "bound without the factor 2"),
    ("recas", "o_kept = (ek / ek.sum(axis=-1, keepdims=True)) @ V[kept]", "o_kept = ek @ V[kept]",
     "kept attention not renormalised"),
    ("recas", "vmax = float(np.sqrt((V * V).sum(axis=-1)).max()) if V.shape[0] else 0.0",
     "vmax = float(np.sqrt((V[kept] * V[kept]).sum(axis=-1)).max()) if V.shape[0] else 0.0",
     "V_max over the kept values only"),
    ("pipeline", "k = int(np.floor(self.rho * self.t))", "k = int(np.floor(self.rho * (self.t - 1)))",
     "recompression length from t - 1"),
    ("pipeline", "self.H[l][g] = self.H[l][g][keep]", "self.H[l][g] = self.H[l][g][:len(keep)]",
     "H does not travel with its token"),
    ("pipeline", "self.qring.pop(0)", "self.qring.pop()", "query ring drops the newest query"),
    ("pipeline", "o[l, g * G:(g + 1) * G] = selkv.decode_attention(qg, self.K[l][g], self.V[l][g])",
     "o[l, g * G:(g + 1) * G] = selkv.decode_attention(qg, self.Kfull[l][g], self.Vfull[l][g])",
     "decode over the full history"),
    ("pipeline", "mask[self.pos[l][g]] = True", "mask[self.pos[l][g][:-1]] = True",
     "probe's kept mask one row short"),
    ("pipeline", "keep = ik.select_topk(ik.union_max(S[l]), int(budgets[l]), w)",
     "keep = ik.select_topk(S[l, 0], int(budgets[l]), w)", "union ranked by the first head only"),
    ("pipeline", "idx[l][g] = ik.select_topk(S[l, g], int(budgets[l]), w)",
     "idx[l][g] = ik.select_topk(S[l, 0], int(budgets[l]), w)", "every head ranked by head 0"),
    ("pipeline", "A[l, g] = ik.window_attention(np.asarray(Qw[l, g * G:(g + 1) * G], np.float64), K[l, g])",
     "A[l, g] = ik.window_attention(np.asarray(Qw[l, g::Hkv], np.float64), K[l, g])",
     "query heads grouped by h mod Hkv (interleaved)"),
    ("pipeline", "hL = np.asarray(hidden[L - 1], np.float64)", "hL = np.asarray(hidden[0], np.float64)",
     "h^(L) taken from the first stored layer"),
    ("pipeline", 'out["S"] = ik.combine(A, out["P"][:, None, :], alpha)',
     'out["S"] = ik.combine(A, out["P"][None, :, :], alpha)', "entropy softmax broadcast over the wrong axis"),
    ("pipeline", 'out["S"] = ik.vatp(A, V)', 'out["S"] = A', "VATP mode without the value norm"),
    ("infokv", "thr = np.sort(cand)[::-1][m - 1]", "thr = np.sort(cand)[::-1][m]",
     "tie-zone threshold one past the k-th candidate"),
    ("infokv", "    cand = S[: n - w_]\n    thr", "    cand = S\n    thr", "tie zone over the recent window too"),
    ("recas", "rank = int(np.ceil((m + 1) * (1.0 - alpha) - 1e-12))",
     "rank = int(np.ceil(m * (1.0 - alpha) - 1e-12))", "quantile rank without the conformal +1"),
    ("recas", "self.res.extend((delta - c * xh).tolist())", "self.res.extend((delta - xh).tolist())",
     "residuals against the uncalibrated predictor"),
    ("recas", "return self.sum_delta / self.sum_x if self.sum_x > 0.0 else 1.0",
     "return self.sum_x / self.sum_delta if self.sum_delta > 0.0 else 1.0", "calibration ratio inverted"),
    ("recas", "xh = np.repeat(np.asarray(x, np.float64), G)", "xh = np.tile(np.asarray(x, np.float64), G)",
     "query heads matched to KV heads by h mod Hkv"),
    ("recas", "return self.c * x, self.c * x + self.q", "return self.c * x, self.c * x",
     "upper bound without the residual quantile"),
    ("recas", "kept_mass = A[n - w_:].sum() + np.concatenate([[0.0], np.cumsum(A[order])])",
     "kept_mass = np.concatenate([[0.0], np.cumsum(A[order])])", "recent window's mass not counted as kept"),
    ("recas", "ok = (ks >= k0) & (c * x + q <= eps)", "ok = (ks >= k0) & (c * x <= eps)",
     "controller ignores the residual quantile"),
    ("recas", "order = cand[np.lexsort((cand, -S[: n - w_]))]", "order = cand[np.lexsort((cand, S[: n - w_]))]",
     "controller re-admits the lowest-utility tokens first"),
    ("recas", "k = int(np.ceil(kappa * n - 1e-12))", "k = int(np.floor(kappa * n - 1e-12))",
     "active count rounded down"),
    ("recas", "tr = (e / e.sum(axis=1, keepdims=True)).mean(axis=0)",
     "tr = (e / e.sum(axis=1, keepdims=True)).sum(axis=0)", "query term summed over the heads"),
    ("recas", "sigma = a_tr * tr + b_hi * (acc / cnt)", "sigma = a_tr * tr + b_hi * acc",
     "history term not normalised by the cached steps"),
    ("recas", "active = np.sort(idx[np.lexsort((idx, -sigma))][:kt])",
     "active = np.sort(idx[np.lexsort((-idx, -sigma))][:kt])", "active-set ties to the higher position"),
    ("recas", "o = pa @ V[active]", "o = (e / e.sum(axis=1, keepdims=True))[:, active] @ V[active]",
     "sparse output not renormalised over the active set"),
    ("recas", "acc_new[active] += pa.mean(axis=0)", "acc_new[active] += pa.sum(axis=0)",
     "history accumulates the head sum"),
    ("recas", "return t_cur - np.maximum(np.asarray(pos), n_prompt)",
     "return t_cur - np.maximum(np.asarray(pos), n_prompt) + 1", "cached steps off by one"),
    ("selkv", "return np.power(float(base), -2.0 * i / d)", "return np.power(float(base), -1.0 * i / d)",
     "rotary frequency exponent i/d"),
    ("selkv", "shift = np.asarray(new_pos, np.float64) - np.asarray(old_pos, np.float64)",
     "shift = np.asarray(old_pos, np.float64) - np.asarray(new_pos, np.float64)", "re-positioning turned backwards"),
    ("selkv", "x1, x2 = K[..., :h], K[..., h:]", "x1, x2 = K[..., 0::2], K[..., 1::2]",
     "interleaved instead of half-split pairs"),
    ("selkv", "return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)",
     "return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)", "rotation sign"),
]


def _pin_cases():
    """Every pin test of test_oracle_pins.py with its parameter sets expanded."""
    for name in sorted(dir(pins)):
        fn = getattr(pins, name)
        if not (name.startswith("test_") and callable(fn)):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            yield name, fn, {}
            continue
        grids = []
        for m in marks:
            names = [s.strip() for s in m.args[0].split(",")]
            grids.append([dict(zip(names, v if len(names) > 1 else (v,))) for v in m.args[1]])
        for combo in itertools.product(*grids):
            kw = {}
            for d in combo:
                kw.update(d)
            yield name, fn, kw


def _first_failing_pin():
    for name, fn, kw in _pin_cases():
        try:
            fn(**kw)
        except Exception:                     # an assertion, or the mutant breaking a call
            return name
    return None


def test_unmutated_oracle_passes_every_pin():
    assert _first_failing_pin() is None


@pytest.mark.parametrize("mod,old,new,what", MUTANTS, ids=[m[3] for m in MUTANTS])
def test_pins_catch_planted_mistake(mod, old, new, what):
    m = importlib.import_module(MODULES[mod])
    src = open(m.__file__).read()
    assert src.count(old) == 1, f"mutation site not unique in {mod}: {old!r}"
    saved = dict(m.__dict__)
    try:
        exec(compile(src.replace(old, new), m.__file__, "exec"), m.__dict__)
        caught = _first_failing_pin()
    finally:
        m.__dict__.clear()
        m.__dict__.update(saved)
    assert caught is not None, f"no pin catches: {what}"
