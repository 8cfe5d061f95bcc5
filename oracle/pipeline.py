"""Prefill compression and decode-time periodic recompression composed from the oracle steps.

Test infrastructure only (fp64).  Pages and readings as in ``infokv``,
``selkv`` and ``recas``; the composition follows:

* [InfoKV] Methodology / Technical details: per layer, score every cached
  token with S = alpha * A + (1 - alpha) * Softmax(D * H) and keep the top
  k_l; compression is applied once after prefill, or during decoding every
  1024 generated tokens (Technical details, "e.g. every 1024 tokens").
* [SelKV] Pipeline overview: VATP importance, selection through the GQA
  union, bucket routing, gated merge, attention compensation.

Readings: R17 - under decode-time compression the budget is
floor(rho * t) of the current total length t (prompt + generated), applied
when the generated count is a multiple of the period; R18 - W = w = 32
where a workload does not state them.
"""
from __future__ import annotations

import numpy as np

from . import infokv as ik
from . import recas
from . import selkv

__all__ = ["prefill_scores", "prefill_select", "DecodeCompressionReplay"]


def prefill_scores(logits, hidden, Qw, K, V=None, *, G: int, alpha: float = 0.9,
                   tau: float = 1.0, topk: int = 256, mode: str = "infokv",
                   H=None, D=None):
    """Signals and scores of every (layer, KV head) row after prefill.

    logits [n][V] (or precomputed H [n]); hidden [L][n][Dh] whose last layer is
    h^(L) (or precomputed D [L][n]); Qw [L][Hq][W][d]; K, V [L][Hkv][n][d].
    mode: "infokv" (S = alpha A + (1 - alpha) P), "vatp" (S = A * ||v||) or
    "attn" (S = A).  Returns a dict with H, D, E, P, Ebar, A and S.
    """
    K = np.asarray(K, np.float64)
    L, Hkv, n, _ = K.shape
    out = {}
    if mode == "infokv":
        if H is None:
            H = ik.topk_entropy(logits, topk)
        if D is None:
            hL = np.asarray(hidden[L - 1], np.float64)
            D = np.stack([ik.repr_change(hidden[l], hL, tau) for l in range(L)])
        E, P, Ebar = ik.entropy_scores(D, np.asarray(H)[None, :])
        out.update(H=np.asarray(H), D=D, E=E, P=P, Ebar=Ebar)
    A = np.zeros((L, Hkv, n))
    for l in range(L):
        for g in range(Hkv):
            A[l, g] = ik.window_attention(np.asarray(Qw[l, g * G:(g + 1) * G], np.float64), K[l, g])
    out["A"] = A
    if mode == "infokv":
        out["S"] = ik.combine(A, out["P"][:, None, :], alpha)
    elif mode == "vatp":
        out["S"] = ik.vatp(A, V)
    else:
        out["S"] = A
    return out


def prefill_select(S, budgets, w: int, sel_mode: str):
    """Kept index lists [L][Hkv] -> array of ascending positions.

    sel_mode "per_kv_head" ranks each KV head by its own S; "gqa_union" ranks
    by max over KV heads and every head of the layer keeps the same set.
    """
    S = np.asarray(S, np.float64)
    L, Hkv, _ = S.shape
    idx = [[None] * Hkv for _ in range(L)]
    for l in range(L):
        if sel_mode == "gqa_union":
            keep = ik.select_topk(ik.union_max(S[l]), int(budgets[l]), w)
            for g in range(Hkv):
                idx[l][g] = keep
        else:
            for g in range(Hkv):
                idx[l][g] = ik.select_topk(S[l, g], int(budgets[l]), w)
    return idx


class DecodeCompressionReplay:
    """One sequence of the decode-time periodic compression workload, replayed in fp64.

    State per (layer, KV head): cached K, V, original positions, and the
    per-token signals H and D^(l) carried along so the token can be rescored
    at the next compression.  A full shadow history is kept for the RECAS
    probe.
    """

    def __init__(self, K, V, H, D, *, n_q_heads: int, W: int, w: int, rho: float,
                 alpha: float, tau: float, period: int, sel_mode: str = "per_kv_head"):
        K = np.asarray(K, np.float64)
        L, Hkv, n, d = K.shape
        self.L, self.Hkv, self.d = L, Hkv, d
        self.G = n_q_heads // Hkv
        self.W, self.w, self.rho = W, w, rho
        self.alpha, self.tau, self.period = alpha, tau, period
        self.sel_mode = sel_mode
        self.n_prompt = n
        self.t = n
        self.generated = 0
        V = np.asarray(V, np.float64)
        H = np.asarray(H, np.float64)
        D = np.asarray(D, np.float64)
        self.K = [[K[l, g].copy() for g in range(Hkv)] for l in range(L)]
        self.V = [[V[l, g].copy() for g in range(Hkv)] for l in range(L)]
        self.pos = [[np.arange(n) for _ in range(Hkv)] for _ in range(L)]
        self.H = [[H.copy() for _ in range(Hkv)] for _ in range(L)]
        self.D = [[D[l].copy() for _ in range(Hkv)] for l in range(L)]
        self.U = [[np.zeros(n) for _ in range(Hkv)] for _ in range(L)]   # RECAS attention history
        self.Kfull = [[K[l, g].copy() for g in range(Hkv)] for l in range(L)]
        self.Vfull = [[V[l, g].copy() for g in range(Hkv)] for l in range(L)]
        self.qring = []          # last W generated queries: list of ([L][Hq][d], position)
        self.kept_history = []   # kept positions after each compression

    def step(self, q, k, v, logits_row, hidden, topk: int = 256, probe: bool = False, sparse=None):
        """Append one generated token and attend with its query.

        q [L][Hq][d]; k, v [L][Hkv][d]; logits_row [V]; hidden [L][Dh].
        sparse = (kappa, a_tr, b_hi): RECAS dynamic sparse decode (recas.sparse_decode_step)
        instead of attention over the whole retained row; each row's attention history
        travels with its tokens.
        Returns o [L][Hq][d] and, when probe is set, the RECAS probe of every
        (layer, query head); with sparse, self.active[(l, g)] holds the active positions.
        """
        L, Hkv, G = self.L, self.Hkv, self.G
        q = np.asarray(q, np.float64)
        k = np.asarray(k, np.float64)
        v = np.asarray(v, np.float64)
        h_new = float(ik.topk_entropy(np.asarray(logits_row, np.float64), topk))
        hid = np.asarray(hidden, np.float64)
        d_new = ik.repr_change(hid, hid[L - 1][None, :], self.tau)
        p = self.t
        for l in range(L):
            for g in range(Hkv):
                self.K[l][g] = np.vstack([self.K[l][g], k[l, g][None]])
                self.V[l][g] = np.vstack([self.V[l][g], v[l, g][None]])
                self.pos[l][g] = np.append(self.pos[l][g], p)
                self.H[l][g] = np.append(self.H[l][g], h_new)
                self.D[l][g] = np.append(self.D[l][g], d_new[l])
                self.U[l][g] = np.append(self.U[l][g], 0.0)
                self.Kfull[l][g] = np.vstack([self.Kfull[l][g], k[l, g][None]])
                self.Vfull[l][g] = np.vstack([self.Vfull[l][g], v[l, g][None]])
        self.t += 1
        self.generated += 1
        self.qring.append((q, p))
        if len(self.qring) > self.W:
            self.qring.pop(0)
        o = np.zeros_like(q)
        probes = {} if probe else None
        self.active = {}
        for l in range(L):
            for g in range(Hkv):
                qg = q[l, g * G:(g + 1) * G]
                if sparse is not None:
                    cnt = recas.cached_steps(self.pos[l][g], self.t, self.n_prompt)
                    og, act, self.U[l][g], _ = recas.sparse_decode_step(qg, self.K[l][g], self.V[l][g], self.U[l][g],
                                                                       cnt, *sparse)
                    o[l, g * G:(g + 1) * G] = og
                    self.active[(l, g)] = act
                else:
                    o[l, g * G:(g + 1) * G] = selkv.decode_attention(qg, self.K[l][g], self.V[l][g])
                if probe:
                    mask = np.zeros(self.t, dtype=bool)
                    mask[self.pos[l][g]] = True
                    probes[(l, g)] = recas.dropped_mass_probe(qg, self.Kfull[l][g], self.Vfull[l][g], mask)
        return o, probes

    def due(self) -> bool:
        return self.generated > 0 and self.generated % self.period == 0

    def scores(self):
        """S and A of every (layer, KV head) row's cached tokens, as a compression scores them:
        window attention with the last W generated queries, Softmax(D * H), the InfoKV mix."""
        L, Hkv, G = self.L, self.Hkv, self.G
        qs = np.stack([qq for qq, _ in self.qring], axis=2)       # [L][Hq][W][d]
        qpos = np.array([pp for _, pp in self.qring])
        out = {}
        for l in range(L):
            for g in range(Hkv):
                A = ik.window_attention(qs[l, g * G:(g + 1) * G], self.K[l][g], qpos=qpos,
                                        kpos=self.pos[l][g])
                _, P, _ = ik.entropy_scores(self.D[l][g], self.H[l][g])
                out[(l, g)] = (ik.combine(A, P, self.alpha), A)
        return out

    def recas_needs(self, scores, eps: float, cals):
        """[RECAS] 2.B controller: every row's need, from floor(rho t), with the calibrators
        cals[l] of this sequence's layers (recas.controller_need)."""
        k0 = int(np.floor(self.rho * self.t))
        n = self.K[0][0].shape[0]
        k0 = min(n, max(min(self.w, n), k0))
        needs = {}
        for l in range(self.L):
            if self.sel_mode == "gqa_union":
                U = ik.union_max(np.stack([scores[(l, g)][0] for g in range(self.Hkv)]))
            for g in range(self.Hkv):
                S, A = scores[(l, g)]
                needs[(l, g)] = recas.controller_need(U if self.sel_mode == "gqa_union" else S, A, self.w, k0,
                                                      cals[l].c, cals[l].q, eps)
        return needs

    def recompress(self, budget=None, scores=None):
        """O12  rescore the cached tokens with the last W generated queries and keep floor(rho * t)
        (or `budget` rows, e.g. the RECAS controller's).  The predictor x of every row (share of
        its window attention on the dropped tokens) is kept in self.x.

        Returns {(l, g): (S of the cached rows, their positions before the compression)}.
        """
        L, Hkv = self.L, self.Hkv
        k = int(np.floor(self.rho * self.t)) if budget is None else int(budget)
        if scores is None:
            scores = self.scores()
        kept_all = []
        before = {key: self.pos[key[0]][key[1]].copy() for key in scores}
        self.x = {}
        for l in range(L):
            if self.sel_mode == "gqa_union":
                shared = ik.select_topk(ik.union_max(np.stack([scores[(l, g)][0] for g in range(Hkv)])),
                                        k, self.w)
            for g in range(Hkv):
                S, A = scores[(l, g)]
                keep = shared if self.sel_mode == "gqa_union" else ik.select_topk(S, k, self.w)
                self.x[(l, g)] = recas.dropped_share(A, keep)
                self.K[l][g] = self.K[l][g][keep]
                self.V[l][g] = self.V[l][g][keep]
                self.pos[l][g] = self.pos[l][g][keep]
                self.H[l][g] = self.H[l][g][keep]
                self.D[l][g] = self.D[l][g][keep]
                self.U[l][g] = self.U[l][g][keep]
                kept_all.append(self.pos[l][g].copy())
        self.kept_history.append(kept_all)
        return {key: (scores[key][0], before[key]) for key in scores}
