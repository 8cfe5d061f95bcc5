"""Host orchestration of the six libkvc calls for the two workloads.

* ``PrefillCompressor``: one-shot compression after prefill - kvc_score ->
  kvc_select -> kvc_compact (optionally kvc_merge), all buffers and
  workspaces allocated once up front so ``run()`` only enqueues kernels.
* ``DecodeTimeCompressor``: decode-time periodic compression of a batch of
  sequences - every step appends one token (K, V and its H / D signals) and
  attends with kvc_decode_attn; every ``period`` generated tokens the batch is
  recompressed with kvc_recompress into a ping-pong buffer.

Nothing here computes on the host: it sizes buffers and launches the calls in
order on the current stream.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import binding as B


class PrefillCompressor:
    def __init__(self, wl, inp, *, budget: str = "uniform", keep_A: bool = False,
                 merge: bool = False, k_cap: Optional[int] = None, device=None):
        self.wl = wl
        self.inp = inp
        dev = device or inp.K.device
        L, Hq, Hkv, d, n = wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n
        self.m = B.model(L, Hq, Hkv, d)
        f32, i32 = torch.float32, torch.int32
        self.mode = B.SCORE_INFOKV if wl.score_mode == "infokv" else B.SCORE_VATP
        self.sel_mode = B.SEL_GQA_UNION if wl.sel_mode == "gqa_union" else B.SEL_PER_KV_HEAD
        self.budget = budget
        self.S = torch.empty(L, Hkv, n, dtype=f32, device=dev)
        self.A = torch.empty(L, Hkv, n, dtype=f32, device=dev) if (keep_A or merge) else None
        infokv = self.mode == B.SCORE_INFOKV
        self.H = torch.empty(n, dtype=f32, device=dev) if infokv else None
        self.D = torch.empty(L, n, dtype=f32, device=dev) if infokv else None
        self.Ebar = torch.empty(L, dtype=f32, device=dev) if infokv else None
        ku = wl.k_uniform
        self.B_total = L * ku
        if k_cap is None:
            k_cap = ku if budget == "uniform" else min(n, 2 * ku)
        self.k_cap = k_cap
        self.k = torch.empty(L, dtype=i32, device=dev)
        self.idx = torch.empty(L, Hkv, k_cap, dtype=i32, device=dev)
        self.Kc = torch.empty(L, Hkv, k_cap, d, dtype=wl.dtype, device=dev)
        self.Vc = torch.empty(L, Hkv, k_cap, d, dtype=wl.dtype, device=dev)
        self.merge = merge
        if merge:
            self.R = torch.empty(L, Hkv, k_cap, dtype=f32, device=dev)
            self.Vm_f32 = None
        self.ws_score = None
        self.ws_select = None

    def score(self, stream=None):
        wl, inp = self.wl, self.inp
        kw = dict(mode=self.mode, n=wl.n, W=wl.W, Qw=inp.Qw, K=inp.K, S=self.S, A=self.A,
                  alpha=wl.alpha, tau=wl.tau, topk=wl.topk, workspace=self.ws_score, stream=stream)
        if self.mode == B.SCORE_INFOKV:
            kw.update(logits=inp.logits, hidden=inp.hidden, H_out=self.H, D_out=self.D, Ebar=self.Ebar)
        else:
            kw.update(V=inp.V)
        self.ws_score = B.kvc_score(self.m, **kw)

    def select(self, stream=None):
        wl = self.wl
        kw = dict(n=wl.n, w=wl.w, S=self.S, k_out=self.k, idx=self.idx, sel_mode=self.sel_mode,
                  workspace=self.ws_select, stream=stream)
        if self.budget == "uniform":
            kw.update(budget_mode=B.BUDGET_UNIFORM, rho=wl.rho)
        else:
            kw.update(budget_mode=B.BUDGET_ADAPTIVE, B_total=self.B_total, Ebar=self.Ebar)
        self.ws_select = B.kvc_select(self.m, **kw)

    def compact(self, stream=None):
        inp = self.inp
        B.kvc_compact(self.m, n=self.wl.n, idx=self.idx, k=self.k, src_K=inp.K, dst_K=self.Kc,
                      src_V=None if self.merge else inp.V, dst_V=None if self.merge else self.Vc,
                      stream=stream)

    def do_merge(self, stream=None, f32_copy: Optional[torch.Tensor] = None):
        B.kvc_merge(self.m, n=self.wl.n, V=self.inp.V, A=self.A, idx=self.idx, k=self.k,
                    dst_V=self.Vc, R=self.R, bucket=self.wl.bucket, dst_V_f32=f32_copy,
                    stream=stream)

    def reposition(self, new0: int = 0, pos_dst=None, stream=None):
        """SelKV step 6: re-embed the compacted keys at positions new0, new0 + 1, ... in place
        (the kept lists in idx are the positions they carry)."""
        B.kvc_rope_reposition(self.m, K=self.Kc, pos=self.idx, k=self.k, base=self.wl.rope_base,
                              new0=new0, pos_dst=pos_dst, stream=stream)

    def run(self, stream=None):
        self.score(stream)
        self.select(stream)
        self.compact(stream)
        if self.merge:
            self.do_merge(stream)


class DecodeAttention:
    """kvc_decode_attn over a [B][L][Hkv][cap][d] cache with preallocated outputs."""

    def __init__(self, m, B_, L, Hq, d, device, probe: bool = False, Hkv: int = 0):
        self.m = m
        self.o = torch.empty(B_, L, Hq, d, dtype=torch.float32, device=device)
        self.ws = {}
        self.probe = probe
        if probe:
            self.delta = torch.empty(B_, L, Hq, dtype=torch.float32, device=device)
            self.err = torch.empty_like(self.delta)
            self.bound = torch.empty_like(self.delta)
            self.vmax = torch.empty(B_, L, Hkv, dtype=torch.float32, device=device)
            self.o_full = torch.empty_like(self.o)
            self.o_kept = torch.empty_like(self.o)

    def __call__(self, q, K, V, lens, max_len, R=None, alpha_c=1.0, stream=None, full=None, lse=None):
        key = full is not None
        kw = dict(q=q, K=K, V=V, lens=lens, max_len=max_len, o=self.o, R=R, alpha_c=alpha_c,
                  lse=lse, stream=stream)
        if full is not None:
            Kf, Vf, lens_f, max_f, bits = full
            kw.update(K_full=Kf, V_full=Vf, lens_full=lens_f, max_len_full=max_f, kept_bits=bits,
                      delta=self.delta, vmax=self.vmax, err=self.err, bound=self.bound,
                      o_full=self.o_full, o_kept=self.o_kept)
        ws = self.ws.get(key)
        need = B.workspace_size(B.OP_DECODE, self.m, B.decode_args(self.m, **kw))
        if ws is None or ws.numel() < need:
            ws = torch.empty(max(need, 1), dtype=torch.uint8, device=self.o.device)
            self.ws[key] = ws
        B.kvc_decode_attn(self.m, workspace=ws, **kw)
        return self.o


class DecodeTimeCompressor:
    """Decode-time periodic compression of a batch of independent sequences.

    Buffers: ping-pong caches K/V [2][B][L][Hkv][cap][d]; per-token side arrays
    pos / H / D [2][B][L][Hkv][cap]; the window-query ring [B][L][Hq][W][d]
    with positions [B][W]; optional full shadow history for the RECAS probe.
    """

    def __init__(self, wl, prompt_K, prompt_V, prompt_H, prompt_D, *, probe: bool = False,
                 recas_eps: Optional[float] = None, recas_alpha: float = 0.1, sparse=None, device=None):
        self.wl = wl
        dev = device or prompt_K.device
        Bn, L, Hq, Hkv, d, W = wl.batch, wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.W
        n0 = wl.n
        self.m = B.model(L, Hq, Hkv, d)
        T = n0 + wl.gen_tokens
        # largest live cache: the compressed length just before a compression
        cap = n0 + wl.period
        j = 1
        while n0 + j * wl.period <= T:
            t = n0 + j * wl.period
            keep = max(min(wl.w, t), math.floor(wl.rho * t))
            cap = max(cap, keep + wl.period)
            j += 1
        self.cap = cap
        dt = wl.dtype
        self.K = torch.zeros(2, Bn, L, Hkv, cap, d, dtype=dt, device=dev)
        self.V = torch.zeros(2, Bn, L, Hkv, cap, d, dtype=dt, device=dev)
        self.pos = torch.zeros(2, Bn, L, Hkv, cap, dtype=torch.int32, device=dev)
        self.Hs = torch.zeros(2, Bn, L, Hkv, cap, dtype=torch.float32, device=dev)
        self.Ds = torch.zeros(2, Bn, L, Hkv, cap, dtype=torch.float32, device=dev)
        # RECAS dynamic sparse decode: (kappa, a_tr, b_hi) and the attention history of
        # every cached token, a side array that travels with it like H and D
        self.sparse = sparse
        self.U = torch.zeros(2, Bn, L, Hkv, cap, dtype=torch.float32, device=dev) if sparse else None
        self.ws_sp = None
        self.cur = 0
        self.len = n0
        self.t = n0
        self.generated = 0
        self.K[0, :, :, :, :n0] = prompt_K
        self.V[0, :, :, :, :n0] = prompt_V
        self.pos[0, :, :, :, :n0] = torch.arange(n0, dtype=torch.int32, device=dev)
        self.Hs[0, :, :, :, :n0] = prompt_H[:, None, None, :]
        self.Ds[0, :, :, :, :n0] = prompt_D[:, :, None, :]
        self.Qring = torch.zeros(Bn, L, Hq, W, d, dtype=dt, device=dev)
        self.qpos = torch.zeros(Bn, W, dtype=torch.int32, device=dev)
        # beside every window query, the log-sum-exp its decode step found over the cache:
        # a recompression whose whole window was decoded (attend() or attend_sparse()) reads
        # these row statistics instead of recomputing them (kvc_recompress's win_lse)
        self.lse_ring = torch.zeros(Bn, L, Hq, W, dtype=torch.float32, device=dev)
        self.lse_streak = 0          # consecutive appended steps a decode step has covered
        self._lse_pending = False    # the last appended step has not been decoded yet
        self.lens = torch.full((Bn, L), n0, dtype=torch.int32, device=dev)
        self.attn = DecodeAttention(self.m, Bn, L, Hq, d, dev, probe=probe, Hkv=Hkv)
        self.probe = probe
        if probe:
            self.Kf = torch.zeros(Bn, L, Hkv, T, d, dtype=dt, device=dev)
            self.Vf = torch.zeros(Bn, L, Hkv, T, d, dtype=dt, device=dev)
            self.Kf[:, :, :, :n0] = prompt_K
            self.Vf[:, :, :, :n0] = prompt_V
            self.nwords = (T + 31) // 32
            self.bits = torch.zeros(Bn, L, Hkv, self.nwords, dtype=torch.int32, device=dev)
            self._set_bits_prefix(n0)
            self.lens_full = torch.full((Bn, L), n0, dtype=torch.int32, device=dev)
        # RECAS adaptive budget: calibration state per (sequence, layer), the predictor of
        # every row's current kept set (nothing dropped yet: 0), the upper bound per row
        self.recas_eps = recas_eps
        self.recas_alpha = recas_alpha
        if recas_eps is not None:
            if not probe:
                raise ValueError("the RECAS budget is calibrated at probe steps: probe=True")
            self.recas_state = B.recas_state(Bn, L, dev)
            self.recas_x = torch.zeros(Bn, L, Hkv, dtype=torch.float32, device=dev)
            self.delta_hat = torch.zeros(Bn, L, Hkv, dtype=torch.float32, device=dev)
            self.delta_bar = torch.full((Bn, L, Hkv), float("inf"), dtype=torch.float32, device=dev)
        # one recompression workspace, sized for the largest cache the run can reach
        self.ws_re = None
        self.ws_re = torch.empty(max(1, self._recompress_ws_bytes()), dtype=torch.uint8, device=dev)

    def _set_bits_prefix(self, n):
        full_words = n // 32
        self.bits.zero_()
        if full_words:
            self.bits[..., :full_words] = -1
        if n % 32:
            self.bits[..., full_words] = (1 << (n % 32)) - 1 if n % 32 < 31 else 0x7fffffff

    def append(self, k, v, H_new, D_new, q, stream=None):
        """Append one generated token per sequence (k, v [B][L][Hkv][d]; H_new [B]; D_new [B][L]):
        the cache row, its position / H / D, its kept bit and its query in the window ring,
        and its row of the full shadow history when the probe is on (one kvc_append)."""
        c = self.cur
        full = dict(K2=self.Kf, V2=self.Vf, lens2=self.lens_full) if self.probe else {}
        B.kvc_append(self.m, k=k, v=v, K=self.K[c], V=self.V[c], lens=self.lens, pos=self.t,
                     side_pos=self.pos[c], side_H=self.Hs[c], side_D=self.Ds[c],
                     side_U=self.U[c] if self.sparse else None, H_new=H_new, D_new=D_new,
                     kept_bits=self.bits if self.probe else None, q=q, Qring=self.Qring, qpos=self.qpos,
                     slot=self.generated % self.wl.W, stream=stream, **full)
        if self._lse_pending:
            self.lse_streak = 0
        self._lse_pending = True
        self.len += 1
        self.t += 1
        self.generated += 1

    def attend(self, q, stream=None, probe: bool = False):
        c = self.cur
        full = None
        if probe and self.probe:
            full = (self.Kf, self.Vf, self.lens_full, self.t, self.bits)
        return self.attn(q, self.K[c], self.V[c], self.lens, self.len, stream=stream, full=full,
                         lse=self._lse_slot())

    def _lse_slot(self):
        """The window ring's slot of the last appended step, for this decode step's log-sum-exp
        over the cache (both decode forms write it); counts the step as decoded."""
        if self.generated == 0:
            return None
        if self._lse_pending:
            self.lse_streak += 1
            self._lse_pending = False
        return self.lse_ring[:, :, :, (self.generated - 1) % self.wl.W]

    def attend_sparse(self, q, stream=None):
        """RECAS dynamic sparse decode over the retained caches (kvc_sparse_decode): the top
        ceil(kappa n) tokens of each row by a_tr tr + b_hi hi attend; every row's attention
        history is updated."""
        c = self.cur
        kappa, a_tr, b_hi = self.sparse
        self.ws_sp = B.kvc_sparse_decode(self.m, q=q, K=self.K[c], V=self.V[c], lens=self.lens, max_len=self.cap,
                                         pos=self.pos[c], acc=self.U[c], t_cur=self.t, n_prompt=self.wl.n,
                                         kappa=kappa, a_tr=a_tr, b_hi=b_hi, o=self.attn.o,
                                         lse=self._lse_slot(), workspace=self.ws_sp, stream=stream)
        return self.attn.o

    def due(self) -> bool:
        return self.generated > 0 and self.generated % self.wl.period == 0

    def _recompress_kw(self, len_, t):
        wl = self.wl
        c, n = self.cur, 1 - self.cur
        kw = dict(len_=len_, t=t, rho=wl.rho, w=wl.w, W=wl.W, Qring=self.Qring, qpos=self.qpos,
                  K=self.K[c], V=self.V[c], pos=self.pos[c], H=self.Hs[c], D=self.Ds[c], K_dst=self.K[n],
                  V_dst=self.V[n], pos_dst=self.pos[n], H_dst=self.Hs[n], D_dst=self.Ds[n],
                  alpha=wl.alpha, tau=wl.tau,
                  sel_mode=B.SEL_GQA_UNION if wl.sel_mode == "gqa_union" else B.SEL_PER_KV_HEAD,
                  k_out=self.lens, kept_bits_dst=self.bits if self.probe else None,
                  U=self.U[c] if self.sparse else None, U_dst=self.U[n] if self.sparse else None,
                  win_lse=self.lse_ring if self.lse_streak >= wl.W else None)
        if self.recas_eps is not None:
            # the budget may grow up to the cache length, but leaves room for a period of appends
            kw.update(recas_state=self.recas_state, recas_eps=self.recas_eps, recas_x=self.recas_x,
                      recas_k_max=self.cap - wl.period)
        return kw

    def _recompress_ws_bytes(self):
        wl = self.wl
        T = wl.n + wl.gen_tokens
        a = B.recompress_args(self.m, **self._recompress_kw(self.cap, max(T, self.cap)))
        return B.workspace_size(B.OP_RECOMPRESS, self.m, a)

    def calibrate(self, stream=None):
        """RECAS calibration after a probe step (attend(..., probe=True)): the exact dropped
        mass of every query head updates the estimate and the residual quantile."""
        B.kvc_recas_calibrate(self.m, delta=self.attn.delta, x=self.recas_x, state=self.recas_state,
                              alpha=self.recas_alpha, delta_hat=self.delta_hat, delta_bar=self.delta_bar,
                              stream=stream)

    def recompress(self, stream=None):
        """kvc_recompress into the other ping-pong buffer; the new row counts land in the
        decode lengths (k_out) and, with the probe, the kept-position bits are rebuilt.
        With the RECAS budget the kept count is decided on the device and read back here
        (one small device-to-host copy per period)."""
        n = 1 - self.cur
        self.ws_re, keep = B.kvc_recompress(self.m, workspace=self.ws_re, stream=stream,
                                            **self._recompress_kw(self.len, self.t))
        if keep < 0:
            keep = int(self.lens[0, 0].item())
        self.cur = n
        self.len = keep
        self.lse_streak = 0          # the ring's statistics describe the cache before this call
        return keep
