"""Seeded synthetic inputs for the KV-cache compression path.

This module only draws random numbers and arranges them into the shapes of
the workloads (Llama-3.2-3B, Llama-3.1-8B and DeepSeek-R1-Distill-Qwen-7B
shaped caches, logits rows and hidden states).  It holds none of the
method's arithmetic: no scores, no selection, no attention.  Both the CUDA
path and the CPU oracle are fed from the tensors it returns.

Every draw comes from a ``torch.Generator`` seeded from the configuration
index and a stream tag, so a given (config, device) pair always yields the
same bits.

Distributions (one per workload family):

* keys, values and window queries ~ N(0, 1); the key of token 0 is scaled
  by 4 (an attention sink);
* final-layer logits row i ~ N(0, sigma_i^2) with sigma_i ~ U(0.5, 4); in the
  bf16 workloads 5 % of rows (Bernoulli per row) get +12 added to one logit
  at a uniformly drawn vocabulary index;
* LM-head inputs: x_i = sigma_i * N(0, 1)^Dh with sigma_i ~ U(0.5, 4) and an
  output projection W ~ N(0, 1 / Dh), so the logits W x_i have the per-row
  spread of the logits rows above (without the dominant-logit rows);
* hidden states: h^(L) ~ N(0, 1) and, for every earlier layer l,
  h^(l) = c * h^(L) + sqrt(1 - c^2) * N(0, 1) with c ~ U(0, 1) drawn per
  (layer, token); the last stored layer is h^(L) itself;
* merge workload: one anchor token per 512-token positional bucket (drawn
  uniformly inside the bucket) whose key is scaled by 3 in every KV head;
  every other token's value is rho * v_anchor + sqrt(1 - rho^2) * N(0, 1)
  with rho ~ U(-0.5, 1), so value cosines to the bucket's anchor span the
  whole gate range.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

# ---------------------------------------------------------------------------
# Workload shapes
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n: int                  # prompt tokens in the cache
    W: int                  # window queries
    w: int                  # recent window always kept
    vocab: int
    hidden: int             # per-layer hidden size
    dtype: torch.dtype      # K/V/Q/logits/hidden storage type
    rho: float              # retention
    sel_mode: str           # "per_kv_head" or "gqa_union"
    score_mode: str         # "infokv" or "vatp"
    alpha: float = 0.9
    tau: float = 1.0
    topk: int = 256
    dominant_rows: bool = True
    bucket: int = 512
    # merge + decode workload
    decode_steps: int = 0
    alpha_c: float = 1.0
    # decode-time periodic compression workload
    batch: int = 1
    gen_tokens: int = 0
    period: int = 1024
    anchors: bool = False
    # rotary base of the keys (Llama-3 shapes 5e5, Qwen-7B 1e6), for re-positioning
    rope_base: float = 500000.0

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def k_uniform(self) -> int:
        return max(min(self.w, self.n), min(self.n, int(math.floor(self.rho * self.n))))

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # tiny InfoKV case that the fp64 oracle finishes in CPU-seconds
    0: Workload("tiny-infokv-fp32", 2, 4, 2, 64, 512, 16, 16, 1000, 256,
                torch.float32, 0.25, "per_kv_head", "infokv", dominant_rows=False),
    # Llama-3.2-3B shaped prefill compression, 16k, 40 % kept, GQA union
    1: Workload("llama3.2-3b-16k-r40", 28, 24, 8, 128, 16384, 32, 32, 128256, 3072,
                torch.bfloat16, 0.40, "gqa_union", "infokv"),
    # Llama-3.1-8B shaped prefill compression, 64k, 20 % kept, per KV head
    2: Workload("llama3.1-8b-64k-r20", 32, 32, 8, 128, 65536, 32, 64, 128256, 4096,
                torch.bfloat16, 0.20, "per_kv_head", "infokv"),
    # SelKV merge + compensated decode at Llama-3.1-8B shape, 100k, 25 % kept
    3: Workload("llama3.1-8b-100k-r25-selkv", 32, 32, 8, 128, 100000, 32, 32, 128256, 4096,
                torch.bfloat16, 0.25, "gqa_union", "vatp", decode_steps=256, anchors=True),
    # decode-time periodic compression at DeepSeek-R1-Distill-Qwen-7B shape
    4: Workload("qwen7b-decode-b8-r12.5", 28, 28, 4, 128, 2048, 32, 32, 152064, 3584,
                torch.bfloat16, 0.125, "per_kv_head", "infokv",
                batch=8, gen_tokens=32768, period=1024, rope_base=1000000.0),
}


def _gen(seed: int, tag: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + tag)
    return g


# ---------------------------------------------------------------------------
# Prefill inputs
# ---------------------------------------------------------------------------


@dataclass
class PrefillInputs:
    wl: Workload
    logits: torch.Tensor            # [n][vocab]
    hidden: torch.Tensor            # [L][n][Dh]; layer L-1 is h^(L)
    Qw: torch.Tensor                # [L][Hq][W][d] window queries (positions n-W .. n-1)
    K: torch.Tensor                 # [L][Hkv][n][d]
    V: torch.Tensor                 # [L][Hkv][n][d]
    anchors: Optional[torch.Tensor] = None   # [ceil(n/bucket)] anchor positions (merge workload)


def gen_logits(rows: int, vocab: int, dtype, seed: int, device, dominant: bool,
               tag: int = 1, chunk: int = 1024, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Logits rows: N(0, sigma_i^2), sigma_i ~ U(0.5, 4); optional +12 on one logit in 5 % of rows."""
    g = _gen(seed, tag, device)
    if out is None:
        out = torch.empty(rows, vocab, dtype=dtype, device=device)
    sig = torch.empty(rows, device=device).uniform_(0.5, 4.0, generator=g)
    dom = torch.rand(rows, device=device, generator=g) < 0.05
    col = torch.randint(0, vocab, (rows,), device=device, generator=g)
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        x = torch.randn(r1 - r0, vocab, device=device, generator=g)
        x.mul_(sig[r0:r1, None])
        if dominant:
            rr = torch.nonzero(dom[r0:r1]).flatten()
            if rr.numel():
                x[rr, col[r0 + rr]] += 12.0
        out[r0:r1].copy_(x.to(dtype))
    return out


def gen_lmhead(n: int, Dh: int, vocab: int, seed: int, device, tag: int = 9, chunk: int = 8192):
    """LM-head input x [n][Dh] = sigma_i * N(0, 1), sigma_i ~ U(0.5, 4), and W [vocab][Dh] ~ N(0, 1/Dh); bf16."""
    g = _gen(seed, tag, device)
    sig = torch.empty(n, device=device).uniform_(0.5, 4.0, generator=g)
    x = torch.empty(n, Dh, dtype=torch.bfloat16, device=device)
    for r0 in range(0, n, chunk):
        r1 = min(n, r0 + chunk)
        x[r0:r1].copy_((torch.randn(r1 - r0, Dh, device=device, generator=g) * sig[r0:r1, None]).to(torch.bfloat16))
    W = torch.empty(vocab, Dh, dtype=torch.bfloat16, device=device)
    for v0 in range(0, vocab, chunk):
        v1 = min(vocab, v0 + chunk)
        W[v0:v1].copy_((torch.randn(v1 - v0, Dh, device=device, generator=g) / math.sqrt(Dh)).to(torch.bfloat16))
    return x, W


def gen_hidden(L: int, n: int, Dh: int, dtype, seed: int, device, tag: int = 2,
               chunk: int = 8192) -> torch.Tensor:
    """[L][n][Dh]: last layer h^(L) ~ N(0,1); layer l < L-1: c*h^(L) + sqrt(1-c^2)*N(0,1)."""
    g = _gen(seed, tag, device)
    out = torch.empty(L, n, Dh, dtype=dtype, device=device)
    c = torch.rand(L, n, device=device, generator=g)
    for t0 in range(0, n, chunk):
        t1 = min(n, t0 + chunk)
        hL = torch.randn(t1 - t0, Dh, device=device, generator=g)
        out[L - 1, t0:t1].copy_(hL.to(dtype))
        for l in range(L - 1):
            cl = c[l, t0:t1, None]
            x = torch.randn(t1 - t0, Dh, device=device, generator=g)
            x.mul_(torch.sqrt(1.0 - cl * cl)).add_(cl * hL)
            out[l, t0:t1].copy_(x.to(dtype))
    return out


def gen_prefill(wl: Workload, seed: int, device="cpu", with_logits: bool = True,
                with_hidden: bool = True) -> PrefillInputs:
    L, Hq, Hkv, d, n, W = wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n, wl.W
    g = _gen(seed, 3, device)
    K = torch.randn(L, Hkv, n, d, device=device, generator=g)
    K[:, :, 0, :] *= 4.0
    V = torch.randn(L, Hkv, n, d, device=device, generator=g)
    Qw = torch.randn(L, Hq, W, d, device=device, generator=g)
    anchors = None
    if wl.anchors:
        nb = (n + wl.bucket - 1) // wl.bucket
        lo = torch.arange(nb, device=device) * wl.bucket
        span = torch.clamp(n - lo, max=wl.bucket)
        anchors = lo + (torch.rand(nb, device=device, generator=g) * span).long()
        anchors = torch.minimum(anchors, lo + span - 1)
        K[:, :, anchors, :] *= 3.0
        rho = torch.empty(L, Hkv, n, 1, device=device).uniform_(-0.5, 1.0, generator=g)
        b_of = torch.arange(n, device=device) // wl.bucket
        va = V[:, :, anchors[b_of], :]
        z = torch.randn(L, Hkv, n, d, device=device, generator=g)
        Vn = rho * va + torch.sqrt(1.0 - rho * rho) * z
        is_anchor = torch.zeros(n, dtype=torch.bool, device=device)
        is_anchor[anchors] = True
        V = torch.where(is_anchor[None, None, :, None], V, Vn)
    dt = wl.dtype
    logits = gen_logits(n, wl.vocab, dt, seed, device, wl.dominant_rows) if with_logits else None
    hidden = gen_hidden(L, n, wl.hidden, dt, seed, device) if with_hidden else None
    return PrefillInputs(wl, logits, hidden, Qw.to(dt), K.to(dt), V.to(dt), anchors)


# ---------------------------------------------------------------------------
# Decode-step inputs
# ---------------------------------------------------------------------------


def gen_decode_queries(wl: Workload, seed: int, step: int, device="cpu") -> torch.Tensor:
    """Decode query for one step: [B][L][Hq][d] ~ N(0, 1)."""
    g = _gen(seed, 100_000 + step, device)
    q = torch.randn(wl.batch, wl.n_layers, wl.n_q_heads, wl.head_dim, device=device, generator=g)
    return q.to(wl.dtype)


def gen_decode_kv(wl: Workload, seed: int, step: int, device="cpu"):
    """Key and value rows appended at one decode step: two [B][L][Hkv][d] ~ N(0, 1)."""
    g = _gen(seed, 200_000 + step, device)
    shape = (wl.batch, wl.n_layers, wl.n_kv_heads, wl.head_dim)
    k = torch.randn(*shape, device=device, generator=g)
    v = torch.randn(*shape, device=device, generator=g)
    return k.to(wl.dtype), v.to(wl.dtype)


def gen_decode_signals(wl: Workload, seed: int, step: int, device="cpu"):
    """Per-step logits rows [B][vocab] and hidden states [B][L][Dh] of the generated token."""
    logits = gen_logits(wl.batch, wl.vocab, wl.dtype, seed, device, wl.dominant_rows,
                        tag=300_000 + step)
    g = _gen(seed, 400_000 + step, device)
    L, Dh = wl.n_layers, wl.hidden
    hL = torch.randn(wl.batch, Dh, device=device, generator=g)
    c = torch.rand(wl.batch, L, 1, device=device, generator=g)
    x = torch.randn(wl.batch, L, Dh, device=device, generator=g)
    h = c * hL[:, None, :] + torch.sqrt(1.0 - c * c) * x
    h[:, L - 1, :] = hL
    return logits, h.to(wl.dtype)


def gen_prompt_batch(wl: Workload, seed: int, device="cpu"):
    """Prompt state for the decode-time workload, one independent prompt per sequence.

    Returns K, V [B][L][Hkv][n][d], prompt logits [B][n][vocab] and prompt
    hidden states [B][L][n][Dh].
    """
    Ks, Vs, Ls, Hs = [], [], [], []
    for b in range(wl.batch):
        p = gen_prefill(wl.scaled(batch=1), seed * 131 + b, device)
        Ks.append(p.K)
        Vs.append(p.V)
        Ls.append(p.logits)
        Hs.append(p.hidden)
    return torch.stack(Ks), torch.stack(Vs), torch.stack(Ls), torch.stack(Hs)
