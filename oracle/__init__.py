"""CPU oracle for the KV-cache compression path: plain, slow, fp64.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this package; only
the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA path: inputs arrive as numpy arrays (bf16 values decoded exactly to
float64 by the caller) and every step below is written out from the pages.

The three pages it restates (cited by title and section throughout):

* [InfoKV] "긴 추론을 위한 정보 인지형 KV 캐시 압축(InfoKV)" - aitrends.kr
  article on information-aware KV-cache compression for long reasoning.
  Sections used: Key contributions, Methodology (방법론), Technical details
  (기술 상세), Glossary (용어 해설).
* [SelKV] "SelKV: Selective KV Cache Merging with Per-Token Merge-or-Drop and
  Attention Compensation" - gist.science explainer.  Sections used:
  1 Problem definition, 2 Methodology / Core components (soft cosine gate,
  attention compensation), Pipeline overview.
* [RECAS] "기술 요약: 긴 문맥 LLM을 위한 추론 인지적 오차 경계 KV-캐시 압축 및
  희소 어텐션" - gist.science technical summary (reasoning-aware error-bounded
  cache compression).  Section used: 2.B error-bounded adaptive compression.

Modules:
  infokv     - O1 top-k entropy, O2 representation change, O3 entropy score,
               O4 window attention, O5 combination, O6 budgets, O7 selection,
               O8 compaction
  selkv      - O9 routing / soft-cosine-gated merge / attention ratio R,
               O10 decode attention with the alpha_c * log R logit bias
  recas      - O11 dropped attention mass and the 2 * V_max * delta bound
  pipeline   - prefill compression and decode-time periodic recompression
               (O12) composed from the steps above
"""
from . import infokv, selkv, recas, pipeline  # noqa: F401
