"""libkvc: B200-native KV-cache scoring, selection, compaction, merging and
compressed decode attention for long-context decoding.

The compute lives in ``_lib/libkvc.so`` (hand-written sm_100a kernels behind
the C ABI of ``include/kvc.h``).  ``binding`` marshals torch tensors into that
ABI; ``pipeline`` strings the calls together for the prefill and
decode-time workloads; ``synth`` draws the seeded synthetic inputs.
"""
from .binding import (  # noqa: F401
    KvcError, kvc_append, kvc_check_status, kvc_compact, kvc_decode_attn, kvc_decode_attn_noalloc,
    kvc_launch_count, kvc_lmhead_entropy, kvc_merge, kvc_recas_calibrate, kvc_recas_control,
    kvc_recompress, kvc_rope_reposition, kvc_score, kvc_select, kvc_sparse_decode, kvc_version, lib,
    lib_path, model,
)

__all__ = ["KvcError", "kvc_append", "kvc_check_status", "kvc_compact", "kvc_decode_attn",
           "kvc_decode_attn_noalloc", "kvc_launch_count", "kvc_lmhead_entropy", "kvc_merge",
           "kvc_recas_calibrate", "kvc_recas_control", "kvc_recompress", "kvc_rope_reposition", "kvc_score",
           "kvc_select", "kvc_sparse_decode", "kvc_version", "lib", "lib_path", "model"]
