"""The C-ABI library loads, exports every function include/kvc.h declares, and
rejects bad arguments on the host before launching anything (no GPU needed)."""
import ctypes as C
import os
import re

import pytest

from long_context_kv_obs_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:kvc_status|const char\s*\*|int|uint64_t)\s+(kvc_\w+)\s*\(", src, re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = B.lib()
    decl = declared_functions()
    assert len(decl) >= 10
    for name in decl:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(B.EXPORTED) <= set(decl)
    assert lib.kvc_version() == 100


def _model(d=128):
    return B.model(4, 8, 2, d)


def _status(call):
    return call


def test_score_validation_errors():
    lib = B.lib()
    m = _model()
    a = B.ScoreArgs()
    n = C.c_size_t(0)
    # missing everything
    assert lib.kvc_workspace_size(B.OP_SCORE, C.byref(m), C.byref(a), C.byref(n)) == 1
    a.n, a.W, a.mode, a.alpha = 100, 8, B.SCORE_ATTN, 0.9
    a.Qw, a.S = 0x10000, 0x20000
    a.K = B.KV(0x30000, B.KVC_BF16, 0, 2 * 100 * 128, 100 * 128, 128)
    assert lib.kvc_workspace_size(B.OP_SCORE, C.byref(m), C.byref(a), C.byref(n)) == 0
    assert n.value > 0
    a.W = 101                                      # W > n
    assert lib.kvc_workspace_size(B.OP_SCORE, C.byref(m), C.byref(a), C.byref(n)) == 1
    a.W = 8
    a.K = B.KV(0x30008, B.KVC_BF16, 0, 2 * 100 * 128, 100 * 128, 128)   # misaligned
    assert lib.kvc_workspace_size(B.OP_SCORE, C.byref(m), C.byref(a), C.byref(n)) == 1
    assert b"aligned" in lib.kvc_last_error()
    a.K = B.KV(0x30000, B.KVC_BF16, 0, 2 * 100 * 128, 100 * 128, 100)   # row stride 200 B
    assert lib.kvc_workspace_size(B.OP_SCORE, C.byref(m), C.byref(a), C.byref(n)) == 1
    m96 = _model(96)
    a.K = B.KV(0x30000, B.KVC_BF16, 0, 2 * 100 * 128, 100 * 128, 128)
    assert lib.kvc_workspace_size(B.OP_SCORE, C.byref(m96), C.byref(a), C.byref(n)) == 2
    a.mode = B.SCORE_INFOKV                        # neither logits nor H_in
    assert lib.kvc_workspace_size(B.OP_SCORE, C.byref(m), C.byref(a), C.byref(n)) == 1
    # too small a workspace is refused before any launch
    a.mode = B.SCORE_ATTN
    assert lib.kvc_score(C.byref(m), C.byref(a), None, 0, None) == 3


def test_select_compact_merge_decode_validation():
    lib = B.lib()
    m = _model()
    s = B.SelectArgs()
    s.n, s.w, s.S, s.k_out, s.idx, s.k_cap = 1000, 16, 0x1000, 0x2000, 0x3000, 100
    s.budget_mode, s.rho = B.BUDGET_UNIFORM, 0.25        # k = 250 > k_cap
    n = C.c_size_t(0)
    assert lib.kvc_workspace_size(B.OP_SELECT, C.byref(m), C.byref(s), C.byref(n)) == 1
    s.k_cap = 250
    assert lib.kvc_workspace_size(B.OP_SELECT, C.byref(m), C.byref(s), C.byref(n)) == 0
    assert n.value >= 2 * 4 * 1000 * 4
    s.budget_mode, s.B_total, s.Ebar = B.BUDGET_ADAPTIVE, 10, 0x4000   # B below L*w
    assert lib.kvc_workspace_size(B.OP_SELECT, C.byref(m), C.byref(s), C.byref(n)) == 1

    c = B.CompactArgs()
    c.n, c.idx, c.k, c.k_cap = 100, 0x1000, 0x2000, 10
    kvt = B.KV(0x10000, B.KVC_BF16, 0, 2 * 100 * 128, 100 * 128, 128)
    c.src_K, c.dst_K = kvt, kvt                           # aliasing
    assert lib.kvc_compact(C.byref(m), C.byref(c), None) == 1
    assert b"alias" in lib.kvc_last_error()
    c.dst_K = B.KV(0x90000, B.KVC_F32, 0, 2 * 10 * 128, 10 * 128, 128)   # dtype mismatch
    assert lib.kvc_compact(C.byref(m), C.byref(c), None) == 1

    g = B.MergeArgs()
    g.n, g.bucket, g.k_cap = 100, 0, 10
    assert lib.kvc_merge(C.byref(m), C.byref(g), None, 0, None) == 2

    d = B.DecodeArgs()
    assert lib.kvc_workspace_size(B.OP_DECODE, C.byref(m), C.byref(d), C.byref(n)) == 1
    d.batch, d.q, d.len, d.o, d.max_len = 1, 0x1000, 0x2000, 0x3000, 64
    d.K = B.KV(0x10000, B.KVC_BF16, 0, 2 * 64 * 128, 64 * 128, 128)
    d.V = B.KV(0x50000, B.KVC_BF16, 0, 2 * 64 * 128, 64 * 128, 128)
    assert lib.kvc_workspace_size(B.OP_DECODE, C.byref(m), C.byref(d), C.byref(n)) == 0
    mg = B.model(2, 36, 2, 128)                           # 18 query heads per KV head
    assert lib.kvc_workspace_size(B.OP_DECODE, C.byref(mg), C.byref(d), C.byref(n)) == 2


def test_rope_reposition_validation():
    lib = B.lib()
    before = B.kvc_launch_count()
    m = _model()
    r = B.RopeArgs()
    r.K = B.KV(0x10000, B.KVC_BF16, 0, 2 * 64 * 128, 64 * 128, 128)
    r.pos, r.pos_s_row, r.k, r.k_cap, r.new0, r.base = 0x2000, 64, 0x3000, 64, 0, 10000.0
    assert lib.kvc_rope_reposition(None, C.byref(r), None) == 1
    r.base = 1.0                                          # base must exceed 1
    assert lib.kvc_rope_reposition(C.byref(m), C.byref(r), None) == 1
    assert b"base" in lib.kvc_last_error()
    r.base, r.pos_s_row = 10000.0, 32                     # rows of pos shorter than k_cap
    assert lib.kvc_rope_reposition(C.byref(m), C.byref(r), None) == 1
    r.pos_s_row, r.new0 = 64, 2 ** 31 - 10                # new positions past int32
    assert lib.kvc_rope_reposition(C.byref(m), C.byref(r), None) == 1
    r.new0, r.pos = 0, None
    assert lib.kvc_rope_reposition(C.byref(m), C.byref(r), None) == 1
    r.pos = 0x2000
    r.K_dst = B.KV(0x90000, B.KVC_F32, 0, 2 * 64 * 128, 64 * 128, 128)   # dtype mismatch
    assert lib.kvc_rope_reposition(C.byref(m), C.byref(r), None) == 1
    r.K_dst = B.KV(0x90008, B.KVC_BF16, 0, 2 * 64 * 128, 64 * 128, 128)  # misaligned
    assert lib.kvc_rope_reposition(C.byref(m), C.byref(r), None) == 1
    assert B.kvc_launch_count() == before


def test_bad_model_rejected():
    lib = B.lib()
    a = B.DecodeArgs()
    n = C.c_size_t(0)
    assert lib.kvc_workspace_size(B.OP_DECODE, None, C.byref(a), C.byref(n)) == 1
    m = B.model(2, 6, 4, 128)                             # Hq not a multiple of Hkv
    assert lib.kvc_workspace_size(B.OP_DECODE, C.byref(m), C.byref(a), C.byref(n)) == 1
    assert lib.kvc_workspace_size(99, C.byref(m), C.byref(a), C.byref(n)) == 1


def test_binding_refuses_host_tensors():
    import torch
    m = _model()
    with pytest.raises(ValueError):
        B.kvc_compact(m, n=4, idx=torch.zeros(4, 2, 2, dtype=torch.int32),
                      k=torch.zeros(4, dtype=torch.int32),
                      src_K=torch.zeros(4, 2, 4, 128, dtype=torch.bfloat16),
                      dst_K=torch.zeros(4, 2, 2, 128, dtype=torch.bfloat16))


def test_rejected_calls_launch_nothing():
    lib = B.lib()
    before = B.kvc_launch_count()
    m = _model()
    a = B.ScoreArgs()
    a.n, a.W, a.mode, a.alpha = 100, 8, B.SCORE_ATTN, 0.9
    a.Qw, a.S = 0x10000, 0x20000
    a.K = B.KV(0x30000, B.KVC_BF16, 0, 2 * 100 * 128, 100 * 128, 128)
    assert lib.kvc_score(C.byref(m), C.byref(a), None, 0, None) == 3     # no workspace
    a.W = 101
    assert lib.kvc_score(C.byref(m), C.byref(a), None, 0, None) == 1     # W > n
    assert B.kvc_launch_count() == before


def test_bench_traffic_record_matches_current_sources():
    """profiles/ holds the entropy kernel's ncu DRAM bytes per row with a hash of its
    sources; bench.py reports roofline traffic only while the hash matches."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    t = bench.profiled_traffic("entropy", 1000)
    assert t is None or 1000 * 128256 * 2 <= t <= 1.3 * 1000 * 128256 * 2
    assert bench.profiled_traffic("no_such_kernel", 1) is None


def test_append_and_recas_validation():
    """kvc_append, kvc_recas_calibrate and kvc_recas_control reject bad arguments before
    anything is launched (fake device addresses: nothing is dereferenced)."""
    lib = B.lib()
    before = B.kvc_launch_count()
    m = _model()
    a = B.AppendArgs()
    assert lib.kvc_append(C.byref(m), C.byref(a), None) == 1                    # everything missing
    a.batch, a.cap, a.k, a.v, a.len, a.pos = 1, 8, 0x10000, 0x20000, 0x30000, 5
    a.K = B.KV(0x40000, B.KVC_BF16, 0, 2 * 8 * 128, 8 * 128, 128)
    a.V = B.KV(0x50000, B.KVC_BF16, 0, 2 * 8 * 128, 8 * 128, 128)
    a.kept_bits, a.bits_words = 0x60000, 0                                        # pos 5 past 0 words
    assert lib.kvc_append(C.byref(m), C.byref(a), None) == 1
    a.bits_words = 1
    a.q, a.Qring, a.qpos, a.W, a.slot = 0x70000, 0x80000, 0x90000, 4, 4          # slot outside [0, W)
    assert lib.kvc_append(C.byref(m), C.byref(a), None) == 1
    a.slot = 0
    a.K2 = B.KV(0xa0000, B.KVC_BF16, 0, 2 * 16 * 128, 16 * 128, 128)            # second cache without V2, len2
    assert lib.kvc_append(C.byref(m), C.byref(a), None) == 1
    a.V2, a.len2, a.cap2 = B.KV(0xb0000, B.KVC_F32, 0, 2 * 16 * 128, 16 * 128, 128), 0xc0000, 16
    assert lib.kvc_append(C.byref(m), C.byref(a), None) == 1                    # V2 dtype differs from K
    a.V2 = B.KV(0xb0000, B.KVC_BF16, 0, 2 * 16 * 128, 16 * 128, 128)
    a.cap2 = 0                                                                     # cap2 below 1
    assert lib.kvc_append(C.byref(m), C.byref(a), None) == 1
    c = B.RecasCalibrateArgs()
    c.batch, c.delta, c.x, c.state, c.alpha = 1, 0x10000, 0x20000, 0x30000, 1.0   # alpha outside (0, 1)
    assert lib.kvc_recas_calibrate(C.byref(m), C.byref(c), None) == 1
    r = B.RecasControlArgs()
    r.batch, r.n, r.w, r.k0, r.S, r.A, r.s_row, r.state, r.need = 1, 16385, 0, 0, 0x1000, 0x2000, 16385, 0x3000, 0x4000
    assert lib.kvc_recas_control(C.byref(m), C.byref(r), None) == 2               # longer than 16384
    r.n, r.s_row, r.k0 = 100, 100, 101                                             # k0 > n
    assert lib.kvc_recas_control(C.byref(m), C.byref(r), None) == 1
    assert B.kvc_launch_count() == before


def test_lmhead_entropy_validation_and_workspace():
    """kvc_lmhead_entropy refuses bad arguments and a short workspace before launching
    anything; its workspace query needs no model (fake device addresses throughout)."""
    lib = B.lib()
    before = B.kvc_launch_count()
    a = B.LmheadEntropyArgs()
    a.n, a.Dh, a.V, a.k, a.dtype = 300, 512, 5000, 256, B.KVC_BF16
    a.x, a.x_stride, a.W, a.W_stride, a.H = 0x10000, 512, 0x20000, 512, 0x30000
    need = B.workspace_size(B.OP_LMHEAD_ENTROPY, None, a)
    assert need > 300 * 256 * 4
    assert lib.kvc_lmhead_entropy(C.byref(a), C.c_void_p(0x100000), need - 1, None) == 3   # short workspace
    for field, bad, code in [("k", 0, 2), ("k", 257, 2), ("dtype", B.KVC_F32, 2), ("x_stride", 516, 1),
                             ("W_stride", 256, 1), ("x", 0x10008, 1), ("n", 0, 1), ("H", 0, 1)]:
        good = getattr(a, field)
        setattr(a, field, bad)
        assert lib.kvc_lmhead_entropy(C.byref(a), C.c_void_p(0x100000), need, None) == code, field
        setattr(a, field, good)
    assert B.kvc_launch_count() == before
