"""kvc_decode_attn_noalloc: decode attention for callers that cannot allocate.

Some callers cannot call cudaMalloc or pass a workspace - a runtime that has
reserved all device memory for its own pool, or code that must avoid the
device-wide synchronisation an allocation may cause.  The no-alloc entry point
keeps its split-K partial results in the library's fixed device array instead.
This checks, through the C ABI, that two calls in a row give the results of
the workspace-taking kvc_decode_attn, and that a call needing more scratch than
the fixed array is refused before anything is launched.  It runs alone in a
fresh process as well as after the other tests.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from long_context_kv_obs_b200 import binding as B
from tests.helpers import OUT_ATOL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(seed, Bn, L, Hq, Hkv, d, lens):
    g = torch.Generator(device=DEV).manual_seed(seed)
    cap = int(max(lens)) + 3
    K = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(torch.bfloat16)
    V = torch.randn(Bn, L, Hkv, cap, d, device=DEV, generator=g).to(torch.bfloat16)
    q = torch.randn(Bn, L, Hq, d, device=DEV, generator=g).to(torch.bfloat16)
    R = 1.0 + 2.0 * torch.rand(Bn, L, Hkv, cap, device=DEV, generator=g)
    lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV).view(Bn, L)
    return K, V, q, R, lens_t


def _noalloc_call(m, K, V, q, R, lens_t, max_len, o):
    a = B.decode_args(m, q=q, K=K, V=V, lens=lens_t, max_len=max_len, o=o, R=R, alpha_c=1.0)
    stream = torch.cuda.current_stream().cuda_stream
    return B.lib().kvc_decode_attn_noalloc(C.byref(m), C.byref(a), C.c_void_p(stream))


def test_noalloc_decode_matches_workspace_decode_twice():
    Bn, L, Hq, Hkv, d = 2, 3, 28, 4, 128
    m = B.model(L, Hq, Hkv, d)
    for seed, lens in ((1, [4100, 17, 1, 2500, 3000, 333]), (2, [64, 5000, 1200, 7, 4096, 900])):
        K, V, q, R, lens_t = _case(seed, Bn, L, Hq, Hkv, d, lens)
        max_len = int(max(lens))
        o_ref = torch.empty(Bn, L, Hq, d, device=DEV)
        B.kvc_decode_attn(m, q=q, K=K, V=V, lens=lens_t, max_len=max_len, o=o_ref, R=R, alpha_c=1.0)
        o = torch.full_like(o_ref, float("nan"))
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        assert _noalloc_call(m, K, V, q, R, lens_t, max_len, o) == 0, B.lib().kvc_last_error()
        torch.cuda.synchronize()
        if seed == 2:
            # after the first call (which may be when the runtime first places the fixed
            # array in device memory) a call takes no device memory
            assert torch.cuda.mem_get_info()[0] == free0
        assert torch.isfinite(o).all()
        np.testing.assert_allclose(o.cpu().numpy(), o_ref.cpu().numpy(), atol=OUT_ATOL, rtol=0)
    assert B.kvc_check_status() == 0


def test_noalloc_refuses_oversized_scratch_before_launch():
    # 64 sequences x 32 layers x 8 KV heads: one partial record per (row, query head) is
    # 16384 * 4 * 130 floats = 34 MB, more than the fixed scratch
    Bn, L, Hq, Hkv, d = 64, 32, 32, 8, 128
    m = B.model(L, Hq, Hkv, d)
    K, V, q, R, lens_t = _case(3, Bn, L, Hq, Hkv, d, [8] * (Bn * L))
    o = torch.zeros(Bn, L, Hq, d, device=DEV)
    need = B.workspace_size(B.OP_DECODE, m, B.decode_args(m, q=q, K=K, V=V, lens=lens_t, max_len=8,
                                                          o=o, R=R))
    assert need > (8 << 20)
    st = _noalloc_call(m, K, V, q, R, lens_t, 8, o)
    assert st == 3                                   # KVC_ERR_WORKSPACE
    assert b"scratch" in B.lib().kvc_last_error()
    torch.cuda.synchronize()
    assert torch.count_nonzero(o) == 0              # nothing ran
