"""ctypes binding of libkvc (include/kvc.h): argument marshalling only.

Every function here packs torch tensors (device memory, owned by the caller)
into the C structs of kvc.h, passes the current CUDA stream, and raises
``KvcError`` on a non-zero status.  All computation happens in libkvc's
kernels; there is no fallback: if the library is missing, loading fails.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libkvc.so")
_lib = None

KVC_F32, KVC_BF16 = 0, 1
SCORE_INFOKV, SCORE_VATP, SCORE_ATTN = 0, 1, 2
SEL_PER_KV_HEAD, SEL_GQA_UNION = 0, 1
BUDGET_UNIFORM, BUDGET_EXPLICIT, BUDGET_ADAPTIVE = 0, 1, 2
(OP_SCORE, OP_SELECT, OP_COMPACT, OP_MERGE, OP_DECODE, OP_RECOMPRESS, OP_SPARSE_DECODE,
 OP_LMHEAD_ENTROPY) = range(8)
STATUS_NAMES = {0: "KVC_OK", 1: "KVC_ERR_ARG", 2: "KVC_ERR_UNSUPPORTED", 3: "KVC_ERR_WORKSPACE",
                4: "KVC_ERR_CUDA", 5: "KVC_ERR_TIMEOUT", 6: "KVC_ERR_DEVICE"}

EXPORTED = ["kvc_workspace_size", "kvc_score", "kvc_select", "kvc_compact", "kvc_merge",
            "kvc_rope_reposition", "kvc_decode_attn", "kvc_recompress", "kvc_append",
            "kvc_recas_calibrate", "kvc_recas_control", "kvc_sparse_decode", "kvc_lmhead_entropy",
            "kvc_check_status", "kvc_last_error", "kvc_version", "kvc_decode_attn_noalloc",
            "kvc_launch_count"]


class KvcError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


# --------------------------------------------------------------------------- C structs

class Model(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int),
                ("head_dim", C.c_int)]


class KV(C.Structure):
    _fields_ = [("ptr", C.c_void_p), ("dtype", C.c_int), ("s_batch", C.c_int64),
                ("s_layer", C.c_int64), ("s_head", C.c_int64), ("s_tok", C.c_int64)]


class ScoreArgs(C.Structure):
    _fields_ = [("mode", C.c_int), ("n", C.c_int), ("W", C.c_int), ("alpha", C.c_float),
                ("tau", C.c_float), ("scale", C.c_float), ("topk", C.c_int),
                ("Qw", C.c_void_p), ("qpos", C.c_void_p), ("K", KV), ("V", KV),
                ("kpos", C.c_void_p), ("kpos_s_layer", C.c_int64), ("kpos_s_head", C.c_int64),
                ("logits", C.c_void_p), ("logits_dtype", C.c_int), ("vocab", C.c_int64),
                ("logits_row_stride", C.c_int64), ("hidden", C.c_void_p), ("hidden_dtype", C.c_int),
                ("hidden_size", C.c_int), ("H_in", C.c_void_p), ("H_s_layer", C.c_int64),
                ("H_s_head", C.c_int64), ("D_in", C.c_void_p), ("D_s_layer", C.c_int64),
                ("D_s_head", C.c_int64), ("S", C.c_void_p), ("A", C.c_void_p), ("H_out", C.c_void_p),
                ("D_out", C.c_void_p), ("Ebar", C.c_void_p), ("window_sms", C.c_int),
                ("wait_limit_ns", C.c_uint64)]


class SelectArgs(C.Structure):
    _fields_ = [("sel_mode", C.c_int), ("n", C.c_int), ("w", C.c_int), ("S", C.c_void_p),
                ("S_s_layer", C.c_int64), ("S_s_head", C.c_int64), ("budget_mode", C.c_int),
                ("rho", C.c_double), ("k_in", C.c_void_p), ("B_total", C.c_int64),
                ("Ebar", C.c_void_p), ("k_out", C.c_void_p), ("idx", C.c_void_p), ("k_cap", C.c_int)]


class CompactArgs(C.Structure):
    _fields_ = [("n", C.c_int), ("src_K", KV), ("src_V", KV), ("dst_K", KV), ("dst_V", KV),
                ("idx", C.c_void_p), ("k_cap", C.c_int), ("k", C.c_void_p),
                ("src_pos", C.c_void_p), ("pos_s_layer", C.c_int64), ("pos_s_head", C.c_int64),
                ("dst_pos", C.c_void_p),
                ("src_H", C.c_void_p), ("H_s_layer", C.c_int64), ("H_s_head", C.c_int64),
                ("dst_H", C.c_void_p),
                ("src_D", C.c_void_p), ("D_s_layer", C.c_int64), ("D_s_head", C.c_int64),
                ("dst_D", C.c_void_p),
                ("src_U", C.c_void_p), ("U_s_layer", C.c_int64), ("U_s_head", C.c_int64),
                ("dst_U", C.c_void_p)]


class MergeArgs(C.Structure):
    _fields_ = [("n", C.c_int), ("bucket", C.c_int), ("V", KV), ("A", C.c_void_p),
                ("A_s_layer", C.c_int64), ("A_s_head", C.c_int64), ("idx", C.c_void_p),
                ("k_cap", C.c_int), ("k", C.c_void_p), ("dst_V", KV), ("R", C.c_void_p),
                ("dst_V_f32", C.c_void_p)]


class RopeArgs(C.Structure):
    _fields_ = [("K", KV), ("K_dst", KV), ("pos", C.c_void_p), ("pos_s_row", C.c_int64),
                ("pos_dst", C.c_void_p), ("k", C.c_void_p), ("k_cap", C.c_int), ("new0", C.c_int64),
                ("base", C.c_double)]


class DecodeArgs(C.Structure):
    _fields_ = [("batch", C.c_int), ("q", C.c_void_p), ("q_dtype", C.c_int), ("K", KV), ("V", KV),
                ("len", C.c_void_p), ("max_len", C.c_int), ("R", C.c_void_p),
                ("R_s_batch", C.c_int64), ("R_s_layer", C.c_int64), ("R_s_head", C.c_int64),
                ("alpha_c", C.c_float), ("scale", C.c_float), ("o", C.c_void_p), ("lse", C.c_void_p),
                ("K_full", KV), ("V_full", KV), ("len_full", C.c_void_p), ("max_len_full", C.c_int),
                ("kept_bits", C.c_void_p), ("bits_s_batch", C.c_int64), ("bits_s_layer", C.c_int64),
                ("bits_s_head", C.c_int64), ("delta", C.c_void_p), ("vmax", C.c_void_p),
                ("err", C.c_void_p), ("bound", C.c_void_p), ("o_full", C.c_void_p),
                ("o_kept", C.c_void_p), ("lse_stride", C.c_int64)]


class RecompressArgs(C.Structure):
    _fields_ = [("batch", C.c_int), ("len", C.c_int), ("t", C.c_int), ("rho", C.c_double),
                ("w", C.c_int), ("alpha", C.c_float), ("tau", C.c_float), ("scale", C.c_float),
                ("sel_mode", C.c_int), ("W", C.c_int), ("Qring", C.c_void_p), ("qpos", C.c_void_p),
                ("K", KV), ("V", KV), ("pos", C.c_void_p), ("H", C.c_void_p), ("D", C.c_void_p),
                ("side_s_row", C.c_int64), ("K_dst", KV), ("V_dst", KV), ("pos_dst", C.c_void_p),
                ("H_dst", C.c_void_p), ("D_dst", C.c_void_p), ("side_dst_s_row", C.c_int64),
                ("U", C.c_void_p), ("U_dst", C.c_void_p),
                ("cap_dst", C.c_int), ("k_out", C.c_void_p), ("kept_bits_dst", C.c_void_p),
                ("bits_s_batch", C.c_int64), ("bits_s_layer", C.c_int64), ("bits_s_head", C.c_int64),
                ("bits_words", C.c_int), ("host_kept", C.c_void_p), ("recas_state", C.c_void_p),
                ("recas_eps", C.c_float), ("recas_x", C.c_void_p), ("recas_k_max", C.c_int),
                ("win_lse", C.c_void_p)]


class SparseDecodeArgs(C.Structure):
    _fields_ = [("batch", C.c_int), ("q", C.c_void_p), ("q_dtype", C.c_int), ("K", KV), ("V", KV),
                ("len", C.c_void_p), ("max_len", C.c_int), ("pos", C.c_void_p), ("acc", C.c_void_p),
                ("side_s_row", C.c_int64), ("t_cur", C.c_int), ("n_prompt", C.c_int), ("kappa", C.c_double),
                ("a_tr", C.c_float), ("b_hi", C.c_float), ("scale", C.c_float), ("o", C.c_void_p),
                ("active", C.c_void_p), ("n_active", C.c_void_p), ("lse", C.c_void_p),
                ("lse_stride", C.c_int64)]


class LmheadEntropyArgs(C.Structure):
    _fields_ = [("n", C.c_int), ("Dh", C.c_int), ("V", C.c_int), ("k", C.c_int), ("dtype", C.c_int),
                ("x", C.c_void_p), ("x_stride", C.c_int64), ("W", C.c_void_p), ("W_stride", C.c_int64),
                ("H", C.c_void_p)]


RECAS_RING = 256
# kvc_recas_cal as float64 words: sum_delta, sum_x, c, q, (count, head as two int32), ring
RECAS_STATE_WORDS = 5 + RECAS_RING


class RecasCalibrateArgs(C.Structure):
    _fields_ = [("batch", C.c_int), ("delta", C.c_void_p), ("x", C.c_void_p), ("alpha", C.c_float),
                ("state", C.c_void_p), ("delta_hat", C.c_void_p), ("delta_bar", C.c_void_p)]


class RecasControlArgs(C.Structure):
    _fields_ = [("sel_mode", C.c_int), ("batch", C.c_int), ("n", C.c_int), ("w", C.c_int), ("k0", C.c_int),
                ("S", C.c_void_p), ("A", C.c_void_p), ("s_row", C.c_int64), ("state", C.c_void_p),
                ("eps", C.c_float), ("need", C.c_void_p), ("budget", C.c_void_p), ("k_max", C.c_int)]


class AppendArgs(C.Structure):
    _fields_ = [("batch", C.c_int), ("cap", C.c_int), ("k", C.c_void_p), ("v", C.c_void_p),
                ("K", KV), ("V", KV), ("len", C.c_void_p), ("pos", C.c_int),
                ("side_pos", C.c_void_p), ("side_H", C.c_void_p), ("side_D", C.c_void_p),
                ("side_R", C.c_void_p), ("side_U", C.c_void_p), ("side_s_row", C.c_int64),
                ("H_new", C.c_void_p),
                ("D_new", C.c_void_p), ("D_new_s_batch", C.c_int64), ("D_new_s_layer", C.c_int64),
                ("kept_bits", C.c_void_p), ("bits_s_batch", C.c_int64), ("bits_s_layer", C.c_int64),
                ("bits_s_head", C.c_int64), ("bits_words", C.c_int), ("q", C.c_void_p),
                ("Qring", C.c_void_p), ("qpos", C.c_void_p), ("W", C.c_int), ("slot", C.c_int),
                ("K2", KV), ("V2", KV), ("len2", C.c_void_p), ("cap2", C.c_int)]


# --------------------------------------------------------------------------- loading

def lib_path() -> str:
    return _LIB_PATH


def lib():
    """The loaded libkvc (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libkvc not built ({_LIB_PATH} missing): run "
                               "`python -m long_context_kv_obs_b200.build`")
        L = C.CDLL(_LIB_PATH)
        for name in ("kvc_score", "kvc_select", "kvc_merge", "kvc_decode_attn", "kvc_recompress"):
            getattr(L, name).argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]
            getattr(L, name).restype = C.c_int
        L.kvc_decode_attn_noalloc.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
        L.kvc_decode_attn_noalloc.restype = C.c_int
        L.kvc_compact.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
        L.kvc_compact.restype = C.c_int
        L.kvc_rope_reposition.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
        L.kvc_rope_reposition.restype = C.c_int
        L.kvc_append.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
        L.kvc_append.restype = C.c_int
        L.kvc_sparse_decode.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]
        L.kvc_sparse_decode.restype = C.c_int
        L.kvc_lmhead_entropy.argtypes = [C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]
        L.kvc_lmhead_entropy.restype = C.c_int
        for name in ("kvc_recas_calibrate", "kvc_recas_control"):
            getattr(L, name).argtypes = [C.c_void_p, C.c_void_p, C.c_void_p]
            getattr(L, name).restype = C.c_int
        L.kvc_workspace_size.argtypes = [C.c_int, C.c_void_p, C.c_void_p, C.POINTER(C.c_size_t)]
        L.kvc_workspace_size.restype = C.c_int
        L.kvc_check_status.argtypes = [C.c_void_p, C.POINTER(C.c_uint32)]
        L.kvc_check_status.restype = C.c_int
        L.kvc_last_error.argtypes = []
        L.kvc_last_error.restype = C.c_char_p
        L.kvc_version.argtypes = []
        L.kvc_version.restype = C.c_int
        L.kvc_launch_count.argtypes = []
        L.kvc_launch_count.restype = C.c_uint64
        _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise KvcError(status, lib().kvc_last_error().decode())


# --------------------------------------------------------------------------- marshalling helpers

def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KVC_BF16
    if t.dtype == torch.float32:
        return KVC_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _p(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor required")
    return t.data_ptr()


def _f32(t: Optional[torch.Tensor], name: str) -> Optional[int]:
    if t is None:
        return None
    if t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32")
    return _p(t)


def _i32(t: Optional[torch.Tensor], name: str) -> Optional[int]:
    if t is None:
        return None
    if t.dtype != torch.int32:
        raise TypeError(f"{name} must be int32")
    return _p(t)


def kv(t: Optional[torch.Tensor]) -> KV:
    """KV descriptor of a [L][H][T][d] or [B][L][H][T][d] tensor with contiguous rows."""
    if t is None:
        return KV()
    if t.stride(-1) != 1:
        raise ValueError("rows must be contiguous")
    if t.dim() == 4:
        sb, (sl, sh, st) = 0, t.stride()[:3]
    elif t.dim() == 5:
        sb, sl, sh, st = t.stride()[:4]
    else:
        raise ValueError("expected a 4-D or 5-D tensor")
    return KV(_p(t), _dt(t), sb, sl, sh, st)


def model(n_layers: int, n_q_heads: int, n_kv_heads: int, head_dim: int) -> Model:
    return Model(n_layers, n_q_heads, n_kv_heads, head_dim)


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def workspace_size(op: int, m: Optional[Model], args) -> int:
    n = C.c_size_t(0)
    _check(lib().kvc_workspace_size(op, C.byref(m) if m is not None else None, C.byref(args), C.byref(n)))
    return n.value


def _ws(op, m, args, workspace: Optional[torch.Tensor], device):
    need = workspace_size(op, m, args)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    elif workspace.numel() < need:
        raise ValueError(f"workspace of {workspace.numel()} bytes < {need}")
    return workspace, need


# --------------------------------------------------------------------------- the six calls

def kvc_score(m: Model, *, mode: int, n: int, W: int, Qw: torch.Tensor, K: torch.Tensor,
              S: torch.Tensor, V: Optional[torch.Tensor] = None, qpos=None, kpos=None,
              kpos_strides=(0, 0), logits=None, hidden=None, H_in=None, H_strides=(0, 0),
              D_in=None, D_strides=(0, 0), alpha: float = 0.9, tau: float = 1.0,
              scale: float = 0.0, topk: int = 256, A=None, H_out=None, D_out=None, Ebar=None,
              window_sms: int = 0, wait_limit_ns: int = 0, workspace=None, stream=None):
    """Scores S[L][Hkv][n] (and optionally A, H, D, E-bar); see kvc.h."""
    a = ScoreArgs()
    a.mode, a.n, a.W, a.alpha, a.tau, a.scale, a.topk = mode, n, W, alpha, tau, scale, topk
    if Qw.dtype != K.dtype or not Qw.is_contiguous():
        raise ValueError("Qw must be contiguous with the dtype of K")
    a.Qw, a.qpos = _p(Qw), _i32(qpos, "qpos")
    a.K, a.V = kv(K), kv(V)
    a.kpos = _i32(kpos, "kpos")
    a.kpos_s_layer, a.kpos_s_head = kpos_strides
    if logits is not None:
        if logits.stride(-1) != 1:
            raise ValueError("logits rows must be contiguous")
        a.logits, a.logits_dtype = _p(logits), _dt(logits)
        a.vocab, a.logits_row_stride = logits.shape[-1], logits.stride(0)
    if hidden is not None:
        if not hidden.is_contiguous():
            raise ValueError("hidden must be contiguous")
        a.hidden, a.hidden_dtype, a.hidden_size = _p(hidden), _dt(hidden), hidden.shape[-1]
    a.H_in = _f32(H_in, "H_in")
    a.H_s_layer, a.H_s_head = H_strides
    a.D_in = _f32(D_in, "D_in")
    a.D_s_layer, a.D_s_head = D_strides
    a.S, a.A = _f32(S, "S"), _f32(A, "A")
    a.H_out, a.D_out, a.Ebar = _f32(H_out, "H_out"), _f32(D_out, "D_out"), _f32(Ebar, "Ebar")
    a.window_sms, a.wait_limit_ns = window_sms, wait_limit_ns
    ws, need = _ws(OP_SCORE, m, a, workspace, K.device)
    _check(lib().kvc_score(C.byref(m), C.byref(a), _p(ws), ws.numel(), _stream(stream)))
    return ws


def kvc_select(m: Model, *, n: int, w: int, S: torch.Tensor, k_out: torch.Tensor,
               idx: torch.Tensor, sel_mode: int = SEL_PER_KV_HEAD, budget_mode: int = BUDGET_UNIFORM,
               rho: float = 0.0, k_in=None, B_total: int = 0, Ebar=None, S_strides=None,
               workspace=None, stream=None):
    """Budgets k_out[L] and ascending kept positions idx[L][Hkv][k_cap]."""
    a = SelectArgs()
    a.sel_mode, a.n, a.w = sel_mode, n, w
    a.S = _f32(S, "S")
    a.S_s_layer, a.S_s_head = S_strides if S_strides else (S.stride(0), S.stride(1))
    a.budget_mode, a.rho, a.k_in, a.B_total = budget_mode, rho, _i32(k_in, "k_in"), B_total
    a.Ebar = _f32(Ebar, "Ebar")
    a.k_out, a.idx, a.k_cap = _i32(k_out, "k_out"), _i32(idx, "idx"), idx.shape[-1]
    ws, need = _ws(OP_SELECT, m, a, workspace, S.device)
    _check(lib().kvc_select(C.byref(m), C.byref(a), _p(ws), ws.numel(), _stream(stream)))
    return ws


def kvc_compact(m: Model, *, n: int, idx: torch.Tensor, k: torch.Tensor, src_K=None, src_V=None,
                dst_K=None, dst_V=None, src_pos=None, pos_strides=(0, 0), dst_pos=None,
                src_H=None, H_strides=(0, 0), dst_H=None, src_D=None, D_strides=(0, 0),
                dst_D=None, src_U=None, U_strides=(0, 0), dst_U=None, stream=None):
    """dst rows j < k_l of every (l, g) = src rows idx(l, g, j), bit-exact."""
    a = CompactArgs()
    a.n = n
    a.src_K, a.src_V, a.dst_K, a.dst_V = kv(src_K), kv(src_V), kv(dst_K), kv(dst_V)
    a.idx, a.k_cap, a.k = _i32(idx, "idx"), idx.shape[-1], _i32(k, "k")
    a.src_pos, (a.pos_s_layer, a.pos_s_head), a.dst_pos = _i32(src_pos, "src_pos"), pos_strides, _i32(dst_pos, "dst_pos")
    a.src_H, (a.H_s_layer, a.H_s_head), a.dst_H = _f32(src_H, "src_H"), H_strides, _f32(dst_H, "dst_H")
    a.src_D, (a.D_s_layer, a.D_s_head), a.dst_D = _f32(src_D, "src_D"), D_strides, _f32(dst_D, "dst_D")
    a.src_U, (a.U_s_layer, a.U_s_head), a.dst_U = _f32(src_U, "src_U"), U_strides, _f32(dst_U, "dst_U")
    _check(lib().kvc_compact(C.byref(m), C.byref(a), _stream(stream)))


def kvc_merge(m: Model, *, n: int, V: torch.Tensor, A: torch.Tensor, idx: torch.Tensor,
              k: torch.Tensor, dst_V: torch.Tensor, R: torch.Tensor, bucket: int = 512,
              dst_V_f32=None, A_strides=None, stream=None):
    """SelKV merge: V' (compacted, merged) and R for every kept slot."""
    a = MergeArgs()
    a.n, a.bucket, a.V = n, bucket, kv(V)
    a.A = _f32(A, "A")
    a.A_s_layer, a.A_s_head = A_strides if A_strides else (A.stride(0), A.stride(1))
    a.idx, a.k_cap, a.k = _i32(idx, "idx"), idx.shape[-1], _i32(k, "k")
    a.dst_V, a.R, a.dst_V_f32 = kv(dst_V), _f32(R, "R"), _f32(dst_V_f32, "dst_V_f32")
    _check(lib().kvc_merge(C.byref(m), C.byref(a), None, 0, _stream(stream)))


def _row_stride(t: torch.Tensor, name: str) -> int:
    """Element stride between the (l, g) rows of an [L][Hkv][C] int32 tensor (rows contiguous)."""
    if t.dim() != 3 or t.stride(2) != 1 or t.stride(0) != t.shape[1] * t.stride(1):
        raise ValueError(f"{name} must be [L][Hkv][C] with evenly spaced contiguous rows")
    return t.stride(1)


def kvc_rope_reposition(m: Model, *, K: torch.Tensor, pos: torch.Tensor, k: torch.Tensor,
                        base: float, new0: int = 0, k_cap: Optional[int] = None, K_dst=None,
                        pos_dst=None, stream=None):
    """SelKV RoPE re-positioning: key row j < k_l of every (l, g), rotated at pos(l, g, j),
    is turned to position new0 + j (in place unless K_dst is given)."""
    a = RopeArgs()
    a.K, a.K_dst = kv(K), kv(K_dst)
    a.pos, a.pos_s_row = _i32(pos, "pos"), _row_stride(pos, "pos")
    if pos_dst is not None and _row_stride(pos_dst, "pos_dst") != a.pos_s_row:
        raise ValueError("pos_dst must have the row stride of pos")
    a.pos_dst = _i32(pos_dst, "pos_dst")
    a.k = _i32(k, "k")
    a.k_cap = k_cap if k_cap is not None else min(K.shape[-2], pos.shape[-1])
    a.new0, a.base = new0, base
    _check(lib().kvc_rope_reposition(C.byref(m), C.byref(a), _stream(stream)))


def _lse(lse):
    """Pointer and element stride of an lse output: [B][L][Hq], contiguous or one slot of a
    [B][L][Hq][W] ring (one element stride between consecutive entries)."""
    if lse is None:
        return None, 0
    s = lse.stride(-1)
    if lse.dim() != 3 or lse.stride(1) != lse.shape[2] * s or lse.stride(0) != lse.shape[1] * lse.shape[2] * s:
        raise ValueError("lse must be [B][L][Hq] with one element stride between entries")
    return _f32(lse, "lse"), s


def decode_args(m: Model, *, q: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                lens: torch.Tensor, max_len: int, o: torch.Tensor, R=None, alpha_c: float = 1.0,
                scale: float = 0.0, lse=None, K_full=None, V_full=None, lens_full=None,
                max_len_full: int = 0, kept_bits=None, delta=None, vmax=None, err=None,
                bound=None, o_full=None, o_kept=None, stream=None) -> DecodeArgs:
    """The DecodeArgs struct for these tensors (see kvc_decode_attn)."""
    a = DecodeArgs()
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    a.batch = q.shape[0]
    a.q, a.q_dtype = _p(q), _dt(q)
    a.K, a.V = kv(K), kv(V)
    a.len, a.max_len = _i32(lens, "lens"), max_len
    if R is not None:
        a.R = _f32(R, "R")
        if R.dim() == 4:
            a.R_s_batch, a.R_s_layer, a.R_s_head = R.stride(0), R.stride(1), R.stride(2)
        else:
            a.R_s_batch, a.R_s_layer, a.R_s_head = 0, R.stride(0), R.stride(1)
    a.alpha_c, a.scale = alpha_c, scale
    a.o = _f32(o, "o")
    a.lse, a.lse_stride = _lse(lse)
    if K_full is not None:
        a.K_full, a.V_full = kv(K_full), kv(V_full)
        a.len_full, a.max_len_full = _i32(lens_full, "lens_full"), max_len_full
        if kept_bits.dtype != torch.int32:
            raise TypeError("kept_bits must be int32 words")
        a.kept_bits = _p(kept_bits)
        a.bits_s_batch, a.bits_s_layer, a.bits_s_head = (kept_bits.stride(0), kept_bits.stride(1),
                                                         kept_bits.stride(2))
        a.delta, a.vmax, a.err, a.bound = (_f32(delta, "delta"), _f32(vmax, "vmax"),
                                           _f32(err, "err"), _f32(bound, "bound"))
        a.o_full, a.o_kept = _f32(o_full, "o_full"), _f32(o_kept, "o_kept")
    return a


def kvc_decode_attn(m: Model, *, workspace=None, stream=None, **kw):
    """Decode attention over K, V [B][L][Hkv][cap][d] for q [B][L][Hq][d] -> o (fp32)."""
    a = decode_args(m, **kw)
    ws, need = _ws(OP_DECODE, m, a, workspace, kw["q"].device)
    _check(lib().kvc_decode_attn(C.byref(m), C.byref(a), _p(ws), ws.numel(), _stream(stream)))
    return ws


def kvc_decode_attn_noalloc(m: Model, *, stream=None, **kw):
    """kvc_decode_attn without a workspace, for callers that cannot allocate device memory.

    The split-K partials use the library's fixed 8 MiB device array (shared by
    every call; overlapping calls on unordered streams race).  The first call
    on a device looks up that array's address: make it before stream capture.
    """
    a = decode_args(m, **kw)
    _check(lib().kvc_decode_attn_noalloc(C.byref(m), C.byref(a), _stream(stream)))


def _bits_strides(bits: torch.Tensor):
    """Word strides and words per row of a [B][L][Hkv][words] int32 kept-bit mask."""
    if bits.dtype != torch.int32 or bits.dim() != 4 or bits.stride(3) != 1:
        raise ValueError("kept bits must be [B][L][Hkv][words] int32 with contiguous rows")
    return bits.stride(0), bits.stride(1), bits.stride(2), bits.shape[3]


def recompress_args(m: Model, *, len_: int, t: int, rho: float, w: int, W: int, Qring, qpos,
                    K, V, pos, H, D, K_dst, V_dst, pos_dst, H_dst, D_dst, alpha: float = 0.9,
                    tau: float = 1.0, scale: float = 0.0, sel_mode: int = SEL_PER_KV_HEAD,
                    k_out=None, kept_bits_dst=None, recas_state=None, recas_eps: float = 0.0,
                    recas_x=None, recas_k_max: int = 0, U=None, U_dst=None, win_lse=None,
                    stream=None) -> RecompressArgs:
    """The RecompressArgs struct for these tensors (see kvc_recompress)."""
    a = RecompressArgs()
    a.batch, a.len, a.t, a.rho, a.w = K.shape[0], len_, t, rho, w
    a.alpha, a.tau, a.scale, a.sel_mode, a.W = alpha, tau, scale, sel_mode, W
    a.Qring, a.qpos = _p(Qring), _i32(qpos, "qpos")
    a.K, a.V = kv(K), kv(V)
    a.pos, a.H, a.D = _i32(pos, "pos"), _f32(H, "H"), _f32(D, "D")
    a.side_s_row = pos.stride(-2)
    a.K_dst, a.V_dst = kv(K_dst), kv(V_dst)
    a.pos_dst, a.H_dst, a.D_dst = _i32(pos_dst, "pos_dst"), _f32(H_dst, "H_dst"), _f32(D_dst, "D_dst")
    a.side_dst_s_row = pos_dst.stride(-2)
    a.U, a.U_dst = _f32(U, "U"), _f32(U_dst, "U_dst")
    if win_lse is not None and not win_lse.is_contiguous():
        raise ValueError("win_lse must be a contiguous [B][L][Hq][W] ring")
    a.win_lse = _f32(win_lse, "win_lse")
    a.cap_dst = K_dst.shape[-2]
    a.k_out = _i32(k_out, "k_out")
    if kept_bits_dst is not None:
        a.kept_bits_dst = _p(kept_bits_dst)
        a.bits_s_batch, a.bits_s_layer, a.bits_s_head, a.bits_words = _bits_strides(kept_bits_dst)
    if recas_state is not None:
        a.recas_state = _recas_state_ptr(recas_state, K.shape[0], m.n_layers)
        a.recas_eps = recas_eps
        a.recas_x = _f32(recas_x, "recas_x")
        a.recas_k_max = recas_k_max
    return a


def kvc_recompress(m: Model, *, workspace=None, stream=None, **kw):
    """Recompress every sequence of a batch from len_ rows to floor(rho * t) rows (or to the
    RECAS budget when recas_state is given).

    Returns (workspace, rows kept per cache row; -1 when the budget is set on the device);
    with kept_bits_dst the RECAS kept-position mask is rebuilt from the kept positions."""
    a = recompress_args(m, **kw)
    kept = C.c_int(-2)
    a.host_kept = C.addressof(kept)
    ws, need = _ws(OP_RECOMPRESS, m, a, workspace, kw["K"].device)
    _check(lib().kvc_recompress(C.byref(m), C.byref(a), _p(ws), ws.numel(), _stream(stream)))
    return ws, kept.value


def sparse_decode_args(m: Model, *, q, K, V, lens, max_len: int, pos, acc, t_cur: int, n_prompt: int,
                       kappa: float, a_tr: float, b_hi: float, o, scale: float = 0.0, active=None,
                       n_active=None, lse=None, stream=None) -> SparseDecodeArgs:
    """The SparseDecodeArgs struct for these tensors (see kvc_sparse_decode)."""
    a = SparseDecodeArgs()
    if not q.is_contiguous():
        raise ValueError("q must be contiguous")
    if pos.stride(-2) != acc.stride(-2) or pos.stride(-1) != 1 or acc.stride(-1) != 1:
        raise ValueError("pos and acc must share one row stride with contiguous rows")
    a.batch, a.q, a.q_dtype = q.shape[0], _p(q), _dt(q)
    a.K, a.V = kv(K), kv(V)
    a.len, a.max_len = _i32(lens, "lens"), max_len
    a.pos, a.acc, a.side_s_row = _i32(pos, "pos"), _f32(acc, "acc"), pos.stride(-2)
    a.t_cur, a.n_prompt, a.kappa, a.a_tr, a.b_hi, a.scale = t_cur, n_prompt, kappa, a_tr, b_hi, scale
    a.o, a.active, a.n_active = _f32(o, "o"), _i32(active, "active"), _i32(n_active, "n_active")
    a.lse, a.lse_stride = _lse(lse)
    return a


def kvc_sparse_decode(m: Model, *, workspace=None, stream=None, **kw):
    """RECAS dynamic sparse decode over the retained caches (see kvc.h); returns the workspace."""
    a = sparse_decode_args(m, **kw)
    ws, need = _ws(OP_SPARSE_DECODE, m, a, workspace, kw["q"].device)
    _check(lib().kvc_sparse_decode(C.byref(m), C.byref(a), _p(ws), ws.numel(), _stream(stream)))
    return ws


def lmhead_entropy_args(*, x: torch.Tensor, W: torch.Tensor, H: torch.Tensor, k: int = 256) -> LmheadEntropyArgs:
    """Argument struct of kvc_lmhead_entropy: x [n][Dh], W [V][Dh] bf16 (unit column stride), H [n] fp32."""
    if x.dtype != torch.bfloat16 or W.dtype != torch.bfloat16:
        raise ValueError("x and W must be bf16")
    if x.dim() != 2 or W.dim() != 2 or x.shape[1] != W.shape[1] or x.stride(1) != 1 or W.stride(1) != 1:
        raise ValueError("x [n][Dh] and W [V][Dh] with unit column stride")
    if H.dtype != torch.float32 or H.dim() != 1 or H.shape[0] != x.shape[0] or H.stride(0) != 1:
        raise ValueError("H must be a contiguous fp32 [n] tensor")
    a = LmheadEntropyArgs()
    a.n, a.Dh, a.V, a.k, a.dtype = x.shape[0], x.shape[1], W.shape[0], k, KVC_BF16
    a.x, a.x_stride, a.W, a.W_stride, a.H = _p(x), x.stride(0), _p(W), W.stride(0), _p(H)
    return a


def kvc_lmhead_entropy(*, x: torch.Tensor, W: torch.Tensor, H: torch.Tensor, k: int = 256, workspace=None,
                       stream=None):
    """Top-k entropy H [n] of softmax(W x_i) without writing the logits (see kvc.h); returns the workspace."""
    a = lmhead_entropy_args(x=x, W=W, H=H, k=k)
    ws, need = _ws(OP_LMHEAD_ENTROPY, None, a, workspace, x.device)
    _check(lib().kvc_lmhead_entropy(C.byref(a), _p(ws), ws.numel(), _stream(stream)))
    return ws


def recas_state(batch: int, n_layers: int, device) -> torch.Tensor:
    """A zeroed RECAS calibration state for every (sequence, layer): the initial state."""
    return torch.zeros(batch, n_layers, RECAS_STATE_WORDS, dtype=torch.float64, device=device)


def _recas_state_ptr(state: torch.Tensor, batch: int, L: int) -> int:
    if state.dtype != torch.float64 or tuple(state.shape) != (batch, L, RECAS_STATE_WORDS) or not state.is_contiguous():
        raise ValueError(f"RECAS state must be a contiguous float64 [{batch}][{L}][{RECAS_STATE_WORDS}] tensor")
    return _p(state)


def recas_fields(state: torch.Tensor) -> dict:
    """Host copy of the readable fields of a RECAS state tensor (c, q, sums, count, ring)."""
    h = state.detach().cpu()
    ints = h[..., 4:5].contiguous().view(torch.int32)
    return {"sum_delta": h[..., 0], "sum_x": h[..., 1], "c": h[..., 2], "q": h[..., 3],
            "count": ints[..., 0], "head": ints[..., 1], "ring": h[..., 5:]}


def kvc_recas_calibrate(m: Model, *, delta, x, state, alpha: float = 0.1, delta_hat=None, delta_bar=None,
                        stream=None):
    """RECAS calibration at a probe step: delta [B][L][Hq], predictors x [B][L][Hkv]."""
    a = RecasCalibrateArgs()
    if not (delta.is_contiguous() and x.is_contiguous()):
        raise ValueError("delta and x must be contiguous")
    a.batch = delta.shape[0]
    a.delta, a.x, a.alpha = _f32(delta, "delta"), _f32(x, "x"), alpha
    a.state = _recas_state_ptr(state, a.batch, m.n_layers)
    a.delta_hat, a.delta_bar = _f32(delta_hat, "delta_hat"), _f32(delta_bar, "delta_bar")
    _check(lib().kvc_recas_calibrate(C.byref(m), C.byref(a), _stream(stream)))


def kvc_recas_control(m: Model, *, S, A, n: int, w: int, k0: int, state, eps: float, need, budget=None,
                      k_max: int = 0, sel_mode: int = SEL_PER_KV_HEAD, stream=None):
    """RECAS controller: each row's need and the largest (budget) for rows S, A [B][L][Hkv][>= n]."""
    a = RecasControlArgs()
    if S.shape != A.shape or S.stride() != A.stride() or S.stride(-1) != 1 or S.dim() != 4:
        raise ValueError("S and A must be [B][L][Hkv][C] with one layout and contiguous rows")
    if S.stride(0) != S.shape[1] * S.shape[2] * S.stride(2) or S.stride(1) != S.shape[2] * S.stride(2):
        raise ValueError("S rows must be evenly spaced")
    a.sel_mode, a.batch, a.n, a.w, a.k0 = sel_mode, S.shape[0], n, w, k0
    a.S, a.A, a.s_row = _f32(S, "S"), _f32(A, "A"), S.stride(2)
    a.state = _recas_state_ptr(state, a.batch, m.n_layers)
    a.eps = eps
    a.need, a.budget, a.k_max = _i32(need, "need"), _i32(budget, "budget"), k_max
    _check(lib().kvc_recas_control(C.byref(m), C.byref(a), _stream(stream)))


def kvc_append(m: Model, *, k, v, K, V, lens, pos: int, side_pos=None, side_H=None, side_D=None,
               side_R=None, side_U=None, H_new=None, D_new=None, kept_bits=None, q=None, Qring=None, qpos=None,
               slot: int = 0, K2=None, V2=None, lens2=None, stream=None):
    """One generated token into every (b, l, g) cache row at row lens[b][l] (then lens += 1).

    k, v [B][L][Hkv][d]; K, V [B][L][Hkv][cap][d]; side arrays [B][L][Hkv][C] (one row stride);
    H_new [B]; D_new [B][L] (any strides); kept_bits [B][L][Hkv][words] int32; q [B][L][Hq][d],
    Qring [B][L][Hq][W][d], qpos [B][W]; K2, V2 [B][L][Hkv][cap2][d] and lens2 [B][L]: a second
    cache receiving the same rows at lens2 (then lens2 += 1), in the same launch."""
    a = AppendArgs()
    if k.dtype != K.dtype or v.dtype != K.dtype or not k.is_contiguous() or not v.is_contiguous():
        raise ValueError("k and v must be contiguous with the dtype of K")
    a.batch, a.cap = K.shape[0], K.shape[-2]
    a.k, a.v = _p(k), _p(v)
    a.K, a.V = kv(K), kv(V)
    a.len, a.pos = _i32(lens, "lens"), pos
    sides = [x for x in (side_pos, side_H, side_D, side_R, side_U) if x is not None]
    if sides:
        rs = {x.stride(-2) for x in sides}
        if len(rs) != 1 or any(x.stride(-1) != 1 for x in sides):
            raise ValueError("side arrays must share one row stride with contiguous rows")
        a.side_s_row = rs.pop()
    a.side_pos, a.side_H = _i32(side_pos, "side_pos"), _f32(side_H, "side_H")
    a.side_D, a.side_R, a.side_U = _f32(side_D, "side_D"), _f32(side_R, "side_R"), _f32(side_U, "side_U")
    a.H_new = _f32(H_new, "H_new")
    if D_new is not None:
        a.D_new = _f32(D_new, "D_new")
        a.D_new_s_batch, a.D_new_s_layer = D_new.stride(0), D_new.stride(1)
    if kept_bits is not None:
        a.kept_bits = _p(kept_bits)
        a.bits_s_batch, a.bits_s_layer, a.bits_s_head, a.bits_words = _bits_strides(kept_bits)
    if q is not None:
        if q.dtype != K.dtype or not q.is_contiguous() or not Qring.is_contiguous():
            raise ValueError("q and Qring must be contiguous with the dtype of K")
        a.q, a.Qring, a.qpos = _p(q), _p(Qring), _i32(qpos, "qpos")
        a.W, a.slot = Qring.shape[-2], slot
    if K2 is not None:
        if K2.dtype != K.dtype or V2.dtype != K.dtype:
            raise ValueError("K2 and V2 must have the dtype of K")
        a.K2, a.V2, a.len2, a.cap2 = kv(K2), kv(V2), _i32(lens2, "lens2"), K2.shape[-2]
    _check(lib().kvc_append(C.byref(m), C.byref(a), _stream(stream)))


def kvc_check_status(stream=None) -> int:
    code = C.c_uint32(0)
    st = lib().kvc_check_status(_stream(stream), C.byref(code))
    if st != 0:
        raise KvcError(st, lib().kvc_last_error().decode())
    return code.value


def kvc_version() -> int:
    return lib().kvc_version()


def kvc_launch_count() -> int:
    """Kernels the library has launched in this process (host-side tally)."""
    return lib().kvc_launch_count()
