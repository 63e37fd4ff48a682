"""ctypes mirror of include/gdr.h and the loader of libgdr.so.

Only argument marshalling lives here.  If the library has not been built the
first call raises at once: there is no other implementation to fall back on.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgdr.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "gdr.h")

GDR_F32 = 0
GDR_BF16 = 1
GDR_DECODE_OVERLAP_STATE_LOAD = 1
GDR_GATE_FROM_RAW = 2
GDR_PREFILL_NOALLOC_MAX_SEQS = 4096

STATUS_NAMES = {
    0: "GDR_OK", 1: "GDR_ERR_INVALID_ARG", 2: "GDR_ERR_UNSUPPORTED", 3: "GDR_ERR_MISALIGNED",
    4: "GDR_ERR_WORKSPACE", 5: "GDR_ERR_CUDA", 6: "GDR_ERR_TIMEOUT",
}

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_f32 = ctypes.c_float


class DecodeArgs(ctypes.Structure):
    _fields_ = [
        ("batch", _i32), ("H_k", _i32), ("H_v", _i32), ("d_k", _i32), ("d_v", _i32),
        ("in_dtype", _i32), ("out_dtype", _i32), ("qk_l2norm", _i32),
        ("scale", _f32), ("eps_l2", _f32), ("eps_norm", _f32), ("flags", _i32),
        ("q_stride", _i64), ("k_stride", _i64), ("v_stride", _i64), ("z_stride", _i64),
        ("gb_stride", _i64), ("out_stride", _i64), ("state_stride", _i64),
        ("q", _vp), ("k", _vp), ("v", _vp), ("z", _vp), ("g", _vp), ("beta", _vp),
        ("state_in", _vp), ("state_out", _vp), ("norm_w", _vp), ("out", _vp),
        ("A_log", _vp), ("dt_bias", _vp),
    ]


class DecodeMultiArgs(ctypes.Structure):
    _fields_ = [
        ("base", DecodeArgs), ("n_tokens", _i32), ("n_slots", _i32),
        ("state_slot", _vp), ("status", _vp),
    ]


class PrefillArgs(ctypes.Structure):
    _fields_ = [
        ("n_seq", _i32), ("H_k", _i32), ("H_v", _i32), ("d_k", _i32), ("d_v", _i32),
        ("chunk", _i32), ("in_dtype", _i32), ("out_dtype", _i32), ("qk_l2norm", _i32),
        ("scale", _f32), ("eps_l2", _f32), ("eps_norm", _f32),
        ("n_tok", _i64),
        ("q_stride", _i64), ("k_stride", _i64), ("v_stride", _i64), ("z_stride", _i64),
        ("gb_stride", _i64), ("out_stride", _i64),
        ("q", _vp), ("k", _vp), ("v", _vp), ("z", _vp), ("g", _vp), ("beta", _vp),
        ("cu_seqlens", _vp), ("cu_seqlens_host", ctypes.POINTER(_i32)),
        ("initial_state", _vp), ("final_state", _vp), ("norm_w", _vp), ("out", _vp),
        ("flags", _i32), ("reserved", _i32), ("A_log", _vp), ("dt_bias", _vp),
    ]


class NormArgs(ctypes.Structure):
    _fields_ = [
        ("rows", _i64), ("d", _i32), ("o_dtype", _i32), ("z_dtype", _i32), ("out_dtype", _i32),
        ("eps", _f32), ("reserved", _i32),
        ("o_stride", _i64), ("z_stride", _i64), ("out_stride", _i64),
        ("o", _vp), ("z", _vp), ("w", _vp), ("out", _vp),
    ]


class AttnDecodeArgs(ctypes.Structure):
    _fields_ = [
        ("batch", _i32), ("H_q", _i32), ("H_kv", _i32), ("d", _i32),
        ("rot_dim", _i32), ("max_len", _i32), ("kv_bound", _i32), ("out_dtype", _i32),
        ("rope_theta", _f32), ("scale", _f32),
        ("q_stride", _i64), ("gate_stride", _i64), ("k_stride", _i64), ("v_stride", _i64),
        ("out_stride", _i64),
        ("q", _vp), ("gate", _vp), ("k", _vp), ("v", _vp),
        ("k_cache", _vp), ("v_cache", _vp), ("cache_len", _vp), ("out", _vp),
    ]


class MoeArgs(ctypes.Structure):
    _fields_ = [
        ("n_tok", _i32), ("hidden", _i32), ("n_exp", _i32), ("top_k", _i32), ("inter", _i32),
        ("s_inter", _i32), ("out_dtype", _i32), ("reserved", _i32),
        ("x_stride", _i64), ("out_stride", _i64),
        ("x", _vp), ("w_router", _vp), ("w_gate_up", _vp), ("w_down", _vp),
        ("ws_gate_up", _vp), ("ws_down", _vp), ("w_sgate", _vp), ("out", _vp),
        ("topk_idx", _vp), ("topk_w", _vp),
    ]


_lib = None


def declared_functions(header: str = HEADER) -> list[str]:
    """Names of the functions include/gdr.h declares."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdr_[a-z_0-9]+)\s*\(", text)))


def lib(path: str = LIB_PATH) -> ctypes.CDLL:
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build the CUDA library first "
            "(python -m linear_attention_recurrence_10_b200.build)")
    h = ctypes.CDLL(path)
    h.gdr_decode_step.argtypes = [ctypes.POINTER(DecodeArgs), _vp]
    h.gdr_decode_step.restype = ctypes.c_int
    h.gdr_prefill_workspace_size.argtypes = [ctypes.POINTER(PrefillArgs),
                                             ctypes.POINTER(ctypes.c_size_t)]
    h.gdr_prefill_workspace_size.restype = ctypes.c_int
    h.gdr_prefill_chunked.argtypes = [ctypes.POINTER(PrefillArgs), _vp, ctypes.c_size_t, _vp]
    h.gdr_prefill_chunked.restype = ctypes.c_int
    h.gdr_prefill_chunked_noalloc.argtypes = [ctypes.POINTER(PrefillArgs), _vp]
    h.gdr_prefill_chunked_noalloc.restype = ctypes.c_int
    h.gdr_prefill_selftest_wait_expiry.argtypes = [ctypes.POINTER(PrefillArgs), _vp,
                                                   ctypes.c_size_t, ctypes.c_uint64, _vp]
    h.gdr_prefill_selftest_wait_expiry.restype = ctypes.c_int
    h.gdr_prefill_noalloc_status.argtypes = [_vp, _vp]
    h.gdr_prefill_noalloc_status.restype = ctypes.c_int
    h.gdr_decode_multi.argtypes = [ctypes.POINTER(DecodeMultiArgs), _vp]
    h.gdr_decode_multi.restype = ctypes.c_int
    h.gdr_rmsnorm_gated.argtypes = [ctypes.POINTER(NormArgs), _vp]
    h.gdr_rmsnorm_gated.restype = ctypes.c_int
    h.gdr_attn_decode_workspace_size.argtypes = [ctypes.POINTER(AttnDecodeArgs),
                                                 ctypes.POINTER(ctypes.c_size_t)]
    h.gdr_attn_decode_workspace_size.restype = ctypes.c_int
    h.gdr_attn_decode_step.argtypes = [ctypes.POINTER(AttnDecodeArgs), _vp, ctypes.c_size_t, _vp]
    h.gdr_attn_decode_step.restype = ctypes.c_int
    h.gdr_moe_workspace_size.argtypes = [ctypes.POINTER(MoeArgs), ctypes.POINTER(ctypes.c_size_t)]
    h.gdr_moe_workspace_size.restype = ctypes.c_int
    h.gdr_moe_decode.argtypes = [ctypes.POINTER(MoeArgs), _vp, ctypes.c_size_t, _vp]
    h.gdr_moe_decode.restype = ctypes.c_int
    h.gdr_status_string.argtypes = [ctypes.c_int]
    h.gdr_status_string.restype = ctypes.c_char_p
    h.gdr_version.argtypes = []
    h.gdr_version.restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = h
    return h
