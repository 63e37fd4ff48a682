"""Gated DeltaNet (gated delta rule) token mixer for B200 -- Python binding.

Thin wrappers over the C ABI of include/gdr.h (libgdr.so, built in-tree by
``python -m linear_attention_recurrence_10_b200.build``).  Each wrapper only
turns torch tensors into pointers, strides and dtype codes and passes the
current CUDA stream; every step of the computation runs in the library's
kernels.  PyTorch is used for device memory and streams only.

    decode_step(q, k, v, g, beta, state, out, ...)        one token per sequence
    prefill_chunked(q, k, v, g, beta, cu_seqlens, out, ...)  packed varlen prompts
    rmsnorm_gated(o, z, out, ...)                          the output gate alone
    attn_decode_step(q, gate, k, v, k_cache, v_cache, cache_len, out, ...)
                                                           gated full-attention decode
    moe_decode(x, w_router, w_gate_up, w_down, out, ...)    routed-expert MoE block
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import GDR_BF16, GDR_F32

__all__ = ["GdrError", "decode_step", "decode_multi", "prefill_chunked", "prefill_chunked_noalloc",
           "prefill_noalloc_status", "prefill_workspace_size", "attn_decode_step",
           "attn_decode_workspace_size", "moe_decode", "moe_workspace_size",
           "rmsnorm_gated", "version", "status_string"]


class GdrError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        name = _abi.STATUS_NAMES.get(self.status, f"status {status}")
        super().__init__(f"{where}: {name}")


def _check(status: int, where: str):
    if status != 0:
        raise GdrError(status, where)


def _dtype_code(t: torch.Tensor, what: str) -> int:
    if t.dtype == torch.bfloat16:
        return GDR_BF16
    if t.dtype == torch.float32:
        return GDR_F32
    raise TypeError(f"{what}: dtype {t.dtype} is not bf16 or fp32")


def _ptr(t):
    # A plain int: every pointer field and argument is declared void* (c_void_p).
    return None if t is None else t.data_ptr()


def _row_stride(t: torch.Tensor, what: str) -> int:
    """Row stride of a [rows, H, d] (or [rows, d]) tensor whose inner dims are packed."""
    if t.is_contiguous():
        return t.stride(0) if t.shape[0] > 1 else 0
    if t.dim() >= 2:
        inner = 1
        for size, stride in zip(reversed(t.shape[1:]), reversed(t.stride()[1:])):
            if size > 1 and stride != inner:
                raise ValueError(f"{what}: inner dimensions must be contiguous")
            inner *= size
    return int(t.stride(0)) if t.shape[0] > 1 else 0


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _f32_tensor(t, what):
    if t is not None and t.dtype != torch.float32:
        raise TypeError(f"{what} must be fp32")
    return t


def version() -> int:
    return _abi.lib().gdr_version()


def status_string(status: int) -> str:
    return _abi.lib().gdr_status_string(int(status)).decode()


def _gate_params(gate_params, H_v):
    """(A_log, dt_bias) fp32 [H_v] tensors, or None: see GDR_GATE_FROM_RAW."""
    if gate_params is None:
        return None, None
    A_log, dt_bias = gate_params
    for t, name in ((A_log, "A_log"), (dt_bias, "dt_bias")):
        _f32_tensor(t, name)
        if t.dim() != 1 or t.shape[0] != H_v or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous fp32 tensor of H_v entries")
    return A_log, dt_bias


def _decode_args(q, k, v, g, beta, state, out, z, norm_w, state_out, scale, eps_l2, eps_norm,
                 qk_l2norm, overlap_state_load, batch, gate_params=None):
    H_k, d = q.shape[1], q.shape[2]
    H_v = v.shape[1]
    for t, name in ((g, "g"), (beta, "beta"), (state, "state"), (norm_w, "norm_w")):
        _f32_tensor(t, name)
    if g.stride() != beta.stride():
        raise ValueError("g and beta must share one layout")
    so = state if state_out is None else _f32_tensor(state_out, "state_out")
    if state.stride() != so.stride():
        raise ValueError("state and state_out must share one layout")
    in_dtype = _dtype_code(q, "q")
    for t, name in ((k, "k"), (v, "v"), (z, "z")):
        if t is not None and _dtype_code(t, name) != in_dtype:
            raise TypeError(f"{name} must have the dtype of q")
    flags = _abi.GDR_DECODE_OVERLAP_STATE_LOAD if overlap_state_load else 0
    A_log, dt_bias = _gate_params(gate_params, H_v)
    if A_log is not None:
        flags |= _abi.GDR_GATE_FROM_RAW
    # One constructor call: ctypes fills the fields in C, a third of the cost of
    # assigning them one by one (this runs on every decode call).
    return _abi.DecodeArgs(
        batch=batch, H_k=H_k, H_v=H_v, d_k=d, d_v=v.shape[2],
        in_dtype=in_dtype, out_dtype=_dtype_code(out, "out"), qk_l2norm=int(bool(qk_l2norm)),
        scale=float(scale), eps_l2=float(eps_l2), eps_norm=float(eps_norm), flags=flags,
        q_stride=_row_stride(q, "q"), k_stride=_row_stride(k, "k"), v_stride=_row_stride(v, "v"),
        z_stride=_row_stride(z, "z") if z is not None else 0, gb_stride=_row_stride(g, "g"),
        out_stride=_row_stride(out, "out"), state_stride=_row_stride(state, "state"),
        q=_ptr(q), k=_ptr(k), v=_ptr(v), z=_ptr(z), g=_ptr(g), beta=_ptr(beta),
        state_in=_ptr(state), state_out=_ptr(so), norm_w=_ptr(norm_w), out=_ptr(out),
        A_log=_ptr(A_log), dt_bias=_ptr(dt_bias))


def decode_step(q, k, v, g, beta, state, out, *, z=None, norm_w=None, state_out=None,
                scale: float = 1.0, eps_l2: float = 1e-6, eps_norm: float = 1e-6,
                qk_l2norm: bool = True, overlap_state_load: bool = False,
                gate_params=None, stream=None) -> torch.Tensor:
    """Advance every sequence of the batch by one token (gdr_decode_step).

    q, k [B, H_k, d]; v, z [B, H_v, d] (bf16 or fp32, same dtype); g, beta
    [B, H_v] fp32; state [B, H_v, d, d] fp32, updated in place unless
    ``state_out`` is given; out [B, H_v, d] bf16 or fp32.  Batch rows may be
    strided views (e.g. one step of a [B, T, H, d] tensor).
    ``overlap_state_load``: GDR_DECODE_OVERLAP_STATE_LOAD -- only when the
    kernel queued just before this call does not write this state.
    ``gate_params`` = (A_log, dt_bias), fp32 [H_v]: g and beta then hold the
    raw projections a, b (GDR_GATE_FROM_RAW).
    """
    a = _decode_args(q, k, v, g, beta, state, out, z, norm_w, state_out, scale, eps_l2, eps_norm,
                     qk_l2norm, overlap_state_load, q.shape[0], gate_params)
    _check(_abi.lib().gdr_decode_step(ctypes.byref(a), _stream(stream, q.device)),
           "gdr_decode_step")
    return out


def decode_multi(q, k, v, g, beta, state, out, *, n_tokens: int, z=None, norm_w=None,
                 state_out=None, slots=None, status=None, scale: float = 1.0,
                 eps_l2: float = 1e-6, eps_norm: float = 1e-6, qk_l2norm: bool = True,
                 overlap_state_load: bool = False, gate_params=None,
                 stream=None) -> torch.Tensor:
    """Advance every sequence by ``n_tokens`` tokens in one call (gdr_decode_multi).

    Token-indexed tensors hold B * n_tokens rows, row b * n_tokens + t being
    token t of sequence b: q, k [B*T, H_k, d]; v, z [B*T, H_v, d]; g, beta
    [B*T, H_v]; out [B*T, H_v, d].  ``slots`` (int32 [B] on the device, or
    None) maps sequence b to its row of ``state`` [n_rows, H_v, d, d];
    ``status`` (int32 [1] on the device) receives GDR_ERR_INVALID_ARG if a
    slot is out of range.
    """
    rows = q.shape[0]
    if n_tokens < 1 or rows % n_tokens != 0:
        raise ValueError("q must hold batch * n_tokens rows")
    batch = rows // n_tokens
    a = _decode_args(q, k, v, g, beta, state, out, z, norm_w, state_out, scale, eps_l2, eps_norm,
                     qk_l2norm, overlap_state_load, batch, gate_params)
    m = _abi.DecodeMultiArgs()
    m.base = a
    m.n_tokens = int(n_tokens)
    m.n_slots = 0
    if slots is not None:
        if slots.dtype != torch.int32 or slots.dim() != 1 or slots.shape[0] != batch:
            raise ValueError("slots must be an int32 tensor of one entry per sequence")
        m.n_slots = state.shape[0]
    m.state_slot = _ptr(slots)
    m.status = _ptr(status)
    _check(_abi.lib().gdr_decode_multi(ctypes.byref(m), _stream(stream, q.device)),
           "gdr_decode_multi")
    return out


def _prefill_args(q, k, v, g, beta, cu_seqlens, out, cu_seqlens_host, z, norm_w,
                  initial_state, final_state, chunk, scale, eps_l2, eps_norm, qk_l2norm,
                  gate_params=None):
    n_tok, H_k, d = q.shape
    H_v = v.shape[1]
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if cu_seqlens_host is None:
        cu_seqlens_host = cu_seqlens.cpu()
    host = (ctypes.c_int32 * len(cu_seqlens_host))(*[int(x) for x in cu_seqlens_host])
    for t, name in ((g, "g"), (beta, "beta"), (initial_state, "initial_state"),
                    (final_state, "final_state"), (norm_w, "norm_w")):
        _f32_tensor(t, name)
    if g.stride() != beta.stride():
        raise ValueError("g and beta must share one layout")
    a = _abi.PrefillArgs()
    a.n_seq = len(cu_seqlens_host) - 1
    a.H_k, a.H_v, a.d_k, a.d_v = H_k, H_v, d, v.shape[2]
    a.chunk = int(chunk)
    a.in_dtype = _dtype_code(q, "q")
    for t, name in ((k, "k"), (v, "v"), (z, "z")):
        if t is not None and _dtype_code(t, name) != a.in_dtype:
            raise TypeError(f"{name} must have the dtype of q")
    a.out_dtype = _dtype_code(out, "out")
    a.qk_l2norm = int(bool(qk_l2norm))
    a.scale, a.eps_l2, a.eps_norm = float(scale), float(eps_l2), float(eps_norm)
    a.n_tok = n_tok
    a.q_stride, a.k_stride = _row_stride(q, "q"), _row_stride(k, "k")
    a.v_stride = _row_stride(v, "v")
    a.z_stride = _row_stride(z, "z") if z is not None else 0
    a.gb_stride = _row_stride(g, "g")
    a.out_stride = _row_stride(out, "out")
    a.q, a.k, a.v, a.z = _ptr(q), _ptr(k), _ptr(v), _ptr(z)
    a.g, a.beta = _ptr(g), _ptr(beta)
    a.cu_seqlens = _ptr(cu_seqlens)
    a.cu_seqlens_host = ctypes.cast(host, ctypes.POINTER(ctypes.c_int32))
    a.initial_state, a.final_state = _ptr(initial_state), _ptr(final_state)
    a.norm_w, a.out = _ptr(norm_w), _ptr(out)
    A_log, dt_bias = _gate_params(gate_params, H_v)
    if A_log is not None:
        a.flags = _abi.GDR_GATE_FROM_RAW
        a.A_log, a.dt_bias = _ptr(A_log), _ptr(dt_bias)
    return a, host


def prefill_workspace_size(q, k, v, g, beta, cu_seqlens, out, *, cu_seqlens_host=None,
                           z=None, chunk: int = 0, **_) -> int:
    a, host = _prefill_args(q, k, v, g, beta, cu_seqlens, out, cu_seqlens_host, z, None, None,
                            None, chunk, 1.0, 1e-6, 1e-6, True)
    n = ctypes.c_size_t(0)
    _check(_abi.lib().gdr_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)),
           "gdr_prefill_workspace_size")
    del host
    return int(n.value)


def prefill_chunked(q, k, v, g, beta, cu_seqlens, out, *, cu_seqlens_host=None, z=None,
                    norm_w=None, initial_state=None, final_state=None, chunk: int = 0,
                    workspace=None, scale: float = 1.0, eps_l2: float = 1e-6,
                    eps_norm: float = 1e-6, qk_l2norm: bool = True, gate_params=None,
                    stream=None) -> torch.Tensor:
    """Chunked prefill of packed variable-length sequences (gdr_prefill_chunked).

    q, k [n_tok, H_k, d]; v, z, out [n_tok, H_v, d]; g, beta [n_tok, H_v] fp32;
    cu_seqlens int32 [n_seq + 1] on the device (``cu_seqlens_host``: the same
    values on the host, read during the call); initial_state / final_state
    [n_seq, H_v, d, d] fp32 or None.  ``workspace``: a uint8 device tensor of
    at least prefill_workspace_size() bytes; allocated here when None.
    ``gate_params`` = (A_log, dt_bias), fp32 [H_v]: g and beta then hold the
    raw projections a, b (GDR_GATE_FROM_RAW).
    """
    a, host = _prefill_args(q, k, v, g, beta, cu_seqlens, out, cu_seqlens_host, z, norm_w,
                            initial_state, final_state, chunk, scale, eps_l2, eps_norm,
                            qk_l2norm, gate_params)
    L = _abi.lib()
    n = ctypes.c_size_t(0)
    _check(L.gdr_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)),
           "gdr_prefill_workspace_size")
    if workspace is None and n.value:
        workspace = torch.empty(int(n.value), dtype=torch.uint8, device=q.device)
    ws_ptr = _ptr(workspace)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(L.gdr_prefill_chunked(ctypes.byref(a), ws_ptr, ws_bytes, _stream(stream, q.device)),
           "gdr_prefill_chunked")
    del host
    return out


def prefill_chunked_noalloc(q, k, v, g, beta, cu_seqlens, out, *, cu_seqlens_host=None,
                            z=None, norm_w=None, initial_state=None, final_state=None,
                            chunk: int = 0, scale: float = 1.0, eps_l2: float = 1e-6,
                            eps_norm: float = 1e-6, qk_l2norm: bool = True, gate_params=None,
                            stream=None) -> torch.Tensor:
    """gdr_prefill_chunked_noalloc: the same prefill, with no workspace to pass and
    nothing allocated -- for callers that cannot allocate device memory here.
    At most 4096 sequences per call; calls must not overlap on the GPU (they
    share one scratch array per device).  Arguments as prefill_chunked."""
    a, host = _prefill_args(q, k, v, g, beta, cu_seqlens, out, cu_seqlens_host, z, norm_w,
                            initial_state, final_state, chunk, scale, eps_l2, eps_norm,
                            qk_l2norm, gate_params)
    _check(_abi.lib().gdr_prefill_chunked_noalloc(ctypes.byref(a), _stream(stream, q.device)),
           "gdr_prefill_chunked_noalloc")
    del host
    return out


def prefill_noalloc_status(stream=None) -> int:
    """The status word of the last prefill_chunked_noalloc call on the current
    device (gdr_prefill_noalloc_status): 0, or GDR_ERR_TIMEOUT if a bounded
    device wait gave up.  ``stream``: a torch CUDA stream (default: the current
    one), which is synchronised, since the value is read back to the host."""
    s = stream if stream is not None else torch.cuda.current_stream()
    host = torch.zeros(1, dtype=torch.int32).pin_memory()
    _check(_abi.lib().gdr_prefill_noalloc_status(host.data_ptr(), ctypes.c_void_p(s.cuda_stream)),
           "gdr_prefill_noalloc_status")
    s.synchronize()
    return int(host.item())


def rmsnorm_gated(o, z, out, *, w=None, eps: float = 1e-6, stream=None) -> torch.Tensor:
    """y = o / sqrt(mean(o^2) + eps) * w * z * sigmoid(z) over the last dim (gdr_rmsnorm_gated).

    o, z, out: [..., d] with packed rows; w [d] fp32 or None."""
    d = o.shape[-1]
    o2, z2, out2 = o.reshape(-1, d), z.reshape(-1, d), out.reshape(-1, d)
    if out2.data_ptr() != out.data_ptr():
        raise ValueError("out must be viewable as [rows, d]")
    _f32_tensor(w, "w")
    a = _abi.NormArgs()
    a.rows, a.d = o2.shape[0], d
    a.o_dtype, a.z_dtype = _dtype_code(o, "o"), _dtype_code(z, "z")
    a.out_dtype = _dtype_code(out, "out")
    a.eps = float(eps)
    a.o_stride, a.z_stride = _row_stride(o2, "o"), _row_stride(z2, "z")
    a.out_stride = _row_stride(out2, "out")
    a.o, a.z, a.w, a.out = _ptr(o2), _ptr(z2), _ptr(w), _ptr(out2)
    _check(_abi.lib().gdr_rmsnorm_gated(ctypes.byref(a), _stream(stream, o.device)),
           "gdr_rmsnorm_gated")
    return out


def _attn_args(q, gate, k, v, k_cache, v_cache, cache_len, out, kv_bound, rot_dim, rope_theta,
               scale):
    B, H_q, d = q.shape
    H_kv = k.shape[1]
    for t, name in ((q, "q"), (gate, "gate"), (k, "k"), (v, "v"), (k_cache, "k_cache"),
                    (v_cache, "v_cache")):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bf16")
    for t, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        if t.dim() != 4 or t.shape[:2] != (B, H_kv) or t.shape[3] != d or not t.is_contiguous():
            raise ValueError(f"{name} must be a packed [batch, H_kv, max_len, d] tensor")
    if cache_len.dtype != torch.int32:
        raise TypeError("cache_len must be int32")
    return _abi.AttnDecodeArgs(
        batch=B, H_q=H_q, H_kv=H_kv, d=d, rot_dim=int(rot_dim), max_len=k_cache.shape[2],
        kv_bound=int(kv_bound), out_dtype=_dtype_code(out, "out"), rope_theta=float(rope_theta),
        scale=float(d ** -0.5 if scale is None else scale),
        q_stride=_row_stride(q, "q"), gate_stride=_row_stride(gate, "gate"),
        k_stride=_row_stride(k, "k"), v_stride=_row_stride(v, "v"),
        out_stride=_row_stride(out, "out"), q=_ptr(q), gate=_ptr(gate), k=_ptr(k), v=_ptr(v),
        k_cache=_ptr(k_cache), v_cache=_ptr(v_cache), cache_len=_ptr(cache_len), out=_ptr(out))


def attn_decode_workspace_size(q, gate, k, v, k_cache, v_cache, cache_len, out, *, kv_bound,
                               rot_dim=64, rope_theta=1e7, scale=None) -> int:
    a = _attn_args(q, gate, k, v, k_cache, v_cache, cache_len, out, kv_bound, rot_dim,
                   rope_theta, scale)
    n = ctypes.c_size_t(0)
    _check(_abi.lib().gdr_attn_decode_workspace_size(ctypes.byref(a), ctypes.byref(n)),
           "gdr_attn_decode_workspace_size")
    return int(n.value)


def attn_decode_step(q, gate, k, v, k_cache, v_cache, cache_len, out, *, kv_bound, rot_dim=64,
                     rope_theta=1e7, scale=None, workspace=None, stream=None) -> torch.Tensor:
    """One decode step of the gated full-attention layer (gdr_attn_decode_step).

    q, gate [B, H_q, 256]; k, v [B, H_kv, 256] (the new token, bf16);
    k_cache, v_cache [B, H_kv, max_len, 256] bf16 (row cache_len[b] receives the
    rotated key and the value); cache_len int32 [B] on the device; ``kv_bound``
    an upper bound of cache_len on the host; out [B, H_q, 256] bf16 or fp32.
    ``workspace``: a uint8 device tensor of attn_decode_workspace_size() bytes,
    allocated here when None.
    """
    a = _attn_args(q, gate, k, v, k_cache, v_cache, cache_len, out, kv_bound, rot_dim,
                   rope_theta, scale)
    L = _abi.lib()
    n = ctypes.c_size_t(0)
    _check(L.gdr_attn_decode_workspace_size(ctypes.byref(a), ctypes.byref(n)),
           "gdr_attn_decode_workspace_size")
    if workspace is None and n.value:
        workspace = torch.empty(int(n.value), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(L.gdr_attn_decode_step(ctypes.byref(a), _ptr(workspace), ws_bytes,
                                  _stream(stream, q.device)), "gdr_attn_decode_step")
    return out


def _moe_args(x, w_router, w_gate_up, w_down, out, top_k, shared, topk_idx, topk_w):
    n_tok, H = x.shape
    E = w_router.shape[0]
    I = w_gate_up.shape[1] // 2
    for t, name in ((x, "x"), (w_router, "w_router"), (w_gate_up, "w_gate_up"),
                    (w_down, "w_down")):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bf16")
    for t, name, shape in ((w_router, "w_router", (E, H)), (w_gate_up, "w_gate_up", (E, 2 * I, H)),
                           (w_down, "w_down", (E, H, I))):
        if tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a packed {list(shape)} tensor")
    ws_gate_up = ws_down = w_sgate = None
    SI = 0
    if shared is not None:
        ws_gate_up, ws_down, w_sgate = shared
        SI = ws_gate_up.shape[0] // 2
        for t, name, shape in ((ws_gate_up, "ws_gate_up", (2 * SI, H)), (ws_down, "ws_down", (H, SI)),
                               (w_sgate, "w_sgate", (H,))):
            if t.dtype != torch.bfloat16 or tuple(t.shape) != shape or not t.is_contiguous():
                raise ValueError(f"{name} must be a packed bf16 {list(shape)} tensor")
    if topk_idx is not None and topk_idx.dtype != torch.int32:
        raise TypeError("topk_idx must be int32")
    _f32_tensor(topk_w, "topk_w")
    return _abi.MoeArgs(
        n_tok=n_tok, hidden=H, n_exp=E, top_k=int(top_k), inter=I, s_inter=SI,
        out_dtype=_dtype_code(out, "out"), reserved=0,
        x_stride=_row_stride(x, "x"), out_stride=_row_stride(out, "out"),
        x=_ptr(x), w_router=_ptr(w_router), w_gate_up=_ptr(w_gate_up), w_down=_ptr(w_down),
        ws_gate_up=_ptr(ws_gate_up), ws_down=_ptr(ws_down), w_sgate=_ptr(w_sgate), out=_ptr(out),
        topk_idx=_ptr(topk_idx), topk_w=_ptr(topk_w))


def moe_workspace_size(x, w_router, w_gate_up, w_down, out, *, top_k=8, shared=None) -> int:
    a = _moe_args(x, w_router, w_gate_up, w_down, out, top_k, shared, None, None)
    n = ctypes.c_size_t(0)
    _check(_abi.lib().gdr_moe_workspace_size(ctypes.byref(a), ctypes.byref(n)),
           "gdr_moe_workspace_size")
    return int(n.value)


def moe_decode(x, w_router, w_gate_up, w_down, out, *, top_k=8, shared=None, topk_idx=None,
               topk_w=None, workspace=None, stream=None) -> torch.Tensor:
    """The routed-expert MoE block for a decode batch (gdr_moe_decode).

    x [n_tok, hidden] bf16; w_router [n_exp, hidden]; w_gate_up [n_exp, 2*inter,
    hidden] (gate rows, then up rows); w_down [n_exp, hidden, inter], all bf16;
    ``shared`` = (ws_gate_up [2*s_inter, hidden], ws_down [hidden, s_inter],
    w_sgate [hidden]) bf16 or None; out [n_tok, hidden] bf16 or fp32;
    ``topk_idx`` (int32) / ``topk_w`` (fp32) [n_tok, top_k] receive the routing.
    """
    a = _moe_args(x, w_router, w_gate_up, w_down, out, top_k, shared, topk_idx, topk_w)
    L = _abi.lib()
    n = ctypes.c_size_t(0)
    _check(L.gdr_moe_workspace_size(ctypes.byref(a), ctypes.byref(n)), "gdr_moe_workspace_size")
    if workspace is None and n.value:
        workspace = torch.empty(int(n.value), dtype=torch.uint8, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(L.gdr_moe_decode(ctypes.byref(a), _ptr(workspace), ws_bytes, _stream(stream, x.device)),
           "gdr_moe_decode")
    return out
