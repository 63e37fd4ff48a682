"""ctypes front end of the fp64 CPU oracle for the Gated DeltaNet mixer.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the CPU-baseline
leg of the benchmark call this module; the product path never does.  It shares
no code with the CUDA library (it does not import the package), and everything
it computes is double precision on the host.

The arithmetic lives in ``gdr_oracle.c`` next to this file.  What it computes is
the gated delta rule named in the Qwen3.5 Chat guide (soniqo.audio, section
"Architektur") and on the Core AI Qwen3.6-35B-A3B card (GVA, first section):

    S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t
    y_t = RMSNorm(o_t) * w * SiLU(z_t)

with the published definition of "Gated Delta Networks" (Yang, Kautz,
Hatamizadeh, ICLR 2025).  Arrays are numpy float64 in the packed layout:

    q, k  [n_tok, H_k, d_k]     v, z  [n_tok, H_v, d_v]     g, beta  [n_tok, H_v]
    cu_seqlens [n_seq + 1] (int)  s0 [n_seq, H_v, d_v, d_k] or None   w [d_v] or None
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
# The gated full-attention decode step (the other mixer of the hybrid decoder).
_SRC_ATTN = os.path.join(_HERE, "gattn_oracle.c")
# The routed-expert MoE feed-forward block.
_SRC_MOE = os.path.join(_HERE, "moe_oracle.c")


def _host_key() -> str:
    """A short key of this host's CPU model and flags: the oracle is compiled
    with -march=native, so a build is only reused on the CPU it was made for."""
    import hashlib
    import platform
    text = platform.machine()
    try:
        with open("/proc/cpuinfo") as f:
            lines = [l for l in f if l.startswith(("model name", "flags", "Features"))]
        text += "".join(sorted(set(lines)))
    except OSError:
        pass
    return hashlib.sha256(text.encode()).hexdigest()[:12]


_LIB = os.path.join(_HERE, "_build", f"liboracle-{_host_key()}.so")

_DP = ctypes.POINTER(ctypes.c_double)


class _Problem(ctypes.Structure):
    _fields_ = [
        ("n_tok", ctypes.c_int64),
        ("n_seq", ctypes.c_int32),
        ("H_k", ctypes.c_int32),
        ("H_v", ctypes.c_int32),
        ("d_k", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("qk_l2norm", ctypes.c_int32),
        ("scale", ctypes.c_double),
        ("eps_l2", ctypes.c_double),
        ("eps_norm", ctypes.c_double),
        ("q", _DP), ("k", _DP), ("v", _DP), ("z", _DP),
        ("g", _DP), ("beta", _DP), ("s0", _DP), ("w", _DP),
        ("cu_seqlens", ctypes.POINTER(ctypes.c_int64)),
    ]


class _AttnProblem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("H_q", ctypes.c_int32), ("H_kv", ctypes.c_int32),
        ("d", ctypes.c_int32), ("rot_dim", ctypes.c_int32), ("max_len", ctypes.c_int32),
        ("theta", ctypes.c_double), ("scale", ctypes.c_double),
        ("q", _DP), ("gate", _DP), ("k", _DP), ("v", _DP),
        ("k_cache", _DP), ("v_cache", _DP),
        ("cache_len", ctypes.POINTER(ctypes.c_int64)),
    ]


class _MoeProblem(ctypes.Structure):
    _fields_ = [
        ("n_tok", ctypes.c_int32), ("hidden", ctypes.c_int32), ("n_exp", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("inter", ctypes.c_int32), ("s_inter", ctypes.c_int32),
        ("x", _DP), ("w_router", _DP), ("w_gate", _DP), ("w_up", _DP), ("w_down", _DP),
        ("ws_gate", _DP), ("ws_up", _DP), ("ws_down", _DP), ("w_sgate", _DP),
    ]


def build(src: str = _SRC, out: str = _LIB, force: bool = False, werror: bool = True,
          attn_src: str = _SRC_ATTN, moe_src: str = _SRC_MOE) -> str:
    """Compile the oracle with the host C compiler: -O3 -march=native, ISO C11 (so
    no floating-point contraction or reassociation: the same arithmetic as any
    other build, only faster).  The file name carries the host's CPU key."""
    srcs = [src, attn_src, moe_src]
    if not force and os.path.exists(out) and all(
            os.path.getmtime(out) >= os.path.getmtime(f) for f in srcs):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(
        ["gcc", "-std=c11", "-O3", "-march=native", "-ffp-contract=off", "-fPIC", "-shared",
         "-Wall", "-Wextra"]
        + (["-Werror"] if werror else []) + ["-o", tmp, *srcs, "-lm", "-lpthread"],
        check=True,
    )
    os.replace(tmp, out)
    return out


_lib_cache: dict[str, ctypes.CDLL] = {}


def load(path: str | None = None) -> ctypes.CDLL:
    """Load (building first if needed) the oracle library; ``path`` selects a
    specific build, which the mutation tests use."""
    path = path or build()
    if path in _lib_cache:
        return _lib_cache[path]
    lib = ctypes.CDLL(path)
    pp = ctypes.POINTER(_Problem)
    lib.orc_gdr_recurrent.argtypes = [pp, _DP, _DP, _DP, ctypes.c_int]
    lib.orc_gdr_recurrent.restype = ctypes.c_int
    lib.orc_gdr_chunked.argtypes = [pp, ctypes.c_int, _DP, _DP, _DP, ctypes.c_int]
    lib.orc_gdr_chunked.restype = ctypes.c_int
    lib.orc_gdr_bruteforce.argtypes = [pp, _DP, _DP, _DP]
    lib.orc_gdr_bruteforce.restype = ctypes.c_int
    lib.orc_rmsnorm_gated.argtypes = [_DP, _DP, _DP, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_double, _DP]
    lib.orc_rmsnorm_gated.restype = None
    lib.orc_gate_from_raw.argtypes = [ctypes.c_int64, ctypes.c_int, _DP, _DP, _DP, _DP, _DP, _DP]
    lib.orc_gate_from_raw.restype = None
    lib.orc_rope_partial.argtypes = [_DP, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_double, ctypes.c_double, _DP]
    lib.orc_rope_partial.restype = None
    lib.orc_gated_attn_decode.argtypes = [ctypes.POINTER(_AttnProblem), _DP, _DP, _DP]
    lib.orc_gated_attn_decode.restype = ctypes.c_int
    ip = ctypes.POINTER(ctypes.c_int32)
    lib.orc_moe_route.argtypes = [ctypes.POINTER(_MoeProblem), _DP, ip, _DP]
    lib.orc_moe_route.restype = None
    lib.orc_moe_forward.argtypes = [ctypes.POINTER(_MoeProblem), ip, _DP, _DP]
    lib.orc_moe_forward.restype = ctypes.c_int
    _lib_cache[path] = lib
    return lib


def _f64(a, shape=None):
    if a is None:
        return None
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"expected shape {tuple(shape)}, got {a.shape}")
    return a


def _ptr(a):
    return a.ctypes.data_as(_DP) if a is not None else None


@dataclass
class Result:
    o: np.ndarray            # [n_tok, H_v, d_v] before the output gate
    y: np.ndarray | None     # [n_tok, H_v, d_v] after RMSNormGated (None without z)
    state: np.ndarray        # [n_seq, H_v, d_v, d_k] state after each sequence


def _problem(q, k, v, g, beta, cu_seqlens, z, s0, w, scale, eps_l2, eps_norm, qk_l2norm):
    q = _f64(q); k = _f64(k); v = _f64(v)
    if q.ndim != 3 or k.shape != q.shape or v.ndim != 3:
        raise ValueError("q, k must be [n_tok, H_k, d_k] and v [n_tok, H_v, d_v]")
    n_tok, H_k, d_k = q.shape
    _, H_v, d_v = v.shape
    if v.shape[0] != n_tok or H_v % H_k:
        raise ValueError("token counts differ or H_v is not a multiple of H_k")
    g = _f64(g, (n_tok, H_v)); beta = _f64(beta, (n_tok, H_v))
    z = _f64(z, (n_tok, H_v, d_v)) if z is not None else None
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    n_seq = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != n_tok or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must rise from 0 to n_tok")
    s0 = _f64(s0, (n_seq, H_v, d_v, d_k)) if s0 is not None else None
    w = _f64(w, (d_v,)) if w is not None else None
    keep = (q, k, v, z, g, beta, s0, w, cu)
    p = _Problem(n_tok, n_seq, H_k, H_v, d_k, d_v, int(bool(qk_l2norm)), float(scale),
                 float(eps_l2), float(eps_norm), _ptr(q), _ptr(k), _ptr(v), _ptr(z),
                 _ptr(g), _ptr(beta), _ptr(s0), _ptr(w),
                 cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
    return p, keep, (n_tok, n_seq, H_v, d_v, d_k)


def _outputs(dims, want_y):
    n_tok, n_seq, H_v, d_v, d_k = dims
    o = np.zeros((n_tok, H_v, d_v))
    y = np.zeros((n_tok, H_v, d_v)) if want_y else None
    s = np.zeros((n_seq, H_v, d_v, d_k))
    return o, y, s


def gdr_recurrent(q, k, v, g, beta, cu_seqlens, *, z=None, s0=None, w=None, scale=1.0,
                  eps_l2=1e-6, eps_norm=1e-6, qk_l2norm=True, threads=1,
                  lib: ctypes.CDLL | None = None) -> Result:
    """The definition, token by token, for every (sequence, value head)."""
    p, keep, dims = _problem(q, k, v, g, beta, cu_seqlens, z, s0, w, scale, eps_l2,
                             eps_norm, qk_l2norm)
    o, y, s = _outputs(dims, z is not None)
    (lib or load()).orc_gdr_recurrent(ctypes.byref(p), _ptr(o), _ptr(y), _ptr(s), int(threads))
    del keep
    return Result(o, y, s)


def gdr_chunked(q, k, v, g, beta, cu_seqlens, *, chunk, z=None, s0=None, w=None,
                scale=1.0, eps_l2=1e-6, eps_norm=1e-6, qk_l2norm=True, threads=1,
                lib: ctypes.CDLL | None = None) -> Result:
    """The chunkwise (WY / UT transform) form with chunks of ``chunk`` tokens."""
    p, keep, dims = _problem(q, k, v, g, beta, cu_seqlens, z, s0, w, scale, eps_l2,
                             eps_norm, qk_l2norm)
    o, y, s = _outputs(dims, z is not None)
    rc = (lib or load()).orc_gdr_chunked(ctypes.byref(p), int(chunk), _ptr(o), _ptr(y),
                                         _ptr(s), int(threads))
    if rc:
        raise ValueError("chunk must be >= 1")
    del keep
    return Result(o, y, s)


def gdr_bruteforce(q, k, v, g, beta, cu_seqlens, *, z=None, s0=None, w=None, scale=1.0,
                   eps_l2=1e-6, eps_norm=1e-6, qk_l2norm=True,
                   lib: ctypes.CDLL | None = None) -> Result:
    """Explicit transition matrices multiplied out; every sequence at most 8 tokens."""
    p, keep, dims = _problem(q, k, v, g, beta, cu_seqlens, z, s0, w, scale, eps_l2,
                             eps_norm, qk_l2norm)
    o, y, s = _outputs(dims, z is not None)
    rc = (lib or load()).orc_gdr_bruteforce(ctypes.byref(p), _ptr(o), _ptr(y), _ptr(s))
    if rc:
        raise ValueError("brute force takes sequences of at most 8 tokens")
    del keep
    return Result(o, y, s)


def gate_from_raw(a, b, A_log, dt_bias, lib: ctypes.CDLL | None = None):
    """(g, beta) from raw per-token gate projections a, b [n_tok, H_v] and the
    per-head A_log, dt_bias [H_v]: g = -exp(A_log) softplus(a + dt_bias),
    beta = sigmoid(b)."""
    a = _f64(a)
    b = _f64(b, a.shape)
    n_tok, H_v = a.shape
    A_log = _f64(A_log, (H_v,))
    dt_bias = _f64(dt_bias, (H_v,))
    g = np.zeros_like(a)
    beta = np.zeros_like(a)
    (lib or load()).orc_gate_from_raw(ctypes.c_int64(n_tok), int(H_v), _ptr(a), _ptr(b),
                                      _ptr(A_log), _ptr(dt_bias), _ptr(g), _ptr(beta))
    return g, beta


def rmsnorm_gated(o, z, w=None, eps=1e-6, lib: ctypes.CDLL | None = None) -> np.ndarray:
    """y = o / sqrt(mean(o^2) + eps) * w * z * sigmoid(z) over the last axis."""
    o = _f64(o); z = _f64(z, o.shape)
    n = o.shape[-1]
    w = _f64(w, (n,)) if w is not None else None
    y = np.zeros_like(o)
    (lib or load()).orc_rmsnorm_gated(_ptr(o), _ptr(z), _ptr(w), o.size // n, n, float(eps),
                                      _ptr(y))
    return y


# ----------------------------------------------------- gated full attention

def rope_partial(x, pos, rot_dim, theta=1e7, lib: ctypes.CDLL | None = None) -> np.ndarray:
    """Rotary embedding of the first rot_dim dims of every row of x [..., d] at
    one position ("rotate half" pairing: dim i with dim i + rot_dim/2)."""
    x = _f64(x)
    d = x.shape[-1]
    out = np.zeros_like(x)
    (lib or load()).orc_rope_partial(_ptr(x), x.size // d, d, int(rot_dim), float(pos),
                                     float(theta), _ptr(out))
    return out


@dataclass
class AttnResult:
    y: np.ndarray        # [batch, H_q, d] after the output gate
    o: np.ndarray        # [batch, H_q, d] attention output before the gate
    k_rot: np.ndarray    # [batch, H_kv, d] rotated key appended at index cache_len[b]


def gated_attn_decode(q, gate, k, v, k_cache, v_cache, cache_len, *, rot_dim, theta=1e7,
                      scale=None, lib: ctypes.CDLL | None = None) -> AttnResult:
    """One decode step of the gated full-attention layer for every sequence:
    q, gate [B, H_q, d]; k, v [B, H_kv, d] (the new token); k_cache, v_cache
    [B, H_kv, max_len, d] with cache_len[b] valid entries; scale defaults to
    d^-1/2."""
    q = _f64(q); gate = _f64(gate, q.shape); k = _f64(k); v = _f64(v, k.shape)
    B, H_q, d = q.shape
    H_kv = k.shape[1]
    k_cache = _f64(k_cache); v_cache = _f64(v_cache, k_cache.shape)
    if k_cache.shape[:2] != (B, H_kv) or k_cache.shape[3] != d:
        raise ValueError("k_cache must be [B, H_kv, max_len, d]")
    cl = np.ascontiguousarray(np.asarray(cache_len, dtype=np.int64))
    p = _AttnProblem(B, H_q, H_kv, d, int(rot_dim), k_cache.shape[2], float(theta),
                     float(d ** -0.5 if scale is None else scale), _ptr(q), _ptr(gate), _ptr(k),
                     _ptr(v), _ptr(k_cache), _ptr(v_cache),
                     cl.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)))
    y = np.zeros((B, H_q, d)); o = np.zeros((B, H_q, d)); kr = np.zeros((B, H_kv, d))
    if (lib or load()).orc_gated_attn_decode(ctypes.byref(p), _ptr(y), _ptr(o), _ptr(kr)):
        raise ValueError("invalid shape or a full cache")
    return AttnResult(y, o, kr)


# ------------------------------------------------------- routed-expert MoE

@dataclass
class MoeRoute:
    probs: np.ndarray    # [n_tok, n_exp] softmax of the router logits
    idx: np.ndarray      # [n_tok, top_k] int32, experts in decreasing probability
    w: np.ndarray        # [n_tok, top_k] renormalised weights


def _moe_problem(x, w_router, w_gate, w_up, w_down, top_k, shared):
    x = _f64(x)
    n_tok, H = x.shape
    w_router = _f64(w_router)
    E = w_router.shape[0]
    w_gate = _f64(w_gate); w_up = _f64(w_up, w_gate.shape)
    I = w_gate.shape[1]
    w_down = _f64(w_down, (E, H, I))
    if shared is not None:
        ws_gate, ws_up, ws_down, w_sgate = (_f64(a) for a in shared)
        SI = ws_gate.shape[0]
    else:
        ws_gate = ws_up = ws_down = w_sgate = None
        SI = 0
    keep = (x, w_router, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, w_sgate)
    p = _MoeProblem(n_tok, H, E, int(top_k), I, SI, _ptr(x), _ptr(w_router), _ptr(w_gate),
                    _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down),
                    _ptr(w_sgate))
    return p, keep, (n_tok, H, E)


def moe_route(x, w_router, top_k, lib: ctypes.CDLL | None = None) -> MoeRoute:
    """Router probabilities, top-k experts and renormalised weights per token."""
    E, H = np.shape(w_router)
    dummy = np.zeros((E, 1, H))
    p, keep, (n_tok, H, E) = _moe_problem(x, w_router, dummy, dummy, np.zeros((E, H, 1)),
                                          top_k, None)
    probs = np.zeros((n_tok, E)); w = np.zeros((n_tok, top_k))
    idx = np.zeros((n_tok, top_k), dtype=np.int32)
    (lib or load()).orc_moe_route(ctypes.byref(p), _ptr(probs),
                                  idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), _ptr(w))
    del keep
    return MoeRoute(probs, idx, w)


def moe_forward(x, w_router, w_gate, w_up, w_down, idx, w, *, shared=None,
                lib: ctypes.CDLL | None = None) -> np.ndarray:
    """The MoE block's output [n_tok, hidden] for the routing (idx, w):
    sum_k w_k SwitchGLU_{idx_k}(x) + sigmoid(w_sgate . x) SwitchGLU_shared(x);
    shared = (ws_gate, ws_up, ws_down, w_sgate) or None."""
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    w = _f64(w, idx.shape)
    p, keep, (n_tok, H, E) = _moe_problem(x, w_router, w_gate, w_up, w_down, idx.shape[1], shared)
    y = np.zeros((n_tok, H))
    if (lib or load()).orc_moe_forward(ctypes.byref(p),
                                       idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                       _ptr(w), _ptr(y)):
        raise ValueError("expert index out of range")
    del keep
    return y
