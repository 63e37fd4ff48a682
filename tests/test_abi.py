"""The C ABI without a GPU: libgdr.so builds and loads, exports every function
include/gdr.h declares, and rejects bad arguments with the documented status
before queueing anything.

The validation cases pass made-up device addresses that are never
dereferenced on the host.  They are only run where no CUDA device is present,
so that a validation bug can never turn into a kernel launch on made-up
addresses."""
import ctypes
import subprocess

import pytest
import torch

from linear_attention_recurrence_10_b200 import _abi, build

OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA = 0, 1, 2, 3, 4, 5
FAKE = 0x7f0000000000  # 16-byte aligned, never dereferenced on the host

host_only = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="host-only validation with made-up addresses")


@pytest.fixture(scope="module")
def lib():
    build.build(quiet=True)
    return _abi.lib()


def test_exports_every_declared_function(lib):
    declared = _abi.declared_functions()
    assert {"gdr_decode_step", "gdr_prefill_chunked", "gdr_prefill_workspace_size",
            "gdr_rmsnorm_gated", "gdr_status_string", "gdr_version"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [f for f in declared if f not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for f in declared:
        assert hasattr(lib, f)


def test_status_strings(lib):
    for code, name in _abi.STATUS_NAMES.items():
        assert lib.gdr_status_string(code).decode().startswith(name)
    assert lib.gdr_status_string(99).decode().startswith("GDR_ERR_UNKNOWN")
    assert lib.gdr_version() >= 100


def _decode_args(**kw):
    a = _abi.DecodeArgs()
    a.batch, a.H_k, a.H_v, a.d_k, a.d_v = 4, 2, 4, 128, 128
    a.in_dtype, a.out_dtype, a.qk_l2norm = 1, 0, 1
    a.scale, a.eps_l2, a.eps_norm = 1.0, 1e-6, 1e-6
    base = FAKE
    for i, name in enumerate(["q", "k", "v", "z", "g", "beta", "state_in", "state_out",
                              "norm_w", "out"]):
        setattr(a, name, base + (i << 32))
    for k, v in kw.items():
        setattr(a, k, v)
    return a


DECODE_CASES = [
    ("null_q", dict(q=None), INVALID),
    ("null_state", dict(state_in=None), INVALID),
    ("null_out", dict(out=None), INVALID),
    ("negative_batch", dict(batch=-1), INVALID),
    ("unknown_flag", dict(flags=2), INVALID),
    ("bad_in_dtype", dict(in_dtype=7), INVALID),
    ("bad_out_dtype", dict(out_dtype=-1), INVALID),
    ("heads_not_multiple", dict(H_k=3, H_v=4), INVALID),
    ("zero_heads", dict(H_k=0), INVALID),
    ("d96", dict(d_k=96, d_v=96), UNSUPPORTED),
    ("dk_ne_dv", dict(d_k=64, d_v=128), UNSUPPORTED),
    ("misaligned_q", dict(q=FAKE + 8), MISALIGNED),
    ("misaligned_state", dict(state_out=FAKE + (7 << 32) + 4), MISALIGNED),
    ("misaligned_g", dict(g=FAKE + (4 << 32) + 2), MISALIGNED),
    ("stride_too_small", dict(q_stride=128), INVALID),
    ("stride_negative", dict(v_stride=-512), INVALID),
    ("stride_not_16B", dict(q_stride=2 * 128 + 4), MISALIGNED),
    ("state_stride_small", dict(state_stride=128 * 128), INVALID),
    ("gb_stride_small", dict(gb_stride=2), INVALID),
    ("state_partial_overlap", dict(state_out=FAKE + (6 << 32) + 4096), INVALID),
    ("raw_gate_without_params", dict(flags=2), INVALID),
    ("raw_gate_without_dt_bias", dict(flags=2, A_log=FAKE + (13 << 32)), INVALID),
    ("raw_gate_misaligned", dict(flags=2, A_log=FAKE + (13 << 32) + 2,
                                 dt_bias=FAKE + (14 << 32)), MISALIGNED),
    ("unknown_flag_4", dict(flags=4), INVALID),
]


@host_only
@pytest.mark.parametrize("name,kw,want", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_validation(lib, name, kw, want):
    assert lib.gdr_decode_step(ctypes.byref(_decode_args(**kw)), None) == want


@host_only
def test_decode_empty_batch_is_noop(lib):
    a = _decode_args(batch=0, q=None, k=None)
    assert lib.gdr_decode_step(ctypes.byref(a), None) == OK
    assert lib.gdr_decode_step(None, None) == INVALID


def _decode_multi_args(base=None, **kw):
    m = _abi.DecodeMultiArgs()
    m.base = base if base is not None else _decode_args()
    m.n_tokens, m.n_slots = 4, 0
    for k, v in kw.items():
        setattr(m, k, v)
    return m


DECODE_MULTI_CASES = [
    ("zero_tokens", dict(n_tokens=0), INVALID),
    ("too_many_tokens", dict(n_tokens=9), INVALID),
    ("slots_without_count", dict(state_slot=FAKE + (11 << 32), n_slots=0), INVALID),
    ("misaligned_slots", dict(state_slot=FAKE + (11 << 32) + 2, n_slots=8), MISALIGNED),
    ("misaligned_status", dict(status=FAKE + (12 << 32) + 1), MISALIGNED),
]


@host_only
@pytest.mark.parametrize("name,kw,want", DECODE_MULTI_CASES, ids=[c[0] for c in DECODE_MULTI_CASES])
def test_decode_multi_validation(lib, name, kw, want):
    assert lib.gdr_decode_multi(ctypes.byref(_decode_multi_args(**kw)), None) == want


@host_only
@pytest.mark.parametrize("name,kw,want", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode_multi_checks_the_step_arguments(lib, name, kw, want):
    m = _decode_multi_args(base=_decode_args(**kw))
    assert lib.gdr_decode_multi(ctypes.byref(m), None) == want


@host_only
def test_decode_multi_slot_pool_overlap(lib):
    # With slots the state buffers span n_slots rows: a separate state_out that
    # starts inside that span overlaps even though `batch` rows alone would not.
    row = 4 * 128 * 128 * 4  # H_v * d * d floats
    base = _decode_args(state_in=FAKE, state_out=FAKE + 6 * row)
    assert lib.gdr_decode_multi(ctypes.byref(_decode_multi_args(base=base)), None) != INVALID
    base = _decode_args(state_in=FAKE, state_out=FAKE + 6 * row)
    m = _decode_multi_args(base=base, state_slot=FAKE + (11 << 32), n_slots=8)
    assert lib.gdr_decode_multi(ctypes.byref(m), None) == INVALID
    assert lib.gdr_decode_multi(None, None) == INVALID


def _prefill_args(lens=(5, 0, 9), **kw):
    a = _abi.PrefillArgs()
    cu = [0]
    for l in lens:
        cu.append(cu[-1] + l)
    host = (ctypes.c_int32 * len(cu))(*cu)
    a.n_seq = len(lens)
    a.H_k, a.H_v, a.d_k, a.d_v = 2, 4, 128, 128
    a.chunk, a.in_dtype, a.out_dtype, a.qk_l2norm = 64, 1, 0, 1
    a.scale, a.eps_l2, a.eps_norm = 1.0, 1e-6, 1e-6
    a.n_tok = cu[-1]
    for i, name in enumerate(["q", "k", "v", "z", "g", "beta", "cu_seqlens", "initial_state",
                              "final_state", "norm_w", "out"]):
        setattr(a, name, FAKE + (i << 32))
    a.cu_seqlens_host = ctypes.cast(host, ctypes.POINTER(ctypes.c_int32))
    for k, v in kw.items():
        setattr(a, k, v)
    return a, host


PREFILL_CASES = [
    ("unknown_flag", dict(flags=1), INVALID),
    ("reserved_set", dict(reserved=1), INVALID),
    ("raw_gate_without_params", dict(flags=2), INVALID),
    ("raw_gate_misaligned", dict(flags=2, A_log=FAKE + (13 << 32) + 1,
                                 dt_bias=FAKE + (14 << 32)), MISALIGNED),
    ("chunk48", dict(chunk=48), UNSUPPORTED),
    ("chunk128", dict(chunk=128), UNSUPPORTED),
    ("d100", dict(d_k=100, d_v=100), UNSUPPORTED),
    ("negative_ntok", dict(n_tok=-1), INVALID),
    ("ntok_mismatch", dict(n_tok=13), INVALID),
    ("null_cu_host", dict(cu_seqlens_host=None), INVALID),
    ("null_cu_dev", dict(cu_seqlens=None), INVALID),
    ("null_v", dict(v=None), INVALID),
    ("misaligned_k", dict(k=FAKE + (1 << 32) + 2), MISALIGNED),
    ("misaligned_initial", dict(initial_state=FAKE + (7 << 32) + 8), MISALIGNED),
    ("misaligned_cu", dict(cu_seqlens=FAKE + (6 << 32) + 2), MISALIGNED),
    ("heads", dict(H_k=4, H_v=6), INVALID),
    ("bad_dtype", dict(in_dtype=3), INVALID),
    ("z_stride_small", dict(z_stride=4), INVALID),
]


@host_only
@pytest.mark.parametrize("name,kw,want", PREFILL_CASES, ids=[c[0] for c in PREFILL_CASES])
def test_prefill_validation(lib, name, kw, want):
    a, host = _prefill_args(**kw)
    assert lib.gdr_prefill_chunked(ctypes.byref(a), None, 0, None) == want


@host_only
def test_prefill_rejects_falling_offsets(lib):
    a, host = _prefill_args()
    host[1], host[2] = 9, 5  # 0, 9, 5, 14: falls
    assert lib.gdr_prefill_chunked(ctypes.byref(a), None, 0, None) == INVALID
    a, host = _prefill_args()
    host[0] = 1
    assert lib.gdr_prefill_chunked(ctypes.byref(a), None, 0, None) == INVALID


@host_only
def test_prefill_workspace_query(lib):
    a, host = _prefill_args()
    n = ctypes.c_size_t(12345)
    assert lib.gdr_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)) == OK
    assert lib.gdr_prefill_workspace_size(ctypes.byref(a), None) == INVALID
    a, host = _prefill_args(chunk=40)
    assert lib.gdr_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)) == UNSUPPORTED


@host_only
def test_prefill_workspace_required(lib):
    # bf16, d = 128, chunk 64 runs on the tensor cores and needs a workspace.
    a, host = _prefill_args()
    n = ctypes.c_size_t(0)
    assert lib.gdr_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)) == OK
    assert n.value >= 16 + 4 * a.n_seq
    # 3 sequences of 5, 0, 9 tokens = 2 chunks of 64 for each of 4 value heads,
    # each with a record holding at least W, P and T diag(beta) (16 KB tiles).
    assert n.value >= 2 * 4 * 3 * 16384
    assert lib.gdr_prefill_chunked(ctypes.byref(a), None, 0, None) == WORKSPACE
    # Below the one-kernel minimum (16 + 4 n_seq, rounded up to 256 bytes).
    assert lib.gdr_prefill_chunked(ctypes.byref(a), FAKE + (12 << 32), 255, None) == WORKSPACE
    assert lib.gdr_prefill_chunked(ctypes.byref(a), FAKE + (12 << 32) + 8, n.value, None) == MISALIGNED
    # fp32 inputs use the CUDA-core path, which needs none.
    a, host = _prefill_args(in_dtype=0)
    assert lib.gdr_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)) == OK and n.value == 0


@host_only
def test_prefill_empty_is_noop(lib):
    a, host = _prefill_args(lens=())
    assert lib.gdr_prefill_chunked(ctypes.byref(a), None, 0, None) == OK


def _norm_args(**kw):
    a = _abi.NormArgs()
    a.rows, a.d, a.o_dtype, a.z_dtype, a.out_dtype, a.eps = 10, 128, 0, 1, 1, 1e-6
    a.o, a.z, a.w, a.out = FAKE, FAKE + (1 << 32), FAKE + (2 << 32), FAKE + (3 << 32)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


NORM_CASES = [
    ("d100", dict(d=100), UNSUPPORTED),
    ("d0", dict(d=0), INVALID),
    ("rows_negative", dict(rows=-2), INVALID),
    ("null_z", dict(z=None), INVALID),
    ("misaligned_w", dict(w=FAKE + (2 << 32) + 4), MISALIGNED),
    ("inplace_dtype_change", dict(out=FAKE), INVALID),
    ("reserved", dict(reserved=2), INVALID),
]


@host_only
@pytest.mark.parametrize("name,kw,want", NORM_CASES, ids=[c[0] for c in NORM_CASES])
def test_norm_validation(lib, name, kw, want):
    assert lib.gdr_rmsnorm_gated(ctypes.byref(_norm_args(**kw)), None) == want


@host_only
def test_norm_zero_rows_is_noop(lib):
    assert lib.gdr_rmsnorm_gated(ctypes.byref(_norm_args(rows=0, o=None)), None) == OK


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        _abi.lib(str(tmp_path / "libgdr.so"))


@host_only
def test_selftest_wait_expiry_host_checks(lib):
    """The wait-expiry self-test refuses, before anything is queued, a wait limit
    outside its range, a shape that does not take the tensor cores, a workspace
    too small for the two-kernel path and an empty batch."""
    f = lib.gdr_prefill_selftest_wait_expiry
    a, host = _prefill_args()
    n = ctypes.c_size_t(0)
    assert lib.gdr_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)) == OK
    ws = FAKE + (40 << 32)
    assert f(ctypes.byref(a), ws, n.value, 10, None) == INVALID                # < 0.1 ms
    assert f(ctypes.byref(a), ws, n.value, 3_000_000_000, None) == INVALID     # > 2 s
    assert f(ctypes.byref(a), ws, 256, 20_000_000, None) == WORKSPACE
    b, host_b = _prefill_args(in_dtype=0)                                      # fp32 inputs
    assert f(ctypes.byref(b), ws, n.value, 20_000_000, None) == UNSUPPORTED
    c, host_c = _prefill_args(lens=())
    assert f(ctypes.byref(c), ws, n.value, 20_000_000, None) == INVALID


@host_only
def test_noalloc_status_rejects_null(lib):
    assert lib.gdr_prefill_noalloc_status(None, None) == INVALID


def _attn_args(**kw):
    a = _abi.AttnDecodeArgs()
    a.batch, a.H_q, a.H_kv, a.d = 4, 16, 2, 256
    a.rot_dim, a.max_len, a.kv_bound, a.out_dtype = 64, 512, 511, 0
    a.rope_theta, a.scale = 1e7, 1.0 / 16
    for i, name in enumerate(["q", "gate", "k", "v", "k_cache", "v_cache", "cache_len", "out"]):
        setattr(a, name, FAKE + (i << 32))
    for k, v in kw.items():
        setattr(a, k, v)
    return a


ATTN_CASES = [
    ("null_q", dict(q=None), INVALID),
    ("null_cache_len", dict(cache_len=None), INVALID),
    ("heads_not_multiple", dict(H_q=15), INVALID),
    ("too_many_query_heads_per_kv", dict(H_q=64, H_kv=2), UNSUPPORTED),
    ("d128", dict(d=128), UNSUPPORTED),
    ("odd_rot_dim", dict(rot_dim=63), INVALID),
    ("rot_dim_past_d", dict(rot_dim=258), INVALID),
    ("bound_past_capacity", dict(kv_bound=512), INVALID),
    ("negative_bound", dict(kv_bound=-1), INVALID),
    ("bad_theta", dict(rope_theta=0.0), INVALID),
    ("bad_out_dtype", dict(out_dtype=4), INVALID),
    ("misaligned_k_cache", dict(k_cache=FAKE + 8), MISALIGNED),
    ("misaligned_cache_len", dict(cache_len=FAKE + 2), MISALIGNED),
    ("stride_too_small", dict(q_stride=256), INVALID),
    ("cache_rows_past_int32", dict(batch=1 << 16, H_kv=2, H_q=16, max_len=1 << 15, kv_bound=100),
     UNSUPPORTED),
]


@host_only
@pytest.mark.parametrize("name,kw,want", ATTN_CASES, ids=[c[0] for c in ATTN_CASES])
def test_attn_validation(lib, name, kw, want):
    a = _attn_args(**kw)
    n = ctypes.c_size_t(1 << 30)
    assert lib.gdr_attn_decode_step(ctypes.byref(a), FAKE + (50 << 32), n, None) == want


@host_only
def test_attn_workspace(lib):
    a = _attn_args()
    n = ctypes.c_size_t(0)
    assert lib.gdr_attn_decode_workspace_size(ctypes.byref(a), ctypes.byref(n)) == OK
    assert n.value > 4 * 2 * 256 * 16 * 4  # at least one split's partials per (b, kv head)
    assert lib.gdr_attn_decode_step(ctypes.byref(a), FAKE + (50 << 32), n.value - 16, None) == WORKSPACE
    assert lib.gdr_attn_decode_step(ctypes.byref(a), None, n.value, None) == WORKSPACE
    empty = _attn_args(batch=0)
    assert lib.gdr_attn_decode_workspace_size(ctypes.byref(empty), ctypes.byref(n)) == OK
    assert n.value == 0
    assert lib.gdr_attn_decode_step(ctypes.byref(empty), None, 0, None) == OK


def _moe_args(**kw):
    a = _abi.MoeArgs()
    a.n_tok, a.hidden, a.n_exp, a.top_k, a.inter, a.s_inter = 4, 2048, 256, 8, 512, 512
    a.out_dtype = 0
    for i, name in enumerate(["x", "w_router", "w_gate_up", "w_down", "ws_gate_up", "ws_down",
                              "w_sgate", "out", "topk_idx", "topk_w"]):
        setattr(a, name, FAKE + (i << 32))
    for k, v in kw.items():
        setattr(a, k, v)
    return a


MOE_CASES = [
    ("null_x", dict(x=None), INVALID),
    ("null_down", dict(w_down=None), INVALID),
    ("shared_without_down", dict(ws_down=None), INVALID),
    ("shared_without_width", dict(s_inter=0), INVALID),
    ("top_k_zero", dict(top_k=0), INVALID),
    ("top_k_past_experts", dict(n_exp=4, top_k=8), INVALID),
    ("top_k_too_large", dict(n_exp=64, top_k=33), UNSUPPORTED),
    ("hidden_not_multiple_of_8", dict(hidden=2044), UNSUPPORTED),
    ("negative_tokens", dict(n_tok=-1), INVALID),
    ("reserved_set", dict(reserved=1), INVALID),
    ("misaligned_weights", dict(w_gate_up=FAKE + 8), MISALIGNED),
    ("misaligned_topk", dict(topk_idx=FAKE + 2), MISALIGNED),
    ("stride_too_small", dict(x_stride=1024), INVALID),
]


@host_only
@pytest.mark.parametrize("name,kw,want", MOE_CASES, ids=[c[0] for c in MOE_CASES])
def test_moe_validation(lib, name, kw, want):
    a = _moe_args(**kw)
    assert lib.gdr_moe_decode(ctypes.byref(a), FAKE + (60 << 32), 1 << 30, None) == want


@host_only
def test_moe_workspace(lib):
    a = _moe_args()
    n = ctypes.c_size_t(0)
    assert lib.gdr_moe_workspace_size(ctypes.byref(a), ctypes.byref(n)) == OK
    # at least the per-pair partial outputs: 4 tokens x (8 + 1) pairs x 2048 fp32
    assert n.value >= 4 * 9 * 2048 * 4
    assert lib.gdr_moe_decode(ctypes.byref(a), FAKE + (60 << 32), n.value - 256, None) == WORKSPACE
    no_shared = _moe_args(ws_gate_up=None, ws_down=None, w_sgate=None, s_inter=0)
    m = ctypes.c_size_t(0)
    assert lib.gdr_moe_workspace_size(ctypes.byref(no_shared), ctypes.byref(m)) == OK
    assert m.value < n.value
    empty = _moe_args(n_tok=0)
    assert lib.gdr_moe_workspace_size(ctypes.byref(empty), ctypes.byref(m)) == OK and m.value == 0
    assert lib.gdr_moe_decode(ctypes.byref(empty), None, 0, None) == OK


@host_only
@pytest.mark.parametrize("kw", [dict(inter=1032), dict(s_inter=2048), dict(n_exp=1025, top_k=8)])
def test_moe_size_limits(lib, kw):
    a = _moe_args(**kw)
    assert lib.gdr_moe_decode(ctypes.byref(a), FAKE + (60 << 32), 1 << 30, None) == UNSUPPORTED
