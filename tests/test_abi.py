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
    # 3 sequences of 5, 0, 9 tokens = 2 chunks of 64 for each of 4 value heads.
    assert n.value >= 2 * 4 * 65536
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
