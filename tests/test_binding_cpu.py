"""The Python binding's marshalling, checked on the host: every field of the argument
struct a decode call hands to gdr_decode_step, for packed tensors and for strided
views; the binding's own refusals; and, with no CUDA device present, each entry
carried through the library's host checks up to the launch.  Nothing runs on a device."""
import pytest
import torch

import linear_attention_recurrence_10_b200 as gdr
from linear_attention_recurrence_10_b200 import _abi

B, H_K, H_V, D = 3, 2, 4, 32


def _inputs(dtype=torch.bfloat16, steps=None):
    """Packed [B, H, d] tensors, or one step of [B, steps, H, d] tensors."""
    def rows(H, dt=dtype):
        if steps is None:
            return torch.randn(B, H, D, dtype=dt)
        return torch.randn(B, steps, H, D, dtype=dt)[:, 1]
    def gates():
        return torch.randn(B, H_V) if steps is None else torch.randn(B, steps, H_V)[:, 1]
    return dict(q=rows(H_K), k=rows(H_K), v=rows(H_V), z=rows(H_V), g=gates(), beta=gates())


def _args(x, state, out, **kw):
    o = dict(z=x["z"], norm_w=torch.ones(D), state_out=None, scale=0.25, eps_l2=1e-6,
             eps_norm=1e-5, qk_l2norm=True, overlap_state_load=False, batch=B,
             gate_params=None)
    o.update(kw)
    return gdr._decode_args(x["q"], x["k"], x["v"], x["g"], x["beta"], state, out, o["z"],
                            o["norm_w"], o["state_out"], o["scale"], o["eps_l2"], o["eps_norm"],
                            o["qk_l2norm"], o["overlap_state_load"], o["batch"],
                            o["gate_params"])


@pytest.mark.parametrize("steps", [None, 5])
def test_decode_fields(steps):
    x = _inputs(steps=steps)
    state = torch.zeros(B, H_V, D, D)
    out = torch.empty(B, H_V, D, dtype=torch.float32)
    a = _args(x, state, out)
    assert (a.batch, a.H_k, a.H_v, a.d_k, a.d_v) == (B, H_K, H_V, D, D)
    assert (a.in_dtype, a.out_dtype) == (_abi.GDR_BF16, _abi.GDR_F32)
    assert a.qk_l2norm == 1 and a.flags == 0
    assert a.scale == 0.25 and a.eps_norm == pytest.approx(1e-5)
    rows = 1 if steps is None else steps
    assert a.q_stride == rows * H_K * D and a.k_stride == rows * H_K * D
    assert a.v_stride == rows * H_V * D and a.z_stride == rows * H_V * D
    assert a.gb_stride == rows * H_V
    assert a.out_stride == H_V * D and a.state_stride == H_V * D * D
    for name in ("q", "k", "v", "z", "g", "beta"):
        assert getattr(a, name) == x[name].data_ptr(), name
    assert a.state_in == state.data_ptr() and a.state_out == state.data_ptr()
    assert a.out == out.data_ptr() and a.A_log is None and a.dt_bias is None


def test_decode_optional_fields():
    x = _inputs(torch.float32)
    state = torch.zeros(B, H_V, D, D)
    state_out = torch.zeros(B, H_V, D, D)
    out = torch.empty(B, H_V, D, dtype=torch.bfloat16)
    A_log, dt_bias = torch.zeros(H_V), torch.ones(H_V)
    a = _args(x, state, out, z=None, norm_w=None, state_out=state_out, overlap_state_load=True,
              qk_l2norm=False, gate_params=(A_log, dt_bias))
    assert a.in_dtype == _abi.GDR_F32 and a.out_dtype == _abi.GDR_BF16
    assert a.z is None and a.z_stride == 0 and a.norm_w is None and a.qk_l2norm == 0
    assert a.state_out == state_out.data_ptr() != a.state_in
    assert a.flags == _abi.GDR_DECODE_OVERLAP_STATE_LOAD | _abi.GDR_GATE_FROM_RAW
    assert a.A_log == A_log.data_ptr() and a.dt_bias == dt_bias.data_ptr()


def test_single_row_has_stride_zero():
    x = {n: t[:1] for n, t in _inputs().items()}
    a = _args(x, torch.zeros(1, H_V, D, D), torch.empty(1, H_V, D), batch=1)
    assert a.q_stride == 0 and a.v_stride == 0 and a.gb_stride == 0 and a.state_stride == 0


def test_binding_refusals():
    x = _inputs()
    state = torch.zeros(B, H_V, D, D)
    out = torch.empty(B, H_V, D)
    bad = dict(x, v=torch.randn(B, D, H_V, dtype=torch.bfloat16).transpose(1, 2))
    with pytest.raises(ValueError):  # inner dimensions not packed
        _args(bad, state, out)
    with pytest.raises(TypeError):   # k of another dtype than q
        _args(dict(x, k=x["k"].float()), state, out)
    with pytest.raises(TypeError):   # fp16 is not an input dtype
        _args(dict(x, q=x["q"].half()), state, out)
    with pytest.raises(ValueError):  # g and beta in different layouts
        _args(dict(x, beta=torch.randn(B, 2, H_V)[:, 0]), state, out)
    with pytest.raises(ValueError):  # gate parameters of the wrong length
        _args(x, state, out, gate_params=(torch.zeros(H_V + 1), torch.zeros(H_V + 1)))


def test_every_entry_reaches_the_launch_without_a_device():
    """With no CUDA device, each binding call marshals its tensors, passes every host
    check of the library, and stops at the launch with GDR_ERR_CUDA: so the binding
    builds arguments the library accepts, through each declared ctypes signature."""
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present: the GPU tests cover these calls")
    H, D = 2, 128
    bf = torch.bfloat16
    w = torch.ones(D)

    def rows(n, dtype=bf):
        return torch.randn(n, H, D, dtype=dtype)

    def gates(n):
        return -torch.rand(n, H), torch.rand(n, H)

    state = torch.zeros(4, H, D, D)
    g, beta = gates(4)
    g8, beta8 = gates(8)
    n_tok = 200
    cu = torch.tensor([0, 80, n_tok], dtype=torch.int32)
    gp, bp = gates(n_tok)
    final = torch.zeros(2, H, D, D)
    pre = dict(cu_seqlens_host=[0, 80, n_tok], z=rows(n_tok), norm_w=w, final_state=final,
               chunk=64, stream=0)
    calls = {
        "gdr_decode_step": lambda: gdr.decode_step(
            rows(4), rows(4), rows(4), g, beta, state, rows(4), z=rows(4), norm_w=w, stream=0),
        "gdr_decode_multi": lambda: gdr.decode_multi(
            rows(8), rows(8), rows(8), g8, beta8, state, rows(8), n_tokens=2, z=rows(8),
            norm_w=w, slots=torch.arange(4, dtype=torch.int32),
            status=torch.zeros(1, dtype=torch.int32), stream=0),
        "gdr_prefill_chunked": lambda: gdr.prefill_chunked(
            rows(n_tok), rows(n_tok), rows(n_tok), gp, bp, cu, rows(n_tok), **pre),
        "gdr_prefill_chunked_noalloc": lambda: gdr.prefill_chunked_noalloc(
            rows(n_tok), rows(n_tok), rows(n_tok), gp, bp, cu, rows(n_tok), **pre),
        "gdr_attn_decode_step": lambda: gdr.attn_decode_step(
            torch.randn(3, 16, 256, dtype=bf), torch.randn(3, 16, 256, dtype=bf),
            torch.randn(3, 2, 256, dtype=bf), torch.randn(3, 2, 256, dtype=bf),
            torch.zeros(3, 2, 64, 256, dtype=bf), torch.zeros(3, 2, 64, 256, dtype=bf),
            torch.tensor([1, 5, 0], dtype=torch.int32), torch.empty(3, 16, 256),
            kv_bound=63, stream=0),
        "gdr_moe_decode": lambda: gdr.moe_decode(
            torch.randn(2, 256, dtype=bf), torch.randn(8, 256, dtype=bf),
            torch.randn(8, 64, 256, dtype=bf), torch.randn(8, 256, 32, dtype=bf),
            torch.empty(2, 256), top_k=2,
            shared=(torch.randn(32, 256, dtype=bf), torch.randn(256, 16, dtype=bf),
                    torch.randn(256, dtype=bf)), stream=0),
        "gdr_rmsnorm_gated": lambda: gdr.rmsnorm_gated(
            rows(10, torch.float32), rows(10, torch.float32), rows(10, torch.float32), w=w,
            stream=0),
    }
    for name, call in calls.items():
        with pytest.raises(gdr.GdrError) as e:
            call()
        assert e.value.status == 5 and name in str(e.value), (name, str(e.value))  # GDR_ERR_CUDA
