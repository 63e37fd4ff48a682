"""Gates from raw projections (GDR_GATE_FROM_RAW) on every GPU path, against the
fp64 oracle fed with oracle.gate_from_raw's g and beta.

The per-head parameters follow the usual initialisation of such layers (the
decay rate A uniform in [1, 16], the step dt log-uniform in [1e-3, 0.1] with
dt_bias its inverse softplus), so the decays cover the range a trained model
sees; a, b ~ N(0, 1) per token."""
import math

import numpy as np
import pytest
import torch

import linear_attention_recurrence_10_b200 as gdr
import oracle
from gdr_testutil import TOL, f64, assert_close, rel_l2, run_decode, run_prefill
from linear_attention_recurrence_10_b200 import synth

pytestmark = pytest.mark.gpu


def raw_gate_problem(lens, H_k, H_v, d, seed, dtype, s0_std=0.02):
    """Inputs whose g, beta hold raw projections, the per-head parameters, and
    the same inputs with the oracle's gate values in their place."""
    inp = synth.make_inputs(lens, H_k, H_v, d, seed=seed, dtype=dtype, s0_std=s0_std)
    n = inp.n_tok
    a = synth.normal((n, H_v), seed, "gate_a")
    b = synth.normal((n, H_v), seed, "gate_b")
    A = synth.uniform((H_v,), seed, "gate_A", 1.0, 16.0)
    dt = torch.exp(synth.uniform((H_v,), seed, "gate_dt", math.log(1e-3), math.log(0.1)))
    A_log = torch.log(A)
    dt_bias = torch.log(torch.expm1(dt))
    g, beta = oracle.gate_from_raw(a.double().numpy(), b.double().numpy(),
                                   A_log.double().numpy(), dt_bias.double().numpy())
    raw = synth.Inputs(inp.q, inp.k, inp.v, inp.z, a.contiguous(), b.contiguous(), inp.s0, inp.w,
                       inp.cu_seqlens, H_k, H_v, d, seed)
    gated = synth.Inputs(inp.q, inp.k, inp.v, inp.z, torch.from_numpy(g).float(),
                         torch.from_numpy(beta).float(), inp.s0, inp.w, inp.cu_seqlens, H_k, H_v,
                         d, seed)
    return raw, gated, (A_log.float().cuda(), dt_bias.float().cuda()), g, beta


def oracle_ref(inp, g, beta):
    return oracle.gdr_recurrent(f64(inp.q), f64(inp.k), f64(inp.v), g, beta,
                                np.array(inp.cu_seqlens), z=f64(inp.z),
                                s0=None if inp.s0 is None else f64(inp.s0), w=f64(inp.w),
                                threads=8)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode(dtype):
    T = 12
    raw, _, params, g, beta = raw_gate_problem([T] * 5, 2, 4, 128, 600, dtype)
    ref = oracle_ref(raw, g, beta)
    out, final = run_decode(raw, T, gate_params=params)
    assert_close(f64(out), ref.y, TOL[dtype]["out"])
    assert_close(f64(final), ref.state, TOL[dtype]["state"])


def test_decode_multi():
    T = 4
    raw, _, params, g, beta = raw_gate_problem([T] * 6, 2, 4, 128, 601, torch.bfloat16)
    ref = oracle_ref(raw, g, beta)
    x = raw.to("cuda")
    state = x.s0.clone()
    out = torch.empty(x.n_tok, 4, 128, device="cuda")
    gdr.decode_multi(x.q, x.k, x.v, x.g, x.beta, state, out, n_tokens=T, z=x.z, norm_w=x.w,
                     gate_params=params)
    torch.cuda.synchronize()
    assert_close(f64(out), ref.y, 2e-3)
    assert_close(f64(state), ref.state, 1e-3)


@pytest.mark.parametrize("path", ["two_kernel", "one_kernel", "cuda_cores"])
def test_prefill(path):
    lens = [300, 64, 1, 190]
    dtype = torch.float32 if path == "cuda_cores" else torch.bfloat16
    d = 64 if path == "cuda_cores" else 128
    raw, _, params, g, beta = raw_gate_problem(lens, 2, 4, d, 610, dtype)
    ref = oracle_ref(raw, g, beta)
    ws = None
    if path == "one_kernel":
        ws = torch.empty((16 + 4 * len(lens) + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
    out, final = run_prefill(raw, chunk=64 if path != "cuda_cores" else 32, workspace=ws,
                             gate_params=params)
    assert_close(f64(out), ref.y, TOL[dtype]["out"])
    assert_close(f64(final), ref.state, TOL[dtype]["state"])


def test_raw_matches_precomputed_gates_on_device():
    """The raw path equals passing the (fp32-rounded) gate values directly, up
    to the fp32 evaluation of softplus and sigmoid."""
    raw, gated, params, _, _ = raw_gate_problem([64, 33], 2, 2, 128, 620, torch.bfloat16)
    out_r, fin_r = run_prefill(raw, gate_params=params)
    out_g, fin_g = run_prefill(gated)
    assert_close(f64(out_r), f64(out_g), 1e-5)
    assert_close(f64(fin_r), f64(fin_g), 1e-5)
