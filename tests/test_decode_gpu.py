"""Decode kernel (gdr_decode_step) against the fp64 oracle on seeded inputs.

Teacher forced: every step reads its token from the seeded inputs, so the GPU
never consumes its own output (the Core ML card for Qwen3.5-0.8B, section
"Fidelity", feeds both sides the same tokens so that disagreement means a
fault, not drift).  The long test watches the error step by step, because a
broken state write shows up as agreement that decays as generation goes on
(same card, defect 2).
"""
import math
import os

import numpy as np
import pytest
import torch

from gdr_testutil import TOL, f64, oracle_full, assert_close, rel_l2, run_decode
from linear_attention_recurrence_10_b200 import synth

pytestmark = pytest.mark.gpu


def _check(inp, out, final, dtype, ref=None, tol_scale=1.0):
    ref = ref or oracle_full(inp)
    tol = TOL[dtype]
    e_out, _ = assert_close(f64(out), ref.y, tol["out"] * tol_scale, "output")
    e_state, _ = assert_close(f64(final), ref.state, tol["state"] * tol_scale, "state")
    return e_out, e_state


def test_tiny_fp32_64_steps():
    """B=1, 2 heads, d=16, 64 steps, fp32, S_0 = 0, seed 0 (the tiny oracle check)."""
    inp = synth.make_inputs([64], 2, 2, 16, seed=0, dtype=torch.float32)
    out, final = run_decode(inp, 64)
    _check(inp, out, final, torch.float32)


@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("heads", [(1, 1), (2, 4), (3, 3)])
def test_shapes(d, dtype, heads):
    H_k, H_v = heads
    inp = synth.make_inputs([9] * 5, H_k, H_v, d, seed=100 + d, dtype=dtype, s0_std=0.02)
    out, final = run_decode(inp, 9)
    _check(inp, out, final, dtype)


@pytest.mark.parametrize("scale", [1.0, 128 ** -0.5])
def test_scale_and_no_gate(scale):
    inp = synth.make_inputs([12] * 3, 2, 4, 128, seed=7, dtype=torch.bfloat16, s0_std=0.02)
    ref = oracle_full(inp, scale=scale)
    out, final = run_decode(inp, 12, scale=scale)
    _check(inp, out, final, torch.bfloat16, ref=ref)
    raw, final2 = run_decode(inp, 12, scale=scale, with_z=False)
    assert_close(f64(raw), ref.o, 2e-3)
    assert torch.equal(final, final2)


def test_out_of_place_and_bf16_output():
    inp = synth.make_inputs([10] * 4, 2, 2, 128, seed=8, dtype=torch.bfloat16, s0_std=0.02)
    ref = oracle_full(inp)
    a_out, a_state = run_decode(inp, 10, in_place=True)
    b_out, b_state = run_decode(inp, 10, in_place=False)
    assert torch.equal(a_out, b_out) and torch.equal(a_state, b_state)
    c_out, _ = run_decode(inp, 10, out_dtype=torch.bfloat16)
    # bf16 output is compared with the oracle rounded to bf16.
    ref_bf16 = torch.from_numpy(ref.y).to(torch.bfloat16).double().numpy()
    assert_close(f64(c_out), ref_bf16, 2e-3, bf16_ulp=True)


def test_no_l2norm_given_unit_vectors():
    inp = synth.make_inputs([8] * 2, 1, 2, 64, seed=9, dtype=torch.float32, s0_std=0.02)
    inp.q = torch.nn.functional.normalize(inp.q, dim=-1)
    inp.k = torch.nn.functional.normalize(inp.k, dim=-1)
    ref = oracle_full(inp, qk_l2norm=False)
    out, final = run_decode(inp, 8, qk_l2norm=False)
    _check(inp, out, final, torch.float32, ref=ref)


def test_reset_by_neg_inf_gate():
    inp = synth.make_inputs([16] * 2, 2, 2, 128, seed=10, dtype=torch.float32, s0_std=0.02)
    g = inp.g.clone()
    g[5] = -math.inf       # sequence 0, token 5
    g[16 + 15] = -math.inf  # sequence 1, last token
    inp.g = g
    out, final = run_decode(inp, 16)
    e = _check(inp, out, final, torch.float32)
    assert np.isfinite(f64(out)).all()


def test_beta_one_retrieval():
    """beta = 1 and q = k: o_t = v_t exactly in exact arithmetic (delta-rule retrieval)."""
    inp = synth.make_inputs([6] * 2, 2, 2, 128, seed=11, dtype=torch.float32, s0_std=0.02)
    inp.beta = torch.ones_like(inp.beta)
    inp.k = inp.q.clone()
    out, _ = run_decode(inp, 6, with_z=False)
    assert_close(f64(out), f64(inp.v), 1e-5)


def test_long_decode_no_drift():
    """512 steps, d=128, bf16: the error after each step must not grow."""
    T = 512
    inp = synth.make_inputs([T] * 2, 2, 2, 128, seed=12, dtype=torch.bfloat16, s0_std=0.02)
    ref = oracle_full(inp)
    out, final = run_decode(inp, T)
    _check(inp, out, final, torch.bfloat16, ref=ref)
    o = f64(out).reshape(2, T, 2, 128)
    r = ref.y.reshape(2, T, 2, 128)
    per_step = [rel_l2(o[:, t], r[:, t]) for t in range(T)]
    first, last = np.mean(per_step[:64]), np.mean(per_step[-64:])
    assert last <= 2.0 * first + 1e-6, f"error grows: {first:.2e} -> {last:.2e}"


def _full_size(B, H_k, H_v, T, seed, dtype=torch.bfloat16):
    """Every output and every final state against the threaded oracle."""
    inp = synth.make_inputs([T] * B, H_k, H_v, 128, seed=seed, dtype=dtype, s0_std=0.02)
    out, final = run_decode(inp, T)
    ref = oracle_full(inp, threads=os.cpu_count() or 8)
    assert_close(f64(out), ref.y, TOL[dtype]["out"], "outputs")
    assert_close(f64(final), ref.state, TOL[dtype]["state"], "final states")
    # And per (sequence, head): no pair may hide behind the others' accuracy.
    o = f64(out).reshape(B, T, H_v, 128)
    r = ref.y.reshape(B, T, H_v, 128)
    fs = f64(final)
    worst = max(rel_l2(o[b, :, h], r[b, :, h]) for b in range(B) for h in range(H_v))
    worst_s = max(rel_l2(fs[b, h], ref.state[b, h]) for b in range(B) for h in range(H_v))
    assert worst <= TOL[dtype]["out"] and worst_s <= TOL[dtype]["state"], (worst, worst_s)


@pytest.mark.slow
def test_qwen35_decode_full_batch32():
    """Qwen3.5-0.8B-shaped decode layer: B=32, 16/16 heads, d=128, bf16, 512 steps,
    S_0 ~ N(0, 0.02); all 512 (sequence, head) pairs against the oracle."""
    _full_size(32, 16, 16, 512, seed=1)


@pytest.mark.slow
@pytest.mark.parametrize("B", [1, 2, 4, 8, 16])
def test_qwen35_decode_small_batches(B):
    _full_size(B, 16, 16, 64, seed=1)


@pytest.mark.slow
def test_qwen36_gva_decode_full():
    """Qwen3.6-35B-A3B-shaped GVA decode: B=64, 16 key / 32 value heads, 256 steps;
    all 2048 (sequence, head) pairs."""
    _full_size(64, 16, 32, 256, seed=3)


def test_empty_batch_is_noop():
    import linear_attention_recurrence_10_b200 as gdr
    e = torch.empty(0, 2, 128, device="cuda", dtype=torch.bfloat16)
    gb = torch.empty(0, 2, device="cuda")
    st = torch.empty(0, 2, 128, 128, device="cuda")
    out = torch.empty(0, 2, 128, device="cuda")
    gdr.decode_step(e, e, e, gb, gb, st, out, z=e)
