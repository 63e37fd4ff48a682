"""Chunked prefill (gdr_prefill_chunked) against the fp64 oracle on seeded inputs.

Besides direct parity, two equivalences from the Swiftlet post ("Correctness &
Validation": incremental decoding matches whole-sequence processing):
decode steps after a prefill equal one longer prefill, and a prefill split in
two with the state handed over equals the whole prefill.
"""
import math
import os

import pytest
import torch

import linear_attention_recurrence_10_b200 as gdr
from gdr_testutil import (TOL, assert_close, f64, oracle_full, oracle_sequence, rel_l2,
                          run_decode, run_prefill)
from linear_attention_recurrence_10_b200 import synth

pytestmark = pytest.mark.gpu


def _check(inp, out, final, dtype, ref=None):
    ref = ref or oracle_full(inp)
    assert_close(f64(out), ref.y, TOL[dtype]["out"], "output")
    assert_close(f64(final), ref.state, TOL[dtype]["state"], "state")
    return ref


def test_tiny_fp32_chunk16():
    """B=1, 2 heads, d=16, T=64, fp32, chunk 16, seed 0: chunked vs the recurrence."""
    inp = synth.make_inputs([64], 2, 2, 16, seed=0, dtype=torch.float32)
    out, final = run_prefill(inp, chunk=16)
    _check(inp, out, final, torch.float32)


@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_shapes_ragged(d, chunk, dtype):
    """Several chunks, ragged last chunks, an empty sequence, GVA heads."""
    lens = [1, chunk + 3, 0, 2 * chunk, 3 * chunk - 5]
    inp = synth.make_inputs(lens, 2, 4, d, seed=200 + d + chunk, dtype=dtype, s0_std=0.02)
    out, final = run_prefill(inp, chunk=chunk)
    _check(inp, out, final, dtype)


def test_no_initial_state_and_no_gate():
    inp = synth.make_inputs([70, 33], 2, 2, 128, seed=21, dtype=torch.bfloat16)
    ref = oracle_full(inp)
    out, final = run_prefill(inp, chunk=64, initial_state=None)
    _check(inp, out, final, torch.bfloat16, ref=ref)
    raw, _ = run_prefill(inp, chunk=64, initial_state=None, with_z=False)
    assert_close(f64(raw), ref.o, 2e-3)


def test_in_place_state():
    inp = synth.make_inputs([40, 90], 1, 2, 64, seed=22, dtype=torch.float32, s0_std=0.02)
    ref = oracle_full(inp)
    x = inp.to("cuda")
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device="cuda")
    out = torch.empty(inp.n_tok, 2, 64, device="cuda")
    st = x.s0.clone()
    gdr.prefill_chunked(x.q, x.k, x.v, x.g, x.beta, cu, out, z=x.z, norm_w=x.w,
                        initial_state=st, final_state=st, chunk=32)
    torch.cuda.synchronize()
    assert_close(f64(st), ref.state, 1e-5)
    assert_close(f64(out), ref.y, 1e-5)


def test_reset_clamp():
    """g = -inf inside chunks: the chunk form clamps g at -64, which changes
    nothing visible next to O(1) terms."""
    inp = synth.make_inputs([100], 2, 2, 128, seed=23, dtype=torch.float32, s0_std=0.02)
    g = inp.g.clone()
    g[[3, 64, 99]] = -math.inf
    inp.g = g
    out, final = run_prefill(inp, chunk=64)
    _check(inp, out, final, torch.float32)


@pytest.mark.parametrize("chunk", [32, 64])
def test_decode_after_prefill_equals_longer_prefill(chunk):
    """Prefill T1 tokens, then T2 decode steps from its final state == one prefill
    of T1 + T2 tokens.  chunk 64 runs on the tensor cores (bf16 MMAs, with hi/lo
    bf16 pairs for the precision-sensitive operands), so the two sides agree to the
    bf16 bars there and to 1e-5 on the CUDA-core path."""
    T1, T2 = 100, 12
    tol_o, tol_s = (2e-3, 1e-3) if chunk == 64 else (1e-5, 1e-5)
    inp = synth.make_inputs([T1 + T2] * 2, 2, 2, 128, seed=24, dtype=torch.bfloat16,
                            s0_std=0.02)
    whole_out, whole_state = run_prefill(inp, chunk=chunk)
    _check(inp, whole_out, whole_state, torch.bfloat16)
    idx = torch.cat([torch.arange(s * (T1 + T2), s * (T1 + T2) + T1) for s in range(2)])
    tail = torch.cat([torch.arange(s * (T1 + T2) + T1, (s + 1) * (T1 + T2)) for s in range(2)])
    a = synth.Inputs(inp.q[idx], inp.k[idx], inp.v[idx], inp.z[idx], inp.g[idx], inp.beta[idx],
                     inp.s0, inp.w, [0, T1, 2 * T1], inp.H_k, inp.H_v, inp.d, inp.seed)
    a_out, a_state = run_prefill(a, chunk=chunk)
    b = synth.Inputs(inp.q[tail], inp.k[tail], inp.v[tail], inp.z[tail], inp.g[tail],
                     inp.beta[tail], a_state.cpu(), inp.w, [0, T2, 2 * T2], inp.H_k, inp.H_v,
                     inp.d, inp.seed)
    b_out, b_state = run_decode(b, T2)
    assert_close(f64(b_state), f64(whole_state), tol_s)
    w = f64(whole_out).reshape(2, T1 + T2, 2, 128)
    assert_close(f64(b_out).reshape(2, T2, 2, 128), w[:, T1:], tol_o)
    assert_close(f64(a_out).reshape(2, T1, 2, 128), w[:, :T1], tol_o)


@pytest.mark.parametrize("chunk", [32, 64])
def test_split_prefill_equals_whole(chunk):
    T, m = 300, 129
    tol_o, tol_s = (2e-3, 1e-3) if chunk == 64 else (1e-5, 1e-5)
    inp = synth.make_inputs([T], 2, 4, 128, seed=25, dtype=torch.bfloat16, s0_std=0.02)
    whole_out, whole_state = run_prefill(inp, chunk=chunk)
    parts = []
    s0 = inp.s0
    for lo, hi in ((0, m), (m, T)):
        sl = slice(lo, hi)
        p = synth.Inputs(inp.q[sl], inp.k[sl], inp.v[sl], inp.z[sl], inp.g[sl], inp.beta[sl],
                         s0, inp.w, [0, hi - lo], inp.H_k, inp.H_v, inp.d, inp.seed)
        o, s = run_prefill(p, chunk=chunk)
        parts.append(o)
        s0 = s.cpu()
    assert_close(f64(s0), f64(whole_state), tol_s)
    assert_close(f64(torch.cat(parts)), f64(whole_out), tol_o)


# ---------------------------------------------------------------- tensor cores
# bf16 inputs, d = 128, chunk 64 run on the tcgen05 kernel.

@pytest.mark.parametrize("lens", [[64], [1], [63, 65, 0, 128, 200], [257, 3, 64 * 5 + 17]])
@pytest.mark.parametrize("heads", [(1, 1), (2, 4), (4, 4)])
def test_tc_ragged_varlen(lens, heads):
    H_k, H_v = heads
    inp = synth.make_inputs(lens, H_k, H_v, 128, seed=300 + sum(lens) + H_v, dtype=torch.bfloat16,
                            s0_std=0.02)
    out, final = run_prefill(inp, chunk=64)
    _check(inp, out, final, torch.bfloat16)


@pytest.mark.parametrize("lens", [[100, 64], [36, 300], [200, 1], [800, 50]])
def test_tc_ragged_tail_never_reads_the_next_sequence(lens):
    """A sequence's ragged last chunk is loaded as whole 64-token boxes, which reach into the
    next sequence's rows: with every q, k and v value of the second sequence NaN, the first
    sequence's outputs and final states are finite and match the oracle (its own inputs
    only). [800, 50] runs as three segments."""
    inp = synth.make_inputs(lens, 2, 4, 128, seed=77 + sum(lens), dtype=torch.bfloat16,
                            s0_std=0.02)
    t1 = inp.cu_seqlens[1]
    for name in ("q", "k", "v"):
        getattr(inp, name)[t1:] = float("nan")
    out, final = run_prefill(inp, chunk=64)
    ref = oracle_sequence(inp, 0)
    o, fs = f64(out[:t1]), f64(final[0:1])
    # (assert_close also requires every value finite)
    assert_close(o, ref.y, 2e-3, what="outputs of the first sequence")
    assert_close(fs, ref.state, 1e-3, what="final states of the first sequence")


@pytest.mark.parametrize("scale", [1.0, 128 ** -0.5])
def test_tc_scale_gate_and_outputs(scale):
    inp = synth.make_inputs([150, 90], 2, 2, 128, seed=31, dtype=torch.bfloat16, s0_std=0.02)
    ref = oracle_full(inp, scale=scale)
    out, final = run_prefill(inp, chunk=64, scale=scale)
    _check(inp, out, final, torch.bfloat16, ref=ref)
    raw, _ = run_prefill(inp, chunk=64, scale=scale, with_z=False)
    assert_close(f64(raw), ref.o, 2e-3)
    o16, _ = run_prefill(inp, chunk=64, scale=scale, out_dtype=torch.bfloat16)
    ref16 = torch.from_numpy(ref.y).to(torch.bfloat16).double().numpy()
    assert_close(f64(o16), ref16, 2e-3, bf16_ulp=True)


def test_tc_long_memory_and_reset():
    """exp(g) in [0.9, 1) (long memory) with a few g = -inf resets."""
    inp = synth.make_inputs([700, 333], 2, 4, 128, seed=32, dtype=torch.bfloat16,
                            g_mode="long", s0_std=0.02)
    g = inp.g.clone()
    g[[5, 64, 400, 900]] = -math.inf
    inp.g = g
    out, final = run_prefill(inp, chunk=64)
    _check(inp, out, final, torch.bfloat16)


@pytest.mark.parametrize("g_scale", [8.0, 40.0])
@pytest.mark.parametrize("one_kernel", [False, True])
def test_tc_strong_decay(g_scale, one_kernel):
    """g = -softplus(N(0,1)) times 8 or 40: the decay across one chunk spans far
    more than fp32's exponent range, so no intermediate may rescale a chunk's
    tokens by e^{+-(gamma_r - gamma_s)} beyond what the recurrence itself applies."""
    lens = [300, 130]
    inp = synth.make_inputs(lens, 2, 4, 128, seed=35, dtype=torch.bfloat16, s0_std=0.02)
    inp.g = (inp.g * g_scale).contiguous()
    ws = None
    if one_kernel:
        ws = torch.empty((16 + 4 * len(lens) + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
    out, final = run_prefill(inp, chunk=64, workspace=ws)
    _check(inp, out, final, torch.bfloat16)


def test_tc_no_l2norm_and_status_word():
    inp = synth.make_inputs([130, 70], 2, 2, 128, seed=33, dtype=torch.bfloat16, s0_std=0.02)
    inp.q = torch.nn.functional.normalize(inp.q.float(), dim=-1).to(torch.bfloat16)
    inp.k = torch.nn.functional.normalize(inp.k.float(), dim=-1).to(torch.bfloat16)
    ref = oracle_full(inp, qk_l2norm=False)
    x = inp.to("cuda")
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device="cuda")
    out = torch.empty(inp.n_tok, 2, 128, device="cuda")
    final = torch.empty(2, 2, 128, 128, device="cuda")
    n = gdr.prefill_workspace_size(x.q, x.k, x.v, x.g, x.beta, cu, out, z=x.z, chunk=64)
    assert n >= 16
    ws = torch.full((n,), 0xAB, dtype=torch.uint8, device="cuda")
    gdr.prefill_chunked(x.q, x.k, x.v, x.g, x.beta, cu, out, z=x.z, norm_w=x.w,
                        initial_state=x.s0, final_state=final, chunk=64, workspace=ws,
                        qk_l2norm=False)
    torch.cuda.synchronize()
    assert ws[:4].view(torch.int32).item() == 0  # no device wait gave up
    assert_close(f64(out), ref.y, 2e-3)
    assert_close(f64(final), ref.state, 1e-3)


def test_tc_workspace_too_small():
    inp = synth.make_inputs([64], 1, 1, 128, seed=34, dtype=torch.bfloat16)
    x = inp.to("cuda")
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device="cuda")
    out = torch.empty(64, 1, 128, device="cuda")
    ws = torch.empty(8, dtype=torch.uint8, device="cuda")
    with pytest.raises(gdr.GdrError, match="WORKSPACE"):
        gdr.prefill_chunked(x.q, x.k, x.v, x.g, x.beta, cu, out, z=x.z, chunk=64, workspace=ws)


def _every_pair(inp, out, final, threads):
    """Each sequence's outputs and final states (every head) against the oracle,
    one sequence at a time; the worst (sequence, head) pair must meet the bars too."""
    for s in range(inp.n_seq):
        ref = oracle_sequence(inp, s, threads=threads)
        t0, t1 = inp.cu_seqlens[s], inp.cu_seqlens[s + 1]
        o = f64(out[t0:t1])
        fs = f64(final[s:s + 1])
        assert_close(o, ref.y, 2e-3, what=f"outputs of sequence {s}")
        assert_close(fs, ref.state, 1e-3, what=f"final states of sequence {s}")
        for h in range(inp.H_v):
            assert rel_l2(o[:, h], ref.y[:, h]) <= 2e-3, (s, h)
            assert rel_l2(fs[0, h], ref.state[0, h]) <= 1e-3, (s, h)


@pytest.mark.slow
def test_qwen35_prefill_full():
    """Qwen3.5-0.8B-shaped prefill: B=4, T=4096, 16 heads, d=128, bf16, chunk 64,
    S_0 = 0; every output and final state against the oracle."""
    inp = synth.make_inputs([4096] * 4, 16, 16, 128, seed=2, dtype=torch.bfloat16)
    out, final = run_prefill(inp, chunk=64)
    _every_pair(inp, out, final, threads=os.cpu_count() or 8)


@pytest.mark.slow
def test_long_context_gva_prefill_full():
    """Long-context GVA prefill: 8 sequences, lengths U{1024..32768} (seed 4),
    16 key / 32 value heads, d=128, bf16, chunk 64, exp(g) in [0.9, 1); every
    output and final state against the oracle."""
    lens = synth.lengths(8, 4, 1024, 32768)
    inp = synth.make_inputs(lens, 16, 32, 128, seed=4, dtype=torch.bfloat16, g_mode="long")
    out, final = run_prefill(inp, chunk=64)
    out, final = out.cpu(), final.cpu()
    _every_pair(inp, out, final, threads=os.cpu_count() or 8)


@pytest.mark.parametrize("lens", [[64], [63, 65, 0, 128, 200], [257, 3, 64 * 5 + 17]])
def test_tc_one_kernel_variant(lens):
    """A workspace too small for the per-chunk records (but holding the sequence
    order) runs the tensor-core prefill as one kernel; same bars."""
    inp = synth.make_inputs(lens, 2, 4, 128, seed=500 + sum(lens), dtype=torch.bfloat16,
                            s0_std=0.02)
    small = (16 + 4 * len(lens) + 255) // 256 * 256
    ws = torch.empty(small, dtype=torch.uint8, device="cuda")
    out, final = run_prefill(inp, chunk=64, workspace=ws)
    _check(inp, out, final, torch.bfloat16)


def _single_pass_workspace(inp, H_v):
    """A workspace one carry buffer short of the segmented layout, which makes
    the library run prep and recurrence as a single pass."""
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device="cuda")
    x = inp.to("cuda")
    out = torch.empty(inp.n_tok, H_v, 128, device="cuda")
    n = gdr.prefill_workspace_size(x.q, x.k, x.v, x.g, x.beta, cu, out,
                                   cu_seqlens_host=inp.cu_seqlens, z=x.z, chunk=64)
    return torch.empty(n - inp.n_seq * H_v * 128 * 128 * 4, dtype=torch.uint8, device="cuda")


# Sequences of 20, 9 (= the first segment boundary, 44% of 20 chunks rounded
# up), 0, 17 and 1 chunks: every segment, an end exactly on a boundary, an empty
# sequence, and a sequence that ends in the first segment.
SEG_LENS = [20 * 64 - 5, 9 * 64, 0, 16 * 64 + 3, 40]


def test_tc_segmented_varlen():
    """Few (sequence, head) chains leave SMs free, so the prefill runs in
    segments whose prep overlaps the previous segment's recurrence; the state
    crosses segment boundaries through the workspace."""
    inp = synth.make_inputs(SEG_LENS, 2, 4, 128, seed=36, dtype=torch.bfloat16, s0_std=0.02)
    out, final = run_prefill(inp, chunk=64)
    _check(inp, out, final, torch.bfloat16)


def test_tc_segmented_equals_single_pass():
    inp = synth.make_inputs(SEG_LENS, 2, 4, 128, seed=37, dtype=torch.bfloat16, s0_std=0.02)
    out_seg, fin_seg = run_prefill(inp, chunk=64)
    out_one, fin_one = run_prefill(inp, chunk=64, workspace=_single_pass_workspace(inp, 4))
    assert torch.equal(out_seg, out_one)
    assert torch.equal(fin_seg, fin_one)
