"""Multi-token decode with state slots (gdr_decode_multi) against the fp64 oracle.

n_tokens tokens of every sequence in one call, the state read and written once;
the Swiftlet post checks that token-by-token decoding matches processing the
tokens together ("Correctness & Validation"), which is what the bit-identity
test below pins: the multi-token call performs exactly the arithmetic of
n_tokens single steps, only without the state round trips through memory.
"""
import numpy as np
import pytest
import torch

import linear_attention_recurrence_10_b200 as gdr
from gdr_testutil import TOL, f64, oracle_full, assert_close, rel_l2, run_decode
from linear_attention_recurrence_10_b200 import synth

pytestmark = pytest.mark.gpu


def run_multi(inp, T, *, out_dtype=torch.float32, with_z=True, state=None, slots=None,
              status=None, out=None, **kw):
    x = inp.to("cuda")
    d = inp.d
    if state is None:
        state = (x.s0.clone() if x.s0 is not None
                 else torch.zeros(inp.n_seq, inp.H_v, d, d, device="cuda"))
    if out is None:
        out = torch.empty(inp.n_tok, inp.H_v, d, device="cuda", dtype=out_dtype)
    gdr.decode_multi(x.q, x.k, x.v, x.g, x.beta, state, out, n_tokens=T,
                     z=x.z if with_z else None, norm_w=x.w, slots=slots, status=status, **kw)
    torch.cuda.synchronize()
    return out, state


@pytest.mark.parametrize("T", [1, 2, 3, 8])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("heads,d", [((2, 4), 128), ((3, 3), 64), ((1, 2), 16)])
def test_matches_oracle(T, dtype, heads, d):
    H_k, H_v = heads
    inp = synth.make_inputs([T] * 6, H_k, H_v, d, seed=400 + T + d, dtype=dtype, s0_std=0.02)
    ref = oracle_full(inp)
    out, state = run_multi(inp, T)
    tol = TOL[dtype]
    assert_close(f64(out), ref.y, tol["out"])
    assert_close(f64(state), ref.state, tol["state"])


@pytest.mark.parametrize("T", [2, 5, 8])
@pytest.mark.parametrize("with_z", [True, False])
def test_bit_identical_to_single_steps(T, with_z):
    inp = synth.make_inputs([T] * 7, 2, 4, 128, seed=410 + T, dtype=torch.bfloat16, s0_std=0.02)
    out_m, state_m = run_multi(inp, T, with_z=with_z)
    out_s, state_s = run_decode(inp, T, with_z=with_z)
    assert torch.equal(out_m, out_s)
    assert torch.equal(state_m, state_s)


def test_state_slots_gather_and_scatter():
    """5 sequences over a pool of 9 states: each reads and writes its own row,
    the untouched rows stay bit-identical."""
    T, pool = 4, 9
    inp = synth.make_inputs([T] * 5, 2, 4, 128, seed=420, dtype=torch.bfloat16, s0_std=0.02)
    slot_of = [7, 0, 4, 8, 2]
    gen = torch.Generator().manual_seed(421)
    pool_state = torch.randn(pool, 4, 128, 128, generator=gen) * 0.02
    for b, s in enumerate(slot_of):
        pool_state[s] = inp.s0[b]
    pool_state = pool_state.cuda()
    before = pool_state.clone()
    slots = torch.tensor(slot_of, dtype=torch.int32, device="cuda")
    out, pool_after = run_multi(inp, T, state=pool_state, slots=slots)
    ref = oracle_full(inp)
    assert_close(f64(out), ref.y, 2e-3)
    assert_close(f64(pool_after[slots.long()]), ref.state, 1e-3)
    untouched = [s for s in range(pool) if s not in slot_of]
    assert torch.equal(pool_after[untouched], before[untouched])


def test_bad_slot_reports_and_leaves_its_sequence_alone():
    T = 3
    inp = synth.make_inputs([T] * 4, 1, 2, 64, seed=430, dtype=torch.float32, s0_std=0.02)
    pool_state = inp.s0.clone().cuda()
    before = pool_state.clone()
    slots = torch.tensor([0, 1, 99, 3], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sentinel = torch.full((inp.n_tok, 2, 64), 7.0, device="cuda")
    out, pool_after = run_multi(inp, T, state=pool_state, slots=slots, status=status,
                                out=sentinel)
    assert int(status.item()) == 1  # GDR_ERR_INVALID_ARG
    assert torch.equal(out[2 * T:3 * T], torch.full_like(out[2 * T:3 * T], 7.0))
    assert torch.equal(pool_after[2], before[2])
    ref = oracle_full(inp)
    good = [0, 1, 3]
    rows = np.concatenate([np.arange(b * T, (b + 1) * T) for b in good])
    assert_close(f64(out[rows]), ref.y[rows], 1e-5)
    assert_close(f64(pool_after[good]), ref.state[good], 1e-5)


def test_many_sequences_full_size():
    """Qwen3.5-0.8B-shaped: 32 sequences x 16 heads x d=128, 4 tokens per call."""
    T = 4
    inp = synth.make_inputs([T] * 32, 16, 16, 128, seed=440, dtype=torch.bfloat16, s0_std=0.02)
    ref = oracle_full(inp, threads=16)
    out, state = run_multi(inp, T)
    assert_close(f64(out), ref.y, 2e-3)
    assert_close(f64(state), ref.state, 1e-3)
