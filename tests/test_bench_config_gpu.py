"""The decode configurations the benchmark times, checked against the fp64 oracle
exactly as they are timed.

bench.py measures the Qwen3.5-0.8B-shaped decode as 18 independent layer states
rotating through HBM, every launch with GDR_DECODE_OVERLAP_STATE_LOAD (the
state loads start while the previous layer's kernel drains), each step's 18
launches replayed from a captured CUDA graph; and the multi-token view the same
way with gdr_decode_multi.  These tests build the benchmark's own objects
(bench.DecodeBench, bench.DecodeMultiBench), replay their graphs step by step,
read every layer's output after every step, and compare all outputs and the
final states of every layer with the oracle fed the same tokens.  Outputs are
stored as bf16 there, so they are compared with the oracle rounded to bf16
(the Core ML card for Qwen3.5-0.8B, section "Fidelity", feeds both sides the
same tokens so that a disagreement means a fault, not drift).
"""
import os

import numpy as np
import pytest
import torch

import bench
import oracle
from gdr_testutil import assert_close, f64

pytestmark = pytest.mark.gpu

THREADS = os.cpu_count() or 8


def _pack(t, n):
    """[L, steps, B, H, d] device tensor -> [L*B*n, H, d] fp64: sequence (l, b)
    holds its first n tokens in order."""
    x = f64(t[:, :n])
    L, _, B = x.shape[:3]
    return np.ascontiguousarray(np.swapaxes(x, 1, 2)).reshape(L * B * n, *x.shape[3:])


def _oracle(q, k, v, z, g, beta, s0, w, n):
    L, B = s0.shape[:2]
    cu = np.arange(0, L * B * n + 1, n)
    return oracle.gdr_recurrent(_pack(q, n), _pack(k, n), _pack(v, n), _pack(g, n),
                                _pack(beta, n), cu, z=_pack(z, n),
                                s0=f64(s0).reshape(L * B, *s0.shape[2:]),
                                w=None if w is None else f64(w), threads=THREADS)


def _bf16(a):
    return torch.from_numpy(a).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("B", [4, 32])
def test_headline_decode_as_benchmarked(B):
    steps = 16
    b = bench.DecodeBench("cuda", seed=1, B=B, slots=steps)
    assert b.overlap, "the benchmark overlaps the state loads of consecutive layers"
    b.capture()  # also runs slot 0 once, as the benchmark does before timing
    s0 = b.state.clone()
    outs = []
    for s in range(steps):
        b.run(s, 1)
        outs.append(b.out.clone())
    torch.cuda.synchronize()
    x = b.x
    ref = _oracle(x.q, x.k, x.v, x.z, x.g, x.beta, s0, x.w, steps)
    L = b.L
    got = torch.stack(outs, 1)  # [L, steps, B, H_v, d]
    got = f64(got.transpose(1, 2)).reshape(L * B * steps, *got.shape[3:])
    assert_close(got, _bf16(ref.y), 2e-3, "outputs (bf16)", bf16_ulp=True)
    fin = f64(b.state).reshape(L * B, *b.state.shape[2:])
    assert_close(fin, ref.state, 1e-3, "final states")
    per_layer = fin.reshape(L, -1)
    want = ref.state.reshape(L, -1)
    for l in range(L):
        assert_close(per_layer[l], want[l], 1e-3, f"final states of layer {l}")


@pytest.mark.parametrize("B", [4, 32])
def test_multi_token_decode_as_benchmarked(B):
    T, calls = 4, 4
    mb = bench.DecodeMultiBench("cuda", seed=12, B=B, slots=calls, T=T)
    mb.capture()  # runs call 0 once before capturing
    s0 = mb.state.clone()
    outs = []
    for c in range(calls):
        mb.run(c, 1)
        outs.append(mb.out.clone())  # [L, B*T, H_v, d]
    torch.cuda.synchronize()
    L = mb.L
    # Back to [L, tokens, B, ...]: call c, row b*T + t is token c*T + t of sequence b.
    unfold = lambda t: t.view(L, calls, B, T, *t.shape[3:]).transpose(2, 3).reshape(
        L, calls * T, B, *t.shape[3:])
    q, k, v, z, g, beta = (unfold(t) for t in (mb.q, mb.k, mb.v, mb.z, mb.g, mb.beta))
    ref = _oracle(q, k, v, z, g, beta, s0, None, calls * T)
    got = torch.stack(outs, 1).view(L, calls, B, T, *mb.out.shape[2:])
    got = f64(got.permute(0, 2, 1, 3, 4, 5)).reshape(L * B * calls * T, *mb.out.shape[2:])
    assert_close(got, _bf16(ref.y), 2e-3, "outputs (bf16)", bf16_ulp=True)
    fin = f64(mb.state).reshape(L * B, *mb.state.shape[2:])
    assert_close(fin, ref.state, 1e-3, "final states")
