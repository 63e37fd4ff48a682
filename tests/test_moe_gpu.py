"""Routed-expert MoE block at decode time (gdr_moe_decode) against the fp64 oracle.

The block is the FFN of the hybrid decoder's MoE models (Core AI card for
Qwen3.6-35B-A3B, first section: router over 256 experts, fp32 softmax, top 8
renormalised, SwitchGLU experts, a sigmoid-gated shared expert).  The oracle
receives the exact bf16 weights and activations widened to fp64.

Routing is a discrete decision: the kernel takes it in fp32 (as the card
states), the oracle in fp64, so the two may differ where two probabilities are
closer than fp32 can tell.  The tests therefore check that the kernel's chosen
set equals the oracle's top-k wherever the oracle's k-th and (k+1)-th
probabilities are apart by more than 1e-4 relative (a tie margin far above fp32
rounding of logits of size ~1), that any other choice is one the margin allows,
and compare the outputs and weights under the kernel's own routing (its chosen
experts with the oracle's renormalised weights).  Arithmetic is fp32 on bf16
inputs with 2048- and 512-term sums: the bar is a relative L2 of 1e-4 with the
element-wise bound of gdr_testutil.
"""
import numpy as np
import pytest
import torch

import linear_attention_recurrence_10_b200 as gdr
import oracle
from gdr_testutil import assert_close, f64

pytestmark = pytest.mark.gpu

TOL = 1e-4
TIE = 1e-4


def _weights(E, H, I, SI, seed):
    g = torch.Generator().manual_seed(seed)
    bf = lambda *s, std=1.0: (torch.randn(*s, generator=g) * std).to(torch.bfloat16)
    W = dict(w_router=bf(E, H, std=H ** -0.5), w_gate_up=bf(E, 2 * I, H, std=H ** -0.5),
             w_down=bf(E, H, I, std=I ** -0.5))
    shared = None
    if SI:
        shared = (bf(2 * SI, H, std=H ** -0.5), bf(H, SI, std=SI ** -0.5), bf(H, std=H ** -0.5))
    return W, shared, g


def _run(x, W, shared, k, out_dtype=torch.float32):
    d = lambda t: t.cuda()
    n, H = x.shape
    out = torch.full((n, H), float("nan"), device="cuda", dtype=out_dtype)
    idx = torch.full((n, k), -1, dtype=torch.int32, device="cuda")
    wts = torch.full((n, k), float("nan"), device="cuda")
    gdr.moe_decode(d(x), d(W["w_router"]), d(W["w_gate_up"]), d(W["w_down"]), out, top_k=k,
                   shared=None if shared is None else tuple(d(t) for t in shared),
                   topk_idx=idx, topk_w=wts)
    torch.cuda.synchronize()
    return out, idx.cpu().numpy(), wts.cpu().numpy()


def _oracle_args(W, shared):
    E, twoI, H = W["w_gate_up"].shape
    I = twoI // 2
    gu = f64(W["w_gate_up"])
    sh = None
    if shared is not None:
        sgu, sd, sg = (f64(t) for t in shared)
        SI = sgu.shape[0] // 2
        sh = (sgu[:SI], sgu[SI:], sd, sg)
    return dict(w_gate=gu[:, :I], w_up=gu[:, I:], w_down=f64(W["w_down"])), sh


def _check(x, W, shared, k, out, idx, wts, out_tol=TOL, bf16_ulp=False):
    ref_route = oracle.moe_route(f64(x), f64(W["w_router"]), k)
    probs = ref_route.probs
    n = x.shape[0]
    for t in range(n):
        order = np.argsort(-probs[t], kind="stable")
        pk, pk1 = probs[t, order[k - 1]], probs[t, order[k]] if k < probs.shape[1] else 0.0
        mine = sorted(idx[t].tolist())
        if pk - pk1 > TIE * pk:
            assert mine == sorted(ref_route.idx[t].tolist()), (t, idx[t], ref_route.idx[t])
        else:  # a near-tie at the boundary: any choice among the tied experts is valid
            lo = pk1 - TIE * pk
            assert all(probs[t, e] >= lo for e in mine), (t, idx[t])
        assert len(set(mine)) == k
        # weights: the oracle's probabilities renormalised over the kernel's choice
        want_w = probs[t, idx[t]] / probs[t, idx[t]].sum()
        assert np.allclose(wts[t], want_w, rtol=1e-5, atol=1e-7), (t, wts[t], want_w)
        assert all(probs[t, idx[t][i]] >= probs[t, idx[t][i + 1]] - TIE * pk for i in range(k - 1))
    ow, sh = _oracle_args(W, shared)
    w_ref = np.stack([probs[t, idx[t]] / probs[t, idx[t]].sum() for t in range(n)])
    y = oracle.moe_forward(f64(x), f64(W["w_router"]), ow["w_gate"], ow["w_up"], ow["w_down"],
                           idx, w_ref, shared=sh)
    if bf16_ulp:
        y = torch.from_numpy(y).to(torch.bfloat16).double().numpy()
    assert_close(f64(out), y, out_tol, "MoE outputs", bf16_ulp=bf16_ulp)


@pytest.mark.parametrize("n_tok", [1, 3, 16])
@pytest.mark.parametrize("with_shared", [True, False])
def test_small_moe_matches_oracle(n_tok, with_shared):
    E, H, I, SI, k = 32, 256, 64, 64, 4
    W, shared, g = _weights(E, H, I, SI if with_shared else 0, seed=800 + n_tok)
    x = torch.randn(n_tok, H, generator=g).to(torch.bfloat16)
    out, idx, wts = _run(x, W, shared, k)
    _check(x, W, shared, k, out, idx, wts)


def test_bf16_output_and_every_expert_chosen():
    """64 tokens over 16 experts with k = 8: nearly every expert is active and
    most see many tokens (the grouped path); bf16 output."""
    E, H, I, SI, k = 16, 512, 128, 96, 8
    W, shared, g = _weights(E, H, I, SI, seed=810)
    x = torch.randn(64, H, generator=g).to(torch.bfloat16)
    out, idx, wts = _run(x, W, shared, k, out_dtype=torch.bfloat16)
    _check(x, W, shared, k, out, idx, wts, bf16_ulp=True)


@pytest.mark.slow
@pytest.mark.parametrize("n_tok", [1, 8])
def test_qwen36_moe_shape(n_tok):
    """Qwen3.6-35B-A3B-shaped block: hidden 2048, 256 experts, top 8, expert
    and shared intermediate 512."""
    E, H, I, SI, k = 256, 2048, 512, 512, 8
    W, shared, g = _weights(E, H, I, SI, seed=820 + n_tok)
    x = torch.randn(n_tok, H, generator=g).to(torch.bfloat16)
    out, idx, wts = _run(x, W, shared, k)
    _check(x, W, shared, k, out, idx, wts)
