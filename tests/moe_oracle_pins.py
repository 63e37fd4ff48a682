"""Checks that pin the fp64 oracle of the routed-expert MoE block to facts other
than itself.

Each ``check_*`` takes an oracle library handle and raises AssertionError on a
mismatch, so the same checks run against the real oracle
(tests/test_moe_oracle.py) and against copies with a planted mistake, where at
least one must fail.

The block (Core AI card for Qwen3.6-35B-A3B, first section): a router
Linear(hidden, 256), a softmax over all experts, the top 8 renormalised by
their sum, SwitchGLU experts gathered by index, an always-on shared MLP scaled
by sigmoid(shared_expert_gate(x)), output = routed sum + gated shared.  What
pins what:
  * routing closed forms: logits ln 1 .. ln 4 give probabilities 0.1 .. 0.4 and
    top-2 weights 4/7, 3/7; zero router weights give 1/E everywhere, the
    lowest k indices and weights 1/k; the top-k are the k largest logits;
  * a SwitchGLU expert worked by hand (silu(ln 3) = 0.75 ln 3, silu(-ln 3) =
    -0.25 ln 3) through a 2 x 2 up/gate/down;
  * the shared expert's gate: sigmoid(0) = 1/2, saturation at +-50;
  * invariants: relabelling the experts changes nothing; the routed output is
    the weighted sum of single-expert outputs; linear in W_down.
"""
from __future__ import annotations

import math

import numpy as np

import oracle


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 0.0)
    assert np.isfinite(a).all() and err <= tol * scale, f"{what}: max error {err:.3e}"


def _weights(rng, E=6, H=8, I=4, SI=3):
    return dict(w_router=rng.standard_normal((E, H)), w_gate=rng.standard_normal((E, I, H)),
                w_up=rng.standard_normal((E, I, H)), w_down=rng.standard_normal((E, H, I)),
                shared=(rng.standard_normal((SI, H)), rng.standard_normal((SI, H)),
                        rng.standard_normal((H, SI)), rng.standard_normal(H)))


def _forward(lib, x, W, idx, w, shared=True):
    return oracle.moe_forward(x, W["w_router"], W["w_gate"], W["w_up"], W["w_down"], idx, w,
                              shared=W["shared"] if shared else None, lib=lib)


def check_moe_route_closed_form(lib):
    """One-hot x, router column ln(1..4): p = 0.1, 0.2, 0.3, 0.4; top-2 = 3, 2 with 4/7, 3/7."""
    x = np.array([[1.0, 0.0]])
    wr = np.array([[math.log(1), 5.0], [math.log(2), -1.0], [math.log(3), 0.0], [math.log(4), 2.0]])
    r = oracle.moe_route(x, wr, 2, lib=lib)
    _close(r.probs[0], [0.1, 0.2, 0.3, 0.4], 1e-15, "probabilities")
    assert r.idx[0].tolist() == [3, 2], r.idx
    _close(r.w[0], [4 / 7, 3 / 7], 1e-15, "renormalised weights")


def check_moe_route_uniform(lib):
    """Zero router weights: every probability 1/E; ties go to the lower index."""
    E, k = 8, 3
    r = oracle.moe_route(np.random.default_rng(1).standard_normal((2, 5)), np.zeros((E, 5)), k,
                         lib=lib)
    _close(r.probs, np.full((2, E), 1 / E), 1e-15, "uniform probabilities")
    assert r.idx.tolist() == [[0, 1, 2], [0, 1, 2]], r.idx
    _close(r.w, np.full((2, k), 1 / k), 1e-15, "uniform weights")


def check_moe_route_topk_are_largest_logits(lib):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 16))
    wr = rng.standard_normal((32, 16))
    r = oracle.moe_route(x, wr, 8, lib=lib)
    logits = x @ wr.T
    for t in range(5):
        want = sorted(range(32), key=lambda e: (-logits[t, e], e))[:8]
        assert r.idx[t].tolist() == want, (t, r.idx[t], want)
    _close(r.probs.sum(1), np.ones(5), 1e-14, "softmax sums to one")
    _close(r.w.sum(1), np.ones(5), 1e-14, "weights sum to one")


def check_moe_expert_by_hand(lib):
    """Expert 1 of 2 (k = 1, weight 1): x = (ln 3, -ln 3), W_gate = I, W_up swaps,
    W_down = [[1, 2], [3, 4]] -> y = (-1.25, -3.25) (ln 3)^2."""
    L = math.log(3.0)
    x = np.array([[L, -L]])
    W = dict(w_router=np.zeros((2, 2)),
             w_gate=np.array([np.zeros((2, 2)), np.eye(2)]),
             w_up=np.array([np.zeros((2, 2)), [[0.0, 1.0], [1.0, 0.0]]]),
             w_down=np.array([np.zeros((2, 2)), [[1.0, 2.0], [3.0, 4.0]]]), shared=None)
    y = _forward(lib, x, W, np.array([[1]]), np.array([[1.0]]), shared=False)
    _close(y[0], [-1.25 * L * L, -3.25 * L * L], 1e-14, "SwitchGLU by hand")


def check_moe_shared_gate(lib):
    """The shared expert's gate: w_sgate . x = 0 adds half of the shared
    SwitchGLU, +50 all of it, -50 none of it."""
    rng = np.random.default_rng(3)
    W = _weights(rng)
    x = rng.standard_normal((3, 8))
    x[:, 0] = 1.0
    sg, su, sd, _ = W["shared"]
    r = oracle.moe_route(x, W["w_router"], 2, lib=lib)
    routed = _forward(lib, x, W, r.idx, r.w, shared=False)

    def shared_part(c):  # w_sgate = c e_0, so w_sgate . x = c for every token
        Wc = dict(W, shared=(sg, su, sd, c * np.eye(8)[0]))
        return _forward(lib, x, Wc, r.idx, r.w) - routed

    half = shared_part(0.0)
    assert np.max(np.abs(half)) > 0
    _close(shared_part(50.0), 2.0 * half, 1e-13, "gate +50")
    _close(shared_part(-50.0), np.zeros_like(half), 1e-13, "gate -50")


def check_moe_relabel(lib):
    rng = np.random.default_rng(4)
    W = _weights(rng)
    x = rng.standard_normal((4, 8))
    r = oracle.moe_route(x, W["w_router"], 3, lib=lib)
    y = _forward(lib, x, W, r.idx, r.w)
    perm = rng.permutation(6)
    Wp = dict(W, w_router=W["w_router"][perm], w_gate=W["w_gate"][perm], w_up=W["w_up"][perm],
              w_down=W["w_down"][perm])
    rp = oracle.moe_route(x, Wp["w_router"], 3, lib=lib)
    assert (perm[rp.idx] == r.idx).all()
    _close(_forward(lib, x, Wp, rp.idx, rp.w), y, 1e-13, "relabelled experts")


def check_moe_weighted_sum_of_experts(lib):
    """The routed part equals the weighted sum of each selected expert alone."""
    rng = np.random.default_rng(5)
    W = _weights(rng)
    x = rng.standard_normal((3, 8))
    r = oracle.moe_route(x, W["w_router"], 4, lib=lib)
    y = _forward(lib, x, W, r.idx, r.w, shared=False)
    acc = np.zeros_like(y)
    for k in range(4):
        acc += r.w[:, k:k + 1] * _forward(lib, x, W, r.idx[:, k:k + 1], np.ones((3, 1)), shared=False)
    _close(y, acc, 1e-13, "sum of single experts")
    W2 = dict(W, w_down=2.0 * W["w_down"])
    _close(_forward(lib, x, W2, r.idx, r.w, shared=False), 2.0 * y, 1e-13, "linear in W_down")


ALL_CHECKS = [
    check_moe_route_closed_form, check_moe_route_uniform, check_moe_route_topk_are_largest_logits,
    check_moe_expert_by_hand, check_moe_shared_gate, check_moe_relabel,
    check_moe_weighted_sum_of_experts,
]
