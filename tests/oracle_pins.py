"""Checks that pin the fp64 oracle to facts other than itself.

Each ``check_*`` takes an oracle library handle (``oracle.load(path)``) and
raises AssertionError on a mismatch, so the same checks can run against the
real oracle (tests/test_oracle.py) and against copies with a planted mistake
(tests/test_oracle_mutations.py), where at least one of them must fail.

What pins what (none of these re-types the oracle's own loops):
  * closed forms of the gated delta rule (Gated Delta Networks, Yang, Kautz,
    Hatamizadeh, ICLR 2025; the mixer named in the Qwen3.5 Chat guide,
    section "Architektur"):
      - beta = 0, g = 0: the state never changes, o_t = S_0 q_t
      - beta = 1, unit k: S_t k_t = v_t (delta-rule retrieval), so q = k gives o_t = v_t
      - g = -inf: the state restarts, S_t = beta_t v_t k_t^T
      - beta = 0: pure decay, S_t = exp(sum g) S_0
      - g = 0, beta = 1, orthonormal keys: S_T = S_0 (I - sum k k^T) + sum v k^T
  * a hand-worked d = 2, T = 2 example (tests/golden/handworked_d2_t2.txt)
  * three forms computed three ways: recurrence, chunkwise WY/UT form (any
    chunk, ragged last chunk) and explicit transition-matrix products (T <= 8)
  * invariants: linearity in (V, S_0); permuting value dimensions; GVA equals
    explicitly repeated key heads (the Core AI Qwen3.6 card: each k/q head
    serves two value heads); packed sequences equal separate runs; splitting a
    sequence and handing the state over equals one run (Swiftlet post,
    "Correctness & Validation": incremental equals whole-sequence); the
    Frobenius contraction bound of each step
  * RMSNormGated: positive-scale invariance, z = 0 gives 0, a hand-worked row
"""
from __future__ import annotations

import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_problem(rng, seqlens, H_k=1, H_v=1, d=4, s0=True, z=True):
    n = int(sum(seqlens))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int64)
    p = dict(
        q=rng.standard_normal((n, H_k, d)),
        k=rng.standard_normal((n, H_k, d)),
        v=rng.standard_normal((n, H_v, d)),
        g=-np.log1p(np.exp(rng.standard_normal((n, H_v)))),
        beta=1.0 / (1.0 + np.exp(-rng.standard_normal((n, H_v)))),
        cu_seqlens=cu,
    )
    if z:
        p["z"] = rng.standard_normal((n, H_v, d))
        p["w"] = 0.5 + rng.random(d)
    if s0:
        p["s0"] = 0.3 * rng.standard_normal((len(seqlens), H_v, d, d))
    return p


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _close(a, b, tol, what):
    a = np.asarray(a); b = np.asarray(b)
    err = np.max(np.abs(a - b)) / max(1.0, np.max(np.abs(b)))
    assert err <= tol, f"{what}: max error {err:.3e} > {tol:.1e}"


# ------------------------------------------------------------- closed forms

def check_beta0_g0_identity(lib):
    rng = np.random.default_rng(1)
    p = _rand_problem(rng, [5, 3], H_k=2, H_v=2, d=4)
    p["beta"][:] = 0.0
    p["g"][:] = 0.0
    for fn in (oracle.gdr_recurrent, oracle.gdr_bruteforce):
        r = fn(**p, eps_l2=0.0, lib=lib)
        _close(r.state, p["s0"], 1e-13, f"{fn.__name__}: state after beta=0,g=0")
        qh = _unit(p["q"])
        for s in range(2):
            for t in range(p["cu_seqlens"][s], p["cu_seqlens"][s + 1]):
                for h in range(2):
                    _close(r.o[t, h], p["s0"][s, h] @ qh[t, h], 1e-13, "o = S_0 q")


def check_retrieval_beta1(lib):
    """beta = 1 with unit keys writes v exactly: S_t k_t = v_t; with q = k, o_t = v_t."""
    rng = np.random.default_rng(2)
    p = _rand_problem(rng, [7, 4], H_k=1, H_v=2, d=5)
    p["beta"][:] = 1.0
    p["q"] = p["k"].copy()
    for fn, kw in ((oracle.gdr_recurrent, {}), (oracle.gdr_chunked, {"chunk": 3}),
                   (oracle.gdr_bruteforce, {})):
        r = fn(**p, eps_l2=0.0, lib=lib, **kw)
        _close(r.o, p["v"], 1e-12, f"{fn.__name__}: retrieval o_t = v_t")
        kh = _unit(p["k"])
        for s, last in enumerate(p["cu_seqlens"][1:] - 1):
            for h in range(2):
                _close(r.state[s, h] @ kh[last, 0], p["v"][last, h], 1e-12,
                       "retrieval S_T k_T = v_T")


def check_reset_neg_inf(lib):
    """g = -inf erases the past: S_t = beta_t v_t k_t^T and o_t = beta_t v_t (k_t . q_t)."""
    rng = np.random.default_rng(3)
    p = _rand_problem(rng, [6], H_k=1, H_v=1, d=4)
    reset = [2, 5]
    p["g"][reset, 0] = -np.inf
    qh = _unit(p["q"]); kh = _unit(p["k"])
    for fn, kw in ((oracle.gdr_recurrent, {}), (oracle.gdr_chunked, {"chunk": 4}),
                   (oracle.gdr_bruteforce, {})):
        r = fn(**p, eps_l2=0.0, lib=lib, **kw)
        for t in reset:
            b = p["beta"][t, 0]
            _close(r.o[t, 0], b * p["v"][t, 0] * (kh[t, 0] @ qh[t, 0]), 1e-12,
                   f"{fn.__name__}: o at a reset")
        _close(r.state[0, 0], p["beta"][5, 0] * np.outer(p["v"][5, 0], kh[5, 0]), 1e-12,
               f"{fn.__name__}: state after a reset")


def check_pure_decay(lib):
    """beta = 0: S_t = exp(g_1 + ... + g_t) S_0 and o_t = S_t q_t."""
    rng = np.random.default_rng(4)
    p = _rand_problem(rng, [9], H_k=1, H_v=1, d=3)
    p["beta"][:] = 0.0
    qh = _unit(p["q"])
    for fn, kw in ((oracle.gdr_recurrent, {}), (oracle.gdr_chunked, {"chunk": 4})):
        r = fn(**p, eps_l2=0.0, lib=lib, **kw)
        G = np.cumsum(p["g"][:, 0])
        for t in range(9):
            _close(r.o[t, 0], math.exp(G[t]) * p["s0"][0, 0] @ qh[t, 0], 1e-12,
                   f"{fn.__name__}: decayed readout")
        _close(r.state[0, 0], math.exp(G[-1]) * p["s0"][0, 0], 1e-12, "decayed state")


def check_orthonormal_keys(lib):
    """g = 0, beta = 1, orthonormal k_1..k_T: S_T = S_0 (I - sum k k^T) + sum v k^T."""
    rng = np.random.default_rng(5)
    d, T = 6, 4
    p = _rand_problem(rng, [T], H_k=1, H_v=1, d=d)
    basis, _ = np.linalg.qr(rng.standard_normal((d, d)))
    p["k"][:, 0] = basis[:, :T].T
    p["g"][:] = 0.0
    p["beta"][:] = 1.0
    want = p["s0"][0, 0] @ (np.eye(d) - p["k"][:, 0].T @ p["k"][:, 0]) + p["v"][:, 0].T @ p["k"][:, 0]
    for fn, kw in ((oracle.gdr_recurrent, {}), (oracle.gdr_chunked, {"chunk": 3}),
                   (oracle.gdr_bruteforce, {})):
        r = fn(**p, eps_l2=0.0, lib=lib, **kw)
        _close(r.state[0, 0], want, 1e-12, f"{fn.__name__}: orthonormal-key closed form")


def read_handworked():
    vals = {}
    with open(os.path.join(GOLDEN, "handworked_d2_t2.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rhs = line.split("=", 1)
            vals[key.strip()] = np.array([float(x) for x in rhs.split()])
    return vals


def check_handworked(lib):
    """The d = 2, T = 2 example worked by hand in tests/golden/handworked_d2_t2.txt."""
    h = read_handworked()
    q = np.stack([h["q1"], h["q2"]])[:, None, :]
    k = np.stack([h["k1"], h["k2"]])[:, None, :]
    v = np.stack([h["v1"], h["v2"]])[:, None, :]
    z = np.stack([h["z1"], h["z2"]])[:, None, :]
    g = np.log(np.array([[h["alpha"][0]], [h["alpha"][1]]]))
    beta = np.array([[h["beta"][0]], [h["beta"][1]]])
    args = dict(q=q, k=k, v=v, g=g, beta=beta, cu_seqlens=[0, 2], z=z, w=h["w"],
                eps_l2=0.0, eps_norm=0.0, qk_l2norm=False)
    for fn, kw in ((oracle.gdr_recurrent, {}), (oracle.gdr_chunked, {"chunk": 2}),
                   (oracle.gdr_bruteforce, {})):
        r = fn(**args, lib=lib, **kw)
        _close(r.o[0, 0], h["o1"], 1e-14, f"{fn.__name__}: hand-worked o_1")
        _close(r.o[1, 0], h["o2"], 1e-14, f"{fn.__name__}: hand-worked o_2")
        _close(r.state[0, 0].ravel(), h["S2"], 1e-14, f"{fn.__name__}: hand-worked S_2")
        _close(r.y[0, 0], h["y1"], 1e-13, f"{fn.__name__}: hand-worked y_1")
        _close(r.y[1, 0], h["y2"], 1e-13, f"{fn.__name__}: hand-worked y_2")


# ------------------------------------------------------- three forms agree

def check_bruteforce_equals_recurrent(lib):
    rng = np.random.default_rng(6)
    p = _rand_problem(rng, [8, 1, 5, 0, 3], H_k=2, H_v=4, d=5)
    a = oracle.gdr_recurrent(**p, lib=lib)
    b = oracle.gdr_bruteforce(**p, lib=lib)
    _close(a.o, b.o, 1e-12, "brute force vs recurrent: o")
    _close(a.y, b.y, 1e-12, "brute force vs recurrent: y")
    _close(a.state, b.state, 1e-12, "brute force vs recurrent: state")


def check_chunked_equals_recurrent(lib):
    rng = np.random.default_rng(7)
    p = _rand_problem(rng, [37, 64, 1, 16, 70], H_k=1, H_v=2, d=8)
    a = oracle.gdr_recurrent(**p, lib=lib)
    for C in (1, 4, 16, 64):
        b = oracle.gdr_chunked(**p, chunk=C, lib=lib)
        _close(b.o, a.o, 1e-12, f"chunked C={C} vs recurrent: o")
        _close(b.y, a.y, 1e-12, f"chunked C={C} vs recurrent: y")
        _close(b.state, a.state, 1e-12, f"chunked C={C} vs recurrent: state")


# ---------------------------------------------------------------- invariants

def check_linearity(lib):
    """o and S are jointly linear in (V, S_0) for fixed q, k, g, beta."""
    rng = np.random.default_rng(8)
    p1 = _rand_problem(rng, [6, 4], H_k=1, H_v=1, d=4, z=False)
    p2 = dict(p1, v=rng.standard_normal(p1["v"].shape), s0=rng.standard_normal(p1["s0"].shape))
    a, b = 0.7, -1.9
    p3 = dict(p1, v=a * p1["v"] + b * p2["v"], s0=a * p1["s0"] + b * p2["s0"])
    r1, r2, r3 = (oracle.gdr_recurrent(**pp, lib=lib) for pp in (p1, p2, p3))
    _close(r3.o, a * r1.o + b * r2.o, 1e-12, "linearity of o")
    _close(r3.state, a * r1.state + b * r2.state, 1e-12, "linearity of S")


def check_value_permutation(lib):
    """Permuting value dimensions of V, S_0 rows, w and z permutes o, y and S rows."""
    rng = np.random.default_rng(9)
    p = _rand_problem(rng, [7], H_k=1, H_v=1, d=5)
    perm = rng.permutation(5)
    pp = dict(p, v=p["v"][..., perm], z=p["z"][..., perm], w=p["w"][perm],
              s0=p["s0"][:, :, perm, :])
    a = oracle.gdr_recurrent(**p, lib=lib)
    b = oracle.gdr_recurrent(**pp, lib=lib)
    _close(b.o, a.o[..., perm], 1e-13, "permuted o")
    _close(b.y, a.y[..., perm], 1e-13, "permuted y")
    _close(b.state, a.state[:, :, perm, :], 1e-13, "permuted S")


def check_gva_equals_expanded(lib):
    """H_v = 2 H_k with shared key heads equals the run with each key head repeated
    for its two value heads (value heads 2j and 2j+1 read key head j)."""
    rng = np.random.default_rng(10)
    p = _rand_problem(rng, [5, 6], H_k=2, H_v=4, d=4)
    pe = dict(p, q=np.repeat(p["q"], 2, axis=1), k=np.repeat(p["k"], 2, axis=1))
    a = oracle.gdr_recurrent(**p, lib=lib)
    b = oracle.gdr_recurrent(**pe, lib=lib)
    assert np.array_equal(a.o, b.o) and np.array_equal(a.state, b.state), "GVA vs expanded"


def check_varlen_equals_separate(lib):
    rng = np.random.default_rng(11)
    lens = [4, 9, 2]
    p = _rand_problem(rng, lens, H_k=1, H_v=2, d=4)
    a = oracle.gdr_recurrent(**p, lib=lib)
    cu = p["cu_seqlens"]
    for s in range(3):
        sl = slice(cu[s], cu[s + 1])
        ps = dict(q=p["q"][sl], k=p["k"][sl], v=p["v"][sl], z=p["z"][sl], g=p["g"][sl],
                  beta=p["beta"][sl], w=p["w"], s0=p["s0"][s:s + 1], cu_seqlens=[0, lens[s]])
        b = oracle.gdr_recurrent(**ps, lib=lib)
        _close(a.o[sl], b.o, 0.0, "packed vs separate: o")
        _close(a.state[s], b.state[0], 0.0, "packed vs separate: state")


def check_split_handoff(lib):
    """Run tokens [0, m) then [m, T) with the state handed over == one run of T."""
    rng = np.random.default_rng(12)
    T, m = 11, 4
    p = _rand_problem(rng, [T], H_k=1, H_v=1, d=4)
    whole = oracle.gdr_recurrent(**p, lib=lib)
    pa = {k: (v[:m] if k in ("q", "k", "v", "z", "g", "beta") else v) for k, v in p.items()}
    pa["cu_seqlens"] = [0, m]
    a = oracle.gdr_recurrent(**pa, lib=lib)
    pb = {k: (v[m:] if k in ("q", "k", "v", "z", "g", "beta") else v) for k, v in p.items()}
    pb["cu_seqlens"] = [0, T - m]
    pb["s0"] = a.state
    b = oracle.gdr_recurrent(**pb, lib=lib)
    _close(np.concatenate([a.o, b.o]), whole.o, 1e-13, "split vs whole: o")
    _close(b.state, whole.state, 1e-13, "split vs whole: state")


def check_contraction_bound(lib):
    """For beta in [0, 1] and unit k, |S_t|_F <= alpha_t |S_{t-1}|_F + beta_t |v_t|."""
    rng = np.random.default_rng(13)
    T = 10
    p = _rand_problem(rng, [T], H_k=1, H_v=1, d=4)
    prev = np.linalg.norm(p["s0"][0, 0])
    s0 = p["s0"]
    for t in range(T):
        pt = {k: (v[t:t + 1] if k in ("q", "k", "v", "z", "g", "beta") else v)
              for k, v in p.items()}
        pt["cu_seqlens"] = [0, 1]
        pt["s0"] = s0
        r = oracle.gdr_recurrent(**pt, eps_l2=0.0, lib=lib)
        cur = np.linalg.norm(r.state[0, 0])
        bound = math.exp(p["g"][t, 0]) * prev + p["beta"][t, 0] * np.linalg.norm(p["v"][t, 0])
        assert cur <= bound * (1 + 1e-12), f"contraction bound broken at t={t}"
        # the step must also actually move the state (rules out a no-op step)
        assert not np.allclose(r.state, s0), f"state did not change at t={t}"
        prev, s0 = cur, r.state


def check_qk_normalisation(lib):
    """With L2 normalisation on, positive rescaling of q and k changes nothing
    (eps_l2 = 0), and `scale` multiplies o."""
    rng = np.random.default_rng(14)
    p = _rand_problem(rng, [6], H_k=1, H_v=1, d=4)
    a = oracle.gdr_recurrent(**p, eps_l2=0.0, lib=lib)
    b = oracle.gdr_recurrent(**dict(p, q=3.0 * p["q"], k=0.25 * p["k"]), eps_l2=0.0, lib=lib)
    _close(b.o, a.o, 1e-13, "q, k rescaling")
    c = oracle.gdr_recurrent(**p, eps_l2=0.0, scale=0.125, lib=lib)
    _close(c.o, 0.125 * a.o, 1e-13, "scale multiplies o")
    _close(c.state, a.state, 1e-13, "scale leaves S alone")


# ----------------------------------------------------------- RMSNormGated

def check_rmsnorm_gated(lib):
    rng = np.random.default_rng(15)
    o = rng.standard_normal((5, 8))
    z = rng.standard_normal((5, 8))
    w = rng.random(8) + 0.5
    y = oracle.rmsnorm_gated(o, z, w, eps=0.0, lib=lib)
    _close(oracle.rmsnorm_gated(7.5 * o, z, w, eps=0.0, lib=lib), y, 1e-13, "scale invariance")
    assert np.all(oracle.rmsnorm_gated(o, np.zeros_like(z), w, eps=0.0, lib=lib) == 0.0)
    # Hand-worked row: o = (3, 4), mean(o^2) = 12.5, so o / rms = (3, 4) / sqrt(12.5);
    # z = (ln 3, -ln 3): sigmoid = (3/4, 1/4), SiLU = (0.75 ln 3, -0.25 ln 3); w = (2, 1).
    l3 = math.log(3.0)
    r = math.sqrt(12.5)
    want = np.array([3.0 / r * 2.0 * 0.75 * l3, 4.0 / r * 1.0 * (-0.25 * l3)])
    got = oracle.rmsnorm_gated(np.array([[3.0, 4.0]]), np.array([[l3, -l3]]),
                               np.array([2.0, 1.0]), eps=0.0, lib=lib)
    _close(got[0], want, 1e-14, "hand-worked RMSNormGated row")
    # eps enters under the root: o = (1, 1), eps = 3 -> 1 / sqrt(1 + 3) = 1/2.
    got = oracle.rmsnorm_gated(np.array([[1.0, 1.0]]), np.array([[l3, l3]]), None, eps=3.0,
                               lib=lib)
    _close(got[0], np.array([0.5 * 0.75 * l3] * 2), 1e-14, "eps of the RMS norm")


def check_gate_from_raw_closed_forms(lib):
    """g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b) (the Gated DeltaNet
    parameterisation; the pages only say the layer is a Gated DeltaNet) at points
    whose values are known exactly: softplus(0) = ln 2, softplus(x) = x + log1p(e^-x)
    for large x, no overflow at +-800, sigmoid(0) = 1/2."""
    a = np.array([[0.0, -3.0], [50.0, -800.0], [800.0, 2.0]])
    b = np.array([[0.0, 1.0], [-1.0, 40.0], [-800.0, 3.0]])
    A_log = np.array([0.0, math.log(2.0)])
    dt_bias = np.array([0.0, 3.0])
    g, beta = oracle.gate_from_raw(a, b, A_log, dt_bias, lib=lib)
    # x = a + dt_bias = 0 -> softplus = ln 2; head 1 scales by exp(ln 2) = 2.
    _close(g[0, 0], -math.log(2.0), 1e-15, "softplus(0)")
    _close(g[0, 1], -2.0 * math.log(2.0), 1e-15, "dt_bias shift and exp(A_log)")
    _close(g[1, 0], -(50.0 + math.log1p(math.exp(-50.0))), 1e-15, "softplus(50)")
    assert g[1, 1] == 0.0, "softplus(-797) underflows to 0"
    _close(g[2, 0], -800.0, 1e-15, "softplus(800) without overflow")
    assert beta[0, 0] == 0.5 and beta[2, 0] == 0.0, "sigmoid(0), sigmoid(-800)"
    assert abs(beta[1, 1] - 1.0) <= 1e-15, "sigmoid(40)"
    _close(beta[0, 1], 1.0 / (1.0 + math.exp(-1.0)), 1e-15, "sigmoid(1)")


def check_gate_from_raw_identities(lib):
    """softplus(x) - softplus(-x) = x and sigmoid(x) + sigmoid(-x) = 1; A_log = -inf
    turns the decay off; decays are never positive; dt_bias shifts the argument."""
    rng = np.random.default_rng(5)
    a = rng.normal(size=(40, 3)) * 4
    b = rng.normal(size=(40, 3)) * 4
    zero = np.zeros(3)
    g_pos, beta_pos = oracle.gate_from_raw(a, b, zero, zero, lib=lib)
    g_neg, beta_neg = oracle.gate_from_raw(-a, -b, zero, zero, lib=lib)
    assert np.max(np.abs(-g_pos + g_neg - a)) <= 1e-13, "softplus(x) - softplus(-x) = x"
    assert np.max(np.abs(beta_pos + beta_neg - 1.0)) <= 1e-15, "sigmoid(x) + sigmoid(-x) = 1"
    g_off, _ = oracle.gate_from_raw(a, b, np.full(3, -np.inf), zero, lib=lib)
    assert np.all(g_off == 0.0) and np.all(g_pos < 0), "no decay at A_log = -inf; g < 0"
    c = np.array([0.5, -1.0, 2.0])
    g1, _ = oracle.gate_from_raw(a, b, zero, c, lib=lib)
    g2, _ = oracle.gate_from_raw(a + c, b, zero, zero, lib=lib)
    assert np.array_equal(g1, g2), "dt_bias shifts the softplus argument"


ALL_CHECKS = [
    check_beta0_g0_identity, check_retrieval_beta1, check_reset_neg_inf, check_pure_decay,
    check_orthonormal_keys, check_handworked, check_bruteforce_equals_recurrent,
    check_chunked_equals_recurrent, check_linearity, check_value_permutation,
    check_gva_equals_expanded, check_varlen_equals_separate, check_split_handoff,
    check_contraction_bound, check_qk_normalisation, check_rmsnorm_gated,
    check_gate_from_raw_closed_forms, check_gate_from_raw_identities,
]
