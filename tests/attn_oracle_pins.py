"""Checks that pin the fp64 oracle of the gated full-attention decode step to
facts other than itself.

Each ``check_*`` takes an oracle library handle and raises AssertionError on a
mismatch, so the same checks run against the real oracle (tests/test_attn_oracle.py)
and against copies with a planted mistake, where at least one must fail.

The layer: standard scaled-dot-product attention over a KV cache with an output
gate (Qwen3.5 Chat guide, section "Architektur"), head_dim 256, GQA 16/2 and
partial rotary embedding with theta = 1e7 (Core AI card for Qwen3.6-35B-A3B,
first section).  What pins what:
  * closed forms of softmax attention: an empty cache returns the new value;
    equal keys give the mean of the values; orthonormal keys with the query
    along one of them give two distinct weights, e^{scale c} and 1;
  * the output gate: sigmoid(0) = 1/2, saturation at +-40;
  * invariants: GQA equals explicitly repeated key/value heads; the cached
    tokens' order does not matter; linearity in the values;
  * the rotary embedding: position 0 is the identity, each pair keeps its
    norm, the dimensions past rot_dim are untouched, rotations compose
    (pos a then b equals a + b), scores depend only on the relative position;
    a unit vector in dimension i turns within the plane (i, i + rot_dim/2) by
    the angle pos * theta^(-2i/rot_dim);
  * the layer rotates q and the new key at the position equal to the cache
    length: its result equals rotating them outside and running without RoPE.
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


def _problem(rng, B=2, H_q=4, H_kv=2, d=16, max_len=12, lens=(5, 9)):
    return dict(
        q=rng.standard_normal((B, H_q, d)), gate=rng.standard_normal((B, H_q, d)),
        k=rng.standard_normal((B, H_kv, d)), v=rng.standard_normal((B, H_kv, d)),
        k_cache=rng.standard_normal((B, H_kv, max_len, d)),
        v_cache=rng.standard_normal((B, H_kv, max_len, d)), cache_len=np.array(lens))


def _run(lib, p, **kw):
    return oracle.gated_attn_decode(p["q"], p["gate"], p["k"], p["v"], p["k_cache"], p["v_cache"],
                                    p["cache_len"], lib=lib, **kw)


def _kv_head(h, H_q, H_kv):
    return h * H_kv // H_q


def check_attn_empty_cache(lib):
    """One token attends only to itself: o = v of its key/value head, whatever q, k."""
    rng = np.random.default_rng(10)
    p = _problem(rng, lens=(0, 0))
    r = _run(lib, p, rot_dim=8)
    for h in range(4):
        _close(r.o[:, h], p["v"][:, _kv_head(h, 4, 2)], 1e-15, "empty cache")


def check_attn_equal_keys(lib):
    """All keys equal (no rotation): uniform weights, o = mean of the values."""
    rng = np.random.default_rng(11)
    p = _problem(rng)
    for b in range(2):
        for g in range(2):
            p["k_cache"][b, g, :] = p["k"][b, g]
    r = _run(lib, p, rot_dim=0)
    for b, L in enumerate(p["cache_len"]):
        for h in range(4):
            g = _kv_head(h, 4, 2)
            want = (p["v_cache"][b, g, :L].sum(0) + p["v"][b, g]) / (L + 1)
            _close(r.o[b, h], want, 1e-13, "equal keys")


def check_attn_orthonormal_keys(lib):
    """Keys e_0 .. e_{L-1} (cached) and e_L (new), query c e_j: weight e^{scale c}
    on token j and 1 on every other one."""
    d, L, c, scale = 16, 6, 3.0, 0.7
    rng = np.random.default_rng(12)
    p = _problem(rng, B=1, H_q=1, H_kv=1, d=d, max_len=8, lens=(L,))
    eye = np.eye(d)
    p["k_cache"][0, 0, :L] = eye[:L]
    p["k"][0, 0] = eye[L]
    for j in (0, 3, L):
        p["q"][0, 0] = c * eye[j]
        r = _run(lib, p, rot_dim=0, scale=scale)
        vals = np.concatenate([p["v_cache"][0, 0, :L], p["v"][0, :1]])
        wj = math.exp(scale * c)
        want = (wj * vals[j] + vals.sum(0) - vals[j]) / (wj + L)
        _close(r.o[0, 0], want, 1e-13, f"orthonormal keys, query along key {j}")


def check_attn_output_gate(lib):
    rng = np.random.default_rng(13)
    p = _problem(rng)
    for gval, factor in ((0.0, 0.5), (40.0, 1.0), (-40.0, 0.0)):
        p["gate"] = np.full_like(p["gate"], gval)
        r = _run(lib, p, rot_dim=8)
        _close(r.y, r.o * factor, 1e-15, f"gate {gval}")


def check_attn_gqa_equals_repeated(lib):
    """16 query heads over 2 key/value heads equal 16 over 16 with each key/value
    head repeated for its 8 consecutive query heads."""
    rng = np.random.default_rng(14)
    p = _problem(rng, H_q=16, H_kv=2)
    r = _run(lib, p, rot_dim=8)
    rep = {k: np.repeat(p[k], 8, axis=1) for k in ("k", "v", "k_cache", "v_cache")}
    q = dict(p, **rep)
    r2 = _run(lib, q, rot_dim=8)
    _close(r.y, r2.y, 0.0, "GQA vs repeated heads")


def check_attn_cache_order(lib):
    """Permuting the cached tokens (keys and values together) changes nothing."""
    rng = np.random.default_rng(15)
    p = _problem(rng)
    r = _run(lib, p, rot_dim=8)
    q = {k: v.copy() for k, v in p.items()}
    for b, L in enumerate(p["cache_len"]):
        perm = rng.permutation(L)
        q["k_cache"][b, :, :L] = p["k_cache"][b, :, perm].transpose(1, 0, 2)
        q["v_cache"][b, :, :L] = p["v_cache"][b, :, perm].transpose(1, 0, 2)
    r2 = _run(lib, q, rot_dim=8)
    _close(r2.y, r.y, 1e-12, "cache order")


def check_attn_linear_in_values(lib):
    rng = np.random.default_rng(16)
    p = _problem(rng)
    r = _run(lib, p, rot_dim=8)
    q = dict(p, v=3.0 * p["v"], v_cache=3.0 * p["v_cache"])
    r2 = _run(lib, q, rot_dim=8)
    _close(r2.o, 3.0 * r.o, 1e-13, "linear in V")


def check_rope_identities(lib):
    rng = np.random.default_rng(17)
    d, rot = 32, 8
    x = rng.standard_normal((5, d))
    y = rng.standard_normal((5, d))
    _close(oracle.rope_partial(x, 0.0, rot, lib=lib), x, 0.0, "position 0")
    for pos in (1.0, 7.0, 4096.0):
        r = oracle.rope_partial(x, pos, rot, lib=lib)
        _close(r[:, rot:], x[:, rot:], 0.0, "dims past rot_dim")
        h = rot // 2
        _close(r[:, :h] ** 2 + r[:, h:rot] ** 2, x[:, :h] ** 2 + x[:, h:rot] ** 2, 1e-13,
               "pair norms")
    a, b = 5.0, 11.0
    _close(oracle.rope_partial(oracle.rope_partial(x, a, rot, lib=lib), b, rot, lib=lib),
           oracle.rope_partial(x, a + b, rot, lib=lib), 1e-12, "composition")
    m, n = 23.0, 9.0
    lhs = np.sum(oracle.rope_partial(x, m, rot, lib=lib) * oracle.rope_partial(y, n, rot, lib=lib), 1)
    rhs = np.sum(oracle.rope_partial(x, m - n, rot, lib=lib) * y, 1)
    _close(lhs, rhs, 1e-12, "relative position")


def check_rope_plane_and_angle(lib):
    """e_i turns within the plane (i, i + rot/2) by pos * theta^(-2i/rot)."""
    d, rot, theta = 16, 8, 1e7
    h = rot // 2
    for i in range(h):
        x = np.zeros((1, d))
        x[0, i] = 1.0
        for pos in (1.0, 3.0):
            r = oracle.rope_partial(x, pos, rot, theta=theta, lib=lib)[0]
            others = np.delete(r, [i, i + h])
            _close(others, np.zeros_like(others), 0.0, f"e_{i} leaves its plane")
            ang = math.atan2(r[i + h], r[i])
            want = math.remainder(pos * theta ** (-2.0 * i / rot), 2 * math.pi)
            assert abs(math.remainder(ang - want, 2 * math.pi)) <= 1e-12, (i, pos, ang, want)


def check_attn_rotates_at_cache_length(lib):
    """RoPE inside the layer == q and the new key rotated outside at position
    cache_len[b], then the layer without RoPE."""
    rng = np.random.default_rng(18)
    rot = 8
    p = _problem(rng)
    r = _run(lib, p, rot_dim=rot)
    q = {k: v.copy() for k, v in p.items()}
    for b, L in enumerate(p["cache_len"]):
        q["q"][b] = oracle.rope_partial(p["q"][b], float(L), rot, lib=lib)
        q["k"][b] = oracle.rope_partial(p["k"][b], float(L), rot, lib=lib)
    r2 = _run(lib, q, rot_dim=0)
    _close(r.y, r2.y, 1e-13, "rotation at the cache length")
    _close(r.k_rot, q["k"], 0.0, "appended key is the rotated new key")


ALL_CHECKS = [
    check_attn_empty_cache, check_attn_equal_keys, check_attn_orthonormal_keys,
    check_attn_output_gate, check_attn_gqa_equals_repeated, check_attn_cache_order,
    check_attn_linear_in_values, check_rope_identities, check_rope_plane_and_angle,
    check_attn_rotates_at_cache_length,
]
