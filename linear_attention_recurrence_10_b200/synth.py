"""Seeded synthetic inputs for the Gated DeltaNet mixer.

This module only draws numbers: it holds none of the mixer's arithmetic, so the
CUDA path and the fp64 oracle can both be fed from it without sharing any of
the method.  Every tensor is drawn from torch's own generator seeded by
(seed, tensor name), so a given (seed, name, shape, device) always yields the
same values.  The CPU and CUDA generators are different streams: tests draw on
the CPU and copy to the GPU; the benchmark draws on the GPU.

Value recipe (the workloads' stated distributions):
    q, k, v, z ~ N(0, 1), rounded once to the input dtype (bf16 by
                 round-to-nearest-even, or fp32)
    beta       = sigmoid(N(0, 1))                          fp32
    g          = -softplus(N(0, 1))  (log of the decay)     fp32
               or log(U[0.9, 1.0))  for the long-memory workload
    s0         ~ N(0, std) fp32, or absent (zeros)
    w          = 1 (fp32)
    lengths    ~ integer U{lo..hi}, inclusive
"""
from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import torch

def _seed_for(seed: int, name: str) -> int:
    return (int(seed) * 1_000_003 + zlib.crc32(name.encode())) & ((1 << 62) - 1)


def generator(seed: int, name: str, device="cpu") -> torch.Generator:
    gen = torch.Generator(device=device)
    gen.manual_seed(_seed_for(seed, name))
    return gen


def normal(shape, seed, name, std=1.0, device="cpu") -> torch.Tensor:
    x = torch.randn(tuple(shape), generator=generator(seed, name, device), device=device,
                    dtype=torch.float32)
    return x * std if std != 1.0 else x


def uniform(shape, seed, name, lo, hi, device="cpu") -> torch.Tensor:
    x = torch.rand(tuple(shape), generator=generator(seed, name, device), device=device,
                   dtype=torch.float64)
    return (lo + (hi - lo) * x).to(torch.float32)


def lengths(n, seed, lo, hi) -> list[int]:
    """n integers uniform in [lo, hi] (inclusive), drawn on the CPU."""
    x = torch.randint(int(lo), int(hi) + 1, (int(n),), generator=generator(seed, "len"))
    return [int(v) for v in x]


@dataclass
class Inputs:
    """Packed variable-length inputs: sequences laid end to end along tokens.

    q, k [n_tok, H_k, d]   v, z [n_tok, H_v, d]   g, beta [n_tok, H_v] fp32
    s0 [n_seq, H_v, d, d] fp32 or None   w [d] fp32   cu_seqlens: host list
    """
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    z: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    s0: torch.Tensor | None
    w: torch.Tensor
    cu_seqlens: list[int]
    H_k: int
    H_v: int
    d: int
    seed: int
    meta: dict = field(default_factory=dict)

    @property
    def n_tok(self) -> int:
        return self.cu_seqlens[-1]

    @property
    def n_seq(self) -> int:
        return len(self.cu_seqlens) - 1

    def to(self, device) -> "Inputs":
        mv = lambda t: None if t is None else t.to(device)
        return Inputs(mv(self.q), mv(self.k), mv(self.v), mv(self.z), mv(self.g),
                      mv(self.beta), mv(self.s0), mv(self.w), list(self.cu_seqlens),
                      self.H_k, self.H_v, self.d, self.seed, dict(self.meta))


def make_inputs(seqlens, H_k, H_v, d, *, seed, dtype=torch.bfloat16, g_mode="softplus",
                s0_std=None, device="cpu") -> Inputs:
    """Draw one packed problem.  ``g_mode`` is "softplus" (g = -softplus(N(0,1)))
    or "long" (g = log U[0.9, 1.0)).  ``s0_std`` None means a zero initial state."""
    seqlens = [int(s) for s in seqlens]
    cu = [0]
    for s in seqlens:
        cu.append(cu[-1] + s)
    n = cu[-1]
    q = normal((n, H_k, d), seed, "q", device=device).to(dtype)
    k = normal((n, H_k, d), seed, "k", device=device).to(dtype)
    v = normal((n, H_v, d), seed, "v", device=device).to(dtype)
    z = normal((n, H_v, d), seed, "z", device=device).to(dtype)
    beta = torch.sigmoid(normal((n, H_v), seed, "beta", device=device))
    if g_mode == "softplus":
        g = -torch.nn.functional.softplus(normal((n, H_v), seed, "g", device=device))
    elif g_mode == "long":
        g = torch.log(uniform((n, H_v), seed, "g", 0.9, 1.0, device=device))
    else:
        raise ValueError(f"unknown g_mode {g_mode!r}")
    s0 = None
    if s0_std is not None:
        s0 = normal((len(seqlens), H_v, d, d), seed, "s0", std=s0_std, device=device)
    w = torch.ones(d, dtype=torch.float32, device=device)
    return Inputs(q, k, v, z, g.contiguous(), beta.contiguous(), s0, w, cu, H_k, H_v, d,
                  seed, {"g_mode": g_mode, "s0_std": s0_std, "dtype": str(dtype)})


@dataclass
class DecodeInputs:
    """Per-step decode inputs for L independent layers: slot t of every tensor is
    the token that step t feeds to each of the B sequences.

    q, k [L, T, B, H_k, d]   v, z [L, T, B, H_v, d]   g, beta [L, T, B, H_v] fp32
    s0 [L, B, H_v, d, d] fp32   w [d] fp32
    """
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    z: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    s0: torch.Tensor
    w: torch.Tensor


def make_decode_inputs(L, T, B, H_k, H_v, d, *, seed, dtype=torch.bfloat16, s0_std=0.02,
                       g_mode="softplus", device="cpu") -> DecodeInputs:
    """Same value recipe as make_inputs, in the [layer, step, batch, head, dim] layout."""
    q = normal((L, T, B, H_k, d), seed, "q", device=device).to(dtype)
    k = normal((L, T, B, H_k, d), seed, "k", device=device).to(dtype)
    v = normal((L, T, B, H_v, d), seed, "v", device=device).to(dtype)
    z = normal((L, T, B, H_v, d), seed, "z", device=device).to(dtype)
    beta = torch.sigmoid(normal((L, T, B, H_v), seed, "beta", device=device))
    if g_mode == "softplus":
        g = -torch.nn.functional.softplus(normal((L, T, B, H_v), seed, "g", device=device))
    elif g_mode == "long":
        g = torch.log(uniform((L, T, B, H_v), seed, "g", 0.9, 1.0, device=device))
    else:
        raise ValueError(f"unknown g_mode {g_mode!r}")
    s0 = normal((L, B, H_v, d, d), seed, "s0", std=s0_std, device=device)
    w = torch.ones(d, dtype=torch.float32, device=device)
    return DecodeInputs(q, k, v, z, g.contiguous(), beta.contiguous(), s0, w)
