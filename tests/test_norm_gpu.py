"""gdr_rmsnorm_gated against the oracle's RMSNormGated (Qwen3.5 Chat guide,
section "Architektur": DeltaNet layers end in RMSNormGated)."""
import numpy as np
import pytest
import torch

import linear_attention_recurrence_10_b200 as gdr
import oracle
from gdr_testutil import f64, assert_close, rel_l2
from linear_attention_recurrence_10_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [16, 32, 64, 128])
@pytest.mark.parametrize("o_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("z_dtype", [torch.float32, torch.bfloat16])
def test_norm(d, o_dtype, z_dtype):
    rows = 1003  # a ragged last block
    o = synth.normal((rows, d), 30, "v").to(o_dtype)
    z = synth.normal((rows, d), 30, "z").to(z_dtype)
    w = synth.uniform((d,), 30, "w", 0.5, 1.5)
    want = oracle.rmsnorm_gated(f64(o), f64(z), f64(w), eps=1e-6)
    out = torch.empty(rows, d, device="cuda")
    gdr.rmsnorm_gated(o.cuda(), z.cuda(), out, w=w.cuda(), eps=1e-6)
    torch.cuda.synchronize()
    assert_close(f64(out), want, 1e-6)
    out16 = torch.empty(rows, d, device="cuda", dtype=torch.bfloat16)
    gdr.rmsnorm_gated(o.cuda(), z.cuda(), out16, w=w.cuda(), eps=1e-6)
    torch.cuda.synchronize()
    want16 = torch.from_numpy(want).to(torch.bfloat16).double().numpy()
    assert_close(f64(out16), want16, 2e-3, bf16_ulp=True)


def test_norm_in_place_and_no_weight():
    o = synth.normal((64, 4, 128), 31, "v").cuda()
    z = synth.normal((64, 4, 128), 31, "z").cuda()
    want = oracle.rmsnorm_gated(f64(o).reshape(-1, 128), f64(z).reshape(-1, 128), None, eps=1e-5)
    gdr.rmsnorm_gated(o, z, o, eps=1e-5)
    torch.cuda.synchronize()
    assert_close(f64(o).reshape(-1, 128), want, 1e-6)


def test_norm_empty():
    e = torch.empty(0, 128, device="cuda")
    gdr.rmsnorm_gated(e, e, e)
