"""The expiry path of the tensor-core prefill's bounded device waits.

Every device-side wait of the prefill's recurrence gives up after a deadline,
records GDR_ERR_TIMEOUT in the workspace status word, waits (bounded) for its
own copies in flight, frees its tensor memory and returns.  The self-test entry
point gdr_prefill_selftest_wait_expiry runs the ordinary two-kernel prefill with
a short deadline and each (sequence, head)'s first key tile never delivered --
a barrier nothing arrives at -- so that path runs without faulting or hanging
anything.  The test checks that the call finishes, that the status word reads
GDR_ERR_TIMEOUT, and that the GPU is left usable with its tensor memory free:
an ordinary prefill right after (whose recurrence allocates all 512 TMEM
columns of an SM) still matches the oracle.
"""
import ctypes
import time

import pytest
import torch

import linear_attention_recurrence_10_b200 as gdr
from gdr_testutil import TOL, assert_close, f64, oracle_full, run_prefill
from linear_attention_recurrence_10_b200 import _abi, synth

pytestmark = pytest.mark.gpu

GDR_ERR_TIMEOUT = 6


def test_wait_expiry_reports_timeout_and_leaves_gpu_usable():
    inp = synth.make_inputs([200, 130], 2, 4, 128, seed=600, dtype=torch.bfloat16, s0_std=0.02)
    x = inp.to("cuda")
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device="cuda")
    out = torch.zeros(inp.n_tok, inp.H_v, inp.d, device="cuda")
    final = torch.zeros(inp.n_seq, inp.H_v, inp.d, inp.d, device="cuda")
    n = gdr.prefill_workspace_size(x.q, x.k, x.v, x.g, x.beta, cu, out,
                                   cu_seqlens_host=inp.cu_seqlens, z=x.z, chunk=64)
    ws = torch.full((n,), 0xAB, dtype=torch.uint8, device="cuda")
    a, host = gdr._prefill_args(x.q, x.k, x.v, x.g, x.beta, cu, out, inp.cu_seqlens, x.z, x.w,
                                x.s0, final, 64, 1.0, 1e-6, 1e-6, True)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    st = _abi.lib().gdr_prefill_selftest_wait_expiry(ctypes.byref(a), ctypes.c_void_p(ws.data_ptr()),
                                                     n, 20_000_000, stream)  # 20 ms
    assert st == 0, gdr.status_string(st)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    del host
    assert ws[:4].view(torch.int32).item() == GDR_ERR_TIMEOUT
    assert elapsed < 5.0, f"unwinding took {elapsed:.2f} s"
    # The device is still usable and no tensor memory was left allocated.
    ref = oracle_full(inp)
    out2, final2 = run_prefill(inp, chunk=64)
    assert_close(f64(out2), ref.y, TOL[torch.bfloat16]["out"], "outputs after the expiry")
    assert_close(f64(final2), ref.state, TOL[torch.bfloat16]["state"], "states after the expiry")
