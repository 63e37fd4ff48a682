"""gdr_prefill_chunked_noalloc: the prefill entry point for callers that cannot
allocate device memory where they run it (for example a runtime that gives all
free device memory to its own pools at start-up).  It takes its workspace from
a fixed array inside the library instead of from the caller.

Checked through the C ABI against gdr_prefill_chunked with a caller-provided
workspace, on two calls in a row with different problems, so that anything the
first call leaves in the shared array would show up in the second.  This file
is named to be collected last."""
import ctypes

import pytest
import torch

import linear_attention_recurrence_10_b200 as gdr
from gdr_testutil import TOL, f64, rel_l2
from linear_attention_recurrence_10_b200 import _abi, synth

pytestmark = pytest.mark.gpu


def _problem(lens, seed):
    inp = synth.make_inputs(lens, 2, 4, 128, seed=seed, dtype=torch.bfloat16, s0_std=0.02)
    x = inp.to("cuda")
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device="cuda")
    return inp, x, cu


def _run(x, inp, cu, noalloc):
    out = torch.empty(inp.n_tok, inp.H_v, inp.d, device="cuda")
    final = torch.empty(inp.n_seq, inp.H_v, inp.d, inp.d, device="cuda")
    a, host = gdr._prefill_args(x.q, x.k, x.v, x.g, x.beta, cu, out, inp.cu_seqlens, x.z, x.w,
                                x.s0, final, 64, 1.0, 1e-6, 1e-6, True)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    lib = _abi.lib()
    if noalloc:
        st = lib.gdr_prefill_chunked_noalloc(ctypes.byref(a), stream)
    else:
        n = ctypes.c_size_t(0)
        assert lib.gdr_prefill_workspace_size(ctypes.byref(a), ctypes.byref(n)) == 0
        ws = torch.empty(max(int(n.value), 16), dtype=torch.uint8, device="cuda")
        st = lib.gdr_prefill_chunked(ctypes.byref(a), ctypes.c_void_p(ws.data_ptr()),
                                     ws.numel(), stream)
    torch.cuda.synchronize()
    assert st == 0, gdr.status_string(st)
    del host
    return out, final


def test_noalloc_matches_workspace_entry_point_twice():
    tol = TOL[torch.bfloat16]
    for lens, seed in (([300, 64, 1, 129], 401), ([70, 0, 513], 402)):
        inp, x, cu = _problem(lens, seed)
        ref_out, ref_state = _run(x, inp, cu, noalloc=False)
        out, state = _run(x, inp, cu, noalloc=True)
        assert rel_l2(f64(out), f64(ref_out)) <= tol["out"]
        assert rel_l2(f64(state), f64(ref_state)) <= tol["state"]


def test_noalloc_rejects_too_many_sequences():
    lens = [1] * (_abi.GDR_PREFILL_NOALLOC_MAX_SEQS + 1)
    inp, x, cu = _problem(lens, 403)
    out = torch.empty(inp.n_tok, inp.H_v, inp.d, device="cuda")
    with pytest.raises(gdr.GdrError, match="WORKSPACE"):
        gdr.prefill_chunked_noalloc(x.q, x.k, x.v, x.g, x.beta, cu, out,
                                    cu_seqlens_host=inp.cu_seqlens, z=x.z, chunk=64)
