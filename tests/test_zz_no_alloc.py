"""gdr_prefill_chunked_noalloc: the prefill entry point for callers that cannot
allocate device memory where they run it (for example a runtime that gives all
free device memory to its own pools at start-up, or a plain C caller with no
memory manager).  It takes its workspace from a fixed array inside the library
instead of from the caller.

Everything goes through the C ABI.  Each case runs the no-alloc call and the
workspace entry point on the same inputs and checks both against the fp64
oracle (and the no-alloc result against the workspace one), two problems in a
row so that anything the first call leaves in the shared array would show up in
the second, and reads the array's status word back through
gdr_prefill_noalloc_status.  The tensor-core path (bf16, d = 128) and the
CUDA-core path (fp32 inputs; d = 64) are both covered, as are a call with no
sequences and one whose sequences are all empty.  This file is named to be
collected last."""
import ctypes

import pytest
import torch

import linear_attention_recurrence_10_b200 as gdr
from gdr_testutil import TOL, assert_close, f64, oracle_full
from linear_attention_recurrence_10_b200 import _abi, synth

pytestmark = pytest.mark.gpu


def _problem(lens, seed, d=128, dtype=torch.bfloat16):
    inp = synth.make_inputs(lens, 2, 4, d, seed=seed, dtype=dtype, s0_std=0.02)
    x = inp.to("cuda")
    cu = torch.tensor(inp.cu_seqlens, dtype=torch.int32, device="cuda")
    return inp, x, cu


def _status():
    host = torch.full((1,), -1, dtype=torch.int32).pin_memory()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert _abi.lib().gdr_prefill_noalloc_status(host.data_ptr(), stream) == 0
    torch.cuda.synchronize()
    return int(host.item())


def _chunk(inp):
    """64 (the tensor cores) for bf16 with d = 128, else 32 (the CUDA cores)."""
    return 64 if inp.d == 128 and inp.q.dtype == torch.bfloat16 else 32


def _run(x, inp, cu, noalloc):
    out = torch.full((inp.n_tok, inp.H_v, inp.d), float("nan"), device="cuda")
    final = torch.full((inp.n_seq, inp.H_v, inp.d, inp.d), float("nan"), device="cuda")
    a, host = gdr._prefill_args(x.q, x.k, x.v, x.g, x.beta, cu, out, inp.cu_seqlens, x.z, x.w,
                                x.s0, final, _chunk(inp), 1.0, 1e-6, 1e-6, True)
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


@pytest.mark.parametrize("case", [
    # (lengths of the two problems in a row, d, input dtype)
    ((([300, 64, 1, 129], 401), ([70, 0, 513], 402)), 128, torch.bfloat16),
    ((([90, 33], 404), ([5, 200, 17], 405)), 128, torch.float32),
    ((([130, 1, 64], 406), ([0, 77], 407)), 64, torch.bfloat16),
], ids=["tensor-cores", "fp32-cuda-cores", "d64-cuda-cores"])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(case):
    problems, d, dtype = case
    tol = TOL[dtype]
    for lens, seed in problems:
        inp, x, cu = _problem(lens, seed, d, dtype)
        ref = oracle_full(inp)
        ws_out, ws_state = _run(x, inp, cu, noalloc=False)
        out, state = _run(x, inp, cu, noalloc=True)
        assert _status() == 0  # no device wait gave up
        assert_close(f64(out), ref.y, tol["out"], "no-alloc outputs")
        assert_close(f64(state), ref.state, tol["state"], "no-alloc final states")
        assert_close(f64(ws_out), ref.y, tol["out"], "workspace outputs")
        assert_close(f64(out), f64(ws_out), tol["out"], "no-alloc vs workspace outputs")
        assert_close(f64(state), f64(ws_state), tol["state"], "no-alloc vs workspace states")


def test_noalloc_no_sequences_and_all_empty():
    # No sequences at all: nothing to do, status word reads 0.
    inp, x, cu = _problem([], 408)
    out = torch.empty(0, inp.H_v, inp.d, device="cuda")
    gdr.prefill_chunked_noalloc(x.q, x.k, x.v, x.g, x.beta, cu, out, cu_seqlens_host=[0],
                                z=x.z, chunk=64)
    assert gdr.prefill_noalloc_status() == 0
    # Sequences that are all empty: the final state is the initial state.
    inp, x, cu = _problem([0, 0], 409)
    out, state = _run(x, inp, cu, noalloc=True)
    assert _status() == 0
    assert torch.equal(state, x.s0)


def test_noalloc_rejects_too_many_sequences():
    lens = [1] * (_abi.GDR_PREFILL_NOALLOC_MAX_SEQS + 1)
    inp, x, cu = _problem(lens, 403)
    out = torch.empty(inp.n_tok, inp.H_v, inp.d, device="cuda")
    with pytest.raises(gdr.GdrError, match="WORKSPACE"):
        gdr.prefill_chunked_noalloc(x.q, x.k, x.v, x.g, x.beta, cu, out,
                                    cu_seqlens_host=inp.cu_seqlens, z=x.z, chunk=64)
