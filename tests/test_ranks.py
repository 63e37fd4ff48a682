"""Multi-rank host logic, on the CPU: splitting work over ranks, the
max-over-ranks time and the whole-job rate, and a world-size-2 gloo run in
which each rank solves its shard of a varlen problem and the gathered result
equals one whole-problem solve (the mixer has no cross-sequence exchange)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from linear_attention_recurrence_10_b200 import ranks, synth


def test_rank_env_defaults_and_torchrun():
    assert ranks.rank_env({}) == ranks.RankEnv(0, 1, 0)
    assert ranks.rank_env({"RANK": "3", "WORLD_SIZE": "4", "LOCAL_RANK": "1"}) == \
        ranks.RankEnv(3, 4, 1)
    with pytest.raises(ValueError):
        ranks.rank_env({"RANK": "4", "WORLD_SIZE": "4"})


@pytest.mark.parametrize("B,world", [(0, 1), (1, 2), (32, 1), (32, 3), (7, 8), (64, 8)])
def test_batch_slice_partitions(B, world):
    seen = []
    sizes = []
    for r in range(world):
        sl = ranks.batch_slice(B, r, world)
        seen.extend(sl)
        sizes.append(len(sl))
    assert seen == list(range(B))  # contiguous, in rank order, no overlap
    assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_partition_by_tokens(world):
    lens = synth.lengths(23, seed=4, lo=1024, hi=32768)
    parts = ranks.partition_by_tokens(lens, world)
    flat = sorted(i for p in parts for i in p)
    assert flat == list(range(len(lens)))
    loads = [sum(lens[i] for i in p) for p in parts]
    # LPT bound: the heaviest rank exceeds the mean by at most one sequence.
    assert max(loads) <= sum(lens) / world + max(lens)
    for p in parts:
        assert p == sorted(p)


def test_partition_by_tokens_optimal_on_small_cases():
    # Brute force on tiny cases: LPT stays within 4/3 of the best split.
    import itertools
    rng = np.random.default_rng(0)
    for _ in range(30):
        lens = [int(x) for x in rng.integers(1, 50, size=6)]
        best = min(max(sum(l for l, a in zip(lens, asg) if a == r) for r in range(2))
                   for asg in itertools.product(range(2), repeat=len(lens)))
        got = max(sum(lens[i] for i in p) for p in ranks.partition_by_tokens(lens, 2))
        assert got <= 4 / 3 * best + 1e-9


def test_weak_scaling_rate():
    assert ranks.weak_scaling_rate(1000, 4, 2.0) == pytest.approx(2e6)
    with pytest.raises(ValueError):
        ranks.weak_scaling_rate(1, 1, 0.0)


def test_shard_inputs_is_the_packed_subset():
    inp = synth.make_inputs([5, 9, 3, 7], 2, 4, 16, seed=3, dtype=torch.float32, s0_std=0.02)
    sub = ranks.shard_inputs(inp, [2, 0])
    assert sub.cu_seqlens == [0, 3, 8]
    assert torch.equal(sub.q[:3], inp.q[14:17]) and torch.equal(sub.q[3:], inp.q[0:5])
    assert torch.equal(sub.s0[0], inp.s0[2]) and torch.equal(sub.s0[1], inp.s0[0])


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, lens, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import oracle
    torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        env = ranks.rank_env()
        assert (env.rank, env.world) == (rank, world)
        # Max over ranks of a per-rank time.
        assert ranks.max_over_ranks(1.5 + rank, world) == 1.5 + world - 1
        # Each rank solves its own sequences; nothing is exchanged until the
        # results are gathered for the check.
        inp = synth.make_inputs(lens, 2, 4, 16, seed=11, dtype=torch.float32, s0_std=0.02)
        mine = ranks.partition_by_tokens(lens, world)[rank]
        sub = ranks.shard_inputs(inp, mine)
        f = lambda t: t.to(torch.float64).numpy()
        r = oracle.gdr_recurrent(f(sub.q), f(sub.k), f(sub.v), f(sub.g), f(sub.beta),
                                 np.array(sub.cu_seqlens), z=f(sub.z), s0=f(sub.s0), w=f(sub.w),
                                 threads=1)
        got = [None] * world
        torch.distributed.all_gather_object(got, {"seqs": mine, "y": r.y, "state": r.state,
                                                  "cu": sub.cu_seqlens})
        if rank == 0:
            full = oracle.gdr_recurrent(f(inp.q), f(inp.k), f(inp.v), f(inp.g), f(inp.beta),
                                        np.array(inp.cu_seqlens), z=f(inp.z), s0=f(inp.s0),
                                        w=f(inp.w), threads=1)
            covered = []
            for part in got:
                for j, s in enumerate(part["seqs"]):
                    a, b = inp.cu_seqlens[s], inp.cu_seqlens[s + 1]
                    pa, pb = part["cu"][j], part["cu"][j + 1]
                    assert np.array_equal(part["y"][pa:pb], full.y[a:b])
                    assert np.array_equal(part["state"][j], full.state[s])
                    covered.append(s)
            assert sorted(covered) == list(range(len(lens)))
            open(os.path.join(out_dir, "ok"), "w").write("ok")
        torch.distributed.barrier()
    finally:
        torch.distributed.destroy_process_group()


def test_two_rank_gloo_shards_match_one_process(tmp_path):
    lens = synth.lengths(7, seed=5, lo=1, hi=40)
    ctx = mp.get_context("spawn")
    world, port = 2, _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, lens, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    assert (tmp_path / "ok").exists()
