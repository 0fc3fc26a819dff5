"""Memory Parallel host logic on the CPU: the shard plan, and the candidate
exchange between 2, 3 and 4 gloo ranks, checked against the oracle's unsharded
routing + top-k.  (The merge kernel itself is checked on the GPU in
test_gpu_parity.py, with the shards emulated in one process.)"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from latent_memory_routing_b200 import memory_parallel as mpar


def _offsets(lengths):
    return oracle.chunk_offsets_from_lengths(np.asarray(lengths))


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_plan_invariants(world):
    rng = np.random.default_rng(world)
    lengths = rng.integers(64, 3000, size=500)
    off = _offsets(lengths)
    k = 16
    plan = mpar.shard_plan(off, world, k)
    assert len(plan) == world
    assert plan[0][0] == 0 and plan[-1][1] == len(lengths)
    C = int(off[-1])
    biggest = int(np.diff(off).max())
    for r, (d0, d1, c0, c1) in enumerate(plan):
        assert d1 - d0 >= k
        assert c0 == off[d0] and c1 == off[d1]
        if r:
            assert d0 == plan[r - 1][1]  # contiguous, increasing
        # cut at the first document reaching r*C/world: within one document
        assert abs(c0 - r * C / world) <= biggest
    local = mpar.local_offsets(off, plan, world - 1)
    assert local[0] == 0 and local[-1] == plan[-1][3] - plan[-1][2]


def test_shard_plan_keeps_k_documents_per_shard():
    # one huge document first: the cut may not leave the first shard short
    off = _offsets([100000] + [64] * 40)
    plan = mpar.shard_plan(off, 2, 8)
    assert plan[0][1] - plan[0][0] >= 8 and plan[1][1] - plan[1][0] >= 8
    with pytest.raises(ValueError):
        mpar.shard_plan(_offsets([64] * 10), 2, 8)


def test_query_block_covers_batch():
    for world in (1, 2, 3, 5):
        for B in (1, 4, 7, 64):
            blocks = [mpar.query_block(B, r, world) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == B
            assert all(blocks[r][1] == blocks[r + 1][0] for r in range(world - 1))


def _bank(seed):
    rng = np.random.default_rng(seed)
    lengths = rng.integers(64, 700, size=60)
    lengths[7] = lengths[50] = 128
    off = _offsets(lengths)
    C, H, D = int(off[-1]), 2, 16
    kr = rng.standard_normal((C, H, D))
    q_r = rng.standard_normal((2, 5, H, D))
    # documents 7 (first shard) and 50 (second shard) are identical and the
    # best for query 0: a tie across shards that must go to the lower id, 7
    kr[off[7]:off[8]] = q_r[0].mean(0) + 0.05 * rng.standard_normal((128 // 64, H, D))
    kr[off[50]:off[51]] = kr[off[7]:off[8]]
    return kr, q_r, off


def _rank_main(rank, world, port, seed, k, fail_q):
    try:
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        kr, q_r, off = _bank(seed)
        plan = mpar.shard_plan(off, world, k)
        d0, d1, c0, c1 = plan[rank]
        # this rank's local routing and top-k (the oracle stands in for the
        # GPU kernels here)
        loc, _ = oracle.route_scores(q_r, kr[c0:c1], mpar.local_offsets(off, plan, rank))
        li, ls = oracle.topk_docs(loc, k)
        cs, ci = mpar.exchange_candidates(torch.from_numpy(ls.astype(np.float32)),
                                          torch.from_numpy(li.astype(np.int32)))
        assert cs.shape == (world, 2, k) and ci.shape == (world, 2, k)
        # merge rule of msa_topk_merge_shards, restated: rank order over the
        # union of candidates by (score desc, global id asc)
        base = np.array([p[0] for p in plan])
        gid = ci.numpy().astype(np.int64) + base[:, None, None]
        full, _ = oracle.route_scores(q_r, kr, off)
        want, _ = oracle.topk_docs(full, k)
        shard = [next(r for r, pr in enumerate(plan) if pr[0] <= d < pr[1]) for d in (7, 50)]
        assert shard[0] < shard[1]  # the tie crosses a shard boundary
        for b in range(2):
            s = cs.numpy()[:, b].reshape(-1).astype(np.float64)
            g = gid[:, b].reshape(-1)
            order = np.lexsort((g, -s))[:k]
            assert g[order].tolist() == want[b].tolist(), (rank, b)
        assert want[0][:2].tolist() == [7, 50]
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:  # report to the parent, then fail the rank
        fail_q.put(f"rank {rank}: {type(e).__name__}: {e}")
        raise


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3, 4])
def test_exchange_and_merge_gloo(world):
    ctx = mp.get_context("spawn")
    fail_q = ctx.SimpleQueue()
    mp.start_processes(_rank_main, args=(world, _free_port(), 3, 4, fail_q), nprocs=world,
                       join=True, start_method="spawn")
    assert fail_q.empty()


def _rank_dies_main(rank, world, port, fail_q, done_q):
    """Rank 1 raises after joining the group and before the exchange; rank 0
    must see its exchange end with an error (the peer's connection closes, or
    the group's short timeout expires) instead of waiting for good."""
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        raise RuntimeError("rank 1 fails before the exchange (injected on the host)")
    s = torch.zeros((2, 4), dtype=torch.float32)
    i = torch.zeros((2, 4), dtype=torch.int32)
    try:
        mpar.exchange_candidates(s, i)
    except Exception as e:  # detected: report and leave
        done_q.put(f"rank 0 detected: {type(e).__name__}")
        return
    fail_q.put("rank 0: the exchange completed without its peer")


def test_rank_failure_before_exchange_is_detected():
    ctx = mp.get_context("spawn")
    fail_q, done_q = ctx.SimpleQueue(), ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_dies_main, args=(r, 2, port, fail_q, done_q))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    alive = [p.pid for p in procs if p.is_alive()]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert not alive, "a rank did not finish"
    assert fail_q.empty(), fail_q.get()
    assert not done_q.empty(), "rank 0 did not report the failure"
    assert done_q.get().startswith("rank 0 detected")
    assert procs[0].exitcode == 0 and procs[1].exitcode != 0
