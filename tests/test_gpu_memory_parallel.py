"""Memory Parallel through the library, in two processes that share the one
GPU: each rank holds only its document range of the prepared routing bank,
routes every query over it with libmsa, takes its local top-k, exchanges
candidates with the other rank over a gloo group (staged through pinned host
memory), merges them with msa_topk_merge_shards and attends for its own block
of queries.  Both ranks' merged top-k and attention outputs are compared with
the oracle's unsharded routing and attention.

The ranks' kernels never wait on each other: the only exchange is the gloo
all-gather on the host, after each rank's own top-k has finished.
"""

import os
import socket
import subprocess

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle

pytestmark = pytest.mark.gpu

ROUTE_ATOL = 2e-3
GAP = 4e-3
ATTN_BF16 = 2e-2
H, D, HQ, T, K = 8, 128, 32, 24, 8
B, N_DOCS = 3, 600


def _bank():
    """The seeded bank every rank (and the parent) draws: pooled bf16 routing
    keys and content rows, 3 routing queries, their attention inputs."""
    from latent_memory_routing_b200 import synth
    gc = torch.Generator().manual_seed(71)
    lengths = torch.randint(1, 900, (N_DOCS,), generator=gc)
    coff_h = oracle.chunk_offsets_from_lengths(lengths.numpy())
    C = int(coff_h[-1])
    g = torch.Generator(device="cuda").manual_seed(72)
    w = {name: synth.randn(shape, torch.bfloat16, "cuda", g) for name, shape in (
        ("kr", (C, H, D)), ("kb", (C, H, D)), ("vb", (C, H, D)), ("q_r", (B, T, H, D)),
        ("q", (B, T, HQ, D)), ("k_loc", (B, T, H, D)), ("v_loc", (B, T, H, D)))}
    return w, coff_h


def _rank_main(rank, world, port, out_q):
    try:
        import torch.distributed as dist

        from latent_memory_routing_b200 import memory_parallel as mpar
        from latent_memory_routing_b200 import msa, pipeline
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        torch.cuda.set_device(0)
        msa.lib()
        w, coff_h = _bank()
        plan = mpar.shard_plan(coff_h, world, K)
        d0, d1, c0, c1 = plan[rank]
        # this rank keeps only its own range of the prepared routing keys
        shard = pipeline.prepare_bank(w["kr"][c0:c1].contiguous())
        del w["kr"]
        local = torch.from_numpy(mpar.local_offsets(coff_h, plan, rank)).cuda()
        m_cap = K * int(np.diff(coff_h).max())
        mp_pipe = mpar.MemoryParallelPipeline(
            shard, local, torch.from_numpy(coff_h).cuda(), w["kb"], w["vb"], plan, rank, B=B,
            T=T, T_loc=T, Hq=HQ, k=K, m_cap=m_cap)
        b0, b1 = mpar.query_block(B, rank, world)
        side = torch.cuda.Stream()  # a non-current stream: the exchange must follow it
        side.wait_stream(torch.cuda.current_stream())
        out = mp_pipe(w["q_r"], w["q"][b0:b1].contiguous(), w["k_loc"][b0:b1].contiguous(),
                      w["v_loc"][b0:b1].contiguous(), stream=side)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        status = msa.msa_device_status(clear=True)
        out_q.put((rank, (b0, b1), mp_pipe.route.idx.cpu().numpy(),
                   mp_pipe.route.top.cpu().numpy(), out[:b1 - b0].float().cpu().numpy(),
                   mp_pipe.mem_len[:b1 - b0].cpu().numpy(), status, None))
        dist.barrier()
        dist.destroy_process_group()
    except BaseException as e:
        out_q.put((rank, None, None, None, None, None, None, f"{type(e).__name__}: {e}"))
        raise


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shared_compute_mode() -> bool:
    try:
        r = subprocess.run(["nvidia-smi", "-i", "0", "--query-gpu=compute_mode",
                            "--format=csv,noheader"], capture_output=True, text=True, timeout=30)
    except (OSError, subprocess.SubprocessError):
        return True
    return "exclusive" not in r.stdout.lower()


def test_memory_parallel_two_processes_vs_oracle(cuda_device):
    if not _shared_compute_mode():
        pytest.skip("the GPU admits one process at a time")
    from latent_memory_routing_b200 import build
    build.build()
    world = 2
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out_q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        # read the results before joining: a child blocks in put() until its
        # (large) result has been read
        for _ in range(world):
            r = out_q.get(timeout=600)
            assert r[7] is None, f"rank {r[0]}: {r[7]}"
            res[r[0]] = r
    finally:
        for p in procs:
            p.join(timeout=120)
        alive = [p.pid for p in procs if p.is_alive()]
        for p in procs:
            if p.is_alive():
                p.kill()
    assert not alive, "a rank did not finish"
    assert sorted(res) == [0, 1] and all(p.exitcode == 0 for p in procs)

    w, coff_h = _bank()
    f64 = lambda t: t.double().cpu().numpy()  # noqa: E731
    ods, _ = oracle.route_scores(f64(w["q_r"]), f64(w["kr"]), coff_h)
    # every rank holds the same global selection
    assert np.array_equal(res[0][2], res[1][2])
    idx = res[0][2]
    for b in range(B):  # the gap rule on the oracle's unsharded scores
        s = ods[b]
        order = np.lexsort((np.arange(N_DOCS), -s))
        srt = s[order]
        if srt[K - 1] - srt[K] > GAP:
            assert set(idx[b].tolist()) == set(order[:K].tolist()), b
        assert np.max(np.abs(res[0][3][b] - s[idx[b]])) <= ROUTE_ATOL
    okm, ovm, oml = oracle.gather_kv(idx, coff_h, f64(w["kb"]), f64(w["vb"]))
    want = oracle.sparse_attn(f64(w["q"]), okm, ovm, f64(w["k_loc"]), f64(w["v_loc"]), K, 10000.0)
    for r in range(world):
        b0, b1 = res[r][1]
        assert res[r][5].tolist() == list(oml[b0:b1])
        got = res[r][4]
        assert np.all(np.isfinite(got))
        assert np.max(np.abs(got - want[b0:b1])) <= ATTN_BF16
        assert res[r][6] == 0
