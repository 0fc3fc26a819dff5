"""Memory Parallel: the routing bank split across GPUs by document range.

Method: "EverMind-AI/MSA: routing top-k compressed documents inside
attention ..." (hysenlabs.com), §"The 100M-token setup depends on host memory
as well as two GPUs": the routing keys are divided among the GPUs, each GPU
scores the query against its own part, and the partial results are reduced
into one global selection, while the content K/V live in host memory.

Here rank r holds the prepared routing keys of a contiguous document range
(``shard_plan``) in its own HBM.  Every rank routes the same queries against
its range and keeps its local top-k; the ranks all-gather their k
(score, local id) candidates (``exchange_candidates``: one all-gather of
B*k floats and B*k ints, NCCL over NVLink for device tensors) and each merges
them with ``msa_topk_merge_shards`` into the same global top-k.  The content
K̄/V̄ sit once in pinned host memory that every GPU maps (tiered storage), so
each rank gathers the selected rows of the queries it serves itself; there is
no peer-to-peer traffic in the data path besides the all-gather.  Rank r
serves the contiguous query block ``query_block(B, rank, world)``.
"""

from __future__ import annotations

import numpy as np

from . import msa as _m
from .pipeline import Attention, Router, gather_kv, topk_workspace, topk_docs


def shard_plan(chunk_offsets, world: int, k: int) -> list[tuple[int, int, int, int]]:
    """Per rank, ``(doc_lo, doc_hi, chunk_lo, chunk_hi)``: contiguous,
    increasing document ranges covering every document, cut where the chunk
    count reaches r*C/world (so shards differ by at most about one document's
    chunks), each holding at least k documents (a local top-k needs k)."""
    off = np.asarray(chunk_offsets, dtype=np.int64)
    n_docs = len(off) - 1
    if world < 1 or k < 1:
        raise ValueError("world and k must be positive")
    if n_docs < world * k:
        raise ValueError(f"{n_docs} documents cannot give {world} shards of at least k={k}")
    C = int(off[-1])
    cuts = [0]
    for r in range(1, world):
        d = int(np.searchsorted(off, r * C / world, side="left"))
        d = max(d, cuts[-1] + k)              # at least k documents behind
        d = min(d, n_docs - (world - r) * k)  # and k for every later shard
        cuts.append(d)
    cuts.append(n_docs)
    return [(cuts[r], cuts[r + 1], int(off[cuts[r]]), int(off[cuts[r + 1]]))
            for r in range(world)]


def query_block(B: int, rank: int, world: int) -> tuple[int, int]:
    """The contiguous block of queries rank serves in the attention stage."""
    return B * rank // world, B * (rank + 1) // world


def local_offsets(chunk_offsets, plan, rank: int):
    """Shard-local chunk offsets (int64, starting at 0) as a NumPy array."""
    off = np.asarray(chunk_offsets, dtype=np.int64)
    d0, d1, c0, _ = plan[rank]
    return off[d0:d1 + 1] - c0


def _torch_stream(stream):
    """A torch stream object for a stream argument of the binding (None,
    a torch.cuda.Stream or a raw cudaStream_t handle)."""
    import torch
    if stream is None or isinstance(stream, torch.cuda.Stream):
        return stream
    return torch.cuda.ExternalStream(int(stream))


def exchange_candidates(scores, ids, group=None, stream=None):
    """All-gathers every rank's ``[B][k]`` local candidates (scores float32,
    local ids int32) into ``[world][B][k]`` tensors on the same device: one
    collective per tensor, every rank in the same order.

    Device tensors: with NCCL the all-gathers are ordered after the work
    queued on ``stream`` (torch's current stream if None) and the results are
    ready for work queued on it afterwards.  With gloo (a CPU group) device
    candidates are staged through pinned host memory -- the copy to the host
    waits for ``stream`` -- and copied back on it."""
    import contextlib

    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    ts = _torch_stream(stream) if scores.is_cuda else None
    ctx = torch.cuda.stream(ts) if ts is not None else contextlib.nullcontext()
    with ctx:
        out_s = torch.empty((world,) + tuple(scores.shape), dtype=scores.dtype,
                            device=scores.device)
        out_i = torch.empty((world,) + tuple(ids.shape), dtype=ids.dtype, device=ids.device)
        staged = scores.is_cuda and dist.get_backend(group) == "gloo"
        if staged:
            hs = torch.empty(scores.shape, dtype=scores.dtype, pin_memory=True)
            hi = torch.empty(ids.shape, dtype=ids.dtype, pin_memory=True)
            hs.copy_(scores)  # synchronous: waits for the stream's top-k
            hi.copy_(ids)
            gs = torch.empty(out_s.shape, dtype=scores.dtype)
            gi = torch.empty(out_i.shape, dtype=ids.dtype)
            dist.all_gather(list(gs.unbind(0)), hs, group=group)
            dist.all_gather(list(gi.unbind(0)), hi, group=group)
            out_s.copy_(gs)
            out_i.copy_(gi)
        else:
            dist.all_gather(list(out_s.unbind(0)), scores.contiguous(), group=group)
            dist.all_gather(list(out_i.unbind(0)), ids.contiguous(), group=group)
    return out_s, out_i


def merge_shards(cand_scores, cand_ids, doc_base, k: int, idx=None, top=None, stream=None):
    """Global top-k from the gathered ``[world][B][k]`` candidates
    (msa_topk_merge_shards); ``doc_base`` [world] int32 holds each shard's
    first global document id."""
    import torch
    world, B, kk = cand_scores.shape
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=cand_scores.device)
    _m.msa_topk_merge_shards(B, world, k, cand_scores, cand_ids, doc_base, idx, top, stream)
    return idx, top


class MemoryParallelRouter:
    """This rank's part of Memory Parallel routing: route the queries over the
    rank's prepared K̄_r shard, take the local top-k, exchange, merge."""

    def __init__(self, kr_hat_shard, local_coff, plan, rank: int, *, B: int, T: int, k: int,
                 group=None):
        import torch
        import torch.distributed as dist
        C, H, D = kr_hat_shard.shape
        dev = kr_hat_shard.device
        self.world = dist.get_world_size(group)
        if len(plan) != self.world:
            raise ValueError("the plan must have one shard per rank")
        self.kr, self.coff, self.group = kr_hat_shard, local_coff, group
        self.n_local = plan[rank][1] - plan[rank][0]
        self.B, self.T, self.k = B, T, k
        self.router = Router(kr_hat_shard.dtype, B, T, H, D, dev, prepared=True)
        self.doc_scores = torch.empty((B, self.n_local), dtype=torch.float32, device=dev)
        self.loc_idx = torch.empty((B, k), dtype=torch.int32, device=dev)
        self.loc_top = torch.empty((B, k), dtype=torch.float32, device=dev)
        self.topk_ws = topk_workspace(B, self.n_local, k, dev)
        self.doc_base = torch.tensor([p[0] for p in plan], dtype=torch.int32, device=dev)
        self.idx = torch.empty((B, k), dtype=torch.int32, device=dev)
        self.top = torch.empty((B, k), dtype=torch.float32, device=dev)

    def __call__(self, q_r, stream=None):
        self.router(q_r, self.kr, self.coff, self.n_local, self.doc_scores, None, stream)
        topk_docs(self.doc_scores, self.k, self.loc_idx, self.loc_top, self.topk_ws, stream)
        cs, ci = exchange_candidates(self.loc_top, self.loc_idx, self.group, stream)
        merge_shards(cs, ci, self.doc_base, self.k, self.idx, self.top, stream)
        return self.idx, self.top


class MemoryParallelPipeline:
    """Route with Memory Parallel, then gather (from the shared host-tier or a
    replicated K̄/V̄ bank, global chunk offsets) and attend for this rank's
    query block."""

    def __init__(self, kr_hat_shard, local_coff, global_coff, k_bar, v_bar, plan, rank: int, *,
                 B: int, T: int, T_loc: int, Hq: int, k: int, m_cap: int, pos0=None,
                 rope_base: float = 10000.0, group=None):
        import torch
        C, H, D = kr_hat_shard.shape
        dev = kr_hat_shard.device
        self.route = MemoryParallelRouter(kr_hat_shard, local_coff, plan, rank, B=B, T=T, k=k,
                                          group=group)
        self.b0, self.b1 = query_block(B, rank, self.route.world)
        nb = self.b1 - self.b0
        self.coff, self.k_bar, self.v_bar, self.m_cap = global_coff, k_bar, v_bar, m_cap
        self.pos0 = k if pos0 is None else pos0
        self.rope_base = rope_base
        self.attn = Attention(kr_hat_shard.dtype, max(nb, 1), T, T_loc, Hq, H, D, m_cap, dev)
        self.k_mem = torch.empty((max(nb, 1), max(m_cap, 1), H, D), dtype=kr_hat_shard.dtype,
                                 device=dev)
        self.v_mem = torch.empty_like(self.k_mem)
        self.mem_len = torch.empty(max(nb, 1), dtype=torch.int32, device=dev)
        self.out = torch.empty((max(nb, 1), T, Hq, D), dtype=kr_hat_shard.dtype, device=dev)

    def __call__(self, q_r, q_blk, k_loc_blk, v_loc_blk, stream=None):
        """q_r: every query (the broadcast routing queries); q_blk, k_loc_blk,
        v_loc_blk: this rank's query block.  Returns the block's output."""
        idx, _ = self.route(q_r, stream)
        if self.b1 == self.b0:
            return self.out[:0]
        gather_kv(idx[self.b0:self.b1], self.coff, self.k_bar, self.v_bar, self.m_cap,
                  self.k_mem, self.v_mem, self.mem_len, stream)
        self.attn(q_blk, self.k_mem, self.v_mem, self.mem_len, k_loc_blk, v_loc_blk, self.pos0,
                  self.rope_base, 0.0, self.out, stream)
        return self.out
