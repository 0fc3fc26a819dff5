"""Buffer management around the libmsa C ABI: allocates device tensors with
torch and chains the entry points encode -> route -> top-k -> gather ->
attend.  No arithmetic of the method happens here; every step is one call
into libmsa.
"""

from __future__ import annotations

import torch

from . import msa as _m


def dt_code(t: torch.Tensor) -> int:
    return _m.dtype_code(t.dtype)


def chunk_offsets(tok_offsets: torch.Tensor, chunk: int = 64, stream=None) -> torch.Tensor:
    """Device chunk offsets [n_docs+1] (int64) from device token offsets."""
    n_docs = tok_offsets.numel() - 1
    out = torch.empty(n_docs + 1, dtype=torch.int64, device=tok_offsets.device)
    _m.msa_chunk_offsets(n_docs, tok_offsets, chunk, out, stream)
    return out


def encode_pool(k_tok, v_tok, kr_tok, tok_offsets, chunk_offs, n_chunks: int,
                rope_base: float = 10000.0, chunk: int = 64, out=None, stream=None):
    """Token-level [L][N][H][D] -> pooled banks [L][C][H][D] (same dtype)."""
    L, N, H, D = k_tok.shape
    n_docs = tok_offsets.numel() - 1
    if out is None:
        out = tuple(torch.empty((L, n_chunks, H, D), dtype=k_tok.dtype, device=k_tok.device)
                    for _ in range(3))
    kb, vb, rb = out
    _m.msa_encode_pool(dt_code(k_tok), L, N, n_docs, H, D, k_tok, v_tok, kr_tok, tok_offsets,
                       chunk_offs, n_chunks, rope_base, chunk, kb, vb, rb, stream)
    return kb, vb, rb


def encode_pool_prepared(k_tok, v_tok, kr_tok, tok_offsets, chunk_offs, n_chunks: int,
                         rope_base: float = 10000.0, chunk: int = 64, keep_raw: bool = False,
                         stream=None):
    """bf16 token-level [L][N][H][D] -> pooled K̄, V̄ and the prepared routing
    bank K̂_r (unit rows, what ``prepare_bank`` makes from K̄_r) in one pass;
    with ``keep_raw`` the raw K̄_r too.  Returns (k_bar, v_bar, kr_hat,
    kr_bar or None)."""
    L, N, H, D = k_tok.shape
    n_docs = tok_offsets.numel() - 1
    mk = lambda: torch.empty((L, n_chunks, H, D), dtype=k_tok.dtype,  # noqa: E731
                             device=k_tok.device)
    kb, vb, rh = mk(), mk(), mk()
    rb = mk() if keep_raw else None
    _m.msa_encode_pool_prepared(dt_code(k_tok), L, N, n_docs, H, D, k_tok, v_tok, kr_tok,
                                tok_offsets, chunk_offs, n_chunks, rope_base, chunk, kb, vb, rb,
                                rh, stream)
    return kb, vb, rh, rb


def prepare_bank(kr_bar, out=None, stream=None):
    """Unit-normalised copy of a bf16 routing bank [C][H][D] (built once per
    bank; see msa_route_prepare_bank)."""
    C, H, D = kr_bar.shape
    if out is None:
        out = torch.empty_like(kr_bar)
    _m.msa_route_prepare_bank(dt_code(kr_bar), C, H, D, kr_bar, out, stream)
    return out


class Router:
    """Holds the workspace of msa_route_scores for fixed (dtype, B, T, H, D).
    ``prepared=True`` routes over a bank made by ``prepare_bank``."""

    def __init__(self, dtype: torch.dtype, B: int, T: int, H: int, D: int, device,
                 prepared: bool = False):
        self.dt = _m.dtype_code(dtype)
        self.B, self.T, self.H, self.D = B, T, H, D
        self.fn = _m.msa_route_scores_prepared if prepared else _m.msa_route_scores
        n = _m.msa_route_workspace_size(self.dt, B, T, H, D)
        self.ws = torch.empty(max(n, 16), dtype=torch.uint8, device=device)

    def __call__(self, q_r, kr_bar, chunk_offs, n_docs, doc_scores=None, chunk_scores=None,
                 stream=None):
        C = kr_bar.shape[0]
        if doc_scores is None:
            doc_scores = torch.empty((self.B, n_docs), dtype=torch.float32, device=q_r.device)
        self.fn(self.dt, self.B, self.T, self.H, self.D, q_r, kr_bar, C, chunk_offs, n_docs,
                doc_scores, chunk_scores, self.ws, self.ws.numel(), stream)
        return doc_scores


def topk_workspace(B: int, n: int, k: int, device):
    n_ws = _m.msa_topk_workspace_size(B, n, k)
    return torch.empty(max(n_ws, 16), dtype=torch.uint8, device=device)


def topk_docs(scores: torch.Tensor, k: int, idx=None, top=None, ws=None, stream=None):
    B, n = scores.shape
    if idx is None:
        idx = torch.empty((B, k), dtype=torch.int32, device=scores.device)
    if ws is None:
        ws = topk_workspace(B, n, k, scores.device)
    _m.msa_topk_docs(B, n, k, scores, idx, top, ws, ws.numel(), stream)
    return idx, top


def gather_kv(idx, chunk_offs, k_bar, v_bar, m_cap: int, k_mem=None, v_mem=None, mem_len=None,
              stream=None):
    B, k = idx.shape
    C, H, D = k_bar.shape
    n_docs = chunk_offs.numel() - 1
    dev = idx.device  # the bank may sit in (pinned, mapped) host memory
    if k_mem is None:
        k_mem = torch.empty((B, m_cap, H, D), dtype=k_bar.dtype, device=dev)
        v_mem = torch.empty((B, m_cap, H, D), dtype=k_bar.dtype, device=dev)
    if mem_len is None:
        mem_len = torch.empty(B, dtype=torch.int32, device=dev)
    _m.msa_gather_kv(dt_code(k_bar), B, k, H, D, idx, chunk_offs, n_docs, k_bar, v_bar, m_cap,
                     k_mem, v_mem, mem_len, stream)
    return k_mem, v_mem, mem_len


def route_backward_workspace(q_r, kr_bar, n_docs: int):
    """The workspace msa_route_backward needs for these shapes (None if none)."""
    B, T, H, D = q_r.shape
    n = _m.msa_route_backward_workspace_size(dt_code(q_r), B, T, H, D, kr_bar.shape[0], n_docs)
    return torch.empty(n, dtype=torch.uint8, device=q_r.device) if n else None


def route_backward(q_r, kr_bar, chunk_offs, d_doc, dq_r=None, dkr_bar=None, ws=None,
                   stream=None):
    """Gradients of the routing inputs from dL/d(doc_scores): ADDS into dq_r
    [B][T][H][D] and dkr_bar [C][H][D] (fp32; zero buffers made if None).
    ``ws``: from route_backward_workspace (made here if None)."""
    B, T, H, D = q_r.shape
    C = kr_bar.shape[0]
    if ws is None:
        ws = route_backward_workspace(q_r, kr_bar, chunk_offs.numel() - 1)
    if dq_r is None:
        dq_r = torch.zeros((B, T, H, D), dtype=torch.float32, device=q_r.device)
    if dkr_bar is None:
        dkr_bar = torch.zeros((C, H, D), dtype=torch.float32, device=q_r.device)
    _m.msa_route_backward(dt_code(q_r), B, T, H, D, q_r, kr_bar, C, chunk_offs,
                          chunk_offs.numel() - 1, d_doc, dq_r, dkr_bar, ws,
                          0 if ws is None else ws.numel(), stream)
    return dq_r, dkr_bar


def encode_pool_backward(dk_bar, dv_bar, dkr_bar, tok_offs, chunk_offs, n_tok: int,
                         rope_base: float = 10000.0, out=None, stream=None):
    """Gradients of the token tensors [L][N][H][D] (fp32) from the pooled
    bank's gradients [L][C][H][D] (fp32); ``out`` = (dk, dv, dkr) to reuse."""
    L, C, H, D = dk_bar.shape
    outs = out if out is not None else tuple(
        torch.empty((L, n_tok, H, D), dtype=torch.float32, device=dk_bar.device)
        for _ in range(3))
    _m.msa_encode_pool_backward(L, n_tok, tok_offs.numel() - 1, H, D, dk_bar, dv_bar, dkr_bar,
                                tok_offs, chunk_offs, C, rope_base, *outs, stream)
    return outs


def to_host_tier(t):
    """A copy of a bank tensor in pinned host memory.  Pinned allocations are
    mapped into every device's address space, so msa_gather_kv reads the
    selected rows straight from it over the host link (tiered storage: the
    routing keys stay in HBM, the content K/V in host DRAM)."""
    import torch
    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    h.copy_(t)
    return h


class Attention:
    """Holds the workspace of msa_sparse_attn for fixed shapes."""

    def __init__(self, dtype, B, T, T_loc, Hq, H, D, m_cap, device):
        self.dt = _m.dtype_code(dtype)
        self.shape = (B, T, T_loc, Hq, H, D, m_cap)
        n = _m.msa_sparse_attn_workspace_size(self.dt, B, T, T_loc, Hq, H, D, m_cap)
        self.ws = torch.empty(max(n, 16), dtype=torch.uint8, device=device)

    def __call__(self, q, k_mem, v_mem, mem_len, k_loc, v_loc, pos0: int,
                 rope_base: float = 10000.0, scale: float = 0.0, out=None, stream=None):
        B, T, T_loc, Hq, H, D, m_cap = self.shape
        if out is None:
            out = torch.empty((B, T, Hq, D), dtype=q.dtype, device=q.device)
        _m.msa_sparse_attn(self.dt, B, T, T_loc, Hq, H, D, q, k_mem, v_mem, mem_len, m_cap,
                           k_loc, v_loc, pos0, rope_base, scale, out, self.ws, self.ws.numel(),
                           stream)
        return out


class FusedAttention:
    """msa_sparse_attn_fused for fixed shapes: attention over the selected
    documents read straight from the bank (no gathered copy)."""

    def __init__(self, dtype, B, T, T_loc, Hq, H, D, k, m_cap, device):
        self.dt = _m.dtype_code(dtype)
        self.shape = (B, T, T_loc, Hq, H, D, k, m_cap)
        n = _m.msa_sparse_attn_fused_workspace_size(self.dt, B, T, T_loc, Hq, H, D, k, m_cap)
        if n == 0:
            raise _m.MsaError("msa_sparse_attn_fused", -2, "unsupported shape")
        self.ws = torch.empty(n, dtype=torch.uint8, device=device)
        self.mem_len = torch.empty(B, dtype=torch.int32, device=device)

    def __call__(self, q, idx, chunk_offs, k_bar, v_bar, k_loc, v_loc, pos0: int,
                 rope_base: float = 10000.0, scale: float = 0.0, out=None, stream=None):
        B, T, T_loc, Hq, H, D, k, m_cap = self.shape
        if out is None:
            out = torch.empty((B, T, Hq, D), dtype=q.dtype, device=q.device)
        _m.msa_sparse_attn_fused(self.dt, B, T, T_loc, Hq, H, D, q, idx, k, chunk_offs,
                                 chunk_offs.numel() - 1, k_bar, v_bar, k_bar.shape[0], m_cap,
                                 k_loc, v_loc, pos0, rope_base, scale, out, self.mem_len,
                                 self.ws, self.ws.numel(), stream)
        return out


class Pipeline:
    """route -> top-k -> gather -> attend over a resident pooled bank (one
    layer), with every buffer allocated once.  With ``prepared=True``,
    ``kr_bar`` is a bank made by ``prepare_bank``."""

    def __init__(self, kr_bar, k_bar, v_bar, chunk_offs, *, B, T, T_loc, Hq, k, m_cap,
                 pos0=None, rope_base=10000.0, prepared=False, fused=False):
        C, H, D = kr_bar.shape
        dev = kr_bar.device
        self.kr_bar, self.k_bar, self.v_bar, self.coff = kr_bar, k_bar, v_bar, chunk_offs
        self.n_docs = chunk_offs.numel() - 1
        self.B, self.T, self.T_loc, self.Hq, self.H, self.D = B, T, T_loc, Hq, H, D
        self.k, self.m_cap = k, m_cap
        self.pos0 = k if pos0 is None else pos0
        self.rope_base = rope_base
        self.router = Router(kr_bar.dtype, B, T, H, D, dev, prepared=prepared)
        self.fused = fused
        self.attn = (FusedAttention(kr_bar.dtype, B, T, T_loc, Hq, H, D, k, m_cap, dev) if fused
                     else Attention(kr_bar.dtype, B, T, T_loc, Hq, H, D, m_cap, dev))
        self.doc_scores = torch.empty((B, self.n_docs), dtype=torch.float32, device=dev)
        self.idx = torch.empty((B, k), dtype=torch.int32, device=dev)
        self.top = torch.empty((B, k), dtype=torch.float32, device=dev)
        self.topk_ws = topk_workspace(B, self.n_docs, k, dev)
        self.k_mem = torch.empty((B, max(m_cap, 1), H, D), dtype=kr_bar.dtype, device=dev)
        self.v_mem = torch.empty_like(self.k_mem)
        self.mem_len = torch.empty(B, dtype=torch.int32, device=dev)
        self.out = torch.empty((B, T, Hq, D), dtype=kr_bar.dtype, device=dev)

    def capture(self, q_r, q, k_loc, v_loc):
        """Records one step over these (fixed) input buffers into a CUDA
        graph and returns it; ``graph.replay()`` reruns the ten launches
        without per-launch host overhead.  Call once eagerly first so every
        one-time set-up (kernel attributes, driver entry points) is done."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self(q_r, q, k_loc, v_loc)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self(q_r, q, k_loc, v_loc)
        return graph

    def capture_from_host(self, q_r_h, q_h, k_loc_h, v_loc_h, out_h, idx_h):
        """Records one step that starts from pinned host inputs and ends with
        the output and the selected documents back in pinned host memory, as
        one CUDA graph: Q_r is uploaded first and routing starts at once,
        while Q and the local K/V are uploaded on a second stream; attention
        waits for both.  ``graph.replay()`` runs the whole step, copies
        included.  Returns the graph (the device-side copies of the inputs
        live in this object)."""
        dev = {name: torch.empty(t.shape, dtype=t.dtype, device=self.kr_bar.device)
               for name, t in (("q_r", q_r_h), ("q", q_h), ("k_loc", k_loc_h),
                               ("v_loc", v_loc_h))}
        self._host_step_inputs = dev
        side = torch.cuda.Stream()

        def step():
            main = torch.cuda.current_stream()
            # Q_r first: the uploads share one copy engine, so the others
            # are made to follow it and run under the routing
            dev["q_r"].copy_(q_r_h, non_blocking=True)
            side.wait_stream(main)
            with torch.cuda.stream(side):  # attention inputs, under the routing
                dev["q"].copy_(q_h, non_blocking=True)
                dev["k_loc"].copy_(k_loc_h, non_blocking=True)
                dev["v_loc"].copy_(v_loc_h, non_blocking=True)
            self.router(dev["q_r"], self.kr_bar, self.coff, self.n_docs, self.doc_scores, None)
            topk_docs(self.doc_scores, self.k, self.idx, self.top, self.topk_ws)
            if not self.fused:
                gather_kv(self.idx, self.coff, self.k_bar, self.v_bar, self.m_cap, self.k_mem,
                          self.v_mem, self.mem_len)
            main.wait_stream(side)
            if self.fused:
                self.attn(dev["q"], self.idx, self.coff, self.k_bar, self.v_bar, dev["k_loc"],
                          dev["v_loc"], self.pos0, self.rope_base, 0.0, self.out)
            else:
                self.attn(dev["q"], self.k_mem, self.v_mem, self.mem_len, dev["k_loc"],
                          dev["v_loc"], self.pos0, self.rope_base, 0.0, self.out)
            out_h.copy_(self.out, non_blocking=True)
            idx_h.copy_(self.idx, non_blocking=True)

        warm = torch.cuda.Stream()
        warm.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(warm):
            step()
        torch.cuda.current_stream().wait_stream(warm)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        return graph

    def __call__(self, q_r, q, k_loc, v_loc, stream=None):
        self.router(q_r, self.kr_bar, self.coff, self.n_docs, self.doc_scores, None, stream)
        topk_docs(self.doc_scores, self.k, self.idx, self.top, self.topk_ws, stream)
        if self.fused:  # attention reads the selected rows from the bank itself
            self.attn(q, self.idx, self.coff, self.k_bar, self.v_bar, k_loc, v_loc, self.pos0,
                      self.rope_base, 0.0, self.out, stream)
            self.mem_len = self.attn.mem_len
            return self.out
        gather_kv(self.idx, self.coff, self.k_bar, self.v_bar, self.m_cap, self.k_mem,
                  self.v_mem, self.mem_len, stream)
        self.attn(q, self.k_mem, self.v_mem, self.mem_len, k_loc, v_loc, self.pos0,
                  self.rope_base, 0.0, self.out, stream)
        return self.out


class HostStream:
    """Consecutive steps of a Pipeline from pinned host buffers, with the
    transfers off the compute stream: step i's inputs are uploaded on an
    upload stream and its output and selected documents read back on a
    download stream, so they overlap the compute of steps i-1 and i+1.  The
    device-side inputs and outputs are double-buffered; each of the two
    buffer sets has its step captured once as a CUDA graph (the Pipeline's
    launches only, no copies), replayed on the compute stream.

    ``step(q_r_h, q_h, k_loc_h, v_loc_h, out_h, idx_h)`` enqueues one step and
    returns at once: the inputs are read from the given pinned host tensors
    and the results written into ``out_h`` / ``idx_h`` (pinned) when the
    step's read-back completes -- ``wait(i)`` waits for step i's read-back,
    ``synchronize()`` for every step enqueued.  A caller may refill an input
    buffer once ``inputs_consumed(i)`` says that step i's uploads are done.
    Ordering between buffer sets: step i + 2 reuses step i's device buffers,
    so its upload waits for step i's compute and its compute for step i's
    read-back (events, no host wait)."""

    def __init__(self, p: Pipeline):
        self.p = p
        dev = p.kr_bar.device
        shapes = {"q_r": (p.B, p.T, p.H, p.D), "q": (p.B, p.T, p.Hq, p.D),
                  "k_loc": (p.B, p.T_loc, p.H, p.D), "v_loc": (p.B, p.T_loc, p.H, p.D)}
        dt = p.kr_bar.dtype
        self.inputs = [{n: torch.empty(sh, dtype=dt, device=dev) for n, sh in shapes.items()}
                       for _ in range(2)]
        self.outs = [torch.empty_like(p.out) for _ in range(2)]
        self.idxs = [torch.empty_like(p.idx) for _ in range(2)]
        self.compute = torch.cuda.current_stream()
        self.up = torch.cuda.Stream()
        self.down = torch.cuda.Stream()
        self.graphs = [self._capture(x) for x in range(2)]
        ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
        self.ev_up, self.ev_comp, self.ev_down = ev(), ev(), ev()
        self.fresh = [True, True]
        self.n = 0

    def _run(self, x):
        p, d = self.p, self.inputs[x]
        out = p.out
        p.out = self.outs[x]  # the step's attention writes this set's output
        try:
            p(d["q_r"], d["q"], d["k_loc"], d["v_loc"])
        finally:
            p.out = out
        self.idxs[x].copy_(p.idx)

    def _capture(self, x):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self._run(x)
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self._run(x)
        return g

    def start_after(self, event):
        """Makes the next step's uploads wait for `event` (e.g. the start of
        a timed region recorded on the compute stream)."""
        self.up.wait_event(event)

    def step(self, q_r_h, q_h, k_loc_h, v_loc_h, out_h, idx_h) -> int:
        x = self.n % 2
        d = self.inputs[x]
        with torch.cuda.stream(self.up):
            if not self.fresh[x]:  # step n-2 has read these device inputs
                self.up.wait_event(self.ev_comp[x])
            for name, h in (("q_r", q_r_h), ("q", q_h), ("k_loc", k_loc_h), ("v_loc", v_loc_h)):
                d[name].copy_(h, non_blocking=True)
            self.ev_up[x].record(self.up)
        self.compute.wait_event(self.ev_up[x])
        if not self.fresh[x]:  # step n-2's outputs have been read back
            self.compute.wait_event(self.ev_down[x])
        with torch.cuda.stream(self.compute):
            self.graphs[x].replay()
            self.ev_comp[x].record(self.compute)
        with torch.cuda.stream(self.down):
            self.down.wait_event(self.ev_comp[x])
            out_h.copy_(self.outs[x], non_blocking=True)
            idx_h.copy_(self.idxs[x], non_blocking=True)
            self.ev_down[x].record(self.down)
        self.fresh[x] = False
        self.n += 1
        return self.n - 1

    def inputs_consumed(self, i: int) -> bool:
        return self.ev_up[i % 2].query() if i >= self.n - 2 else True

    def wait(self, i: int):
        if i >= self.n - 2:
            self.ev_down[i % 2].synchronize()

    def synchronize(self):
        self.down.synchronize()
        self.compute.synchronize()
