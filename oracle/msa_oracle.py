"""Float64 CPU oracle of the MSA hot path (vectorised NumPy).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by
the CPU-baseline leg of the benchmark, never by the product library.

Sources (web pages about EverMind-AI's Memory Sparse Attention), cited below
by title and section:

* [DEEP] "深度分析MSA:把超长文档组织成可检索内部记忆的工程路径"
  (yeyulingfeng.com) -- sections "三、文档如何变成 memory" (document
  encoding, "2. chunk 压缩", "3. memory bank 构建") and "五、推理阶段：memory
  的使用方式" (Step 2 routing, Step 3 local generation).
* [HYSEN] "EverMind-AI/MSA: routing top-k compressed documents inside
  attention, and where the 100M-token claim stops" (hysenlabs.com) --
  sections "Routing happens inside attention, not in a retrieval service in
  front of the model", "Document-wise RoPE resets every document to position
  zero", "Memory must be encoded offline before a query can reach it".

Readings taken where the pages are silent (each is repeated at its function):

* RoPE pairs element i with element i + D/2 ("rotate half"), inverse
  frequency base^(-2i/D), i in [0, D/2).
* Only token K is rotated document-wise; V and K_r are pooled unrotated.
* The cosine uses max(|x|, 1e-12) for each norm, so a zero vector scores 0.
* A document's score is the maximum over its chunks' scores.
* Top-k ties go to the lower document index; output is in rank order.
* Memory rows keep their document-wise rotation; only the query and its local
  keys take global positions starting at offset k.  Every memory row is
  visible to every query token; local keys are causal.
* Softmax scale 1/sqrt(D); query head h reads KV head floor(h * H / Hq).

Everything is computed in float64 from inputs upcast to float64.
Parity of these readings with the upstream implementation is unpinned (its
code is not available); each reading is pinned by closed forms in the tests.
"""

from __future__ import annotations

import numpy as np

CHUNK = 64  # [DEEP] "2. chunk 压缩": every 64 tokens form one chunk
EPS = 1e-12


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------
# Chunking -- [DEEP] "2. chunk 压缩" (64 tokens per chunk; 180 tokens -> 3)
# ----------------------------------------------------------------------------

def chunk_counts(lengths, chunk: int = CHUNK) -> np.ndarray:
    """Number of chunks of each document: ceil(len / chunk).

    A trailing partial chunk is kept, which is what makes a 180-token document
    give 3 chunks ([DEEP] "2. chunk 压缩").  Empty documents are rejected.
    """
    lengths = np.asarray(lengths, dtype=np.int64)
    if lengths.ndim != 1:
        raise ValueError("lengths must be 1-D")
    if np.any(lengths <= 0):
        raise ValueError("every document must hold at least one token")
    if chunk <= 0:
        raise ValueError("chunk must be positive")
    return (lengths + chunk - 1) // chunk


def chunk_offsets_from_lengths(lengths, chunk: int = CHUNK) -> np.ndarray:
    """Exclusive prefix sum of the chunk counts: doc d owns chunk rows
    [off[d], off[d+1])."""
    counts = chunk_counts(lengths, chunk)
    off = np.zeros(counts.shape[0] + 1, dtype=np.int64)
    np.cumsum(counts, out=off[1:])
    return off


def chunk_token_ranges(length: int, chunk: int = CHUNK):
    """Token ranges [a, b) of the chunks of one document of ``length`` tokens."""
    n = int(chunk_counts([length], chunk)[0])
    return [(j * chunk, min((j + 1) * chunk, int(length))) for j in range(n)]


# ----------------------------------------------------------------------------
# RoPE -- [HYSEN] "Document-wise RoPE resets every document to position zero"
# ----------------------------------------------------------------------------

def rope_inv_freq(D: int, base: float) -> np.ndarray:
    """Inverse frequencies base^(-2i/D), i = 0 .. D/2-1 (float64)."""
    if D % 2:
        raise ValueError("head dim must be even")
    i = np.arange(D // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / D)


def rope_rotate(x, pos, base: float) -> np.ndarray:
    """Rotate rows of ``x`` by RoPE at positions ``pos``.

    ``x`` has shape [n, ..., D] (axis 0 indexes rows, which take positions
    ``pos[n]``).  Pair (x_i, x_{i+D/2}) at angle theta = p * base^(-2i/D)
    maps to (x_i cos - x_{i+D/2} sin, x_{i+D/2} cos + x_i sin).
    """
    x = _f64(x)
    pos = _f64(pos).reshape(-1)
    if pos.shape[0] != x.shape[0]:
        raise ValueError("one position per row")
    D = x.shape[-1]
    half = D // 2
    theta = pos.reshape((-1,) + (1,) * (x.ndim - 1)) * rope_inv_freq(D, base)
    c, s = np.cos(theta), np.sin(theta)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ----------------------------------------------------------------------------
# Memory encoding -- [DEEP] "三、文档如何变成 memory"; [HYSEN] "Memory must be
# encoded offline before a query can reach it"
# ----------------------------------------------------------------------------

def encode_pool_doc(k_doc, v_doc, kr_doc, rope_base: float = 10000.0,
                    chunk: int = CHUNK):
    """Pool one document.

    ``k_doc``, ``v_doc``, ``kr_doc``: [len][H][D] token rows of one layer.
    K is rotated with document-wise positions 0..len-1, then K, V and K_r are
    mean-pooled over each chunk (a partial tail chunk is the mean of the
    tokens it holds).  Returns (k_bar, v_bar, kr_bar), each [n_chunks][H][D].
    """
    k_doc, v_doc, kr_doc = _f64(k_doc), _f64(v_doc), _f64(kr_doc)
    n = k_doc.shape[0]
    k_rot = rope_rotate(k_doc, np.arange(n), rope_base)
    ranges = chunk_token_ranges(n, chunk)
    kb = np.stack([k_rot[a:b].mean(axis=0) for a, b in ranges])
    vb = np.stack([v_doc[a:b].mean(axis=0) for a, b in ranges])
    rb = np.stack([kr_doc[a:b].mean(axis=0) for a, b in ranges])
    return kb, vb, rb


def encode_pool(k_tok, v_tok, kr_tok, tok_offsets, rope_base: float = 10000.0,
                chunk: int = CHUNK):
    """Encode every document of every layer into the chunk-level bank.

    ``*_tok``: [L][N][H][D]; ``tok_offsets``: [n_docs+1].  Returns
    (k_bar, v_bar, kr_bar, chunk_offsets) with banks [L][C][H][D].
    """
    k_tok, v_tok, kr_tok = _f64(k_tok), _f64(v_tok), _f64(kr_tok)
    tok_offsets = np.asarray(tok_offsets, dtype=np.int64)
    lengths = np.diff(tok_offsets)
    coff = chunk_offsets_from_lengths(lengths, chunk)
    L, _, H, D = k_tok.shape
    C = int(coff[-1])
    kb = np.empty((L, C, H, D))
    vb = np.empty((L, C, H, D))
    rb = np.empty((L, C, H, D))
    for l in range(L):
        for d in range(lengths.shape[0]):
            t0, t1 = int(tok_offsets[d]), int(tok_offsets[d + 1])
            c0, c1 = int(coff[d]), int(coff[d + 1])
            kb[l, c0:c1], vb[l, c0:c1], rb[l, c0:c1] = encode_pool_doc(
                k_tok[l, t0:t1], v_tok[l, t0:t1], kr_tok[l, t0:t1],
                rope_base, chunk)
    return kb, vb, rb, coff


# ----------------------------------------------------------------------------
# Routing -- [HYSEN] "Routing happens inside attention ...": cosine
# similarity, mean over heads, then maximum over query tokens; [DEEP]
# "五、推理阶段" Step 2: Q_r x K̄_r -> score -> top-k
# ----------------------------------------------------------------------------

def cosine(q, k, eps: float = EPS) -> np.ndarray:
    """cos(q, k) = q.k / (max(|q|, eps) max(|k|, eps)) over the last axis."""
    q, k = _f64(q), _f64(k)
    qn = np.maximum(np.linalg.norm(q, axis=-1), eps)
    kn = np.maximum(np.linalg.norm(k, axis=-1), eps)
    return np.sum(q * k, axis=-1) / (qn * kn)


def route_chunk_scores(q_r, kr_bar, eps: float = EPS,
                       block: int = 16384) -> np.ndarray:
    """Chunk scores s[b, c] = max_t (1/H) sum_h cos(Q_r[b,t,h], K̄_r[c,h]).

    ``q_r``: [B][T][H][D]; ``kr_bar``: [C][H][D] (one layer).  Returns [B][C].
    Chunk rows are independent, so they are processed in blocks of ``block``
    rows only to bound memory; each score is the formula above as written.
    """
    q = _f64(q_r)
    k = _f64(kr_bar)
    B, T, H, D = q.shape
    C = k.shape[0]
    qn = q / np.maximum(np.linalg.norm(q, axis=-1, keepdims=True), eps)
    out = np.empty((B, C))
    for c0 in range(0, C, block):
        kblk = k[c0:c0 + block]
        kn = kblk / np.maximum(np.linalg.norm(kblk, axis=-1, keepdims=True), eps)
        for b in range(B):
            head_sum = np.zeros((T, kblk.shape[0]))
            for h in range(H):
                head_sum += qn[b, :, h, :] @ kn[:, h, :].T  # cosines [T][c]
            head_mean = head_sum / H
            out[b, c0:c0 + kblk.shape[0]] = head_mean.max(axis=0)
    return out


def doc_max(chunk_scores, chunk_offsets) -> np.ndarray:
    """Document score = maximum of its chunks' scores (the pages leave the
    document-level aggregation open; this library takes the maximum)."""
    s = _f64(chunk_scores)
    coff = np.asarray(chunk_offsets, dtype=np.int64)
    if np.any(np.diff(coff) <= 0):
        raise ValueError("every document must own at least one chunk")
    return np.maximum.reduceat(s, coff[:-1], axis=1)


def route_scores(q_r, kr_bar, chunk_offsets, eps: float = EPS):
    """Returns (doc_scores [B][n_docs], chunk_scores [B][C])."""
    cs = route_chunk_scores(q_r, kr_bar, eps)
    return doc_max(cs, chunk_offsets), cs


def topk_docs(doc_scores, k: int):
    """Top-k documents per query, ordered by (score descending, index
    ascending), so ties go to the lower document index.

    Returns (idx [B][k] int64, scores [B][k] float64).
    """
    s = _f64(doc_scores)
    if s.ndim != 2:
        raise ValueError("doc_scores must be [B][n_docs]")
    B, n = s.shape
    if not 0 < k <= n:
        raise ValueError("need 0 < k <= n_docs")
    idx = np.empty((B, k), dtype=np.int64)
    for b in range(B):
        order = np.lexsort((np.arange(n), -s[b]))  # primary: -score
        idx[b] = order[:k]
    return idx, np.take_along_axis(s, idx, axis=1)


# ----------------------------------------------------------------------------
# Context assembly -- [HYSEN] "Memory must be encoded offline ...": only the
# selected K/V are loaded and joined with the local context
# ----------------------------------------------------------------------------

def gather_kv(idx, chunk_offsets, k_bar, v_bar):
    """Concatenate the chunk rows of the selected documents in rank order.

    ``idx``: [B][k]; banks [C][H][D].  Returns (k_mem, v_mem, mem_len) where
    k_mem[b], v_mem[b] are [M_b][H][D] float64 arrays and mem_len[b] = M_b.
    """
    coff = np.asarray(chunk_offsets, dtype=np.int64)
    kb, vb = _f64(k_bar), _f64(v_bar)
    k_mem, v_mem, mem_len = [], [], []
    for row in np.asarray(idx, dtype=np.int64):
        rows = np.concatenate([np.arange(coff[d], coff[d + 1]) for d in row])
        k_mem.append(kb[rows])
        v_mem.append(vb[rows])
        mem_len.append(rows.shape[0])
    return k_mem, v_mem, np.asarray(mem_len, dtype=np.int64)


# ----------------------------------------------------------------------------
# Sparse attention -- [HYSEN] "Routing happens inside attention ..." (selected
# compressed K/V concatenated with the query's local K/V) and "Document-wise
# RoPE ..." (global RoPE, query start offset by k)
# ----------------------------------------------------------------------------

def sparse_attn(q, k_mem, v_mem, k_loc, v_loc, pos0: int,
                rope_base: float = 10000.0, scale: float | None = None):
    """GQA attention over [memory rows ; local causal rows].

    ``q``: [B][T][Hq][D]; ``k_mem[b]``/``v_mem[b]``: [M_b][H][D] (already
    carrying their document-wise rotation, not rotated again);
    ``k_loc``/``v_loc``: [B][T_loc][H][D] with T <= T_loc.  Local key j sits
    at global position pos0 + j and is rotated there; query token i is local
    token T_loc - T + i, at position pos0 + T_loc - T + i.  Local key j is
    visible to query i iff j <= T_loc - T + i; memory rows are always visible.
    Returns O [B][T][Hq][D].
    """
    q, k_loc, v_loc = _f64(q), _f64(k_loc), _f64(v_loc)
    B, T, Hq, D = q.shape
    T_loc, H = k_loc.shape[1], k_loc.shape[2]
    if T > T_loc:
        raise ValueError("T must not exceed T_loc")
    if Hq % H:
        raise ValueError("Hq must be a multiple of H")
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.empty((B, T, Hq, D))
    q_pos = pos0 + (T_loc - T) + np.arange(T)
    k_pos = pos0 + np.arange(T_loc)
    i_idx = np.arange(T)[:, None]
    j_idx = np.arange(T_loc)[None, :]
    local_ok = j_idx <= (T_loc - T) + i_idx  # [T][T_loc]
    for b in range(B):
        km, vm = _f64(k_mem[b]), _f64(v_mem[b])
        M = km.shape[0]
        for hq in range(Hq):
            g = (hq * H) // Hq
            qr = rope_rotate(q[b, :, hq, :], q_pos, rope_base)       # [T][D]
            kl = rope_rotate(k_loc[b, :, g, :], k_pos, rope_base)    # [T_loc][D]
            keys = np.concatenate([km[:, g, :].reshape(M, D), kl], axis=0)
            vals = np.concatenate([vm[:, g, :].reshape(M, D), v_loc[b, :, g, :]],
                                  axis=0)
            logits = (qr @ keys.T) * scale                           # [T][M+T_loc]
            ok = np.concatenate([np.ones((T, M), dtype=bool), local_ok], axis=1)
            logits = np.where(ok, logits, -np.inf)
            m = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - m)
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, hq, :] = p @ vals
    return out


def msa_forward(k_tok, v_tok, kr_tok, tok_offsets, q_r, q, k_loc, v_loc,
                k: int, rope_base: float = 10000.0, chunk: int = CHUNK,
                pos0: int | None = None):
    """Whole path on one layer: encode -> route -> top-k -> gather -> attend.

    Token tensors are [1][N][H][D] (one routed layer).  ``pos0`` defaults to
    ``k``, the number of retrieved documents.  Returns a dict of every
    intermediate.
    """
    kb, vb, rb, coff = encode_pool(k_tok, v_tok, kr_tok, tok_offsets,
                                   rope_base, chunk)
    doc_s, chunk_s = route_scores(q_r, rb[0], coff)
    idx, top_s = topk_docs(doc_s, k)
    k_mem, v_mem, mem_len = gather_kv(idx, coff, kb[0], vb[0])
    o = sparse_attn(q, k_mem, v_mem, k_loc, v_loc,
                    k if pos0 is None else pos0, rope_base)
    return dict(k_bar=kb, v_bar=vb, kr_bar=rb, chunk_offsets=coff,
                doc_scores=doc_s, chunk_scores=chunk_s, topk_idx=idx,
                topk_scores=top_s, k_mem=k_mem, v_mem=v_mem, mem_len=mem_len,
                out=o)
