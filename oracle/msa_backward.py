"""Float64 CPU oracle of the backward pass of chunk pooling and routing.

TEST INFRASTRUCTURE ONLY: imported by the tests, never by the product
library.

Source: "深度分析MSA:把超长文档组织成可检索内部记忆的工程路径"
(yeyulingfeng.com), section "四、训练阶段：学习 memory 与路由": a training
step encodes the documents (token K/V/K_r, then chunk pooling into the
memory), routes Q_r against the pooled routing keys, and its routing
auxiliary loss -- BCE or InfoNCE over the documents' scores -- sends
gradients back to Q_r and, through the pooling, to the token-level K_r (the
language-model loss reaches Q, K and V).  The loss itself is the caller's:
this module takes the gradient of the loss with respect to the document
scores and returns the gradients of the routing inputs, and takes the
gradients of the pooled bank and returns those of the token tensors.

Readings taken where the page is silent:

* The gradient of a maximum goes entirely to its first maximiser: a
  document's score is that of its best (chunk, query token) pair, the lowest
  chunk index among equal chunk scores and, inside that chunk, the lowest
  token index among equal head-mean cosines.
* The cosine divides by max(|x|, 1e-12) for each vector; below 1e-12 that
  norm is the constant 1e-12 (its gradient has no norm term).
* Chunk pooling is linear, so its backward is its adjoint: the gradient of a
  pooled row, divided by the chunk's token count, reaches each of its tokens,
  and for K it is rotated back by the token's document-wise position
  (R(p) is orthogonal, R(p)^T = R(-p)).

Everything is computed in float64.
"""

from __future__ import annotations

import numpy as np

from .msa_oracle import CHUNK, EPS, _f64, chunk_offsets_from_lengths, chunk_token_ranges, rope_rotate


def cosine_grad(q, k, eps: float = EPS):
    """Gradients of cos(q, k) = q.k / (max(|q|, eps) max(|k|, eps)) with
    respect to q and k (vectors on the last axis)."""
    q, k = _f64(q), _f64(k)
    lq = np.linalg.norm(q, axis=-1, keepdims=True)
    lk = np.linalg.norm(k, axis=-1, keepdims=True)
    nq, nk = np.maximum(lq, eps), np.maximum(lk, eps)
    c = (q * k).sum(axis=-1, keepdims=True) / (nq * nk)
    dq = k / (nq * nk) - np.where(lq >= eps, c * q / (nq * nq), 0.0)
    dk = q / (nq * nk) - np.where(lk >= eps, c * k / (nk * nk), 0.0)
    return dq, dk


def route_argmax(q_r, kr_bar, chunk_offsets, eps: float = EPS):
    """Per (query b, document d): the score max over (chunk, token) of the
    head-mean cosine, and the first maximiser (chunk c*, token t*).

    Returns (doc_scores [B][n_docs], c_star, t_star), the index arrays
    [B][n_docs] int64 (c* is a global chunk index)."""
    q, k = _f64(q_r), _f64(kr_bar)
    coff = np.asarray(chunk_offsets, dtype=np.int64)
    B, T, H, D = q.shape
    n_docs = len(coff) - 1
    qn = q / np.maximum(np.linalg.norm(q, axis=-1, keepdims=True), eps)
    kn = k / np.maximum(np.linalg.norm(k, axis=-1, keepdims=True), eps)
    scores = np.empty((B, n_docs))
    c_star = np.empty((B, n_docs), dtype=np.int64)
    t_star = np.empty((B, n_docs), dtype=np.int64)
    for d in range(n_docs):
        c0, c1 = int(coff[d]), int(coff[d + 1])
        # s[b, c, t] = (1/H) sum_h cos(Q_r[b,t,h], K_r[c,h])
        s = np.einsum("bthd,chd->bct", qn, kn[c0:c1]) / H
        flat = s.reshape(B, -1)
        j = flat.argmax(axis=1)  # first maximum: lowest chunk, then lowest token
        scores[:, d] = flat[np.arange(B), j]
        c_star[:, d] = c0 + j // T
        t_star[:, d] = j % T
    return scores, c_star, t_star


def route_scores_backward(q_r, kr_bar, chunk_offsets, d_doc, eps: float = EPS):
    """Gradients of L with respect to Q_r [B][T][H][D] and K̄_r [C][H][D],
    given dL/d(doc_scores) [B][n_docs]: each document's score is
    (1/H) sum_h cos(Q_r[b,t*,h], K̄_r[c*,h]) at its first maximiser."""
    q, k = _f64(q_r), _f64(kr_bar)
    g = _f64(d_doc)
    B, T, H, D = q.shape
    _, c_star, t_star = route_argmax(q, k, chunk_offsets, eps)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    for b in range(B):
        for d in np.nonzero(g[b])[0]:
            c, t = int(c_star[b, d]), int(t_star[b, d])
            gq, gk = cosine_grad(q[b, t], k[c], eps)  # [H][D] each
            dq[b, t] += g[b, d] / H * gq
            dk[c] += g[b, d] / H * gk
    return dq, dk


def encode_pool_backward(dk_bar, dv_bar, dkr_bar, tok_offsets, rope_base: float = 10000.0,
                         chunk: int = CHUNK):
    """Adjoint of encode_pool: gradients of the pooled banks [L][C][H][D] ->
    gradients of the token tensors [L][N][H][D]."""
    dk_bar, dv_bar, dkr_bar = _f64(dk_bar), _f64(dv_bar), _f64(dkr_bar)
    tok_offsets = np.asarray(tok_offsets, dtype=np.int64)
    lengths = np.diff(tok_offsets)
    coff = chunk_offsets_from_lengths(lengths, chunk)
    L, C, H, D = dk_bar.shape
    N = int(tok_offsets[-1])
    dk = np.zeros((L, N, H, D))
    dv = np.zeros((L, N, H, D))
    dkr = np.zeros((L, N, H, D))
    for d, n in enumerate(lengths):
        t0 = int(tok_offsets[d])
        for j, (a, b) in enumerate(chunk_token_ranges(int(n), chunk)):
            c = int(coff[d]) + j
            cnt = b - a
            dv[:, t0 + a:t0 + b] = dv_bar[:, c][:, None] / cnt
            dkr[:, t0 + a:t0 + b] = dkr_bar[:, c][:, None] / cnt
            # K was rotated by its document-wise position p before pooling:
            # the gradient is rotated back, R(p)^T = R(-p)
            for lyr in range(L):
                rows = np.repeat(dk_bar[lyr, c][None] / cnt, cnt, axis=0)
                dk[lyr, t0 + a:t0 + b] = rope_rotate(rows, -np.arange(a, b), rope_base)
    return dk, dv, dkr
