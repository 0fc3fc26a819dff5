"""Loop-only float64 restatement of the MSA hot path, for tiny shapes.

TEST INFRASTRUCTURE ONLY.  It re-derives every step element by element with
Python scalars and ``math`` so that the vectorised oracle in ``msa_oracle``
can be checked against a structurally different program (no NumPy
broadcasting, no matmul, no reduceat, no lexsort).  Citations and readings are
the same as in ``msa_oracle``:

* chunking and pooling: "深度分析MSA:把超长文档组织成可检索内部记忆的工程路径",
  § "三、文档如何变成 memory" / "2. chunk 压缩";
* RoPE, routing, sparse attention: "EverMind-AI/MSA: routing top-k compressed
  documents inside attention, and where the 100M-token claim stops",
  §§ "Document-wise RoPE resets every document to position zero" and
  "Routing happens inside attention, not in a retrieval service in front of
  the model".

Tensors are nested Python lists (or anything indexable) of floats.
"""

from __future__ import annotations

import math


def n_chunks(length: int, chunk: int = 64) -> int:
    n = 0
    start = 0
    while start < length:  # one chunk per started group of `chunk` tokens
        n += 1
        start += chunk
    return n


def rope_vec(x, p: int, base: float):
    """Rotate one head vector x (length D) to position p, pair (i, i+D/2)."""
    D = len(x)
    half = D // 2
    y = [0.0] * D
    for i in range(half):
        w = base ** (-(2.0 * i) / D)
        a = p * w
        c, s = math.cos(a), math.sin(a)
        y[i] = x[i] * c - x[i + half] * s
        y[i + half] = x[i + half] * c + x[i] * s
    return y


def encode_doc(k_doc, v_doc, kr_doc, base: float, chunk: int = 64):
    """k_doc etc: [len][H][D] lists.  Returns pooled ([n][H][D],)*3."""
    length = len(k_doc)
    H = len(k_doc[0])
    D = len(k_doc[0][0])
    kb, vb, rb = [], [], []
    for j in range(n_chunks(length, chunk)):
        a = j * chunk
        b = min(a + chunk, length)
        cnt = b - a
        ks = [[0.0] * D for _ in range(H)]
        vs = [[0.0] * D for _ in range(H)]
        rs = [[0.0] * D for _ in range(H)]
        for t in range(a, b):
            for h in range(H):
                kr = rope_vec(k_doc[t][h], t, base)  # position within doc
                for d in range(D):
                    ks[h][d] += kr[d]
                    vs[h][d] += float(v_doc[t][h][d])
                    rs[h][d] += float(kr_doc[t][h][d])
        kb.append([[x / cnt for x in row] for row in ks])
        vb.append([[x / cnt for x in row] for row in vs])
        rb.append([[x / cnt for x in row] for row in rs])
    return kb, vb, rb


def cos_scalar(q, k, eps: float = 1e-12) -> float:
    dot = 0.0
    qq = 0.0
    kk = 0.0
    for a, b in zip(q, k):
        dot += a * b
        qq += a * a
        kk += b * b
    return dot / (max(math.sqrt(qq), eps) * max(math.sqrt(kk), eps))


def chunk_score(q_r_b, kr_c) -> float:
    """q_r_b: [T][H][D], kr_c: [H][D] -> max_t mean_h cos."""
    best = -math.inf
    H = len(kr_c)
    for t in range(len(q_r_b)):
        acc = 0.0
        for h in range(H):
            acc += cos_scalar(q_r_b[t][h], kr_c[h])
        best = max(best, acc / H)
    return best


def route(q_r, kr_bar, chunk_offsets):
    """Returns (doc_scores [B][n_docs], chunk_scores [B][C]) as lists."""
    n_docs = len(chunk_offsets) - 1
    doc_s, chunk_s = [], []
    for b in range(len(q_r)):
        cs = [chunk_score(q_r[b], kr_bar[c]) for c in range(len(kr_bar))]
        ds = []
        for d in range(n_docs):
            best = -math.inf
            for c in range(chunk_offsets[d], chunk_offsets[d + 1]):
                if cs[c] > best:
                    best = cs[c]
            ds.append(best)
        chunk_s.append(cs)
        doc_s.append(ds)
    return doc_s, chunk_s


def topk(scores_b, k: int):
    """Selection by repeated arg-max: strictly greater score wins, equal
    scores keep the lower index."""
    taken = [False] * len(scores_b)
    out = []
    for _ in range(k):
        best = -1
        for i, s in enumerate(scores_b):
            if taken[i]:
                continue
            if best < 0 or s > scores_b[best]:
                best = i
        taken[best] = True
        out.append(best)
    return out


def attend(q_b, kmem_b, vmem_b, kloc_b, vloc_b, pos0: int, base: float):
    """One query batch element.  q_b: [T][Hq][D]; kmem_b: [M][H][D];
    kloc_b: [T_loc][H][D].  Returns [T][Hq][D]."""
    T = len(q_b)
    Hq = len(q_b[0])
    D = len(q_b[0][0])
    T_loc = len(kloc_b)
    H = len(kloc_b[0])
    M = len(kmem_b)
    scale = 1.0 / math.sqrt(D)
    out = []
    for i in range(T):
        row = []
        for hq in range(Hq):
            g = (hq * H) // Hq
            qv = rope_vec(q_b[i][hq], pos0 + T_loc - T + i, base)
            logits, vals = [], []
            for m in range(M):
                logits.append(sum(a * b for a, b in zip(qv, kmem_b[m][g])) * scale)
                vals.append(vmem_b[m][g])
            for j in range(T_loc):
                if j > T_loc - T + i:
                    continue
                kv = rope_vec(kloc_b[j][g], pos0 + j, base)
                logits.append(sum(a * b for a, b in zip(qv, kv)) * scale)
                vals.append(vloc_b[j][g])
            mx = max(logits)
            ws = [math.exp(x - mx) for x in logits]
            tot = sum(ws)
            o = [0.0] * D
            for w, v in zip(ws, vals):
                for d in range(D):
                    o[d] += w * float(v[d]) / tot
            row.append(o)
        out.append(row)
    return out
