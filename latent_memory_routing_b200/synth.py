"""Seeded synthetic inputs for the MSA hot path.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no RoPE, pooling, chunking, scoring or attention), so
both the CUDA path and the float64 oracle can be fed from it.  Chunk offsets,
where a generator needs them (pooled banks, pooled needles), are passed in by
the caller.

Workloads (sizes follow the method's published setting: 64-token chunks,
8 routing/KV heads of dim 128 and 32 query heads for the 4B-class backbone,
top-16 documents, banks of 1M to 100M tokens):

``tiny``      16 docs x 180 tokens, H=2, D=64, Hq=4, fp32, planted needle in
              doc 5, top-2, global RoPE offset 2.
``bank_1m``   1,000 docs, lengths U[256,1792], token-level bf16, one
              128-token prefill query, 4 planted needles, top-16.
``bank_10m``  10,000 docs, lengths log-normal (median 800, sigma 0.65,
              clipped to [64, 8192]); pooled bf16 bank drawn directly; 64
              single-token decode queries with 2,048 local tokens, top-16.
``bank_100m`` 100,000 docs, lengths U[500,1500]; pooled bf16 bank drawn
              directly (~1.56M chunks); one 256-token prefill query,
              8 planted needles, top-16.
``encode_4l`` 4 routed layers x 1M tokens, lengths U[100,4000], token-level
              bf16 K/V/K_r for encoding throughput.

Values are i.i.d. N(0,1).  A planted needle document has routing keys equal
to the query's mean routing direction u_h = normalise(mean_t Q_r[t,h]) plus
noise (0.1 N(0,1) per token; for banks drawn at chunk level the noise of a
full 64-token chunk mean, 0.1/8 N(0,1)).
"""

from __future__ import annotations

import math

import torch

SEEDS = {"tiny": 1001, "bank_1m": 1002, "bank_10m": 1003,
         "bank_100m": 1004, "encode_4l": 1005, "backward_1m": 1006}

NEEDLE_SIGMA_TOKEN = 0.1
NEEDLE_SIGMA_POOLED = 0.1 / 8.0


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn(shape, dtype, device, gen) -> torch.Tensor:
    return torch.randn(*shape, dtype=torch.float32, device=device,
                       generator=gen).to(dtype)


def tok_offsets(lengths: torch.Tensor) -> torch.Tensor:
    """Prefix sum of document lengths with a leading 0 (int64, CPU)."""
    lengths = lengths.to(torch.int64).cpu()
    out = torch.zeros(lengths.numel() + 1, dtype=torch.int64)
    out[1:] = torch.cumsum(lengths, 0)
    return out


def lengths_uniform(n_docs: int, lo: int, hi: int, gen_cpu) -> torch.Tensor:
    return torch.randint(lo, hi + 1, (n_docs,), generator=gen_cpu,
                         dtype=torch.int64)


def lengths_lognormal(n_docs: int, median: float, sigma: float, lo: int,
                      hi: int, gen_cpu) -> torch.Tensor:
    z = torch.randn(n_docs, generator=gen_cpu, dtype=torch.float64)
    x = torch.exp(math.log(median) + sigma * z)
    return torch.clamp(torch.round(x), lo, hi).to(torch.int64)


def lengths_to_total(total: int, lo: int, hi: int, gen_cpu) -> torch.Tensor:
    """Draw U[lo,hi] lengths until they cover ``total`` tokens; the last
    document is cut so the lengths sum to exactly ``total``."""
    out, acc = [], 0
    while acc < total:
        n = int(torch.randint(lo, hi + 1, (1,), generator=gen_cpu).item())
        n = min(n, total - acc)
        out.append(n)
        acc += n
    return torch.tensor(out, dtype=torch.int64)


def mean_direction(q_r_b: torch.Tensor) -> torch.Tensor:
    """u_h = normalise(mean over tokens of Q_r[t, h]); q_r_b: [T][H][D].
    Input construction for planted needles only."""
    m = q_r_b.float().mean(dim=0)
    return m / m.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def plant_token_needles(kr_tok: torch.Tensor, toff: torch.Tensor, docs,
                        q_r_b: torch.Tensor, gen, layer: int = 0,
                        sigma: float = NEEDLE_SIGMA_TOKEN) -> None:
    """Overwrite the token-level routing keys of ``docs`` (in place)."""
    u = mean_direction(q_r_b).to(kr_tok.device)
    for d in docs:
        t0, t1 = int(toff[d]), int(toff[d + 1])
        noise = randn((t1 - t0,) + tuple(u.shape), torch.float32,
                      kr_tok.device, gen)
        kr_tok[layer, t0:t1] = (u.unsqueeze(0) + sigma * noise).to(kr_tok.dtype)


def plant_pooled_needles(kr_bar: torch.Tensor, chunk_offsets, docs,
                         q_r_b: torch.Tensor, gen,
                         sigma: float = NEEDLE_SIGMA_POOLED) -> None:
    """Overwrite the pooled routing-key rows of ``docs`` (in place).
    ``chunk_offsets`` comes from the caller."""
    u = mean_direction(q_r_b).to(kr_bar.device)
    for d in docs:
        c0, c1 = int(chunk_offsets[d]), int(chunk_offsets[d + 1])
        noise = randn((c1 - c0,) + tuple(u.shape), torch.float32,
                      kr_bar.device, gen)
        kr_bar[c0:c1] = (u.unsqueeze(0) + sigma * noise).to(kr_bar.dtype)


# ----------------------------------------------------------------------------
# Workloads
# ----------------------------------------------------------------------------

def tiny(device="cpu") -> dict:
    """16 docs x 180 tokens, fp32, H=2, D=64, Hq=4, needle in doc 5."""
    g = _gen(device, SEEDS["tiny"])
    H, D, Hq, T = 2, 64, 4, 16
    lengths = torch.full((16,), 180, dtype=torch.int64)
    toff = tok_offsets(lengths)
    N = int(toff[-1])
    dt = torch.float32
    w = dict(name="tiny", dtype=dt, H=H, D=D, Hq=Hq, L=1, T=T, T_loc=T,
             B=1, k=2, pos0=2, rope_base=10000.0, chunk=64,
             lengths=lengths, tok_offsets=toff, needles=[5])
    w["k_tok"] = randn((1, N, H, D), dt, device, g)
    w["v_tok"] = randn((1, N, H, D), dt, device, g)
    w["kr_tok"] = randn((1, N, H, D), dt, device, g)
    w["q"] = randn((1, T, Hq, D), dt, device, g)
    w["q_r"] = randn((1, T, H, D), dt, device, g)
    w["k_loc"] = randn((1, T, H, D), dt, device, g)
    w["v_loc"] = randn((1, T, H, D), dt, device, g)
    plant_token_needles(w["kr_tok"], toff, [5], w["q_r"][0], g)
    return w


def bank_1m(device="cpu", n_docs: int = 1000, T: int = 128) -> dict:
    """Token-level bf16 bank of ~1M tokens with 4 needles; one prefill
    query of T tokens.  ``n_docs`` can be lowered for quick tests."""
    gc = _gen("cpu", SEEDS["bank_1m"])
    g = _gen(device, SEEDS["bank_1m"] + 100)
    H, D, Hq = 8, 128, 32
    lengths = lengths_uniform(n_docs, 256, 1792, gc)
    needles = torch.randperm(n_docs, generator=gc)[:min(4, n_docs)].tolist()
    toff = tok_offsets(lengths)
    N = int(toff[-1])
    dt = torch.bfloat16
    w = dict(name="bank_1m", dtype=dt, H=H, D=D, Hq=Hq, L=1, T=T, T_loc=T,
             B=1, k=16, pos0=16, rope_base=10000.0, chunk=64,
             lengths=lengths, tok_offsets=toff, needles=needles)
    w["k_tok"] = randn((1, N, H, D), dt, device, g)
    w["v_tok"] = randn((1, N, H, D), dt, device, g)
    w["kr_tok"] = randn((1, N, H, D), dt, device, g)
    w["q"] = randn((1, T, Hq, D), dt, device, g)
    w["q_r"] = randn((1, T, H, D), dt, device, g)
    w["k_loc"] = randn((1, T, H, D), dt, device, g)
    w["v_loc"] = randn((1, T, H, D), dt, device, g)
    plant_token_needles(w["kr_tok"], toff, needles, w["q_r"][0], g)
    return w


def backward_1m(chunk_offsets, n_tok: int, device="cpu", T: int = 128) -> dict:
    """Inputs of the backward of routing and pooling over the bank_1m
    document set (lengths as ``bank_1m`` draws them; ``chunk_offsets`` and
    ``n_tok`` from the caller): a pooled routing bank and one T-token query
    (bf16 N(0,1)), a dense dL/d(doc score) over every document (the shape of
    an InfoNCE gradient: softmax(scores) - one-hot, drawn here as N(0,1)/n_docs)
    and fp32 N(0,1) gradients of the pooled K, V and K_r banks."""
    g = _gen(device, SEEDS["backward_1m"])
    H, D = 8, 128
    C = int(chunk_offsets[-1])
    n_docs = len(chunk_offsets) - 1
    w = dict(name="backward_1m", H=H, D=D, T=T, B=1, n_docs=n_docs, n_tok=n_tok)
    w["q_r"] = randn((1, T, H, D), torch.bfloat16, device, g)
    w["kr_bar"] = randn((C, H, D), torch.bfloat16, device, g)
    w["d_doc"] = torch.randn((1, n_docs), generator=g, device=device) / n_docs
    for name in ("dk_bar", "dv_bar", "dkr_bar"):
        w[name] = torch.randn((1, C, H, D), generator=g, device=device)
    return w


def bank_1m_lengths(n_docs: int = 1000) -> torch.Tensor:
    """The document lengths ``bank_1m`` draws (its generator's first draw)."""
    return lengths_uniform(n_docs, 256, 1792, _gen("cpu", SEEDS["bank_1m"]))


def bank_10m_lengths(n_docs: int = 10000) -> torch.Tensor:
    gc = _gen("cpu", SEEDS["bank_10m"])
    return lengths_lognormal(n_docs, 800.0, 0.65, 64, 8192, gc)


def bank_10m(chunk_offsets, device="cpu", B: int = 64, T_loc: int = 2048,
             n_docs: int = 10000) -> dict:
    """Pooled bf16 bank for the 10M-token decode workload.  ``chunk_offsets``
    (from the caller) sizes the bank."""
    lengths = bank_10m_lengths(n_docs)
    g = _gen(device, SEEDS["bank_10m"] + 100)
    H, D, Hq = 8, 128, 32
    C = int(chunk_offsets[-1])
    dt = torch.bfloat16
    w = dict(name="bank_10m", dtype=dt, H=H, D=D, Hq=Hq, L=1, T=1,
             T_loc=T_loc, B=B, k=16, pos0=16, rope_base=10000.0, chunk=64,
             lengths=lengths, tok_offsets=tok_offsets(lengths), needles=[])
    w["kr_bar"] = randn((C, H, D), dt, device, g)
    w["k_bar"] = randn((C, H, D), dt, device, g)
    w["v_bar"] = randn((C, H, D), dt, device, g)
    w["q"] = randn((B, 1, Hq, D), dt, device, g)
    w["q_r"] = randn((B, 1, H, D), dt, device, g)
    w["k_loc"] = randn((B, T_loc, H, D), dt, device, g)
    w["v_loc"] = randn((B, T_loc, H, D), dt, device, g)
    return w


def bank_100m_lengths(n_docs: int = 100000) -> torch.Tensor:
    gc = _gen("cpu", SEEDS["bank_100m"])
    return lengths_uniform(n_docs, 500, 1500, gc)


def bank_100m(chunk_offsets, device="cpu", T: int = 256,
              n_docs: int = 100000, n_needles: int = 8) -> dict:
    """Pooled bf16 bank for the 100M-token prefill workload, with planted
    needles.  ``chunk_offsets`` (from the caller) sizes the bank."""
    lengths = bank_100m_lengths(n_docs)
    gc = _gen("cpu", SEEDS["bank_100m"] + 1)
    needles = torch.randperm(n_docs, generator=gc)[:n_needles].tolist()
    g = _gen(device, SEEDS["bank_100m"] + 100)
    H, D, Hq = 8, 128, 32
    C = int(chunk_offsets[-1])
    dt = torch.bfloat16
    w = dict(name="bank_100m", dtype=dt, H=H, D=D, Hq=Hq, L=1, T=T, T_loc=T,
             B=1, k=16, pos0=16, rope_base=10000.0, chunk=64,
             lengths=lengths, tok_offsets=tok_offsets(lengths),
             needles=needles)
    w["kr_bar"] = randn((C, H, D), dt, device, g)
    w["k_bar"] = randn((C, H, D), dt, device, g)
    w["v_bar"] = randn((C, H, D), dt, device, g)
    w["q"] = randn((1, T, Hq, D), dt, device, g)
    w["q_r"] = randn((1, T, H, D), dt, device, g)
    w["k_loc"] = randn((1, T, H, D), dt, device, g)
    w["v_loc"] = randn((1, T, H, D), dt, device, g)
    plant_pooled_needles(w["kr_bar"], chunk_offsets, needles, w["q_r"][0], g)
    return w


def encode_4l(device="cpu", L: int = 4, n_tok: int = 1_000_000) -> dict:
    """Token-level bf16 K/V/K_r for encoding throughput ([L][N][8][128])."""
    gc = _gen("cpu", SEEDS["encode_4l"])
    g = _gen(device, SEEDS["encode_4l"] + 100)
    H, D = 8, 128
    lengths = lengths_to_total(n_tok, 100, 4000, gc)
    dt = torch.bfloat16
    w = dict(name="encode_4l", dtype=dt, H=H, D=D, L=L, rope_base=10000.0,
             chunk=64, lengths=lengths, tok_offsets=tok_offsets(lengths))
    w["k_tok"] = randn((L, n_tok, H, D), dt, device, g)
    w["v_tok"] = randn((L, n_tok, H, D), dt, device, g)
    w["kr_tok"] = randn((L, n_tok, H, D), dt, device, g)
    return w
