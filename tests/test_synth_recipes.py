"""The seeded input recipes (latent_memory_routing_b200.synth) on the CPU:
document counts, length ranges, token and chunk totals of each workload, as
the design notes and the benchmark's config state them, and the planted
needle of the tiny workload.  The values are fixed by the seeds, so a change
to a recipe shows up here."""

import numpy as np
import torch

import oracle
from latent_memory_routing_b200 import synth


def _stats(lengths):
    c = oracle.chunk_offsets_from_lengths(lengths.numpy())
    return len(lengths), int(lengths.sum()), int(c[-1]), int(lengths.min()), int(lengths.max())


def test_bank_1m_lengths():
    n, tok, chunks, lo, hi = _stats(synth.bank_1m_lengths())
    assert (n, chunks) == (1000, 16312)
    assert 256 <= lo and hi <= 1792 and tok == 1012871


def test_bank_10m_lengths():
    n, tok, chunks, lo, hi = _stats(synth.bank_10m_lengths())
    assert (n, tok, chunks) == (10000, 9913039, 159814)
    assert 64 <= lo and hi <= 8192


def test_bank_100m_lengths():
    n, tok, chunks, lo, hi = _stats(synth.bank_100m_lengths())
    assert (n, tok, chunks) == (100000, 100024189, 1612509)
    assert 500 <= lo and hi <= 1500


def test_encode_4l_lengths_cover_exactly_one_million_tokens():
    gc = synth._gen("cpu", synth.SEEDS["encode_4l"])
    n, tok, chunks, lo, hi = _stats(synth.lengths_to_total(1_000_000, 100, 4000, gc))
    assert (n, tok, chunks) == (491, 1_000_000, 15866)
    assert 1 <= lo and hi <= 4000


def test_recipes_are_deterministic():
    assert torch.equal(synth.bank_10m_lengths(), synth.bank_10m_lengths())
    a, b = synth.tiny("cpu"), synth.tiny("cpu")
    for key in ("k_tok", "v_tok", "kr_tok", "q", "q_r", "k_loc", "v_loc"):
        assert torch.equal(a[key], b[key]), key


def test_tiny_workload_shapes_and_needle():
    w = synth.tiny("cpu")
    assert w["k_tok"].shape == (1, 16 * 180, 2, 64) and w["k_tok"].dtype == torch.float32
    assert w["q"].shape == (1, 16, 4, 64) and w["q_r"].shape == (1, 16, 2, 64)
    assert w["tok_offsets"].tolist() == [180 * d for d in range(17)]
    # the needle document's routing keys point along the mean query direction
    u = synth.mean_direction(w["q_r"][0]).double().numpy()          # [H][D]
    kr = w["kr_tok"][0].double().numpy()                            # [N][H][D]
    cos = np.einsum("nhd,hd->nh", kr, u) / np.linalg.norm(kr, axis=-1)
    per_doc = cos.reshape(16, 180, 2).mean(axis=(1, 2))
    assert int(np.argmax(per_doc)) == 5
    assert per_doc[5] > 0.6 and np.max(np.delete(per_doc, 5)) < 0.2
