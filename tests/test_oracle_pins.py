"""Pins of the float64 oracle against facts that do not come from the oracle.

Each test checks the oracle against something fixed outside it: the worked
example printed on the pages (tests/golden/), closed forms, invariants, a
library routine on a special case, or the loop-only restatement on tiny
inputs.  They are chosen so that a dropped term, a wrong sign, a wrong index
or a transposed operand in the oracle fails at least one of them; the
``TestPlantedMistakes`` class plants such mistakes in the oracle and checks
that a pin fires.
"""

import os

import numpy as np
import pytest
import torch

import oracle
from oracle import msa_loops as loops
from oracle import msa_oracle as mo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *rest = line.split()
            vals[key] = [int(x) for x in rest]
    return vals


# ---------------------------------------------------------------- chunking

class TestChunking:
    def test_worked_example_180_tokens(self):
        g = _read_golden("chunking_180.txt")
        length, chunk = g["length"][0], g["chunk"][0]
        assert oracle.chunk_counts([length], chunk).tolist() == g["n_chunks"]
        sizes = [b - a for a, b in oracle.chunk_token_ranges(length, chunk)]
        assert sizes == g["sizes"]
        assert loops.n_chunks(length, chunk) == g["n_chunks"][0]

    def test_offsets_and_ranges_cover_documents(self):
        lengths = [1, 63, 64, 65, 128, 129, 180, 4000]
        off = oracle.chunk_offsets_from_lengths(lengths)
        assert off[0] == 0
        for d, n in enumerate(lengths):
            r = oracle.chunk_token_ranges(n)
            assert len(r) == off[d + 1] - off[d] == loops.n_chunks(n)
            assert r[0][0] == 0 and r[-1][1] == n
            assert all(a2 == b1 for (_, b1), (a2, _) in zip(r, r[1:]))
            assert all(0 < b - a <= 64 for a, b in r)

    def test_empty_document_rejected(self):
        with pytest.raises(ValueError):
            oracle.chunk_counts([5, 0, 3])


# -------------------------------------------------------------------- RoPE

class TestRope:
    def test_frequency_values(self):
        # base^(-2i/D): D=4, base=10000 -> 1 and 10000^(-1/2) = 0.01
        np.testing.assert_allclose(oracle.rope_inv_freq(4, 10000.0),
                                   [1.0, 0.01], rtol=0, atol=1e-15)

    def test_identity_at_position_zero(self):
        x = _rng(1).standard_normal((3, 2, 8))
        np.testing.assert_array_equal(oracle.rope_rotate(x, [0, 0, 0], 1e4), x)

    def test_norm_preserved(self):
        x = _rng(2).standard_normal((50, 3, 64))
        y = oracle.rope_rotate(x, np.arange(50) * 37, 10000.0)
        np.testing.assert_allclose(np.linalg.norm(y, axis=-1),
                                   np.linalg.norm(x, axis=-1), rtol=1e-13)

    def test_equals_complex_multiplication(self):
        # pair (x_i, x_{i+D/2}) as the complex number x_i + j x_{i+D/2},
        # multiplied by exp(j p w_i): an independent statement of the rotation
        D, base = 16, 500.0
        x = _rng(3).standard_normal((7, D))
        pos = np.array([0, 1, 2, 5, 11, 100, 1234])
        w = np.array([base ** (-(2.0 * i) / D) for i in range(D // 2)])
        z = (x[:, :D // 2] + 1j * x[:, D // 2:]) * np.exp(1j * np.outer(pos, w))
        want = np.concatenate([z.real, z.imag], axis=1)
        np.testing.assert_allclose(oracle.rope_rotate(x, pos, base), want,
                                   rtol=0, atol=1e-12)

    def test_relative_position_property(self):
        rng = _rng(4)
        q, k = rng.standard_normal(32), rng.standard_normal(32)
        def dot(m, n):
            return float(oracle.rope_rotate(q[None], [m], 1e4)[0]
                         @ oracle.rope_rotate(k[None], [n], 1e4)[0])
        for m, n, s in [(3, 7, 11), (100, 5, 900), (0, 0, 64)]:
            assert dot(m, n) == pytest.approx(dot(m + s, n + s), abs=1e-10)

    def test_loop_twin(self):
        x = _rng(5).standard_normal((4, 8))
        pos = [0, 3, 9, 70]
        got = oracle.rope_rotate(x, pos, 10000.0)
        for r in range(4):
            np.testing.assert_allclose(got[r], loops.rope_vec(list(x[r]), pos[r], 1e4),
                                       atol=1e-13)


# ---------------------------------------------------------------- encoding

class TestEncode:
    def _doc(self, n, H=2, D=4, seed=6):
        rng = _rng(seed)
        return [rng.standard_normal((n, H, D)) for _ in range(3)]

    def test_pool_equals_brute_force_sums(self):
        for n, chunk in [(5, 2), (7, 3), (180, 64), (64, 64), (1, 64)]:
            k, v, r = self._doc(n)
            got = oracle.encode_pool_doc(k, v, r, 10000.0, chunk)
            want = loops.encode_doc(k.tolist(), v.tolist(), r.tolist(), 10000.0, chunk)
            for g, w in zip(got, want):
                np.testing.assert_allclose(g, np.array(w), rtol=1e-12, atol=1e-12)

    def test_constant_chunk_pools_to_itself(self):
        n = 180
        rng = _rng(7)
        c = rng.standard_normal((1, 2, 4))
        tok = np.repeat(c, n, axis=0)
        _, vb, rb = oracle.encode_pool_doc(tok, tok, tok, 10000.0)
        np.testing.assert_allclose(vb, np.repeat(c, 3, axis=0), rtol=1e-14)
        np.testing.assert_allclose(rb, np.repeat(c, 3, axis=0), rtol=1e-14)

    def test_pooled_rotated_key_geometric_series(self):
        # D=2, inverse frequency 1: a constant key z rotated to positions
        # a..b-1 and averaged is z * sum_p e^{jp} / n, a geometric series.
        # This pins the doc-wise origin (positions restart at 0), the
        # direction of rotation and the 1/count normalisation.
        z = complex(0.3, -1.7)
        n = 180
        tok = np.tile(np.array([[z.real, z.imag]]), (n, 1)).reshape(n, 1, 2)
        kb, _, _ = oracle.encode_pool_doc(tok, tok, tok, 10000.0, 64)
        for j, (a, b) in enumerate([(0, 64), (64, 128), (128, 180)]):
            cnt = b - a
            geo = (np.exp(1j * a) - np.exp(1j * b)) / (1 - np.exp(1j)) / cnt
            want = z * geo
            assert kb[j, 0, 0] == pytest.approx(want.real, abs=1e-12)
            assert kb[j, 0, 1] == pytest.approx(want.imag, abs=1e-12)

    def test_multi_doc_multi_layer_layout(self):
        rng = _rng(8)
        lengths = [70, 5, 130]
        toff = np.concatenate([[0], np.cumsum(lengths)])
        L, H, D = 2, 2, 4
        k, v, r = (rng.standard_normal((L, toff[-1], H, D)) for _ in range(3))
        kb, vb, rb, coff = oracle.encode_pool(k, v, r, toff, 10000.0)
        assert coff.tolist() == [0, 2, 3, 6]
        for l in range(L):
            for d in range(3):
                t0, t1 = toff[d], toff[d + 1]
                want = loops.encode_doc(k[l, t0:t1].tolist(), v[l, t0:t1].tolist(),
                                        r[l, t0:t1].tolist(), 10000.0)
                for got, w in zip((kb, vb, rb), want):
                    np.testing.assert_allclose(got[l, coff[d]:coff[d + 1]], np.array(w),
                                               atol=1e-12)


# ----------------------------------------------------------------- routing

class TestRoute:
    def test_cosine_special_cases(self):
        rng = _rng(9)
        x = rng.standard_normal(64)
        assert oracle.cosine(x, x) == pytest.approx(1.0, abs=1e-15)
        assert oracle.cosine(x, -x) == pytest.approx(-1.0, abs=1e-15)
        assert oracle.cosine(x, 5.0 * x) == pytest.approx(1.0, abs=1e-15)
        assert oracle.cosine(x, np.zeros(64)) == 0.0
        e0, e1 = np.eye(64)[0], np.eye(64)[1]
        assert oracle.cosine(e0, e1) == 0.0

    def test_scores_bounded(self):
        rng = _rng(10)
        q = rng.standard_normal((2, 5, 3, 16))
        k = rng.standard_normal((40, 3, 16))
        s = oracle.route_chunk_scores(q, k)
        assert np.all(s <= 1.0 + 1e-15) and np.all(s >= -1.0 - 1e-15)

    def test_head_mean_then_token_max(self):
        # token 0 matches head 0 only, token 1 matches head 1 only:
        # mean over heads then max over tokens gives 0.5 (max-then-mean
        # would give 1, mean-over-tokens would give 0.5 too but fails below)
        e = np.eye(4)
        q = np.array([[[e[0], e[2]], [e[3], e[1]]]])      # [1][T=2][H=2][4]
        k = np.array([[e[0], e[1]]])                        # [C=1][H=2][4]
        assert oracle.route_chunk_scores(q, k)[0, 0] == pytest.approx(0.5)
        # token 0 matches both heads, token 1 anti-matches both: max over
        # tokens of the head mean is 1 (a mean over tokens would give 0)
        q2 = np.array([[[e[0], e[1]], [-e[0], -e[1]]]])
        assert oracle.route_chunk_scores(q2, k)[0, 0] == pytest.approx(1.0)

    def test_parallel_keys_score_one(self):
        rng = _rng(11)
        q = rng.standard_normal((1, 6, 4, 32))
        k = 3.0 * q[0, 2][None]                             # chunk || token 2
        k = np.concatenate([k, rng.standard_normal((5, 4, 32))])
        s = oracle.route_chunk_scores(q, k)
        assert s[0, 0] == pytest.approx(1.0, abs=1e-14)
        assert np.all(s[0, 1:] < 1.0)

    def test_doc_max(self):
        cs = np.array([[0.1, 0.5, -0.2, 0.3, 0.9, 0.0]])
        assert oracle.doc_max(cs, [0, 2, 3, 6]).tolist() == [[0.5, -0.2, 0.9]]

    def test_loop_twin(self):
        rng = _rng(12)
        q = rng.standard_normal((2, 3, 2, 8))
        k = rng.standard_normal((7, 2, 8))
        coff = [0, 2, 3, 7]
        ds, cs = oracle.route_scores(q, k, coff)
        lds, lcs = loops.route(q.tolist(), k.tolist(), coff)
        np.testing.assert_allclose(cs, np.array(lcs), atol=1e-13)
        np.testing.assert_allclose(ds, np.array(lds), atol=1e-13)


# ------------------------------------------------------------------- top-k

class TestTopk:
    def test_equals_full_sort(self):
        rng = _rng(13)
        s = rng.standard_normal((3, 200))
        idx, top = oracle.topk_docs(s, 16)
        for b in range(3):
            want = sorted(range(200), key=lambda i: (-s[b, i], i))[:16]
            assert idx[b].tolist() == want
            np.testing.assert_array_equal(top[b], s[b, want])

    def test_ties_go_to_lower_index(self):
        s = np.array([[0.5, 0.9, 0.5, 0.9, 0.1, 0.5]])
        idx, _ = oracle.topk_docs(s, 4)
        assert idx[0].tolist() == [1, 3, 0, 2]
        assert loops.topk(s[0].tolist(), 4) == [1, 3, 0, 2]

    def test_permutation(self):
        rng = _rng(14)
        s = rng.permutation(50).astype(float)[None]
        idx, _ = oracle.topk_docs(s, 50)
        assert s[0, idx[0]].tolist() == list(range(49, -1, -1))

    def test_k_bounds(self):
        with pytest.raises(ValueError):
            oracle.topk_docs(np.zeros((1, 3)), 4)


# ------------------------------------------------------------------ gather

class TestGather:
    def test_rank_order_concatenation(self):
        coff = np.array([0, 2, 3, 6, 8])
        kb = np.arange(8 * 2 * 2, dtype=float).reshape(8, 2, 2)
        km, vm, ml = oracle.gather_kv([[2, 0], [1, 3]], coff, kb, -kb)
        assert ml.tolist() == [5, 3]
        np.testing.assert_array_equal(km[0], kb[[3, 4, 5, 0, 1]])
        np.testing.assert_array_equal(km[1], kb[[2, 6, 7]])
        np.testing.assert_array_equal(vm[1], -kb[[2, 6, 7]])


# --------------------------------------------------------------- attention

def _sdpa_reference(q, keys_mem, vals_mem, k_loc, v_loc, pos0, base):
    """torch scaled_dot_product_attention in float64 on inputs rotated by
    the (separately pinned) RoPE, with an explicit visibility mask."""
    B, T, Hq, D = q.shape
    T_loc, H = k_loc.shape[1], k_loc.shape[2]
    out = np.empty_like(q)
    for b in range(B):
        qr = oracle.rope_rotate(q[b], pos0 + T_loc - T + np.arange(T), base)
        kl = oracle.rope_rotate(k_loc[b], pos0 + np.arange(T_loc), base)
        K = np.concatenate([keys_mem[b], kl], 0)             # [M+T_loc][H][D]
        V = np.concatenate([vals_mem[b], v_loc[b]], 0)
        M = keys_mem[b].shape[0]
        rep = Hq // H
        qt = torch.from_numpy(qr).permute(1, 0, 2)                       # [Hq][T][D]
        kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(rep, 0)
        vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(rep, 0)
        mask = torch.ones(T, M + T_loc, dtype=torch.bool)
        for i in range(T):
            mask[i, M + (T_loc - T + i) + 1:] = False
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
        out[b] = o.permute(1, 0, 2).numpy()
    return out


class TestAttention:
    def test_no_memory_is_textbook_causal_attention(self):
        rng = _rng(15)
        B, T, Hq, H, D = 2, 9, 4, 2, 16
        q = rng.standard_normal((B, T, Hq, D))
        kl = rng.standard_normal((B, T, H, D))
        vl = rng.standard_normal((B, T, H, D))
        empty = [np.zeros((0, H, D))] * B
        got = oracle.sparse_attn(q, empty, empty, kl, vl, pos0=3)
        # textbook: torch's causal SDPA on rotated q, k, with KV heads repeated
        rep = Hq // H
        for b in range(B):
            qr = oracle.rope_rotate(q[b], 3 + np.arange(T), 1e4)
            kr = oracle.rope_rotate(kl[b], 3 + np.arange(T), 1e4)
            o = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(qr).permute(1, 0, 2),
                torch.from_numpy(kr).permute(1, 0, 2).repeat_interleave(rep, 0),
                torch.from_numpy(vl[b]).permute(1, 0, 2).repeat_interleave(rep, 0),
                is_causal=True)
            np.testing.assert_allclose(got[b], o.permute(1, 0, 2).numpy(), atol=1e-12)

    def test_with_memory_matches_masked_sdpa(self):
        rng = _rng(16)
        B, T, T_loc, Hq, H, D = 2, 3, 7, 8, 2, 16
        q = rng.standard_normal((B, T, Hq, D))
        kl = rng.standard_normal((B, T_loc, H, D))
        vl = rng.standard_normal((B, T_loc, H, D))
        km = [rng.standard_normal((m, H, D)) for m in (5, 11)]
        vm = [rng.standard_normal((m, H, D)) for m in (5, 11)]
        got = oracle.sparse_attn(q, km, vm, kl, vl, pos0=16)
        want = _sdpa_reference(q, km, vm, kl, vl, 16, 1e4)
        np.testing.assert_allclose(got, want, atol=1e-12)

    def test_single_key_returns_its_value(self):
        rng = _rng(17)
        q = rng.standard_normal((1, 1, 2, 8))
        kl = rng.standard_normal((1, 1, 1, 8))
        vl = rng.standard_normal((1, 1, 1, 8))
        empty = [np.zeros((0, 1, 8))]
        got = oracle.sparse_attn(q, empty, empty, kl, vl, pos0=5)
        np.testing.assert_allclose(got[0, 0, 0], vl[0, 0, 0], atol=1e-15)
        np.testing.assert_allclose(got[0, 0, 1], vl[0, 0, 0], atol=1e-15)

    def test_equal_logits_give_mean_of_visible_values(self):
        rng = _rng(18)
        T, T_loc, D = 2, 4, 8
        q = np.zeros((1, T, 1, D))
        kl = rng.standard_normal((1, T_loc, 1, D))
        vl = rng.standard_normal((1, T_loc, 1, D))
        km = [rng.standard_normal((3, 1, D))]
        vm = [rng.standard_normal((3, 1, D))]
        got = oracle.sparse_attn(q, km, vm, kl, vl, pos0=2)
        for i in range(T):
            vis = np.concatenate([vm[0][:, 0], vl[0, :T_loc - T + i + 1, 0]])
            np.testing.assert_allclose(got[0, i, 0], vis.mean(0), atol=1e-14)

    def test_memory_order_invariance(self):
        rng = _rng(19)
        q = rng.standard_normal((1, 2, 2, 8))
        kl = rng.standard_normal((1, 4, 1, 8))
        vl = rng.standard_normal((1, 4, 1, 8))
        km = rng.standard_normal((6, 1, 8))
        vm = rng.standard_normal((6, 1, 8))
        p = rng.permutation(6)
        a = oracle.sparse_attn(q, [km], [vm], kl, vl, 3)
        b = oracle.sparse_attn(q, [km[p]], [vm[p]], kl, vl, 3)
        np.testing.assert_allclose(a, b, atol=1e-13)

    def test_loop_twin(self):
        rng = _rng(20)
        B, T, T_loc, Hq, H, D = 1, 3, 5, 4, 2, 8
        q = rng.standard_normal((B, T, Hq, D))
        kl = rng.standard_normal((B, T_loc, H, D))
        vl = rng.standard_normal((B, T_loc, H, D))
        km = [rng.standard_normal((4, H, D))]
        vm = [rng.standard_normal((4, H, D))]
        got = oracle.sparse_attn(q, km, vm, kl, vl, 7)
        want = loops.attend(q[0].tolist(), km[0].tolist(), vm[0].tolist(),
                            kl[0].tolist(), vl[0].tolist(), 7, 1e4)
        np.testing.assert_allclose(got[0], np.array(want), atol=1e-12)


# ------------------------------------------------------- needles / pipeline

def _np(t):
    return t.double().cpu().numpy()


class TestNeedle:
    def test_tiny_workload_needle_ranks_first(self):
        from latent_memory_routing_b200 import synth
        w = synth.tiny()
        r = oracle.msa_forward(_np(w["k_tok"]), _np(w["v_tok"]), _np(w["kr_tok"]),
                               w["tok_offsets"].numpy(), _np(w["q_r"]), _np(w["q"]),
                               _np(w["k_loc"]), _np(w["v_loc"]), k=w["k"])
        assert r["topk_idx"][0, 0] == 5
        assert r["chunk_offsets"][-1] == 48
        assert r["mem_len"][0] == 6
        s = r["doc_scores"][0]
        assert s[5] - np.sort(s)[-2] > 0.05
        assert np.all(np.abs(r["chunk_scores"]) <= 1.0)

    def test_rank_one_query_needle_wins_by_margin(self):
        rng = _rng(21)
        T, H, D = 8, 4, 32
        tok = rng.standard_normal((1, H, D))
        q = np.repeat(tok[None], T, axis=1)                 # identical tokens
        bank = rng.standard_normal((30, H, D))
        bank[17:19] = tok + 0.1 * rng.standard_normal((2, H, D))
        coff = [0, 5, 10, 17, 19, 30]
        ds, _ = oracle.route_scores(q, bank, coff)
        idx, top = oracle.topk_docs(ds, 2)
        assert idx[0, 0] == 3
        assert top[0, 0] - top[0, 1] > 0.5


# -------------------------------------------- pins fire on planted mistakes

class TestPlantedMistakes:
    """Each case plants one plausible mistake in the oracle (on the CPU,
    through monkeypatch) and checks that the pins above catch it."""

    def test_wrong_frequency_exponent_is_caught(self, monkeypatch):
        monkeypatch.setattr(mo, "rope_inv_freq",
                            lambda D, base: np.power(float(base), -np.arange(D // 2) / D))
        with pytest.raises(AssertionError):
            TestRope().test_equals_complex_multiplication()

    def test_wrong_rotation_sign_is_caught(self, monkeypatch):
        real = mo.rope_rotate
        monkeypatch.setattr(mo, "rope_rotate",
                            lambda x, pos, base: real(x, -np.asarray(pos), base))
        with pytest.raises(AssertionError):
            TestEncode().test_pooled_rotated_key_geometric_series()

    def test_token_mean_instead_of_max_is_caught(self, monkeypatch):
        def bad(q_r, kr_bar, eps=mo.EPS, block=16384):
            q = np.asarray(q_r, float)
            k = np.asarray(kr_bar, float)
            qn = q / np.linalg.norm(q, axis=-1, keepdims=True)
            kn = k / np.linalg.norm(k, axis=-1, keepdims=True)
            return np.einsum("bthd,chd->btc", qn, kn).mean(1) / q.shape[2]
        monkeypatch.setattr(mo, "route_chunk_scores", bad)
        monkeypatch.setattr(oracle, "route_chunk_scores", bad)
        with pytest.raises(AssertionError):
            TestRoute().test_head_mean_then_token_max()

    def test_causal_off_by_one_is_caught(self, monkeypatch):
        src = mo.sparse_attn

        def shifted(q, k_mem, v_mem, k_loc, v_loc, pos0, rope_base=1e4, scale=None):
            # a query that also sees the next local token
            k_loc = np.asarray(k_loc, float)
            v_loc = np.asarray(v_loc, float)
            pad = np.zeros_like(k_loc[:, :1])
            return src(q, k_mem, v_mem, np.concatenate([k_loc, pad], 1),
                       np.concatenate([v_loc, pad], 1), pos0, rope_base, scale)
        monkeypatch.setattr(oracle, "sparse_attn", shifted)
        with pytest.raises(AssertionError):
            TestAttention().test_no_memory_is_textbook_causal_attention()
