"""GPU parity of every libmsa entry point against the float64 oracle.

Inputs come from ``latent_memory_routing_b200.synth`` (seeded); both sides
consume the same bytes (the GPU tensor, and its copy upcast to float64 for
the oracle).  No expected value comes from the CUDA path.  Tolerances:

* pooled K̄/V̄/K̄_r: normwise relative error (max |gpu-oracle| / max |oracle|
  per tensor) <= 1e-5 in fp32, <= 1e-2 in bf16;
* routing scores: <= 2e-3 absolute;
* top-k: identical to the oracle on identical scores; on routed scores,
  identical wherever the oracle's gap between consecutive ranks exceeds
  4e-3;
* attention: <= 2e-2 max-abs in bf16; <= 1e-4 in fp32 (fp32 sums over at
  most a few thousand keys plus a 2e-7 RoPE angle error stay below 1e-5;
  1e-4 leaves a 10x margin).

Full-size workloads are checked on sampled outputs that the oracle computes
one by one.
"""


import numpy as np
import pytest
import torch

import oracle
from latent_memory_routing_b200 import memory_parallel as mpar
from latent_memory_routing_b200 import msa, pipeline, synth

pytestmark = pytest.mark.gpu

RTOL_F32 = 1e-5
RTOL_BF16 = 1e-2
ROUTE_ATOL = 2e-3
GAP = 4e-3
ATTN_BF16 = 2e-2
ATTN_F32 = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from latent_memory_routing_b200 import build
    build.build()
    msa.lib()
    msa.msa_device_status(clear=True)
    yield
    torch.cuda.synchronize()


def f64(t):
    return t.detach().double().cpu().numpy()


def normwise(gpu, ref):
    ref = np.asarray(ref)
    return float(np.max(np.abs(np.asarray(gpu) - ref)) / max(np.max(np.abs(ref)), 1e-30))


def status_ok():
    torch.cuda.synchronize()
    assert msa.msa_device_status(clear=True) == 0


# ------------------------------------------------------------------ chunking

@pytest.mark.parametrize("lengths", [
    [180] * 16, [1], [64], [65], [1, 2, 3, 64, 128, 129, 8192],
    list(synth.bank_10m_lengths().numpy()), list(synth.bank_100m_lengths().numpy()),
])
def test_chunk_offsets_bit_exact(lengths):
    toff = synth.tok_offsets(torch.tensor(lengths)).cuda()
    got = pipeline.chunk_offsets(toff).cpu().numpy()
    want = oracle.chunk_offsets_from_lengths(lengths)
    np.testing.assert_array_equal(got, want)
    status_ok()


# ------------------------------------------------------------------ encoding

def _encode_case(dtype, L, lengths, H, D, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    toff_c = synth.tok_offsets(torch.tensor(lengths))
    N = int(toff_c[-1])
    k, v, r = (synth.randn((L, N, H, D), dtype, "cuda", g) for _ in range(3))
    toff = toff_c.cuda()
    coff = pipeline.chunk_offsets(toff)
    C = int(coff[-1])
    kb, vb, rb = pipeline.encode_pool(k, v, r, toff, coff, C)
    torch.cuda.synchronize()
    return k, v, r, toff_c, coff.cpu().numpy(), (kb, vb, rb)


@pytest.mark.parametrize("dtype,L,H,D,tol", [
    (torch.float32, 1, 2, 64, RTOL_F32),
    (torch.float32, 2, 8, 128, RTOL_F32),
    (torch.bfloat16, 2, 8, 128, RTOL_BF16),
    (torch.bfloat16, 1, 4, 64, RTOL_BF16),
    (torch.bfloat16, 3, 16, 128, RTOL_BF16),
])
def test_encode_ragged(dtype, L, H, D, tol):
    lengths = [1, 5, 63, 64, 65, 127, 128, 129, 180, 300, 777, 2, 4000]
    k, v, r, toff, coff, (kb, vb, rb) = _encode_case(dtype, L, lengths, H, D, 7)
    ok, ov, orr, ocoff = oracle.encode_pool(f64(k), f64(v), f64(r), toff.numpy(), 10000.0)
    np.testing.assert_array_equal(coff, ocoff)
    assert normwise(f64(kb), ok) <= tol
    assert normwise(f64(vb), ov) <= tol
    assert normwise(f64(rb), orr) <= tol
    status_ok()


@pytest.mark.parametrize("L,H,D,keep_raw", [
    (2, 8, 128, True), (1, 3, 128, False), (1, 4, 64, True), (3, 16, 128, False),
])
def test_encode_prepared_bank_equals_the_preparation_step(L, H, D, keep_raw):
    """msa_encode_pool_prepared writes K̄ and V̄ as msa_encode_pool does and
    the prepared routing bank byte for byte as msa_route_prepare_bank makes
    it from K̄_r (H = 3 leaves idle lanes in the pooling kernel's head
    groups; one document's routing keys are all zero, so its rows hit the
    1e-12 floor); the prepared rows are the oracle's pooled K_r rows over
    their norms, within the bf16 tolerance."""
    lengths = [1, 5, 63, 64, 65, 127, 128, 129, 180, 300, 777, 2, 4000]
    dtype = torch.bfloat16
    g = torch.Generator(device="cuda").manual_seed(31 + H)
    toff_c = synth.tok_offsets(torch.tensor(lengths))
    N = int(toff_c[-1])
    k, v, r = (synth.randn((L, N, H, D), dtype, "cuda", g) for _ in range(3))
    r[:, int(toff_c[4]):int(toff_c[5])] = 0.0  # document 4: zero routing keys
    toff = toff_c.cuda()
    coff = pipeline.chunk_offsets(toff)
    C = int(coff[-1])
    kb, vb, rb = pipeline.encode_pool(k, v, r, toff, coff, C)
    kb2, vb2, rh, rb2 = pipeline.encode_pool_prepared(k, v, r, toff, coff, C, keep_raw=keep_raw)
    torch.cuda.synchronize()
    assert torch.equal(kb, kb2) and torch.equal(vb, vb2)
    assert (rb2 is not None) == keep_raw
    if keep_raw:
        assert torch.equal(rb, rb2)
    for l in range(L):
        assert torch.equal(rh[l], pipeline.prepare_bank(rb[l].contiguous()))
    _, _, orr, ocoff = oracle.encode_pool(f64(k), f64(v), f64(r), toff_c.numpy(), 10000.0)
    onorm = np.linalg.norm(orr, axis=-1, keepdims=True)
    ounit = orr / np.maximum(onorm, 1e-12)
    c4 = slice(int(ocoff[4]), int(ocoff[5]))
    assert np.all(f64(rh)[:, c4] == 0.0)
    assert normwise(f64(rh), ounit) <= RTOL_BF16
    status_ok()


def test_encode_tiny_workload_fp32():
    w = synth.tiny("cuda")
    toff = w["tok_offsets"].cuda()
    coff = pipeline.chunk_offsets(toff)
    kb, vb, rb = pipeline.encode_pool(w["k_tok"], w["v_tok"], w["kr_tok"], toff, coff, 48)
    ok, ov, orr, _ = oracle.encode_pool(f64(w["k_tok"]), f64(w["v_tok"]), f64(w["kr_tok"]),
                                        w["tok_offsets"].numpy(), 10000.0)
    for got, want in ((kb, ok), (vb, ov), (rb, orr)):
        assert normwise(f64(got), want) <= RTOL_F32
    status_ok()


def test_encode_4_layers_1m_tokens_sampled():
    w = synth.encode_4l("cuda")
    toff = w["tok_offsets"].cuda()
    coff = pipeline.chunk_offsets(toff)
    C = int(coff[-1])
    kb, vb, rb = pipeline.encode_pool(w["k_tok"], w["v_tok"], w["kr_tok"], toff, coff, C)
    torch.cuda.synchronize()
    coff_h = coff.cpu().numpy()
    toff_h = w["tok_offsets"].numpy()
    n_docs = len(toff_h) - 1
    rng = np.random.default_rng(5)
    docs = sorted(set(rng.choice(n_docs, 24, replace=False).tolist()) | {0, n_docs - 1})
    for d in docs:
        t0, t1 = int(toff_h[d]), int(toff_h[d + 1])
        c0, c1 = int(coff_h[d]), int(coff_h[d + 1])
        for l in range(w["L"]):
            want = oracle.encode_pool_doc(f64(w["k_tok"][l, t0:t1]), f64(w["v_tok"][l, t0:t1]),
                                          f64(w["kr_tok"][l, t0:t1]), 10000.0)
            for got, ref in zip((kb, vb, rb), want):
                assert normwise(f64(got[l, c0:c1]), ref) <= RTOL_BF16, (d, l)
    status_ok()


# ------------------------------------------------------------------- routing

def _pooled_bank(n_docs, lo, hi, H, D, dtype, seed, needle_q=None):
    g = torch.Generator(device="cuda").manual_seed(seed)
    gc = torch.Generator().manual_seed(seed)
    lengths = torch.randint(lo, hi + 1, (n_docs,), generator=gc)
    coff_h = oracle.chunk_offsets_from_lengths(lengths.numpy())
    C = int(coff_h[-1])
    kr = synth.randn((C, H, D), dtype, "cuda", g)
    if needle_q is not None:
        synth.plant_pooled_needles(kr, coff_h, [n_docs // 3], needle_q, g)
    return kr, torch.from_numpy(coff_h).cuda(), coff_h


def _route(q_r, kr, coff, n_docs, with_chunks=True, prepared=False):
    """Routes q_r over the raw bank kr, or over its prepared (unit-row) copy
    made by msa_route_prepare_bank."""
    B, T, H, D = q_r.shape
    router = pipeline.Router(q_r.dtype, B, T, H, D, "cuda", prepared=prepared)
    bank = pipeline.prepare_bank(kr) if prepared else kr
    cs = torch.empty((B, kr.shape[0]), dtype=torch.float32, device="cuda") if with_chunks else None
    ds = router(q_r, bank, coff, n_docs, chunk_scores=cs)
    torch.cuda.synchronize()
    return ds, cs


@pytest.mark.parametrize("prepared", [False, True])
@pytest.mark.parametrize("B,T,H,D,n_docs", [
    (1, 256, 8, 128, 150),    # one pass, N = 256 (the 100M prefill shape)
    (1, 128, 8, 128, 90),     # N = 128
    (64, 1, 8, 128, 60),      # N = 64, one column per query (decode shape)
    (3, 7, 8, 128, 40),       # N = 64 with 21 live columns
    (3, 48, 8, 128, 40),      # N = 256, query 2 straddles the column halves
    (2, 150, 8, 128, 40),     # 300 columns: two passes over the bank
    (1, 64, 2, 64, 70),       # D = 64, H = 2
    (5, 3, 1, 128, 33),       # H = 1
    (100, 1, 8, 128, 50),     # N = 128, one column per query
    (12, 10, 8, 128, 45),     # N = 128, ten-token queries
])
def test_route_bf16_vs_oracle(B, T, H, D, n_docs, prepared):
    g = torch.Generator(device="cuda").manual_seed(100 + B * T)
    q_r = synth.randn((B, T, H, D), torch.bfloat16, "cuda", g)
    kr, coff, coff_h = _pooled_bank(n_docs, 1, 900, H, D, torch.bfloat16, 11 + T,
                                    needle_q=q_r[0])
    ds, cs = _route(q_r, kr, coff, n_docs, prepared=prepared)
    ods, ocs = oracle.route_scores(f64(q_r), f64(kr), coff_h)
    assert np.max(np.abs(f64(cs) - ocs)) <= ROUTE_ATOL
    assert np.max(np.abs(f64(ds) - ods)) <= ROUTE_ATOL
    status_ok()


def test_route_fp32_tiny():
    w = synth.tiny("cuda")
    ok, ov, orr, coff_h = oracle.encode_pool(f64(w["k_tok"]), f64(w["v_tok"]), f64(w["kr_tok"]),
                                             w["tok_offsets"].numpy(), 10000.0)
    kr = torch.from_numpy(orr[0]).float().cuda()  # oracle bank as the common input
    ds, cs = _route(w["q_r"], kr, torch.from_numpy(coff_h).cuda(), 16)
    ods, ocs = oracle.route_scores(f64(w["q_r"]), f64(kr), coff_h)
    assert np.max(np.abs(f64(cs) - ocs)) <= 1e-5
    assert np.max(np.abs(f64(ds) - ods)) <= 1e-5
    assert int(torch.argmax(ds[0])) == 5
    status_ok()


def test_prepared_bank_rows_are_unit_and_scores_agree():
    H, D = 8, 128
    g = torch.Generator(device="cuda").manual_seed(77)
    kr = synth.randn((3000, H, D), torch.bfloat16, "cuda", g) * 3.0
    kr[5] = 0.0
    hat = pipeline.prepare_bank(kr)
    n = hat.float().norm(dim=-1).cpu().numpy()
    assert np.all(np.abs(n[np.arange(3000) != 5] - 1.0) <= 4e-3)
    assert np.all(n[5] == 0.0)
    q = synth.randn((2, 40, H, D), torch.bfloat16, "cuda", g)
    coff_h = np.arange(0, 3001, 30)
    coff = torch.from_numpy(coff_h).cuda()
    a, _ = _route(q, kr, coff, 100)
    b, _ = _route(q, kr, coff, 100, prepared=True)
    assert np.max(np.abs(f64(a) - f64(b))) <= 1e-4
    status_ok()


def test_route_zero_key_scores_zero():
    H, D = 8, 128
    kr = torch.zeros((130, H, D), dtype=torch.bfloat16, device="cuda")
    kr[:65] = 1.0
    coff_h = np.array([0, 65, 130])
    q = torch.ones((1, 4, H, D), dtype=torch.bfloat16, device="cuda")
    ds, cs = _route(q, kr, torch.from_numpy(coff_h).cuda(), 2)
    assert abs(float(ds[0, 0]) - 1.0) <= ROUTE_ATOL
    assert float(ds[0, 1]) == 0.0
    status_ok()


def _check_topk_on_routed(idx, oracle_scores, k):
    """Indices must match the oracle wherever the oracle ranking is
    unambiguous by more than GAP."""
    idx = np.asarray(idx)
    for b in range(oracle_scores.shape[0]):
        s = oracle_scores[b]
        order = np.lexsort((np.arange(s.shape[0]), -s))
        srt = s[order]
        if srt[k - 1] - srt[k] > GAP:
            assert set(idx[b].tolist()) == set(order[:k].tolist()), b
        for r in range(k):
            left = srt[r - 1] - srt[r] if r > 0 else np.inf
            right = srt[r] - srt[r + 1]
            if left > GAP and right > GAP:
                assert idx[b, r] == order[r], (b, r)


@pytest.mark.parametrize("prepared", [False, True])
def test_route_topk_10m_decode_full(prepared):
    lengths = synth.bank_10m_lengths()
    coff_h = oracle.chunk_offsets_from_lengths(lengths.numpy())
    w = synth.bank_10m(coff_h, "cuda")
    coff = torch.from_numpy(coff_h).cuda()
    ds, _ = _route(w["q_r"], w["kr_bar"], coff, len(lengths), with_chunks=False,
                   prepared=prepared)
    ods, _ = oracle.route_scores(f64(w["q_r"]), f64(w["kr_bar"]), coff_h)
    assert np.max(np.abs(f64(ds) - ods)) <= ROUTE_ATOL
    idx, _ = pipeline.topk_docs(ds, 16)
    _check_topk_on_routed(idx.cpu().numpy(), ods, 16)
    status_ok()


@pytest.mark.parametrize("prepared", [False, True])
def test_route_100m_prefill_sampled(prepared):
    lengths = synth.bank_100m_lengths()
    coff_h = oracle.chunk_offsets_from_lengths(lengths.numpy())
    w = synth.bank_100m(coff_h, "cuda")
    coff = torch.from_numpy(coff_h).cuda()
    n_docs = len(lengths)
    ds, cs = _route(w["q_r"], w["kr_bar"], coff, n_docs, prepared=prepared)
    idx, _ = pipeline.topk_docs(ds, 16)
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    C = int(coff_h[-1])
    q = f64(w["q_r"])
    chunks = np.unique(np.concatenate([rng.choice(C, 6000, replace=False),
                                       np.arange(C - 300, C), np.arange(0, 300)]))
    ocs = oracle.route_chunk_scores(q, f64(w["kr_bar"][torch.from_numpy(chunks).cuda()]))
    assert np.max(np.abs(f64(cs)[0, chunks] - ocs[0])) <= ROUTE_ATOL
    docs = np.unique(np.concatenate([rng.choice(n_docs, 300, replace=False), w["needles"],
                                     idx[0].cpu().numpy()]))
    for d in docs:
        rows = torch.arange(int(coff_h[d]), int(coff_h[d + 1]), device="cuda")
        od = oracle.route_chunk_scores(q, f64(w["kr_bar"][rows])).max()
        assert abs(float(ds[0, d]) - od) <= ROUTE_ATOL, d
    # top-k is exact on the GPU's own scores: every unselected score is below
    # the k-th (or equal with a higher index), selection is in rank order
    s = ds[0].cpu().numpy()
    sel = idx[0].cpu().numpy()
    kth = s[sel[-1]]
    assert np.all(np.diff(s[sel]) <= 0)
    rest = np.setdiff1d(np.arange(n_docs), sel)
    assert np.all((s[rest] < kth) | ((s[rest] == kth) & (rest > sel[-1])))
    status_ok()


# --------------------------------------------------------------------- top-k

@pytest.mark.parametrize("B,n,k,quant", [
    (1, 16, 2, None), (4, 1000, 16, None), (64, 10000, 16, None), (1, 100000, 16, None),
    (3, 5000, 1024, None), (2, 300, 300, None), (2, 5000, 16, 8.0), (1, 4096, 64, 1.0),
    (2, 16384, 16, None), (2, 16385, 16, 64.0),          # one segment / two segments
    (1, 200000, 1024, None),                              # 8 segments of 25K keys (L2 keys)
    (3, 70000, 100, 16.0), (1, 1000000, 16, None),        # many ties; 1M documents
    (2, 2048, 32, None), (2, 2049, 32, 4.0),              # small-k path: one / two segments
    (1, 50000, 1, None), (1, 70000, 33, None),            # k = 1; just above the small path
])
def test_topk_identical_to_oracle(B, n, k, quant):
    g = torch.Generator(device="cuda").manual_seed(n + k)
    s = torch.randn((B, n), device="cuda", generator=g)
    if quant is not None:  # many exact ties
        s = torch.round(s * quant) / quant
    idx, top = torch.empty((B, k), dtype=torch.int32, device="cuda"), \
        torch.empty((B, k), device="cuda")
    pipeline.topk_docs(s, k, idx, top)
    oi, ot = oracle.topk_docs(f64(s), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), oi)
    np.testing.assert_array_equal(f64(top), ot)
    status_ok()


@pytest.mark.parametrize("k", [16, 32, 200])
def test_topk_sorted_inputs(k):
    """Ascending scores (every batch of the small-k path improves its list)
    and descending ones, with runs of exact ties."""
    n = 40000
    base = torch.arange(n, device="cuda", dtype=torch.float32) // 3
    for s in (base[None, :], base.flip(0)[None, :], -base[None, :]):
        s = s.contiguous()
        top = torch.empty((1, k), device="cuda")
        idx, _ = pipeline.topk_docs(s, k, top=top)
        oi, ot = oracle.topk_docs(f64(s), k)
        np.testing.assert_array_equal(idx.cpu().numpy(), oi)
        np.testing.assert_array_equal(f64(top), ot)
    status_ok()


def test_topk_special_values():
    s = torch.tensor([[0.5, float("nan"), -float("inf"), 0.5, float("inf"), -0.0, 0.0]],
                     device="cuda")
    idx, _ = pipeline.topk_docs(s, 7)
    # +inf, the two 0.5 by index, -0.0 and 0.0 as equal scores by index,
    # -inf, NaN last
    assert idx[0].tolist() == [4, 0, 3, 5, 6, 2, 1]
    oi, _ = oracle.topk_docs(f64(s), 7)
    assert oi[0].tolist() == idx[0].tolist()
    status_ok()


# ----------------------------------------------------- Memory Parallel merge

def test_merge_shards_vs_oracle_special_values():
    """msa_topk_merge_shards over hand-made candidates: ties across shards go
    to the lower global id, -0 == +0, NaN last; compared with the oracle's
    top-k over the dense score vector the candidates describe."""
    world, B, k = 3, 2, 5
    base = [0, 100, 200]
    rng = np.random.default_rng(5)
    cs = np.zeros((world, B, k), np.float32)
    ci = np.zeros((world, B, k), np.int32)
    for r in range(world):
        for b in range(B):
            ci[r, b] = rng.choice(100, k, replace=False)
            cs[r, b] = np.round(rng.standard_normal(k), 1)  # coarse: many ties
    cs[1, 0, 0], cs[2, 0, 1] = 0.0, -0.0
    cs[0, 1, 2] = np.nan
    dense = np.full((B, 300), np.nan)
    for r in range(world):
        for b in range(B):
            dense[b, ci[r, b] + base[r]] = cs[r, b]
    want, wscore = oracle.topk_docs(dense, k)
    idx, top = mpar.merge_shards(torch.from_numpy(cs).cuda(), torch.from_numpy(ci).cuda(),
                                 torch.tensor(base, dtype=torch.int32, device="cuda"), k,
                                 top=torch.empty((B, k), device="cuda"))
    torch.cuda.synchronize()
    assert idx.cpu().tolist() == want.tolist()
    np.testing.assert_array_equal(top.cpu().numpy(), wscore.astype(np.float32))
    status_ok()


@pytest.mark.parametrize("world", [2, 3])
def test_memory_parallel_emulated_matches_single_gpu(world):
    """Memory Parallel with its shards emulated in one process: each shard's
    prepared routing + local top-k, the stacked candidates merged by
    msa_topk_merge_shards, equal bit for bit to the unsharded route + top-k
    (each chunk's score does not depend on the shard it sits in).  Two
    identical best documents in the first and last shard: the lower id wins."""
    H, D, B, T, k = 8, 128, 3, 32, 16
    kr, coff, coff_h = _pooled_bank(1500, 1, 900, H, D, torch.bfloat16, 41)
    g = torch.Generator(device="cuda").manual_seed(42)
    q_r = synth.randn((B, T, H, D), torch.bfloat16, "cuda", g)
    plan = mpar.shard_plan(coff_h, world, k)
    counts = np.diff(coff_h)
    da = plan[0][0] + 5
    db = next(d for d in range(plan[-1][0], plan[-1][1]) if counts[d] == counts[da])
    kr[coff_h[da]:coff_h[da + 1]] = q_r[0, 0]  # cosine 1 with query 0's first token
    kr[coff_h[db]:coff_h[db + 1]] = kr[coff_h[da]:coff_h[da + 1]]
    hat = pipeline.prepare_bank(kr)
    n_docs = len(counts)
    router = pipeline.Router(torch.bfloat16, B, T, H, D, "cuda", prepared=True)
    ds = torch.empty((B, n_docs), dtype=torch.float32, device="cuda")
    router(q_r, hat, coff, n_docs, ds)
    gi, gt = pipeline.topk_docs(ds, k, top=torch.empty((B, k), device="cuda"))
    cs = torch.empty((world, B, k), dtype=torch.float32, device="cuda")
    ci = torch.empty((world, B, k), dtype=torch.int32, device="cuda")
    for r, (d0, d1, c0, c1) in enumerate(plan):
        lc = torch.from_numpy(mpar.local_offsets(coff_h, plan, r)).cuda()
        dsr = torch.empty((B, d1 - d0), dtype=torch.float32, device="cuda")
        router(q_r, hat[c0:c1], lc, d1 - d0, dsr)
        pipeline.topk_docs(dsr, k, ci[r], cs[r])
    base = torch.tensor([p[0] for p in plan], dtype=torch.int32, device="cuda")
    idx, top = mpar.merge_shards(cs, ci, base, k, top=torch.empty((B, k), device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(idx, gi) and torch.equal(top, gt)
    assert idx[0, :2].tolist() == [da, db]
    status_ok()


# -------------------------------------------------------------------- gather

def test_gather_bit_exact_and_capacity():
    H, D = 8, 128
    kr, coff, coff_h = _pooled_bank(50, 1, 700, H, D, torch.bfloat16, 21)
    g = torch.Generator(device="cuda").manual_seed(22)
    kb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    vb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    idx = torch.tensor([[7, 3, 49, 0], [12, 12, 5, 30]], dtype=torch.int32, device="cuda")
    counts = np.diff(coff_h)
    need = [int(counts[r].sum()) for r in idx.cpu().numpy()]
    m_cap = max(need) + 3
    km, vm, ml = pipeline.gather_kv(idx, coff, kb, vb, m_cap)
    okm, ovm, oml = oracle.gather_kv(idx.cpu().numpy(), coff_h, f64(kb), f64(vb))
    assert ml.cpu().tolist() == oml.tolist()
    for b in range(2):
        np.testing.assert_array_equal(f64(km[b, :oml[b]]), okm[b])
        np.testing.assert_array_equal(f64(vm[b, :oml[b]]), ovm[b])
    status_ok()
    # capacity overflow: rows past m_cap dropped, status word set
    small = min(need) - 1
    km2, vm2, ml2 = pipeline.gather_kv(idx, coff, kb, vb, small)
    torch.cuda.synchronize()
    assert ml2.cpu().tolist() == [small, small]
    np.testing.assert_array_equal(f64(km2[0]), okm[0][:small])
    assert msa.msa_device_status(clear=True) == -3


def test_gather_tiered_host_bank():
    """Tiered storage: K̄/V̄ in pinned host memory, read by the same gather
    kernel over the host link; bit-identical to the device-resident gather."""
    H, D = 8, 128
    kr, coff, coff_h = _pooled_bank(300, 1, 700, H, D, torch.bfloat16, 23)
    g = torch.Generator(device="cuda").manual_seed(24)
    kb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    vb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    kh, vh = pipeline.to_host_tier(kb), pipeline.to_host_tier(vb)
    assert kh.is_pinned() and not kh.is_cuda
    idx = torch.stack([torch.randperm(300, generator=torch.Generator().manual_seed(s))[:16]
                       for s in range(3)]).int().cuda()
    counts = np.diff(coff_h)
    m_cap = max(int(counts[r].sum()) for r in idx.cpu().numpy())
    km, vm, ml = pipeline.gather_kv(idx, coff, kh, vh, m_cap)
    kd, vd, mld = pipeline.gather_kv(idx, coff, kb, vb, m_cap)
    torch.cuda.synchronize()
    assert km.is_cuda and ml.tolist() == mld.tolist()
    okm, ovm, oml = oracle.gather_kv(idx.cpu().numpy(), coff_h, f64(kb), f64(vb))
    for b in range(3):
        n = int(oml[b])
        assert torch.equal(km[b, :n], kd[b, :n]) and torch.equal(vm[b, :n], vd[b, :n])
        np.testing.assert_array_equal(f64(km[b, :n]), okm[b])
        np.testing.assert_array_equal(f64(vm[b, :n]), ovm[b])
    status_ok()


def test_gather_fp32_tiny():
    w = synth.tiny("cuda")
    ok, ov, orr, coff_h = oracle.encode_pool(f64(w["k_tok"]), f64(w["v_tok"]), f64(w["kr_tok"]),
                                             w["tok_offsets"].numpy(), 10000.0)
    kb = torch.from_numpy(ok[0]).float().cuda()
    vb = torch.from_numpy(ov[0]).float().cuda()
    idx = torch.tensor([[5, 0]], dtype=torch.int32, device="cuda")
    km, vm, ml = pipeline.gather_kv(idx, torch.from_numpy(coff_h).cuda(), kb, vb, 6)
    okm, ovm, oml = oracle.gather_kv([[5, 0]], coff_h, f64(kb), f64(vb))
    assert int(ml[0]) == 6
    np.testing.assert_array_equal(f64(km[0]), okm[0])
    np.testing.assert_array_equal(f64(vm[0]), ovm[0])
    status_ok()


# ----------------------------------------------------------------- attention

def _attn_case(dtype, B, T, T_loc, Hq, H, D, m_cap, mem_lens, pos0, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = synth.randn((B, T, Hq, D), dtype, "cuda", g)
    km = synth.randn((B, max(m_cap, 1), H, D), dtype, "cuda", g)
    vm = synth.randn((B, max(m_cap, 1), H, D), dtype, "cuda", g)
    kl = synth.randn((B, T_loc, H, D), dtype, "cuda", g)
    vl = synth.randn((B, T_loc, H, D), dtype, "cuda", g)
    ml = torch.tensor(mem_lens, dtype=torch.int32, device="cuda")
    att = pipeline.Attention(dtype, B, T, T_loc, Hq, H, D, m_cap, "cuda")
    out = att(q, km, vm, ml, kl, vl, pos0)
    torch.cuda.synchronize()
    okm = [f64(km[b, :mem_lens[b]]) for b in range(B)]
    ovm = [f64(vm[b, :mem_lens[b]]) for b in range(B)]
    want = oracle.sparse_attn(f64(q), okm, ovm, f64(kl), f64(vl), pos0, 10000.0)
    return f64(out), want


@pytest.mark.parametrize("dtype,B,T,T_loc,Hq,H,D,m_cap,mem_lens,pos0,tol", [
    (torch.float32, 1, 16, 16, 4, 2, 64, 6, [6], 2, ATTN_F32),          # tiny workload shape
    (torch.float32, 2, 5, 9, 8, 2, 128, 40, [33, 0], 16, ATTN_F32),     # chunked prefill, empty mem
    (torch.float32, 3, 1, 300, 32, 8, 128, 100, [100, 7, 64], 16, ATTN_F32),  # decode
    (torch.bfloat16, 1, 128, 128, 32, 8, 128, 300, [257], 16, ATTN_BF16),
    (torch.bfloat16, 1, 256, 256, 32, 8, 128, 384, [371], 16, ATTN_BF16),
    (torch.bfloat16, 2, 40, 100, 16, 2, 64, 50, [50, 0], 3, ATTN_BF16),
    (torch.bfloat16, 8, 1, 2048, 32, 8, 128, 2048, [250, 0, 2048, 1, 100, 300, 17, 64], 16,
     ATTN_BF16),
    (torch.bfloat16, 2, 3, 7, 8, 8, 128, 5, [5, 2], 0, ATTN_BF16),      # G = 1
])
def test_attention_vs_oracle(dtype, B, T, T_loc, Hq, H, D, m_cap, mem_lens, pos0, tol):
    got, want = _attn_case(dtype, B, T, T_loc, Hq, H, D, m_cap, mem_lens, pos0, 31 + T)
    assert np.max(np.abs(got - want)) <= tol
    status_ok()


@pytest.mark.parametrize("B,T,T_loc,Hq,H,D,m_cap,mem_lens", [
    (2, 300, 700, 32, 8, 128, 500, [500, 129]),   # several key tiles each side
    (3, 64, 64, 8, 8, 64, 130, [128, 0, 1]),       # G = 1, empty and 1-row memory
    (1, 17, 1000, 16, 1, 128, 256, [256]),         # G = 16, chunked prefill
    (1, 64, 4096, 32, 8, 128, 384, [300]),         # long local context: key-tile splits
])
def test_attention_prefill_tensor_core_shapes(B, T, T_loc, Hq, H, D, m_cap, mem_lens):
    """Rows past mem_len are filled with NaN: they must not reach the
    output (the kernel loads whole 128-key tiles)."""
    g = torch.Generator(device="cuda").manual_seed(T + T_loc)
    dt = torch.bfloat16
    q = synth.randn((B, T, Hq, D), dt, "cuda", g)
    km = synth.randn((B, m_cap, H, D), dt, "cuda", g)
    vm = synth.randn((B, m_cap, H, D), dt, "cuda", g)
    for b, n in enumerate(mem_lens):
        km[b, n:] = float("nan")
        vm[b, n:] = float("nan")
    kl = synth.randn((B, T_loc, H, D), dt, "cuda", g)
    vl = synth.randn((B, T_loc, H, D), dt, "cuda", g)
    ml = torch.tensor(mem_lens, dtype=torch.int32, device="cuda")
    att = pipeline.Attention(dt, B, T, T_loc, Hq, H, D, m_cap, "cuda")
    out = att(q, km, vm, ml, kl, vl, 16)
    torch.cuda.synchronize()
    want = oracle.sparse_attn(f64(q), [f64(km[b, :n]) for b, n in enumerate(mem_lens)],
                              [f64(vm[b, :n]) for b, n in enumerate(mem_lens)],
                              f64(kl), f64(vl), 16, 10000.0)
    got = f64(out)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - want)) <= ATTN_BF16
    status_ok()


@pytest.mark.parametrize("B,T,Hq,H,m_cap,mem_lens", [
    (16, 512, 32, 8, 384, [384] * 8 + [0, 1, 127, 128, 129, 255, 256, 383]),  # ~7 items per CTA
    (2, 64, 32, 8, 3072, [3072, 0]),  # 3 key splits; batch 1's splits past its one tile are empty
])
def test_attention_prefill_persistent_items_repeat_bit_exactly(B, T, Hq, H, m_cap, mem_lens):
    """The prefill's persistent CTAs claim their items at run time from a
    counter that the RoPE preparation zeroes: on one workspace, two more
    eager calls and three replays of a CUDA graph of the call reproduce the
    first call bit for bit (each item is computed whole by one CTA, in a
    fixed order, whatever CTA claims it), and the first call matches the
    oracle on sampled rows of the first and last batch element."""
    D, pos0 = 128, 16
    g = torch.Generator(device="cuda").manual_seed(B * T + m_cap)
    dt = torch.bfloat16
    q = synth.randn((B, T, Hq, D), dt, "cuda", g)
    km = synth.randn((B, m_cap, H, D), dt, "cuda", g)
    vm = synth.randn((B, m_cap, H, D), dt, "cuda", g)
    for b, n in enumerate(mem_lens):
        km[b, n:] = float("nan")
        vm[b, n:] = float("nan")
    kl = synth.randn((B, T, H, D), dt, "cuda", g)
    vl = synth.randn((B, T, H, D), dt, "cuda", g)
    ml = torch.tensor(mem_lens, dtype=torch.int32, device="cuda")
    att = pipeline.Attention(dt, B, T, T, Hq, H, D, m_cap, "cuda")
    first = att(q, km, vm, ml, kl, vl, pos0).clone()
    out = torch.empty_like(first)
    for _ in range(2):
        att(q, km, vm, ml, kl, vl, pos0, out=out)
        torch.cuda.synchronize()
        assert torch.equal(out, first)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on the capture stream
        att(q, km, vm, ml, kl, vl, pos0, out=out)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        att(q, km, vm, ml, kl, vl, pos0, out=out)
    for _ in range(3):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, first)
    del graph
    worst = 0.0
    for b in sorted({0, B - 1}):
        n = mem_lens[b]
        for i0 in sorted({0, T // 2 - 4, T - 8}):
            i1 = i0 + 8
            want = oracle.sparse_attn(f64(q[b:b + 1, i0:i1]), [f64(km[b, :n])], [f64(vm[b, :n])],
                                      f64(kl[b:b + 1, :i1]), f64(vl[b:b + 1, :i1]), pos0,
                                      10000.0)
            got = f64(first[b:b + 1, i0:i1])
            assert np.all(np.isfinite(got))
            worst = max(worst, float(np.max(np.abs(got - want))))
    assert worst <= ATTN_BF16, worst
    status_ok()


def _prefill_sweep_points():
    import bench
    return list(bench.PREFILL_SWEEP)


@pytest.mark.parametrize("B,T,M", _prefill_sweep_points())
def test_attention_prefill_sweep_point_sampled(B, T, M):
    """Each point of the benchmark's prefill sweep (T = T_loc up to 32K, B up
    to 16), run at its own size with the inputs the sweep draws, checked on
    sampled blocks of query rows: rows i0 .. i0+7 of a prefill of T tokens
    are the last 8 rows of a prefill of i0+8 tokens over the same keys, so
    the oracle computes them from that prefix (first rows, rows across the
    first key-tile boundary, the middle and the last rows)."""
    Hq, H, D, pos0 = 32, 8, 128, 16
    g = torch.Generator(device="cuda").manual_seed(B * T)
    dt = torch.bfloat16
    q = synth.randn((B, T, Hq, D), dt, "cuda", g)
    km = synth.randn((B, M, H, D), dt, "cuda", g)
    vm = synth.randn((B, M, H, D), dt, "cuda", g)
    kl = synth.randn((B, T, H, D), dt, "cuda", g)
    vl = synth.randn((B, T, H, D), dt, "cuda", g)
    ml = torch.full((B,), M, dtype=torch.int32, device="cuda")
    att = pipeline.Attention(dt, B, T, T, Hq, H, D, M, "cuda")
    out = att(q, km, vm, ml, kl, vl, pos0)
    torch.cuda.synchronize()
    worst = 0.0
    for b in sorted({0, B - 1}):
        for i0 in (0, 124, T // 2 - 4, T - 8):
            i1 = i0 + 8
            want = oracle.sparse_attn(f64(q[b:b + 1, i0:i1]), [f64(km[b])], [f64(vm[b])],
                                      f64(kl[b:b + 1, :i1]), f64(vl[b:b + 1, :i1]), pos0,
                                      10000.0)
            got = f64(out[b:b + 1, i0:i1])
            assert np.all(np.isfinite(got))
            worst = max(worst, float(np.max(np.abs(got - want))))
    assert worst <= ATTN_BF16, worst
    status_ok()


@pytest.mark.parametrize("B,T_loc,Hq,H,m_cap,mem_lens", [
    (3, 1, 32, 8, 70, [70, 0, 65]),         # one local token, ragged memory tile
    (2, 65, 8, 8, 64, [64, 1]),             # G = 1, local tail of one key
    (2, 200, 16, 8, 130, [129, 3]),         # G = 2
    (2, 129, 64, 8, 200, [200, 77]),        # G = 8
    (1, 100, 16, 1, 500, [500]),            # G = 16, one KV head
    (2, 90, 32, 8, 64, [0, 0]),             # no memory rows at all
    (4, 4096, 32, 8, 1024, [1000, 0, 1024, 513]),  # long context, several splits
    (48, 130, 16, 8, 300, [0, 1, 127, 128, 129, 255, 256, 300] * 6),  # many items per CTA
])
def test_attention_decode_shapes(B, T_loc, Hq, H, m_cap, mem_lens):
    """bf16 decode over 64-key tiles: rows past mem_len hold NaN and must not
    reach the output; the relative-RoPE local tiles must match absolute
    positions."""
    D = 128
    g = torch.Generator(device="cuda").manual_seed(T_loc + m_cap)
    dt = torch.bfloat16
    q = synth.randn((B, 1, Hq, D), dt, "cuda", g)
    km = synth.randn((B, m_cap, H, D), dt, "cuda", g)
    vm = synth.randn((B, m_cap, H, D), dt, "cuda", g)
    for b, n in enumerate(mem_lens):
        km[b, n:] = float("nan")
        vm[b, n:] = float("nan")
    kl = synth.randn((B, T_loc, H, D), dt, "cuda", g)
    vl = synth.randn((B, T_loc, H, D), dt, "cuda", g)
    ml = torch.tensor(mem_lens, dtype=torch.int32, device="cuda")
    att = pipeline.Attention(dt, B, 1, T_loc, Hq, H, D, m_cap, "cuda")
    out = att(q, km, vm, ml, kl, vl, 16)
    torch.cuda.synchronize()
    want = oracle.sparse_attn(f64(q), [f64(km[b, :n]) for b, n in enumerate(mem_lens)],
                              [f64(vm[b, :n]) for b, n in enumerate(mem_lens)],
                              f64(kl), f64(vl), 16, 10000.0)
    got = f64(out)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - want)) <= ATTN_BF16
    status_ok()


@pytest.mark.parametrize("B,T,T_loc,Hq,H,k,n_docs", [
    (5, 1, 300, 32, 8, 6, 40),      # decode, GQA 4:1, ragged documents
    (3, 1, 65, 16, 1, 9, 30),       # decode, G = 16, one KV head
    (4, 1, 200, 8, 8, 3, 12),       # decode, G = 1
    (2, 64, 64, 32, 8, 6, 40),      # prefill
    (1, 256, 256, 32, 8, 16, 60),   # prefill at the 100M-bank step's shape
    (2, 300, 700, 16, 8, 7, 25),    # chunked prefill, several key tiles, G = 2
])
def test_attention_fused_vs_oracle(B, T, T_loc, Hq, H, k, n_docs):
    """Fused assembly + attention: rows read from the bank in 8-row groups
    (documents of 1..40 rows, most not a multiple of 8, one document shared
    by two queries) against the oracle's gather + attention."""
    D = 128
    g = torch.Generator(device="cuda").manual_seed(T_loc + n_docs)
    gc = torch.Generator().manual_seed(T_loc)
    counts = torch.randint(1, 41, (n_docs,), generator=gc).numpy()
    counts[0] = 1
    coff_h = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    C = int(coff_h[-1])
    kb = synth.randn((C, H, D), torch.bfloat16, "cuda", g)
    vb = synth.randn((C, H, D), torch.bfloat16, "cuda", g)
    idx_h = np.stack([np.random.default_rng(b).choice(n_docs, k, replace=False) for b in range(B)])
    if B > 1:
        idx_h[1, 0] = idx_h[0, 0]
    if 0 not in idx_h[0]:
        idx_h[0, -1] = 0  # the one-row document
    idx = torch.from_numpy(idx_h).int().cuda()
    q = synth.randn((B, T, Hq, D), torch.bfloat16, "cuda", g)
    kl = synth.randn((B, T_loc, H, D), torch.bfloat16, "cuda", g)
    vl = synth.randn((B, T_loc, H, D), torch.bfloat16, "cuda", g)
    m_cap = int(max(counts[r].sum() for r in idx_h))
    att = pipeline.FusedAttention(torch.bfloat16, B, T, T_loc, Hq, H, D, k, m_cap, "cuda")
    out = att(q, idx, torch.from_numpy(coff_h).cuda(), kb, vb, kl, vl, k)
    torch.cuda.synchronize()
    okm, ovm, oml = oracle.gather_kv(idx_h, coff_h, f64(kb), f64(vb))
    assert att.mem_len.cpu().tolist() == list(oml)
    want = oracle.sparse_attn(f64(q), okm, ovm, f64(kl), f64(vl), k, 10000.0)
    got = f64(out)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - want)) <= ATTN_BF16
    status_ok()


@pytest.mark.parametrize("B,T,T_loc,Hq,H,k", [
    (3, 1, 200, 32, 8, 6),       # decode
    (2, 64, 64, 32, 8, 6),       # prefill
    (1, 256, 256, 32, 8, 16),    # prefill at the 100M-bank step's shape
])
def test_attention_fused_ignores_non_finite_rows_past_a_document(B, T, T_loc, Hq, H, k):
    """The rows of a selected document's last 8-row group past its end belong
    to the next document.  Here every odd document is NaN in K and in V and
    only even documents are selected, so each selected document is followed
    by NaN rows that its last group reads: they must be masked and their V
    zeroed, giving a finite output equal to the oracle's over the selected
    rows alone."""
    D, n_docs = 128, 48
    g = torch.Generator(device="cuda").manual_seed(400 + T)
    gc = torch.Generator().manual_seed(401 + T)
    counts = torch.randint(1, 30, (n_docs,), generator=gc).numpy()
    counts[1::2] = np.maximum(counts[1::2], 8)  # a whole group of NaN after each
    counts[0] = 1
    coff_h = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    C = int(coff_h[-1])
    kb = synth.randn((C, H, D), torch.bfloat16, "cuda", g)
    vb = synth.randn((C, H, D), torch.bfloat16, "cuda", g)
    for d in range(1, n_docs, 2):
        kb[coff_h[d]:coff_h[d + 1]] = float("nan")
        vb[coff_h[d]:coff_h[d + 1]] = float("inf") if d % 4 == 1 else float("nan")
    idx_h = np.stack([2 * np.random.default_rng(50 + b).choice(n_docs // 2, k, replace=False)
                      for b in range(B)])
    idx_h[0, -1] = 0  # the one-row document: seven NaN rows in its group
    idx = torch.from_numpy(idx_h).int().cuda()
    q = synth.randn((B, T, Hq, D), torch.bfloat16, "cuda", g)
    kl = synth.randn((B, T_loc, H, D), torch.bfloat16, "cuda", g)
    vl = synth.randn((B, T_loc, H, D), torch.bfloat16, "cuda", g)
    m_cap = int(max(counts[r].sum() for r in idx_h))
    att = pipeline.FusedAttention(torch.bfloat16, B, T, T_loc, Hq, H, D, k, m_cap, "cuda")
    out = att(q, idx, torch.from_numpy(coff_h).cuda(), kb, vb, kl, vl, k)
    torch.cuda.synchronize()
    okm, ovm, oml = oracle.gather_kv(idx_h, coff_h, f64(kb), f64(vb))
    assert all(np.all(np.isfinite(x)) for x in okm + ovm)
    assert att.mem_len.cpu().tolist() == list(oml)
    want = oracle.sparse_attn(f64(q), okm, ovm, f64(kl), f64(vl), k, 10000.0)
    got = f64(out)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - want)) <= ATTN_BF16
    status_ok()


def test_attention_fused_capacity_and_bad_index():
    """Fewer groups than the documents need: rows past the capacity are
    dropped (mem_len says how many were used) and MSA_ERR_CAPACITY is
    recorded."""
    D, H, Hq, T_loc, k = 128, 8, 32, 64, 4
    counts = np.array([30, 30, 30, 30, 30])
    coff_h = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    g = torch.Generator(device="cuda").manual_seed(3)
    kb = synth.randn((int(coff_h[-1]), H, D), torch.bfloat16, "cuda", g)
    vb = synth.randn((int(coff_h[-1]), H, D), torch.bfloat16, "cuda", g)
    idx = torch.tensor([[0, 1, 2, 3]], dtype=torch.int32, device="cuda")
    q = synth.randn((1, 1, Hq, D), torch.bfloat16, "cuda", g)
    kl = synth.randn((1, T_loc, H, D), torch.bfloat16, "cuda", g)
    att = pipeline.FusedAttention(torch.bfloat16, 1, 1, T_loc, Hq, H, D, k, 40, "cuda")
    out = att(q, idx, torch.from_numpy(coff_h).cuda(), kb, vb, kl, kl, k)
    torch.cuda.synchronize()
    # max_groups = ceil(40/8) + 4 = 9 groups; each document takes 4
    assert int(att.mem_len[0]) == 30 + 30 + 8
    assert np.all(np.isfinite(f64(out)))
    assert msa.msa_device_status(clear=True) == -3


def test_attention_decode_10m_workload_full():
    lengths = synth.bank_10m_lengths()
    coff_h = oracle.chunk_offsets_from_lengths(lengths.numpy())
    w = synth.bank_10m(coff_h, "cuda")
    B = w["B"]
    rng = np.random.default_rng(9)
    # 16 documents per query, as the router would select
    idx = np.stack([rng.choice(len(lengths), 16, replace=False) for _ in range(B)])
    counts = np.diff(coff_h)
    m_cap = int(max(counts[r].sum() for r in idx))
    km, vm, ml = pipeline.gather_kv(torch.from_numpy(idx).int().cuda(),
                                    torch.from_numpy(coff_h).cuda(), w["k_bar"], w["v_bar"], m_cap)
    att = pipeline.Attention(torch.bfloat16, B, 1, 2048, 32, 8, 128, m_cap, "cuda")
    out = att(w["q"], km, vm, ml, w["k_loc"], w["v_loc"], 16)
    fatt = pipeline.FusedAttention(torch.bfloat16, B, 1, 2048, 32, 8, 128, 16, m_cap, "cuda")
    fout = fatt(w["q"], torch.from_numpy(idx).int().cuda(), torch.from_numpy(coff_h).cuda(),
                w["k_bar"], w["v_bar"], w["k_loc"], w["v_loc"], 16)
    torch.cuda.synchronize()
    okm, ovm, oml = oracle.gather_kv(idx, coff_h, f64(w["k_bar"]), f64(w["v_bar"]))
    want = oracle.sparse_attn(f64(w["q"]), okm, ovm, f64(w["k_loc"]), f64(w["v_loc"]), 16)
    assert np.max(np.abs(f64(out) - want)) <= ATTN_BF16
    assert np.max(np.abs(f64(fout) - want)) <= ATTN_BF16  # the same, read from the bank
    assert fatt.mem_len.cpu().tolist() == list(oml)
    status_ok()


# ------------------------------------------------------------ whole pipeline

def test_tiny_pipeline_end_to_end_fp32():
    w = synth.tiny("cuda")
    toff = w["tok_offsets"].cuda()
    coff = pipeline.chunk_offsets(toff)
    kb, vb, rb = pipeline.encode_pool(w["k_tok"], w["v_tok"], w["kr_tok"], toff, coff, 48)
    p = pipeline.Pipeline(rb[0], kb[0], vb[0], coff, B=1, T=16, T_loc=16, Hq=4, k=2, m_cap=6)
    out = p(w["q_r"], w["q"], w["k_loc"], w["v_loc"])
    torch.cuda.synchronize()
    ref = oracle.msa_forward(f64(w["k_tok"]), f64(w["v_tok"]), f64(w["kr_tok"]),
                             w["tok_offsets"].numpy(), f64(w["q_r"]), f64(w["q"]),
                             f64(w["k_loc"]), f64(w["v_loc"]), k=2)
    assert p.idx[0].tolist() == ref["topk_idx"][0].tolist() == [5, p.idx[0, 1].item()]
    assert int(p.mem_len[0]) == 6
    assert np.max(np.abs(f64(p.doc_scores) - ref["doc_scores"])) <= 1e-5
    assert np.max(np.abs(f64(out) - ref["out"])) <= ATTN_F32
    status_ok()


def test_pipeline_tiered_matches_resident():
    """Routing keys in HBM, content K̄/V̄ in pinned host memory: the whole
    step (route, top-k, gather over the host link, prefill attention) gives
    the same bytes as the all-HBM pipeline, and matches the oracle."""
    H, D, Hq, T, k = 8, 128, 32, 64, 8
    kr, coff, coff_h = _pooled_bank(400, 1, 600, H, D, torch.bfloat16, 25)
    g = torch.Generator(device="cuda").manual_seed(26)
    kb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    vb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    q_r = synth.randn((1, T, H, D), torch.bfloat16, "cuda", g)
    q = synth.randn((1, T, Hq, D), torch.bfloat16, "cuda", g)
    kl = synth.randn((1, T, H, D), torch.bfloat16, "cuda", g)
    vl = synth.randn((1, T, H, D), torch.bfloat16, "cuda", g)
    m_cap = k * int(np.diff(coff_h).max())
    outs = []
    for kk, vv in ((kb, vb), (pipeline.to_host_tier(kb), pipeline.to_host_tier(vb))):
        p = pipeline.Pipeline(kr, kk, vv, coff, B=1, T=T, T_loc=T, Hq=Hq, k=k, m_cap=m_cap,
                              pos0=k)
        outs.append((p(q_r, q, kl, vl).clone(), p.idx.clone(), p.mem_len.clone()))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][1], outs[1][1]) and torch.equal(outs[0][2], outs[1][2])
    assert torch.equal(outs[0][0], outs[1][0])
    idx = outs[1][1].cpu().numpy()
    okm, ovm, _ = oracle.gather_kv(idx, coff_h, f64(kb), f64(vb))
    want = oracle.sparse_attn(f64(q), okm, ovm, f64(kl), f64(vl), k, 10000.0)
    assert np.max(np.abs(f64(outs[1][0]) - want)) <= ATTN_BF16
    status_ok()


@pytest.mark.parametrize("fused", [False, True])
def test_pipeline_step_from_host_graph(fused):
    """One CUDA graph from pinned host inputs to pinned host outputs (inputs
    uploaded on two streams, attention after both): replayed twice with new
    host inputs, it gives the same bytes as the device-resident step."""
    H, D, Hq, T, k = 8, 128, 32, 128, 8
    kr, coff, coff_h = _pooled_bank(300, 1, 900, H, D, torch.bfloat16, 31)
    g = torch.Generator(device="cuda").manual_seed(32)
    kb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    vb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    m_cap = k * int(np.diff(coff_h).max())
    p = pipeline.Pipeline(kr, kb, vb, coff, B=1, T=T, T_loc=T, Hq=Hq, k=k, m_cap=m_cap, pos0=k,
                          fused=fused)
    shapes = {"q_r": (1, T, H, D), "q": (1, T, Hq, D), "k_loc": (1, T, H, D),
              "v_loc": (1, T, H, D)}
    host = {n: torch.empty(sh, dtype=torch.bfloat16).pin_memory() for n, sh in shapes.items()}
    out_h = torch.empty((1, T, Hq, D), dtype=torch.bfloat16).pin_memory()
    idx_h = torch.empty((1, k), dtype=torch.int32).pin_memory()
    graph = p.capture_from_host(host["q_r"], host["q"], host["k_loc"], host["v_loc"], out_h,
                                idx_h)
    for rep in range(2):
        dev = {n: synth.randn(sh, torch.bfloat16, "cuda", g) for n, sh in shapes.items()}
        for n in host:
            host[n].copy_(dev[n].cpu())
        graph.replay()
        torch.cuda.synchronize()
        got_out, got_idx = out_h.clone(), idx_h.clone()
        want = p(dev["q_r"], dev["q"], dev["k_loc"], dev["v_loc"])
        torch.cuda.synchronize()
        assert torch.equal(got_idx, p.idx.cpu())
        assert torch.equal(got_out, want.cpu())
    status_ok()


def test_host_stream_steps_match_device_steps():
    """HostStream runs consecutive steps from pinned host buffers with the
    uploads and read-backs on their own streams (double-buffered device
    buffers, two graphs): five steps with different inputs, each read back
    while the next computes, give the device-resident step's bytes."""
    H, D, Hq, T, k = 8, 128, 32, 64, 8
    kr, coff, coff_h = _pooled_bank(300, 1, 900, H, D, torch.bfloat16, 61)
    g = torch.Generator(device="cuda").manual_seed(62)
    kb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    vb = synth.randn(kr.shape, torch.bfloat16, "cuda", g)
    m_cap = k * int(np.diff(coff_h).max())
    p = pipeline.Pipeline(kr, kb, vb, coff, B=1, T=T, T_loc=T, Hq=Hq, k=k, m_cap=m_cap, pos0=k)
    shapes = {"q_r": (1, T, H, D), "q": (1, T, Hq, D), "k_loc": (1, T, H, D),
              "v_loc": (1, T, H, D)}
    steps = []
    for i in range(5):
        dev = {n: synth.randn(sh, torch.bfloat16, "cuda", g) for n, sh in shapes.items()}
        host = {n: t.cpu().pin_memory() for n, t in dev.items()}
        out_h = torch.empty((1, T, Hq, D), dtype=torch.bfloat16).pin_memory()
        idx_h = torch.empty((1, k), dtype=torch.int32).pin_memory()
        steps.append((dev, host, out_h, idx_h))
    hs = pipeline.HostStream(p)
    for dev, host, out_h, idx_h in steps:
        hs.step(host["q_r"], host["q"], host["k_loc"], host["v_loc"], out_h, idx_h)
    hs.synchronize()
    for dev, host, out_h, idx_h in steps:
        want = p(dev["q_r"], dev["q"], dev["k_loc"], dev["v_loc"])
        torch.cuda.synchronize()
        assert torch.equal(idx_h, p.idx.cpu())
        assert torch.equal(out_h, want.cpu())
    status_ok()


def _oracle_route_bank(q64, bank, rows: int = 32768):
    """The oracle's routing over a device bank, upcast slice by slice (the
    whole bank in float64 would not fit in host memory)."""
    C = bank.shape[0]
    out = np.empty((q64.shape[0], C))
    for c0 in range(0, C, rows):
        out[:, c0:c0 + rows] = oracle.route_chunk_scores(q64, f64(bank[c0:c0 + rows]))
    return out


def _check_step_memory_and_attention(p, w, coff_h, k_bar_dev, v_bar_dev):
    """The gathered rows of the GPU's selection equal the oracle's gather of
    the same documents bit for bit; the attention output matches the
    oracle's attention over those rows element by element."""
    idx = p.idx.cpu().numpy()
    okm, ovm, oml = oracle.gather_kv(idx, coff_h, f64(k_bar_dev), f64(v_bar_dev))
    ml = p.mem_len.cpu().tolist()
    assert ml == list(oml)
    for b in range(idx.shape[0]):
        np.testing.assert_array_equal(f64(p.k_mem[b, :ml[b]]), okm[b])
        np.testing.assert_array_equal(f64(p.v_mem[b, :ml[b]]), ovm[b])
    want = oracle.sparse_attn(f64(w["q"]), okm, ovm, f64(w["k_loc"]), f64(w["v_loc"]), w["pos0"],
                              10000.0)
    got = f64(p.out)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - want)) <= ATTN_BF16
    return idx, okm, ovm, want


def test_100m_step_vs_oracle():
    """The whole step at the 100M-token bank (1,612,509 chunks, one
    256-token prefill query, top-16): route over the prepared bank, top-k,
    gather and attention, as the benchmark runs it.  The oracle routes the
    full bank (the same bank bytes, float64): every document score within
    2e-3, the selected documents equal to the oracle's wherever its
    k-th/(k+1)-th gap exceeds 4e-3 (and each rank where both neighbouring
    gaps do), the gathered rows bit-exact and the attention output within
    2e-2 of the oracle's attention over the selected rows; the fused path
    gives the same attention from the bank."""
    lengths = synth.bank_100m_lengths()
    coff_h = oracle.chunk_offsets_from_lengths(lengths.numpy())
    w = synth.bank_100m(coff_h, "cuda")
    coff = torch.from_numpy(coff_h).cuda()
    hat = pipeline.prepare_bank(w["kr_bar"])
    m_cap = w["k"] * int(np.diff(coff_h).max())
    p = pipeline.Pipeline(hat, w["k_bar"], w["v_bar"], coff, B=1, T=w["T"], T_loc=w["T_loc"],
                          Hq=w["Hq"], k=w["k"], m_cap=m_cap, pos0=w["pos0"], prepared=True)
    p(w["q_r"], w["q"], w["k_loc"], w["v_loc"])
    torch.cuda.synchronize()
    ods = oracle.doc_max(_oracle_route_bank(f64(w["q_r"]), w["kr_bar"]), coff_h)
    assert np.max(np.abs(f64(p.doc_scores) - ods)) <= ROUTE_ATOL
    idx, okm, ovm, want = _check_step_memory_and_attention(p, w, coff_h, w["k_bar"], w["v_bar"])
    _check_topk_on_routed(idx, ods, w["k"])
    fatt = pipeline.FusedAttention(torch.bfloat16, 1, w["T"], w["T_loc"], w["Hq"], 8, 128,
                                   w["k"], m_cap, "cuda")
    fout = fatt(w["q"], p.idx, coff, w["k_bar"], w["v_bar"], w["k_loc"], w["v_loc"], w["pos0"])
    torch.cuda.synchronize()
    assert np.max(np.abs(f64(fout) - want)) <= ATTN_BF16
    status_ok()


@pytest.mark.parametrize("prepared", [False, True])
def test_1m_step_vs_oracle(prepared):
    """The whole step at the 1M-token bank (1,000 token-level documents, one
    128-token prefill query, top-16): encode on the GPU, route, top-k,
    gather, attention.

    Two oracle comparisons.  Same bytes: the oracle routes the GPU's own
    bf16 bank -- every document score within 2e-3, the top-16 by the 4e-3
    gap rule, the gathered rows bit-exact and the attention within 2e-2.
    Chained: the oracle encodes the token tensors itself (float64) and
    routes and attends over its own bank -- the pooled banks within 1e-2
    normwise, the document scores within 4e-3 (the 2e-3 routing tolerance
    plus the bf16 rounding of the GPU's pooled K̄_r, whose rows are means of
    64 N(0,1) tokens: up to 2^-9 relative, which moves a cosine by up to
    ~2e-3), and the attention over the oracle's own rows of the selected
    documents within 2e-2."""
    w = synth.bank_1m("cuda")
    toff = w["tok_offsets"].cuda()
    coff = pipeline.chunk_offsets(toff)
    coff_h = coff.cpu().numpy()
    C = int(coff_h[-1])
    kb, vb, rb = pipeline.encode_pool(w["k_tok"], w["v_tok"], w["kr_tok"], toff, coff, C)
    bank = pipeline.prepare_bank(rb[0]) if prepared else rb[0]
    m_cap = w["k"] * int(np.diff(coff_h).max())
    p = pipeline.Pipeline(bank, kb[0], vb[0], coff, B=1, T=w["T"], T_loc=w["T_loc"], Hq=w["Hq"],
                          k=w["k"], m_cap=m_cap, pos0=w["pos0"], prepared=prepared)
    p(w["q_r"], w["q"], w["k_loc"], w["v_loc"])
    torch.cuda.synchronize()
    q = f64(w["q_r"])
    # same bytes: the oracle routes the GPU's pooled bank
    ods = oracle.doc_max(oracle.route_chunk_scores(q, f64(rb[0])), coff_h)
    ds = f64(p.doc_scores)
    assert np.max(np.abs(ds - ods)) <= ROUTE_ATOL
    idx, _, _, want = _check_step_memory_and_attention(p, w, coff_h, kb[0], vb[0])
    _check_topk_on_routed(idx, ods, w["k"])
    # chained: the oracle's own encoding of every document
    toff_h = w["tok_offsets"].numpy()
    okb = np.empty((C, 8, 128))
    ovb = np.empty((C, 8, 128))
    orb = np.empty((C, 8, 128))
    for d in range(len(toff_h) - 1):
        t0, t1 = int(toff_h[d]), int(toff_h[d + 1])
        c0, c1 = int(coff_h[d]), int(coff_h[d + 1])
        okb[c0:c1], ovb[c0:c1], orb[c0:c1] = oracle.encode_pool_doc(
            f64(w["k_tok"][0, t0:t1]), f64(w["v_tok"][0, t0:t1]), f64(w["kr_tok"][0, t0:t1]),
            10000.0)
    for got, ref in ((kb[0], okb), (vb[0], ovb), (rb[0], orb)):
        assert normwise(f64(got), ref) <= RTOL_BF16
    ods_chain = oracle.doc_max(oracle.route_chunk_scores(q, orb), coff_h)
    assert np.max(np.abs(ds - ods_chain)) <= ROUTE_ATOL + 2e-3
    ckm, cvm, _ = oracle.gather_kv(idx, coff_h, okb, ovb)
    want_chain = oracle.sparse_attn(f64(w["q"]), ckm, cvm, f64(w["k_loc"]), f64(w["v_loc"]),
                                    w["pos0"], 10000.0)
    assert np.max(np.abs(f64(p.out) - want_chain)) <= ATTN_BF16
    status_ok()


# ------------------------------------------------------------------ backward

def _rel(got, want):
    return np.max(np.abs(got - want)) / max(np.max(np.abs(want)), 1e-30)


def test_encode_pool_backward_vs_oracle():
    """Token gradients from pooled gradients: /count per chunk, K rotated
    back by -p; two layers, documents with partial tails and a 1-token one."""
    L, H, D = 2, 8, 128
    lengths = np.array([180, 64, 1, 300, 77])
    toff_h = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    coff_h = oracle.chunk_offsets_from_lengths(lengths)
    N, C = int(toff_h[-1]), int(coff_h[-1])
    g = torch.Generator(device="cuda").manual_seed(77)
    dk, dv, dr = (torch.randn((L, C, H, D), generator=g, device="cuda") for _ in range(3))
    gk, gv, gr = pipeline.encode_pool_backward(dk, dv, dr, torch.from_numpy(toff_h).cuda(),
                                               torch.from_numpy(coff_h).cuda(), N)
    torch.cuda.synchronize()
    ok, ov, orr = oracle.encode_pool_backward(f64(dk), f64(dv), f64(dr), toff_h)
    for got, want in ((gk, ok), (gv, ov), (gr, orr)):
        assert _rel(f64(got), want) <= 1e-5
    status_ok()


def _clear_gap_grad(q64, k64, coff_h, gap, rng, frac=0.6):
    """dL/d(doc score): N(0,1) on a random subset of the (query, document)
    pairs whose best and second-best (chunk, token) head-mean cosines differ
    by more than `gap` (their first maximiser is then the same in any
    precision within that gap), 0 elsewhere."""
    B, T, H, _ = q64.shape
    n_docs = len(coff_h) - 1
    qn = q64 / np.linalg.norm(q64, axis=-1, keepdims=True)
    kn = k64 / np.linalg.norm(k64, axis=-1, keepdims=True)
    d_doc = np.zeros((B, n_docs))
    for b in range(B):
        for d in range(n_docs):
            s = np.einsum("thd,chd->ct", qn[b], kn[coff_h[d]:coff_h[d + 1]]).ravel() / H
            top2 = np.sort(s)[-2:] if s.size > 1 else np.array([-np.inf, s[0]])
            if top2[1] - top2[0] > gap and rng.random() < frac:
                d_doc[b, d] = rng.standard_normal()
    return d_doc


# (B, T): one 128-column pass; one 64-column pass; 300 query columns in two
# 256-column passes, the second query's tokens split across them
@pytest.mark.parametrize("dtype,B,T,H,D", [
    (torch.float32, 2, 40, 8, 128), (torch.bfloat16, 2, 40, 8, 128),
    (torch.bfloat16, 1, 40, 8, 128), (torch.bfloat16, 2, 150, 8, 128),
    (torch.bfloat16, 3, 20, 4, 64),                      # D = 64 scan, 64 columns
])
def test_route_backward_vs_oracle(dtype, B, T, H, D):
    """dQ_r and dK̄_r from dL/d(doc_scores), against the oracle, on the
    (query, document) pairs whose first maximiser is decided beyond rounding:
    a gap above 1e-4 for the fp32 CUDA-core path, above 4e-3 (the routing
    score tolerance) for the bf16 path, whose maximisers come from the
    tensor-core scan of bf16 unit rows."""
    n_docs = 30
    g = torch.Generator(device="cuda").manual_seed(5 + B * T)
    gc = torch.Generator().manual_seed(5)
    lengths = torch.randint(1, 900, (n_docs,), generator=gc).numpy()
    coff_h = oracle.chunk_offsets_from_lengths(lengths)
    C = int(coff_h[-1])
    q_r = synth.randn((B, T, H, D), dtype, "cuda", g)
    kr = synth.randn((C, H, D), dtype, "cuda", g)
    q64, k64 = f64(q_r), f64(kr)
    gap = 1e-4 if dtype == torch.float32 else 4e-3
    d_doc = _clear_gap_grad(q64, k64, coff_h, gap, np.random.default_rng(5))
    assert np.count_nonzero(d_doc) >= 10
    dq, dk = pipeline.route_backward(q_r, kr, torch.from_numpy(coff_h).cuda(),
                                     torch.from_numpy(d_doc).float().cuda())
    torch.cuda.synchronize()
    oq, ok = oracle.route_scores_backward(q64, k64, coff_h, d_doc.astype(np.float32))
    assert _rel(f64(dq), oq) <= 1e-4
    assert _rel(f64(dk), ok) <= 1e-4
    status_ok()


def test_route_backward_first_maximiser_ties():
    """Exact ties go to the first maximiser: two identical chunk rows and two
    identical query tokens make four equal best pairs in document 1; the
    gradient must reach only (its lower chunk, the lower token)."""
    B, T, H, D = 1, 24, 8, 128
    lengths = np.array([300, 640, 200])
    coff_h = oracle.chunk_offsets_from_lengths(lengths)
    C = int(coff_h[-1])
    g = torch.Generator(device="cuda").manual_seed(11)
    q_r = synth.randn((B, T, H, D), torch.bfloat16, "cuda", g)
    kr = synth.randn((C, H, D), torch.bfloat16, "cuda", g)
    q_r[0, 17] = q_r[0, 6]
    c_a, c_b = int(coff_h[1]) + 2, int(coff_h[1]) + 7
    row = (q_r[0, 6].float() + 0.8 * synth.randn((H, D), torch.float32, "cuda", g))
    kr[c_a] = row.to(torch.bfloat16)
    kr[c_b] = kr[c_a]
    d_doc = torch.zeros((B, 3), dtype=torch.float32, device="cuda")
    d_doc[0, 1] = 1.0
    dq, dk = pipeline.route_backward(q_r, kr, torch.from_numpy(coff_h).cuda(), d_doc)
    torch.cuda.synchronize()
    oq, ok = oracle.route_scores_backward(f64(q_r), f64(kr), coff_h, f64(d_doc))
    _, c_star, t_star = oracle.route_argmax(f64(q_r), f64(kr), coff_h)
    assert (int(c_star[0, 1]), int(t_star[0, 1])) == (c_a, 6)
    dq_h, dk_h = f64(dq), f64(dk)
    assert np.count_nonzero(dq_h[0, 17]) == 0 and np.count_nonzero(dk_h[c_b]) == 0
    assert np.count_nonzero(dq_h[0, 6]) > 0 and np.count_nonzero(dk_h[c_a]) > 0
    assert _rel(dq_h, oq) <= 1e-4
    assert _rel(dk_h, ok) <= 1e-4
    status_ok()


def test_route_backward_workspace_contract():
    """bf16 takes the tensor-core path and needs its workspace; fp32 needs
    none; a short workspace is refused before any launch."""
    B, T, H, D, C, n_docs = 1, 16, 8, 128, 40, 4
    assert msa.msa_route_backward_workspace_size(msa.MSA_BF16, B, T, H, D, C, n_docs) > 0
    assert msa.msa_route_backward_workspace_size(msa.MSA_F32, B, T, H, D, C, n_docs) == 0
    q = torch.zeros((B, T, H, D), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((C, H, D), dtype=torch.bfloat16, device="cuda")
    coff = torch.tensor([0, 10, 20, 30, 40], dtype=torch.int64, device="cuda")
    dd = torch.zeros((B, n_docs), dtype=torch.float32, device="cuda")
    dq = torch.zeros((B, T, H, D), dtype=torch.float32, device="cuda")
    dk = torch.zeros((C, H, D), dtype=torch.float32, device="cuda")
    with pytest.raises(msa.MsaError):
        msa.msa_route_backward(msa.MSA_BF16, B, T, H, D, q, k, C, coff, n_docs, dd, dq, dk,
                               None, 0)
    status_ok()
