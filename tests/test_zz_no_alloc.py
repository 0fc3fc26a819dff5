"""msa_route_scores_noalloc: routing for callers that cannot allocate device
memory (an engine whose memory is all owned by its own pool allocator, or a
latency-critical loop where cudaMalloc, which may synchronise the device, is
not acceptable).  It must give the same scores as msa_route_scores with a
caller workspace, call after call, through the C ABI.

This file is collected last on purpose (test_zz_*), so a run that stops at
the first failure has already run every other test.  It builds the library
itself, so it also passes alone in a fresh process.
"""

import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

# Both paths launch the same deterministic kernels on the same bytes; only
# the scratch's address differs, so the scores must agree bit for bit.

MSA_F32, MSA_BF16 = 0, 1


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latent_memory_routing_b200 import build, msa
    build.build()
    return msa.lib()


def _case(B, T, n_docs, seed, H=8, D=128, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda").manual_seed(seed)
    gc = torch.Generator().manual_seed(seed)
    counts = torch.randint(1, 30, (n_docs,), generator=gc)
    coff = torch.zeros(n_docs + 1, dtype=torch.int64)
    coff[1:] = torch.cumsum(counts, 0)
    C = int(coff[-1])
    q = torch.randn((B, T, H, D), device="cuda", generator=g).to(dtype)
    kr = torch.randn((C, H, D), device="cuda", generator=g).to(dtype)
    return q, kr, coff.cuda(), C


def _dt(q):
    return MSA_F32 if q.dtype == torch.float32 else MSA_BF16


def _with_workspace(lib, q, kr, coff, C, n_docs):
    B, T, H, D = q.shape
    n = lib.msa_route_workspace_size(_dt(q), B, T, H, D)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    ds = torch.full((B, n_docs), float("nan"), device="cuda")
    cs = torch.full((B, C), float("nan"), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    rc = lib.msa_route_scores(_dt(q), B, T, H, D, q.data_ptr(), kr.data_ptr(), C,
                              coff.data_ptr(), n_docs, ds.data_ptr(), cs.data_ptr(),
                              ws.data_ptr(), n, s)
    assert rc == 0
    return ds, cs


def _no_alloc(lib, q, kr, coff, C, n_docs):
    B, T, H, D = q.shape
    ds = torch.full((B, n_docs), float("nan"), device="cuda")
    cs = torch.full((B, C), float("nan"), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    rc = lib.msa_route_scores_noalloc(_dt(q), B, T, H, D, q.data_ptr(), kr.data_ptr(), C,
                                      coff.data_ptr(), n_docs, ds.data_ptr(), cs.data_ptr(), s)
    assert rc == 0
    return ds, cs


def _status_clear(lib):
    st = ctypes.c_int32(0)
    assert lib.msa_device_status(ctypes.addressof(st), 1,
                                 torch.cuda.current_stream().cuda_stream) == 0
    return st.value


@pytest.mark.parametrize("shapes", [
    # bf16: a full 256-column pass that fills the 512 KiB scratch exactly, then
    # a 99-column call whose padded query rows must not see the first call's
    # contents
    [(1, 256, 400, 1, 8, 128, torch.bfloat16), (3, 33, 250, 2, 8, 128, torch.bfloat16)],
    # fp32 (the CUDA-core path through the same scratch), two calls in a row
    [(2, 16, 40, 4, 2, 64, torch.float32), (1, 7, 33, 5, 2, 64, torch.float32)],
], ids=["bf16", "fp32"])
def test_no_alloc_matches_workspace_path_on_two_calls_in_a_row(lib, shapes):
    assert _status_clear(lib) == 0
    for B, T, n_docs, seed, H, D, dtype in shapes:
        q, kr, coff, C = _case(B, T, n_docs, seed, H, D, dtype)
        if dtype == torch.bfloat16 and B * T == 256:
            assert lib.msa_route_workspace_size(MSA_BF16, B, T, H, D) == \
                lib.msa_route_noalloc_scratch_bytes()
        a_ds, a_cs = _with_workspace(lib, q, kr, coff, C, n_docs)
        b_ds, b_cs = _no_alloc(lib, q, kr, coff, C, n_docs)
        torch.cuda.synchronize()
        assert torch.isfinite(a_ds).all() and torch.isfinite(a_cs).all()
        assert torch.equal(a_ds, b_ds)
        assert torch.equal(a_cs, b_cs)
        assert _status_clear(lib) == 0


def test_no_alloc_rejects_shapes_beyond_its_scratch(lib):
    cap = lib.msa_route_noalloc_scratch_bytes()
    assert cap == 512 * 1024
    # 257 query columns need a second 256-column pass: 1 MiB of scratch
    assert lib.msa_route_workspace_size(MSA_BF16, 1, 257, 8, 128) > cap
    q, kr, coff, C = _case(1, 257, 50, 3)
    ds = torch.empty((1, 50), device="cuda")
    rc = lib.msa_route_scores_noalloc(MSA_BF16, 1, 257, 8, 128, q.data_ptr(), kr.data_ptr(), C,
                                      coff.data_ptr(), 50, ds.data_ptr(), None,
                                      torch.cuda.current_stream().cuda_stream)
    assert rc == -6  # MSA_ERR_WORKSPACE
