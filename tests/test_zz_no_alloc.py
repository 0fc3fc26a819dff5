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

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROUTE_ATOL = 2e-3  # the routing-score tolerance of the parity tests


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from latent_memory_routing_b200 import build, msa
    build.build()
    return msa.lib()


def _case(B, T, n_docs, seed, H=8, D=128):
    g = torch.Generator(device="cuda").manual_seed(seed)
    gc = torch.Generator().manual_seed(seed)
    counts = torch.randint(1, 30, (n_docs,), generator=gc)
    coff = torch.zeros(n_docs + 1, dtype=torch.int64)
    coff[1:] = torch.cumsum(counts, 0)
    C = int(coff[-1])
    q = torch.randn((B, T, H, D), device="cuda", generator=g).to(torch.bfloat16)
    kr = torch.randn((C, H, D), device="cuda", generator=g).to(torch.bfloat16)
    return q, kr, coff.cuda(), C


def _with_workspace(lib, q, kr, coff, C, n_docs):
    B, T, H, D = q.shape
    n = lib.msa_route_workspace_size(1, B, T, H, D)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    ds = torch.empty((B, n_docs), device="cuda")
    cs = torch.empty((B, C), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    rc = lib.msa_route_scores(1, B, T, H, D, q.data_ptr(), kr.data_ptr(), C, coff.data_ptr(),
                              n_docs, ds.data_ptr(), cs.data_ptr(), ws.data_ptr(), n, s)
    assert rc == 0
    return ds, cs


def _no_alloc(lib, q, kr, coff, C, n_docs):
    B, T, H, D = q.shape
    ds = torch.empty((B, n_docs), device="cuda")
    cs = torch.empty((B, C), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    rc = lib.msa_route_scores_noalloc(1, B, T, H, D, q.data_ptr(), kr.data_ptr(), C,
                                      coff.data_ptr(), n_docs, ds.data_ptr(), cs.data_ptr(), s)
    assert rc == 0
    return ds, cs


def test_no_alloc_matches_workspace_path_on_two_calls_in_a_row(lib):
    # a full 256-column pass, then a smaller shape whose padded query rows
    # must not see the first call's contents
    for B, T, n_docs, seed in [(1, 256, 400, 1), (3, 33, 250, 2)]:
        q, kr, coff, C = _case(B, T, n_docs, seed)
        a_ds, a_cs = _with_workspace(lib, q, kr, coff, C, n_docs)
        b_ds, b_cs = _no_alloc(lib, q, kr, coff, C, n_docs)
        torch.cuda.synchronize()
        assert np.max(np.abs(a_ds.cpu().numpy() - b_ds.cpu().numpy())) <= ROUTE_ATOL
        assert np.max(np.abs(a_cs.cpu().numpy() - b_cs.cpu().numpy())) <= ROUTE_ATOL
        st = ctypes.c_int32(0)
        assert lib.msa_device_status(ctypes.addressof(st), 1,
                                     torch.cuda.current_stream().cuda_stream) == 0
        assert st.value == 0


def test_no_alloc_rejects_shapes_beyond_its_scratch(lib):
    cap = lib.msa_route_noalloc_scratch_bytes()
    assert cap == 512 * 1024
    # 257 query columns need a second 256-column pass: 1 MiB of scratch
    assert lib.msa_route_workspace_size(1, 1, 257, 8, 128) > cap
    q, kr, coff, C = _case(1, 257, 50, 3)
    ds = torch.empty((1, 50), device="cuda")
    rc = lib.msa_route_scores_noalloc(1, 1, 257, 8, 128, q.data_ptr(), kr.data_ptr(), C,
                                      coff.data_ptr(), 50, ds.data_ptr(), None,
                                      torch.cuda.current_stream().cuda_stream)
    assert rc == -6  # MSA_ERR_WORKSPACE
