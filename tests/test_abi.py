"""CPU checks of the C ABI boundary: libmsa.so loads, exports every function
include/msa.h declares, and rejects bad arguments on the host before any
CUDA work (no GPU needed for these paths)."""


import pytest

from latent_memory_routing_b200 import msa


@pytest.fixture(scope="module")
def lib():
    return msa.lib()


def test_header_declares_the_hot_path(lib):
    names = msa.header_symbols()
    for required in ("msa_encode_pool", "msa_route_scores", "msa_topk_docs",
                     "msa_gather_kv", "msa_sparse_attn"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in msa.header_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_header():
    assert set(msa.header_symbols()) == set(msa._SIGS)


def test_status_strings(lib):
    for code in range(-6, 1):
        assert msa.msa_status_string(code)
    assert msa.msa_status_string(12345) == "unknown status"
    assert "sm_100a" in msa.msa_version()


NULL = None


def test_host_validation_topk(lib):
    f = lib.msa_topk_docs
    assert f(1, 10, 11, 16, 16, NULL, NULL, 0, NULL) == -1      # k > n_docs
    assert f(1, 10, 0, 16, 16, NULL, NULL, 0, NULL) == -1       # k == 0
    assert f(1, 10, 2, NULL, 16, NULL, NULL, 0, NULL) == -1     # NULL scores


def test_host_validation_bounded_wait(lib):
    f = lib.msa_check_bounded_wait
    assert f(999, 0, NULL) == -1                  # limit below 1 us
    assert f(10_000_000_001, 0, NULL) == -1       # limit above 10 s
    assert f(-5, 1, NULL) == -1


def test_host_validation_route(lib):
    f = lib.msa_route_scores
    p = 256
    assert f(1, 1, 4, 0, 128, p, p, 10, p, 2, p, NULL, p, 1 << 20, NULL) == -1   # H == 0
    assert f(1, 1, 4, 8, 96, p, p, 10, p, 2, p, NULL, p, 1 << 20, NULL) == -2    # D == 96
    assert f(1, 1, 4, 9, 128, p, p, 10, p, 2, p, NULL, p, 1 << 20, NULL) == -2   # bf16 H > 8
    assert f(1, 1, 4, 8, 128, p + 4, p, 10, p, 2, p, NULL, p, 1 << 20, NULL) == -1  # misaligned
    assert f(1, 1, 4, 8, 128, p, p, 10, p, 2, p, NULL, NULL, 0, NULL) == -6      # no workspace


def test_host_validation_encode_gather_attn(lib):
    p = 256
    assert lib.msa_encode_pool(1, 1, 100, 2, 8, 128, p, p, p, p, p, 4, 1e4, 65,
                               p, p, p, NULL) == -1                              # chunk > 64
    assert lib.msa_encode_pool(1, 1, 100, 2, 8, 100, p, p, p, p, p, 4, 1e4, 64,
                               p, p, p, NULL) == -2                              # D == 100
    assert lib.msa_gather_kv(1, 1, 3, 8, 128, p, p, 2, p, p, 16, p, p, p, NULL) == -1  # k > n
    assert lib.msa_sparse_attn(1, 1, 5, 4, 32, 8, 128, p, p, p, p, 16, p, p, 16, 1e4, 0.0,
                               p, p, 1 << 20, NULL) == -1                        # T > T_loc
    assert lib.msa_sparse_attn(1, 1, 1, 4, 30, 8, 128, p, p, p, p, 16, p, p, 16, 1e4, 0.0,
                               p, p, 1 << 20, NULL) == -2                        # Hq % H
    assert lib.msa_device_status(NULL, 0, NULL) == -1


def test_workspace_sizes_are_monotone(lib):
    a = msa.msa_route_workspace_size(1, 1, 256, 8, 128)
    b = msa.msa_route_workspace_size(1, 2, 256, 8, 128)
    assert 0 < a < b
    assert msa.msa_route_workspace_size(1, 0, 256, 8, 128) == 0


@pytest.fixture(scope="module")
def debug_lib():
    """libmsa_debug.so (same sources built with -DMSA_DEBUG), loaded beside
    the release library under its own handle."""
    import ctypes

    from latent_memory_routing_b200 import build
    handle = ctypes.CDLL(build.build(debug=True))
    for name, (res, args) in msa._SIGS.items():
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    return handle


def test_debug_library_exports_every_call(debug_lib):
    missing = [n for n in msa.header_symbols() if not hasattr(debug_lib, n)]
    assert not missing, missing


def test_debug_library_rejects_the_same_host_arguments(debug_lib):
    f = debug_lib.msa_topk_docs
    assert f(1, 10, 11, 16, 16, NULL, NULL, 0, NULL) == -1
    p = 256
    g = debug_lib.msa_route_scores
    assert g(1, 1, 4, 8, 96, p, p, 10, p, 2, p, NULL, p, 1 << 20, NULL) == -2
    assert g(1, 1, 4, 8, 128, p, p, 10, p, 2, p, NULL, NULL, 0, NULL) == -6


def test_input_checks_exist_only_in_the_debug_build(debug_lib):
    """The release library carries none of the debug build's checks (they
    compile away), the debug library carries all three."""
    import subprocess

    from latent_memory_routing_b200 import build

    def checks(path):
        out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True,
                             text=True, check=True).stdout
        return {n for n in ("debug_check_offsets", "debug_check_mem_len", "debug_finish")
                if n in out}

    assert checks(build.LIB_DEBUG) == {"debug_check_offsets", "debug_check_mem_len",
                                       "debug_finish"}
    assert checks(build.LIB) == set()


class _StubLib:
    """Stands in for libmsa.so: records which entry points were reached."""

    def __init__(self):
        self.called = []

    def __getattr__(self, name):
        def fn(*args):
            self.called.append(name)
            return 0
        return fn


@pytest.fixture
def stub(monkeypatch):
    """The stubbed library, with CPU tensors standing in for device tensors
    (the placement check is exercised on its own below)."""
    s = _StubLib()
    monkeypatch.setattr(msa, "lib", lambda *a, **k: s)
    monkeypatch.setattr(msa, "_device_ok", lambda t, host_ok: True)
    return s


@pytest.fixture
def stub_strict(monkeypatch):
    """The stubbed library with the binding's real placement check: on a
    machine without a GPU every tensor is a host tensor."""
    s = _StubLib()
    monkeypatch.setattr(msa, "lib", lambda *a, **k: s)
    return s


def test_binding_rejects_other_element_types(stub):
    """A tensor of another type than the call reads would be misread by the
    kernel: a narrower one (bf16 where fp32 is declared, int32 offsets where
    int64 are read) overrun, a wider one (fp32 q in a bf16 call, int64 ids
    where int32 are read) reinterpreted.  The binding refuses both before
    the library is called."""
    import torch
    f32, bf16 = torch.float32, torch.bfloat16
    i32, i64 = torch.int32, torch.int64
    with pytest.raises(ValueError, match="scores is torch.bfloat16"):
        msa.msa_topk_docs(1, 10, 2, torch.zeros(10, dtype=bf16), torch.zeros(2, dtype=i32),
                          None, None, 0, stream=0)
    with pytest.raises(ValueError, match="idx is torch.int64"):
        msa.msa_topk_docs(1, 10, 2, torch.zeros(10, dtype=f32), torch.zeros(2, dtype=i64),
                          None, None, 0, stream=0)
    with pytest.raises(ValueError, match="tok_offsets is torch.int32"):
        msa.msa_chunk_offsets(3, torch.zeros(4, dtype=i32), 64, torch.zeros(4, dtype=i64),
                              stream=0)
    with pytest.raises(ValueError, match="q_r is torch.float32"):
        msa.msa_route_scores(msa.MSA_BF16, 1, 1, 8, 128, torch.zeros(1024, dtype=f32),
                             torch.zeros(10 * 1024, dtype=bf16), 10,
                             torch.zeros(4, dtype=i64), 3, torch.zeros(3), None, None, 0,
                             stream=0)
    with pytest.raises(ValueError, match="mem_len is torch.int64"):
        msa.msa_gather_kv(msa.MSA_BF16, 1, 2, 8, 128, torch.zeros(2, dtype=i32),
                          torch.zeros(4, dtype=i64), 3, torch.zeros(1024, dtype=bf16),
                          torch.zeros(1024, dtype=bf16), 4, torch.zeros(4096, dtype=bf16),
                          torch.zeros(4096, dtype=bf16), torch.zeros(1, dtype=i64), stream=0)
    assert stub.called == []
    B, T, T_loc, Hq, H, D, m_cap = 1, 2, 2, 4, 2, 64, 3
    ok = dict(q=torch.zeros(B * T * Hq * D, dtype=f32),
              k_mem=torch.zeros(B * m_cap * H * D, dtype=f32),
              v_mem=torch.zeros(B * m_cap * H * D, dtype=f32),
              mem_len=torch.zeros(B, dtype=i32),
              k_loc=torch.zeros(B * T_loc * H * D, dtype=f32),
              v_loc=torch.zeros(B * T_loc * H * D, dtype=f32),
              out=torch.zeros(B * T * Hq * D, dtype=f32))

    def attn(**kw):
        a = {**ok, **kw}
        msa.msa_sparse_attn(msa.MSA_F32, B, T, T_loc, Hq, H, D, a["q"], a["k_mem"], a["v_mem"],
                            a["mem_len"], m_cap, a["k_loc"], a["v_loc"], 2, 10000.0, 0.0,
                            a["out"], None, 0, stream=0)

    attn()  # matching types reach the library
    assert stub.called == ["msa_sparse_attn"]
    for name in ("q", "k_mem", "v_mem", "k_loc", "v_loc", "out"):
        with pytest.raises(ValueError, match=name):
            attn(**{name: ok[name].to(bf16)})
    with pytest.raises(ValueError, match="mem_len"):
        attn(mem_len=torch.zeros(B, dtype=torch.int16))
    with pytest.raises(ValueError, match="mem_len"):
        attn(mem_len=torch.zeros(B, dtype=torch.int64))
    assert stub.called == ["msa_sparse_attn"]  # no refused call reached it


def test_binding_refuses_a_workspace_smaller_than_ws_bytes(stub):
    """The library trusts ws_bytes: a tensor holding fewer bytes would be
    written past its end, so the binding compares the two first."""
    import torch
    q = torch.zeros(1024, dtype=torch.bfloat16)
    kr = torch.zeros(10 * 1024, dtype=torch.bfloat16)
    coff = torch.zeros(4, dtype=torch.int64)
    ws = torch.zeros(4096, dtype=torch.uint8)
    with pytest.raises(ValueError, match="ws holds 4096 bytes, ws_bytes says 8192"):
        msa.msa_route_scores(msa.MSA_BF16, 1, 1, 8, 128, q, kr, 10, coff, 3, torch.zeros(3),
                             None, ws, 8192, stream=0)
    with pytest.raises(ValueError, match="ws holds"):
        msa.msa_topk_docs(1, 10, 2, torch.zeros(10), torch.zeros(2, dtype=torch.int32), None,
                          torch.zeros(16, dtype=torch.uint8), 17, stream=0)
    assert stub.called == []
    msa.msa_route_scores(msa.MSA_BF16, 1, 1, 8, 128, q, kr, 10, coff, 3, torch.zeros(3),
                         None, ws, 4096, stream=0)
    assert stub.called == ["msa_route_scores"]


def test_binding_refuses_host_tensors(stub_strict):
    """A pageable host tensor's address would reach the kernels as if it were
    device memory: refused.  Pinned host memory is accepted only for the
    bank of a tiered gather or fused attention (read over the host link);
    on this machine no tensor is pinned, so the bank is refused too."""
    import torch
    with pytest.raises(ValueError, match="scores is on cpu .pageable.; the kernels read it "
                                         "from the current CUDA device$"):
        msa.msa_topk_docs(1, 10, 2, torch.zeros(10), torch.zeros(2, dtype=torch.int32), None,
                          None, 0, stream=0)
    with pytest.raises(ValueError, match="k_bar .* or pinned host memory"):
        msa.msa_gather_kv(msa.MSA_BF16, 1, 2, 8, 128, 1 << 20, 1 << 20, 3,
                          torch.zeros(1024, dtype=torch.bfloat16), 1 << 20, 4, 1 << 20,
                          1 << 20, 1 << 20, stream=0)
    assert stub_strict.called == []
    # raw integer addresses are the caller's responsibility
    msa.msa_topk_docs(1, 10, 2, 1 << 20, 1 << 20, None, None, 0, stream=0)
    assert stub_strict.called == ["msa_topk_docs"]


def test_binding_rejects_short_offsets_and_outputs(stub):
    import torch
    with pytest.raises(ValueError, match="chunk_offsets"):
        msa.msa_route_scores(msa.MSA_BF16, 1, 1, 8, 128, torch.zeros(1024, dtype=torch.bfloat16),
                             torch.zeros(10 * 1024, dtype=torch.bfloat16), 10,
                             torch.zeros(3, dtype=torch.int64), 3,
                             torch.zeros(3), None, None, 0, stream=0)
    with pytest.raises(ValueError, match="top_scores"):
        msa.msa_topk_docs(2, 10, 4, torch.zeros(20), torch.zeros(8, dtype=torch.int32),
                          torch.zeros(7), None, 0, stream=0)
    assert stub.called == []
