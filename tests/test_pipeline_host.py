"""Pipeline's host logic on the CPU, with the library stubbed: one step
calls the entry points in the path's order (route -> top-k -> gather ->
attend, or route -> top-k -> fused attend), on buffers whose sizes and
element types pass the binding's checks; wrong input types are refused
before any call."""

import pytest
import torch

from latent_memory_routing_b200 import msa, pipeline


class _StubLib:
    def __init__(self):
        self.called = []

    def __getattr__(self, name):
        def fn(*args):
            if not name.endswith("_size"):
                self.called.append(name)
            return 4096 if name.endswith("_size") else 0
        return fn


@pytest.fixture
def stub(monkeypatch):
    s = _StubLib()
    monkeypatch.setattr(msa, "lib", lambda *a, **k: s)
    monkeypatch.setattr(msa, "_stream", lambda stream: 0)
    # CPU tensors stand in for device tensors here
    monkeypatch.setattr(msa, "_device_ok", lambda t, host_ok: True)
    return s


def _bank(n_docs=12, H=8, D=128):
    counts = torch.arange(1, n_docs + 1)
    coff = torch.zeros(n_docs + 1, dtype=torch.int64)
    coff[1:] = torch.cumsum(counts, 0)
    C = int(coff[-1])
    bf = torch.bfloat16
    return (torch.zeros((C, H, D), dtype=bf), torch.zeros((C, H, D), dtype=bf),
            torch.zeros((C, H, D), dtype=bf), coff)


def _inputs(B=2, T=16, Hq=32, H=8, D=128, dt=torch.bfloat16):
    return (torch.zeros((B, T, H, D), dtype=dt), torch.zeros((B, T, Hq, D), dtype=dt),
            torch.zeros((B, T, H, D), dtype=dt), torch.zeros((B, T, H, D), dtype=dt))


@pytest.mark.parametrize("fused", [False, True])
def test_step_calls_the_path_in_order(stub, fused):
    kr, kb, vb, coff = _bank()
    p = pipeline.Pipeline(kr, kb, vb, coff, B=2, T=16, T_loc=16, Hq=32, k=4, m_cap=4 * 12,
                          prepared=True, fused=fused)
    stub.called.clear()
    out = p(*_inputs())
    want = ["msa_route_scores_prepared", "msa_topk_docs"]
    want += ["msa_sparse_attn_fused"] if fused else ["msa_gather_kv", "msa_sparse_attn"]
    assert stub.called == want
    assert out.shape == (2, 16, 32, 128) and out.dtype == torch.bfloat16
    assert p.idx.dtype == torch.int32 and p.doc_scores.dtype == torch.float32


def test_step_refuses_inputs_of_a_narrower_type(stub):
    kr, kb, vb, coff = _bank()
    p = pipeline.Pipeline(kr, kb, vb, coff, B=2, T=16, T_loc=16, Hq=32, k=4, m_cap=48,
                          prepared=True)
    q_r, q, kl, vl = _inputs()
    stub.called.clear()
    with pytest.raises(ValueError, match="q_r is torch.int8"):
        p(torch.zeros(q_r.shape, dtype=torch.int8), q, kl, vl)
    assert stub.called == []


def test_unprepared_router_and_fp32_attention(stub):
    """An fp32 pipeline over a raw bank routes with msa_route_scores and
    attends in fp32 (its buffers carry the bank's dtype)."""
    H, D = 2, 64
    n_docs = 5
    coff = torch.tensor([0, 3, 5, 6, 9, 12], dtype=torch.int64)
    kr = torch.zeros((12, H, D))
    p = pipeline.Pipeline(kr, kr.clone(), kr.clone(), coff, B=1, T=16, T_loc=16, Hq=4, k=2,
                          m_cap=6)
    stub.called.clear()
    out = p(*_inputs(B=1, T=16, Hq=4, H=H, D=D, dt=torch.float32))
    assert stub.called[0] == "msa_route_scores" and stub.called[-1] == "msa_sparse_attn"
    assert out.dtype == torch.float32 and p.k_mem.shape == (1, 6, H, D)
    assert n_docs == p.n_docs
