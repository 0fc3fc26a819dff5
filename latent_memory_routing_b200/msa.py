"""ctypes binding of libmsa (include/msa.h), with the same names.

Argument marshalling only: every step of the MSA hot path runs in the CUDA
kernels of ``libmsa.so``.  Tensor arguments may be torch tensors (their
device pointer is passed; shapes are checked against the sizes given) or raw
integer device addresses.  ``stream`` defaults to torch's current stream on
the current device.  A non-zero status raises ``MsaError``; the library must
have been built (``python -m latent_memory_routing_b200.build``) -- there is
no fallback.

With ``MSA_DEBUG=1`` in the environment the binding loads
``libmsa_debug.so`` (``python -m latent_memory_routing_b200.build --debug``)
instead: the same kernels, with every call first checking the device-side
index arrays it is given and then waiting for its own work, so that a
device-detected error is raised by the call that caused it.
"""

from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmsa_debug.so" if os.environ.get("MSA_DEBUG") == "1"
                         else "libmsa.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "msa.h")

MSA_F32 = 0
MSA_BF16 = 1

_STATUS = {0: "MSA_OK", -1: "MSA_ERR_INVALID_ARG", -2: "MSA_ERR_UNSUPPORTED",
           -3: "MSA_ERR_CAPACITY", -4: "MSA_ERR_CUDA", -5: "MSA_ERR_TIMEOUT",
           -6: "MSA_ERR_WORKSPACE"}


class MsaError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        self.status = status
        super().__init__(f"{fn} -> {_STATUS.get(status, status)}"
                         + (f" ({detail})" if detail else ""))


_lib = None

c_i = ctypes.c_int
c_i64 = ctypes.c_int64
c_f = ctypes.c_float
c_sz = ctypes.c_size_t
c_p = ctypes.c_void_p

_SIGS = {
    "msa_status_string": (ctypes.c_char_p, [c_i]),
    "msa_last_cuda_error": (c_i, []),
    "msa_version": (ctypes.c_char_p, []),
    "msa_device_status": (c_i, [c_p, c_i, c_p]),
    "msa_check_bounded_wait": (c_i, [c_i64, c_i, c_p]),
    "msa_chunk_offsets": (c_i, [c_i, c_p, c_i, c_p, c_p]),
    "msa_encode_pool": (c_i, [c_i, c_i, c_i64, c_i, c_i, c_i, c_p, c_p, c_p, c_p, c_p,
                              c_i64, c_f, c_i, c_p, c_p, c_p, c_p]),
    "msa_encode_pool_prepared": (c_i, [c_i, c_i, c_i64, c_i, c_i, c_i, c_p, c_p, c_p, c_p, c_p,
                                       c_i64, c_f, c_i, c_p, c_p, c_p, c_p, c_p]),
    "msa_route_workspace_size": (c_sz, [c_i, c_i, c_i, c_i, c_i]),
    "msa_route_scores": (c_i, [c_i, c_i, c_i, c_i, c_i, c_p, c_p, c_i64, c_p, c_i, c_p, c_p,
                               c_p, c_sz, c_p]),
    "msa_route_prepare_bank": (c_i, [c_i, c_i64, c_i, c_i, c_p, c_p, c_p]),
    "msa_route_scores_prepared": (c_i, [c_i, c_i, c_i, c_i, c_i, c_p, c_p, c_i64, c_p, c_i, c_p,
                                        c_p, c_p, c_sz, c_p]),
    "msa_route_noalloc_scratch_bytes": (c_sz, []),
    "msa_route_scores_noalloc": (c_i, [c_i, c_i, c_i, c_i, c_i, c_p, c_p, c_i64, c_p, c_i, c_p,
                                       c_p, c_p]),
    "msa_topk_workspace_size": (c_sz, [c_i, c_i, c_i]),
    "msa_topk_docs": (c_i, [c_i, c_i, c_i, c_p, c_p, c_p, c_p, c_sz, c_p]),
    "msa_topk_merge_shards": (c_i, [c_i, c_i, c_i, c_p, c_p, c_p, c_p, c_p, c_p]),
    "msa_gather_kv": (c_i, [c_i, c_i, c_i, c_i, c_i, c_p, c_p, c_i, c_p, c_p, c_i, c_p, c_p,
                            c_p, c_p]),
    "msa_sparse_attn_workspace_size": (c_sz, [c_i, c_i, c_i, c_i, c_i, c_i, c_i, c_i]),
    "msa_sparse_attn_fused_workspace_size": (c_sz, [c_i] * 9),
    "msa_route_backward_workspace_size": (c_sz, [c_i, c_i, c_i, c_i, c_i, c_i64, c_i]),
    "msa_route_backward": (c_i, [c_i, c_i, c_i, c_i, c_i, c_p, c_p, c_i64, c_p, c_i, c_p, c_p,
                                 c_p, c_p, c_sz, c_p]),
    "msa_encode_pool_backward": (c_i, [c_i, c_i64, c_i, c_i, c_i, c_p, c_p, c_p, c_p, c_p,
                                       c_i64, c_f, c_p, c_p, c_p, c_p]),
    "msa_sparse_attn_fused": (c_i, [c_i, c_i, c_i, c_i, c_i, c_i, c_i, c_p, c_p, c_i, c_p, c_i,
                                    c_p, c_p, c_i64, c_i, c_p, c_p, c_i, c_f, c_f, c_p, c_p,
                                    c_p, c_sz, c_p]),
    "msa_sparse_attn": (c_i, [c_i, c_i, c_i, c_i, c_i, c_i, c_i, c_p, c_p, c_p, c_p, c_i, c_p,
                              c_p, c_i, c_f, c_f, c_p, c_p, c_sz, c_p]),
}


def header_symbols(path: str = HEADER) -> list[str]:
    """Function names declared in include/msa.h."""
    with open(path, encoding="utf-8") as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z0-9_]+)\s*\(", text)))


def lib(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libmsa.so (once) and declares every signature."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with "
                              "`python -m latent_memory_routing_b200.build`")
        handle = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def dtype_code(t) -> int:
    import torch
    if t == torch.float32:
        return MSA_F32
    if t == torch.bfloat16:
        return MSA_BF16
    raise ValueError(f"unsupported dtype {t}")


def _check(name: str, rc: int):
    if rc != 0:
        detail = ""
        if rc == -4:
            detail = f"cudaError {lib().msa_last_cuda_error()}"
        raise MsaError(name, rc, detail)


# Element type of each tensor argument: the call's `dt` for floating-point
# tensors, and these fixed types for the rest.
F32, I32, I64 = "f32", "i32", "i64"


def _torch_dtype(kind):
    import torch
    return {MSA_F32: torch.float32, MSA_BF16: torch.bfloat16, F32: torch.float32,
            I32: torch.int32, I64: torch.int64}.get(kind)


def _es(dt):
    """The element type of a `dt`-typed tensor (None for an unknown dt, which
    the library itself rejects)."""
    return dt if dt in (MSA_F32, MSA_BF16) else None


def _device_ok(t, host_ok: bool) -> bool:
    """A tensor the kernels may read: on the current CUDA device, or (where
    the call reads a tiered bank over the host link) in pinned host memory."""
    import torch
    if t.is_cuda:
        return t.device.index == torch.cuda.current_device()
    return host_ok and t.is_pinned()


def _numel_ok(t, n, what, kind=None, host_ok=False):
    """Checks a tensor argument before its address goes to the library:
    contiguous, of exactly the element type the call reads (`kind`: a dt code
    or F32/I32/I64), holding at least n elements, and on the current device
    (pinned host memory only where ``host_ok``).  Raw integer addresses are
    the caller's responsibility and pass unchecked."""
    if t is None or isinstance(t, int):
        return
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    want = _torch_dtype(kind)
    if want is not None and t.dtype != want:
        raise ValueError(f"{what} is {t.dtype}, the call reads {want}")
    if t.numel() < n:
        raise ValueError(f"{what} holds {t.numel()} elements, needs {n}")
    if not _device_ok(t, host_ok):
        where = "the current CUDA device or pinned host memory" if host_ok else \
            "the current CUDA device"
        raise ValueError(f"{what} is on {t.device}{' (pageable)' if not t.is_cuda else ''}; "
                         f"the kernels read it from {where}")


def _ws_ok(ws, ws_bytes):
    """A workspace tensor must lie on the current device and hold at least
    the ws_bytes the library is told it may use."""
    if ws is None or isinstance(ws, int):
        return
    if not ws.is_contiguous():
        raise ValueError("ws must be contiguous")
    if ws.numel() * ws.element_size() < ws_bytes:
        raise ValueError(f"ws holds {ws.numel() * ws.element_size()} bytes, "
                         f"ws_bytes says {ws_bytes}")
    if not _device_ok(ws, False):
        raise ValueError(f"ws is on {ws.device}; it must be on the current CUDA device")


# ---------------------------------------------------------------- entry points

def msa_status_string(status: int) -> str:
    return lib().msa_status_string(status).decode()


def msa_version() -> str:
    return lib().msa_version().decode()


def msa_last_cuda_error() -> int:
    return lib().msa_last_cuda_error()


def msa_device_status(clear: bool = True, stream=None) -> int:
    out = ctypes.c_int32(0)
    _check("msa_device_status",
           lib().msa_device_status(ctypes.addressof(out), int(clear), _stream(stream)))
    return out.value


def msa_check_bounded_wait(limit_ns: int, arrive: bool, stream=None):
    _check("msa_check_bounded_wait",
           lib().msa_check_bounded_wait(int(limit_ns), int(arrive), _stream(stream)))


def msa_chunk_offsets(n_docs, tok_offsets, chunk, chunk_offsets, stream=None):
    _numel_ok(tok_offsets, n_docs + 1, "tok_offsets", I64)
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    _check("msa_chunk_offsets", lib().msa_chunk_offsets(
        n_docs, _ptr(tok_offsets), chunk, _ptr(chunk_offsets), _stream(stream)))


def msa_encode_pool(dt, L, n_tok, n_docs, H, D, k_tok, v_tok, kr_tok, tok_offsets,
                    chunk_offsets, n_chunks, rope_base, chunk, k_bar, v_bar, kr_bar,
                    stream=None):
    for t, what in ((k_tok, "k_tok"), (v_tok, "v_tok"), (kr_tok, "kr_tok")):
        _numel_ok(t, L * n_tok * H * D, what, _es(dt))
    for t, what in ((k_bar, "k_bar"), (v_bar, "v_bar"), (kr_bar, "kr_bar")):
        _numel_ok(t, L * n_chunks * H * D, what, _es(dt))
    _numel_ok(tok_offsets, n_docs + 1, "tok_offsets", I64)
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    _check("msa_encode_pool", lib().msa_encode_pool(
        dt, L, n_tok, n_docs, H, D, _ptr(k_tok), _ptr(v_tok), _ptr(kr_tok),
        _ptr(tok_offsets), _ptr(chunk_offsets), n_chunks, rope_base, chunk,
        _ptr(k_bar), _ptr(v_bar), _ptr(kr_bar), _stream(stream)))


def msa_encode_pool_prepared(dt, L, n_tok, n_docs, H, D, k_tok, v_tok, kr_tok, tok_offsets,
                             chunk_offsets, n_chunks, rope_base, chunk, k_bar, v_bar, kr_bar,
                             kr_hat, stream=None):
    for t, what in ((k_tok, "k_tok"), (v_tok, "v_tok"), (kr_tok, "kr_tok")):
        _numel_ok(t, L * n_tok * H * D, what, _es(dt))
    for t, what in ((k_bar, "k_bar"), (v_bar, "v_bar"), (kr_bar, "kr_bar"), (kr_hat, "kr_hat")):
        _numel_ok(t, L * n_chunks * H * D, what, _es(dt))
    _numel_ok(tok_offsets, n_docs + 1, "tok_offsets", I64)
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    _check("msa_encode_pool_prepared", lib().msa_encode_pool_prepared(
        dt, L, n_tok, n_docs, H, D, _ptr(k_tok), _ptr(v_tok), _ptr(kr_tok),
        _ptr(tok_offsets), _ptr(chunk_offsets), n_chunks, rope_base, chunk,
        _ptr(k_bar), _ptr(v_bar), _ptr(kr_bar), _ptr(kr_hat), _stream(stream)))


def msa_route_workspace_size(dt, B, T, H, D) -> int:
    return lib().msa_route_workspace_size(dt, B, T, H, D)


def msa_route_scores(dt, B, T, H, D, q_r, kr_bar, n_chunks, chunk_offsets, n_docs,
                     doc_scores, chunk_scores, ws, ws_bytes, stream=None):
    _numel_ok(q_r, B * T * H * D, "q_r", _es(dt))
    _numel_ok(kr_bar, n_chunks * H * D, "kr_bar", _es(dt))
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    _numel_ok(doc_scores, B * n_docs, "doc_scores", F32)
    _numel_ok(chunk_scores, B * n_chunks, "chunk_scores", F32)
    _ws_ok(ws, ws_bytes)
    _check("msa_route_scores", lib().msa_route_scores(
        dt, B, T, H, D, _ptr(q_r), _ptr(kr_bar), n_chunks, _ptr(chunk_offsets), n_docs,
        _ptr(doc_scores), _ptr(chunk_scores), _ptr(ws), ws_bytes, _stream(stream)))


def msa_route_prepare_bank(dt, n_chunks, H, D, kr_bar, kr_hat, stream=None):
    _numel_ok(kr_bar, n_chunks * H * D, "kr_bar", _es(dt))
    _numel_ok(kr_hat, n_chunks * H * D, "kr_hat", _es(dt))
    _check("msa_route_prepare_bank", lib().msa_route_prepare_bank(
        dt, n_chunks, H, D, _ptr(kr_bar), _ptr(kr_hat), _stream(stream)))


def msa_route_scores_prepared(dt, B, T, H, D, q_r, kr_hat, n_chunks, chunk_offsets, n_docs,
                              doc_scores, chunk_scores, ws, ws_bytes, stream=None):
    _numel_ok(q_r, B * T * H * D, "q_r", _es(dt))
    _numel_ok(kr_hat, n_chunks * H * D, "kr_hat", _es(dt))
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    _numel_ok(doc_scores, B * n_docs, "doc_scores", F32)
    _numel_ok(chunk_scores, B * n_chunks, "chunk_scores", F32)
    _ws_ok(ws, ws_bytes)
    _check("msa_route_scores_prepared", lib().msa_route_scores_prepared(
        dt, B, T, H, D, _ptr(q_r), _ptr(kr_hat), n_chunks, _ptr(chunk_offsets), n_docs,
        _ptr(doc_scores), _ptr(chunk_scores), _ptr(ws), ws_bytes, _stream(stream)))


def msa_route_noalloc_scratch_bytes() -> int:
    return lib().msa_route_noalloc_scratch_bytes()


def msa_route_scores_noalloc(dt, B, T, H, D, q_r, kr_bar, n_chunks, chunk_offsets, n_docs,
                             doc_scores, chunk_scores, stream=None):
    """msa_route_scores with the library's fixed scratch array instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    _numel_ok(q_r, B * T * H * D, "q_r", _es(dt))
    _numel_ok(kr_bar, n_chunks * H * D, "kr_bar", _es(dt))
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    _numel_ok(doc_scores, B * n_docs, "doc_scores", F32)
    _numel_ok(chunk_scores, B * n_chunks, "chunk_scores", F32)
    _check("msa_route_scores_noalloc", lib().msa_route_scores_noalloc(
        dt, B, T, H, D, _ptr(q_r), _ptr(kr_bar), n_chunks, _ptr(chunk_offsets), n_docs,
        _ptr(doc_scores), _ptr(chunk_scores), _stream(stream)))


def msa_topk_workspace_size(B, n_docs, k) -> int:
    return lib().msa_topk_workspace_size(B, n_docs, k)


def msa_topk_merge_shards(B, world, k, cand_scores, cand_idx, doc_base, idx, top_scores,
                          stream=None):
    _numel_ok(cand_scores, world * B * k, "cand_scores", F32)
    _numel_ok(cand_idx, world * B * k, "cand_idx", I32)
    _numel_ok(doc_base, world, "doc_base", I32)
    _numel_ok(idx, B * k, "idx", I32)
    _numel_ok(top_scores, B * k, "top_scores", F32)
    _check("msa_topk_merge_shards", lib().msa_topk_merge_shards(
        B, world, k, _ptr(cand_scores), _ptr(cand_idx), _ptr(doc_base), _ptr(idx),
        _ptr(top_scores), _stream(stream)))


def msa_topk_docs(B, n_docs, k, scores, idx, top_scores, ws, ws_bytes, stream=None):
    _numel_ok(scores, B * n_docs, "scores", F32)
    _numel_ok(idx, B * k, "idx", I32)
    _numel_ok(top_scores, B * k, "top_scores", F32)
    _ws_ok(ws, ws_bytes)
    _check("msa_topk_docs", lib().msa_topk_docs(
        B, n_docs, k, _ptr(scores), _ptr(idx), _ptr(top_scores), _ptr(ws), ws_bytes,
        _stream(stream)))


def msa_gather_kv(dt, B, k, H, D, idx, chunk_offsets, n_docs, k_bar, v_bar, m_cap, k_mem,
                  v_mem, mem_len, stream=None):
    _numel_ok(idx, B * k, "idx", I32)
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    # the bank's row count sits on the device (chunk_offsets[n_docs]); its
    # type and placement are checked here: device or pinned host tier
    for t, what in ((k_bar, "k_bar"), (v_bar, "v_bar")):
        _numel_ok(t, 0, what, _es(dt), host_ok=True)
    _numel_ok(k_mem, B * m_cap * H * D, "k_mem", _es(dt))
    _numel_ok(v_mem, B * m_cap * H * D, "v_mem", _es(dt))
    _numel_ok(mem_len, B, "mem_len", I32)
    _check("msa_gather_kv", lib().msa_gather_kv(
        dt, B, k, H, D, _ptr(idx), _ptr(chunk_offsets), n_docs, _ptr(k_bar), _ptr(v_bar),
        m_cap, _ptr(k_mem), _ptr(v_mem), _ptr(mem_len), _stream(stream)))


def msa_sparse_attn_workspace_size(dt, B, T, T_loc, Hq, H, D, m_cap) -> int:
    return lib().msa_sparse_attn_workspace_size(dt, B, T, T_loc, Hq, H, D, m_cap)


def msa_sparse_attn(dt, B, T, T_loc, Hq, H, D, q, k_mem, v_mem, mem_len, m_cap, k_loc, v_loc,
                    pos0, rope_base, scale, out, ws, ws_bytes, stream=None):
    _numel_ok(q, B * T * Hq * D, "q", _es(dt))
    _numel_ok(k_mem, B * m_cap * H * D, "k_mem", _es(dt))
    _numel_ok(v_mem, B * m_cap * H * D, "v_mem", _es(dt))
    _numel_ok(mem_len, B, "mem_len", I32)
    _numel_ok(k_loc, B * T_loc * H * D, "k_loc", _es(dt))
    _numel_ok(v_loc, B * T_loc * H * D, "v_loc", _es(dt))
    _numel_ok(out, B * T * Hq * D, "out", _es(dt))
    _ws_ok(ws, ws_bytes)
    _check("msa_sparse_attn", lib().msa_sparse_attn(
        dt, B, T, T_loc, Hq, H, D, _ptr(q), _ptr(k_mem), _ptr(v_mem), _ptr(mem_len), m_cap,
        _ptr(k_loc), _ptr(v_loc), pos0, rope_base, scale, _ptr(out), _ptr(ws), ws_bytes,
        _stream(stream)))


def msa_sparse_attn_fused_workspace_size(dt, B, T, T_loc, Hq, H, D, k, m_cap) -> int:
    return lib().msa_sparse_attn_fused_workspace_size(dt, B, T, T_loc, Hq, H, D, k, m_cap)


def msa_sparse_attn_fused(dt, B, T, T_loc, Hq, H, D, q, idx, k, chunk_offsets, n_docs, k_bar,
                          v_bar, n_chunks, m_cap, k_loc, v_loc, pos0, rope_base, scale, out,
                          mem_len, ws, ws_bytes, stream=None):
    _numel_ok(q, B * T * Hq * D, "q", _es(dt))
    _numel_ok(idx, B * k, "idx", I32)
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    _numel_ok(k_bar, n_chunks * H * D, "k_bar", _es(dt), host_ok=True)
    _numel_ok(v_bar, n_chunks * H * D, "v_bar", _es(dt), host_ok=True)
    _numel_ok(k_loc, B * T_loc * H * D, "k_loc", _es(dt))
    _numel_ok(v_loc, B * T_loc * H * D, "v_loc", _es(dt))
    _numel_ok(out, B * T * Hq * D, "out", _es(dt))
    _numel_ok(mem_len, B, "mem_len", I32)
    _ws_ok(ws, ws_bytes)
    _check("msa_sparse_attn_fused", lib().msa_sparse_attn_fused(
        dt, B, T, T_loc, Hq, H, D, _ptr(q), _ptr(idx), k, _ptr(chunk_offsets), n_docs,
        _ptr(k_bar), _ptr(v_bar), n_chunks, m_cap, _ptr(k_loc), _ptr(v_loc), pos0, rope_base,
        scale, _ptr(out), _ptr(mem_len), _ptr(ws), ws_bytes, _stream(stream)))


def msa_route_backward_workspace_size(dt, B, T, H, D, n_chunks, n_docs) -> int:
    return lib().msa_route_backward_workspace_size(dt, B, T, H, D, n_chunks, n_docs)


def msa_route_backward(dt, B, T, H, D, q_r, kr_bar, n_chunks, chunk_offsets, n_docs, d_doc,
                       dq_r, dkr_bar, ws=None, ws_bytes=0, stream=None):
    _numel_ok(q_r, B * T * H * D, "q_r", _es(dt))
    _numel_ok(kr_bar, n_chunks * H * D, "kr_bar", _es(dt))
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    _numel_ok(d_doc, B * n_docs, "d_doc", F32)
    _numel_ok(dq_r, B * T * H * D, "dq_r", F32)
    _numel_ok(dkr_bar, n_chunks * H * D, "dkr_bar", F32)
    _ws_ok(ws, ws_bytes)
    _check("msa_route_backward", lib().msa_route_backward(
        dt, B, T, H, D, _ptr(q_r), _ptr(kr_bar), n_chunks, _ptr(chunk_offsets), n_docs,
        _ptr(d_doc), _ptr(dq_r), _ptr(dkr_bar), _ptr(ws), ws_bytes, _stream(stream)))


def msa_encode_pool_backward(L, n_tok, n_docs, H, D, dk_bar, dv_bar, dkr_bar, tok_offsets,
                             chunk_offsets, n_chunks, rope_base, dk_tok, dv_tok, dkr_tok,
                             stream=None):
    for t, nm in ((dk_bar, "dk_bar"), (dv_bar, "dv_bar"), (dkr_bar, "dkr_bar")):
        _numel_ok(t, L * n_chunks * H * D, nm, F32)
    for t, nm in ((dk_tok, "dk_tok"), (dv_tok, "dv_tok"), (dkr_tok, "dkr_tok")):
        _numel_ok(t, L * n_tok * H * D, nm, F32)
    _numel_ok(tok_offsets, n_docs + 1, "tok_offsets", I64)
    _numel_ok(chunk_offsets, n_docs + 1, "chunk_offsets", I64)
    _check("msa_encode_pool_backward", lib().msa_encode_pool_backward(
        L, n_tok, n_docs, H, D, _ptr(dk_bar), _ptr(dv_bar), _ptr(dkr_bar), _ptr(tok_offsets),
        _ptr(chunk_offsets), n_chunks, rope_base, _ptr(dk_tok), _ptr(dv_tok), _ptr(dkr_tok),
        _stream(stream)))
