"""B200-native Memory Sparse Attention (MSA) hot path.

``libmsa.so`` (built from ``csrc/`` by ``python -m
latent_memory_routing_b200.build``) implements, as hand-written sm_100a CUDA
kernels behind the C ABI of ``include/msa.h``: document-wise RoPE with
64-token chunk pooling, cosine routing with head-mean / token-max /
document-max, top-k document selection, K/V gather and GQA sparse attention
with global RoPE offset by k.  ``msa`` is the ctypes binding (same names as
the C functions), ``pipeline`` allocates buffers and chains the calls, and
``synth`` draws the seeded synthetic workloads.
"""

from . import msa  # noqa: F401
from .msa import (  # noqa: F401
    MSA_BF16,
    MSA_F32,
    MsaError,
    msa_check_bounded_wait,
    msa_chunk_offsets,
    msa_device_status,
    msa_encode_pool,
    msa_encode_pool_backward,
    msa_gather_kv,
    msa_last_cuda_error,
    msa_route_backward,
    msa_route_backward_workspace_size,
    msa_route_prepare_bank,
    msa_route_scores,
    msa_route_scores_prepared,
    msa_route_workspace_size,
    msa_sparse_attn,
    msa_sparse_attn_fused,
    msa_sparse_attn_fused_workspace_size,
    msa_sparse_attn_workspace_size,
    msa_status_string,
    msa_topk_docs,
    msa_topk_merge_shards,
    msa_topk_workspace_size,
    msa_version,
)
