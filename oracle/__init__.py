"""Plain float64 CPU oracle for the Memory Sparse Attention (MSA) hot path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline / reference arm of ``bench.py`` may
import or execute anything in this package.  The product path
(``latent_memory_routing_b200`` and its CUDA library) never imports it, and
this package never imports the product: the two share no code.

Modules
-------
msa_oracle
    Vectorised NumPy float64 implementation of each step, written from the
    definitions on the pages (cited per function).
msa_loops
    A second, deliberately loop-only implementation for tiny shapes, used to
    pin ``msa_oracle`` against a structurally different restatement.
msa_backward
    The backward pass of chunk pooling and routing (gradients of the token
    tensors and of the routing query / bank from the gradients of the pooled
    bank and of the document scores), for training with a routing loss.
"""

from .msa_oracle import (  # noqa: F401
    CHUNK,
    EPS,
    chunk_counts,
    chunk_offsets_from_lengths,
    rope_inv_freq,
    rope_rotate,
    encode_pool,
    cosine,
    route_chunk_scores,
    doc_max,
    encode_pool_doc,
    chunk_token_ranges,
    route_scores,
    topk_docs,
    gather_kv,
    sparse_attn,
    msa_forward,
)
from .msa_backward import (  # noqa: F401,E402
    cosine_grad,
    encode_pool_backward,
    route_argmax,
    route_scores_backward,
)
