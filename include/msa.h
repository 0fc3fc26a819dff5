/*
 * libmsa -- C ABI of the Memory Sparse Attention (MSA) hot path on NVIDIA
 * B200 (sm_100a).
 *
 * The path, as the pages describing MSA define it:
 *   1. encode:  document-wise RoPE on token K, then 64-token chunk means of
 *               K, V and the routing key K_r  (msa_encode_pool);
 *   2. route:   cosine of Q_r against each pooled K̄_r, mean over heads, max
 *               over query tokens, max over a document's chunks
 *               (msa_route_scores), then the top-k documents (msa_topk_docs);
 *   3. attend:  gather the selected documents' pooled K̄/V̄ in rank order
 *               (msa_gather_kv) and run GQA attention over [memory ; local
 *               causal context] with global RoPE starting at offset k
 *               (msa_sparse_attn).
 *
 * Sources, cited by page title and section:
 *   [DEEP]  "深度分析MSA:把超长文档组织成可检索内部记忆的工程路径"
 *           (yeyulingfeng.com), §"三、文档如何变成 memory" and
 *           §"五、推理阶段：memory 的使用方式".
 *   [HYSEN] "EverMind-AI/MSA: routing top-k compressed documents inside
 *           attention, and where the 100M-token claim stops"
 *           (hysenlabs.com), §"Routing happens inside attention, not in a
 *           retrieval service in front of the model", §"Document-wise RoPE
 *           resets every document to position zero", §"Memory must be
 *           encoded offline before a query can reach it".
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers owned by the caller, row-major
 *     and contiguous, in the layouts stated per function.  Integer
 *     arguments are host values.  The library keeps no pointer after a call
 *     returns and allocates no device memory: scratch comes from the
 *     caller's workspace (sizes from the *_workspace_size functions).
 *     A workspace holds a call's state while its kernels run (rotated
 *     copies, split partials, the tensor-core prefill's work-item counter),
 *     so calls that share one must run in order: on one stream, or ordered
 *     by events.
 *   - `dt` selects the element type of every floating-point tensor of the
 *     call (MSA_F32 = float, MSA_BF16 = __nv_bfloat16); arithmetic is fp32.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and never synchronises the host.
 *   - Errors the host can see (bad sizes, NULL or misaligned pointers,
 *     unsupported shapes) are returned before anything is launched; a
 *     failing CUDA launch returns MSA_ERR_CUDA and msa_last_cuda_error()
 *     gives the cudaError_t.  Errors only the device can see (a gather that
 *     overflows its capacity, a bounded wait that ran out) are recorded in a
 *     per-device status word read with msa_device_status().
 *   - Tensors read with 16-byte vector loads must be 16-byte aligned; this
 *     is checked and reported as MSA_ERR_INVALID_ARG.
 *   - Environment switches, read once per process, choose between kernels
 *     that compute the same results (for comparison and profiling):
 *       MSA_ROUTE_PAIRS=0   prepared-bank routing on single CTAs instead of
 *                           CTA pairs;
 *       MSA_DECODE_TC=0     decode attention on the CUDA cores instead of
 *                           the tensor cores;
 *       MSA_ENCODE_TMA=0    chunk pooling by per-chunk CTAs with plain loads
 *                           instead of bulk copies;
 *       MSA_ROUTE_BWD_TC=0  the routing backward's maximisers recomputed on
 *                           the CUDA cores (fp32) instead of the tensor-core
 *                           scan;
 *       MSA_ATTN_SPLITS=n   at most n (1..16) key-tile splits in prefill
 *                           attention (default 3).
 *   - Debug build (libmsa_debug.so: the same sources compiled with
 *     -DMSA_DEBUG).  Its kernels are the release kernels.  What changes is
 *     that every compute entry point, after its host checks, validates on
 *     the device the index arrays it is given:
 *       - CSR offsets must be non-negative, non-decreasing and within the
 *         tensor they index;
 *       - memory lengths must lie in [0, m_cap].
 *     The call waits for that check and returns MSA_ERR_INVALID_ARG before
 *     any of its kernels reads through a bad array.  At its end it waits for
 *     its own work and returns a CUDA error or the status word's first
 *     error, such as MSA_ERR_CAPACITY.  The word is read, not cleared, so an
 *     earlier unread error is returned too.  While the stream is being
 *     captured into a CUDA graph nothing waits: the checks are captured with
 *     the call and record into the status word.  msa_check_bounded_wait is
 *     not wrapped.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* msa_stream_t;

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = -1,  /* NULL/misaligned pointer, bad size, k > n_docs, ... */
  MSA_ERR_UNSUPPORTED = -2,  /* shape outside what the kernels implement          */
  MSA_ERR_CAPACITY = -3,     /* gather: selected rows exceed m_cap (device word)  */
  MSA_ERR_CUDA = -4,         /* a CUDA call failed; see msa_last_cuda_error()     */
  MSA_ERR_TIMEOUT = -5,      /* a bounded device wait ran out (device word)       */
  MSA_ERR_WORKSPACE = -6     /* workspace NULL or smaller than required           */
} msa_status;

typedef enum { MSA_F32 = 0, MSA_BF16 = 1 } msa_dtype;

/* Static, NUL-terminated description of a status code. Never NULL. */
const char* msa_status_string(int status);

/* cudaError_t of the last CUDA failure seen by a libmsa call on the calling
 * host thread (0 if none). */
int msa_last_cuda_error(void);

/* Library version string, e.g. "libmsa 0.1.0 sm_100a". */
const char* msa_version(void);

/* Reads (and, if clear != 0, resets) the status word of the current device:
 * MSA_OK or the first device-detected error (MSA_ERR_CAPACITY,
 * MSA_ERR_TIMEOUT) since the last reset.  Ordered after the work already
 * queued on `stream`; blocks the host until that work is done. */
int msa_device_status(int32_t* host_out, int clear, msa_stream_t stream);

/* Failure-detection check of the bounded device waits.  Every pipelined
 * kernel (routing scan, chunk pooling, prefill and decode attention) waits on
 * mbarriers for at most a fixed time; a wait that runs out records
 * MSA_ERR_TIMEOUT in the device status word and the kernel winds down, so a
 * lost arrival becomes an error status instead of a hung GPU.  This call runs
 * that path alone: one thread initialises an mbarrier expecting one arrival
 * and waits for its first phase for at most limit_ns nanoseconds.
 *   arrive != 0  the thread arrives first: the wait succeeds at once and
 *                nothing is recorded;
 *   arrive == 0  nothing arrives: the wait expires after limit_ns and
 *                MSA_ERR_TIMEOUT is recorded in the device status word.
 * The kernel holds no asynchronous copy and no tensor memory, so the context
 * stays usable either way.  1000 <= limit_ns <= 10^10 (10 s), else
 * MSA_ERR_INVALID_ARG (checked before any CUDA call).  Asynchronous on
 * `stream`; read the outcome with msa_device_status. */
int msa_check_bounded_wait(int64_t limit_ns, int arrive, msa_stream_t stream);

/* Chunk offsets of the bank -- [DEEP] §"三、文档如何变成 memory",
 * "2. chunk 压缩": every `chunk` (64) tokens of a document form one chunk and
 * a trailing partial chunk is kept (180 tokens -> 3 chunks).
 *   tok_offsets   [n_docs+1] int64, device: document d owns token rows
 *                 [tok_offsets[d], tok_offsets[d+1]).
 *   chunk_offsets [n_docs+1] int64, device, written: exclusive prefix sum of
 *                 ceil(len_d / chunk); document d owns chunk rows
 *                 [chunk_offsets[d], chunk_offsets[d+1]).
 * An empty document (len <= 0) gets no chunk and records
 * MSA_ERR_INVALID_ARG in the device status word.  1 <= chunk <= 64. */
int msa_chunk_offsets(int n_docs, const int64_t* tok_offsets, int chunk,
                      int64_t* chunk_offsets, msa_stream_t stream);

/* Memory encoding -- [HYSEN] §"Document-wise RoPE resets every document to
 * position zero" and §"Memory must be encoded offline before a query can
 * reach it"; [DEEP] "2. chunk 压缩".
 *   k_tok, v_tok, kr_tok   [L][n_tok][H][D] (dt): token-level K, V, K_r of
 *                          L routed layers, laid out contiguously.
 *   tok_offsets, chunk_offsets  [n_docs+1] int64 (device), as above;
 *                          n_chunks = chunk_offsets[n_docs].
 *   k_bar, v_bar, kr_bar   [L][n_chunks][H][D] (dt), written.
 * K row t of document d is rotated to position t - tok_offsets[d] (RoPE,
 * pairs (i, i+D/2), inverse frequency rope_base^(-2i/D)); K, V and K_r are
 * then averaged over each chunk's tokens (fp32 sums, one rounding to dt).
 * Supported: D in {64,128}, 1 <= H <= 16, 1 <= chunk <= 64. */
int msa_encode_pool(msa_dtype dt, int L, int64_t n_tok, int n_docs, int H,
                    int D, const void* k_tok, const void* v_tok,
                    const void* kr_tok, const int64_t* tok_offsets,
                    const int64_t* chunk_offsets, int64_t n_chunks,
                    float rope_base, int chunk, void* k_bar, void* v_bar,
                    void* kr_bar, msa_stream_t stream);

/* Memory encoding that also writes the prepared routing bank -- [HYSEN]
 * §"Memory must be encoded offline before a query can reach it": the routing
 * keys' per-row normalisation depends on the bank alone, so it is done in
 * the same pass that pools them.  As msa_encode_pool (same arguments,
 * layouts and limits), plus:
 *   kr_hat  [L][n_chunks][H][D] bf16, written: each (chunk, head) row of
 *           K̄_r (as rounded to bf16) divided by max(|row|, 1e-12) and
 *           rounded to bf16 -- byte for byte what msa_route_prepare_bank
 *           writes from K̄_r, ready for msa_route_scores_prepared;
 *   kr_bar  may be NULL: then only the prepared bank is kept, so building
 *           the memory takes one pass and one routing bank (the raw K̄_r is
 *           needed only by msa_route_backward).
 * bf16 only (MSA_ERR_UNSUPPORTED otherwise); always runs the bulk-copy
 * pooling kernel, whatever MSA_ENCODE_TMA says.  kr_hat may not alias any
 * other argument. */
int msa_encode_pool_prepared(msa_dtype dt, int L, int64_t n_tok, int n_docs, int H,
                             int D, const void* k_tok, const void* v_tok,
                             const void* kr_tok, const int64_t* tok_offsets,
                             const int64_t* chunk_offsets, int64_t n_chunks,
                             float rope_base, int chunk, void* k_bar, void* v_bar,
                             void* kr_bar, void* kr_hat, msa_stream_t stream);

/* Routing -- [HYSEN] §"Routing happens inside attention ...": relevance is
 * the cosine similarity of Q_r and K̄_r, averaged over heads, then the
 * maximum over query tokens; [DEEP] §"五、推理阶段" Step 2.  A document's
 * score is the maximum over its chunks (the pages leave this aggregation
 * open).
 *   q_r          [B][T][H][D] (dt): routing queries, B independent queries
 *                of T tokens.
 *   kr_bar       [n_chunks][H][D] (dt): one layer of the pooled bank.
 *   chunk_offsets [n_docs+1] int64 (device).
 *   doc_scores   [B][n_docs] float, written (-inf for an empty document).
 *   chunk_scores [B][n_chunks] float, written when not NULL.
 *   ws           workspace of >= msa_route_workspace_size(...) bytes.
 * cos(q,k) = q.k / (max(|q|,1e-12) max(|k|,1e-12)).  MSA_BF16 runs the
 * contraction on the tcgen05 tensor cores (bf16 operands, fp32 accumulate);
 * MSA_F32 runs it on the CUDA cores in fp32.
 * Supported: D in {64,128}, 1 <= H <= 8 (bf16) or 16 (fp32), B*T >= 1. */
size_t msa_route_workspace_size(msa_dtype dt, int B, int T, int H, int D);
int msa_route_scores(msa_dtype dt, int B, int T, int H, int D,
                     const void* q_r, const void* kr_bar, int64_t n_chunks,
                     const int64_t* chunk_offsets, int n_docs,
                     float* doc_scores, float* chunk_scores, void* ws,
                     size_t ws_bytes, msa_stream_t stream);

/* Routing over a prepared bank.  The per-row normalisation of K̄_r depends
 * only on the bank, so it can be done once when the bank is built (the
 * pages encode the memory offline, [HYSEN] §"Memory must be encoded offline
 * before a query can reach it") instead of on every query:
 *   msa_route_prepare_bank writes kr_hat[c][h] = K̄_r[c][h] /
 *     max(|K̄_r[c][h]|, 1e-12), rounded to bf16 ([n_chunks][H][D], may not
 *     alias kr_bar);
 *   msa_route_scores_prepared takes kr_hat in place of kr_bar and returns
 *     the same scores as msa_route_scores (identical rounding: the raw scan
 *     normalises the rows the same way in shared memory).
 * bf16 only (MSA_ERR_UNSUPPORTED otherwise).  Same workspace, layouts and
 * errors as msa_route_scores. */
int msa_route_prepare_bank(msa_dtype dt, int64_t n_chunks, int H, int D,
                           const void* kr_bar, void* kr_hat, msa_stream_t stream);
int msa_route_scores_prepared(msa_dtype dt, int B, int T, int H, int D,
                              const void* q_r, const void* kr_hat,
                              int64_t n_chunks, const int64_t* chunk_offsets,
                              int n_docs, float* doc_scores,
                              float* chunk_scores, void* ws, size_t ws_bytes,
                              msa_stream_t stream);

/* Routing without any device allocation.  The paper has no counterpart: this
 * is a deployment variant of msa_route_scores for callers that cannot call
 * cudaMalloc -- an engine whose device memory is all owned by its own pool
 * allocator, or a latency-critical loop where an allocation (which may
 * synchronise the device) is not acceptable.  It computes exactly what
 * msa_route_scores computes, with the same arguments minus the workspace:
 * the scratch is a fixed array of msa_route_noalloc_scratch_bytes() bytes
 * (512 KiB) compiled into the library, one per device, held by every GPU
 * that loads the library until the process exits.  The caller still owns
 * and passes every input and output.
 *   - A shape whose workspace (msa_route_workspace_size) exceeds the array
 *     -- e.g. more than 256 query columns at 8 x 128 in bf16 -- returns
 *     MSA_ERR_WORKSPACE before anything is launched.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture begins.
 *   - All calls on a device share the array: calls that overlap on the GPU
 *     race on it and must be ordered (one stream, or events).  Each call
 *     rewrites every byte it reads, so nothing carries over between calls. */
size_t msa_route_noalloc_scratch_bytes(void);
int msa_route_scores_noalloc(msa_dtype dt, int B, int T, int H, int D,
                             const void* q_r, const void* kr_bar,
                             int64_t n_chunks, const int64_t* chunk_offsets,
                             int n_docs, float* doc_scores, float* chunk_scores,
                             msa_stream_t stream);

/* Top-k documents -- [HYSEN] §"Routing happens inside attention ...": the
 * router selects the top-k documents.  Ties go to the lower document index.
 *   scores      [B][n_docs] float (device).
 *   idx         [B][k] int32, written, in rank order (best first).
 *   top_scores  [B][k] float, written when not NULL.
 * NaN scores rank below every number.  1 <= k <= min(n_docs, 1024). */
size_t msa_topk_workspace_size(int B, int n_docs, int k);
int msa_topk_docs(int B, int n_docs, int k, const float* scores,
                  int32_t* idx, float* top_scores, void* ws, size_t ws_bytes,
                  msa_stream_t stream);

/* Memory Parallel merge -- [HYSEN] §"The 100M-token setup depends on host
 * memory as well as two GPUs": the routing keys are split across GPUs, each
 * scores the query against its part, and the partial results are reduced
 * into one selection.  A shard is a contiguous document range; shard r's
 * local top-k (msa_topk_docs over its own documents) has been all-gathered.
 *   cand_scores [world][B][k] float (device), shard r's scores in rank order.
 *   cand_idx    [world][B][k] int32 (device), the matching shard-local ids.
 *   doc_base    [world] int32 (device): global id of shard r's document 0;
 *               shards hold disjoint, increasing document ranges.
 *   idx         [B][k] int32, written: the global top-k ids in rank order.
 *   top_scores  [B][k] float, written when not NULL.
 * Same order as msa_topk_docs: score descending, lower global id first,
 * NaN last, -0 == +0.  Candidate ids must be distinct (they are, when each
 * shard returns each of its documents at most once).  world * k <= 4096,
 * else MSA_ERR_UNSUPPORTED; a global id outside int32 records
 * MSA_ERR_INVALID_ARG in the device status word. */
int msa_topk_merge_shards(int B, int world, int k, const float* cand_scores,
                          const int32_t* cand_idx, const int32_t* doc_base,
                          int32_t* idx, float* top_scores, msa_stream_t stream);

/* Context assembly -- [HYSEN] §"Memory must be encoded offline ...": only
 * the selected documents' K/V are loaded and joined with the local context.
 *   idx          [B][k] int32 (device), document ids in rank order.
 *   k_bar, v_bar [n_chunks][H][D] (dt), one layer of the pooled bank.
 *   k_mem, v_mem [B][m_cap][H][D] (dt), written: rows 0..mem_len[b]-1 are
 *                the chunk rows of idx[b][0], idx[b][1], ... concatenated.
 *   mem_len      [B] int32, written: min(total rows, m_cap).
 * If a query's rows exceed m_cap, rows past m_cap are dropped and
 * MSA_ERR_CAPACITY is recorded in the device status word.  An index outside
 * [0, n_docs) contributes no rows and records MSA_ERR_INVALID_ARG there.
 * Tiered storage -- [HYSEN] §"The 100M-token setup depends on host memory as
 * well as two GPUs" and [WIKI] §6 (routing keys on the GPU, content K/V in
 * host memory): k_bar and v_bar may instead point into pinned host memory
 * that is mapped into the device's address space (cudaHostAlloc, or
 * cudaHostRegister with mapping; the unified address is passed).  The same
 * kernel then reads only the selected rows over the host link; idx,
 * chunk_offsets and the outputs stay in device memory. */
int msa_gather_kv(msa_dtype dt, int B, int k, int H, int D,
                  const int32_t* idx, const int64_t* chunk_offsets,
                  int n_docs, const void* k_bar, const void* v_bar,
                  int m_cap, void* k_mem, void* v_mem, int32_t* mem_len,
                  msa_stream_t stream);

/* Sparse attention, prefill (T > 1) and decode (T = 1) -- [HYSEN]
 * §"Routing happens inside attention ..." (the selected compressed K/V are
 * concatenated with the query's local K/V) and §"Document-wise RoPE ..."
 * (global RoPE: the query's start index is offset by k).
 *   q            [B][T][Hq][D] (dt): the last T of the T_loc local tokens.
 *   k_mem, v_mem [B][m_cap][H][D] (dt) with mem_len [B] int32 (device):
 *                memory rows, used as stored (they keep their
 *                document-wise rotation).
 *   k_loc, v_loc [B][T_loc][H][D] (dt): local context, unrotated.
 *   out          [B][T][Hq][D] (dt), written.
 * Local key j is rotated to position pos0 + j, query token i to
 * pos0 + T_loc - T + i; query i sees every memory row and local keys
 * j <= T_loc - T + i.  Query head h reads KV head floor(h*H/Hq).  scale <= 0
 * selects 1/sqrt(D).  Softmax and accumulation in fp32.
 * Supported: D in {64,128}, Hq % H == 0, Hq/H <= 16, 1 <= T <= T_loc. */
size_t msa_sparse_attn_workspace_size(msa_dtype dt, int B, int T, int T_loc,
                                      int Hq, int H, int D, int m_cap);
int msa_sparse_attn(msa_dtype dt, int B, int T, int T_loc, int Hq, int H,
                    int D, const void* q, const void* k_mem,
                    const void* v_mem, const int32_t* mem_len, int m_cap,
                    const void* k_loc, const void* v_loc, int pos0,
                    float rope_base, float scale, void* out, void* ws,
                    size_t ws_bytes, msa_stream_t stream);

/* Backward of the routing score -- "深度分析MSA" §"四、训练阶段：学习 memory
 * 与路由": the routing auxiliary loss (BCE or InfoNCE on the document
 * scores) trains Q_r and K_r.  Given dL/d(doc_scores) it ADDS to the
 * caller's (zeroed) gradient buffers:
 *   d_doc    [B][n_docs] float (device): dL/d(doc score); zero entries cost
 *            nothing.
 *   dq_r     [B][T][H][D] float, accumulated.
 *   dkr_bar  [n_chunks][H][D] float, accumulated (gradient of the raw,
 *            unnormalised pooled routing keys).
 *   q_r, kr_bar, chunk_offsets: as msa_route_scores (dt f32 or bf16).
 * A document's score is that of its best (chunk, query token) pair; the
 * gradient goes to the first maximiser (lowest chunk, then lowest token) and
 * is computed in fp32 from q_r and kr_bar.
 * bf16 with D in {64,128}, H <= 8 and n_chunks * T < 2^32: the maximisers are
 * found by one tensor-core scan of the bank (as msa_route_scores, the
 * cosines of bf16 unit rows summed in fp32; pairs whose best two cosines lie
 * within that rounding may take either) and the gradient kernel visits only
 * pairs with a non-zero gradient; ws must hold
 * msa_route_backward_workspace_size() bytes (16-byte aligned) or the call
 * returns MSA_ERR_WORKSPACE.  Otherwise (fp32, or MSA_ROUTE_BWD_TC=0 in the
 * environment) the maximisers are recomputed in fp32 on the CUDA cores, one
 * pass over the document's chunks and the query's tokens per pair with a
 * non-zero gradient, and ws is unused (workspace size 0).
 * Supported: D in {64,128}, H <= 16, H*D <= 1024. */
size_t msa_route_backward_workspace_size(msa_dtype dt, int B, int T, int H, int D,
                                         int64_t n_chunks, int n_docs);
int msa_route_backward(msa_dtype dt, int B, int T, int H, int D, const void* q_r,
                       const void* kr_bar, int64_t n_chunks, const int64_t* chunk_offsets,
                       int n_docs, const float* d_doc, float* dq_r, float* dkr_bar,
                       void* ws, size_t ws_bytes, msa_stream_t stream);

/* Backward of the memory encoding (chunk pooling with document-wise RoPE on
 * K) -- the same training step: the gradient of the pooled bank reaches the
 * token tensors.  All float:
 *   dk_bar, dv_bar, dkr_bar  [L][n_chunks][H][D] (device).
 *   dk_tok, dv_tok, dkr_tok  [L][n_tok][H][D], written.
 * Each token gets its chunk's gradient / (tokens in the chunk); K's is
 * rotated back by the token's document-wise position.  D in {64,128}. */
int msa_encode_pool_backward(int L, int64_t n_tok, int n_docs, int H, int D,
                             const float* dk_bar, const float* dv_bar, const float* dkr_bar,
                             const int64_t* tok_offsets, const int64_t* chunk_offsets,
                             int64_t n_chunks, float rope_base, float* dk_tok, float* dv_tok,
                             float* dkr_tok, msa_stream_t stream);

/* Fused context assembly + sparse attention -- [HYSEN] §"Memory must be
 * encoded offline ..." (only the selected documents' K/V are loaded and
 * joined with the local context) and §"Routing happens inside attention
 * ...": the same attention as msa_gather_kv followed by msa_sparse_attn,
 * reading the selected documents' pooled rows straight from the bank (no
 * gathered copy).
 *   idx          [B][k] int32 (device): document ids in rank order.
 *   chunk_offsets[n_docs+1] int64 (device); k_bar, v_bar [n_chunks][H][D]
 *                (dt): one layer of the bank (device or pinned, mapped host
 *                memory).
 *   m_cap        upper bound of a query's memory rows (sizes the workspace;
 *                rows past it are dropped and MSA_ERR_CAPACITY is recorded).
 *   mem_len      [B] int32, written when not NULL: memory rows used.
 *   q, k_loc, v_loc, pos0, rope_base, scale, out: as msa_sparse_attn.
 * Each document's rows are read in 8-row groups; the rows of its last group
 * past its end are other bank rows, masked out of the softmax and with their
 * V zeroed, so whatever they hold (NaN included) does not reach the output.
 * Supported (else MSA_ERR_UNSUPPORTED): bf16, D = 128, Hq/H in
 * {1,2,4,8,16}, 1 <= k <= min(n_docs, 1024), n_chunks < 2^31, and either
 *   T = 1 (decode, on the tensor-core decode kernel), or
 *   2 <= T <= T_loc (prefill, on the tensor-core prefill kernel), with
 *   B <= 65535 and B*T, B*T_loc and B*8*(ceil(m_cap/8) + k) each <= 2^30
 *   (a query's memory is padded to whole 8-row groups per document).
 * The workspace size is 0 for unsupported shapes. */
size_t msa_sparse_attn_fused_workspace_size(msa_dtype dt, int B, int T, int T_loc, int Hq,
                                            int H, int D, int k, int m_cap);
int msa_sparse_attn_fused(msa_dtype dt, int B, int T, int T_loc, int Hq, int H, int D,
                          const void* q, const int32_t* idx, int k,
                          const int64_t* chunk_offsets, int n_docs, const void* k_bar,
                          const void* v_bar, int64_t n_chunks, int m_cap, const void* k_loc,
                          const void* v_loc, int pos0, float rope_base, float scale,
                          void* out, int32_t* mem_len, void* ws, size_t ws_bytes,
                          msa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */
