/*
 * dsa.h — C ABI of the B200 (sm_100a) DSA sparse-attention layer.
 *
 * The layer replaces full-attention MLA in 24 of the 93 layers of
 * Kimi-K3.1-Pro (llama.cpp b12180 news: aiaulis.com paragraphs 2-3;
 * aiunderstanding.org "What happened"; devotd.net section 1 and its
 * configuration table).  It runs in three steps:
 *
 *   1. a lightning indexer of 32 heads x 128 dims, no RoPE, scores every
 *      earlier cached token of each query:
 *        I[q,s] = sum_h w[q,h] * ReLU( q_idx[q,h,:] . k_idx[s,:] ),  s <= p(q)
 *      (the pages name the scorer but print no formula; this is the usual
 *      lightning-indexer form and is an assumption of this library);
 *   2. the top_k highest-scoring positions are kept (top_k = 2048 in the
 *      released checkpoint), ties broken by lower position;
 *   3. attention runs only over the kept rows of a shared key-only latent
 *      cache: K = the whole 576-wide row, V = its first 512 entries
 *      (devotd.net section 2: a key-only cache per DSA layer).
 *
 * With top_k >= p+1 for every query the result is full causal attention
 * (aiaulis.com paragraph 7; devotd.net section 4).
 *
 * Conventions for every call
 * --------------------------
 *  - Numbers: bf16 tensors are passed as uint16_t bit patterns; scores,
 *    weights, outputs are IEEE fp32.  Products are exact, accumulation is
 *    fp32, softmax runs in fp32.
 *  - Memory: every tensor pointer is a DEVICE pointer owned by the caller,
 *    except the h_* fields of dsa_batch, which are HOST mirrors used to plan
 *    the launch without a device sync.  The library allocates nothing, keeps
 *    no state between calls and is re-entrant; calls on different streams
 *    must use different workspaces.  The one exception is
 *    dsa_sparse_attn_noalloc, which keeps its scratch in a static device
 *    array shared by all of its calls (see its declaration: calls of it
 *    that may overlap on the GPU must be serialised).  A workspace must be
 *    zero-filled (e.g. cudaMemset) before its first use: its first 256
 *    bytes are a control block holding the kernels' error word, which calls
 *    leave zero unless a kernel-side failure sets it, and
 *    dsa_check_device_status clears.
 *  - Asynchrony: all work is enqueued on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  Nothing synchronises except
 *    dsa_check_device_status.
 *  - Errors: every call validates all arguments before it launches anything;
 *    on any error it returns a non-OK status and writes nothing.  No C++
 *    exception crosses this boundary.  Kernel-side failures (a bounded wait
 *    that ran out, an index entry outside 0..p) set an error word in the
 *    workspace, read back and cleared by dsa_check_device_status.  The error
 *    word is sticky: while it is set, the kernels of later calls on the same
 *    workspace skip their work, and the outputs of the failing call and of
 *    those later calls are undefined.
 *  - Alignment: every tensor pointer must be 16-byte aligned.
 *  - Fixed shapes: indexer 32 heads x 128, latent row 576, value width 512,
 *    1 <= top_k <= 2048, 1 <= H <= 128.  Other values give
 *    DSA_ERR_UNSUPPORTED.
 */
#ifndef DSA_B200_H_
#define DSA_B200_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_INDEX_HEADS 32   /* indexer heads (devotd.net configuration table) */
#define DSA_INDEX_DIM 128    /* indexer key length (same table) */
#define DSA_LATENT_DIM 576   /* latent key row width */
#define DSA_VALUE_DIM 512    /* V = first 512 entries of the latent row */
#define DSA_MAX_TOPK 2048    /* keys kept per query (same table) */
#define DSA_MAX_HEADS 128    /* attention heads per query */

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,    /* null pointer, bad size, inconsistent batch */
  DSA_ERR_UNSUPPORTED = 2,    /* shape outside the fixed set, misaligned pointer */
  DSA_ERR_WORKSPACE = 3,      /* ws NULL or smaller than the call needs */
  DSA_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed */
  DSA_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait ran out (device side) */
  DSA_ERR_NOT_SM100 = 6,      /* current device is not compute capability 10.0 */
  DSA_ERR_BAD_INDEX = 7       /* an index entry outside -1..p was skipped (device side) */
} dsa_status;

/* Flags (bitwise OR); every bit not listed here is reserved and must be 0. */
/* dsa_indexer_score and dsa_topk: build, then use, the per-row histogram of
 * the scores that the fused layer builds (see those calls). */
#define DSA_FLAG_SCORE_HISTOGRAM 0x1u
/* dsa_layer_forward, for tests of the timeout path only: the indexer's TMA
 * producer issues no load, so every wait of the indexer runs out after its
 * time limit (about a second); the call then leaves DSA_ERR_DEVICE_TIMEOUT in
 * the workspace, and its outputs are undefined. */
#define DSA_FLAG_TEST_STALL 0x80000000u
/* dsa_workspace_size: the size also covers dsa_masked_attn on the batch. */
#define DSA_FLAG_MASKED_ROUTE 0x2u

/*
 * A batch of sequences.  Sequence b owns
 *   - query rows [q_offsets[b], q_offsets[b+1]) of every per-query tensor
 *     (nq_b = q_offsets[b+1] - q_offsets[b] >= 0, q_offsets[0] = 0,
 *     q_offsets[B] = Nq);
 *   - positions 0..ctx_lens[b]-1 of the caches k_idx and kv (the two caches
 *     share row numbering), with nq_b <= ctx_lens[b].
 * Where position s of sequence b lives:
 *   - contiguous caches (page_size = 0): row kv_offsets[b] + s, inside
 *     [kv_offsets[b], kv_offsets[b+1]), so ctx_lens[b] <= kv_offsets[b+1] -
 *     kv_offsets[b];
 *   - paged caches (page_size > 0, a power of two >= 64): row
 *     block_table[b * max_blocks + s / page_size] * page_size
 *     + s % page_size; every listed page is < cache_rows / page_size and
 *     ctx_lens[b] <= max_blocks * page_size; kv_offsets is not used (may be
 *     NULL).
 * The current tokens are already appended to the caches: the j-th query of
 * sequence b sits at position p = ctx_lens[b] - nq_b + j and sees positions
 * 0..p, its own included (decode: nq_b = 1, p = L-1; prefill: nq_b = L).
 * The device arrays and their host mirrors must hold the same values.
 */
typedef struct {
  int32_t B;                    /* sequences, >= 0 */
  int32_t Nq;                   /* total query rows = q_offsets[B] */
  const int32_t* q_offsets;     /* device, [B+1] */
  const int64_t* kv_offsets;    /* device, [B+1] */
  const int32_t* ctx_lens;      /* device, [B] */
  const int32_t* h_q_offsets;   /* host mirror, [B+1] */
  const int64_t* h_kv_offsets;  /* host mirror, [B+1] */
  const int32_t* h_ctx_lens;    /* host mirror, [B] */
  /* paged caches (all zero / NULL for contiguous caches) */
  int32_t page_size;            /* 0, or rows per page: a power of two >= 64 */
  int32_t max_blocks;           /* block-table entries per sequence */
  const int32_t* block_table;   /* device, [B][max_blocks] page numbers */
  const int32_t* h_block_table; /* host mirror */
  int64_t cache_rows;           /* rows of k_idx and kv (paged caches) */
} dsa_batch;

/* Bytes of workspace that dsa_layer_forward needs for this batch; it is also
 * enough for every other call on the same batch, H and top_k (with
 * DSA_FLAG_MASKED_ROUTE in `flags`, for dsa_masked_attn too; otherwise pass
 * 0).  Returns 0 for an invalid batch or flag. */
DSA_API size_t dsa_workspace_size(const dsa_batch* batch, int H, int top_k, uint32_t flags);

/*
 * Step 1, the lightning indexer (aiaulis.com paragraph 2: a light indexer
 * scores earlier tokens; devotd.net configuration table: 32 heads, key
 * length 128; aiunderstanding.org "What happened": no RoPE).
 *   q_idx   [Nq, 32, 128] bf16   indexer queries (no rotary embedding applied)
 *   w       [Nq, 32]      fp32   per-query head weights
 *   k_idx   [rows, 128]   bf16   indexer key cache
 *   scores  [Nq, ld_scores] fp32 out: scores[r, s] for s = 0..p(r);
 *                                entries past p(r) are left untouched.
 *   ld_scores >= max_b ctx_lens[b], a multiple of 4.
 *   ws      workspace: at least 256 bytes; with DSA_FLAG_SCORE_HISTOGRAM, at
 *           least dsa_workspace_size(batch, 1, 1, 0) bytes.
 *   flags   0, or DSA_FLAG_SCORE_HISTOGRAM: also count every score of each
 *           row into a 4096-bin histogram of its top 12 order-preserving key
 *           bits, kept in the workspace for a following dsa_topk with the
 *           same flag (as the fused layer does for decode).
 * Runs on tcgen05 tensor cores (bf16 products, fp32 accumulation).
 */
DSA_API dsa_status dsa_indexer_score(const dsa_batch* batch, const uint16_t* q_idx, const float* w,
                             const uint16_t* k_idx, float* scores, int64_t ld_scores, void* ws,
                             size_t ws_bytes, uint32_t flags, void* stream);

/*
 * Step 2, top-k selection (aiaulis.com paragraphs 2-3: attention only for the
 * highest-scored tokens, 2048 of them; devotd.net configuration table).
 *   scores [Nq, ld_scores] fp32, read for s = 0..p(r) only.
 *   idx    [Nq, top_k] int32 out: the n = min(top_k, p+1) positions with the
 *          largest (score, -position), i.e. score descending with ties to the
 *          lower position, written in ascending position order, followed by
 *          top_k - n entries of -1.  Positions are sequence-relative.
 *   -0.0 and +0.0 are the same score.  NaN scores are not supported.
 *   ws     workspace: at least 256 bytes; with DSA_FLAG_SCORE_HISTOGRAM, at
 *          least dsa_workspace_size(batch, 1, top_k, 0) bytes.
 *   flags  0, or DSA_FLAG_SCORE_HISTOGRAM: the histograms that the preceding
 *          dsa_indexer_score call with that flag left in this workspace, for
 *          these same scores, drive the selection (one filtering pass over
 *          each row) wherever few long rows make that path pay; the result
 *          is the same either way.
 */
DSA_API dsa_status dsa_topk(const dsa_batch* batch, const float* scores, int64_t ld_scores, int top_k,
                    int32_t* idx, void* ws, size_t ws_bytes, uint32_t flags, void* stream);

/*
 * Step 3, attention over the selected rows only (aiaulis.com paragraph 2;
 * devotd.net section 2: the key-only cache serves as both K and V).
 *   q    [Nq, H, 576] bf16     attention queries
 *   kv   [rows, 576]  bf16     shared latent cache; V = first 512 entries
 *   idx  [Nq, top_k]  int32    sequence-relative positions, -1 = unused slot;
 *                              every other entry must satisfy 0 <= idx <= p(r):
 *                              an entry outside -1..p(r) is checked on the
 *                              device, skipped (no memory is read for it) and
 *                              reported as DSA_ERR_BAD_INDEX by
 *                              dsa_check_device_status
 *   out  [Nq, H, 512] fp32     out: softmax_s(scale * q.kv[s]) weighted sum of
 *                              kv[s, :512] over the listed s
 *   lse  [Nq, H] fp32 or NULL  out: natural-log log-sum-exp of the logits
 *   A row whose idx holds no valid entry gets out = 0 and lse = -inf.
 */
DSA_API dsa_status dsa_sparse_attn(const dsa_batch* batch, const uint16_t* q, int H, const uint16_t* kv,
                           const int32_t* idx, int top_k, float scale, float* out, float* lse,
                           void* ws, size_t ws_bytes, void* stream);

/*
 * Step 3 the way the pages describe llama.cpp doing it, kept as a measured
 * comparison (aiaulis.com paragraph 4; devotd.net section 2: the selection
 * is applied as a mask over the whole cache so that the existing sparse
 * flash attention can be reused; off that path the cost is full-cache
 * attention).  Same arguments, result and error rules as dsa_sparse_attn
 * (results agree within the library's tolerances), but it reads every cached
 * row 0..p of each query and masks the logits of the rows idx does not list,
 * instead of gathering only the listed rows.  Needs the workspace size that
 * dsa_workspace_size reports with DSA_FLAG_MASKED_ROUTE; contexts up to 2^21.
 */
DSA_API dsa_status dsa_masked_attn(const dsa_batch* batch, const uint16_t* q, int H,
                                   const uint16_t* kv, const int32_t* idx, int top_k, float scale,
                                   float* out, float* lse, void* ws, size_t ws_bytes,
                                   void* stream);

/*
 * The whole DSA layer: dsa_indexer_score -> dsa_topk -> dsa_sparse_attn,
 * with the scores kept in the workspace.  Arguments as above; `idx` receives
 * the selected index sets, `out`/`lse` the attention output.  `flags` is 0
 * (or DSA_FLAG_TEST_STALL, in tests of the timeout path only).
 */
DSA_API dsa_status dsa_layer_forward(const dsa_batch* batch, const uint16_t* q, int H,
                             const uint16_t* q_idx, const float* w, const uint16_t* k_idx,
                             const uint16_t* kv, int top_k, float scale, float* out, float* lse,
                             int32_t* idx, void* ws, size_t ws_bytes, uint32_t flags,
                             void* stream);

/*
 * The indexer's input step for the new tokens of a batch (aiunderstanding.org
 * "What happened": the indexer's q_b, k and projection tensors are kept out
 * of quantization; devotd.net section 2: a DSA layer keeps an indexer key
 * cache).  The pages give no widths and no normalisation; the three maps are
 * taken as plain linear maps.  For every query row t (the j-th new token of
 * sequence b, at position p = ctx_lens[b] - nq_b + j):
 *   q_idx[t] = c_q[t] . w_q_b^T     [Nq, 32, 128] bf16 out
 *   k        = x[t]   . w_k^T       written to k_idx row kv_offsets[b] + p (bf16)
 *   w[t]     = x[t]   . w_proj^T    [Nq, 32] fp32 out
 * Inputs, bf16: x [Nq, d_model] (hidden states), c_q [Nq, d_q] (query
 * latents); weights [out, in]: w_q_b [4096, d_q], w_k [128, d_model],
 * w_proj [32, d_model].  d_model and d_q are multiples of 64 in [64, 65536].
 * Rows of k_idx other than the new tokens' are not touched.  Products are
 * exact, sums fp32, outputs rounded to bf16 (to nearest even) except w.
 * Runs as one tcgen05 GEMM; the workspace holds split-K partials
 * (dsa_indexer_project_workspace_size bytes, zero-filled before first use
 * like every workspace).
 */
DSA_API size_t dsa_indexer_project_workspace_size(const dsa_batch* batch, int64_t d_model,
                                                  int64_t d_q);
DSA_API dsa_status dsa_indexer_project(const dsa_batch* batch, const uint16_t* x, int64_t d_model,
                                       const uint16_t* c_q, int64_t d_q, const uint16_t* w_q_b,
                                       const uint16_t* w_k, const uint16_t* w_proj,
                                       uint16_t* q_idx, uint16_t* k_idx, float* w, void* ws,
                                       size_t ws_bytes, void* stream);

/*
 * dsa_sparse_attn without a workspace, for callers that cannot allocate
 * device memory when they run the layer (a fixed pre-sized memory pool, a
 * runtime that hands kernels only the tensors it owns, a plugin host that
 * forbids allocation after start-up).  There is no counterpart on the source
 * pages: this is a deployment convenience of this library.
 *
 * Arguments, results and errors are those of dsa_sparse_attn, minus ws and
 * ws_bytes.  Its scratch (the partial results of a query's selected set split
 * over CTAs) lives in one static device array of 10 MiB that every GPU
 * holding this library keeps until process exit; a launch needing more
 * returns DSA_ERR_WORKSPACE and runs nothing (no shape within the fixed limits
 * needs more than about 9.3 MiB).  It allocates nothing and calls no
 * allocating routine.  The first call on each device looks up the array's
 * address, which under lazy module loading (the CUDA 12 default) also loads
 * the module and commits the array's memory: make that first call at
 * start-up, before device memory fills up and before capturing a stream into
 * a CUDA graph (a failed lookup returns DSA_ERR_CUDA).  Calls share
 * the array: calls that may overlap on the GPU (different streams) race and
 * must be serialised by the caller.  It always runs the CUDA-core attention
 * kernels, so results agree with dsa_sparse_attn within the library's
 * tolerances (not bit for bit).  Index entries outside -1..p(r) are skipped
 * as in dsa_sparse_attn, but with no workspace there is no error word to
 * report them in.
 */
DSA_API dsa_status dsa_sparse_attn_noalloc(const dsa_batch* batch, const uint16_t* q, int H,
                                           const uint16_t* kv, const int32_t* idx, int top_k,
                                           float scale, float* out, float* lse, void* stream);

/* Synchronises `stream`, then reads and clears the device error word that the
 * kernels of earlier calls on this workspace may have set.  Returns DSA_OK,
 * DSA_ERR_DEVICE_TIMEOUT (a bounded wait ran out; takes precedence),
 * DSA_ERR_BAD_INDEX (an index entry outside -1..p was skipped), or
 * DSA_ERR_CUDA if the stream itself reports an error. */
DSA_API dsa_status dsa_check_device_status(void* ws, size_t ws_bytes, void* stream);

/* Static, human-readable name of a status code. */
DSA_API const char* dsa_status_string(dsa_status status);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_H_ */
