/*
 * dsa.h -- C ABI of the DeepSeek Sparse Attention (DSA) hot path on one NVIDIA B200 (sm_100a).
 *
 * The method (pages "How GLM5.3 Sparse Attention Affects HBM Memory Usage" and its Chinese
 * original on InferenceX, sections "Lightning Indexer", "Sparse MLA", "MLA Modifications"):
 *   1. a lightning indexer scores every visible KV position s for each query token t,
 *        I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:])       (multi-head query, one-head key);
 *   2. the K highest-scoring positions are selected per query (shared by all attention heads);
 *      a query that sees fewer than K positions keeps all of them (dense attention);
 *   3. MLA runs in MQA ("absorbed") mode over only the selected rows of the latent KV cache:
 *      each row is a 512-d latent plus a 64-d RoPE key; the full row is the key, its first
 *      d_v dims are the value; all heads share the rows.
 *
 * Conventions shared by every entry point
 *   - Ownership: the caller owns and allocates every buffer (device memory unless stated).
 *     The library never allocates device memory; scratch is passed in by the caller.
 *   - Asynchrony: every compute call only enqueues kernels on `stream` (a cudaStream_t, NULL for
 *     the legacy default stream) and returns; there is no host synchronisation inside a call,
 *     except in dsa_get_device_error, which is documented as synchronous.
 *   - Positions: query t belongs to request q_req[t] and sits at absolute position q_pos[t];
 *     it sees positions 0..q_pos[t] of its request (causal, including itself).  Selected
 *     indices are logical positions within the request; only kernels that read a paged cache
 *     apply the block table: row = block_table[req][pos / block_size] * block_size
 *     + pos % block_size.
 *   - Errors: shapes, dtypes, alignment and NULL pointers are checked on the host before
 *     anything is launched (DSA_ERR_INVALID_ARG); valid but unimplemented combinations return
 *     DSA_ERR_UNSUPPORTED; a failed launch returns DSA_ERR_CUDA.  Faults that only the device
 *     can see (a block id outside the pool, a selected index outside 0..q_pos, a request id
 *     outside the batch, a NaN score, a bounded wait that ran out) never trap: the kernel sets
 *     a bit in the library's device error word (DSA_DEVERR_*), skips the offending element,
 *     and the host reads the word with dsa_get_device_error.
 *   - Tensor cores: production shapes (indexer 64 heads x 128, MLA 128 heads over 512 + 64,
 *     bf16 operands, e4m3 or bf16 indexer keys) run on tcgen05/TMA kernels; any other shape runs
 *     on a generic CUDA-core path of the same library.  There is no CPU fallback.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_ABI_VERSION 2

typedef enum dsa_status {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,
  DSA_ERR_UNSUPPORTED = 2,
  DSA_ERR_CUDA = 3,
  DSA_ERR_DEVICE_FAULT = 4
} dsa_status;

typedef enum dsa_dtype {
  DSA_F32 = 0,
  DSA_BF16 = 1,
  DSA_E4M3 = 2 /* OCP FP8 E4M3 ("fn": no infinities), used with a per-token f32 scale */
} dsa_dtype;

/* Bits of the device error word. */
#define DSA_DEVERR_BLOCK_ID 1      /* block_table entry outside [0, num_blocks) */
#define DSA_DEVERR_INDEX 2         /* selected index outside [-1, q_pos[t]] */
#define DSA_DEVERR_REQUEST 4       /* q_req[t] outside [0, num_reqs) or q_pos[t] >= max_context */
#define DSA_DEVERR_NAN_SCORE 8     /* NaN indexer score met by the selection */
#define DSA_DEVERR_TIMEOUT 16      /* a bounded wait inside a kernel gave up */
#define DSA_DEVERR_QUERY_GROUP 32  /* queries of one group are not in one request */

typedef void* dsa_stream; /* cudaStream_t */

/* A paged per-token cache: `data` is [num_blocks, block_size, dim] of `dtype`, row-major, in
 * device memory, 16-byte aligned, one token per row.  For DSA_E4M3, `scale` is the per-token
 * dequantisation scale [num_blocks, block_size] f32 (value = code * scale, scale > 0); it is
 * NULL for the other dtypes.  block_size is 64. */
typedef struct dsa_paged_cache {
  const void* data;
  const float* scale;
  int64_t num_blocks;
  int32_t block_size;
  int32_t dim;
  int32_t dtype; /* dsa_dtype */
  int32_t reserved;
} dsa_paged_cache;

/* The queries of one call.  q_req, q_pos and block_table are device int32 arrays:
 * q_req [num_queries], q_pos [num_queries], block_table [num_reqs, max_blocks].
 * max_context is a host-side bound: every q_pos[t] < max_context (it sizes score rows).
 * query_group G >= 1 is a host-side promise that queries come in runs of G consecutive t
 * (num_queries a multiple of G) sharing one request; a prefill chunk passes 4, decode passes 1.
 * It only selects kernels: a broken promise sets DSA_DEVERR_QUERY_GROUP. */
typedef struct dsa_batch {
  int32_t num_queries;
  int32_t num_reqs;
  const int32_t* q_req;
  const int32_t* q_pos;
  const int32_t* block_table;
  int32_t max_blocks;
  int32_t max_context;
  int32_t query_group;
  int32_t reserved;
} dsa_batch;

/*
 * Lightning-indexer scores (page "How GLM5.3 Sparse Attention Affects HBM Memory Usage",
 * section "Lightning Indexer": dot product, ReLU, weighted sum over the query heads; no value,
 * no softmax).
 *   scores[t * ld + s] = sum_h w[t,h] * max(0, sum_i q[t,h,i] * khat[s,i]),  0 <= s <= q_pos[t]
 *   khat = key row (f32/bf16), or e4m3 code * per-token scale.
 *   q[t,h,:] as stored (f32/bf16), or e4m3 code * q_scale[t,h].
 * q: device [num_queries, Hi, Di] of q_dtype (DSA_F32, DSA_BF16 or DSA_E4M3); q_scale: device f32
 * [num_queries, Hi] for DSA_E4M3 queries (per query and head), ignored otherwise; w: device
 * [num_queries, Hi] f32; keys: paged indexer-key cache with dim == Di, same block table as the
 * batch; scores: device f32 [num_queries, ld], ld >= max_context.  Entries s > q_pos[t] are not
 * written.  Tensor-core path: Hi == 64, Di == 128, and bf16 q with bf16 or e4m3 keys, or e4m3 q
 * with e4m3 keys; bf16 queries take any bf16 value (with e4m3 keys each head row is carried as
 * two e4m3 terms at a power-of-two scale, exact to bf16 precision for every element down to 2^-10
 * of the row's largest).  Other combinations run on the generic kernels.
 * key_hist: NULL, or device uint32 [num_queries, 4096] (16-byte aligned) to which the call adds,
 * per query, how many of its scores fall in each bin of the top 12 bits of the selection's
 * order key (the key dsa_topk_select compares: sign, exponent and three mantissa bits of the
 * score); dsa_topk_select takes it to place its threshold.  It is filled by the tensor-core
 * kernel for bf16 keys with query_group 1 and by the generic kernels; the other tensor-core
 * configurations leave it untouched.
 */
dsa_status dsa_indexer_scores(const void* q, int32_t q_dtype, const float* q_scale, int32_t Hi,
                              int32_t Di, const float* w, const dsa_paged_cache* keys,
                              const dsa_batch* batch, float* scores, int64_t ld,
                              uint32_t* key_hist, dsa_stream stream);

/*
 * Top-K selection (same page, section "Lightning Indexer": the K highest indexer scores are
 * kept per query and shared by all heads; a query seeing fewer than K positions keeps all).
 * For query t with n = q_pos[t] + 1 visible scores scores[t * ld + 0 .. n-1]:
 *   n <= k: idx[t] = 0, 1, ..., n-1, then -1;
 *   n >  k: the k positions first in the order (score descending, position ascending), written
 *           in ascending position order.
 * -0.0 and +0.0 are equal scores; a NaN score sets DSA_DEVERR_NAN_SCORE (it ranks lowest).
 * scores: device f32 [T, ld]; q_pos: device int32 [T] with q_pos[t] < ld (a larger value sets
 * DSA_DEVERR_REQUEST and only the first ld scores are used); idx: device int32 [T, k].
 * k in [1, 4096].  Needs no scratch memory.
 * key_hist: NULL, or the order-key digit histogram of each row's scores as dsa_indexer_scores
 * builds it ([T, 4096] uint32, 16-byte aligned): the call places its threshold from it instead of
 * sampling the row, and leaves it zero-filled for the next call.  The result never depends on
 * it: a histogram that does not match the scores only costs time.
 */
dsa_status dsa_topk_select(const float* scores, int64_t ld, const int32_t* q_pos, int32_t T,
                           int32_t k, int32_t* idx, uint32_t* key_hist, dsa_stream stream);

/*
 * Indexer scores fused with the top-K selection (same page, section "Lightning Indexer": the
 * indexer exists to pick each query's top K).  `scores` is caller-owned scratch of
 * [num_queries, ld] f32 (ld >= max_context) that receives the scores; idx is device int32
 * [num_queries, k].  Same semantics as the two calls above.  With a workspace of
 * dsa_indexer_topk_workspace_size(num_queries) bytes (16-byte aligned) the indexer kernel builds
 * each query's order-key digit histogram as it writes the scores (where dsa_indexer_scores
 * fills key_hist), and the selection takes its threshold from it (no sampling pass); the
 * workspace must be zero-filled before its first use and every call leaves it zero-filled
 * again.  Without a workspace, or where the indexer builds no histogram, the selection samples.
 */
dsa_status dsa_indexer_topk(const void* q, int32_t q_dtype, const float* q_scale, int32_t Hi,
                            int32_t Di, const float* w, const dsa_paged_cache* keys,
                            const dsa_batch* batch, int32_t k, float* scores, int64_t ld,
                            int32_t* idx, void* workspace, size_t workspace_bytes,
                            dsa_stream stream);

/* Bytes of the dsa_indexer_topk workspace for num_queries queries (4096 uint32 counters each). */
size_t dsa_indexer_topk_workspace_size(int32_t num_queries);

/*
 * Sparse MLA in MQA mode over the selected rows (same page, sections "Sparse MLA" and "MLA
 * Modifications": P = Q[H, d+r] K^T over the selected latent rows, O = P V, where V is the
 * first d of each row; the softmax is the usual scaled one).  For query t and head h:
 *   logit_j = softmax_scale * (q[t,h,:] . row(idx[t,j]))           (all d_v + d_rope dims)
 *   out[t,h,:] = sum_j softmax_j(logit) * row(idx[t,j])[0:d_v]
 *   lse[t,h]   = ln sum_j exp(logit_j)          (-inf and out = 0 when nothing is selected)
 * Entries idx[t,j] == -1 are skipped; any other index outside 0..q_pos[t] sets
 * DSA_DEVERR_INDEX and is skipped.
 * Dense case (same page, section "Lightning Indexer": a query that sees fewer than K positions
 * keeps all of them): idx == NULL attends every visible position 0..q_pos[t], with no selection;
 * then k >= max_context is required (k bounds the rows per query).  A caller whose queries all
 * see at most K positions skips the indexer and the selection and calls this directly.
 * q: device [num_queries, H, d_v + d_rope] of q_dtype; latent: paged cache with
 * dim == d_v + d_rope and dtype == q_dtype (f32 or bf16); idx: device int32 [num_queries, k]
 * or NULL (dense);
 * out: device [num_queries, H, d_v] of q_dtype; lse: device f32 [num_queries, H] or NULL.
 * workspace: device scratch of at least dsa_mla_workspace_size(num_queries, H, d_v, k) bytes,
 * 256-byte aligned (may be NULL when that size is 0).
 * The decode entry point splits each query's k rows across CTAs and merges the partial
 * results (log-sum-exp combine); the prefill entry point gives each query whole CTAs.
 * Fast path: H == 128, d_v == 512, d_rope == 64, bf16.
 */
dsa_status dsa_sparse_mla_decode(const void* q, int32_t q_dtype, int32_t H, int32_t d_v,
                                 int32_t d_rope, const dsa_paged_cache* latent,
                                 const dsa_batch* batch, const int32_t* idx, int32_t k,
                                 float softmax_scale, void* out, float* lse, void* workspace,
                                 size_t workspace_bytes, dsa_stream stream);

dsa_status dsa_sparse_mla_prefill(const void* q, int32_t q_dtype, int32_t H, int32_t d_v,
                                  int32_t d_rope, const dsa_paged_cache* latent,
                                  const dsa_batch* batch, const int32_t* idx, int32_t k,
                                  float softmax_scale, void* out, float* lse, void* workspace,
                                  size_t workspace_bytes, dsa_stream stream);

/*
 * Sparse MLA decode without caller-provided workspace.  The pages have no counterpart: this is a
 * convenience entry point for callers that cannot allocate device memory (for example code that
 * runs inside another framework's memory pool, or on a path where allocation is not allowed).
 * Same inputs, outputs and results as dsa_sparse_mla_decode; the split partials go to a fixed
 * 32 MiB scratch array inside the library.  Calls whose partials need more than that (the same
 * split plan as dsa_sparse_mla_decode; shapes that take the generic kernels need none) return
 * DSA_ERR_INVALID_ARG with a message: use dsa_sparse_mla_decode with a workspace then.
 * Set-up: the first call on each device looks up the scratch address (cudaGetSymbolAddress).
 * Under lazy module loading, the CUDA default, that lookup is when the scratch is reserved on the
 * device (32 MiB, held until the process exits), and it may synchronise the device.  Make the
 * first call on each device during set-up, before timing-critical work and before any stream
 * capture; later calls allocate nothing and do not synchronise.  After a device reset the next
 * call looks the address up again.  All calls on a device share the scratch: calls whose kernels
 * overlap on the GPU race; calls ordered on one stream are safe.  Nothing in the scratch needs
 * clearing.
 */
dsa_status dsa_sparse_mla_decode_noalloc(const void* q, int32_t q_dtype, int32_t H, int32_t d_v,
                                         int32_t d_rope, const dsa_paged_cache* latent,
                                         const dsa_batch* batch, const int32_t* idx, int32_t k,
                                         float softmax_scale, void* out, float* lse,
                                         dsa_stream stream);

/* Bytes of workspace dsa_sparse_mla_decode needs for these sizes (0 when none). Host only. */
size_t dsa_mla_workspace_size(int32_t num_queries, int32_t H, int32_t d_v, int32_t k);

/* Diagnostic of the bounded waits (no counterpart on the pages): enqueues one kernel whose single
 * thread waits on an mbarrier phase that never completes, with the same bounded wait the
 * tensor-core kernels use but a limit of `limit_cycles` SM cycles (1 .. 4e9).  The wait gives up,
 * the kernel sets DSA_DEVERR_TIMEOUT in the device error word and returns; the context stays
 * usable.  Read the word with dsa_get_device_error. */
dsa_status dsa_selftest_bounded_wait(int64_t limit_cycles, dsa_stream stream);

/* Diagnostic of the sparse MLA's row-gather rate (no counterpart on the pages): enqueues one
 * kernel of num_ctas CTAs (1 .. 1024) that gathers latent rows exactly as the tensor-core sparse
 * MLA does -- 64-row tiles, each row's nine 128-byte column blocks by TMA tile::gather4, a
 * two-stage shared-memory ring -- and does nothing else with them.  CTA c gathers the pool rows
 * rows[(c * tiles_per_cta + j) * 64 + i] (tile j = 0 .. tiles_per_cta-1, i = 0 .. 63; a device
 * int32 array of num_ctas * tiles_per_cta * 64 entries, each a row index of the pool, block *
 * 64 + offset) and writes its SM cycles from the start of its gathers to the landing of its last
 * tile to cycles[c] (device int64; -1 when a bounded wait gave up).  A row index outside the pool
 * sets DSA_DEVERR_INDEX and reads as zeros.  latent: bf16, block_size 64, dim 576, data 16-byte
 * aligned (the tensor-core MLA's shape).  tiles_per_cta: 1 .. 65536. */
dsa_status dsa_selftest_gather_rate(const dsa_paged_cache* latent, const int32_t* rows, int32_t tiles_per_cta,
                                    int32_t num_ctas, int64_t* cycles, dsa_stream stream);

/* Synchronises `stream`, then reads the device error word of the current device into *code
 * (0 = no fault).  Not for use inside stream capture. */
dsa_status dsa_get_device_error(int32_t* code, dsa_stream stream);

/* Enqueues a reset of the current device's error word to 0 on `stream`. */
dsa_status dsa_clear_device_error(dsa_stream stream);

/* Static description of a status code; detail of the last failed call on this host thread. */
const char* dsa_status_string(dsa_status status);
const char* dsa_last_error_message(void);

int32_t dsa_abi_version(void);

/* Number of kernels this library has enqueued in this process so far (all devices).  Host only;
 * a diagnostic for counting launches inside a timed region. */
int64_t dsa_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
