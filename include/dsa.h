/*
 * dsa.h - C ABI of the B200 (sm_100a) gated Indexer + Top-K sparse-attention layer.
 *
 * The layer, for every query row t of a ragged batch:
 *   1. indexer  s[t,j] = sum_h w_h * max(0, c * q_idx[t,h,:] . k_idx[j,h,:]),  j = 0..p(t)
 *   2. Top-K    the K positions with the largest s[t,j] (ties: lower j wins), or all
 *               p(t)+1 positions when there are no more than K
 *   3. attention o[t,h] = softmax_j(scale * q[t,h] . k[j,g(h)]) . v[j,g(h)] over the
 *               selected j only (exact softmax over the subset)
 *   4. gate     out[t,h,e] = sigmoid(gate[t,h,e]) * o[t,h,e]
 *
 * Pages this interface follows (web articles on one model release):
 *   [HSA] "Hybrid Sparse Attention for Long-Context LLMs: How Linear Attention and
 *          Indexer + Top-K Work Together": section "Indexer + Top-K: How Fine-Grained
 *          Sparse Attention Works", steps 1-4 and the pseudocode below them.
 *   [ITK] "Optimizing LLM Long-Context Inference with Indexed Top-K Sparse Attention":
 *          sections "Introducing Indexed Top-K Sparse Attention" (indexing stage, Top-K
 *          stage, K = 2048) and "Interface Design for Practical Implementation"
 *          (sparse_attn_forward(query, key, value, top_k); index consistency across
 *          heads; variable sequence lengths across a batch).
 *   [FGS] "How Fine-Grained Sparse Attention Reshapes Long-Context Architecture in Large
 *          Models": section "How Indexer + Top-K Works at Runtime" (retrieve, read
 *          precisely, fuse; one index set per query over the KV cache).
 *   [SAE] "Sparse Attention in Long-Context LLM Inference: Engineering Trade-offs and
 *          Architecture Choices": section "5. Abstract Implementation Sketch of
 *          Indexer + Top-K" (scale 1/sqrt(dim); cross-head sharing).
 *   [GSA] "From Linear Attention to Gated Sparse Attention: Dissecting a Hybrid LLM
 *          Architecture Trade-off": sections "2. The Core Change" (gate(q) * out) and
 *          "4. The Role of Gating and Engineering Considerations" (indexer precision,
 *          fused Top-K).
 * The pages give no indexer formula; the per-head ReLU dot product with a weighted head
 * sum in step 1 is the reading this library implements.  One score row and one index
 * set per query are shared by all attention heads.
 *
 * Conventions for every entry point
 *  - Ownership: the caller owns every buffer and the stream.  The library never
 *    allocates device memory; scratch comes from a caller-provided workspace (or, for
 *    dsa_decode_noalloc only, a fixed array inside the library).  The library keeps no
 *    per-call state and may be called from several host threads.
 *  - Synchrony: every compute call is asynchronous on `stream` (a cudaStream_t; NULL
 *    is the legacy default stream).  Argument errors are returned before anything is
 *    launched; a failed launch returns DSA_ERR_CUDA.  No exception crosses the ABI.
 *  - Device pointers: all tensor arguments are device pointers unless a field says
 *    "host".  Tensors are row-major and packed ragged: query-side tensors have
 *    total_q rows (sequence b owns rows q_offsets[b] .. q_offsets[b+1]-1), cache-side
 *    tensors have total_kv rows (sequence b owns rows kv_offsets[b] ..).
 *  - Positions: sequence b has L_b = kv_offsets[b+1]-kv_offsets[b] cache positions and
 *    Q_b = q_offsets[b+1]-q_offsets[b] <= L_b queries, the last Q_b positions: query i
 *    of b sits at p = L_b - Q_b + i and sees positions 0..p (itself included).  Index
 *    values are positions within the sequence (0-based).
 *  - Bad device data is never trapped: index entries < 0 are padding; entries > p are
 *    skipped and counted in `err_count` when one is given.  A bounded wait inside a
 *    kernel that runs out records DSA_ERR_TIMEOUT in the device status word
 *    (dsa_device_status) and the kernel returns.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1, /* a pointer, size, stride or alignment is invalid     */
  DSA_ERR_UNSUPPORTED = 2, /* valid but outside what this build implements        */
  DSA_ERR_WORKSPACE = 3,   /* workspace missing, too small or misaligned          */
  DSA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed         */
  DSA_ERR_TIMEOUT = 5      /* (device status only) a bounded in-kernel wait ended */
} dsa_status;

typedef enum {
  DSA_BF16 = 0,     /* bfloat16                                  */
  DSA_FP8_E4M3 = 1  /* OCP fp8 e4m3 (indexer tensors only)       */
} dsa_dtype;

/* Ragged batch description. */
typedef struct {
  int32_t batch;              /* B >= 1                                            */
  const int32_t* q_offsets;   /* device [B+1], q_offsets[0] = 0, non-decreasing    */
  const int32_t* kv_offsets;  /* device [B+1], kv_offsets[0] = 0, non-decreasing   */
  int32_t max_q_len;          /* host: >= max_b Q_b                                */
  int32_t max_kv_len;         /* host: >= max_b L_b                                */
  int64_t total_q;            /* host: q_offsets[B]                                */
  int64_t total_kv;           /* host: kv_offsets[B] (contiguous); with a block table,
                                 the rows of the cache arrays (pages * page_size)   */
  /* Paged cache (optional).  NULL block_table: sequence b's cache rows are rows
   * kv_offsets[b] .. kv_offsets[b+1]-1 of k_idx / k_cache / v_cache.  Otherwise position
   * j of sequence b lives in row block_table[b * max_pages + j / page_size] * page_size
   * + j % page_size of those arrays, and kv_offsets only gives the lengths
   * L_b = kv_offsets[b+1] - kv_offsets[b].  This is the serving layout of a cache that is
   * "no longer contiguous" ([FGS] "How Indexer + Top-K Works at Runtime", engineering
   * details).  page_size: a power of two >= 128 (a 128-position indexer tile never
   * straddles pages); max_pages >= ceil(max_kv_len / page_size); every referenced page id
   * in [0, total_kv / page_size). */
  const int32_t* block_table; /* device [B, max_pages] or NULL                     */
  int32_t max_pages;
  int32_t page_size;
  /* Host copies of q_offsets and kv_offsets (optional, NULL when not given; the same
   * values as the device arrays).  With them dsa_prefill and dsa_workspace_size plan per
   * sequence: in a batch that mixes long query groups (Q_b >= 128, prefill chunks) with
   * short ones (Q_b < 128, e.g. one new token per sequence), steps 1-2 run over each stretch
   * of consecutive sequences of one kind with the tiles that suit it -- the fused indexer ->
   * Top-K over 128-row query tiles for the long groups, key-split score tiles of 16 queries
   * for the short ones -- and the attention then runs once over all rows.  A serving
   * scheduler has these lengths on the host already; without them such a batch takes the
   * score-matrix path planned from the totals above. */
  const int32_t* q_offsets_host;   /* host [B+1] or NULL */
  const int32_t* kv_offsets_host;  /* host [B+1] or NULL */
} dsa_ragged;

/* Layer shape and numerics.  Supported by this build: idx_dim = 64,
 * 1 <= n_idx_heads <= 4, head_dim = 128, n_kv_heads divides n_q_heads with
 * n_q_heads / n_kv_heads <= 16, 1 <= top_k <= 16384. */
typedef struct {
  int32_t n_idx_heads;   /* H_i: indexer heads                                        */
  int32_t idx_dim;       /* D_i: indexer head dimension                               */
  int32_t n_q_heads;     /* Hq: attention query heads                                 */
  int32_t n_kv_heads;    /* Hkv: attention KV heads; query head h reads KV head h/(Hq/Hkv) */
  int32_t head_dim;      /* d                                                         */
  int32_t top_k;         /* K                                                         */
  int32_t idx_dtype;     /* dsa_dtype of q_idx and k_idx                              */
  float idx_scale_q;     /* dequantisation scale of q_idx (1 for bf16)                */
  float idx_scale_k;     /* dequantisation scale of k_idx (1 for bf16); c = scale_q*scale_k */
  float attn_scale;      /* softmax logit scale; 0 selects 1/sqrt(head_dim)           */
  int32_t w_row_stride;  /* 0: w is [H_i], shared by all rows; else w[row*stride + h] */
} dsa_params;

/* Human-readable name of a status code (static string). */
const char* dsa_status_string(dsa_status s);

/* Library ABI version (major*10000 + minor*100 + patch): 102 (dsa_ragged gained the
 * optional host offsets). */
int32_t dsa_version(void);

/*
 * Step 1 - indexer scores ([HSA] step 1; [ITK] "Two Engineering Considerations",
 * 1. Indexer Computational Cost: low-dimensional and cheap).
 *   q_idx  [total_q, H_i, D_i]  bf16 or e4m3 (params->idx_dtype)
 *   k_idx  [total_kv, H_i, D_i] same dtype
 *   w      fp32, [H_i] or [total_q, w_row_stride] (see dsa_params)
 *   scores fp32 [q_count, ld_scores]: row i belongs to packed query row q_begin+i and
 *          receives s[j] for j = 0..p of that row.  Entries beyond p are not written.
 * Requirements: 0 <= q_begin, q_begin+q_count <= total_q; ld_scores >= max_kv_len and a
 * multiple of 4; q_idx, k_idx 16-byte aligned; row strides H_i*D_i*elem a multiple of
 * 16 bytes.  Runs on tcgen05 tensor cores fed by TMA.
 */
dsa_status dsa_index_scores(const dsa_params* params, const dsa_ragged* ragged,
                            const void* q_idx, const void* k_idx, const float* w,
                            int64_t q_begin, int64_t q_count, float* scores, int64_t ld_scores,
                            void* stream);

/*
 * Step 2 - Top-K selection ([HSA] step 2; [ITK] "Introducing Indexed Top-K Sparse
 * Attention", Top-K Selection Stage).
 *   scores fp32 [q_count, ld_scores] as written by dsa_index_scores (only 0..p read)
 *   idx    int32 [q_count, ld_idx]: the selected positions of row i in ascending order,
 *          min(K, p+1) of them, then -1 up to K.  Ties at the threshold keep the lower
 *          positions; -0.0 equals +0.0.  NaN scores are not supported.
 *   cnt    int32 [q_count] or NULL: number selected per row.
 * Requirements: ld_scores a multiple of 4 and scores 16-byte aligned; ld_idx >= K.
 */
dsa_status dsa_topk(const dsa_params* params, const dsa_ragged* ragged, const float* scores,
                    int64_t ld_scores, int64_t q_begin, int64_t q_count, int32_t* idx,
                    int64_t ld_idx, int32_t* cnt, void* stream);

/*
 * Steps 1-2 fused - the index rows of dsa_index_scores followed by dsa_topk, without
 * writing the score matrix ([GSA] section 4: whether the Top-K selection can be fused
 * into kernels; [HSA] "Engineering and Evaluation Recommendations": dedicated fused
 * Top-K kernels).  The pages name the fusion as an engineering goal and give no method;
 * this one is exact:
 *   a. the indexer over every 16th key position gives each row a sample of its scores;
 *   b. from the sample, a threshold t per row with, with overwhelming probability, at
 *      least K of the row's scores >= t and not many more;
 *   c. the indexer over all keys keeps only the (position, score) pairs with score >= t;
 *   d. when a row has between K and the slot count of such candidates they contain its
 *      Top-K with every tie, and an exact radix select over them gives the result;
 *      a row whose threshold missed has its scores recomputed (CUDA cores, fp32) and
 *      selected exactly.
 * Output: exactly what dsa_index_scores + dsa_topk give on inputs whose scores are exact
 * in fp32 (e.g. dyadic values); otherwise the Top-K of fp32 scores whose rounding may
 * differ in the last bit for a row that was recomputed in step d.
 *   q_idx, k_idx, w   as dsa_index_scores
 *   idx, ld_idx, cnt  as dsa_topk (rows q_begin .. q_begin+q_count-1)
 *   workspace device, 256-byte aligned, ws_bytes >= the minimum of
 *             dsa_index_topk_workspace_size; rows are processed in passes of as many
 *             as it holds (the recommended size holds all q_count rows).  Nothing in it
 *             has to be initialised; its contents are undefined afterwards.
 * Returns DSA_ERR_UNSUPPORTED when K is too large for the candidate slots (about
 * K > 4500) or max_kv_len exceeds 314496; dsa_index_scores + dsa_topk cover those.
 */
dsa_status dsa_index_topk_workspace_size(const dsa_params* params, const dsa_ragged* ragged,
                                         int64_t q_count, size_t* min_bytes, size_t* rec_bytes);
dsa_status dsa_index_topk(const dsa_params* params, const dsa_ragged* ragged, const void* q_idx,
                          const void* k_idx, const float* w, int64_t q_begin, int64_t q_count,
                          int32_t* idx, int64_t ld_idx, int32_t* cnt, void* workspace,
                          size_t ws_bytes, void* stream);

/*
 * Steps 1-2 at block granularity ([HSA] "Indexer + Top-K: How Fine-Grained Sparse
 * Attention Works", steps 1-2: score and keep positions "or blocks").  The pages define no
 * block score; here a block of `block` consecutive positions scores as the largest indexer
 * score among its positions (up to p), the top_k blocks with the largest scores are kept
 * (ties to the lower block; all blocks when the row has no more than top_k), and the row's
 * selection is their positions.
 *   params->top_k  number of blocks kept per row (Kb)
 *   block          positions per block: a power of two, 32 .. 4096
 *   idx    int32 [q_count, ld_idx], ld_idx >= Kb * block: the selected positions of row i
 *          ascending, then -1 up to Kb * block.  Pass it to dsa_sparse_attn_gated with a
 *          params copy whose top_k is Kb * block.
 *   cnt    int32 [q_count] or NULL: positions selected per row.
 *   workspace device, 256-byte aligned, ws_bytes >= the minimum of
 *          dsa_index_topk_blocks_workspace_size (one row's 32-position maxima, block scores
 *          and block list); rows are processed in passes of as many as it holds.
 * The indexer stores one value per 32 positions (the maximum) instead of 32 scores, so the
 * Top-K works on n / block entries per row.  Every other argument as dsa_index_scores.
 * Returns DSA_ERR_INVALID_ARG for a block size outside the range or ld_idx < Kb * block.
 */
dsa_status dsa_index_topk_blocks_workspace_size(const dsa_params* params,
                                                const dsa_ragged* ragged, int32_t block,
                                                int64_t q_count, size_t* min_bytes,
                                                size_t* rec_bytes);
dsa_status dsa_index_topk_blocks(const dsa_params* params, const dsa_ragged* ragged,
                                 const void* q_idx, const void* k_idx, const float* w,
                                 int32_t block, int64_t q_begin, int64_t q_count, int32_t* idx,
                                 int64_t ld_idx, int32_t* cnt, void* workspace, size_t ws_bytes,
                                 void* stream);

/*
 * Steps 3-4 - exact softmax attention over the selected rows with the sigmoid output
 * gate fused in ([HSA] steps 3-4 and pseudocode; [SAE] section 5; [GSA] section 2).
 *   q        bf16 [total_q, Hq, d]
 *   k_cache  bf16 [total_kv, Hkv, d]; v_cache likewise
 *   idx      int32 [q_count, ld_idx], row i for packed query row q_begin+i: positions
 *            within the sequence, any order; entries < 0 are padding
 *   gate     bf16 [total_q, Hq, d] gate logits, or NULL for no gate
 *   out      bf16 [total_q, Hq, d] (rows q_begin..q_begin+q_count-1 written)
 *   lse      fp32 [q_count, Hq] or NULL: log(sum_j exp(scale * q.k_j)) over the
 *            selected j (natural log; -inf for a row with nothing selected)
 *   err_count int32 [1] or NULL: incremented once per index entry > p (skipped)
 * A row with nothing selected gets out = 0.  All rows read the same index set for all
 * heads; the gather of a KV head is shared by the query heads of its group.
 * Precision: logits, the running maximum and the softmax sums are fp32, the softmax
 * weights enter the P.V product rounded to bf16 (fp32 accumulation), and out is rounded
 * to bf16 (nearest even).  A row's result does not depend on q_begin / q_count (how the
 * rows are split into calls).
 * Addressing of the gathered rows: a 32-bit offset per row when each of k_cache and v_cache
 * spans at most 64 GiB, a general form otherwise; the environment variable
 * DSA_ATTN_ADDR_ROWS=1 (read once per process) forces the general form, for tests.  The
 * choice changes no result bit.
 * Requirements: q, k_cache, v_cache, gate, out 16-byte aligned.
 */
dsa_status dsa_sparse_attn_gated(const dsa_params* params, const dsa_ragged* ragged,
                                 const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* idx, int64_t ld_idx, int64_t q_begin,
                                 int64_t q_count, const void* gate, void* out, float* lse,
                                 int32_t* err_count, void* stream);

/*
 * Steps 3-4 with the layer's second branch mixed in by the gate ([HSA] "Indexer + Top-K:
 * How Fine-Grained Sparse Attention Works", step 4 and the last line of its pseudocode,
 * g * o_sparse + (1 - g) * o_linear; [FGS] "How Indexer + Top-K Works at Runtime", step 3
 * "Fuse": g * precise + (1 - g) * compressed_context):
 *   out[t,h,e] = sigmoid(gate[t,h,e]) * o[t,h,e] + (1 - sigmoid(gate[t,h,e])) * other[t,h,e]
 * with o the exact sparse attention of dsa_sparse_attn_gated.  The second branch (the
 * linear or compressed-context attention output) is an input computed elsewhere.
 *   other  bf16 [total_q, Hq, d], 16-byte aligned; gate is required here.
 * Every other argument, the LSE (of the sparse branch) and the error behaviour are as for
 * dsa_sparse_attn_gated.
 */
dsa_status dsa_sparse_attn_gated_mix(const dsa_params* params, const dsa_ragged* ragged,
                                     const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* idx, int64_t ld_idx, int64_t q_begin,
                                     int64_t q_count, const void* gate, const void* other,
                                     void* out, float* lse, int32_t* err_count, void* stream);

/*
 * Workspace for dsa_prefill / dsa_decode.  *min_bytes: the least that works (one query
 * row of scores per pass); *rec_bytes: the size this build recommends for throughput
 * (fewer, larger passes).  Either pointer may be NULL.  dsa_prefill runs steps 1-2 as
 * dsa_index_topk does when the batch is prefill-shaped (at least 256 query rows per
 * sequence on average), its score matrix would exceed 256 MiB, the fused path supports
 * K and max_kv_len, and the workspace holds fused passes of at least 2048 rows (or all
 * rows); *rec_bytes then covers one fused pass over every row.
 */
dsa_status dsa_workspace_size(const dsa_params* params, const dsa_ragged* ragged, int is_decode,
                              size_t* min_bytes, size_t* rec_bytes);

/*
 * Whole layer for a ragged batch of prefill chunks (any Q_b <= L_b): steps 1-4 in
 * passes over the query rows, each pass sized to the workspace (scores and, when
 * idx_out is NULL, index rows live there).  Fused Top-K and gather per [HSA]
 * "Engineering and Evaluation Recommendations" (inference side) and chunked prefill.
 *   idx_out  int32 [total_q, K] or NULL: the selected positions (as dsa_topk).
 *   err_count int32 [1] or NULL (as dsa_sparse_attn_gated).
 *   workspace device, 256-byte aligned, ws_bytes >= the minimum of dsa_workspace_size.
 */
dsa_status dsa_prefill(const dsa_params* params, const dsa_ragged* ragged, const void* q_idx,
                       const void* k_idx, const float* w, const void* q, const void* k_cache,
                       const void* v_cache, const void* gate, void* out, int32_t* idx_out,
                       int32_t* err_count, void* workspace, size_t ws_bytes, void* stream);

/* Buffers of one layer call: the ragged offsets and the layer's inputs and output. */
typedef struct {
  const int32_t* q_offsets;   /* [batch+1] */
  const int32_t* kv_offsets;  /* [batch+1] */
  const void* q_idx;
  const void* k_idx;
  const float* w;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const void* gate;           /* NULL: no gate */
  void* out;
} dsa_layer_buffers;

/*
 * dsa_prefill from host memory, with the transfers overlapped with the computation: the
 * packed query rows are split into n_chunks ranges (n_chunks <= 0: up to 16, one per 2048
 * rows); for each range one copy stream uploads its query-side rows (q_idx, q, gate) and
 * the cache rows its queries see that are not on the device yet, the caller's stream runs
 * the layer on the range as soon as they have landed, and a second copy stream brings its
 * output rows back.
 *   order  1: ranges in row order (the cache arrives progressively); 2: last range first;
 *          0: 2 when the batch has at least 256 query rows per sequence on average, else 1.
 *          (Used when the layer runs per range, see below.)
 * When the workspace also holds the index rows of every row (K int32 each) next to one pass
 * of steps 1-2 over all rows (the dsa_workspace_size recommendation does for a prefill whose
 * steps 1-2 run fused), steps 1-2 run once as soon as q_idx and k_idx have landed, and only
 * the attention runs per range (in row order; the last of the n_chunks ranges is then cut in
 * halves of halves, at most three times and not below 256 rows, since its attention and
 * read-back are what remains after the last upload); otherwise the whole layer runs per
 * range.
 *   host  every input and the output in host memory (page-locked memory lets the copies
 *         run asynchronously and overlap); host->q_offsets / kv_offsets are also read by
 *         the host to plan the ranges.
 *   dev   device buffers of the same sizes and layouts (caller-owned; overwritten with the
 *         inputs, dev->out with the output).  R gives the sizes; its offset pointers are
 *         replaced by dev's.
 *   workspace as dsa_prefill.
 * The call returns once everything is enqueued; `stream` completes after the last output
 * row is back in host memory.  The device buffers must not be touched by other streams
 * until then.  The library's two copy streams per device are shared by all such calls
 * (calls from several host threads enqueue one at a time and their copies queue behind each
 * other).  Contiguous caches only (DSA_ERR_UNSUPPORTED with a block table).
 */
dsa_status dsa_prefill_from_host(const dsa_params* params, const dsa_ragged* ragged,
                                 const dsa_layer_buffers* host, const dsa_layer_buffers* dev,
                                 int32_t n_chunks, int32_t order, void* workspace,
                                 size_t ws_bytes, void* stream);

/*
 * Whole layer for one new token per sequence (every Q_b = 1, so max_q_len must be 1 and
 * total_q = batch).  Same arguments and outputs as dsa_prefill; tiles are sized for a
 * single query per sequence (the indexer becomes a bandwidth-bound scan of k_idx).
 */
dsa_status dsa_decode(const dsa_params* params, const dsa_ragged* ragged, const void* q_idx,
                      const void* k_idx, const float* w, const void* q, const void* k_cache,
                      const void* v_cache, const void* gate, void* out, int32_t* idx_out,
                      int32_t* err_count, void* workspace, size_t ws_bytes, void* stream);

/*
 * dsa_decode without a workspace argument, for callers that cannot allocate device
 * memory: code embedded in a host framework whose allocator owns the whole device
 * (a side allocation would break its accounting or pools), decode loops that must not
 * allocate after warm-up because an allocation can synchronise the device, and plugin
 * interfaces that hand over tensors but no allocator.  The pages have no counterpart;
 * this is a deployment convenience.
 *   Arguments and outputs are those of dsa_decode minus workspace / ws_bytes.
 *   Scratch: a fixed 32 MiB array inside the library on each device (reserved on every
 *   GPU that loads the library until the process exits).  The layer runs in as many
 *   passes as that needs; a single query row must fit, i.e. 4 * roundup(max_kv_len, 32)
 *   (+ 4 * K when idx_out is NULL) <= 32 MiB, otherwise DSA_ERR_WORKSPACE is returned
 *   before anything is launched (max_kv_len up to about 8.3 million at K = 2048).
 *   This entry point calls no cudaMalloc, cudaFree or other allocating routine.
 *   The first call on a device looks up the scratch's device address
 *   (cudaGetSymbolAddress), so make that first call before any stream capture.  The
 *   address is tied to the device's CUDA context; a call made in a new context (after
 *   cudaDeviceReset, say) looks it up again, so that call too should precede any capture.
 *   All calls on a device share the one scratch array: calls that can overlap on the
 *   GPU (different streams, or different host threads) race and must be serialised by
 *   the caller.  No part of the scratch needs to be zeroed between calls.
 */
dsa_status dsa_decode_noalloc(const dsa_params* params, const dsa_ragged* ragged,
                              const void* q_idx, const void* k_idx, const float* w,
                              const void* q, const void* k_cache, const void* v_cache,
                              const void* gate, void* out, int32_t* idx_out, int32_t* err_count,
                              void* stream);

/*
 * Device status word of the current device: synchronises `stream`, stores the status
 * recorded by kernels since the last clear (DSA_OK or DSA_ERR_TIMEOUT) in *status (host),
 * and clears it when clear != 0.
 */
dsa_status dsa_device_status(void* stream, int32_t* status, int clear);

/* Number of kernels this library has launched from the calling host thread. */
int64_t dsa_launch_count(void);

/* Number of query rows whose steps 1-2 the calling host thread ran through the fused
 * indexer -> Top-K path (dsa_index_topk, and the rows dsa_prefill planned that way) since
 * the last reset; reset != 0 clears the count after reading it.  Lets a caller see which
 * path a layer call took. */
int64_t dsa_fused_rows(int reset);

/*
 * Per-stage device timing, for measurement.  While enabled, each stage launch made
 * from the calling host thread is bracketed by CUDA events on its stream.
 * dsa_stage_times synchronises those events and returns, per stage (0 indexer,
 * 1 Top-K, 2 attention), the summed milliseconds and launch counts since the last
 * reset; the arrays are host [3].
 */
dsa_status dsa_stage_timing(int enable);
dsa_status dsa_stage_times(double* ms, int64_t* launches, int reset);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
