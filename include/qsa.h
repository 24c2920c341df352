/*
 * qsa.h — C ABI of the decode-time Qwen Sparse Attention (QSA) library
 * (libqsa.so, hand-written CUDA kernels for sm_100a).
 *
 * The method (sources cited by page title and section):
 *   - "Qwen 4 QSA 迎来解码上下文并行：深入解读 vLLM 针对 Qwen3.8-Flash-Next 的草稿 PR"
 *     (orcarouter.ai), section "拉取请求实际改变了什么": a light indexer
 *     compresses keys into micro-blocks at compression ratio 4, scores them
 *     and keeps the best 512 blocks (about 2,048 token positions); the final
 *     softmax and value aggregation still run on the uncompressed K and V.
 *     Under decode context parallelism each rank reads its own slice of the
 *     KV cache and the partial attention results are merged at the end; the
 *     selector and its side caches are replicated and live in the same cache
 *     group as the main KV cache.
 *   - "PR #53896 完整报告" (prhub.com.cn), sections "执行摘要" / "实现拆解"
 *     (weight-free top-k selector over a compressed-key cache; a circular
 *     raw-key cache; MTP step 0 selects, later steps reuse the indices;
 *     start-up check that the block size is divisible by the compress
 *     ratio) and the QSAIndexer.forward excerpt under "关键源码片段"
 *     (caches are updated and compressed before selection; the result is a
 *     fixed-width row of request-relative indices padded with -1).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or keeps them.  Layouts are dense,
 *     row-major (last index fastest) unless stated.
 *   - Every call is asynchronous: it validates its host-side arguments,
 *     enqueues kernels on `stream` and returns.  Arguments that can be
 *     checked on the host are checked before anything is launched
 *     (QSA_ERR_INVALID_ARG / QSA_ERR_UNSUPPORTED; nothing is launched then).
 *   - Problems only visible on the device (a block-table entry out of range,
 *     a context length that does not fit the block table, a malformed
 *     selection row, a wait that ran out) are recorded in a per-device error
 *     word and the offending access is skipped; read (and clear) it with
 *     qsa_get_device_error().  No kernel traps.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).
 */
#ifndef QSA_H_
#define QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *qsa_stream_t; /* same type as cudaStream_t */

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1, /* a host-side argument is malformed            */
  QSA_ERR_UNSUPPORTED = 2, /* a valid but unsupported shape or dtype        */
  QSA_ERR_BOUNDS = 3,      /* device saw an out-of-range page / position    */
  QSA_ERR_CUDA = 4,        /* a CUDA runtime call failed                    */
  QSA_ERR_TIMEOUT = 5,     /* a bounded device wait ran out                 */
  QSA_ERR_BAD_INPUT = 6    /* device saw malformed data (lengths, selection) */
} qsa_status;

typedef enum { QSA_F32 = 0, QSA_BF16 = 1, QSA_FP8_E4M3 = 2 } qsa_dtype;

/* Paged caches of one attention layer.  The main K/V cache, the compressed
 * indexer-key cache and the block table form one cache group: the same
 * block-table entry names the same physical page in all of them. */
typedef struct {
  int32_t num_pages;    /* physical pages in each cache                       */
  int32_t page_size;    /* tokens per page P; a multiple of the compress
                           ratio 4 (whole 4-token micro-blocks per page)     */
  int32_t num_kv_heads; /* Hkv                                                */
  int32_t head_dim;     /* D: 64 or 128                                       */
  int32_t idx_dim;      /* indexer dim d: 32, 64 or 128                       */
  int32_t kv_dtype;     /* qsa_dtype of k_cache / v_cache                     */
  const void *k_cache;  /* [num_pages, P, Hkv, D] of kv_dtype                 */
  const void *v_cache;  /* [num_pages, P, Hkv, D] of kv_dtype                 */
  const float *k_scale; /* [num_pages, Hkv] dequant scale (FP8 only, else NULL) */
  const float *v_scale; /* [num_pages, Hkv] dequant scale (FP8 only, else NULL) */
  uint8_t *kc;          /* [num_pages, qsa_kc_page_bytes(P, d)] packed compressed
                           keys (sums of 4 int8 keys), 16-byte aligned; layout
                           at qsa_kc_page_bytes                               */
  int8_t *ring;         /* [ring_rows, 4, d] raw keys of the newest positions:
                           slot p % 4 of row r holds request r's key at p     */
  int32_t ring_rows;    /* rows of `ring` (>= batch of every call)            */
  const int32_t *block_table; /* [B, max_pages_per_req] physical page of each
                                 logical page; -1 = none                     */
  int32_t max_pages_per_req;  /* row stride of block_table                    */
} qsa_cache;

/* Human-readable name of a status code (static string). */
const char *qsa_status_string(int32_t status);

/* Library ABI version (incremented on any incompatible change). */
int32_t qsa_abi_version(void);

/*
 * qsa_kc_page_bytes — bytes of one page of the packed compressed-key cache,
 * or 0 for an unsupported geometry (page_size not a positive multiple of 4,
 * idx_dim not 32, 64 or 128).
 *
 * A compressed key value v of micro-block b, dim j (the sum of 4 int8 keys,
 * -512 <= v <= 508) is stored losslessly in 10 bits: its low byte v & 255
 * and a 2-bit high field f = (v >> 8) + 2 in [0, 3], so v = 256 (f - 2) +
 * low byte.  A page of P tokens (R = P/4 micro-blocks, d = idx_dim) holds
 *   bytes [0, R*d)             R rows of d low bytes (row = micro-block in
 *                              the page, column = dim),
 *   bytes [R*d, R*d + R*d/4)   d/16 * R little-endian 32-bit words of high
 *                              fields: word w*R + row holds dims 16w ..
 *                              16w+15 of that row, dim 16w + 4s + k (s, k
 *                              in [0, 4)) at bits 8k + 2s,
 * then zero padding to a multiple of 16 bytes.  (The int16 layout would move
 * 2d bytes per micro-block through the scan of qsa_index_topk; this one
 * 1.25 d.)
 */
size_t qsa_kc_page_bytes(int32_t page_size, int32_t idx_dim);

/*
 * qsa_compress_append — write new tokens' raw indexer keys and refresh the
 * compressed key of every micro-block they touch.
 *
 * Passage: blog "拉取请求实际改变了什么" (keys compressed into micro-blocks
 * at ratio 4); PR #53896 report, QSAIndexer.forward excerpt (token keys go
 * to a circular raw-key cache, complete blocks are pooled into the
 * compressed-key cache, before any selection).  Pooling is the plain
 * integer sum: kc[b] = sum over tokens t in [4b, min(4b+4, end)) of k[t],
 * so a partial tail block holds the sum of the tokens present.
 *
 *   B              requests in this call (<= cache->ring_rows)
 *   pos0   [B]     int32, logical position of request r's first new token
 *   cu_new [B+1]   int32, request r's new tokens are rows cu_new[r] ..
 *                  cu_new[r+1]-1 of k_new (cu_new[0] = 0)
 *   k_new  [N, d]  int8 raw indexer keys, N = cu_new[B]
 *   max_new_per_req  host upper bound of cu_new[r+1]-cu_new[r] (sizes the
 *                  launch; a request above it is an error on the device)
 * Positions are appended in order: the raw keys of positions
 * 4*floor(pos0/4) .. pos0-1 must have been appended by an earlier call (they
 * are read back from ring row r).  A decode step passes T new tokens per
 * request; a prefill passes whole chunks (complete blocks are pooled
 * straight from k_new).  Errors: QSA_ERR_INVALID_ARG for null pointers,
 * B < 0, B > ring_rows or page_size % 4 != 0 (PR #53896 report, 实现拆解:
 * the block size must be divisible by the compress ratio);
 * QSA_ERR_UNSUPPORTED for an unsupported idx_dim.
 */
qsa_status qsa_compress_append(const qsa_cache *cache, int32_t B, const int32_t *pos0,
                               const int32_t *cu_new, const int8_t *k_new,
                               int32_t max_new_per_req, qsa_stream_t stream);

/* Workspace bytes qsa_index_topk needs for B requests of at most
 * max_blocks micro-blocks each. */
size_t qsa_index_topk_workspace_bytes(int32_t B, int32_t max_blocks);

/*
 * qsa_index_topk — score every competing micro-block against the indexer
 * query and keep the best `topk`.
 *
 * Passage: blog "拉取请求实际改变了什么" (score the micro-blocks, keep the
 * best 512); PR #53896 report "执行摘要" (weight-free top-k selection) and
 * QSAIndexer.forward excerpt (fixed-width int32 output padded with -1).
 *
 *   score[r][b] = sum_j q_idx[r][j] * kc_r[b][j]   (exact int32), b < n_r
 *   n_r = n_sel[r] if n_sel != NULL else ceil(ctx_lens[r] / 4)
 *   sel[r] = the topk blocks with the highest score (ties: lower block index
 *            wins), listed in ascending block order, padded with -1
 *
 *   q_idx    [B, d] int8 indexer query (MTP: of query token 0)
 *   ctx_lens [B] int32 tokens in each request's cache (>= 1)
 *   n_sel    [B] int32 or NULL (MTP: floor((L - T) / 4) + 1)
 *   max_blocks  host upper bound of n_r (row stride of the score buffer)
 *   topk     1 .. 4096
 *   sel      [B, topk] int32 output
 *   scores   [B, max_blocks] int32 output of every score, or NULL
 *   workspace  >= qsa_index_topk_workspace_bytes(B, max_blocks) bytes,
 *            16-byte aligned, any contents: it holds the maxima of the
 *            scan's groups of 2048/d consecutive blocks, and the scores when
 *            `scores` is NULL (with `scores` given, 64 KiB + the maxima,
 *            4 * B * ceil(max_blocks / 16) bytes rounded up to 256, are
 *            enough); calls that overlap on the GPU need separate
 *            workspaces.  Two kernels run: a scan that writes every score
 *            and the group maxima, then a selection with one CTA per
 *            request, which reads only the groups whose maximum can reach
 *            the top k (all scores when the request has fewer groups than
 *            topk).
 * The compressed-key pages are read through the block table.  Errors:
 * QSA_ERR_INVALID_ARG (null pointer, topk or max_blocks out of range,
 * workspace too small or misaligned, kc not 16-byte aligned).
 */
qsa_status qsa_index_topk(const qsa_cache *cache, int32_t B, const int8_t *q_idx,
                          const int32_t *ctx_lens, const int32_t *n_sel, int32_t max_blocks,
                          int32_t topk, int32_t *sel, int32_t *scores, void *workspace,
                          size_t workspace_bytes, qsa_stream_t stream);

/*
 * qsa_index_topk_tokens — the selection as a token budget: fixed-width rows
 * of request-relative token indices, padded with -1.
 *
 * Passage: PR #53896 report, QSAIndexer.forward excerpt (the indexer's
 * budget is a token count, token_topk = indexer_budget; forward returns
 * fixed-width request-relative token indices padded with -1; MTP step 0
 * selects for the target row and later steps reuse it).
 *
 * Selects topk = budget / 4 micro-blocks exactly as qsa_index_topk does,
 * then lists their tokens: with p0 = ctx_lens[r] - T (query token 0),
 *   tokens[r][4k + j] = 4 b_k + j   if 4 b_k + j <= p0, else -1
 * for the k-th kept block b_k in ascending order, and -1 in the groups of
 * four past the kept blocks.  Only the block holding p0 can be cut, and it
 * is the last kept one, so every row is ascending and its -1 sit at its end.
 *
 *   T        1 .. 4 query tokens per request (p0 as above)
 *   budget   4 .. 16384, a multiple of 4 (the compress ratio)
 *   tokens   [B, budget] int32 output, 16-byte aligned
 *   sel      [B, budget / 4] int32 output of the kept blocks, or NULL
 *   other arguments as for qsa_index_topk (topk = budget / 4)
 * Errors: as qsa_index_topk; QSA_ERR_INVALID_ARG also for a budget that is
 * not a positive multiple of 4, T out of range or a misaligned `tokens`.
 */
qsa_status qsa_index_topk_tokens(const qsa_cache *cache, int32_t B, const int8_t *q_idx,
                                 const int32_t *ctx_lens, const int32_t *n_sel, int32_t T,
                                 int32_t max_blocks, int32_t budget, int32_t *tokens,
                                 int32_t *sel, int32_t *scores, void *workspace,
                                 size_t workspace_bytes, qsa_stream_t stream);

/* Workspace bytes qsa_sparse_decode needs. */
size_t qsa_sparse_decode_workspace_bytes(int32_t B, int32_t T, int32_t Hq, int32_t Hkv,
                                         int32_t D, int32_t topk, int32_t num_splits);

/*
 * qsa_sparse_decode — exact softmax attention over the selected tokens of
 * the uncompressed paged K/V, split into KV partitions.
 *
 * Passage: blog "拉取请求实际改变了什么" (final softmax and value
 * aggregation on the uncompressed K/V; each decode-context-parallel rank
 * reads its own slice of the cache, results merged at the end); PR #53896
 * report "实现拆解" (MTP step 0 selects, later steps reuse the indices).
 *
 * Query token t of request r sits at position p_t = L - T + t (p0 = L - T).
 * It attends the set
 *     { i in selected blocks : i <= p_t }  U  (p0, p_t]
 * (the speculative tail is always visible, no token counted twice), with
 * logits sm_scale * q . k_i and query head h reading kv head h / (Hq/Hkv).
 * Split s owns logical pages [floor(s*NP/S), floor((s+1)*NP/S)),
 * NP = ceil(L / P); it writes
 *     lse_s = log sum_{i in split} exp(logit_i),
 *     o_s   = sum_{i in split} exp(logit_i - lse_s) v_i,
 * and an empty split writes o_s = 0, lse_s = -inf.  FP8 K/V values are
 * code * scale[page][kv head].
 * Numerics: products on tensor cores with fp32 accumulation (bf16 caches:
 * bf16 operands; fp8 caches: f16 operands, which hold every E4M3 code
 * exactly, with Q scaled into f16 range by a power of two per row); the
 * softmax weights enter the value product as a hi + lo pair; fp32 caches
 * run in fp32.  Outputs stay within 1e-2 absolute and 2e-3 relative L2 (o)
 * and 1e-4 (lse) of the exact result.
 *
 *   q        [B, T, Hq, D] of q_dtype (QSA_F32 or QSA_BF16; BF16 for
 *            BF16/FP8 caches, F32 for F32 caches)
 *   sel      [B, topk] int32, ascending block indices padded with -1 (the
 *            output of qsa_index_topk)
 *   T        1 .. 4; (Hq/Hkv) * T <= 32; Hq % Hkv == 0
 *   num_splits  1 .. 16
 *   o_part   [S, B, T, Hq, D] float32 output
 *   lse_part [S, B, T, Hq] float32 output (natural log)
 *   workspace  >= qsa_sparse_decode_workspace_bytes(...), 16-byte aligned,
 *            any contents.  BF16 caches (the stream-K decode) keep the
 *            requests' split boundaries and the workers' partials there,
 *            all written before they are read.  FP8 and F32 caches (the
 *            chunked decode) keep a header with a work counter and
 *            per-split tickets, which the call zeroes itself (a one-CTA
 *            kernel ahead of the decode kernel), then the chunk partials.
 *            Calls that overlap on the GPU need separate workspaces.
 * Errors: QSA_ERR_INVALID_ARG / QSA_ERR_UNSUPPORTED on the host
 * (QSA_ERR_UNSUPPORTED also when num_pages * page_size * Hkv exceeds
 * 2^31 - 1 cache rows); page or position violations -> QSA_ERR_BOUNDS on the
 * device.
 */
qsa_status qsa_sparse_decode(const qsa_cache *cache, int32_t B, int32_t T, int32_t Hq,
                             const void *q, int32_t q_dtype, const int32_t *ctx_lens,
                             const int32_t *sel, int32_t topk, float sm_scale,
                             int32_t num_splits, float *o_part, float *lse_part,
                             void *workspace, size_t workspace_bytes, qsa_stream_t stream);

/*
 * qsa_sparse_decode_merged — qsa_sparse_decode followed by the split merge
 * (qsa_lse_merge of o_part / lse_part into o / lse), in one call: the two
 * kernels go back to back on the stream.
 *
 * Passage: as qsa_sparse_decode and qsa_lse_merge (blog "拉取请求实际改变了
 * 什么": partial results of the context slices are merged at the end).
 *
 *   o    [B, T, Hq, D] float32 output, 16-byte aligned
 *   lse  [B, T, Hq] float32 output
 *   other arguments as for qsa_sparse_decode; o_part / lse_part are still
 *   written (same values as qsa_sparse_decode)
 * o / lse are those of qsa_lse_merge(num_splits, B*T*Hq, D, o_part,
 * lse_part, o, lse).
 * Errors: as qsa_sparse_decode and qsa_lse_merge.
 */
qsa_status qsa_sparse_decode_merged(const qsa_cache *cache, int32_t B, int32_t T, int32_t Hq,
                                    const void *q, int32_t q_dtype, const int32_t *ctx_lens,
                                    const int32_t *sel, int32_t topk, float sm_scale,
                                    int32_t num_splits, float *o_part, float *lse_part, float *o,
                                    float *lse, void *workspace, size_t workspace_bytes,
                                    qsa_stream_t stream);

/*
 * qsa_sparse_decode_splits — qsa_sparse_decode for the splits
 * [split_lo, split_hi) of num_splits only: what one rank of decode context
 * parallelism computes when it holds one slice of the KV pages.
 *
 * Passage: blog "拉取请求实际改变了什么" (each decode-context-parallel rank
 * reads its own slice of the cache; the partial results are merged at the
 * end).
 *
 * Split s still owns logical pages [floor(s*NP/S), floor((s+1)*NP/S)) of
 * S = num_splits. Pages outside the computed splits are never read, so the
 * block table may leave them unmapped (-1).
 *   o_part   [split_hi - split_lo, B, T, Hq, D] float32: split split_lo + i
 *            in o_part[i]
 *   lse_part [split_hi - split_lo, B, T, Hq] float32
 *   0 <= split_lo < split_hi <= num_splits
 *   other arguments as for qsa_sparse_decode (same workspace size for
 *   num_splits)
 * The computed splits are bit-identical to the same splits of a
 * qsa_sparse_decode call with the same arguments.
 * Errors: as qsa_sparse_decode; QSA_ERR_INVALID_ARG for an empty or
 * out-of-range split range.
 */
qsa_status qsa_sparse_decode_splits(const qsa_cache *cache, int32_t B, int32_t T, int32_t Hq,
                                    const void *q, int32_t q_dtype, const int32_t *ctx_lens,
                                    const int32_t *sel, int32_t topk, float sm_scale,
                                    int32_t num_splits, int32_t split_lo, int32_t split_hi,
                                    float *o_part, float *lse_part, void *workspace,
                                    size_t workspace_bytes, qsa_stream_t stream);

/*
 * qsa_lse_merge — merge KV-partition partial results by log-sum-exp.
 *
 * Passage: blog "拉取请求实际改变了什么" (attention results from the ranks
 * are merged at the end).
 *   lse = log sum_s exp(lse_s),  o = sum_s exp(lse_s - lse) o_s;
 *   when every lse_s is -inf: o = 0, lse = -inf.
 *
 *   o_part [S, rows, D], lse_part [S, rows] float32 (rows = B*T*Hq)
 *   o [rows, D], lse [rows] float32 outputs (may not alias the inputs)
 *   1 <= S <= 64, D % 4 == 0, all pointers 16-byte aligned.
 */
qsa_status qsa_lse_merge(int32_t num_splits, int64_t rows, int32_t D, const float *o_part,
                         const float *lse_part, float *o, float *lse, qsa_stream_t stream);

/*
 * Normalised-pooling indexer variant: float compressed keys and scores.
 *
 * Passage: PR #53896 report, QSAIndexer.forward excerpt under 关键源码片段
 * (raw token keys are pooled by the compress ratio and normalised before
 * they enter the compressed-key cache) and 实现拆解 (an RMS norm of the
 * indexer, apply_qsa_rmsnorm).  Reading: pooling = mean of the tokens present
 * in the micro-block; normalisation = RMS normalisation,
 *     k_c[b] = m_b / sqrt(mean_j m_b[j]^2 + eps) * (1 + w),  m_b = block mean,
 * w an optional per-dim weight; score[r][b] = q_r . k_c[b] in float; the
 * selection rule is qsa_index_topk's (highest score first, ties: lower block
 * index; ascending; -1 padded).
 *
 * Storage (separate from the integer indexer's caches; same block table):
 *   kcn   [num_pages, qsa_kcn_page_bytes(P, d)] bytes: page = [P/4 rows][d]
 *         float16 compressed keys, 16-byte aligned
 *   ring  [ring_rows, 4, d] bfloat16: slot p % 4 of row r holds request r's
 *         raw key at position p, 16-byte aligned
 * Numerics: sums, the mean square and the dot products in float32; k_c is
 * rounded to float16 (relative error <= 2^-11), so a score is within
 * 2^-10 * |q|_2 * sqrt(d) * max_j |1 + w_j| of the exact one, and blocks whose
 * scores are that close to the top-k threshold may be ordered either way.
 *
 * qsa_kcn_page_bytes: (P/4) * d * 2, or 0 for page_size not a positive
 * multiple of 4 or idx_dim not 32, 64 or 128.
 *
 * qsa_compress_append_norm: as qsa_compress_append (pos0, cu_new,
 * max_new_per_req, ring_rows and the append order are the same), with
 *   k_new        [N, d] bfloat16 raw keys, 16-byte aligned
 *   norm_weight  [d] float32 w, or NULL for none
 *   eps          > 0 (1e-6 in the tests)
 * Errors: QSA_ERR_INVALID_ARG for null or misaligned pointers, B out of
 * range, eps <= 0; QSA_ERR_UNSUPPORTED for an unsupported idx_dim.
 *
 * qsa_index_topk_norm: as qsa_index_topk (ctx_lens, n_sel, max_blocks,
 * topk, sel, workspace of qsa_index_topk_workspace_bytes), with
 *   q_idx   [B, d] bfloat16 indexer query, 16-byte aligned
 *   scores  [B, max_blocks] float32 output of every score, or NULL
 * Two kernels: a scan of the float16 keys and the selection on float keys.
 */
size_t qsa_kcn_page_bytes(int32_t page_size, int32_t idx_dim);
qsa_status qsa_compress_append_norm(const qsa_cache *cache, void *kcn, void *ring,
                                    const float *norm_weight, float eps, int32_t B,
                                    const int32_t *pos0, const int32_t *cu_new, const void *k_new,
                                    int32_t max_new_per_req, qsa_stream_t stream);
qsa_status qsa_index_topk_norm(const qsa_cache *cache, const void *kcn, int32_t B,
                               const void *q_idx, const int32_t *ctx_lens, const int32_t *n_sel,
                               int32_t max_blocks, int32_t topk, int32_t *sel, float *scores,
                               void *workspace, size_t workspace_bytes, qsa_stream_t stream);

/*
 * qsa_sparse_prefill — QSA attention of a prefill chunk: many query tokens
 * per request, each with its own selection.
 *
 * Passage: blog "为什么一篇关于未发布架构的 serving PR 仍然值得你花时间" (a native
 * sparse-prefill kernel for the QSA path, PR #59010); what it computes is
 * read from the decode path of the same pages: query token p of a request is
 * a causal query over [0, p].  Its candidate blocks are 0 .. floor(p/4), the
 * block holding p summing only its tokens <= p; they are scored against p's
 * own indexer query, the best `topk` kept (ties: lower block index), and p
 * attends the kept blocks' tokens up to p:
 *   sel[i]  = the kept blocks of token i, ascending, -1 padded
 *   o[i]    = sum_t softmax(sm_scale * q[i] . k_t) v_t,  lse[i] = log sum exp
 * (GQA: query head h reads kv head h / (Hq/Hkv)).  A token of the first
 * 2,048 positions keeps every block: dense causal attention.
 *
 * Preconditions: the chunk's tokens are the NEWEST cached tokens of each
 * request: their K/V rows and raw indexer keys were written (K/V into the
 * paged cache, keys through qsa_compress_append) before this call, so
 * request r holds ctx_lens[r] tokens and its query tokens sit at positions
 * ctx_lens[r] - n_r .. ctx_lens[r] - 1 (n_r = cu_q[r+1] - cu_q[r]).
 *
 *   B, n_tokens    requests, and query tokens in all (= cu_q[B])
 *   max_q_per_req  host bound of n_r (sizes the launch)
 *   cu_q     [B+1] int32 row offsets of each request's query tokens
 *   ctx_lens [B] int32 cached tokens of each request (>= n_r)
 *   q_idx    [n_tokens, d] int8 indexer queries, 16-byte aligned
 *   k_chunk  [n_tokens, d] int8 raw indexer keys of the query tokens (as
 *            appended), 4-byte aligned
 *   q        [n_tokens, Hq, D] of q_dtype (as qsa_sparse_decode)
 *   max_blocks  host bound of ceil(ctx_lens[r] / 4) (score row stride)
 *   topk     1 .. 4096
 *   sel      [n_tokens, topk] int32 output
 *   o        [n_tokens, Hq, D] float32 output, 16-byte aligned
 *   lse      [n_tokens, Hq] float32 output
 *   workspace >= qsa_sparse_prefill_workspace_bytes(n_tokens, max_blocks,
 *            Hq, Hkv, D, topk) bytes, 256-byte aligned, any contents
 * Kernels: a tensor-core scan (tcgen05.mma kind::i8, int32 accumulators in
 * tensor memory) of every token's indexer query against its prefix's
 * compressed keys, a per-token fix-up of the block holding the token, the
 * selection of qsa_index_topk per token, and the decode kernels of
 * qsa_sparse_decode with one split per token.
 * Errors: QSA_ERR_INVALID_ARG for null / misaligned pointers or sizes out of
 * range; QSA_ERR_UNSUPPORTED for n_tokens or B above 65535 or an
 * unsupported idx_dim / head shape; device problems as qsa_sparse_decode.
 */
size_t qsa_sparse_prefill_workspace_bytes(int32_t n_tokens, int32_t max_blocks, int32_t Hq,
                                          int32_t Hkv, int32_t D, int32_t topk);
qsa_status qsa_sparse_prefill(const qsa_cache *cache, int32_t B, int32_t n_tokens,
                              int32_t max_q_per_req, const int32_t *cu_q, const int32_t *ctx_lens,
                              const int8_t *q_idx, const int8_t *k_chunk, const void *q,
                              int32_t q_dtype, int32_t Hq, int32_t max_blocks, int32_t topk,
                              float sm_scale, int32_t *sel, float *o, float *lse, void *workspace,
                              size_t workspace_bytes, qsa_stream_t stream);

/*
 * qsa_index_topk_noalloc — qsa_index_topk without a caller workspace.
 *
 * The source pages have no counterpart to this entry point; it exists for
 * callers that cannot hand the library device memory of their own: code that
 * runs where cudaMalloc is not allowed or not wanted (inside a plugin of a
 * framework that owns all allocations, or on a latency-critical path where an
 * allocation would synchronise the device), and that therefore cannot
 * provide the score workspace.
 *
 * Same arguments and results as qsa_index_topk (sel only; no score output).
 * The scores go to a fixed array compiled into libqsa.so: 8,388,608 int32
 * (32 MiB), held on every GPU that loads the library until the process
 * exits.  Calls with B * max_blocks above that are rejected with
 * QSA_ERR_UNSUPPORTED before anything is launched.  Nothing is allocated:
 * the first call on a device looks up the array's device address (with
 * that device current) and keeps it, so make that first call before any
 * stream capture.  All calls share the array: calls that overlap on the GPU
 * (two streams, or two devices' threads racing on the same device) race on
 * it; calls in order on one stream do not.  QSA_ERR_CUDA if the address
 * lookup fails.  The looked-up address is kept for the life of the process,
 * so after cudaDeviceReset on a device this entry point must not be called
 * on that device again in the same process.  Each call's scan writes every
 * score its selection reads, so the array needs no clearing between calls.
 */
qsa_status qsa_index_topk_noalloc(const qsa_cache *cache, int32_t B, const int8_t *q_idx,
                                  const int32_t *ctx_lens, const int32_t *n_sel,
                                  int32_t max_blocks, int32_t topk, int32_t *sel,
                                  qsa_stream_t stream);

/*
 * qsa_get_device_error — synchronise `stream`, then read and clear the
 * current device's error word.  Returns QSA_OK when no kernel recorded a
 * problem, else the first recorded code (QSA_ERR_BOUNDS, QSA_ERR_TIMEOUT,
 * QSA_ERR_BAD_INPUT); *flags_out (if not NULL) receives every bit seen.
 * The word is shared by all streams of the device.
 */
qsa_status qsa_get_device_error(qsa_stream_t stream, uint32_t *flags_out);

/*
 * Decode session — one decode step per call, host buffers in and out, with
 * the transfers overlapped with the kernels.
 *
 * The pages' path runs inside a serving runtime that owns the transfers;
 * they have no counterpart for this call.  It exists so that an end-to-end
 * step (inputs from host memory, o / lse back to host memory) costs no more
 * than the kernels:
 * - The session owns two slots of device input and output buffers, plus
 *   the selection, split partials and workspaces.
 * - Its upload stream copies step k+1's inputs while step k computes on the
 *   compute stream, and its download stream copies step k-1's o / lse back.
 *   Events order the three streams.
 * - A step runs exactly qsa_compress_append, qsa_index_topk and
 *   qsa_sparse_decode_merged (sm_scale, num_splits).
 *
 * qsa_session_create allocates every buffer (cudaMalloc, the decode
 * workspace zero-filled) and two non-blocking streams. It copies *cache
 * (the caches stay the caller's).
 *   T, Hq, topk, num_splits, max_blocks as for the calls above
 *   q_dtype         QSA_BF16 (bf16 / fp8 caches) or QSA_F32 (fp32 caches)
 *   max_new_tokens  bound on cu_new[B] (tokens appended per step)
 *   compute_stream  stream for the kernels, or NULL for a session-owned one
 *   *out            receives the session
 *
 * qsa_session_step_host enqueues one step and returns without waiting:
 *   pos0 [B], cu_new [B+1], k_new [cu_new[B], d], q_idx [B, d],
 *   q [B, T, Hq, D] of q_dtype, ctx_lens [B], n_sel [B] or NULL
 *     host inputs; cu_new is also read on the host
 *   o [B, T, Hq, D] float32, lse [B, T, Hq] float32
 *     host outputs
 * Host buffers should be pinned (cudaHostAlloc or registered) for the
 * copies to overlap. Pageable memory works, but the copies then block.
 * Inputs must stay unchanged and outputs untouched until
 * qsa_session_synchronize returns.
 *
 * qsa_session_streams reports the three streams, for events and waits.
 * qsa_session_synchronize waits for every enqueued step.
 * qsa_session_destroy synchronises and frees the session.
 *
 * Errors: QSA_ERR_INVALID_ARG for bad sizes, null pointers or cu_new[B] >
 * max_new_tokens; QSA_ERR_CUDA when an allocation, copy or stream call
 * fails; otherwise the status of the failing library call.
 */
typedef struct qsa_session qsa_session;

qsa_status qsa_session_create(const qsa_cache *cache, int32_t B, int32_t T, int32_t Hq,
                              int32_t q_dtype, int32_t topk, int32_t num_splits,
                              int32_t max_blocks, int32_t max_new_tokens, float sm_scale,
                              qsa_stream_t compute_stream, qsa_session **out);
qsa_status qsa_session_step_host(qsa_session *s, const int32_t *pos0, const int32_t *cu_new,
                                 const int8_t *k_new, const int8_t *q_idx, const void *q,
                                 const int32_t *ctx_lens, const int32_t *n_sel, float *o,
                                 float *lse);
qsa_status qsa_session_streams(const qsa_session *s, qsa_stream_t *h2d, qsa_stream_t *compute,
                               qsa_stream_t *d2h);
qsa_status qsa_session_synchronize(qsa_session *s);
qsa_status qsa_session_destroy(qsa_session *s);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H_ */
