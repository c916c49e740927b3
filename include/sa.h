/*
 * sa.h -- C ABI of libsa.so: fine-grained top-K sparse attention on B200.
 *
 * The method (three stages, all queries of a token sharing one selection over
 * one shared KV head):
 *   1. a lightweight indexer scores every causal (query t, key s) pair,
 *        I[t,s] = sum_j w[t,j] * ReLU(qI[t,j] . kI[s])
 *      ("Sparse Attention for Long-Context LLM Inference", section "Where
 *      Sparse Attention Is Actually Sparse": a lightweight indexer scores the
 *      history and hands candidate indices to attention; "Sparse Attention in
 *      2026", "The designs that shipped": the lightning indexer is a small,
 *      few-head, low-precision scorer feeding top-k 2048), optionally after a
 *      coarse pass over mean-pooled 64-token blocks ("Why fine-grained sparse
 *      attention ...", section "What Fine-Grained Means");
 *   2. each query keeps its K best keys (ties -> lower position) and always
 *      the W most recent positions ("Sparse Attention", completesystemdesign,
 *      mask diagrams: "+ always the local window");
 *   3. exact softmax(q.k/sqrt(d)) v over only the selected keys
 *      ("A Guide to Sparse Attention in Large Models", section 2, masked form
 *      with Mask[i,j] = 1 iff j in S(i); section 4.2, index-based path).
 *
 * Conventions shared by every entry point
 *   - Every pointer named in an argument list is DEVICE memory owned by the
 *     caller, unless the comment says "host".  The library never allocates,
 *     frees, or keeps a pointer past the call.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream).  The library never synchronises.
 *   - The return value reports synchronous argument checks.  On any status
 *     other than SA_OK nothing has been enqueued.
 *   - `dev_status` (device int32, may be NULL) receives errors found while
 *     kernels run: kernels OR SA_DEV_* bits into it.  The caller zeroes it
 *     before the call and reads it after synchronising.  An out-of-range index
 *     or page id is never dereferenced: the access is skipped and the bit set.
 *   - bf16 values are passed as raw 16-bit patterns (sa_bf16), e4m3 values
 *     as raw bytes (sa_e4m3).
 *   - Supported shapes: d (attention head dim) in {64, 128}; D_I (indexer
 *     dim) in {32, 64} with bf16 operands, {64, 128} with e4m3 operands and
 *     for the fused decode select; H_I in {1, 2, 4, 8} (1 .. 8 for the fused
 *     decode select); 1 <= Hq <= 64 query heads; page_size 64.  Other shapes
 *     return SA_ERR_UNSUPPORTED.  There is no fallback path.
 */
#ifndef FINE_GRAINED_TOP_SA_H
#define FINE_GRAINED_TOP_SA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t sa_bf16;                 /* raw bfloat16 bits */
typedef uint8_t sa_e4m3;                  /* raw OCP FP8 e4m3 bits (no inf; 0x7F/0xFF NaN) */
typedef struct CUstream_st *sa_stream;    /* same type as cudaStream_t */

typedef enum {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,   /* NULL pointer, negative size, bad stride ...  */
    SA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set              */
    SA_ERR_CUDA = 3,          /* a CUDA runtime call failed (launch, attr)    */
    SA_ERR_TIMEOUT = 4,       /* (decoded from dev_status) a bounded wait gave up */
    SA_ERR_INDEX = 5,         /* (decoded from dev_status) bad index / page id */
    SA_ERR_WORKSPACE = 6      /* caller's workspace is smaller than required  */
} sa_status;

/* bits OR-ed into *dev_status by kernels */
#define SA_DEV_INDEX   0x1    /* an index, candidate or page id out of range   */
#define SA_DEV_ORDER   0x2    /* a top-K / candidate row not strictly ascending */
#define SA_DEV_TIMEOUT 0x4    /* a bounded pipeline wait ran out               */

/* Human-readable name of a status (static storage). */
const char *sa_status_string(sa_status s);

/* Maps a dev_status word (read back by the caller) to a status:
 * SA_OK, SA_ERR_TIMEOUT or SA_ERR_INDEX. */
sa_status sa_dev_status_decode(int word);

/* Library ABI version (major * 100 + minor). */
int sa_version(void);

/* ------------------------------------------------------------------------
 * Stage 1 -- indexer scores (tensor cores: tcgen05 MMA into TMEM, TMA loads)
 *
 *   scores[(b*T + t) * ld_scores + s] =
 *       sum_{j < H_I} w[b,t,j] * max(0, sum_{c < D_I} qI[b,t,j,c] * kI_b[s,c])
 *   for 0 <= s < n_valid[b*T + t]; no 1/sqrt(D_I), no softmax, no positional
 *   term ("Where Sparse Attention Is Actually Sparse": the indexer omits
 *   positional encoding).  Sums are fp32 (exact for the integer-valued inputs
 *   used by the tests).  Columns s >= n_valid of a row are NOT written: their
 *   contents are unspecified and every consumer bounds rows by n_valid.
 *
 *   qI        [B, T, H_I, D_I] bf16
 *   w         [B, T, H_I] bf16
 *   kI        contiguous (page_table == NULL): [B, S, D_I] bf16, sequence b's
 *             key s at row b*S + s;
 *             paged: a pool [P, page_size, D_I]; key s of sequence b at row
 *             page_table[b*max_pages + s/page_size]*page_size + s%page_size.
 *   n_valid   [B*T] number of leading key columns scored for each query row
 *             (0 .. S); NULL means causal prefill with the T queries at the
 *             last T of S positions: n_valid = S - T + t + 1.
 *   scores    [B*T, ld_scores] fp32, ld_scores >= S and a multiple of 4.
 *   Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_CUDA; device:
 *   SA_DEV_INDEX for a page id outside [0, P) (P = pool_pages), or an
 *   n_valid entry outside [0, S]; SA_DEV_TIMEOUT.
 * ---------------------------------------------------------------------- */
sa_status sa_indexer_scores(const sa_bf16 *qI, const sa_bf16 *w,
                            const sa_bf16 *kI, const int32_t *page_table,
                            int max_pages, int pool_pages, int page_size,
                            int B, int T, int S, int H_I, int D_I,
                            const int32_t *n_valid, float *scores,
                            int64_t ld_scores, int *dev_status,
                            sa_stream stream);

/* Indexer scores with FP8 operands ("Sparse Attention in 2026", "The designs
 * that shipped": the shipped lightning indexer is a small FP8 network).
 *   The same definition, layouts, n_valid rule, errors and unwritten columns
 *   as sa_indexer_scores, with qI and kI held as e4m3 bytes: the products
 *   run on the tensor cores as tcgen05.mma kind::f8f6f4 (each e4m3 x e4m3
 *   product is exact) and sums are fp32.  w stays bf16.
 *   qI [B, T, H_I, D_I] e4m3, kI contiguous [B, S, D_I] or a paged pool
 *   [P, 64, D_I] e4m3, both 16-byte aligned; D_I in {64, 128} (rows of 64
 *   or 128 bytes).
 *   Scores equal sa_indexer_scores applied to the decoded values whenever
 *   the fp32 sums are exact (e.g. the integers -3..3 of the tests, which e4m3
 *   holds exactly). */
sa_status sa_indexer_scores_fp8(const sa_e4m3 *qI, const sa_bf16 *w,
                                const sa_e4m3 *kI, const int32_t *page_table,
                                int max_pages, int pool_pages, int page_size,
                                int B, int T, int S, int H_I, int D_I,
                                const int32_t *n_valid, float *scores,
                                int64_t ld_scores, int *dev_status,
                                sa_stream stream);

/* Quantise n bf16 values to e4m3 (for indexer keys entering the cache and
 * indexer queries): round to nearest, ties to even; finite values beyond
 * +-448 and infinities become +-448; NaN becomes NaN (0x7F with the sign).
 *   src [n] bf16, dst [n] e4m3, device memory, not overlapping; any n >= 0
 *   and any alignment (16-byte src and 8-byte dst take the vector path).
 *   Errors: SA_ERR_INVALID_ARG (n < 0, NULL with n > 0), SA_ERR_CUDA. */
sa_status sa_convert_e4m3(const sa_bf16 *src, sa_e4m3 *dst, int64_t n,
                          sa_stream stream);

/* Indexer scores over an explicit candidate list per query (the fine pass of
 * the two-stage selection, "What Fine-Grained Means": the fine pass scores
 * individual tokens inside the coarse candidates).
 *   scores[t*ld_scores + i] = I[t, cand[t*ld_cand + i]] for i < n_cand[t];
 *   entries i >= n_cand[t] are not written.
 *   qI [T, H_I, D_I], w [T, H_I], kI [S, D_I] (contiguous), cand int32 with
 *   every used entry in [0, S) (else SA_DEV_INDEX, entry skipped).
 *   n_cand[t] must lie in [0, ld_cand] and ld_scores >= ld_cand. */
sa_status sa_indexer_scores_candidates(const sa_bf16 *qI, const sa_bf16 *w,
                                       const sa_bf16 *kI, int T, int S,
                                       int H_I, int D_I, const int32_t *cand,
                                       int64_t ld_cand, const int32_t *n_cand,
                                       float *scores, int64_t ld_scores,
                                       int *dev_status, sa_stream stream);

/* Fine-pass scores of the two-stage selection, computed block by block on
 * the tensor cores: the same values and layout as sa_indexer_scores_candidates
 * applied to the candidates that sa_expand_blocks writes for the same
 * `blocks`, i.e. for query t at position p = S - T + t:
 *   scores[t*ld_scores + i*block + j] = I[t, blocks[t,i']*block + j] for the
 *   i-th valid kept block i' (j < block), then
 *   scores[t*ld_scores + n_kept*block + j] = I[t, (p/block)*block + j] for the
 *   query's own block, j <= p - (p/block)*block; other entries are not written.
 * ("What Fine-Grained Means": the fine pass scores tokens inside the coarse
 * candidates; "Sparse Attention in 2026", "The designs that shipped": the
 * loop runs over KV blocks and gathers the queries that chose each one.)
 * Each 64-token block's keys are read once and multiplied (tcgen05, TMEM)
 * against the gathered indexer queries of every query that kept it.
 *   qI [T, H_I, D_I], w [T, H_I], kI [S, D_I], blocks [T, keep] (ascending,
 *   -1 padded, ids < p/block), block = 64, keep <= 255, T < 2^24,
 *   ld_scores >= keep*block + block.
 *   workspace: device memory of at least sa_block_scores_workspace_bytes(T,
 *   S, keep) bytes, 256-byte aligned, caller-owned; it holds the per-block
 *   query lists (contents on entry do not matter).
 *   Errors: SA_ERR_WORKSPACE, SA_ERR_UNSUPPORTED (block != 64 ...); device
 *   SA_DEV_INDEX for a block id >= p/block (skipped), SA_DEV_TIMEOUT. */
size_t sa_block_scores_workspace_bytes(int T, int S, int keep);

sa_status sa_indexer_scores_blocks(const sa_bf16 *qI, const sa_bf16 *w,
                                   const sa_bf16 *kI, int T, int S, int H_I,
                                   int D_I, const int32_t *blocks, int keep,
                                   int block, float *scores,
                                   int64_t ld_scores, void *workspace,
                                   size_t workspace_bytes, int *dev_status,
                                   sa_stream stream);

/* ------------------------------------------------------------------------
 * Stage 2 -- top-K select ("Where Sparse Attention Is Actually Sparse": Top-K
 * caps how many history positions take part in exact attention)
 *
 *   For each row r, among columns 0 <= col < n_valid[r] of
 *   scores[r*ld_scores + col], keep the min(K, n_valid[r]) largest scores;
 *   equal scores are ranked by lower position.  The position of a column is
 *   the column itself, or cand_map[r*ld_cand + col] when cand_map != NULL, in
 *   which case each row of cand_map must be strictly ascending over its valid
 *   columns (as sa_expand_blocks writes it) so that "lower column" means
 *   "lower position" (SA_DEV_ORDER otherwise).
 *   topk[r*K + i], i < K: the kept positions in ascending order, then -1.
 *   The result is unique, so it is bit-exact.
 *
 *   n_valid   [rows] or NULL (NULL: causal rows at the last `rows` of
 *             `row_len` positions, n_valid = row_len - rows + r + 1).
 *   Order-preserving keys: NaN scores are not supported; -inf sorts last.
 *   Limits: row_len <= 524288; K >= 0.
 *   Rows of at most 1024 columns are selected by one warp holding the row
 *   in registers; longer rows are split over a thread-block cluster
 *   (1..16 CTAs, distributed shared memory for the histograms).  No
 *   workspace is needed.
 * ---------------------------------------------------------------------- */
sa_status sa_topk_select(const float *scores, int64_t ld_scores, int rows,
                         int row_len, const int32_t *n_valid,
                         const int32_t *cand_map, int64_t ld_cand, int K,
                         int32_t *topk, int *dev_status, sa_stream stream);

/* The same select over the two-stage candidates, given by the kept block ids
 * instead of a position map ("What Fine-Grained Means": the fine pass picks
 * top-K tokens inside the blocks the coarse pass kept).
 *
 *   T queries at positions p = S - T + t.  Row t's columns are the tokens of
 *   the valid ids of blocks[t*keep .. t*keep + keep) (as sa_topk_select wrote
 *   them: ascending, each < p / block, then -1 padding), `block` columns per
 *   id, followed by the query's own block p / block up to p -- the layout
 *   sa_indexer_scores_blocks writes its scores in.  Column c of the n =
 *   n_kept * block + (p % block + 1) valid columns is position
 *   blocks[t, c / block] * block + c % block (c < n_kept * block), else
 *   (p / block) * block + c - n_kept * block.
 *   scores: [T, ld_scores] fp32, ld_scores >= keep*block + block, a multiple
 *   of 4, 16-byte aligned.  topk: [T, K], ascending positions, then -1.
 *   Device errors: an id >= p / block sets SA_DEV_INDEX, ids out of order
 *   SA_DEV_ORDER.  Limits: keep*block + block <= 524288 (SA_ERR_UNSUPPORTED).
 *   No workspace; blocks may be NULL when keep == 0.
 */
sa_status sa_topk_select_blocks(const float *scores, int64_t ld_scores, int T,
                                int S, const int32_t *blocks, int keep,
                                int block, int K, int32_t *topk,
                                int *dev_status, sa_stream stream);

/* ------------------------------------------------------------------------
 * Stages 1 + 2 fused, decode -- indexer scores and top-K select in one
 * kernel ("A Guide to Sparse Attention in Large Models", section 4.3: the
 * fused operator; "Where Sparse Attention Is Actually Sparse": the indexer
 * feeds Top-K).  The scores are never written to memory.
 *
 *   For each sequence b (one query each):
 *     I_b[s] = sum_{j < H_I} w[b,j] * max(0, sum_{c < D_I} qI[b,j,c] * kI_b[s,c])
 *   for 0 <= s < seq_lens[b], then topk[b*K + i], i < K: the min(K,
 *   seq_lens[b]) positions of the largest I_b[s], equal scores ranked by
 *   lower position, in ascending order, then -1.
 *   The same result as sa_indexer_scores (T = 1, n_valid = seq_lens)
 *   followed by sa_topk_select whenever the fp32 sums are exact (e.g. the
 *   integer-valued inputs of the tests); otherwise the two may order their
 *   sums differently.
 *
 *   qI        [B, H_I, D_I] bf16, 16-byte aligned; w [B, H_I] bf16
 *   kI        contiguous (page_table == NULL): [B, S, D_I] bf16, 16-byte
 *             aligned; paged: a pool [pool_pages, 64, D_I] through
 *             page_table [B, max_pages] (page_size must be 64)
 *   seq_lens  [B] keys per sequence, 0 .. S
 *   Limits: H_I <= 8, D_I in {64, 128}, S <= 524288 (and shared memory for
 *   the longest rows with D_I = 128: SA_ERR_UNSUPPORTED when it does not fit).
 *   Each sequence's row is split over a thread-block cluster; every CTA
 *   computes the scores of its chunk of keys on the tensor cores (mma.sync
 *   bf16 -> fp32) into shared memory and selects there.  No workspace.
 *   Errors: SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_CUDA; device:
 *   SA_DEV_INDEX for a seq_lens entry outside [0, S] or a page id outside
 *   [0, pool_pages) among the pages of the keys that are scored (a sequence
 *   of at most K keys keeps all of them without reading its pages).
 * ---------------------------------------------------------------------- */
sa_status sa_indexer_topk_decode(const sa_bf16 *qI, const sa_bf16 *w,
                                 const sa_bf16 *kI, const int32_t *page_table,
                                 int max_pages, int pool_pages, int page_size,
                                 int B, int S, int H_I, int D_I,
                                 const int32_t *seq_lens, int K,
                                 int32_t *topk, int *dev_status,
                                 sa_stream stream);

/* ------------------------------------------------------------------------
 * Stage 3a -- sparse attention, prefill
 *
 *   Query t (t < T) sits at position p = S - T + t.  Its key set is
 *     S(t) = {s in topk[t, :] : 0 <= s <= p - W} U {max(0, p-W+1) .. p}
 *   (top-K entries inside the window are taken once, from the window), and
 *     out[t,h,:] = sum_{s in S(t)} softmax_s(q[t,h,:] . k[s,:] * scale) v[s,:]
 *   for every head h < Hq; all heads share S(t) and the single KV head.
 *   lse[t,h] = log(sum_s exp(q.k*scale)) (natural log), if lse != NULL.
 *   q [T, Hq, d], k/v [S, d], topk [T, K] ascending, -1 padded (as
 *   sa_topk_select writes it), out [T, Hq, d] bf16, lse [T, Hq] fp32.
 *   Softmax and accumulation are fp32; probabilities are rounded to bf16 for
 *   the P.V product; out is rounded to bf16 (nearest even).
 *   Two kinds of kernel compute this.  Gathered: each query's selected K/V
 *   rows are gathered into shared memory (the only kind when workspace is
 *   NULL): on tcgen05 tiles with keys on M for d = 128, Hq <= 32, K <= 2048,
 *   else on mma.sync tiles.  Masked tensor-core tiles: when every query keeps a large share of
 *   its causal keys (S * Hq <= 256 * (K + W), Hq in {4, 8, 16, 32}, d in
 *   {64, 128}), groups of 128 / Hq queries stream the causal K/V once in
 *   128-key tiles through tcgen05 MMAs, masked by a per-query selection
 *   bitmap that is built in `workspace`.  Both give the same result within
 *   rounding.
 *   workspace: NULL, or device memory of at least
 *   sa_prefill_workspace_bytes(T, S, K, W, Hq, d) bytes (0 when the masked
 *   path does not apply), 256-byte aligned, caller-owned, contents ignored.
 *   Device errors: a top-K entry > p sets SA_DEV_INDEX and is skipped; a row
 *   that is not strictly ascending sets SA_DEV_ORDER.
 *   Limit: K + W <= 32768 (each query's key list is held in shared memory). 
 *   Every key set must be non-empty (a softmax over no keys is undefined):
 *   K + W = 0 returns SA_ERR_INVALID_ARG, and with W = 0 every top-K row
 *   must hold a valid entry (rows from sa_topk_select always do, since
 *   they keep min(K, p + 1) positions <= p); the out and lse rows of a query
 *   whose set is empty anyway are unspecified.
 * ---------------------------------------------------------------------- */
size_t sa_prefill_workspace_bytes(int T, int S, int K, int W, int Hq, int d);

sa_status sa_sparse_attn_prefill(const sa_bf16 *q, const sa_bf16 *k,
                                 const sa_bf16 *v, const int32_t *topk, int K,
                                 int W, int T, int S, int Hq, int d,
                                 float scale, sa_bf16 *out, float *lse,
                                 void *workspace, size_t workspace_bytes,
                                 int *dev_status, sa_stream stream);

/* ------------------------------------------------------------------------
 * Stage 3b -- sparse attention, decode (one new query per sequence)
 *
 *   Sequence b has seq_lens[b] tokens; its query sits at p = seq_lens[b] - 1
 *   (its own k/v/kI already appended).  Key set and output as in prefill.
 *   k_cache/v_cache: contiguous (page_table == NULL) [B, S_max, d]; paged:
 *   pools [P, page_size, d] addressed through page_table [B, max_pages].
 *   Each sequence's selection is split into chunks processed by separate
 *   CTAs, whose partial softmax states are merged by log-sum-exp.  When
 *   every chunk fits one CTA of a thread-block cluster (G = min(16,
 *   max(ceil((K+W)/128), ceil(Hq/8))) CTAs per sequence, at most 1024 keys
 *   each), the merge runs inside the same kernel through distributed shared
 *   memory and `workspace` is not touched.  Otherwise the partial states go to
 *   `workspace` and a second kernel merges them.  workspace: device memory of
 *   at least
 *   sa_decode_workspace_bytes(B, Hq, d, K, W) bytes, 256-byte aligned, owned
 *   by the caller; contents on entry do not matter.
 *   Errors: SA_ERR_WORKSPACE if too small; SA_ERR_UNSUPPORTED if B * S_max
 *   (contiguous) or pool_pages * 64 (paged) exceeds INT32_MAX rows; device
 *   SA_DEV_INDEX for a bad top-K entry or page id (skipped), SA_DEV_ORDER for
 *   a non-ascending row.
 * ---------------------------------------------------------------------- */
size_t sa_decode_workspace_bytes(int B, int Hq, int d, int K, int W);

sa_status sa_sparse_attn_decode(const sa_bf16 *q, const sa_bf16 *k_cache,
                                const sa_bf16 *v_cache,
                                const int32_t *page_table, int max_pages,
                                int pool_pages, int page_size, int S_max,
                                const int32_t *seq_lens, const int32_t *topk,
                                int K, int W, int B, int Hq, int d,
                                float scale, sa_bf16 *out, float *lse,
                                void *workspace, size_t workspace_bytes,
                                int *dev_status, sa_stream stream);

/* ------------------------------------------------------------------------
 * Decode without a caller workspace.  The pages have no counterpart: this is
 * an interface convenience for callers that cannot allocate device memory --
 * for example a plugin inside an engine that has reserved the GPU's memory for
 * its own KV-cache pool and passes plugins only inputs and outputs, or a
 * latency-critical loop where cudaMalloc / cudaFree (which may synchronise
 * the device) must not run.
 *
 *   Same arguments, results and device errors as sa_sparse_attn_decode, minus
 *   the workspace.  The split partials go to one fixed device array of
 *   SA_DECODE_NOALLOC_SCRATCH_BYTES that every GPU loading this library holds
 *   until the process exits.  Calls needing more than that
 *   (sa_decode_workspace_bytes(B, Hq, d, K, W) > SA_DECODE_NOALLOC_SCRATCH_BYTES)
 *   return SA_ERR_WORKSPACE and enqueue nothing.
 *   All calls on a device share the array: calls that overlap on the GPU (two
 *   streams, two host threads) race and must be serialised by the caller.
 *   The array keeps the previous call's contents; nothing in it needs to start
 *   at zero.  The first call on a device looks up the array's address on that
 *   device (set-up, once per device); make that first call before any stream
 *   capture.  The address stays cached for the life of the process; after
 *   cudaDeviceReset on a device, do not call this entry point on it again.  This entry point never calls cudaMalloc, cudaFree or any
 *   allocating routine.
 * ---------------------------------------------------------------------- */
#define SA_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)

sa_status sa_sparse_attn_decode_noalloc(const sa_bf16 *q,
                                        const sa_bf16 *k_cache,
                                        const sa_bf16 *v_cache,
                                        const int32_t *page_table,
                                        int max_pages, int pool_pages,
                                        int page_size, int S_max,
                                        const int32_t *seq_lens,
                                        const int32_t *topk, int K, int W,
                                        int B, int Hq, int d, float scale,
                                        sa_bf16 *out, float *lse,
                                        int *dev_status, sa_stream stream);

/* ------------------------------------------------------------------------
 * Two-stage selection helpers ("What Fine-Grained Means": a coarse block pass
 * picks candidate regions cheaply, a fine pass picks top-K tokens inside
 * them; section 2 "Learned Block Routing": blocks are mean-pooled over
 * complete blocks and scored by dot product).
 * ---------------------------------------------------------------------- */

/* kB[b, c] = bf16(mean of kI[b*block + i, c], i < block) for the S/block
 * complete blocks (a partial tail block is dropped).  The mean is an fp32 sum
 * divided by `block`, rounded to bf16 (exact for integer-valued keys with
 * |sum| <= 256 and a power-of-two block). */
sa_status sa_pool_index_keys(const sa_bf16 *kI, int S, int D_I, int block,
                             sa_bf16 *kB, sa_stream stream);

/* n_blocks[t] = floor((S - T + t) / block): the number of complete blocks
 * that lie entirely before the block holding query t -- the coarse pass's
 * eligible blocks (and its n_valid for sa_indexer_scores / sa_topk_select). */
sa_status sa_coarse_block_counts(int T, int S, int block, int32_t *n_blocks,
                                 sa_stream stream);

/* Candidates of the fine pass for query t at position p = S - T + t:
 *   the tokens of the kept blocks (blocks[t, :keep], ascending, -1 padded, as
 *   sa_topk_select writes it), then the tokens of p's own block up to p.
 *   cand[t*ld_cand + i] for i < n_cand[t] (ascending); ld_cand >= keep*block +
 *   block.  A block id >= floor(p/block) sets SA_DEV_INDEX and is skipped. */
sa_status sa_expand_blocks(const int32_t *blocks, int T, int S, int keep,
                           int block, int32_t *cand, int64_t ld_cand,
                           int32_t *n_cand, int *dev_status, sa_stream stream);

/* ------------------------------------------------------------------------
 * Health check (no counterpart on the pages): one thread waits on a barrier
 * that nothing arrives at, giving up after limit_us microseconds (1 .. 10^6)
 * exactly as every pipeline wait in this library does; *dev_status then holds
 * SA_DEV_TIMEOUT and the CUDA context stays usable.
 * ---------------------------------------------------------------------- */
sa_status sa_selftest_wait_timeout(int limit_us, int *dev_status,
                                   sa_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* FINE_GRAINED_TOP_SA_H */
