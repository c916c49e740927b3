// sa_api.cu -- the exported C ABI (include/sa.h): synchronous argument checks,
// then kernel launches on the caller's stream.  Nothing is enqueued when a
// check fails; no C++ exception crosses the boundary; nothing is allocated.
#include <stdint.h>

#include "../../include/sa.h"
#include "internal.h"

using namespace sa;

namespace {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool head_dim_ok(int d) { return d == 64 || d == 128; }
inline bool index_dim_ok(int D) { return D == 32 || D == 64; }
inline bool index_dim_fp8_ok(int D) { return D == 64 || D == 128; }
inline bool index_heads_ok(int H) { return H == 1 || H == 2 || H == 4 || H == 8; }
inline cudaStream_t cs(sa_stream s) { return reinterpret_cast<cudaStream_t>(s); }

template <class F>
sa_status guarded(F &&f) {
    try {
        return f();
    } catch (...) {
        return SA_ERR_CUDA;
    }
}

}  // namespace

extern "C" {

const char *sa_status_string(sa_status s) {
    switch (s) {
        case SA_OK: return "SA_OK";
        case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
        case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
        case SA_ERR_CUDA: return "SA_ERR_CUDA";
        case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
        case SA_ERR_INDEX: return "SA_ERR_INDEX";
        case SA_ERR_WORKSPACE: return "SA_ERR_WORKSPACE";
    }
    return "SA_ERR_UNKNOWN";
}

sa_status sa_dev_status_decode(int word) {
    if (word & SA_DEV_TIMEOUT) return SA_ERR_TIMEOUT;
    if (word & (SA_DEV_INDEX | SA_DEV_ORDER)) return SA_ERR_INDEX;
    return SA_OK;
}

int sa_version(void) { return 101; }

// Shared by the bf16 and e4m3 entry points: identical argument rules, the
// element type only changes the row bytes the kernel sees.
static sa_status indexer_scores(const void *qI, const sa_bf16 *w, const void *kI, bool fp8,
                                const int32_t *page_table, int max_pages, int pool_pages, int page_size, int B,
                                int T, int S, int H_I, int D_I, const int32_t *n_valid, float *scores,
                                int64_t ld_scores, int *dev_status, sa_stream stream) {
    if (B < 0 || T < 0 || S < 0 || ld_scores < S || (ld_scores & 3)) return SA_ERR_INVALID_ARG;
    if (!index_heads_ok(H_I) || !(fp8 ? index_dim_fp8_ok(D_I) : index_dim_ok(D_I))) return SA_ERR_UNSUPPORTED;
    if (B == 0 || T == 0 || S == 0) return SA_OK;
    if (!qI || !w || !kI || !scores || !aligned16(qI) || !aligned16(kI)) return SA_ERR_INVALID_ARG;
    if (n_valid == nullptr && T > S) return SA_ERR_INVALID_ARG;
    if ((int64_t)B * T * H_I > INT32_MAX || (int64_t)B * S > INT32_MAX) return SA_ERR_UNSUPPORTED;
    if (page_table) {
        if (page_size != 64) return SA_ERR_UNSUPPORTED;
        if (max_pages <= 0 || pool_pages <= 0 || (int64_t)max_pages * 64 < S) return SA_ERR_INVALID_ARG;
        if ((int64_t)pool_pages * 64 > INT32_MAX) return SA_ERR_UNSUPPORTED;
    }
    return guarded([&] {
        IndexerArgs a;
        a.qI = qI; a.w = w; a.kI = kI; a.fp8 = fp8; a.page_table = page_table;
        a.max_pages = max_pages; a.pool_pages = pool_pages; a.page_size = page_size;
        a.B = B; a.T = T; a.S = S; a.H_I = H_I; a.D_I = D_I;
        a.n_valid = n_valid; a.scores = scores; a.ld = ld_scores; a.dev_status = dev_status;
        return launch_indexer(a, cs(stream));
    });
}

sa_status sa_indexer_scores(const sa_bf16 *qI, const sa_bf16 *w, const sa_bf16 *kI, const int32_t *page_table,
                            int max_pages, int pool_pages, int page_size, int B, int T, int S, int H_I, int D_I,
                            const int32_t *n_valid, float *scores, int64_t ld_scores, int *dev_status,
                            sa_stream stream) {
    return indexer_scores(qI, w, kI, false, page_table, max_pages, pool_pages, page_size, B, T, S, H_I, D_I,
                          n_valid, scores, ld_scores, dev_status, stream);
}

sa_status sa_indexer_scores_fp8(const sa_e4m3 *qI, const sa_bf16 *w, const sa_e4m3 *kI,
                                const int32_t *page_table, int max_pages, int pool_pages, int page_size, int B,
                                int T, int S, int H_I, int D_I, const int32_t *n_valid, float *scores,
                                int64_t ld_scores, int *dev_status, sa_stream stream) {
    return indexer_scores(qI, w, kI, true, page_table, max_pages, pool_pages, page_size, B, T, S, H_I, D_I,
                          n_valid, scores, ld_scores, dev_status, stream);
}

sa_status sa_convert_e4m3(const sa_bf16 *src, sa_e4m3 *dst, int64_t n, sa_stream stream) {
    if (n < 0) return SA_ERR_INVALID_ARG;
    if (n == 0) return SA_OK;
    if (!src || !dst) return SA_ERR_INVALID_ARG;
    return guarded([&] { return launch_convert_e4m3(src, dst, n, cs(stream)); });
}

sa_status sa_indexer_scores_candidates(const sa_bf16 *qI, const sa_bf16 *w, const sa_bf16 *kI, int T, int S,
                                       int H_I, int D_I, const int32_t *cand, int64_t ld_cand,
                                       const int32_t *n_cand, float *scores, int64_t ld_scores, int *dev_status,
                                       sa_stream stream) {
    if (T < 0 || S < 0 || ld_cand < 0 || ld_scores < ld_cand) return SA_ERR_INVALID_ARG;
    if (!index_heads_ok(H_I) || !index_dim_ok(D_I)) return SA_ERR_UNSUPPORTED;
    if (T == 0) return SA_OK;
    if (!qI || !w || !kI || !cand || !n_cand || !scores || !aligned16(kI)) return SA_ERR_INVALID_ARG;
    return guarded([&] {
        CandArgs a;
        a.qI = qI; a.w = w; a.kI = kI; a.T = T; a.S = S; a.H_I = H_I; a.D_I = D_I;
        a.cand = cand; a.ld_cand = ld_cand; a.n_cand = n_cand; a.scores = scores; a.ld = ld_scores;
        a.dev_status = dev_status;
        return launch_indexer_candidates(a, cs(stream));
    });
}

size_t sa_block_scores_workspace_bytes(int T, int S, int keep) {
    if (T < 0 || S < 0 || keep < 0) return 0;
    return block_scores_workspace_bytes(T, S, keep);
}

sa_status sa_indexer_scores_blocks(const sa_bf16 *qI, const sa_bf16 *w, const sa_bf16 *kI, int T, int S, int H_I,
                                   int D_I, const int32_t *blocks, int keep, int block, float *scores,
                                   int64_t ld_scores, void *workspace, size_t workspace_bytes, int *dev_status,
                                   sa_stream stream) {
    if (T < 0 || S < T || keep < 0 || block <= 0) return SA_ERR_INVALID_ARG;
    if (!index_heads_ok(H_I) || !index_dim_ok(D_I) || block != 64 || keep > 255 || T >= (1 << 24))
        return SA_ERR_UNSUPPORTED;
    if (ld_scores < (int64_t)keep * block + block) return SA_ERR_INVALID_ARG;
    if (T == 0) return SA_OK;
    if (!qI || !w || !kI || !scores || (keep > 0 && !blocks) || !aligned16(qI) || !aligned16(kI))
        return SA_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SA_ERR_INVALID_ARG;
    if (workspace_bytes < block_scores_workspace_bytes(T, S, keep)) return SA_ERR_WORKSPACE;
    return guarded([&] {
        BlockScoreArgs a;
        a.qI = qI; a.w = w; a.kI = kI; a.T = T; a.S = S; a.H_I = H_I; a.D_I = D_I; a.blocks = blocks;
        a.keep = keep; a.scores = scores; a.ld = ld_scores; a.workspace = workspace; a.dev_status = dev_status;
        return launch_block_scores(a, cs(stream));
    });
}

sa_status sa_topk_select(const float *scores, int64_t ld_scores, int rows, int row_len, const int32_t *n_valid,
                         const int32_t *cand_map, int64_t ld_cand, int K, int32_t *topk, int *dev_status,
                         sa_stream stream) {
    if (rows < 0 || row_len < 0 || K < 0 || ld_scores < row_len || (ld_scores & 3)) return SA_ERR_INVALID_ARG;
    if (cand_map && ld_cand < row_len) return SA_ERR_INVALID_ARG;
    if (row_len > topk_max_row_len()) return SA_ERR_UNSUPPORTED;
    if (rows == 0 || K == 0) return SA_OK;
    if (!scores || !topk || !aligned16(scores)) return SA_ERR_INVALID_ARG;
    return guarded([&] {
        TopkArgs a;
        a.scores = scores; a.ld = ld_scores; a.rows = rows; a.row_len = row_len; a.n_valid = n_valid;
        a.cand = cand_map; a.ld_cand = ld_cand; a.K = K; a.out = topk; a.dev_status = dev_status; a.chunk = 0;
        return launch_topk(a, cs(stream));
    });
}

sa_status sa_topk_select_blocks(const float *scores, int64_t ld_scores, int T, int S, const int32_t *blocks, int keep,
                                int block, int K, int32_t *topk, int *dev_status, sa_stream stream) {
    if (T < 0 || S < T || keep < 0 || block <= 0 || K < 0) return SA_ERR_INVALID_ARG;
    const int64_t row_len = (int64_t)keep * block + block;
    if (ld_scores < row_len || (ld_scores & 3)) return SA_ERR_INVALID_ARG;
    if (row_len > topk_max_row_len()) return SA_ERR_UNSUPPORTED;
    if (T == 0 || K == 0) return SA_OK;
    if (!scores || !topk || (keep > 0 && !blocks) || !aligned16(scores)) return SA_ERR_INVALID_ARG;
    return guarded([&] {
        TopkArgs a;
        a.scores = scores; a.ld = ld_scores; a.rows = T; a.row_len = (int)row_len; a.n_valid = nullptr;
        a.cand = nullptr; a.ld_cand = 0; a.K = K; a.out = topk; a.dev_status = dev_status; a.chunk = 0;
        a.by_blocks = true; a.blocks = keep > 0 ? blocks : nullptr; a.keep = keep; a.block = block; a.S = S;
        return launch_topk(a, cs(stream));
    });
}

sa_status sa_indexer_topk_decode(const sa_bf16 *qI, const sa_bf16 *w, const sa_bf16 *kI, const int32_t *page_table,
                                 int max_pages, int pool_pages, int page_size, int B, int S, int H_I, int D_I,
                                 const int32_t *seq_lens, int K, int32_t *topk, int *dev_status, sa_stream stream) {
    if (B < 0 || S < 0 || K < 0 || H_I < 1) return SA_ERR_INVALID_ARG;
    if (page_table && (page_size != 64 || max_pages < 0 || pool_pages < 1 || (int64_t)max_pages * 64 < S))
        return page_size != 64 ? SA_ERR_UNSUPPORTED : SA_ERR_INVALID_ARG;
    if (H_I > 8 || (D_I != 64 && D_I != 128) || S > topk_max_row_len()) return SA_ERR_UNSUPPORTED;
    if (B == 0 || K == 0) return SA_OK;
    if (!qI || !w || !kI || !seq_lens || !topk) return SA_ERR_INVALID_ARG;
    if (!aligned16(qI) || !aligned16(kI) || (reinterpret_cast<uintptr_t>(w) & 1u)) return SA_ERR_INVALID_ARG;
    return guarded([&] {
        TopkArgs a;
        a.scores = nullptr; a.ld = 0; a.rows = B; a.row_len = S; a.n_valid = seq_lens;
        a.cand = nullptr; a.ld_cand = 0; a.K = K; a.out = topk; a.dev_status = dev_status; a.chunk = 0;
        a.fused = true; a.f_qI = qI; a.f_w = w; a.f_kI = kI; a.f_page_table = page_table;
        a.f_max_pages = max_pages; a.f_pool_pages = pool_pages; a.f_HI = H_I; a.f_DI = D_I; a.f_S = S;
        return launch_topk(a, cs(stream));
    });
}

size_t sa_prefill_workspace_bytes(int T, int S, int K, int W, int Hq, int d) {
    if (T < 0 || S < 0 || K < 0 || W < 0) return 0;
    PrefillArgs a = {};
    a.T = T; a.S = S; a.K = K; a.W = W; a.Hq = Hq; a.d = d;
    return prefill_tc_supported(a) ? prefill_tc_workspace_bytes(T, S) : 0;
}

sa_status sa_sparse_attn_prefill(const sa_bf16 *q, const sa_bf16 *k, const sa_bf16 *v, const int32_t *topk, int K,
                                 int W, int T, int S, int Hq, int d, float scale, sa_bf16 *out, float *lse,
                                 void *workspace, size_t workspace_bytes, int *dev_status, sa_stream stream) {
    if (K < 0 || W < 0 || T < 0 || S < 0 || T > S) return SA_ERR_INVALID_ARG;
    if (T > 0 && K + W == 0) return SA_ERR_INVALID_ARG;   // every key set would be empty
    if (!head_dim_ok(d) || Hq < 1 || Hq > 64) return SA_ERR_UNSUPPORTED;
    if ((int64_t)K + W > 32768) return SA_ERR_UNSUPPORTED;   // the per-query key list lives in shared memory
    if (T == 0) return SA_OK;
    if (!q || !k || !v || !out || (K > 0 && !topk)) return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SA_ERR_INVALID_ARG;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SA_ERR_INVALID_ARG;
    return guarded([&] {
        PrefillArgs a;
        a.q = q; a.k = k; a.v = v; a.topk = topk; a.K = K; a.W = W; a.T = T; a.S = S; a.Hq = Hq; a.d = d;
        a.scale = scale; a.out = out; a.lse = lse; a.dev_status = dev_status;
        a.workspace = workspace;
        a.workspace_bytes = workspace_bytes;
        return launch_prefill(a, cs(stream));
    });
}

size_t sa_decode_workspace_bytes(int B, int Hq, int d, int K, int W) {
    if (B < 0 || Hq < 0 || d < 0 || K < 0 || W < 0) return 0;
    return decode_workspace_bytes(B, Hq, d, K, W);
}

sa_status sa_sparse_attn_decode(const sa_bf16 *q, const sa_bf16 *k_cache, const sa_bf16 *v_cache,
                                const int32_t *page_table, int max_pages, int pool_pages, int page_size, int S_max,
                                const int32_t *seq_lens, const int32_t *topk, int K, int W, int B, int Hq, int d,
                                float scale, sa_bf16 *out, float *lse, void *workspace, size_t workspace_bytes,
                                int *dev_status, sa_stream stream) {
    const sa_status chk = check_decode_args(q, k_cache, v_cache, page_table, max_pages, pool_pages, page_size,
                                            S_max, seq_lens, topk, K, W, B, Hq, d, out);
    if (chk != SA_OK || B == 0) return chk;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SA_ERR_INVALID_ARG;
    if (workspace_bytes < decode_workspace_bytes(B, Hq, d, K, W)) return SA_ERR_WORKSPACE;
    return guarded([&] {
        DecodeArgs a;
        a.q = q; a.k = k_cache; a.v = v_cache; a.page_table = page_table; a.max_pages = max_pages;
        a.pool_pages = pool_pages; a.page_size = page_size; a.S_max = page_table ? max_pages * 64 : S_max;
        a.seq_lens = seq_lens; a.topk = topk; a.K = K; a.W = W; a.B = B; a.Hq = Hq; a.d = d; a.scale = scale;
        a.out = out; a.lse = lse; a.workspace = workspace; a.dev_status = dev_status;
        return launch_decode(a, cs(stream));
    });
}

sa_status sa_pool_index_keys(const sa_bf16 *kI, int S, int D_I, int block, sa_bf16 *kB, sa_stream stream) {
    if (S < 0 || block <= 0) return SA_ERR_INVALID_ARG;
    if (!index_dim_ok(D_I)) return SA_ERR_UNSUPPORTED;
    if (S / block == 0) return SA_OK;
    if (!kI || !kB) return SA_ERR_INVALID_ARG;
    return guarded([&] { return launch_pool(kI, S, D_I, block, kB, cs(stream)); });
}

sa_status sa_coarse_block_counts(int T, int S, int block, int32_t *n_blocks, sa_stream stream) {
    if (T < 0 || S < T || block <= 0) return SA_ERR_INVALID_ARG;
    if (T == 0) return SA_OK;
    if (!n_blocks) return SA_ERR_INVALID_ARG;
    return guarded([&] { return launch_block_counts(T, S, block, n_blocks, cs(stream)); });
}

sa_status sa_expand_blocks(const int32_t *blocks, int T, int S, int keep, int block, int32_t *cand,
                           int64_t ld_cand, int32_t *n_cand, int *dev_status, sa_stream stream) {
    if (T < 0 || S < T || keep < 0 || block <= 0) return SA_ERR_INVALID_ARG;
    if (ld_cand < (int64_t)keep * block + block) return SA_ERR_INVALID_ARG;
    if (T == 0) return SA_OK;
    if (!cand || !n_cand || (keep > 0 && !blocks)) return SA_ERR_INVALID_ARG;
    return guarded([&] {
        return launch_expand(blocks, T, S, keep, block, cand, ld_cand, n_cand, dev_status, cs(stream));
    });
}

}  // extern "C"
