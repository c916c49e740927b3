// internal.h -- launchers shared between the C-ABI layer (sa_api.cu) and the
// kernel files.  Nothing here is exported from libsa.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/sa.h"

namespace sa {

struct TopkArgs {
    const float *scores;
    int64_t ld;
    int rows, row_len;
    const int32_t *n_valid;
    const int32_t *cand;
    int64_t ld_cand;
    int K;
    int32_t *out;
    int *dev_status;
    int chunk;   // columns per CTA (set by the launcher)
    // two-stage candidates given by block ids instead of a position map:
    // columns are the tokens of the valid (ascending) ids of blocks[r, :keep],
    // then the query's own block up to its position p = S - rows + r
    bool by_blocks = false;
    const int32_t *blocks = nullptr;   // [rows, keep]; may be NULL when keep == 0
    int keep = 0, block = 0, S = 0;
    // fused indexer (decode, one query per row): the scores of row r are
    // computed in shared memory from qI [rows, H_I, D_I], w [rows, H_I] and
    // the row's keys of kI (contiguous [rows, f_S, D_I], or a pool of 64-key
    // pages through f_page_table [rows, f_max_pages]) instead of read from
    // `scores`; n_valid gives each row's key count
    bool fused = false;
    const uint16_t *f_qI = nullptr, *f_w = nullptr, *f_kI = nullptr;
    const int32_t *f_page_table = nullptr;
    int f_max_pages = 0, f_pool_pages = 0, f_HI = 0, f_DI = 0, f_S = 0;
    int ring_off = 0;   // (set by the launcher) words from the chunk start to the key-tile ring
};
sa_status launch_topk(TopkArgs a, cudaStream_t st);
int topk_max_row_len();

struct IndexerArgs {
    const void *qI, *kI;   // bf16 or e4m3 elements (fp8)
    const uint16_t *w;
    bool fp8;
    const int32_t *page_table;
    int max_pages, pool_pages, page_size;
    int B, T, S, H_I, D_I;
    const int32_t *n_valid;
    float *scores;
    int64_t ld;
    int *dev_status;
};
sa_status launch_indexer(const IndexerArgs &a, cudaStream_t st);
sa_status launch_convert_e4m3(const uint16_t *src, uint8_t *dst, int64_t n, cudaStream_t st);

struct CandArgs {
    const uint16_t *qI, *w, *kI;
    int T, S, H_I, D_I;
    const int32_t *cand;
    int64_t ld_cand;
    const int32_t *n_cand;
    float *scores;
    int64_t ld;
    int *dev_status;
};
sa_status launch_indexer_candidates(const CandArgs &a, cudaStream_t st);

struct BlockScoreArgs {
    const uint16_t *qI, *w, *kI;
    int T, S, H_I, D_I;
    const int32_t *blocks;
    int keep;
    float *scores;
    int64_t ld;
    void *workspace;
    int *dev_status;
};
size_t block_scores_workspace_bytes(int T, int S, int keep);
sa_status launch_block_scores(const BlockScoreArgs &a, cudaStream_t st);

struct PrefillArgs {
    const uint16_t *q, *k, *v;
    const int32_t *topk;
    int K, W, T, S, Hq, d;
    float scale;
    uint16_t *out;
    float *lse;
    void *workspace;          // selection bitmap for the masked tensor-core path, or NULL
    size_t workspace_bytes;
    int *dev_status;
};
sa_status launch_prefill(const PrefillArgs &a, cudaStream_t st);
bool prefill_tc_supported(const PrefillArgs &a);
size_t prefill_tc_workspace_bytes(int T, int S);
sa_status launch_prefill_tc(const PrefillArgs &a, cudaStream_t st);
bool prefill_gather_supported(const PrefillArgs &a);
sa_status launch_prefill_gather(const PrefillArgs &a, cudaStream_t st);

struct DecodeArgs {
    const uint16_t *q, *k, *v;
    const int32_t *page_table;
    int max_pages, pool_pages, page_size, S_max;
    const int32_t *seq_lens, *topk;
    int K, W, B, Hq, d;
    float scale;
    uint16_t *out;
    float *lse;
    void *workspace;
    int *dev_status;
    bool force_split_k = false;   // always take the split-K path through `workspace`
};
size_t decode_workspace_bytes(int B, int Hq, int d, int K, int W);
sa_status launch_decode(const DecodeArgs &a, cudaStream_t st);

// Argument rules shared by every decode entry point (with or without a caller
// workspace): SA_OK when the call may proceed to its workspace checks.  A call
// with B == 0 passes and enqueues nothing.
inline sa_status check_decode_args(const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *page_table, int max_pages, int pool_pages, int page_size,
                                   int S_max, const int32_t *seq_lens, const int32_t *topk, int K, int W, int B,
                                   int Hq, int d, const void *out) {
    if (K < 0 || W < 0 || B < 0 || S_max < 0) return SA_ERR_INVALID_ARG;
    if (!(d == 64 || d == 128) || Hq < 1 || Hq > 64) return SA_ERR_UNSUPPORTED;
    if (B == 0) return SA_OK;
    if (!q || !k_cache || !v_cache || !seq_lens || !out || (K > 0 && !topk)) return SA_ERR_INVALID_ARG;
    const uintptr_t mis = (reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k_cache) |
                           reinterpret_cast<uintptr_t>(v_cache)) & 15u;
    if (mis) return SA_ERR_INVALID_ARG;
    if (page_table) {
        if (page_size != 64) return SA_ERR_UNSUPPORTED;
        if (max_pages <= 0 || pool_pages <= 0) return SA_ERR_INVALID_ARG;
        if ((int64_t)pool_pages * 64 > INT32_MAX) return SA_ERR_UNSUPPORTED;
    } else if ((int64_t)B * S_max > INT32_MAX) {
        return SA_ERR_UNSUPPORTED;
    }
    return SA_OK;
}

sa_status launch_pool(const uint16_t *kI, int S, int D_I, int block, uint16_t *kB, cudaStream_t st);
sa_status launch_block_counts(int T, int S, int block, int32_t *n_blocks, cudaStream_t st);
sa_status launch_expand(const int32_t *blocks, int T, int S, int keep, int block, int32_t *cand,
                        int64_t ld_cand, int32_t *n_cand, int *dev_status, cudaStream_t st);

inline sa_status cuda_ok(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

// Raise a kernel's dynamic shared-memory limit (and allow clusters wider than
// 8 CTAs) on the current device.  The attributes are set once per device and
// kernel; later launches skip the runtime calls.  Concurrent first calls may
// both set the same attributes, which is harmless.
template <auto Kern>
cudaError_t prepare_kernel(size_t smem, bool wide_cluster) {
    static std::atomic<unsigned> done[64];   // per device: bit 31 wide clusters, low bits smem bytes
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned st = (dev >= 0 && dev < 64) ? done[dev].load(std::memory_order_relaxed) : 0u;
    const unsigned have_smem = st & 0x7fffffffu;
    const bool have_wide = (st >> 31) != 0;
    if (have_smem >= smem && (!wide_cluster || have_wide)) return cudaSuccess;
    if (smem > have_smem) {
        e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    if (wide_cluster && !have_wide) {
        e = cudaFuncSetAttribute(Kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    if (dev >= 0 && dev < 64) {
        const unsigned ns = (unsigned)(smem > have_smem ? smem : have_smem) |
                            ((wide_cluster || have_wide) ? 0x80000000u : 0u);
        done[dev].store(ns, std::memory_order_relaxed);
    }
    return cudaSuccess;
}

}  // namespace sa
