// two_stage.cu -- the coarse-then-fine selection helpers.
//
// "Why fine-grained sparse attention is becoming the new ..." (mg6.net),
// section "What Fine-Grained Means": a coarse block-selection pass finds
// candidate regions cheaply, then a fine pass picks top-K tokens inside them;
// section 2 "Learned Block Routing": block keys are the mean over complete
// blocks (a partial tail block is dropped), scored by dot product.
//
// The coarse scores reuse the indexer kernel with the pooled keys in place of
// kI and n_valid = the eligible block count; the coarse top-k reuses the
// top-K kernel.  These kernels supply the pieces in between.
#include "internal.h"
#include "ptx.cuh"

namespace sa {

// kB[blk, c] = bf16(fp32 sum of the block's rows / block), one thread per (blk, c)
__global__ void pool_keys_kernel(const uint16_t *__restrict__ kI, int n_blocks, int D_I, int block,
                                 uint16_t *__restrict__ kB) {
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (int64_t)n_blocks * D_I) return;
    const int blk = (int)(idx / D_I), c = (int)(idx % D_I);
    const uint16_t *src = kI + (int64_t)blk * block * D_I + c;
    float s = 0.f;
    for (int i = 0; i < block; ++i) s += __uint_as_float((uint32_t)src[(int64_t)i * D_I] << 16);
    const __nv_bfloat16 m = __float2bfloat16_rn(s / (float)block);
    kB[idx] = *reinterpret_cast<const uint16_t *>(&m);
}

__global__ void block_counts_kernel(int T, int S, int block, int32_t *__restrict__ n_blocks) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t < T) n_blocks[t] = (S - T + t) / block;
}

// One warp per query: compact the valid kept block ids (in order), then write
// their tokens followed by the query's own block up to its position.
__global__ void __launch_bounds__(256) expand_kernel(const int32_t *__restrict__ blocks, int T, int S, int keep,
                                                     int block, int32_t *__restrict__ cand, int64_t ld_cand,
                                                     int32_t *__restrict__ n_cand, int *dev_status) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    const int p = S - T + t;
    const int own = p / block;
    const int32_t *br = blocks + (int64_t)t * keep;
    int32_t *out = cand + (int64_t)t * ld_cand;
    int n_kept = 0;
    int prev = -1;
    for (int i0 = 0; i0 < keep; i0 += 32) {
        const int i = i0 + lane;
        int bid = (i < keep) ? br[i] : -1;
        bool ok = bid >= 0;
        if (ok && bid >= own) { report(dev_status, SA_DEV_INDEX); ok = false; }
        // strictly ascending among the valid ids (checked against the previous lane / round)
        const int left = __shfl_up_sync(0xffffffffu, ok ? bid : -1, 1);
        const int before = (lane == 0) ? prev : left;
        if (ok && before >= 0 && before >= bid) report(dev_status, SA_DEV_ORDER);
        const uint32_t bal = __ballot_sync(0xffffffffu, ok);
        const int slot = n_kept + __popc(bal & lanemask_lt());
        // each valid id writes its block's tokens; lanes cooperate per block below
        for (int src = 0; src < 32; ++src) {
            if (!((bal >> src) & 1u)) continue;
            const int b_id = __shfl_sync(0xffffffffu, bid, src);
            const int sl = __shfl_sync(0xffffffffu, slot, src);
            for (int j = lane; j < block; j += 32) out[(int64_t)sl * block + j] = b_id * block + j;
        }
        n_kept += __popc(bal);
        const int last_valid = bal ? 31 - __clz(bal) : -1;
        if (last_valid >= 0) prev = __shfl_sync(0xffffffffu, bid, last_valid);
    }
    const int own0 = own * block;
    const int n_own = p - own0 + 1;
    for (int j = lane; j < n_own; j += 32) out[(int64_t)n_kept * block + j] = own0 + j;
    if (lane == 0) n_cand[t] = n_kept * block + n_own;
}

sa_status launch_pool(const uint16_t *kI, int S, int D_I, int block, uint16_t *kB, cudaStream_t st) {
    const int nb = S / block;
    const int64_t n = (int64_t)nb * D_I;
    if (n == 0) return SA_OK;
    pool_keys_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(kI, nb, D_I, block, kB);
    return cuda_ok(cudaGetLastError());
}

sa_status launch_block_counts(int T, int S, int block, int32_t *n_blocks, cudaStream_t st) {
    if (T == 0) return SA_OK;
    block_counts_kernel<<<(T + 255) / 256, 256, 0, st>>>(T, S, block, n_blocks);
    return cuda_ok(cudaGetLastError());
}

sa_status launch_expand(const int32_t *blocks, int T, int S, int keep, int block, int32_t *cand, int64_t ld_cand,
                        int32_t *n_cand, int *dev_status, cudaStream_t st) {
    if (T == 0) return SA_OK;
    expand_kernel<<<(T + 7) / 8, 256, 0, st>>>(blocks, T, S, keep, block, cand, ld_cand, n_cand, dev_status);
    return cuda_ok(cudaGetLastError());
}

}  // namespace sa
