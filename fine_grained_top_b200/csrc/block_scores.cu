// block_scores.cu -- fine-pass indexer scores of the two-stage selection,
// computed block by block on the tensor cores.
//
// "Why fine-grained sparse attention is becoming the new ..." (mg6.net),
// section "What Fine-Grained Means": a coarse pass picks candidate blocks,
// then the fine pass scores individual tokens inside them.  "Sparse Attention
// in 2026" (Acing AI), "The designs that shipped", names the access pattern
// used here for MiniMax's kernels: loop over KV blocks and gather the queries
// that chose them ("KV-outer-gather-Q").
//
// Each query's candidates are whole 64-token blocks, so the score work is
// grouped by block: block b is read once into shared memory and multiplied
// against the gathered indexer queries of every query that kept it.
//   1. invert the kept-block lists: per block, the (query, slot) pairs that
//      use it (per-CTA shared-memory histograms, one global reservation per
//      block and CTA, then a scatter); the query's own block is included;
//   2. for each block and each group of 128 / H_I such queries:
//        D[(t,j), s] = qI[t,j] . kI[s]     M = 128 query-head rows (gathered),
//                                          N = 64 keys, K = D_I (tcgen05, TMEM)
//      and the epilogue reduces w[t,j] * ReLU(D) over the H_I heads of each
//      query (adjacent TMEM lanes) and writes the block's 64 scores into the
//      query's slot, the same layout sa_expand_blocks gives the candidates.
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

constexpr int kBlk = 64;              // tokens per block (one MMA N)
constexpr int kInvThreads = 1024;
constexpr int kInvRows = 1024;        // query rows per inversion CTA
constexpr int kScoreThreads = 128;    // 4 warps: one TMEM lane quadrant each

struct BlockWs {                      // carved out of the caller's workspace
    int32_t *cnt;                     // [nb] (query, slot) pairs per block
    int32_t *cursor;                  // [nb] fill position per block
    int32_t *off;                     // [nb + 1] start of each block's list
    uint32_t *list;                   // [T * (keep + 1)]: t << 8 | slot
};

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t block_scores_workspace_bytes(int T, int S, int keep) {
    const size_t nb = (size_t)S / kBlk + 1;
    return 3 * align256(nb * 4 + 4) + align256((size_t)T * (keep + 1) * 4);
}

static BlockWs carve(void *ws, int T, int S, int keep) {
    const size_t nb = (size_t)S / kBlk + 1;
    uint8_t *p = reinterpret_cast<uint8_t *>(ws);
    BlockWs w;
    w.cnt = reinterpret_cast<int32_t *>(p);
    p += align256(nb * 4 + 4);
    w.cursor = reinterpret_cast<int32_t *>(p);
    p += align256(nb * 4 + 4);
    w.off = reinterpret_cast<int32_t *>(p);
    p += align256(nb * 4 + 4);
    w.list = reinterpret_cast<uint32_t *>(p);
    (void)T; (void)keep;
    return w;
}

// The blocks of query row t (position p = S - T + t): the kept blocks
// (valid entries of blocks[t, :keep], each < p / 64) in slots 0.., then the
// own block p / 64 in the next slot.  Calls f(block, slot) for each.
template <class F>
__device__ __forceinline__ void for_each_block(const int32_t *blocks, int keep, int S, int T, int t,
                                               int *dev_status, F &&f) {
    const int own = (S - T + t) / kBlk;
    int slot = 0;
    for (int i = 0; i < keep; ++i) {
        const int b = blocks[(int64_t)t * keep + i];
        if (b < 0) continue;
        if (b >= own) { report(dev_status, SA_DEV_INDEX); continue; }
        f(b, slot++);
    }
    f(own, slot);
}

// Pass 1: per-block pair counts (shared-memory histogram per CTA).
__global__ void __launch_bounds__(kInvThreads) invert_count_kernel(const int32_t *blocks, int keep, int S, int T,
                                                                   int nb, BlockWs ws, int *dev_status) {
    extern __shared__ int32_t hist[];   // [nb]
    for (int i = threadIdx.x; i < nb; i += kInvThreads) hist[i] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kInvRows;
    for (int t = t0 + threadIdx.x; t < min(T, t0 + kInvRows); t += kInvThreads)
        for_each_block(blocks, keep, S, T, t, dev_status, [&](int b, int) { atomicAdd(&hist[b], 1); });
    __syncthreads();
    for (int i = threadIdx.x; i < nb; i += kInvThreads)
        if (hist[i]) atomicAdd(&ws.cnt[i], hist[i]);
}

// Pass 2: exclusive scan of the counts (one CTA); cursors start at the offsets.
__global__ void __launch_bounds__(kInvThreads) invert_scan_kernel(int nb, BlockWs ws) {
    __shared__ int32_t part[kInvThreads / 32];
    __shared__ int32_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < nb; base += kInvThreads) {
        const int i = base + threadIdx.x;
        const int v = i < nb ? ws.cnt[i] : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) part[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int p = lane < kInvThreads / 32 ? part[lane] : 0, q = p;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, q, o);
                if (lane >= o) q += y;
            }
            if (lane < kInvThreads / 32) part[lane] = q - p;
        }
        __syncthreads();
        const int excl = carry + part[warp] + x - v;
        if (i < nb) { ws.off[i] = excl; ws.cursor[i] = excl; }
        __syncthreads();
        if (threadIdx.x == kInvThreads - 1) carry = excl + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) ws.off[nb] = carry;
}

// Pass 3: scatter.  Each CTA counts its pairs per block again, reserves one
// range per block with a single global atomic, then fills it.
__global__ void __launch_bounds__(kInvThreads) invert_scatter_kernel(const int32_t *blocks, int keep, int S, int T,
                                                                     int nb, BlockWs ws, int *dev_status) {
    extern __shared__ int32_t sm[];     // hist[nb], base[nb]
    int32_t *hist = sm, *base = sm + nb;
    for (int i = threadIdx.x; i < nb; i += kInvThreads) hist[i] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kInvRows;
    for (int t = t0 + threadIdx.x; t < min(T, t0 + kInvRows); t += kInvThreads)
        for_each_block(blocks, keep, S, T, t, nullptr, [&](int b, int) { atomicAdd(&hist[b], 1); });
    __syncthreads();
    for (int i = threadIdx.x; i < nb; i += kInvThreads) {
        base[i] = hist[i] ? atomicAdd(&ws.cursor[i], hist[i]) : 0;
        hist[i] = 0;
    }
    __syncthreads();
    for (int t = t0 + threadIdx.x; t < min(T, t0 + kInvRows); t += kInvThreads)
        for_each_block(blocks, keep, S, T, t, nullptr, [&](int b, int slot) {
            const int pos = base[b] + atomicAdd(&hist[b], 1);
            ws.list[pos] = ((uint32_t)t << 8) | (uint32_t)slot;
        });
    (void)dev_status;
}

// Pass 4: scores.  A persistent CTA takes an equal range of the pairs; for
// each block in it, it loads the block's keys once and runs over its query
// groups with the next group's gather in flight while the current one is
// multiplied.
template <int D_I, int H_I>
__global__ void __launch_bounds__(kScoreThreads) block_scores_kernel(const uint16_t *qI, const uint16_t *w,
                                                                     const uint16_t *kI, int T, int S, int nb,
                                                                     BlockWs ws, float *scores, int64_t ld,
                                                                     int *dev_status) {
    constexpr int QG = 128 / H_I;                  // queries per group (M = 128 rows)
    constexpr int ROWB = D_I * 2;                  // 128 or 64 bytes per row
    constexpr int CH = ROWB / 16;                  // 16-byte chunks per row
    constexpr int A_BYTES = 128 * ROWB, B_BYTES = kBlk * ROWB;
    constexpr uint32_t SBO = 8 * ROWB;             // 8-row core group stride
    constexpr uint32_t LAYOUT = (D_I == 64) ? 2 : 4;
    constexpr uint32_t idesc = idesc_bf16_f32(128, kBlk);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sB = sm;                              // [64][D_I] keys of the block
    uint8_t *sA = sm + 1024 * ((B_BYTES + 1023) / 1024);   // [2][128][D_I] gathered queries
    __shared__ uint64_t mma_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ uint32_t s_entry[2][QG];            // (t << 8 | slot), 0xffffffff = none

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        mbar_init(&mma_bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_slot, 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_slot;

    // byte offset of chunk c of row r under the TMA-style swizzle the UMMA
    // descriptor expects (128B: c ^ (r & 7); 64B: c ^ ((r >> 1) & 3))
    auto swz = [](int r, int c) -> uint32_t {
        return (D_I == 64) ? (uint32_t)(r * ROWB + ((c ^ (r & 7)) << 4))
                           : (uint32_t)(r * ROWB + ((c ^ ((r >> 1) & 3)) << 4));
    };
    // the QG pairs of list entries [lo, min(lo + QG, hi)) into buffer buf
    auto gather_queries = [&](int lo, int hi, int buf) {
        if (tid < QG) s_entry[buf][tid] = (lo + tid < hi) ? ws.list[lo + tid] : 0xffffffffu;
        for (int idx = tid; idx < 128 * CH; idx += kScoreThreads) {
            const int r = idx / CH, c = idx % CH;
            const int e = lo + r / H_I;
            uint8_t *dst = sA + buf * A_BYTES + swz(r, c);
            if (e < hi) {
                const int t = (int)(ws.list[e] >> 8);
                cp_async16(dst, qI + ((int64_t)t * H_I + (r % H_I)) * D_I + c * 8);
            } else {
                *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
            }
        }
    };

    // This CTA's share: an equal contiguous range [p0, p1) of the (query,
    // slot) pairs of all blocks (the lists are grouped by block, and early
    // blocks are kept by many more queries than late ones, so whole blocks
    // per CTA would leave a few CTAs with most of the work).
    const int total = ws.off[nb];
    const int per = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int p0 = min(total, (int)blockIdx.x * per), p1 = min(total, p0 + per);
    int b0 = 0;   // the block whose list holds pair p0: the last b with off[b] <= p0
    {
        int hi_b = nb;
        while (hi_b - b0 > 1) {
            const int mid = (b0 + hi_b) >> 1;
            if (ws.off[mid] <= p0) b0 = mid;
            else hi_b = mid;
        }
    }
    uint32_t phase = 0;
    for (int b = b0; b < nb && p0 < p1; ++b) {
        const int r0 = max(ws.off[b], p0), r1 = min(ws.off[b + 1], p1);
        if (r0 >= p1) break;
        if (r1 <= r0) continue;
        const int groups = (r1 - r0 + QG - 1) / QG;
        __syncthreads();   // the previous block's MMAs and epilogues are done with sB / sA
        for (int idx = tid; idx < kBlk * CH; idx += kScoreThreads) {
            const int r = idx / CH, c = idx % CH;
            const int s = b * kBlk + r;
            uint8_t *dst = sB + swz(r, c);
            if (s < S) cp_async16(dst, kI + (int64_t)s * D_I + c * 8);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
        }
        gather_queries(r0, r1, 0);
        cp_async_commit();
        for (int g = 0; g < groups; ++g) {
            const int buf = g & 1;
            if (g + 1 < groups) gather_queries(r0 + (g + 1) * QG, r1, buf ^ 1);
            cp_async_commit();
            cp_async_wait<1>();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // cp.async writes -> tensor core reads
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t a_addr = smem_u32(sA + buf * A_BYTES), b_addr = smem_u32(sB);
#pragma unroll
                for (int kk = 0; kk < D_I / 16; ++kk)
                    tc_mma_f16(tmem, smem_desc(a_addr + kk * 32, SBO, LAYOUT), smem_desc(b_addr + kk * 32, SBO, LAYOUT),
                               idesc, kk > 0 ? 1u : 0u);
                tc_commit(&mma_bar);
            }
            // this thread's TMEM lane: row r = (query qi, head j)
            const int r = warp * 32 + lane, qi = r / H_I, j = r % H_I;
            const uint32_t e = s_entry[buf][qi];
            const bool valid = e != 0xffffffffu;
            const int t = valid ? (int)(e >> 8) : 0, slot = valid ? (int)(e & 255u) : 0;
            const float wv = valid ? __uint_as_float((uint32_t)w[(int64_t)t * H_I + j] << 16) : 0.f;
            const int own = (S - T + t) / kBlk;
            const int last = (b == own) ? (S - T + t) - b * kBlk : kBlk - 1;   // own block: keys <= position
            {
                volatile int no_abort = 0;
                if (!mbar_wait(&mma_bar, phase, &no_abort)) report(dev_status, SA_DEV_TIMEOUT);
            }
            phase ^= 1u;
            tc_fence_after();
            float* out = scores + (int64_t)t * ld + slot * kBlk;
            // w_j ReLU(.) of the 64 keys for this lane's head, then the sum over
            // the H_I heads (adjacent lanes) as a transposing butterfly: at each
            // step a lane keeps one half of its values and adds the partner's
            // copy of that half, so every lane ends with kBlk / H_I finished
            // sums of consecutive keys (no lane idles in the stores)
            float sc[kBlk];
#pragma unroll
            for (int c0 = 0; c0 < kBlk; c0 += 16) {
                uint32_t v[16];
                tmem_ld_x16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; ++k) sc[c0 + k] = wv * fmaxf(__uint_as_float(v[k]), 0.f);
            }
            int ko = 0;   // first key of this lane's finished sums
#pragma unroll
            for (int o = 1, L = kBlk; o < H_I; o <<= 1, L >>= 1) {
                const bool upper = (lane & o) != 0;   // keep the upper half of the current L values
#pragma unroll
                for (int i = 0; i < L / 2; ++i) {
                    const float keep = upper ? sc[L / 2 + i] : sc[i];
                    const float send = upper ? sc[i] : sc[L / 2 + i];
                    sc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
                ko += upper ? L / 2 : 0;
            }
            constexpr int NF = kBlk / H_I;   // finished sums per lane
            if (valid) {
                if (ko + NF - 1 <= last) {
#pragma unroll
                    for (int k = 0; k < NF; k += 4)
                        *reinterpret_cast<float4 *>(out + ko + k) = make_float4(sc[k], sc[k + 1], sc[k + 2], sc[k + 3]);
                } else {
#pragma unroll
                    for (int k = 0; k < NF; ++k)
                        if (ko + k <= last) out[ko + k] = sc[k];
                }
            }
            tc_fence_before();
            __syncthreads();   // TMEM and this buffer are free for the next group
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

template <int D_I>
static sa_status launch_scores_h(const uint16_t *qI, const uint16_t *w, const uint16_t *kI, int T, int S, int H_I,
                                 int nb, const BlockWs &ws, float *scores, int64_t ld, int *ds, cudaStream_t st) {
    constexpr int ROWB = D_I * 2;
    const size_t smem = 1024 + 1024 * ((kBlk * ROWB + 1023) / 1024) + 2 * 128 * ROWB;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = std::min(nb, 4 * sms);
#define SA_SCORES_CASE(H)                                                                              \
    case H: {                                                                                          \
        if (prepare_kernel<block_scores_kernel<D_I, H>>(smem, false) != cudaSuccess) return SA_ERR_CUDA; \
        block_scores_kernel<D_I, H><<<grid, kScoreThreads, smem, st>>>(qI, w, kI, T, S, nb, ws, scores, ld, ds); \
        break;                                                                                         \
    }
    switch (H_I) {
        SA_SCORES_CASE(1)
        SA_SCORES_CASE(2)
        SA_SCORES_CASE(4)
        SA_SCORES_CASE(8)
        default: return SA_ERR_UNSUPPORTED;
    }
#undef SA_SCORES_CASE
    return cuda_ok(cudaGetLastError());
}

sa_status launch_block_scores(const BlockScoreArgs &a, cudaStream_t st) {
    if (a.T == 0) return SA_OK;
    const int nb = (a.S + kBlk - 1) / kBlk;   // own blocks may be partial
    BlockWs ws = carve(a.workspace, a.T, a.S, a.keep);
    if (cudaMemsetAsync(ws.cnt, 0, (size_t)nb * 4, st) != cudaSuccess) return SA_ERR_CUDA;
    const int inv_grid = (a.T + kInvRows - 1) / kInvRows;
    const size_t h1 = (size_t)nb * 4, h2 = 2 * (size_t)nb * 4;
    if (prepare_kernel<invert_count_kernel>(h1, false) != cudaSuccess ||
        prepare_kernel<invert_scatter_kernel>(h2, false) != cudaSuccess)
        return SA_ERR_CUDA;
    invert_count_kernel<<<inv_grid, kInvThreads, h1, st>>>(a.blocks, a.keep, a.S, a.T, nb, ws, a.dev_status);
    invert_scan_kernel<<<1, kInvThreads, 0, st>>>(nb, ws);
    invert_scatter_kernel<<<inv_grid, kInvThreads, h2, st>>>(a.blocks, a.keep, a.S, a.T, nb, ws, a.dev_status);
    if (cudaGetLastError() != cudaSuccess) return SA_ERR_CUDA;
    if (a.D_I == 64) return launch_scores_h<64>(a.qI, a.w, a.kI, a.T, a.S, a.H_I, nb, ws, a.scores, a.ld, a.dev_status, st);
    if (a.D_I == 32) return launch_scores_h<32>(a.qI, a.w, a.kI, a.T, a.S, a.H_I, nb, ws, a.scores, a.ld, a.dev_status, st);
    return SA_ERR_UNSUPPORTED;
}

}  // namespace sa
