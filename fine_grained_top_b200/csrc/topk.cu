// topk.cu -- per-row top-K select with ties to the lower position.
//
// "Sparse Attention for Long-Context LLM Inference", section "Where Sparse
// Attention Is Actually Sparse": Top-K caps how many history positions take
// part in exact attention.  Here: the K largest scores of a row, equal
// scores ranked by lower position, emitted in ascending position order.
//
// Design (sm_100a):
//   * one row per thread-block cluster of G = 1..8 CTAs; CTA c of the cluster
//     owns a contiguous chunk of the row, loaded once from HBM with 16-byte
//     vector loads into shared memory as order-preserving uint32 keys;
//   * exact radix select over the keys, 4 passes of 8 bits: per-CTA
//     histograms (warp-aggregated shared atomics via match.any), summed over
//     the cluster through distributed shared memory (no global workspace);
//   * after the passes the K-th key tau is known exactly, together with how
//     many keys equal to tau must be taken (the lowest-positioned ones);
//   * ordered compaction: warp ballots count "> tau" and "== tau" keys in
//     column order, a scan over warps and over the cluster's CTAs gives every
//     kept key its output slot, so the output comes out ascending.
#include "internal.h"
#include "ptx.cuh"

namespace sa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkChunkTarget = 16384;   // columns per CTA before adding CTAs
constexpr int kTopkMaxChunk = 49152;      // 192 KB of keys per CTA
constexpr int kTopkMaxCluster = 8;

int topk_max_row_len() { return kTopkMaxChunk * kTopkMaxCluster; }

template <int G>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a) {
    extern __shared__ __align__(16) uint32_t keys[];   // [chunk]
    __shared__ uint32_t hist_local[2][256];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t warp_gt[kTopkWarps], warp_eq[kTopkWarps];
    __shared__ uint32_t cta_counts[2];
    __shared__ uint32_t sel_digit, sel_above;

    const int r = blockIdx.x / G;
    const uint32_t rank = (G > 1) ? cluster_rank() : 0u;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    int n;
    if (a.n_valid) {
        n = a.n_valid[r];
        if (n < 0 || n > a.row_len) {
            if (rank == 0 && tid == 0) report(a.dev_status, SA_DEV_INDEX);
            n = n < 0 ? 0 : a.row_len;
        }
    } else {
        n = a.row_len - a.rows + r + 1;
        n = n < 0 ? 0 : (n > a.row_len ? a.row_len : n);
    }
    const int c0 = (int)rank * a.chunk;
    const int c1 = min(c0 + a.chunk, n);
    const int len = max(0, c1 - c0);
    int32_t *out = a.out + (int64_t)r * a.K;
    const float *row = a.scores + (int64_t)r * a.ld;
    const int32_t *cand = a.cand ? a.cand + (int64_t)r * a.ld_cand : nullptr;

    if (cand) {   // the position map must be strictly ascending and non-negative
        for (int i = tid; i < len; i += kTopkThreads) {
            const int col = c0 + i;
            const int32_t c = cand[col];
            if (c < 0) report(a.dev_status, SA_DEV_INDEX);
            if (col > 0 && cand[col - 1] >= c) report(a.dev_status, SA_DEV_ORDER);
        }
    }

    if (n <= a.K) {   // every candidate is kept: no select needed
        for (int i = tid; i < len; i += kTopkThreads) out[c0 + i] = cand ? cand[c0 + i] : c0 + i;
        if (rank == 0)
            for (int i = n + tid; i < a.K; i += kTopkThreads) out[i] = -1;
        return;   // uniform over the cluster: no distributed smem was touched
    }

    // ---- load the chunk as order-preserving keys
    {
        const int len4 = len >> 2;   // c0 and ld are multiples of 4, base 16-byte aligned
        const float4 *src4 = reinterpret_cast<const float4 *>(row + c0);
        for (int i = tid; i < len4; i += kTopkThreads) {
            const float4 f = src4[i];
            uint4 k;
            k.x = order_key(f.x); k.y = order_key(f.y); k.z = order_key(f.z); k.w = order_key(f.w);
            reinterpret_cast<uint4 *>(keys)[i] = k;
        }
        for (int i = (len4 << 2) + tid; i < len; i += kTopkThreads) keys[i] = order_key(row[c0 + i]);
    }

    // ---- exact radix select of the K-th largest key
    uint32_t prefix = 0u, mask = 0u;
    uint32_t need = (uint32_t)a.K;   // keys still to take among those matching `prefix`
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        uint32_t *hl = hist_local[pass & 1];
        if (tid < 256) hl[tid] = 0u;
        __syncthreads();
        for (int base = 0; base < len; base += kTopkThreads) {
            const int i = base + tid;
            uint32_t bin = 256u;   // sentinel: not counted
            if (i < len) {
                const uint32_t u = keys[i];
                if ((u & mask) == prefix) bin = (u >> shift) & 255u;
            }
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&hl[bin], (uint32_t)__popc(peers));
        }
        __syncthreads();
        if (G > 1) {
            cluster_sync();
            if (tid < 256) {
                uint32_t s = 0;
#pragma unroll
                for (int c = 0; c < G; ++c) s += dsmem_ld_u32(&hl[tid], (uint32_t)c);
                hist[tid] = s;
            }
        } else if (tid < 256) {
            hist[tid] = hl[tid];
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns bins 255-8l .. 248-8l, scanned from the top down
            uint32_t cnt[8], lsum = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) { cnt[k] = hist[255 - 8 * lane - k]; lsum += cnt[k]; }
            uint32_t incl = lsum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const uint32_t excl = incl - lsum;
            if (excl < need && need <= incl) {
                uint32_t acc = excl;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (acc + cnt[k] >= need) {
                        sel_digit = 255u - 8u * lane - k;
                        sel_above = acc;
                        break;
                    }
                    acc += cnt[k];
                }
            }
        }
        __syncthreads();
        need -= sel_above;
        prefix |= sel_digit << shift;
        mask |= 0xFFu << shift;
    }
    const uint32_t tau = prefix;   // the K-th largest key; `need` keys equal to it are kept

    // ---- ordered compaction
    const int sub = ((len + kTopkThreads - 1) / kTopkThreads) * 32;   // per-warp span, multiple of 32
    const int w0 = warp * sub, w1 = min(w0 + sub, len);
    uint32_t gt = 0, eq = 0;
    for (int i = w0 + lane; i < w0 + sub; i += 32) {
        const bool valid = i < w1;
        const uint32_t u = valid ? keys[i] : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, valid && u > tau));
        eq += __popc(__ballot_sync(0xffffffffu, valid && u == tau));
    }
    if (lane == 0) { warp_gt[warp] = gt; warp_eq[warp] = eq; }
    __syncthreads();
    if (tid == 0) {
        uint32_t g = 0, e = 0;
        for (int w = 0; w < kTopkWarps; ++w) {
            const uint32_t tg = warp_gt[w], te = warp_eq[w];
            warp_gt[w] = g; warp_eq[w] = e;
            g += tg; e += te;
        }
        cta_counts[0] = g; cta_counts[1] = e;
    }
    __syncthreads();
    uint32_t base_gt = 0, base_eq = 0;
    if (G > 1) {
        cluster_sync();
        for (uint32_t c = 0; c < rank; ++c) {
            base_gt += dsmem_ld_u32(&cta_counts[0], c);
            base_eq += dsmem_ld_u32(&cta_counts[1], c);
        }
    }
    uint32_t run_gt = base_gt + warp_gt[warp], run_eq = base_eq + warp_eq[warp];
    const uint32_t lt = lanemask_lt();
    for (int i = w0 + lane; i < w0 + sub; i += 32) {
        const bool valid = i < w1;
        const uint32_t u = valid ? keys[i] : 0u;
        const bool is_gt = valid && u > tau, is_eq = valid && u == tau;
        const uint32_t bg = __ballot_sync(0xffffffffu, is_gt), be = __ballot_sync(0xffffffffu, is_eq);
        const uint32_t gt_before = run_gt + __popc(bg & lt), eq_before = run_eq + __popc(be & lt);
        if (is_gt || (is_eq && eq_before < need)) {
            const uint32_t slot = gt_before + min(eq_before, need);
            const int col = c0 + i;
            out[slot] = cand ? cand[col] : col;
        }
        run_gt += __popc(bg);
        run_eq += __popc(be);
    }
    if (G > 1) cluster_sync();   // peers may still read this CTA's counters
}

template <int G>
static sa_status launch_topk_g(const TopkArgs &a, size_t smem, cudaStream_t st) {
    auto kern = topk_kernel<G>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return SA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.rows * G));
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_ok(cudaLaunchKernelEx(&cfg, kern, a));
}

sa_status launch_topk(TopkArgs a, cudaStream_t st) {
    int g = 1;
    while (g < kTopkMaxCluster && (a.row_len + g - 1) / g > kTopkChunkTarget) g *= 2;
    int chunk = (a.row_len + g - 1) / g;
    chunk = (chunk + 3) & ~3;
    if (chunk > kTopkMaxChunk) return SA_ERR_UNSUPPORTED;
    a.chunk = chunk;
    const size_t smem = (size_t)chunk * 4 + 16;
    switch (g) {
        case 1: return launch_topk_g<1>(a, smem, st);
        case 2: return launch_topk_g<2>(a, smem, st);
        case 4: return launch_topk_g<4>(a, smem, st);
        default: return launch_topk_g<8>(a, smem, st);
    }
}

}  // namespace sa
