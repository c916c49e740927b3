// topk.cu -- per-row top-K select with ties to the lower position.
//
// "Sparse Attention for Long-Context LLM Inference", section "Where Sparse
// Attention Is Actually Sparse": Top-K caps how many history positions take
// part in exact attention.  Here: the K largest scores of a row, equal
// scores ranked by lower position, emitted in ascending position order.
//
// Design (sm_100a):
//   * rows of at most 1024 columns: one warp per row, the keys in registers,
//     a bitwise search for the K-th key (topk_rows_kernel);
//   * longer rows: one row per thread-block cluster of G = 1..16 CTAs; CTA c of the
//     cluster owns a contiguous chunk of the row, copied once from HBM into
//     shared memory with 16-byte cp.async (issued first, so the copy overlaps
//     the row's argument checks) and rewritten there as order-preserving
//     uint32 keys;
//   * exact radix select over the keys in three passes of 11, 11 and 10 bits
//     (12, 10 and 10 for a cluster row).
//     The first histogram is built while the keys are rewritten; the later
//     passes only count keys that match the prefix chosen so far.  Per-CTA
//     histograms are summed over the cluster through distributed shared
//     memory (no global workspace).  When the threshold bin is taken whole,
//     the remaining passes are skipped;
//   * the K-th key tau (to the resolved precision) is then known, together
//     with how many keys equal to it must be taken (the lowest-positioned);
//   * ordered compaction: each warp counts "> tau" and "== tau" keys of its
//     span in column order (4 keys per lane per step, both counts packed in
//     one word), a scan over lanes, warps and the cluster's CTAs gives every
//     kept key its output slot, so the output comes out ascending.
#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

// Threads per CTA: 256 for a single-CTA row (rows of at most 8192 columns:
// more rows resident per SM), 512 for the CTAs of a cluster row (chunks of up
// to 32768 columns).
template <int G> constexpr int topk_threads() { return G == 1 ? 256 : 512; }
#ifndef SA_TOPK_CHUNK
#define SA_TOPK_CHUNK 8192
#endif
constexpr int kTopkChunkTarget = SA_TOPK_CHUNK;   // columns per CTA before adding CTAs
constexpr int kTopkMaxChunk = 32768;      // 128 KB of keys per CTA
constexpr int kTopkMaxCluster = 16;
// First digit: the top 11 bits for a single-CTA row (then 11 and 10), the
// top 12 bits for a cluster row (then 10 and 10: smaller refinement
// histograms to sum across the cluster).
template <int G> constexpr int bits_a() { return G == 1 ? 11 : 12; }
constexpr int kBinsMax = 4096;

int topk_max_row_len() { return kTopkMaxChunk * kTopkMaxCluster; }

// Sum the CTAs' histograms (G > 1) and find the bin holding the need-th
// largest key.  Every thread returns (digit, count above it, count in it).
// The cluster sum is a reduce-scatter plus all-gather over distributed shared
// memory: CTA r adds up bin slice r from every CTA (all G loads in flight at
// once) and stores the sums into slice r of every CTA's `hsum`.
template <int G, int BINS, int NT>
__device__ __forceinline__ void find_threshold(uint32_t *hl, uint32_t *hsum, uint32_t need,
                                               uint32_t *scan_tmp, uint32_t *sel, int tid) {
    constexpr int PER = BINS / NT;   // bins per thread
    const int lane = tid & 31, warp = tid >> 5;
    const uint32_t *h = hl;
    if (G > 1) {
        constexpr int SLICE = BINS / G;
        const uint32_t rank = cluster_rank();
        cluster_sync();   // every CTA's histogram is complete
        for (int i = tid; i < SLICE; i += NT) {
            const int bin = (int)rank * SLICE + i;
            uint32_t v[G];
#pragma unroll
            for (int c = 0; c < G; ++c) v[c] = dsmem_ld_u32(&hl[bin], (uint32_t)c);
            uint32_t s = 0;
#pragma unroll
            for (int c = 0; c < G; ++c) s += v[c];
#pragma unroll
            for (int c = 0; c < G; ++c) dsmem_st_u32(&hsum[bin], (uint32_t)c, s);
        }
        cluster_sync();   // every slice has reached every CTA
        h = hsum;
    }
    // thread i owns bins BINS-1-PER*i .. BINS-PER*i (scanned from the top down),
    // read as PER/4 16-byte vectors
    static_assert(PER % 4 == 0 || PER == 2, "bins per thread");
    uint32_t cnt[PER], lsum = 0;
    if constexpr (PER % 4 == 0) {
#pragma unroll
        for (int q4 = 0; q4 < PER / 4; ++q4) {
            const uint4 b = reinterpret_cast<const uint4 *>(h + BINS - PER * (tid + 1))[PER / 4 - 1 - q4];
            cnt[4 * q4 + 0] = b.w; cnt[4 * q4 + 1] = b.z; cnt[4 * q4 + 2] = b.y; cnt[4 * q4 + 3] = b.x;
        }
    } else {
        const uint2 b = reinterpret_cast<const uint2 *>(h + BINS - PER * (tid + 1))[0];
        cnt[0] = b.y; cnt[1] = b.x;
    }
#pragma unroll
    for (int k = 0; k < PER; ++k) lsum += cnt[k];
    uint32_t incl = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) scan_tmp[warp] = incl;
    __syncthreads();
    // bins above this warp's: the totals of the warps before it
    const uint32_t wexcl = __reduce_add_sync(0xffffffffu, lane < warp ? scan_tmp[lane] : 0u);
    const uint32_t excl = wexcl + incl - lsum;
    if (excl < need && need <= excl + lsum) {
        uint32_t acc = excl;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            if (acc + cnt[k] >= need) {
                sel[0] = (uint32_t)(BINS - 1 - PER * tid - k);
                sel[1] = acc;
                sel[2] = cnt[k];
                break;
            }
            acc += cnt[k];
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------- fused indexer
// Decode rows with the indexer fused in: the scores of columns [c0, c0 + len)
// of row r (keys c0 .. of sequence r),
//   I[s] = sum_{j < H_I} w[j] * max(0, qI[j, :] . kI[s, :]),
// are computed on the tensor cores and written straight into keys[] as
// order-preserving keys while the first histogram is counted; they never
// reach global memory.  mma.sync m16n8k16 (bf16 x bf16 -> fp32) with M = 16
// keys, N = 8 heads (H_I <= 8, missing heads zero), K = 16 dims; the key rows
// come through a ring of four 32 KB tiles in shared memory, three in flight
// while one is used (16-byte cp.async, 16-byte chunks XOR-swizzled by row for
// conflict-free ldmatrix).  The head sum runs over the four lanes of a quad (two heads per
// lane), so for integer-valued inputs every sum is exact and the result equals
// the unfused indexer's.
constexpr int kFusedSlotBytes = 32768;   // one ring slot: 256 keys of 128 bytes (128 of 256)
constexpr int kFusedStages = 4;          // ring slots (up to three tiles in flight while one is used)

template <int ROWB>
__device__ __forceinline__ uint32_t ring_swz(int row, int c) {
    return (uint32_t)(row * ROWB + ((c ^ (row & 7)) << 4));
}

template <int NT, int D_I, int SHIFT>
__device__ void fused_scores(const TopkArgs &a, int r, int c0, int len, uint32_t *keys, uint32_t *hist0,
                             uint8_t *ring, int tid) {
    constexpr int ROWB = D_I * 2, CH = ROWB / 16, KS = D_I / 16, NW = NT / 32;
    constexpr int TILE = kFusedSlotBytes / ROWB;   // keys per slot
    const int lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
    const int H = a.f_HI;
    // B fragments (K x N = dims x heads, "col"): head g, dims 16 ks + 2t, +1
    // and 16 ks + 2t + 8, +9 (two consecutive bf16 in each 32-bit register)
    uint32_t bq[KS][2];
    const uint32_t *q32 = reinterpret_cast<const uint32_t *>(a.f_qI + (int64_t)r * H * D_I);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        bq[ks][0] = g < H ? q32[(g * D_I + 16 * ks + 2 * t) >> 1] : 0u;
        bq[ks][1] = g < H ? q32[(g * D_I + 16 * ks + 2 * t + 8) >> 1] : 0u;
    }
    // this lane's heads in the accumulator: 2t and 2t + 1
    const uint16_t *wr = a.f_w + (int64_t)r * H;
    const float w0 = 2 * t < H ? __uint_as_float((uint32_t)wr[2 * t] << 16) : 0.f;
    const float w1 = 2 * t + 1 < H ? __uint_as_float((uint32_t)wr[2 * t + 1] << 16) : 0.f;
    const int32_t *pt = a.f_page_table ? a.f_page_table + (int64_t)r * a.f_max_pages : nullptr;

    // tile `tile` into slot tile % kFusedStages; one commit group per call
    auto issue = [&](int tile) {
        uint8_t *dst = ring + (tile % kFusedStages) * kFusedSlotBytes;
        const int k0 = tile * TILE;
        for (int idx = tid; idx < TILE * CH; idx += NT) {
            const int i = idx / CH, c = idx % CH;
            if (k0 + i >= len) break;   // idx grows with i: the rest of this thread's copies are past the chunk
            const int s = c0 + k0 + i;  // key position in the sequence
            int64_t row;
            if (pt) {
                int pid = pt[s >> 6];
                if (pid < 0 || pid >= a.f_pool_pages) {
                    if (c == 0) report(a.dev_status, SA_DEV_INDEX);
                    pid = 0;   // any valid row: the result is flagged
                }
                row = (int64_t)pid * 64 + (s & 63);
            } else {
                row = (int64_t)r * a.f_S + s;
            }
            cp_async16(dst + ring_swz<ROWB>(i, c), a.f_kI + row * D_I + c * 8);
        }
    };
    const int ntile = (len + TILE - 1) / TILE;
#pragma unroll
    for (int p = 0; p < kFusedStages - 1; ++p) {
        if (p < ntile) issue(p);
        cp_async_commit();   // (empty groups keep the count uniform)
    }
    for (int tile = 0; tile < ntile; ++tile) {
        cp_async_wait<kFusedStages - 2>();   // this thread's copies of `tile` have landed
        __syncthreads();                     // ... everyone's; and every warp is past tile - 1
        if (tile + kFusedStages - 1 < ntile) issue(tile + kFusedStages - 1);   // into the slot of tile - 1
        cp_async_commit();
        const uint8_t *buf = ring + (tile % kFusedStages) * kFusedSlotBytes;
        for (int mt = warp; mt < TILE / 16; mt += NW) {
            const int k0 = tile * TILE + mt * 16;   // first column of the 16-key group
            if (k0 >= len) break;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t af[4];
                const int row = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                ldmatrix_x4(af, buf + ring_swz<ROWB>(row, ks * 2 + (lane >> 4)));
                mma_bf16_16816(acc, af, bq[ks]);
            }
            // acc: (key g, heads 2t, 2t+1), (key g + 8, heads 2t, 2t+1)
            float s_lo = w0 * fmaxf(acc[0], 0.f) + w1 * fmaxf(acc[1], 0.f);
            float s_hi = w0 * fmaxf(acc[2], 0.f) + w1 * fmaxf(acc[3], 0.f);
            s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
            s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
            s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
            s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
            const int col = k0 + g + (t == 1 ? 8 : 0);
            if (t < 2 && col < len) {
                const uint32_t u = order_key(t == 0 ? s_lo : s_hi);
                keys[col] = u;
                atomicAdd(&hist0[u >> SHIFT], 1u);
            }
        }
    }
    cp_async_wait<0>();
    __syncthreads();
}

template <int G, bool FUSED>
__device__ __forceinline__ void topk_body(const TopkArgs &a) {
    constexpr int NT = topk_threads<G>(), NW = NT / 32;
    // dynamic smem: keys[chunk] | hist_local[4096] | (G > 1) hist_sum[4096]
    // (peers read this CTA's histogram of a pass only between that pass's two
    // cluster barriers, so one local buffer serves every pass)
    extern __shared__ __align__(16) uint32_t dsm[];
    uint32_t *keys = dsm;
    uint32_t *hist0 = dsm + a.chunk;
    constexpr int BA = bits_a<G>(), SA_ = 32 - BA, BINS_A = 1 << BA, BINS_1 = 1 << (SA_ - 10);
    uint32_t *hsum = (G > 1) ? hist0 + BINS_A : nullptr;
    __shared__ uint32_t scan_tmp[64];
    __shared__ uint32_t sel[3];
    __shared__ uint32_t warp_gt[NW];   // packed per-warp counts
    __shared__ uint32_t cta_counts[2];
    __shared__ uint32_t low_bits[2];   // OR, AND of the last digit over the first refinement's keys

    const int r = blockIdx.x / G;
    const uint32_t rank = (G > 1) ? cluster_rank() : 0u;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // Start copying this CTA's chunk of the row into shared memory before
    // anything waits.  With block-id candidates the row's valid length is
    // known only after the ids are checked, so that copy runs to the row's
    // allocated length; columns past the valid length are never read back.
    const int c0 = (int)rank * a.chunk;
    const float *row = FUSED ? nullptr : a.scores + (int64_t)r * a.ld;
    int n_bound = a.row_len;
    {
        if (!a.by_blocks) {
            n_bound = a.n_valid ? a.n_valid[r] : a.row_len - a.rows + r + 1;
            n_bound = n_bound < 0 ? 0 : (n_bound > a.row_len ? a.row_len : n_bound);
        }
        if (!FUSED) {
            const int pre4 = max(0, min(c0 + a.chunk, n_bound) - c0) >> 2;   // c0 and ld are multiples of 4
            const float4 *src4 = reinterpret_cast<const float4 *>(row + c0);
            for (int i = tid; i < pre4; i += NT) cp_async16(keys + 4 * i, src4 + i);
        }
    }

    int n;
    int n_kept = 0, own0 = 0;   // block-id candidates: valid kept blocks, first token of the own block
    const bool byb = a.by_blocks;
    const int32_t *brow = (byb && a.keep > 0) ? a.blocks + (int64_t)r * a.keep : nullptr;
    if (byb) {
        const int p = a.S - a.rows + r, own = p / a.block;
        own0 = own * a.block;
        // the valid ids form a prefix, strictly ascending, each below the own block
        if (tid == 0) cta_counts[0] = 0u;
        __syncthreads();
        uint32_t valid = 0;
        for (int i = tid; i < a.keep; i += NT) {
            const int b = brow[i];
            if (b >= 0) {
                ++valid;
                if (rank == 0 && b >= own) report(a.dev_status, SA_DEV_INDEX);
                if (rank == 0 && i > 0 && !(brow[i - 1] >= 0 && brow[i - 1] < b)) report(a.dev_status, SA_DEV_ORDER);
            }
        }
        valid = __reduce_add_sync(0xffffffffu, valid);
        if (lane == 0 && valid) atomicAdd(&cta_counts[0], valid);
        __syncthreads();
        n_kept = (int)cta_counts[0];
        __syncthreads();
        n = n_kept * a.block + (p - own0 + 1);
        if (n > a.row_len) {
            if (rank == 0 && tid == 0) report(a.dev_status, SA_DEV_INDEX);
            n = a.row_len;
        }
    } else if (a.n_valid) {
        n = a.n_valid[r];
        if (n < 0 || n > a.row_len) {
            if (rank == 0 && tid == 0) report(a.dev_status, SA_DEV_INDEX);
            n = n < 0 ? 0 : a.row_len;
        }
    } else {
        n = a.row_len - a.rows + r + 1;
        n = n < 0 ? 0 : (n > a.row_len ? a.row_len : n);
    }
    const int c1 = min(c0 + a.chunk, n);
    const int len = max(0, c1 - c0);
    int32_t *out = a.out + (int64_t)r * a.K;
    const int32_t *cand = a.cand ? a.cand + (int64_t)r * a.ld_cand : nullptr;
    // position of column col: through the block ids, the position map, or itself
    // (a power-of-two block size, the usual case, takes shifts instead of divisions)
    const int bshift = (a.block > 0 && (a.block & (a.block - 1)) == 0) ? __ffs(a.block) - 1 : -1;
    auto pos = [&](int col) -> int32_t {
        if (byb) {
            const int kb = n_kept * a.block;
            if (col >= kb) return own0 + (col - kb);
            if (bshift >= 0) return (brow[col >> bshift] << bshift) + (col & (a.block - 1));
            return brow[col / a.block] * a.block + col % a.block;
        }
        return cand ? cand[col] : col;
    };

    if (cand) {   // the position map must be strictly ascending and non-negative
        for (int i = tid; i < len; i += NT) {
            const int col = c0 + i;
            const int32_t c = cand[col];
            if (c < 0) report(a.dev_status, SA_DEV_INDEX);
            if (col > 0 && cand[col - 1] >= c) report(a.dev_status, SA_DEV_ORDER);
        }
    }

    if (n <= a.K) {   // every candidate is kept: no select needed
        for (int i = tid; i < len; i += NT) out[c0 + i] = pos(c0 + i);
        if (rank == 0)
            for (int i = n + tid; i < a.K; i += NT) out[i] = -1;
        cp_async_wait_all();   // the copies into this CTA's shared memory end before it exits
        return;   // uniform over the cluster: no distributed smem was touched
    }

    // ---- the chunk as order-preserving keys, counting the top 11 bits
    for (int i = tid; i < BINS_A / 4; i += NT) reinterpret_cast<uint4 *>(hist0)[i] = make_uint4(0u, 0u, 0u, 0u);
    cp_async_wait_all();
    __syncthreads();
    if (FUSED) {
        uint8_t *ring = reinterpret_cast<uint8_t *>(keys + a.ring_off);
        if (a.f_DI == 64) fused_scores<NT, 64, SA_>(a, r, c0, len, keys, hist0, ring, tid);
        else fused_scores<NT, 128, SA_>(a, r, c0, len, keys, hist0, ring, tid);
    } else {
        const int len4 = len >> 2;
        for (int i = tid; i < len4; i += NT) {
            const uint4 f = reinterpret_cast<const uint4 *>(keys)[i];
            uint4 u;
            u.x = order_key(__uint_as_float(f.x)); u.y = order_key(__uint_as_float(f.y));
            u.z = order_key(__uint_as_float(f.z)); u.w = order_key(__uint_as_float(f.w));
            reinterpret_cast<uint4 *>(keys)[i] = u;
            atomicAdd(&hist0[u.x >> SA_], 1u);
            atomicAdd(&hist0[u.y >> SA_], 1u);
            atomicAdd(&hist0[u.z >> SA_], 1u);
            atomicAdd(&hist0[u.w >> SA_], 1u);
        }
        for (int i = (len4 << 2) + tid; i < len; i += NT) {   // the last len % 4 columns
            const uint32_t k = order_key(row[c0 + i]);
            keys[i] = k;
            atomicAdd(&hist0[k >> SA_], 1u);
        }
    }
    __syncthreads();

    uint32_t need = (uint32_t)a.K;      // keys still to take among those matching `prefix`
    find_threshold<G, BINS_A, NT>(hist0, hsum, need, scan_tmp, sel, tid);
    uint32_t prefix = sel[0] << SA_, mask = 0xFFFFFFFFu << SA_;
    need -= sel[1];
    bool whole = sel[2] == need;        // the threshold bin is taken entirely
    // refinements (11 or 10 bits, then 10) over the keys that match the prefix.  A single-CTA
    // row also takes, in the first, the OR and AND of the last digit (bits
    // 9..0) over those keys: when they agree, every key of the bin shares its
    // last digit and the second refinement is decided without a pass (keys with
    // few mantissa bits, e.g. integer-valued or FP8-product scores).
#pragma unroll 1
    for (int pass = 1; pass < 3 && !whole; ++pass) {
        const int shift = pass == 1 ? 10 : 0;
        const uint32_t dmask = pass == 1 ? (uint32_t)BINS_1 - 1u : 1023u;   // the digit: bits SA_-1..10, then 9..0
        const bool track = G == 1 && pass == 1;
        uint32_t *hl = hist0;
        for (int i = tid; i < (int)(dmask + 1) / 4; i += NT)
            reinterpret_cast<uint4 *>(hl)[i] = make_uint4(0u, 0u, 0u, 0u);
        if (track && tid == 0) { low_bits[0] = 0u; low_bits[1] = 1023u; }
        __syncthreads();
        uint32_t lor = 0u, land = 1023u;
        auto count = [&](uint32_t u) {
            if ((u & mask) == prefix) {
                atomicAdd(&hl[(u >> shift) & dmask], 1u);
                if (track) {
                    lor |= u & 1023u;
                    land &= u & 1023u;
                }
            }
        };
        const int len4 = len >> 2;
        for (int i = tid; i < len4; i += NT) {
            const uint4 k = reinterpret_cast<const uint4 *>(keys)[i];
            count(k.x);
            count(k.y);
            count(k.z);
            count(k.w);
        }
        for (int i = (len4 << 2) + tid; i < len; i += NT) count(keys[i]);
        if (track) {
            lor = __reduce_or_sync(0xffffffffu, lor);
            land = __reduce_and_sync(0xffffffffu, land);
            if (lane == 0) {
                atomicOr(&low_bits[0], lor);
                atomicAnd(&low_bits[1], land);
            }
        }
        __syncthreads();
        if (pass == 1)
            find_threshold<G, BINS_1, NT>(hl, hsum, need, scan_tmp, sel, tid);
        else
            find_threshold<G, 1024, NT>(hl, hsum, need, scan_tmp, sel, tid);
        prefix |= sel[0] << shift;
        mask |= dmask << shift;
        need -= sel[1];
        whole = sel[2] == need;
        if (track && !whole && low_bits[0] == low_bits[1]) {   // the last digit is the same for all
            prefix |= low_bits[0];
            mask = 0xFFFFFFFFu;
            break;
        }
    }
    const uint32_t tau = prefix, tmask = mask;   // keep: (u&tmask) > tau, and `need` of (u&tmask) == tau

    // ---- ordered compaction.  Warp w owns keys [w0, w0 + sub) of the chunk and
    // visits them 128 at a time, 4 consecutive keys per lane; per-lane counts
    // of "> tau" (low 16 bits) and "== tau" (high 16 bits) are packed into one
    // word, so one warp sum or scan handles both (a CTA holds < 65536 keys).
    const int sub = ((len + 4 * NT - 1) / (4 * NT)) * 128;
    const int w0 = warp * sub, w1 = min(w0 + sub, len);
    auto load4 = [&](int p, uint32_t (&u)[4]) {
        if (p + 3 < w1) {
            const uint4 k = reinterpret_cast<const uint4 *>(keys)[p >> 2];
            u[0] = k.x; u[1] = k.y; u[2] = k.z; u[3] = k.w;
        } else {   // the ragged end of the span (or past it)
#pragma unroll
            for (int e = 0; e < 4; ++e) u[e] = p + e < w1 ? keys[p + e] : 0u;
        }
    };
    // per lane and 128-key group: bits 0..3 "key e > tau", bits 4..7 "key e == tau",
    // kept for the write sweep in the first histogram's storage (free by now)
    uint32_t *flags = hist0 + warp * (sub / 4);   // sub / 128 groups x 32 lanes per warp
    auto flags4 = [&](int p, uint32_t (&u)[4]) -> uint32_t {
        uint32_t f = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const uint32_t k = u[e] & tmask;
            const bool valid = p + e < w1;
            f |= (valid && k > tau) ? (1u << e) : 0u;
            f |= (valid && k == tau) ? (16u << e) : 0u;
        }
        return f;
    };
    uint32_t wtot = 0;
    for (int j = w0, g = 0; j < w0 + sub; j += 128, ++g) {
        uint32_t u[4];
        load4(j + 4 * lane, u);
        const uint32_t f = flags4(j + 4 * lane, u);
        flags[g * 32 + lane] = f;
        wtot += (uint32_t)__popc(f & 15u) + ((uint32_t)__popc(f >> 4) << 16);
    }
    wtot = __reduce_add_sync(0xffffffffu, wtot);   // this warp's packed counts
    if (lane == 0) warp_gt[warp] = wtot;
    __syncthreads();
    const uint32_t wbase = __reduce_add_sync(0xffffffffu, lane < warp ? warp_gt[lane] : 0u);   // warps before
    if (tid == NT - 1) {
        cta_counts[0] = (wbase + wtot) & 0xFFFFu;
        cta_counts[1] = (wbase + wtot) >> 16;
    }
    uint32_t base_gt = 0, base_eq = 0;
    if (G > 1) {
        cluster_sync();   // every CTA's totals are written
        for (uint32_t c = 0; c < rank; ++c) {
            base_gt += dsmem_ld_u32(&cta_counts[0], c);
            base_eq += dsmem_ld_u32(&cta_counts[1], c);
        }
    }
    uint32_t run = wbase;   // packed counts before the current 128-key group of this warp
    for (int j = w0, g = 0; j < w0 + sub; j += 128, ++g) {
        const int p = j + 4 * lane;
        const uint32_t f = flags[g * 32 + lane];
        const uint32_t c = (uint32_t)__popc(f & 15u) + ((uint32_t)__popc(f >> 4) << 16);
        uint32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (f != 0u) {   // this lane keeps or ties at least one of its keys
            const uint32_t before = run + incl - c;
            uint32_t gt_before = base_gt + (before & 0xFFFFu), eq_before = base_eq + (before >> 16);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool is_gt = (f >> e) & 1u, is_eq = (f >> (4 + e)) & 1u;
                if (is_gt || (is_eq && eq_before < need)) {
                    out[gt_before + min(eq_before, need)] = pos(c0 + p + e);
                }
                gt_before += is_gt ? 1u : 0u;
                eq_before += is_eq ? 1u : 0u;
            }
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (G > 1) cluster_sync();   // peers may still read this CTA's counters
}

// The select alone, and the select with the indexer fused in (which keeps
// its operand fragments and key tiles in registers and shared memory, so it
// asks for one resident CTA's worth of registers rather than the select's
// occupancy).
template <int G>
__global__ void __launch_bounds__(topk_threads<G>()) topk_kernel(TopkArgs a) { topk_body<G, false>(a); }
template <int G>
__global__ void __launch_bounds__(topk_threads<G>(), 1) topk_fused_kernel(TopkArgs a) { topk_body<G, true>(a); }

// Short rows (the coarse block selection, small prefills): a group of W warps
// per row (W = 1 for the rows of at most 1024 columns it is used for), the row's keys
// in registers, thread t of the group holding the PER consecutive columns
// from t * PER.  The K-th largest key tau is found bit by bit from the top:
// a candidate bit is kept when at least K keys are >= the candidate (counts
// summed over the group).  The kept keys are then written in column order
// after one scan of the "> tau" and "== tau" counts over the group, the
// lowest-positioned ties first.
constexpr int kRowsThreads = 256;

template <int PER, int W>
__global__ void __launch_bounds__(kRowsThreads) topk_rows_kernel(TopkArgs a) {
    constexpr int GT = 32 * W;                        // threads per row
    constexpr int RPC = kRowsThreads / GT;            // rows per CTA
    __shared__ uint32_t red[RPC][2][W];               // per-warp partial counts (double-buffered by round)
    __shared__ uint32_t scan[RPC][W];
    const int grp = threadIdx.x / GT, t = threadIdx.x % GT, lane = t & 31, wg = t >> 5;
    const int r = blockIdx.x * RPC + grp;
    if (r >= a.rows) return;   // whole groups leave together (rows are group-uniform)
    auto group_sync = [&]() {
        if (W > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(GT) : "memory");
    };
    // sum of v over the group (a shuffle butterfly: the warp reduction
    // instruction runs on a slower pipe); `round` alternates the exchange
    // buffer, so one barrier per sum suffices
    auto group_sum = [&](uint32_t v, int round) -> uint32_t {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (W == 1) return v;
        if (lane == 0) red[grp][round & 1][wg] = v;
        group_sync();
        uint32_t s2 = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) s2 += red[grp][round & 1][w];
        return s2;
    };
    int n;
    int n_kept = 0, own0 = 0;   // block-id candidates: valid kept blocks, first token of the own block
    const bool byb = a.by_blocks;
    const int32_t *brow = (byb && a.keep > 0) ? a.blocks + (int64_t)r * a.keep : nullptr;
    if (byb) {
        const int p = a.S - a.rows + r, own = p / a.block;
        own0 = own * a.block;
        // the valid ids form a prefix, strictly ascending, each below the own block
        uint32_t valid = 0;
        for (int i = t; i < a.keep; i += GT) {
            const int b = brow[i];
            if (b >= 0) {
                ++valid;
                if (b >= own) report(a.dev_status, SA_DEV_INDEX);
                if (i > 0 && !(brow[i - 1] >= 0 && brow[i - 1] < b)) report(a.dev_status, SA_DEV_ORDER);
            }
        }
        n_kept = (int)group_sum(valid, 0);
        group_sync();   // the count's exchange buffer is reused by the search
        n = n_kept * a.block + (p - own0 + 1);
        if (n > a.row_len) {
            if (t == 0) report(a.dev_status, SA_DEV_INDEX);
            n = a.row_len;
        }
    } else if (a.n_valid) {
        n = a.n_valid[r];
        if (n < 0 || n > a.row_len) {
            if (t == 0) report(a.dev_status, SA_DEV_INDEX);
            n = n < 0 ? 0 : a.row_len;
        }
    } else {
        n = a.row_len - a.rows + r + 1;
        n = n < 0 ? 0 : (n > a.row_len ? a.row_len : n);
    }
    int32_t *out = a.out + (int64_t)r * a.K;
    const float *row = a.scores + (int64_t)r * a.ld;
    const int32_t *cand = a.cand ? a.cand + (int64_t)r * a.ld_cand : nullptr;
    // position of column col: through the block ids, the position map, or itself
    // (a power-of-two block size, the usual case, takes shifts instead of divisions)
    const int bshift = (a.block > 0 && (a.block & (a.block - 1)) == 0) ? __ffs(a.block) - 1 : -1;
    auto pos = [&](int col) -> int32_t {
        if (byb) {
            const int kb = n_kept * a.block;
            if (col >= kb) return own0 + (col - kb);
            if (bshift >= 0) return (brow[col >> bshift] << bshift) + (col & (a.block - 1));
            return brow[col / a.block] * a.block + col % a.block;
        }
        return cand ? cand[col] : col;
    };
    const int c_lo = t * PER;
    if (cand) {   // the position map must be strictly ascending and non-negative
        for (int col = t; col < n; col += GT) {
            const int32_t c = cand[col];
            if (c < 0) report(a.dev_status, SA_DEV_INDEX);
            if (col > 0 && cand[col - 1] >= c) report(a.dev_status, SA_DEV_ORDER);
        }
    }
    if (n <= a.K) {   // every column is kept
        for (int col = t; col < a.K; col += GT) out[col] = col < n ? pos(col) : -1;
        return;
    }
    uint32_t key[PER];
    if (PER % 4 == 0 && c_lo + PER <= n) {   // 16-byte loads (rows start 16-byte aligned, PER % 4 == 0)
#pragma unroll
        for (int e = 0; e < PER; e += 4) {
            const float4 f = __ldg(reinterpret_cast<const float4 *>(row + c_lo + e));
            key[e] = order_key(f.x); key[e + 1] = order_key(f.y);
            key[e + 2] = order_key(f.z); key[e + 3] = order_key(f.w);
        }
    } else {
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int col = c_lo + e;
            key[e] = col < n ? order_key(__ldg(row + col)) : 0u;   // 0 ranks below every score
        }
    }
    // Bits on which every valid key agrees need no count: tau takes them from
    // the keys (integer-valued or short-mantissa scores leave most low bits
    // constant).  OR and AND over the row's valid keys:
    uint32_t kor = 0u, kand = 0xffffffffu;
#pragma unroll
    for (int e = 0; e < PER; ++e)
        if (c_lo + e < n) { kor |= key[e]; kand &= key[e]; }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kor |= __shfl_xor_sync(0xffffffffu, kor, o);
        kand &= __shfl_xor_sync(0xffffffffu, kand, o);
    }
    if (W > 1) {
        if (lane == 0) { red[grp][0][wg] = kor; red[grp][1][wg] = kand; }
        group_sync();
        kor = 0u; kand = 0xffffffffu;
#pragma unroll
        for (int w = 0; w < W; ++w) { kor |= red[grp][0][w]; kand &= red[grp][1][w]; }
        group_sync();   // the buffers are reused by the counts below
    }
    const uint32_t varying = kor ^ kand;
    // tau = the largest value with at least K keys >= tau, bit by bit from the top
    uint32_t tau = 0u;
    int round = 0;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
        if (!((varying >> bit) & 1u)) {
            tau |= kand & (1u << bit);
            continue;
        }
        const uint32_t c = tau | (1u << bit);
        uint32_t cnt = 0;
#pragma unroll
        for (int e = 0; e < PER; ++e) cnt += key[e] >= c ? 1u : 0u;
        if (group_sum(cnt, round++) >= (uint32_t)a.K) tau = c;
    }
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        gt += key[e] > tau ? 1u : 0u;
        eq += key[e] == tau ? 1u : 0u;
    }
    // packed (eq << 16 | gt) counts: exclusive scan over the group's threads
    const uint32_t packed = gt | (eq << 16);
    uint32_t incl = packed;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    uint32_t before_w = 0, total = incl;
    if (W > 1) {
        if (lane == 31) scan[grp][wg] = incl;
        group_sync();
        total = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const uint32_t v = scan[grp][w];
            before_w += w < wg ? v : 0u;
            total += v;
        }
    } else {
        total = __shfl_sync(0xffffffffu, incl, 31);
    }
    const uint32_t need = (uint32_t)a.K - (total & 0xFFFFu);   // ties to take
    const uint32_t excl = before_w + incl - packed;
    uint32_t gt_before = excl & 0xFFFFu, eq_before = excl >> 16;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const bool is_gt = key[e] > tau, is_eq = key[e] == tau;
        if (is_gt || (is_eq && eq_before < need)) {
            out[gt_before + min(eq_before, need)] = pos(c_lo + e);
        }
        gt_before += is_gt ? 1u : 0u;
        eq_before += is_eq ? 1u : 0u;
    }
}

template <int PER, int W>
static sa_status launch_topk_rows(const TopkArgs &a, cudaStream_t st) {
    constexpr int RPC = kRowsThreads / (32 * W);
    topk_rows_kernel<PER, W><<<(a.rows + RPC - 1) / RPC, kRowsThreads, 0, st>>>(a);
    return cuda_ok(cudaGetLastError());
}

template <int G, bool FUSED>
static sa_status launch_topk_g(const TopkArgs &a, size_t smem, cudaStream_t st) {
    auto kern = FUSED ? topk_fused_kernel<G> : topk_kernel<G>;
    if ((FUSED ? prepare_kernel<topk_fused_kernel<G>>(smem, G > 8) : prepare_kernel<topk_kernel<G>>(smem, G > 8)) !=
        cudaSuccess)
        return SA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.rows * G));
    cfg.blockDim = dim3(topk_threads<G>());
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
    // Rows of at most 1024 columns: the register search (32 rounds over at most
    // 32 keys per lane).  Longer rows: the histogram select, whose passes cost
    // a few operations per key rather than 32.
    // (The fused indexer lives in the histogram kernel only.)
    if (!a.fused && a.row_len <= 256) return launch_topk_rows<8, 1>(a, st);
    if (!a.fused && a.row_len <= 512) return launch_topk_rows<16, 1>(a, st);
    if (!a.fused && a.row_len <= 1024) return launch_topk_rows<32, 1>(a, st);
    int g = 1;
    while (g < kTopkMaxCluster && (a.row_len + g - 1) / g > kTopkChunkTarget) g *= 2;
    int chunk = (a.row_len + g - 1) / g;
    chunk = (chunk + 3) & ~3;
    if (chunk > kTopkMaxChunk) return SA_ERR_UNSUPPORTED;
    a.chunk = chunk;
    // histograms, later reused for the compaction's per-lane flags (one word
    // per lane and 128-key group of each warp's span)
    const size_t nt = g > 1 ? topk_threads<2>() : topk_threads<1>();
    const size_t flag_words = (nt / 32) * (((size_t)chunk + 4 * nt - 1) / (4 * nt)) * 32;
    const size_t hist_words = std::max((g > 1) ? 2 * (size_t)kBinsMax : (size_t)kBinsMax / 2, flag_words);
    size_t smem = ((size_t)chunk + hist_words) * 4;
    if (a.fused) {   // then the key-tile ring, 128-byte aligned
        a.ring_off = (int)((((size_t)chunk + hist_words) + 31) & ~(size_t)31);
        smem = (size_t)a.ring_off * 4 + (size_t)kFusedStages * kFusedSlotBytes;
        if (smem > 227 * 1024) return SA_ERR_UNSUPPORTED;
        switch (g) {
            case 1: return launch_topk_g<1, true>(a, smem, st);
            case 2: return launch_topk_g<2, true>(a, smem, st);
            case 4: return launch_topk_g<4, true>(a, smem, st);
            case 8: return launch_topk_g<8, true>(a, smem, st);
            default: return launch_topk_g<16, true>(a, smem, st);
        }
    }
    switch (g) {
        case 1: return launch_topk_g<1, false>(a, smem, st);
        case 2: return launch_topk_g<2, false>(a, smem, st);
        case 4: return launch_topk_g<4, false>(a, smem, st);
        case 8: return launch_topk_g<8, false>(a, smem, st);
        default: return launch_topk_g<16, false>(a, smem, st);
    }
}

}  // namespace sa
