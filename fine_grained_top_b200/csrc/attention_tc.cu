// attention_tc.cu -- prefill sparse attention as masked tensor-core tiles.
//
// Same result as sparse_attn_kernel (attention.cu):
//   O[t,h] = sum_{s in S(t)} softmax_s(q[t,h] . k[s] * scale) v[s],
//   S(t) = {s in TopK(t) : s <= p - W} U {max(0, p-W+1) .. p}
// ("A Guide to Sparse Attention in Large Models", section 2: the masked form
// softmax(QK^T * Mask + (1 - Mask)(-inf)) V with Mask[i,j] = 1 iff j in S(i)).
//
// When each query selects a large share of its causal keys, gathering the
// selected rows per query costs more L2 traffic than streaming the keys once
// for a group of queries.  This kernel takes GQ = 128 / Hq consecutive queries
// (M = GQ x Hq = 128 query-head rows) and walks the causal key range in
// contiguous 128-key tiles:
//   S = Q K^T         tcgen05.mma M=128, N=128, K=d  -> TMEM (double buffer)
//   P = masked softmax of S, one thread per row (the row's query's selection
//       as a 128-bit mask per tile), written to shared memory as bf16
//   O += P V          tcgen05.mma M=128, N=d, K=128 (V as an MN-major operand)
//                     -> TMEM
// The running maximum is only raised when a tile exceeds it by more than 2^8
// (then O is rescaled in TMEM), so P stays below 256.
//
// The selection of each query is first expanded into a bitmap (one bit per
// key; selection_bitmap_kernel, which also validates the top-K rows), so that
// the TMA producer can fetch each tile's [GQ x 128-bit] mask with the K and V
// tiles and no warp waits on index loads.
//
// Warp roles: 0 TMA producer (Q once; K, V and mask rings of 2) and TMEM
// allocator; 1 MMA issuer; 2..5 softmax (TMEM lane quadrant = warp % 4).
// Every wait is bounded.
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

namespace {

constexpr int kTile = 128;                  // keys per tile
constexpr int kTcThreads = 6 * 32;
constexpr int kBitmapThreads = 256;

struct TcParams {
    int T, S, Hq;
    float scale_log2;
    uint16_t *out;
    float *lse;
    int *dev_status;
    int n_groups;
};

template <int D>
struct TcCfg {
    static constexpr int kHalf = 128 * 128;                 // one 64-column SW128 half of a 128-row tile
    static constexpr int kQBytes = 128 * D * 2;             // 128 rows x D
    static constexpr int kKVBytes = kTile * D * 2;          // 128 keys x D
    static constexpr int kPBytes = 128 * kTile * 2;         // 128 rows x 128 keys
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + 2 * kKVBytes;
    static constexpr int kOffP = kOffV + 2 * kKVBytes;
    static constexpr int kOffMask = kOffP + kPBytes;           // [2 slots of 512 B][GQ rows][4 words]
    static constexpr int kOffBar = kOffMask + 2 * 512;
    static constexpr size_t kSmem = 1024 + kOffBar + 256;
};

__device__ __forceinline__ uint64_t desc_k(uint32_t addr) { return smem_desc(addr, 1024, 2); }

// MN-major SW128 operand (V as B: N = head dims contiguous, K = keys):
// 64-element MN chunks LBO bytes apart, 8-row K groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mn(uint32_t addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((1024 >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Set bits [a, b] (inclusive, tile-relative, clipped to [0, 127]) of m[4].
__device__ __forceinline__ void set_range(uint32_t (&m)[4], int a, int b) {
    a = max(a, 0);
    b = min(b, kTile - 1);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const int lo = max(a, 32 * w), hi = min(b, 32 * w + 31);
        if (lo <= hi) {
            const int n = hi - lo + 1;
            const uint32_t bits = (n == 32) ? 0xffffffffu : (((1u << n) - 1u) << (lo - 32 * w));
            m[w] |= bits;
        }
    }
}

// Row t of the bitmap: bit s of word s / 32 is set iff s is in S(t) (for the
// query at position p = S - T + t): the top-K entries <= p - W and the window
// {max(0, p-W+1) .. p}.  Built in shared memory, written whole (zeros past p).
// Entries beyond p are reported (SA_DEV_INDEX) and skipped; a row that is not
// strictly ascending before its -1 padding sets SA_DEV_ORDER.
__global__ void __launch_bounds__(kBitmapThreads) selection_bitmap_kernel(const int32_t *topk, int K, int W, int T,
                                                                          int S, int words, uint32_t *bitmap,
                                                                          int *dev_status) {
    extern __shared__ uint32_t rowbits[];   // [words]
    const int t = blockIdx.x;
    const int p = S - T + t;
    for (int i = threadIdx.x; i < words; i += kBitmapThreads) rowbits[i] = 0u;
    __syncthreads();
    const int32_t *row = topk + (int64_t)t * K;
    bool bad_idx = false, bad_ord = false;
    for (int i = threadIdx.x; i < K; i += kBitmapThreads) {
        const int e = __ldg(row + i);
        if (e < 0) continue;
        if (i > 0) {
            const int prev = __ldg(row + i - 1);
            if (!(prev >= 0 && prev < e)) bad_ord = true;
        }
        if (e > p) { bad_idx = true; continue; }
        if (e <= p - W) atomicOr(&rowbits[e >> 5], 1u << (e & 31));
    }
    if (bad_idx) report(dev_status, SA_DEV_INDEX);
    if (bad_ord) report(dev_status, SA_DEV_ORDER);
    const int w0 = max(0, p - W + 1);
    for (int wi = (w0 >> 5) + (int)threadIdx.x; wi <= (p >> 5) && W > 0; wi += kBitmapThreads) {
        const int a = max(w0, wi * 32), b = min(p, wi * 32 + 31);
        const int n = b - a + 1;
        atomicOr(&rowbits[wi], (n == 32) ? 0xffffffffu : (((1u << n) - 1u) << (a - wi * 32)));
    }
    __syncthreads();
    uint32_t *dst = bitmap + (int64_t)t * words;
    for (int i = threadIdx.x; i < words; i += kBitmapThreads) dst[i] = rowbits[i];
}

template <int D, int HQ>
__global__ void __launch_bounds__(kTcThreads, 1)
    masked_attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                          const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_m,
                          TcParams P) {
    using C = TcCfg<D>;
    constexpr int GQ = 128 / HQ;   // queries per CTA
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + C::kOffBar);
    uint64_t *q_full = bar + 0;
    uint64_t *k_full = bar + 1, *k_empty = bar + 3;      // [2]
    uint64_t *v_full = bar + 5, *v_empty = bar + 7;      // [2]
    uint64_t *s_full = bar + 9, *s_empty = bar + 11;     // [2]
    uint64_t *p_full = bar + 13, *o_done = bar + 14;
    uint64_t *m_full = bar + 15, *m_empty = bar + 17;    // [2]
    uint64_t *drain = bar + 19;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 20);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint32_t *masks = reinterpret_cast<uint32_t *>(sm + C::kOffMask);   // [2][GQ][4]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = P.n_groups - 1 - blockIdx.x;                  // heavy (late) groups first
    const int t0 = g * GQ;
    const int nq = min(GQ, P.T - t0);
    const int p_last = P.S - P.T + t0 + nq - 1;                 // position of the group's last query
    const int n_tiles = p_last / kTile + 1;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
            mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
            mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 4);
            mbar_init(&m_full[i], 1); mbar_init(&m_empty[i], 4);
        }
        mbar_init(p_full, 4);
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&map_q);
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_v);
        tma_prefetch_desc(&map_m);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t t_s = tmem, t_o = tmem + 256;                // S buffers at columns 0, 128; O at 256

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            mbar_arrive_expect_tx(q_full, C::kQBytes);
            for (int h = 0; h < D / 64; ++h)
                tma_load_2d(sm + C::kOffQ + h * C::kHalf, &map_q, h * 64, t0 * HQ, q_full);
            for (int kt = 0; kt < n_tiles && ok; ++kt) {
                const int s = kt & 1;
                const uint32_t par = ((uint32_t)(kt >> 1) & 1u) ^ 1u;
                ok = mbar_wait(&k_empty[s], par, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&k_full[s], C::kKVBytes);
                for (int h = 0; h < D / 64; ++h)
                    tma_load_2d(sm + C::kOffK + s * C::kKVBytes + h * C::kHalf, &map_k, h * 64, kt * kTile, &k_full[s]);
                ok = mbar_wait(&m_empty[s], par, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&m_full[s], GQ * 16);
                tma_load_2d(masks + s * 128, &map_m, kt * 4, t0, &m_full[s]);
                ok = mbar_wait(&v_empty[s], par, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&v_full[s], C::kKVBytes);
                for (int h = 0; h < D / 64; ++h)
                    tma_load_2d(sm + C::kOffV + s * C::kKVBytes + h * C::kHalf, &map_v, h * 64, kt * kTile, &v_full[s]);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTile);
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D) | (1u << 16);   // B (V) MN-major
            const uint32_t qa = smem_u32(sm + C::kOffQ);
            const uint32_t pa = smem_u32(sm + C::kOffP);
            bool ok = mbar_wait(q_full, 0, abort_flag);
            auto issue_s = [&](int kt) -> bool {
                const int s = kt & 1;
                const uint32_t use = (uint32_t)(kt >> 1) & 1u;
                if (!mbar_wait(&k_full[s], use, abort_flag) || !mbar_wait(&s_empty[s], use ^ 1u, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t ka = smem_u32(sm + C::kOffK + s * C::kKVBytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (uint32_t)((kk >> 2) * C::kHalf + (kk & 3) * 32);
                    tc_mma_f16(t_s + (uint32_t)(s * kTile), desc_k(qa + off), desc_k(ka + off), idesc_s, kk > 0);
                }
                tc_commit(&k_empty[s]);
                tc_commit(&s_full[s]);
                return true;
            };
            if (ok) ok = issue_s(0);
            if (ok && n_tiles > 1) ok = issue_s(1);
            for (int kt = 0; kt < n_tiles && ok; ++kt) {
                const int s = kt & 1;
                ok = mbar_wait(p_full, (uint32_t)kt & 1u, abort_flag) &&
                     mbar_wait(&v_full[s], (uint32_t)(kt >> 1) & 1u, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t va = smem_u32(sm + C::kOffV + s * C::kKVBytes);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint32_t poff = (uint32_t)((kk >> 2) * C::kHalf + (kk & 3) * 32);
                    tc_mma_f16(t_o, desc_k(pa + poff), desc_mn(va + (uint32_t)kk * 2048u, C::kHalf), idesc_o,
                               (kt > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&v_empty[s]);
                tc_commit(o_done);
                if (kt + 2 < n_tiles) ok = issue_s(kt + 2);
            }
            tc_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, &no_abort);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax (one thread per row)
        const int quad = warp & 3;
        const int r = quad * 32 + lane;            // TMEM lane = row = (query, head)
        const int q = r / HQ, h = r % HQ;
        const bool act = q < nq;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        uint8_t *prow = sm + C::kOffP + r * 128;   // this row in each 64-key half of P
        float m_used = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        for (int kt = 0; kt < n_tiles && ok; ++kt) {
            const int s = kt & 1;
            const uint32_t use = (uint32_t)(kt >> 1) & 1u;
            ok = __all_sync(0xffffffffu, mbar_wait(&m_full[s], use, abort_flag) && mbar_wait(&s_full[s], use, abort_flag));
            if (!ok) break;
            tc_fence_after();
            uint32_t mk[4];
            {
                const uint32_t *src = masks + s * 128 + (act ? q : 0) * 4;
                mk[0] = act ? src[0] : 0u; mk[1] = act ? src[1] : 0u;
                mk[2] = act ? src[2] : 0u; mk[3] = act ? src[3] : 0u;
            }
            // the row's 128 scores, masked and scaled in place (one register array)
            float x[kTile];
#pragma unroll
            for (int c = 0; c < kTile; c += 16) {
                uint32_t tmp[16];
                tmem_ld_x16(t_s + lane_off + (uint32_t)(s * kTile + c), tmp);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) x[c + i] = __uint_as_float(tmp[i]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) { mbar_arrive(&s_empty[s]); mbar_arrive(&m_empty[s]); }
            float tmax = -CUDART_INF_F;
#pragma unroll
            for (int c = 0; c < kTile; ++c) {
                const bool on = (mk[c >> 5] >> (c & 31)) & 1u;
                x[c] = on ? x[c] * P.scale_log2 : -CUDART_INF_F;
                tmax = fmaxf(tmax, x[c]);
            }
            // PV of the previous tile must be done before O is rescaled or P rewritten
            if (kt > 0) {
                ok = __all_sync(0xffffffffu, mbar_wait(o_done, (uint32_t)(kt - 1) & 1u, abort_flag));
                if (!ok) break;
                tc_fence_after();
            }
            const bool raise = tmax > m_used + 8.f;
            if (__any_sync(0xffffffffu, raise && l > 0.f)) {
                // rescale this warp's O rows whose maximum rose (rare)
                const float f = (raise && l > 0.f) ? exp2f(m_used - tmax) : 1.f;
#pragma unroll
                for (int c = 0; c < D; c += 16) {
                    uint32_t o[16];
                    tmem_ld_x16(t_o + lane_off + (uint32_t)c, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st_x16(t_o + lane_off + (uint32_t)c, o);
                }
                tmem_st_wait();
            }
            if (raise) {
                if (l > 0.f) l *= exp2f(m_used - tmax);
                m_used = tmax;
            }
            const float base = (m_used == -CUDART_INF_F) ? 0.f : m_used;
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < kTile; c += 8) {
                uint32_t pk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float a = exp2f(x[c + 2 * i] - base), b2 = exp2f(x[c + 2 * i + 1] - base);
                    rs += a + b2;
                    pk[i] = pack_bf16(a, b2);
                }
                // chunk (c / 8) of the row: 64-key half c / 64, 16-byte chunk (c % 64) / 8, SW128
                const int half = c >> 6, ch = (c & 63) >> 3;
                *reinterpret_cast<uint4 *>(prow + half * C::kHalf + ((ch ^ (r & 7)) << 4)) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            l += rs;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // P writes -> tensor core reads
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // ---- epilogue: O / l
        if (ok && __all_sync(0xffffffffu, mbar_wait(o_done, (uint32_t)(n_tiles - 1) & 1u, abort_flag))) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const int t = t0 + q;
            uint16_t *orow = P.out + ((int64_t)t * HQ + h) * D;
#pragma unroll
            for (int c = 0; c < D; c += 16) {
                uint32_t o[16];
                tmem_ld_x16(t_o + lane_off + (uint32_t)c, o);
                tmem_ld_wait();
                if (act) {
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        pk[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            if (act && P.lse)
                P.lse[(int64_t)t * HQ + h] = (l > 0.f ? m_used + __log2f(l) : -CUDART_INF_F) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) report(P.dev_status, SA_DEV_TIMEOUT);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// rows x D bf16 row-major, box = 128 rows x 64 columns, 128B swizzle
bool map_rows(CUtensorMap *m, const void *base, uint64_t rows, int D) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// selection bitmap [T rows x words] uint32, box = GQ rows x 4 words (one 128-key tile)
bool map_bitmap(CUtensorMap *m, const void *base, uint64_t rows, int words, int gq) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)words, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)words * 4};
    cuuint32_t box[2] = {4, (cuuint32_t)gq};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int bitmap_words(int S) { return (S + kTile - 1) / kTile * 4; }

template <int D, int HQ>
sa_status launch_tc(const PrefillArgs &a, cudaStream_t st) {
    using C = TcCfg<D>;
    constexpr int GQ = 128 / HQ;
    TcParams p;
    p.T = a.T; p.S = a.S; p.Hq = a.Hq;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out = a.out; p.lse = a.lse; p.dev_status = a.dev_status;
    p.n_groups = (a.T + GQ - 1) / GQ;
    const int words = bitmap_words(a.S);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(a.workspace);
    CUtensorMap mq, mk, mv, mm;
    if (!map_rows(&mq, a.q, (uint64_t)a.T * HQ, D) || !map_rows(&mk, a.k, (uint64_t)a.S, D) ||
        !map_rows(&mv, a.v, (uint64_t)a.S, D) || !map_bitmap(&mm, bitmap, (uint64_t)a.T, words, GQ))
        return SA_ERR_CUDA;
    const size_t bsmem = (size_t)words * 4;
    if (prepare_kernel<selection_bitmap_kernel>(bsmem, false) != cudaSuccess) return SA_ERR_CUDA;
    selection_bitmap_kernel<<<a.T, kBitmapThreads, bsmem, st>>>(a.topk, a.K, a.W, a.T, a.S, words, bitmap,
                                                               a.dev_status);
    if (prepare_kernel<masked_attn_tc_kernel<D, HQ>>(C::kSmem, false) != cudaSuccess) return SA_ERR_CUDA;
    masked_attn_tc_kernel<D, HQ><<<p.n_groups, kTcThreads, C::kSmem, st>>>(mq, mk, mv, mm, p);
    return cuda_ok(cudaGetLastError());
}

}  // namespace

// Masked tensor-core prefill: head dim 64 / 128, Hq in {4, 8, 16, 32} (a
// 128-row tile holds whole queries), and selections dense enough that
// streaming every causal key once per query group beats gathering the
// selected rows per query (S * Hq <= 256 * (K + W)).  Needs the bitmap
// workspace of prefill_tc_workspace_bytes.
bool prefill_tc_supported(const PrefillArgs &a) {
    return (a.d == 64 || a.d == 128) && (a.Hq == 4 || a.Hq == 8 || a.Hq == 16 || a.Hq == 32) &&
           (int64_t)a.S * a.Hq <= 256 * ((int64_t)a.K + a.W) && bitmap_words(a.S) * 4 <= 200 * 1024;
}

size_t prefill_tc_workspace_bytes(int T, int S) { return (size_t)T * bitmap_words(S) * 4; }

sa_status launch_prefill_tc(const PrefillArgs &a, cudaStream_t st) {
    if (a.T == 0) return SA_OK;
#define SA_TC_CASE(DD, HH) \
    if (a.d == DD && a.Hq == HH) return launch_tc<DD, HH>(a, st);
    SA_TC_CASE(128, 16) SA_TC_CASE(128, 4) SA_TC_CASE(128, 8) SA_TC_CASE(128, 32)
    SA_TC_CASE(64, 16) SA_TC_CASE(64, 4) SA_TC_CASE(64, 8) SA_TC_CASE(64, 32)
#undef SA_TC_CASE
    return SA_ERR_UNSUPPORTED;
}

}  // namespace sa
