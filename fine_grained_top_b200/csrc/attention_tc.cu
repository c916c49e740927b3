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
// for a group of queries.  A CTA takes 2 GQ consecutive queries, GQ = 128 / Hq,
// as two 128-row tiles A and B (row = (query, head)), and walks the causal key
// range in contiguous 128-key tiles (starting at a tile that differs between
// neighbouring CTAs), each K and V tile serving both:
//   S_X = Q_X K^T       tcgen05.mma M=128, N=128, K=d -> TMEM
//   P_X = masked softmax of S_X (the row's query's selection as a 128-bit
//         mask per tile), bf16, written back over S_X in TMEM
//   O_X += P_X V        tcgen05.mma M=128, N=d, K=128, A (= P_X) from TMEM,
//                       V as an MN-major shared-memory operand -> TMEM
// The tensor core alternates between the tiles (P V and the next S of A,
// then of B), so the softmax of one tile runs while the other's matrix
// products execute.  The running maximum is only raised when a tile exceeds
// it by more than 2^8 (then O_X is rescaled in TMEM), so P stays below 256.
//
// The selection of each query is first expanded into a bitmap (one bit per
// key; selection_bitmap_kernel, which also validates the top-K rows), so that
// the TMA producer can fetch each tile's [2 GQ x 128-bit] mask with the K and
// V tiles and no warp waits on index loads.
//
// Warp roles: 0 TMA producer (Q once; a ring whose step i carries K and the
// mask of tile i with V of tile i - 1) and TMEM allocator; 1 MMA issuer;
// 2..5 softmax of tile A and 6..9 of tile B, one thread per row (TMEM lane
// quadrant = warp % 4) holding the row's 128 scores in registers.  Every wait
// is bounded.
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

namespace {

constexpr int kTile = 128;                  // keys per tile
constexpr int kTcThreads = 10 * 32;
constexpr int kBitmapThreads = 256;        // up to 4 rows of the selection bitmap per CTA
constexpr int kBitmapRowThreads = 64;
constexpr size_t kSmemLimit = 232448;       // opt-in dynamic shared memory per CTA

struct TcParams {
    int T, S, Hq;
    float scale_log2;
    uint16_t *out;
    float *lse;
    int *dev_status;
    int n_groups;
};

template <int D, int HQ>
struct TcCfg {
    static constexpr int GQ = 128 / HQ;                     // queries per 128-row tile
    static constexpr int kHalf = 128 * 128;                 // one 64-column SW128 half of a 128-row tile
    static constexpr int kQBytes = 128 * D * 2;             // 128 rows x D
    static constexpr int kKVBytes = kTile * D * 2;          // 128 keys x D
    static constexpr int kMaskBytes = 2 * GQ * 16;          // [2 GQ queries][4 words]
    // Step i of the ring carries K and the mask of tile i and V of tile i - 1.
    static constexpr size_t bytes(int ns) {
        return 1024 + 2 * kQBytes + (size_t)ns * (2 * kKVBytes + kMaskBytes) + 256;
    }
    static constexpr int kNS = bytes(3) <= kSmemLimit ? 3 : 2;
    static constexpr int kOffQ = 0;                         // [2 tiles]
    static constexpr int kOffK = 2 * kQBytes;               // [kNS]
    static constexpr int kOffV = kOffK + kNS * kKVBytes;    // [kNS]
    static constexpr int kOffMask = kOffV + kNS * kKVBytes;  // [kNS]
    static constexpr int kOffBar = kOffMask + kNS * kMaskBytes;
    static constexpr size_t kSmem = bytes(kNS);
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

// D (TMEM) += A (TMEM: row i in lane i, two bf16 per 32-bit column) x B (smem descriptor).
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0;"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same two forms with the accumulator always read (no predicate register).
__device__ __forceinline__ void tc_mma_ss_acc(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc) {
    asm volatile(
        "{ .reg .pred p; setp.eq.u32 p, 1, 1;"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc)
        : "memory");
}
__device__ __forceinline__ void tc_mma_ts_acc(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc) {
    asm volatile(
        "{ .reg .pred p; setp.eq.u32 p, 1, 1;"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc)
        : "memory");
}

__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x with flush-to-zero (the ex2.approx.ftz PTX instruction); 2^-inf = 0.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float y;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
    return y;
}
// Named barrier `id` over `n` threads (warps may reach it from different code).
__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// Packed pairs of f32 (one 64-bit register pair) for the f32x2 instructions.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// 2^y for a pair, on the FMA pipe instead of the ex2 unit.  Range reduction:
// adding 1.5 * 2^23 rounds y to the nearest integer r in the low mantissa bits
// of t (exact for |y| < 2^22), f = y - r lies in [-1/2, 1/2], and 2^f is the
// cubic of least maximum relative error on [-1/2, 1/2] (the minimax fit, found
// by the Remez exchange algorithm: max 7.48e-5, well below bf16's 2^-8
// spacing).  r is added to the exponent field of 2^f: the shifter's own bits
// shifted left by 23 vanish mod 2^32, so t_bits << 23 == r << 23.  y is first
// raised to -126, where 2^y is below 2^-125 (masked keys, y = -inf, end there
// rather than at 0; callers judge "nothing selected" by the running maximum).
constexpr float kExpShift = 12582912.0f;   // 1.5 * 2^23
constexpr float kExp2C0 = 9.999280572e-01f, kExp2C1 = 6.932609677e-01f, kExp2C2 = 2.426111400e-01f,
                kExp2C3 = 5.517166853e-02f;
__device__ __forceinline__ void exp2_pair_fma(uint64_t y, float &a, float &b) {
    float y0, y1;
    f2_split(y, y0, y1);
    const uint64_t yc = f2(fmaxf(y0, -126.f), fmaxf(y1, -126.f));
    const uint64_t t = add2(yc, f2(kExpShift, kExpShift));
    const uint64_t r = add2(t, f2(-kExpShift, -kExpShift));
    const uint64_t fr = fma2(r, f2(-1.f, -1.f), yc);
    uint64_t p = fma2(f2(kExp2C3, kExp2C3), fr, f2(kExp2C2, kExp2C2));
    p = fma2(p, fr, f2(kExp2C1, kExp2C1));
    p = fma2(p, fr, f2(kExp2C0, kExp2C0));
    float t0, t1, p0, p1;
    f2_split(t, t0, t1);
    f2_split(p, p0, p1);
    a = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
    b = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

// Row t of the bitmap: bit s of word s / 32 is set iff s is in S(t) (for the
// query at position p = S - T + t): the top-K entries <= p - W and the window
// {max(0, p-W+1) .. p}.  Built in shared memory, written whole (zeros past p).
// Entries beyond p are reported (SA_DEV_INDEX) and skipped; a row that is not
// strictly ascending before its -1 padding sets SA_DEV_ORDER.  64 threads
// build one row; a CTA holds blockDim.x / 64 rows.
__global__ void __launch_bounds__(kBitmapThreads) selection_bitmap_kernel(const int32_t *topk, int K, int W, int T,
                                                                          int S, int words, uint32_t *bitmap,
                                                                          int *dev_status) {
    extern __shared__ uint4 bits4[];   // [rows per CTA][words / 4]
    const int rows = (int)blockDim.x / kBitmapRowThreads;
    const int sub = (int)threadIdx.x / kBitmapRowThreads, lt = (int)threadIdx.x % kBitmapRowThreads;
    const int t = (int)blockIdx.x * rows + sub;
    const bool live = t < T;
    uint32_t *rowbits = reinterpret_cast<uint32_t *>(bits4) + (size_t)sub * words;
    if (live)
        for (int i = lt; i < words / 4; i += kBitmapRowThreads)
            reinterpret_cast<uint4 *>(rowbits)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    bool bad_idx = false, bad_ord = false;
    if (live) {
        const int p = S - T + t;
        const int32_t *row = topk + (int64_t)t * K;
        auto take = [&](int i, int e, int prev) {   // entry i holds e; prev is entry i - 1
            if (e < 0) return;
            if (i > 0 && !(prev >= 0 && prev < e)) bad_ord = true;
            if (e > p) {
                bad_idx = true;
                return;
            }
            if (e <= p - W) atomicOr(&rowbits[e >> 5], 1u << (e & 31));
        };
        if ((K & 3) == 0 && (reinterpret_cast<uintptr_t>(topk) & 15u) == 0) {
            const int4 *row4 = reinterpret_cast<const int4 *>(row);
            for (int i4 = lt; i4 < K / 4; i4 += kBitmapRowThreads) {
                const int4 v = __ldg(row4 + i4);
                const int prev = i4 > 0 ? __ldg(row + 4 * i4 - 1) : 0;
                take(4 * i4, v.x, prev);
                take(4 * i4 + 1, v.y, v.x);
                take(4 * i4 + 2, v.z, v.y);
                take(4 * i4 + 3, v.w, v.z);
            }
        } else {
            for (int i = lt; i < K; i += kBitmapRowThreads) take(i, __ldg(row + i), i > 0 ? __ldg(row + i - 1) : 0);
        }
        const int w0 = max(0, p - W + 1);
        for (int wi = (w0 >> 5) + lt; wi <= (p >> 5) && W > 0; wi += kBitmapRowThreads) {
            const int lo = max(w0, wi * 32), hi = min(p, wi * 32 + 31);
            const int n = hi - lo + 1;
            atomicOr(&rowbits[wi], (n == 32) ? 0xffffffffu : (((1u << n) - 1u) << (lo - wi * 32)));
        }
    }
    if (bad_idx) report(dev_status, SA_DEV_INDEX);
    if (bad_ord) report(dev_status, SA_DEV_ORDER);
    __syncthreads();
    if (live) {
        uint4 *dst = reinterpret_cast<uint4 *>(bitmap + (int64_t)t * words);
        for (int i = lt; i < words / 4; i += kBitmapRowThreads) dst[i] = reinterpret_cast<const uint4 *>(rowbits)[i];
    }
}

template <int D, int HQ>
__global__ void __launch_bounds__(kTcThreads, 1)
    masked_attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                          const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_m,
                          TcParams P) {
    using C = TcCfg<D, HQ>;
    constexpr int GQ = C::GQ;
    constexpr int NS = C::kNS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + C::kOffBar);
    uint64_t *q_full = bar;
    uint64_t *kv_full = bar + 1, *kv_empty = kv_full + NS;   // [NS] K(i), V(i - 1) of step i
    uint64_t *m_full = kv_empty + NS, *m_empty = m_full + NS; // [NS] mask of tile i
    uint64_t *s_full = m_empty + NS;                          // [2 tiles] S_X(kt) in TMEM
    uint64_t *p_full = s_full + 2;                            // [2 tiles] P_X(kt) written over it
    uint64_t *o_done = p_full + 2;                            // [2 tiles] the last P_X V done
    uint64_t *drain = o_done + 2;
    constexpr int kSlotWord = 8 + 4 * NS;                     // tmem_slot, abort flag after the barriers
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + kSlotWord);
    static_assert(kSlotWord * 8 + 8 <= 256, "barrier region");
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    uint32_t *masks = reinterpret_cast<uint32_t *>(sm + C::kOffMask);   // [NS][2 GQ][4]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = P.n_groups - 1 - blockIdx.x;                  // heavy (late) groups first
    const int t0 = g * 2 * GQ;
    const int nq = min(2 * GQ, P.T - t0);
    const int p_last = P.S - P.T + t0 + nq - 1;                 // position of the CTA's last query
    const int n_tiles = p_last / kTile + 1;
    // The CTA visits its key tiles starting from a different one than its
    // neighbours (the softmax does not depend on the order), so that CTAs
    // running at the same time read different K/V tiles from L2.
    const int rot = (int)(blockIdx.x % (unsigned)n_tiles);
    auto tile_of = [&](int i) { return i + rot < n_tiles ? i + rot : i + rot - n_tiles; };

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int i = 0; i < NS; ++i) {
            mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1);
            mbar_init(&m_full[i], 1); mbar_init(&m_empty[i], 8);
        }
        for (int i = 0; i < 2; ++i) { mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 4); mbar_init(&o_done[i], 1); }
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
    const uint32_t tmem = *tmem_slot;   // S_A, S_B at columns 0, 128; O_A, O_B at 256, 256 + D

    if (warp < 2) {
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            mbar_arrive_expect_tx(q_full, 2 * C::kQBytes);
            for (int x = 0; x < 2; ++x)
                for (int h = 0; h < D / 64; ++h)
                    tma_load_2d(sm + C::kOffQ + x * C::kQBytes + h * C::kHalf, &map_q, h * 64, (t0 + x * GQ) * HQ,
                                q_full);
            // step i: K and the mask of tile i, V of tile i - 1
            for (int i = 0; i <= n_tiles && ok; ++i) {
                const int ns = i % NS;
                const uint32_t par = ((uint32_t)(i / NS) & 1u) ^ 1u;
                ok = mbar_wait(&kv_empty[ns], par, abort_flag);
                if (!ok) break;
                mbar_arrive_expect_tx(&kv_full[ns], (i < n_tiles ? C::kKVBytes : 0) + (i >= 1 ? C::kKVBytes : 0));
                if (i < n_tiles)
                    for (int h = 0; h < D / 64; ++h)
                        tma_load_2d(sm + C::kOffK + ns * C::kKVBytes + h * C::kHalf, &map_k, h * 64,
                                    tile_of(i) * kTile, &kv_full[ns]);
                if (i >= 1)
                    for (int h = 0; h < D / 64; ++h)
                        tma_load_2d(sm + C::kOffV + ns * C::kKVBytes + h * C::kHalf, &map_v, h * 64,
                                    tile_of(i - 1) * kTile, &kv_full[ns]);
                if (i < n_tiles) {
                    ok = mbar_wait(&m_empty[ns], par, abort_flag);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&m_full[ns], C::kMaskBytes);
                    tma_load_2d(sm + C::kOffMask + ns * C::kMaskBytes, &map_m, tile_of(i) * 4, t0, &m_full[ns]);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTile);
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, D) | (1u << 16);   // B (V) MN-major
            // Descriptors are built once; an operand at byte offset o from a base
            // is base + (o >> 4) (the 14-bit address field never carries over).
            const uint64_t q_d = desc_k(smem_u32(sm + C::kOffQ));
            const uint64_t k_d = desc_k(smem_u32(sm + C::kOffK));
            const uint64_t v_d = desc_mn(smem_u32(sm + C::kOffV), C::kHalf);
            // S_X(kt) = Q_X K(kt)^T over the columns of S_X, which last held
            // P_X(kt - 1), read by P V of tile kt - 1 that this thread issued
            // earlier (the tensor core runs one thread's MMAs in order).
            auto s_mma = [&](int x, int kt) {
                const uint64_t qd = q_d + (uint64_t)(x * (C::kQBytes >> 4));
                const uint64_t kd = k_d + (uint64_t)((kt % NS) * (C::kKVBytes >> 4));
                const uint32_t dt = tmem + (uint32_t)(x * kTile);
                tc_mma_f16(dt, qd, kd, idesc_s, 0u);
#pragma unroll
                for (int kk = 1; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * C::kHalf + (kk & 3) * 32) >> 4);
                    tc_mma_ss_acc(dt, qd + off, kd + off, idesc_s);
                }
                tc_commit(&s_full[x]);
            };
            // O_X += P_X V: P_X in the first 64 columns of S_X, V(kt) MN-major
            auto pv_mma = [&](int x, int kt, uint64_t vd) {
                const uint32_t dt = tmem + 256u + (uint32_t)(x * D), at = tmem + (uint32_t)(x * kTile);
                tc_mma_f16_ts(dt, at, vd, idesc_o, kt > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 1; kk < kTile / 16; ++kk)
                    tc_mma_ts_acc(dt, at + (uint32_t)(kk * 8), vd + (uint64_t)((kk * 2048) >> 4), idesc_o);
                if (kt == n_tiles - 1) tc_commit(&o_done[x]);
            };
            bool ok = mbar_wait(q_full, 0, abort_flag) && mbar_wait(&kv_full[0], 0, abort_flag);
            if (ok) {
                tc_fence_after();
                s_mma(0, 0);
                s_mma(1, 0);
                tc_commit(&kv_empty[0]);
            }
            // step kt + 1 holds V(kt) and K(kt + 1); one commit releases both
            for (int kt = 0; kt < n_tiles && ok; ++kt) {
                const int kn = kt + 1, ns = kn % NS;
                const uint32_t par = (uint32_t)kt & 1u;
                ok = mbar_wait(&kv_full[ns], (uint32_t)(kn / NS) & 1u, abort_flag) &&
                     mbar_wait(&p_full[0], par, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint64_t vd = v_d + (uint64_t)(ns * (C::kKVBytes >> 4));
                pv_mma(0, kt, vd);
                if (kn < n_tiles) s_mma(0, kn);
                ok = mbar_wait(&p_full[1], par, abort_flag);
                if (!ok) break;
                tc_fence_after();
                pv_mma(1, kt, vd);
                if (kn < n_tiles) s_mma(1, kn);
                tc_commit(&kv_empty[ns]);
            }
            tc_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, &no_abort);
        }
        __syncwarp();
    }
    // Once all warps are past their last TMEM access, warp 0 frees TMEM.
    tc_fence_before();
    named_sync(1, kTcThreads);
    if (warp == 0) {
        uint8_t *smb = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
        uint32_t *slot = reinterpret_cast<uint32_t *>(reinterpret_cast<uint64_t *>(smb + C::kOffBar) + kSlotWord);
        if (lane == 0 && *reinterpret_cast<volatile int *>(slot + 1)) report(P.dev_status, SA_DEV_TIMEOUT);
        tc_fence_after();
        tmem_dealloc(*slot, 512);
    }
    } else {
        // ------------------------------------------------------------ softmax (one thread per row)
        const int x = (warp - 2) >> 2;             // tile A (0) or B (1)
        const int quad = warp & 3;
        const int r = quad * 32 + lane;            // TMEM lane = row = (query, head)
        const int qi = x * GQ + r / HQ, h = r % HQ;
        const bool act = qi < nq;
        const uint32_t lane_t = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t s_t = lane_t + (uint32_t)(x * kTile);
        const uint32_t o_t = lane_t + 256u + (uint32_t)(x * D);
        const float sl2 = P.scale_log2;
        const uint64_t sl2x2 = f2(sl2, sl2);
        float m_used = -CUDART_INF_F;              // log2 units: score x scale x log2 e
        uint64_t l2 = f2(0.f, 0.f);                // row sum, as two partial sums
        bool ok = true;
        for (int kt = 0; kt < n_tiles; ++kt) {
            const int ks = kt % NS;
            ok = __all_sync(0xffffffffu, mbar_wait(&m_full[ks], (uint32_t)(kt / NS) & 1u, abort_flag) &&
                                             mbar_wait(&s_full[x], (uint32_t)kt & 1u, abort_flag));
            if (!ok) break;
            tc_fence_after();
            uint32_t mk[4] = {0u, 0u, 0u, 0u};
            if (act) {
                const uint4 m4 = *reinterpret_cast<const uint4 *>(masks + ks * (C::kMaskBytes / 4) + qi * 4);
                mk[0] = m4.x; mk[1] = m4.y; mk[2] = m4.z; mk[3] = m4.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&m_empty[ks]);
            // the row's 128 scores, -inf outside the selection, and their maximum
            uint32_t v[128];
#pragma unroll
            for (int c = 0; c < 128; c += 16)
                tmem_ld_x16(s_t + (uint32_t)c, *reinterpret_cast<uint32_t(*)[16]>(&v[c]));
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 128; ++c) asm volatile("" : "+r"(v[c]));   // keep uses after the wait
            float mx[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
            for (int c = 0; c < 128; ++c)
                if (!((mk[c >> 5] >> (c & 31)) & 1u)) v[c] = 0xff800000u;   // -inf
#pragma unroll
            for (int c = 0; c < 128; c += 2) {
                const int a = (c >> 1) & 3;
                mx[a] = max3(mx[a], __uint_as_float(v[c]), __uint_as_float(v[c + 1]));
            }
            const float tmax = fmaxf(max3(mx[0], mx[1], mx[2]), mx[3]) * sl2;
            const bool raise = tmax > m_used + 8.f;
            const bool resc = raise && m_used != -CUDART_INF_F;   // O_X holds earlier tiles
            if (__any_sync(0xffffffffu, resc)) {
                // P_X V of tile kt - 1 is done: this thread saw S_X(kt), issued after it
                const float f = resc ? ex2(m_used - tmax) : 1.f;
#pragma unroll 1
                for (int c = 0; c < D; c += 16) {
                    uint32_t o[16];
                    tmem_ld_x16(o_t + (uint32_t)c, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st_x16(o_t + (uint32_t)c, o);
                }
            }
            if (raise) {
                if (resc) {
                    const float f = ex2(m_used - tmax);
                    l2 = fma2(l2, f2(f, f), f2(0.f, 0.f));
                } else {
                    l2 = f2(0.f, 0.f);
                }
                m_used = tmax;
            }
            const float nb = (m_used == -CUDART_INF_F) ? 0.f : -m_used;
            const uint64_t nbx2 = f2(nb, nb);
            // P = 2^(x scale log2 e - m_used), keys 2i, 2i + 1 -> column i of S_X
            // (all of S_X has been read into registers)
#pragma unroll
            for (int c = 0; c < 128; c += 32) {
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float a, b;
                    const uint64_t y =
                        fma2(f2(__uint_as_float(v[c + 2 * i]), __uint_as_float(v[c + 2 * i + 1])), sl2x2, nbx2);
                    if ((i & 7) == 7) {   // one pair in eight on the FMA pipe, the rest on the ex2 unit
                        exp2_pair_fma(y, a, b);
                    } else {
                        f2_split(y, a, b);
                        a = ex2(a);
                        b = ex2(b);
                    }
                    l2 = add2(l2, f2(a, b));
                    pk[i] = pack_bf16(a, b);
                }
                tmem_st_x16(s_t + (uint32_t)(c / 2), pk);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[x]);
        }
        // ---- epilogue: O_X / l
        if (ok && __all_sync(0xffffffffu, mbar_wait(&o_done[x], 0u, abort_flag))) {
            tc_fence_after();
            float la, lb;
            f2_split(l2, la, lb);
            const float l = la + lb;
            // no selected key at all leaves the maximum at -inf (l then only holds
            // the polynomial's floor values of masked keys)
            const bool any = m_used != -CUDART_INF_F;
            const float inv = any && l > 0.f ? 1.f / l : 0.f;
            const int t = t0 + qi;
            uint16_t *orow = P.out + ((int64_t)t * HQ + h) * D;
#pragma unroll
            for (int c = 0; c < D; c += 16) {
                uint32_t o[16];
                tmem_ld_x16(o_t + (uint32_t)c, o);
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
                P.lse[(int64_t)t * HQ + h] = (any && l > 0.f ? m_used + __log2f(l) : -CUDART_INF_F) * 0.69314718055994531f;
        }
        tc_fence_before();
        named_sync(1, kTcThreads);   // TMEM is freed by warp 0 after this
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

// selection bitmap [T rows x words] uint32, box = `rows_box` rows x 4 words (one 128-key tile)
bool map_bitmap(CUtensorMap *m, const void *base, uint64_t rows, int words, int rows_box) {
    auto enc = encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)words, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)words * 4};
    cuuint32_t box[2] = {4, (cuuint32_t)rows_box};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int bitmap_words(int S) { return (S + kTile - 1) / kTile * 4; }

template <int D, int HQ>
sa_status launch_tc(const PrefillArgs &a, cudaStream_t st) {
    using C = TcCfg<D, HQ>;
    constexpr int GQ = C::GQ;
    static_assert(C::kSmem <= kSmemLimit, "shared memory");
    TcParams p;
    p.T = a.T; p.S = a.S; p.Hq = a.Hq;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out = a.out; p.lse = a.lse; p.dev_status = a.dev_status;
    p.n_groups = (a.T + 2 * GQ - 1) / (2 * GQ);
    const int words = bitmap_words(a.S);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(a.workspace);
    CUtensorMap mq, mk, mv, mm;
    if (!map_rows(&mq, a.q, (uint64_t)a.T * HQ, D) || !map_rows(&mk, a.k, (uint64_t)a.S, D) ||
        !map_rows(&mv, a.v, (uint64_t)a.S, D) || !map_bitmap(&mm, bitmap, (uint64_t)a.T, words, 2 * GQ))
        return SA_ERR_CUDA;
    // 4 rows per CTA while their bitmap rows fit in 48 KB, else one
    const int brows = (size_t)words * 4 * 4 <= 48 * 1024 ? 4 : 1;
    const size_t bsmem = (size_t)words * 4 * brows;
    if (prepare_kernel<selection_bitmap_kernel>(bsmem, false) != cudaSuccess) return SA_ERR_CUDA;
    selection_bitmap_kernel<<<(a.T + brows - 1) / brows, kBitmapRowThreads * brows, bsmem, st>>>(
        a.topk, a.K, a.W, a.T, a.S, words, bitmap, a.dev_status);
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
