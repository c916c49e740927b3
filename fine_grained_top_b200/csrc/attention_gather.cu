// attention_gather.cu -- prefill sparse attention over gathered key rows on
// the tensor cores (tcgen05, TMEM), for selections that are sparse in the
// causal range (each query keeps a small share of its keys).
//
//   S(t) = {s in TopK(t) : s <= p - W}  U  {max(0, p-W+1) .. p}
//   O[t,h] = sum_{s in S(t)} softmax_s(q[t,h] . k[s] * scale) v[s]
//
// ("A Guide to Sparse Attention in Large Models", section 2: the masked
// form with Mask[i,j] = 1 iff j in S(i); section 4.2: the index-based
// implementation computes only on the selected subset.)  All query heads of a
// token share S(t) and the single KV head.
//
// The selected rows of different queries barely overlap, so every query
// gathers its own K/V rows; the kernel is built to keep that gather at the
// L2 -> shared-memory rate.  Per query, keys go on the MMA's M dimension and
// the query's heads on N (N = Hq rounded up to 16), so a 128-key tile is one
// tcgen05.mma group:
//   S^T = K Q^T         M = 128 keys, N = heads, K = d        -> TMEM
//   P^T = softmax over keys of S^T (per head; one thread per key lane)
//   O^T += V^T P^T      M = d (V as an MN-major operand), N = heads,
//                       K = 128 keys (P^T, MN-major, from shared memory) -> TMEM
// The running maximum of a head is raised only when a tile exceeds it by more
// than 2^8 (then O^T and the row sums are rescaled), so P stays below 256.
//
// Persistent CTAs (one per SM) take queries T-1-c, T-1-c-G, ... (heavy first)
// and stream their tiles through a pipeline of warp roles (kGW = 2 gather
// warps per side; four per side measured slower: fewer registers per thread):
//   index builder (one warp): copies the query's top-K row to shared memory,
//               validates it (SA_DEV_INDEX / SA_DEV_ORDER), finds the prefix
//               of entries <= p - W, writes the byte offsets of each 128-key
//               tile's cache rows (top-K prefix, then the window; a slot past
//               the selection repeats the tile's first row, whose score is
//               masked) into a ring, and publishes the tile's record to the
//               MMA and softmax warps
//   gather (warps 0 .. 2 kGW - 1): 16-byte cp.async of every selected K row
//               (with the query's Q rows at its first tile) and V row into
//               128B-swizzled tiles of separate K and V rings; completion is
//               tracked by the slot's mbarrier (cp.async.mbarrier.arrive.noinc)
//   S issuer (one thread) and TMEM owner
//   P V issuer (one thread)
//   softmax (eight warps): tile g in two groups of four warps, each group
//               owning half of the heads (TMEM lane quadrant = warp % 4), one
//               vote per tile, P^T written MN-major (16-byte rows of 8 heads);
//               each query's epilogue (O^T / l -> out bf16, lse) runs once its
//               last P V is known to be done
// Every wait is bounded (SA_DEV_TIMEOUT), and the softmax warps take each
// wait's outcome together (bar.red) before any barrier among them.
#include <math_constants.h>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

namespace {

constexpr int kGTile = 128;                  // keys per tile (MMA M)
#ifndef SA_GATHER_WARPS_PER_SIDE
#define SA_GATHER_WARPS_PER_SIDE 2
#endif
constexpr int kGW = SA_GATHER_WARPS_PER_SIDE;   // gather warps per side (K, V)
constexpr int kGKeys = kGTile / kGW;            // keys of a tile per gather warp
constexpr int kWarpSmx = 2 * kGW;               // first softmax warp
// warp roles: 0..2 kGW - 1 gather (K side first), then eight softmax warps (two
// groups of four, each owning half of the heads), then the S issuer (TMEM
// owner), the index builder, the P V issuer
constexpr int kWarpS = kWarpSmx + 8, kWarpBuild = kWarpS + 1, kWarpPV = kWarpS + 2;
constexpr int kGThreads = (kWarpPV + 1) * 32;
constexpr int kGRing = 6;                    // row-index tiles the builder runs ahead
constexpr int kGMaxK = 2048;                 // top-K entries held in shared memory per query
constexpr int kGInfo = 16;                   // tile records in flight (built .. read by the P V issuer)
constexpr int kGSB = 4;                      // S^T buffers in TMEM
constexpr int kGPB = 3;                      // P^T buffers in shared memory
constexpr size_t kGSmemLimit = 232448;

struct GParams {
    const uint16_t *q, *k, *v;
    const int32_t *topk;
    int K, W, T, S, Hq;
    float scale_log2;
    uint16_t *out;
    float *lse;
    int *dev_status;
};

// Per-tile record passed from the index builder to the gather warps, and from
// the gather warps to the MMA and softmax warps.
struct TileHdr {
    int end;      // 1: no more tiles
    int t;        // query row
    int j;        // the CTA's query counter (buffer parity)
    int i;        // tile index within the query
    int nvalid;   // selected keys in this tile (the rest is padding)
    int last;     // 1: last tile of the query
    int p;        // query position
    int pad;
};

template <int HQP>
struct GCfg {
    static constexpr int kD = 128;
    static constexpr int kHalf = kGTile * 128;                 // one 64-column SW128 half of a K or V tile
    static constexpr int kKV = 2 * kHalf;                      // 128 keys x 256 bytes
    static constexpr int kQHalf = HQP * 128;
    static constexpr int kQ = 2 * kQHalf;                      // HQP rows x 256 bytes
    static constexpr int kP = 2 * kQHalf;                      // HQP heads x 128 keys bf16
    // everything but the K and V rings (barriers counted for 3 + 3 ring slots)
    static constexpr size_t fixed() {
        return 1024 + 2 * (size_t)kQ + kGPB * (size_t)kP + kGRing * (kGTile * 4 + sizeof(TileHdr)) +
               kGInfo * sizeof(TileHdr) + kGMaxK * 4 + 4 * 4 * HQP * 4 + 8 +
               (4 * 3 + 2 * kGRing + 2 * kGInfo + 2 * kGSB + kGPB + 2 * 4) * 8 + 16;
    }
    // K and V tiles live in separate rings: K(g) is released when S(g) is
    // done, V(g) when P V(g) is done
    static constexpr int kNK = fixed() + 6 * (size_t)kKV <= kGSmemLimit ? 3 : 2;
    static constexpr int kNV = kNK;
    static constexpr int kOffK = 0;                                    // [kNK] K tiles
    static constexpr int kOffV = kOffK + kNK * kKV;                    // [kNV] V tiles
    static constexpr int kOffQ = kOffV + kNV * kKV;                    // [2]
    static constexpr int kOffP = kOffQ + 2 * kQ;                       // [kGPB]
    static constexpr int kOffRows = kOffP + kGPB * kP;                 // [kGRing][128] row byte offsets
    static constexpr int kOffRowHdr = kOffRows + kGRing * kGTile * 4;  // [kGRing] TileHdr
    static constexpr int kOffTi = kOffRowHdr + kGRing * (int)sizeof(TileHdr);   // [kGInfo] TileHdr
    static constexpr int kOffList = kOffTi + kGInfo * (int)sizeof(TileHdr);    // [kGMaxK] int32
    static constexpr int kOffRed = kOffList + kGMaxK * 4;              // [4][HQP] max, [4][HQP] sums, [2][2][HQP] m, l
    static constexpr int kOffBar = (kOffRed + 4 * 4 * HQP * 4 + 7) & ~7;
    // k_full/k_empty [kNK], v_full/v_empty [kNV], row_full/row_empty [kGRing],
    // ti_full / ti_empty [kGInfo], s_full / p_full [kGSB], p_empty [kGPB], four
    // pairs (o_full, o_empty, q_empty, drain)
    static constexpr int kNumBar = 2 * kNK + 2 * kNV + 2 * kGRing + 2 * kGInfo + 2 * kGSB + kGPB + 2 * 4;
    static constexpr size_t kSmem = 1024 + (size_t)kOffBar + kNumBar * 8 + 16;
    static constexpr int kCols = (kGSB + 2) * HQP;              // S^T buffers, then O^T [2]
    static constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : (kCols <= 64 ? 64 : (kCols <= 128 ? 128 : 256));
};

// ------------------------------------------------------------------ PTX helpers
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival counts against the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Bounded wait for a phase that parks the thread in mbarrier.try_wait (with a
// suspend-time hint of 20 us) instead of polling: eleven warps wait on
// barriers most of the time here, and polling waits flood the issue slots
// and the pipe that executes the barrier tests.  Gives up like mbar_wait.
__device__ __forceinline__ bool try_wait_parked(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool gwait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (try_wait_parked(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (try_wait_parked(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            *abort = 1;
            return false;
        }
    }
}
// The two MMA-issuing threads poll with plain mbarrier.try_wait (no suspend
// hint): each is one thread, and a parked issuer wakes late and delays the
// hand-off it waits for.
__device__ __forceinline__ bool try_wait_issuer(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool iwait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (try_wait_issuer(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        for (int i = 0; i < 16; ++i) if (try_wait_issuer(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer() - t0 > kWaitLimitNs) { *abort = 1; return false; }
    }
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// Barrier `id` over `n` threads that also returns the OR / AND of a predicate.
__device__ __forceinline__ bool bar_or(int id, int n, bool p) {
    uint32_t r;
    asm volatile(
        "{ .reg .pred a, b; setp.ne.u32 a, %1, 0; bar.red.or.pred b, %2, %3, a; selp.u32 %0, 1, 0, b; }"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool bar_and(int id, int n, bool p) {
    uint32_t r;
    asm volatile(
        "{ .reg .pred a, b; setp.ne.u32 a, %1, 0; bar.red.and.pred b, %2, %3, a; selp.u32 %0, 1, 0, b; }"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void bar_sync_n(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_st_wait_all() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void mma_acc(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t acc) {
    tc_mma_f16(d_tmem, a_desc, b_desc, idesc, acc);
}
// MN-major SW128 operand: 64-element MN chunks `lbo` bytes apart, 8-row K
// groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mn128(uint32_t addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((1024 >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// MN-major operand without swizzle: 8 x 16-byte core matrices (8 K rows of 8
// MN elements, 128 contiguous bytes); K groups of 8 rows `kgroup` bytes apart,
// MN chunks of 8 elements `mnchunk` bytes apart.  (For this layout the
// descriptor's leading offset is the K-group stride and its stride offset the
// MN-chunk stride.)
__device__ __forceinline__ uint64_t desc_mn_plain(uint32_t addr, uint32_t kgroup, uint32_t mnchunk) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((kgroup >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((mnchunk >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;   // layout type 0 (no swizzle) in bits 61-63
    return d;
}

// Byte offset of 16-byte chunk `ch` (0..15) of row `r` in a 128B-swizzled
// tile of 256-byte rows held as two 64-column halves `half` bytes apart.
__device__ __forceinline__ uint32_t sw_off(int r, int ch, int half) {
    return (uint32_t)((ch >> 3) * half + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

template <int HQP>
__global__ void __launch_bounds__(kGThreads, 1) gather_attn_tc_kernel(GParams P) {
    using C = GCfg<HQP>;
    constexpr int NK = C::kNK, NV = C::kNV;
    constexpr int D = C::kD;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int32_t *rows = reinterpret_cast<int32_t *>(sm + C::kOffRows);
    TileHdr *rhdr = reinterpret_cast<TileHdr *>(sm + C::kOffRowHdr);
    TileHdr *ti = reinterpret_cast<TileHdr *>(sm + C::kOffTi);
    int32_t *list = reinterpret_cast<int32_t *>(sm + C::kOffList);
    float *redmax = reinterpret_cast<float *>(sm + C::kOffRed);     // [2 groups][4 warps][HQP / 2]
    float *redsum = redmax + 4 * HQP;                                // [2 groups][4 warps][HQP / 2]
    float *epi_m = redsum + 4 * HQP, *epi_l = epi_m + 2 * HQP;       // [2 queries][HQP]
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + C::kOffBar);
    uint64_t *k_full = bar, *k_empty = k_full + NK, *v_full = k_empty + NK, *v_empty = v_full + NV;
    uint64_t *row_full = v_empty + NV, *row_empty = row_full + kGRing, *ti_full = row_empty + kGRing;
    uint64_t *ti_empty = ti_full + kGInfo;
    uint64_t *s_full = ti_empty + kGInfo, *p_full = s_full + kGSB, *p_empty = p_full + kGSB;
    uint64_t *o_full = p_empty + kGPB, *o_empty = o_full + 2;
    uint64_t *q_empty = o_empty + 2, *drain = q_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + C::kNumBar);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = (int)gridDim.x;
    const int n_mine = P.T > (int)blockIdx.x ? (P.T - 1 - (int)blockIdx.x) / G + 1 : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NK; ++i) {
            mbar_init(&k_full[i], 32 * kGW);   // one cp.async arrival per K-side thread
            mbar_init(&k_empty[i], 1);
        }
        for (int i = 0; i < NV; ++i) {
            mbar_init(&v_full[i], 32 * kGW);   // one cp.async arrival per V-side thread
            mbar_init(&v_empty[i], 1);
        }
        for (int i = 0; i < kGInfo; ++i) {
            mbar_init(&ti_full[i], 1);
            mbar_init(&ti_empty[i], 1);   // the P V issuer has read the record
        }
        for (int i = 0; i < kGRing; ++i) {
            mbar_init(&row_full[i], 1);
            mbar_init(&row_empty[i], 2 * kGW);   // every gather warp has issued the tile
        }
        for (int i = 0; i < kGSB; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 8);
        }
        for (int i = 0; i < kGPB; ++i) mbar_init(&p_empty[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&o_full[i], 1);
            mbar_init(&o_empty[i], 8);
            mbar_init(&q_empty[i], 1);
        }
        mbar_init(&drain[0], 1);
        mbar_init(&drain[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // zero both Q buffers once: rows >= Hq stay zero
    for (int i = threadIdx.x; i < 2 * C::kQ / 16; i += kGThreads)
        reinterpret_cast<uint4 *>(sm + C::kOffQ)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    if (warp == kWarpS) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;   // S[0], S[1] at columns 0, HQP; O[0], O[1] at 2 HQP, 3 HQP

    if (warp == kWarpBuild) {
        // ------------------------------------------------------------ index builder
        int g = 0;
        bool ok = true;
        for (int j = 0; j < n_mine && ok; ++j) {
            const int t = P.T - 1 - ((int)blockIdx.x + j * G);
            const int p = P.S - P.T + t;
            const int lim = p - P.W;   // top-K entries <= lim are kept; the window covers the rest
            const int32_t *trow = P.topk + (int64_t)t * P.K;
            // the row -> shared memory; prefix length and validation
            int first_out = P.K;        // first entry that is not in [0, lim]
            bool bad_idx = false, bad_ord = false;
            auto check = [&](int k, int e) {
                list[k] = e;
                if (e > p) bad_idx = true;
                if (!(e >= 0 && e <= lim)) first_out = min(first_out, k);
            };
            if ((P.K & 3) == 0 && (reinterpret_cast<uintptr_t>(P.topk) & 15u) == 0) {
                // 16-byte loads, the whole batch in flight (every row starts 16-byte aligned)
                for (int base = 0; base < P.K; base += 128 * 16) {
                    int4 e[16];
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        const int k = base + 128 * v + 4 * lane;
                        e[v] = k < P.K ? __ldg(reinterpret_cast<const int4 *>(trow + k)) : make_int4(-1, -1, -1, -1);
                    }
#pragma unroll
                    for (int v = 0; v < 16; ++v) {
                        const int k = base + 128 * v + 4 * lane;
                        if (k < P.K) {
                            check(k, e[v].x); check(k + 1, e[v].y); check(k + 2, e[v].z); check(k + 3, e[v].w);
                        }
                    }
                }
            } else {
                for (int base = 0; base < P.K; base += 32 * 8) {
                    int e[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int k = base + 32 * u + lane;
                        e[u] = k < P.K ? __ldg(trow + k) : -1;
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int k = base + 32 * u + lane;
                        if (k < P.K) check(k, e[u]);
                    }
                }
            }
            first_out = (int)__reduce_min_sync(0xffffffffu, (unsigned)first_out);
            __syncwarp();
            for (int k = lane + 1; k < P.K; k += 32) {
                const int e = list[k];
                if (e >= 0) {
                    const int prev = list[k - 1];
                    if (!(prev >= 0 && prev < e)) bad_ord = true;
                }
            }
            if (__any_sync(0xffffffffu, bad_idx) && lane == 0) report(P.dev_status, SA_DEV_INDEX);
            if (__any_sync(0xffffffffu, bad_ord) && lane == 0) report(P.dev_status, SA_DEV_ORDER);
            const int n_top = first_out;
            const int w0 = max(0, p - P.W + 1);
            const int n_keys = n_top + (p >= 0 ? p - w0 + 1 : 0);
            const int n_tiles = (n_keys + kGTile - 1) / kGTile;
            for (int i = 0; i < n_tiles && ok; ++i, ++g) {
                const int slot = g % kGRing;
                ok = __all_sync(0xffffffffu, gwait(&row_empty[slot], ((uint32_t)(g / kGRing) & 1u) ^ 1u,
                                                       abort_flag));
                if (!ok) break;
                // Byte offsets of the tile's 128 rows, in the order the gather
                // lanes read them: key kk = kGKeys pw + 2 it + sub sits at
                // kGKeys pw + (kGKeys / 2) sub + it.  A slot past the selection
                // repeats the tile's first row: its score is masked to -inf, so
                // its P is exactly 0.
                int32_t *rr = rows + slot * kGTile;
                int first_row = 0;
#pragma unroll
                for (int u = 0; u < kGTile / 32; ++u) {
                    const int kk = i * kGTile + u * 32 + lane;
                    int row = kk < n_top ? list[kk] : (kk < n_keys ? w0 + (kk - n_top) : -1);
                    if (u == 0) first_row = __shfl_sync(0xffffffffu, row, 0);
                    if (row < 0) row = first_row;
                    const int kt = u * 32 + lane;   // key within the tile
                    rr[(kt / kGKeys) * kGKeys + (kt & 1) * (kGKeys / 2) + ((kt % kGKeys) >> 1)] =
                        (int32_t)((uint32_t)row * (uint32_t)(D * 2));
                }
                // the tile's record for the gather warps, and for the MMA and
                // softmax warps (once the P V issuer has read the record of tile
                // g - kGInfo from the slot)
                if (g >= kGInfo)
                    ok = __all_sync(0xffffffffu, gwait(&ti_empty[g % kGInfo], ((uint32_t)(g / kGInfo) & 1u) ^ 1u,
                                                       abort_flag));
                if (!ok) break;
                if (lane == 0) {
                    TileHdr h;
                    h.end = 0; h.t = t; h.j = j; h.i = i;
                    h.nvalid = min(kGTile, n_keys - i * kGTile);
                    h.last = (i == n_tiles - 1); h.p = p; h.pad = 0;
                    rhdr[slot] = h;
                    ti[g % kGInfo] = h;
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&row_full[slot]);
                    mbar_arrive(&ti_full[g % kGInfo]);
                }
            }
            __syncwarp();   // the list is rewritten for the next query
        }
        if (ok) {   // end marker
            const int slot = g % kGRing;
            ok = __all_sync(0xffffffffu, gwait(&row_empty[slot], ((uint32_t)(g / kGRing) & 1u) ^ 1u, abort_flag));
            if (ok && g >= kGInfo)
                ok = __all_sync(0xffffffffu, gwait(&ti_empty[g % kGInfo], ((uint32_t)(g / kGInfo) & 1u) ^ 1u, abort_flag));
            if (ok && lane == 0) {
                TileHdr h = {};
                h.end = 1;
                rhdr[slot] = h;
                ti[g % kGInfo] = h;
                mbar_arrive(&row_full[slot]);
                mbar_arrive(&ti_full[g % kGInfo]);
            }
        }
        __syncwarp();
    } else if (warp < kWarpSmx) {
        // ------------------------------------------------------------ gather
        // The first kGW warps copy K rows (and a query's Q rows with its first
        // tile), the next kGW copy V rows, each side on its own ring: K(g)
        // waits only for S(g - kNK) to finish with its slot, V(g) only for
        // P V(g - kNV).
        const bool kside = warp < kGW;
        const int pw = warp % kGW, ts = pw * 32 + lane;   // thread within the side
        const int sub = lane >> 4, ch = lane & 15;
        const uint8_t *base = reinterpret_cast<const uint8_t *>(kside ? P.k : P.v) + ch * 16;
        bool ok = true;
        for (int g = 0; ok; ++g) {
            const int slot = g % kGRing;
            ok = gwait(&row_full[slot], (uint32_t)(g / kGRing) & 1u, abort_flag);
            if (!ok) break;
            const TileHdr h = rhdr[slot];
            if (!h.end) {
                uint8_t *dst;
                if (kside) {
                    ok = gwait(&k_empty[g % NK], ((uint32_t)(g / NK) & 1u) ^ 1u, abort_flag);
                    if (ok && h.i == 0 && h.j >= 2)   // Q buffer j % 2, once the S products of query j - 2 are done
                        ok = gwait(&q_empty[h.j & 1], ((uint32_t)(h.j >> 1) & 1u) ^ 1u, abort_flag);
                    if (!ok) break;
                    if (h.i == 0) {
                        uint8_t *sq = sm + C::kOffQ + (h.j & 1) * C::kQ;
                        const uint16_t *qrow = P.q + (int64_t)h.t * P.Hq * D;
                        for (int idx = ts; idx < P.Hq * 16; idx += 32 * kGW) {
                            const int r = idx >> 4, c = idx & 15;
                            cp_async16(sq + sw_off(r, c, C::kQHalf), qrow + (int64_t)r * D + c * 8);
                        }
                    }
                    dst = sm + C::kOffK + (g % NK) * C::kKV;
                } else {
                    ok = gwait(&v_empty[g % NV], ((uint32_t)(g / NV) & 1u) ^ 1u, abort_flag);
                    if (!ok) break;
                    dst = sm + C::kOffV + (g % NV) * C::kKV;
                }
                // this warp's kGKeys keys (key kGKeys pw + 2 it + sub for lane
                // half sub): the byte offsets as 16-byte loads, then the copies
                constexpr int NIT = kGKeys / 2;
                const uint4 *rr = reinterpret_cast<const uint4 *>(rows + slot * kGTile + pw * kGKeys + sub * NIT);
                uint32_t ro[NIT];
#pragma unroll
                for (int q = 0; q < NIT / 4; ++q) {
                    const uint4 o = rr[q];
                    ro[4 * q] = o.x; ro[4 * q + 1] = o.y; ro[4 * q + 2] = o.z; ro[4 * q + 3] = o.w;
                }
#pragma unroll
                for (int it = 0; it < NIT; ++it) {
                    const int key = pw * kGKeys + 2 * it + sub;
                    cp_async16(dst + sw_off(key, ch, C::kHalf), base + ro[it]);
                }
            }
            if (kside) {
                if (!h.end) cp_async_arrive_noinc(&k_full[g % NK]);
            } else if (!h.end) {
                cp_async_arrive_noinc(&v_full[g % NV]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&row_empty[slot]);
            if (h.end) break;
        }
        cp_async_wait_all();
    } else if (warp == kWarpS) {
        // ------------------------------------------------------------ S issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, HQP);
            const uint64_t k_d = smem_desc(smem_u32(sm + C::kOffK), 1024, 2);
            const uint64_t q_d = smem_desc(smem_u32(sm + C::kOffQ), 1024, 2);
            for (int g = 0;; ++g) {
                // the tile's record, K(g), and S buffer g % kGSB read by the
                // softmax of tile g - kGSB
                bool ok = iwait(&ti_full[g % kGInfo], (uint32_t)(g / kGInfo) & 1u, abort_flag);
                if (!ok) break;
                const TileHdr h = ti[g % kGInfo];
                if (h.end) break;
                ok = iwait(&k_full[g % NK], (uint32_t)(g / NK) & 1u, abort_flag);
                if (ok && g >= kGSB)   // S buffer g % kGSB, read by the softmax of tile g - kGSB
                    ok = iwait(&p_full[g % kGSB], ((uint32_t)(g / kGSB) & 1u) ^ 1u, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t dt = tmem + (uint32_t)((g % kGSB) * HQP);
                const uint64_t kd = k_d + (uint64_t)(((g % NK) * C::kKV) >> 4);
                const uint64_t qd = q_d + (uint64_t)(((h.j & 1) * C::kQ) >> 4);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ka = (uint64_t)(((kk >> 2) * C::kHalf + (kk & 3) * 32) >> 4);
                    const uint64_t qa = (uint64_t)(((kk >> 2) * C::kQHalf + (kk & 3) * 32) >> 4);
                    mma_acc(dt, kd + ka, qd + qa, idesc_s, kk > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[g % kGSB]);
                tc_commit(&k_empty[g % NK]);
                if (h.last) tc_commit(&q_empty[h.j & 1]);
            }
            tc_commit(&drain[0]);
            volatile int no_abort = 0;
            iwait(&drain[0], 0, &no_abort);
        }
        __syncwarp();
    } else if (warp == kWarpPV) {
        // ------------------------------------------------------------ P V issuer
        if (lane == 0) {
            // A (V^T) and B (P^T) both MN-major
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, HQP) | (1u << 15) | (1u << 16);
            const uint64_t v_d = desc_mn128(smem_u32(sm + C::kOffV), C::kHalf);
            const uint64_t p_d = desc_mn_plain(smem_u32(sm + C::kOffP), HQP * 16, 128);
            for (int g = 0;; ++g) {
                bool ok = iwait(&ti_full[g % kGInfo], (uint32_t)(g / kGInfo) & 1u, abort_flag);
                if (!ok) break;
                const TileHdr h = ti[g % kGInfo];
                if (h.end) break;
                mbar_arrive(&ti_empty[g % kGInfo]);   // every reader of the record is done with it
                // P(g) written, V(g) landed and, for a query's first tile, its O
                // buffer read by the epilogue of query j - 2
                ok = iwait(&p_full[g % kGSB], (uint32_t)(g / kGSB) & 1u, abort_flag) &&
                     iwait(&v_full[g % NV], (uint32_t)(g / NV) & 1u, abort_flag);
                if (ok && h.i == 0 && h.j >= 2)
                    ok = iwait(&o_empty[h.j & 1], ((uint32_t)(h.j >> 1) & 1u) ^ 1u, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t dt = tmem + (uint32_t)((kGSB + (h.j & 1)) * HQP);
                const uint64_t vd = v_d + (uint64_t)(((g % NV) * C::kKV) >> 4);
                const uint64_t pd = p_d + (uint64_t)(((g % kGPB) * C::kP) >> 4);
#pragma unroll
                for (int kk = 0; kk < kGTile / 16; ++kk) {
                    const uint64_t pa = (uint64_t)((kk * 2 * HQP * 16) >> 4);   // 16 keys = two key groups
                    mma_acc(dt, vd + (uint64_t)((kk * 2048) >> 4), pd + pa, idesc_o, (h.i == 0 && kk == 0) ? 0u : 1u);
                }
                tc_commit(&p_empty[g % kGPB]);
                tc_commit(&v_empty[g % NV]);
                if (h.last) tc_commit(&o_full[h.j & 1]);
            }
            tc_commit(&drain[1]);
            volatile int no_abort = 0;
            iwait(&drain[1], 0, &no_abort);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue (eight warps)
        constexpr int HG = HQP / 2;                       // heads of this group
        const int quad = warp & 3, hg = (warp - kWarpSmx) >> 2, h0 = hg * HG;
        const int bar_red = 2 + 2 * hg, bar_x = 3 + 2 * hg;   // this group's named barriers
        const int key = quad * 32 + lane;                 // TMEM lane: key (S^T) or head dim (O^T)
        const uint32_t lane_t = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)h0;
        float *gmax = redmax + hg * 4 * HG, *gsum = redsum + hg * 4 * HG;
        const float sl2 = P.scale_log2;
        float m[HG], l[HG];
#pragma unroll
        for (int h = 0; h < HG; ++h) { m[h] = -CUDART_INF_F; l[h] = 0.f; }
        auto tload = [&](uint32_t col, float (&v)[HG]) {
#pragma unroll
            for (int c = 0; c < HG; c += 8) {
                uint32_t u[8];
                tmem_ld_x8(lane_t + col + (uint32_t)c, u);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e) v[c + e] = __uint_as_float(u[e]);
            }
        };
        // The epilogue of a query (O^T / l -> out, lse) runs kGPB tiles after
        // its last one, when that tile's P V is known to be done (the P buffer
        // wait of the current tile covers it), or earlier at the next query's
        // last tile (one pending query at a time) or at the end.
        int pend_j = -1, pend_t = 0, pend_g = 0;
        auto epilogue = [&]() -> bool {
            if (pend_j < 0) return true;
            const int jb = pend_j & 1;
            if (!bar_and(bar_red, 128, gwait(&o_full[jb], (uint32_t)(pend_j >> 1) & 1u, abort_flag))) return false;
            tc_fence_after();
            float o[HG];
            tload((uint32_t)((kGSB + jb) * HQP), o);
            uint16_t *orow = P.out + (int64_t)pend_t * P.Hq * D;
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) {
                if (h0 + hh < P.Hq) {
                    const float L = epi_l[jb * HQP + h0 + hh];
                    const __nv_bfloat16 ob = __float2bfloat16_rn(o[hh] * (L > 0.f ? 1.f / L : 0.f));
                    orow[(int64_t)(h0 + hh) * D + key] = *reinterpret_cast<const uint16_t *>(&ob);
                }
            }
            if (P.lse && quad == 0 && lane < HG && h0 + lane < P.Hq) {
                const float L = epi_l[jb * HQP + h0 + lane];
                P.lse[(int64_t)pend_t * P.Hq + h0 + lane] =
                    (L > 0.f ? epi_m[jb * HQP + h0 + lane] + __log2f(L) : -CUDART_INF_F) * 0.69314718055994531f;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_empty[jb]);
            pend_j = -1;
            return true;
        };
        bool ok = true;
        for (int g = 0; ok; ++g) {
            const int sb = g % kGSB, pb_i = g % kGPB;
            // the tile's record, its S^T, and P buffer g % kGPB (free once P V of
            // tile g - kGPB is done); the waits are decided together
            bool w = gwait(&ti_full[g % kGInfo], (uint32_t)(g / kGInfo) & 1u, abort_flag);
            TileHdr h = {};
            if (w) {
                h = ti[g % kGInfo];
                if (!h.end) w = gwait(&s_full[sb], (uint32_t)(g / kGSB) & 1u, abort_flag);
                if (!h.end && w && g >= kGPB)
                    w = gwait(&p_empty[pb_i], ((uint32_t)(g / kGPB) & 1u) ^ 1u, abort_flag);
            }
            // One vote per tile decides the common case: nobody stopped (a
            // wait that ran out, or the end marker) and no head needs a new
            // maximum.  (After a failed wait the S^T read below returns
            // whatever TMEM holds; the vote discards it.)
            const bool stop = !w || h.end;
            tc_fence_after();
            float x[HG];
            tload((uint32_t)(sb * HQP), x);
            if (key >= h.nvalid) {   // a lane past the selection (a query's last tile)
#pragma unroll
                for (int hh = 0; hh < HG; ++hh) x[hh] = -CUDART_INF_F;
            }
            // e[h] = log2 of P before rounding: the scaled score less the
            // head's running maximum.  Is any more than 8 (P above 2^8)?
            // (Always decided anew at a query's first tile, where the maximum is set.)
            float e[HG];
            float emax = -CUDART_INF_F;
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) {
                e[hh] = fmaf(x[hh], sl2, -m[hh]);
                emax = fmaxf(emax, e[hh]);
            }
            bool need = h.i == 0 || emax > 8.f;
            if (!bar_or(bar_red, 128, need || stop)) {
                need = false;
            } else if (bar_or(bar_red, 128, stop)) {
                ok = bar_and(bar_red, 128, w);   // every wait succeeded: the end marker for all
                if (ok) ok = epilogue();
                break;
            } else {
                need = true;
            }
            if (need) {
                // exact tile maximum of every head over the 128 key lanes:
                // butterfly within each warp, then across the group's four warps
#pragma unroll
                for (int hh = 0; hh < HG; ++hh) {
                    float v = x[hh] * sl2;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                    if (lane == 0) gmax[quad * HG + hh] = v;
                }
                bar_sync_n(bar_x, 128);
                float f[HG];
                bool resc = false;
#pragma unroll
                for (int hh = 0; hh < HG; ++hh) {
                    const float tm = fmaxf(fmaxf(gmax[hh], gmax[HG + hh]), fmaxf(gmax[2 * HG + hh], gmax[3 * HG + hh]));
                    f[hh] = 1.f;
                    if (h.i == 0) {
                        m[hh] = tm;
                        l[hh] = 0.f;
                    } else if (tm > m[hh] + 8.f) {
                        f[hh] = ex2f(m[hh] - tm);
                        m[hh] = tm;
                        l[hh] *= f[hh];
                        resc = true;
                    }
                }
                if (resc) {
                    // O^T holds the query's earlier tiles: wait for P V of tile g - 1
                    ok = bar_and(bar_red, 128, gwait(&p_empty[(g - 1) % kGPB], (uint32_t)((g - 1) / kGPB) & 1u,
                                                       abort_flag));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t ot = lane_t + (uint32_t)((kGSB + (h.j & 1)) * HQP);
#pragma unroll
                    for (int c = 0; c < HG; c += 8) {
                        uint32_t o[8];
                        tmem_ld_x8(ot + (uint32_t)c, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f[c + e]);
                        tmem_st8(ot + (uint32_t)c, o);
                    }
                    tmem_st_wait_all();
                }
#pragma unroll
                for (int hh = 0; hh < HG; ++hh) e[hh] = fmaf(x[hh], sl2, -m[hh]);
            }
            // P^T as an MN-major operand without swizzle: 16-byte rows of 8
            // heads, the rows of 8 keys 16 bytes apart, the head chunks of a
            // key group 128 bytes apart, key groups HQP * 16 bytes apart; each
            // thread (one key) stores its heads h0 .. as whole 16-byte rows
            uint8_t *pbuf = sm + C::kOffP + pb_i * C::kP + (key >> 3) * (HQP * 16) + (key & 7) * 16;
#pragma unroll
            for (int c = 0; c < HG; c += 8) {
                uint32_t u[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float p0 = ex2f(e[c + 2 * q]);
                    const float p1 = ex2f(e[c + 2 * q + 1]);
                    l[c + 2 * q] += p0;
                    l[c + 2 * q + 1] += p1;
                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);   // p0 in the low half
                    u[q] = *reinterpret_cast<const uint32_t *>(&b2);
                }
                *reinterpret_cast<uint4 *>(pbuf + ((h0 + c) >> 3) * 128) = make_uint4(u[0], u[1], u[2], u[3]);
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[sb]);
            // a pending epilogue, now that this tile is handed over
            if (pend_j >= 0 && (g - pend_g >= kGPB || h.last))
                if (!(ok = epilogue())) break;
            if (h.last) {
                // the query's row sums over all 128 key lanes and its maxima,
                // kept for its epilogue
#pragma unroll
                for (int hh = 0; hh < HG; ++hh) {
                    float v = l[hh];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    if (lane == 0) gsum[quad * HG + hh] = v;
                }
                bar_sync_n(bar_x, 128);
                if (quad == 0 && lane < HG) {
                    const int jb = h.j & 1;
                    epi_l[jb * HQP + h0 + lane] = (gsum[lane] + gsum[HG + lane]) + (gsum[2 * HG + lane] + gsum[3 * HG + lane]);
#pragma unroll
                    for (int hh = 0; hh < HG; ++hh)
                        if (hh == lane) epi_m[jb * HQP + h0 + lane] = m[hh];
                }
                bar_sync_n(bar_x, 128);   // epi_* written before any warp's epilogue reads them
                pend_j = h.j;
                pend_t = h.t;
                pend_g = g;
            }
        }
    }
    // Once every role is past its last TMEM access, the S issuer's warp frees TMEM.
    tc_fence_before();
    bar_sync_n(1, kGThreads);
    if (warp == kWarpS) {
        if (lane == 0 && *abort_flag) report(P.dev_status, SA_DEV_TIMEOUT);
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

template <int HQP>
sa_status launch_gather(const PrefillArgs &a, cudaStream_t st) {
    using C = GCfg<HQP>;
    static_assert(C::kSmem <= kGSmemLimit, "shared memory");
    GParams p;
    p.q = a.q; p.k = a.k; p.v = a.v; p.topk = a.topk;
    p.K = a.K; p.W = a.W; p.T = a.T; p.S = a.S; p.Hq = a.Hq;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.out = a.out; p.lse = a.lse; p.dev_status = a.dev_status;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SA_ERR_CUDA;
    const int grid = a.T < sms ? a.T : sms;
    if (prepare_kernel<gather_attn_tc_kernel<HQP>>(C::kSmem, false) != cudaSuccess) return SA_ERR_CUDA;
    gather_attn_tc_kernel<HQP><<<grid, kGThreads, C::kSmem, st>>>(p);
    return cuda_ok(cudaGetLastError());
}

}  // namespace

// Gathered tensor-core prefill: head dim 128, up to 32 query heads, and top-K
// rows of at most 2048 entries (each query's row is staged in shared memory).
bool prefill_gather_supported(const PrefillArgs &a) { return a.d == 128 && a.Hq >= 1 && a.Hq <= 32 && a.K <= kGMaxK; }

sa_status launch_prefill_gather(const PrefillArgs &a, cudaStream_t st) {
    if (a.T == 0) return SA_OK;
    if (a.Hq <= 16) return launch_gather<16>(a, st);
    return launch_gather<32>(a, st);
}

}  // namespace sa
