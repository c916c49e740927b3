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
//                       K = 128 keys (P^T from shared memory) -> TMEM
// The running maximum of a head is raised only when a tile exceeds it by more
// than 2^8 (then O^T and the row sums are rescaled), so P stays below 256.
//
// Persistent CTAs (one per SM) take queries T-1-c, T-1-c-G, ... (heavy first)
// and stream their tiles through a pipeline of warp roles:
//   warp 9      index builder: copies the query's top-K row to shared memory,
//               validates it (SA_DEV_INDEX / SA_DEV_ORDER), finds the prefix
//               of entries <= p - W and writes the cache rows of each
//               128-key tile (top-K prefix, then the window) into a ring
//   warps 0..3  gather: 16-byte cp.async of every selected K and V row into a
//               128B-swizzled tile (rows past the selection are zero-filled),
//               the query's Q rows with its first tile; completion is tracked
//               by the stage's mbarrier (cp.async.mbarrier.arrive.noinc)
//   warp 8      MMA issuer (one thread) and TMEM owner
//   warps 4..7  softmax of tile g (TMEM lane quadrant = warp % 4), then the
//               epilogue of each query: O^T / l -> out (bf16), lse
// Every wait is bounded (SA_DEV_TIMEOUT), and the softmax warps take each
// wait's outcome together (bar.red) before any barrier among them.
#include <math_constants.h>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

namespace {

constexpr int kGTile = 128;                  // keys per tile (MMA M)
constexpr int kGThreads = 10 * 32;
constexpr int kGRing = 8;                    // row-index tiles the builder runs ahead
constexpr int kGMaxK = 2048;                 // top-K entries held in shared memory per query
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
    static constexpr int kHalf = kGTile * 128;                 // one 64-column SW128 half of a K/V tile
    static constexpr int kKV = 2 * kHalf;                      // 128 keys x 256 bytes
    static constexpr int kStage = 2 * kKV;                     // K + V
    static constexpr int kQHalf = HQP * 128;
    static constexpr int kQ = 2 * kQHalf;                      // HQP rows x 256 bytes
    static constexpr int kP = 2 * kQHalf;                      // HQP heads x 128 keys bf16
    static constexpr size_t fixed() {
        return 1024 + 2 * (size_t)kQ + 2 * (size_t)kP + kGRing * (kGTile * 4 + sizeof(TileHdr)) + kGMaxK * 4 +
               2 * 4 * HQP * 4 + 1024;
    }
    static constexpr int kNS = fixed() + 3 * (size_t)kStage <= kGSmemLimit ? 3 : 2;
    static constexpr int kOffKV = 0;                                   // [kNS] stages
    static constexpr int kOffQ = kOffKV + kNS * kStage;                // [2]
    static constexpr int kOffP = kOffQ + 2 * kQ;                       // [2]
    static constexpr int kOffRows = kOffP + 2 * kP;                    // [kGRing][128] int32
    static constexpr int kOffRowHdr = kOffRows + kGRing * kGTile * 4;  // [kGRing] TileHdr
    static constexpr int kOffTi = kOffRowHdr + kGRing * (int)sizeof(TileHdr);   // [kNS] TileHdr
    static constexpr int kOffList = kOffTi + kNS * (int)sizeof(TileHdr);       // [kGMaxK] int32
    static constexpr int kOffRed = kOffList + kGMaxK * 4;              // [2][4][HQP] f32
    static constexpr int kOffBar = (kOffRed + 2 * 4 * HQP * 4 + 7) & ~7;
    // kv_full/kv_empty [kNS], row_full/row_empty [kGRing], six pairs (s_full,
    // p_full, p_empty, o_full, o_empty, q_empty) and drain
    static constexpr int kNumBar = 2 * kNS + 2 * kGRing + 2 * 6 + 1;
    static constexpr size_t kSmem = 1024 + (size_t)kOffBar + kNumBar * 8 + 16;
    static constexpr uint32_t kTmemCols = 4 * HQP <= 32 ? 32 : (4 * HQP <= 64 ? 64 : (4 * HQP <= 128 ? 128 : 256));
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ void cp_async16_zfill(void *smem_dst, const void *gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
                 "r"(src_bytes)
                 : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival counts against the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ float warp_max(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}
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
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
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

// Byte offset of 16-byte chunk `ch` (0..15) of row `r` in a 128B-swizzled
// tile of 256-byte rows held as two 64-column halves `half` bytes apart.
__device__ __forceinline__ uint32_t sw_off(int r, int ch, int half) {
    return (uint32_t)((ch >> 3) * half + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

template <int HQP>
__global__ void __launch_bounds__(kGThreads, 1) gather_attn_tc_kernel(GParams P) {
    using C = GCfg<HQP>;
    constexpr int NS = C::kNS;
    constexpr int D = C::kD;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int32_t *rows = reinterpret_cast<int32_t *>(sm + C::kOffRows);
    TileHdr *rhdr = reinterpret_cast<TileHdr *>(sm + C::kOffRowHdr);
    TileHdr *ti = reinterpret_cast<TileHdr *>(sm + C::kOffTi);
    int32_t *list = reinterpret_cast<int32_t *>(sm + C::kOffList);
    float *redmax = reinterpret_cast<float *>(sm + C::kOffRed);     // [4][HQP]
    float *redsum = redmax + 4 * HQP;                                // [4][HQP]
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + C::kOffBar);
    uint64_t *kv_full = bar, *kv_empty = bar + NS;
    uint64_t *row_full = bar + 2 * NS, *row_empty = row_full + kGRing;
    uint64_t *s_full = row_empty + kGRing, *p_full = s_full + 2, *p_empty = p_full + 2;
    uint64_t *o_full = p_empty + 2, *o_empty = o_full + 2;
    uint64_t *q_empty = o_empty + 2, *drain = q_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + C::kNumBar);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = (int)gridDim.x;
    const int n_mine = P.T > (int)blockIdx.x ? (P.T - 1 - (int)blockIdx.x) / G + 1 : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&kv_full[i], 128 + 1);   // 128 cp.async arrivals + the header writer
            mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < kGRing; ++i) {
            mbar_init(&row_full[i], 1);
            mbar_init(&row_empty[i], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&p_empty[i], 1);
            mbar_init(&o_full[i], 1);
            mbar_init(&o_empty[i], 4);
            mbar_init(&q_empty[i], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // zero both Q buffers once: rows >= Hq stay zero
    for (int i = threadIdx.x; i < 2 * C::kQ / 16; i += kGThreads)
        reinterpret_cast<uint4 *>(sm + C::kOffQ)[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    if (warp == 8) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;   // S[0], S[1] at columns 0, HQP; O[0], O[1] at 2 HQP, 3 HQP

    if (warp == 9) {
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
                ok = __all_sync(0xffffffffu, mbar_wait(&row_empty[slot], ((uint32_t)(g / kGRing) & 1u) ^ 1u,
                                                       abort_flag));
                if (!ok) break;
                int32_t *rr = rows + slot * kGTile;
#pragma unroll
                for (int u = 0; u < kGTile / 32; ++u) {
                    const int kk = i * kGTile + u * 32 + lane;
                    rr[u * 32 + lane] = kk < n_top ? list[kk] : (kk < n_keys ? w0 + (kk - n_top) : -1);
                }
                if (lane == 0) {
                    TileHdr h;
                    h.end = 0; h.t = t; h.j = j; h.i = i;
                    h.nvalid = min(kGTile, n_keys - i * kGTile);
                    h.last = (i == n_tiles - 1); h.p = p; h.pad = 0;
                    rhdr[slot] = h;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&row_full[slot]);
            }
            __syncwarp();   // the list is rewritten for the next query
        }
        if (ok) {   // end marker
            const int slot = g % kGRing;
            ok = __all_sync(0xffffffffu, mbar_wait(&row_empty[slot], ((uint32_t)(g / kGRing) & 1u) ^ 1u, abort_flag));
            if (ok && lane == 0) {
                TileHdr h = {};
                h.end = 1;
                rhdr[slot] = h;
                mbar_arrive(&row_full[slot]);
            }
        }
        __syncwarp();
    } else if (warp < 4) {
        // ------------------------------------------------------------ gather
        const int tid = threadIdx.x;   // 0..127
        const int sub = lane >> 4, ch = lane & 15;
        bool ok = true;
        for (int g = 0; ok; ++g) {
            const int slot = g % kGRing, s = g % NS;
            ok = mbar_wait(&row_full[slot], (uint32_t)(g / kGRing) & 1u, abort_flag) &&
                 mbar_wait(&kv_empty[s], ((uint32_t)(g / NS) & 1u) ^ 1u, abort_flag);
            if (!ok) break;
            const TileHdr h = rhdr[slot];
            if (h.end) {
                if (tid == 0) ti[s] = h;
                cp_async_arrive_noinc(&kv_full[s]);
                if (tid == 0) mbar_arrive(&kv_full[s]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&row_empty[slot]);
                break;
            }
            uint8_t *sk = sm + C::kOffKV + s * C::kStage, *sv = sk + C::kKV;
            if (h.i == 0) {
                // the query's Q rows into buffer j % 2, once the S products of
                // query j - 2 are done with it
                if (h.j >= 2) {
                    ok = mbar_wait(&q_empty[h.j & 1], ((uint32_t)(h.j >> 1) & 1u) ^ 1u, abort_flag);
                    if (!ok) break;
                }
                uint8_t *sq = sm + C::kOffQ + (h.j & 1) * C::kQ;
                const uint16_t *qrow = P.q + (int64_t)h.t * P.Hq * D;
                for (int idx = tid; idx < P.Hq * 16; idx += 128) {
                    const int r = idx >> 4, c = idx & 15;
                    cp_async16(sq + sw_off(r, c, C::kQHalf), qrow + (int64_t)r * D + c * 8);
                }
            }
            const int32_t *rr = rows + slot * kGTile;
#pragma unroll 4
            for (int it = 0; it < 16; ++it) {
                const int key = warp * 32 + 2 * it + sub;
                const int row = rr[key];
                const uint32_t off = sw_off(key, ch, C::kHalf);
                if (key < h.nvalid && row >= 0) {
                    cp_async16(sk + off, P.k + (int64_t)row * D + ch * 8);
                    cp_async16(sv + off, P.v + (int64_t)row * D + ch * 8);
                } else {
                    cp_async16_zfill(sk + off, P.k, 0u);
                    cp_async16_zfill(sv + off, P.v, 0u);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&row_empty[slot]);
            if (tid == 0) ti[s] = h;
            cp_async_arrive_noinc(&kv_full[s]);
            if (tid == 0) mbar_arrive(&kv_full[s]);
        }
        cp_async_wait_all();
    } else if (warp == 8) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, HQP);
            constexpr uint32_t idesc_o = idesc_bf16_f32(128, HQP) | (1u << 15);   // A (V^T) MN-major
            const uint64_t kv_d = smem_desc(smem_u32(sm + C::kOffKV), 1024, 2);
            const uint64_t v_d = desc_mn128(smem_u32(sm + C::kOffKV + C::kKV), C::kHalf);
            const uint64_t q_d = smem_desc(smem_u32(sm + C::kOffQ), 1024, 2);
            const uint64_t p_d = smem_desc(smem_u32(sm + C::kOffP), 1024, 2);
            int gs = 0, gp = 0, g_end = 0x7fffffff;
            int info_j[2] = {0, 0}, info_first[2] = {0, 0}, info_last[2] = {0, 0};
            bool ok = true;
            unsigned long long t0 = globaltimer();
            while (gp < g_end && ok) {
                bool progressed = false;
                // S(gs) = K(gs) Q^T once the tile landed and S buffer gs % 2 is free
                if (gs < g_end && gs < gp + 2 && mbar_try_wait(&kv_full[gs % NS], (uint32_t)(gs / NS) & 1u)) {
                    const TileHdr h = ti[gs % NS];
                    if (h.end) {
                        g_end = gs;
                    } else {
                        tc_fence_after();
                        const uint32_t dt = tmem + (uint32_t)((gs & 1) * HQP);
                        const uint64_t kd = kv_d + (uint64_t)(((gs % NS) * C::kStage) >> 4);
                        const uint64_t qd = q_d + (uint64_t)(((h.j & 1) * C::kQ) >> 4);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t ka = (uint64_t)(((kk >> 2) * C::kHalf + (kk & 3) * 32) >> 4);
                            const uint64_t qa = (uint64_t)(((kk >> 2) * C::kQHalf + (kk & 3) * 32) >> 4);
                            mma_acc(dt, kd + ka, qd + qa, idesc_s, kk > 0 ? 1u : 0u);
                        }
                        tc_commit(&s_full[gs & 1]);
                        if (h.last) tc_commit(&q_empty[h.j & 1]);
                        info_j[gs & 1] = h.j;
                        info_first[gs & 1] = h.i == 0;
                        info_last[gs & 1] = h.last;
                        ++gs;
                    }
                    progressed = true;
                }
                // O^T += V^T P^T once the softmax wrote P(gp) (and, for a
                // query's first tile, the epilogue of query j - 2 read its O)
                if (gp < gs && mbar_try_wait(&p_full[gp & 1], (uint32_t)(gp >> 1) & 1u)) {
                    const int j = info_j[gp & 1];
                    const bool first = info_first[gp & 1] != 0;
                    if (!first || j < 2 || mbar_try_wait(&o_empty[j & 1], ((uint32_t)(j >> 1) & 1u) ^ 1u)) {
                        tc_fence_after();
                        const uint32_t dt = tmem + (uint32_t)((2 + (j & 1)) * HQP);
                        const uint64_t vd = v_d + (uint64_t)(((gp % NS) * C::kStage) >> 4);
                        const uint64_t pd = p_d + (uint64_t)(((gp & 1) * C::kP) >> 4);
#pragma unroll
                        for (int kk = 0; kk < kGTile / 16; ++kk) {
                            const uint64_t pa = (uint64_t)(((kk >> 2) * C::kQHalf + (kk & 3) * 32) >> 4);
                            mma_acc(dt, vd + (uint64_t)((kk * 2048) >> 4), pd + pa, idesc_o,
                                    (first && kk == 0) ? 0u : 1u);
                        }
                        tc_commit(&p_empty[gp & 1]);
                        tc_commit(&kv_empty[gp % NS]);
                        if (info_last[gp & 1]) tc_commit(&o_full[j & 1]);
                        ++gp;
                        progressed = true;
                    }
                }
                if (progressed) {
                    t0 = globaltimer();
                } else if (*abort_flag || globaltimer() - t0 > kWaitLimitNs) {
                    *abort_flag = 1;
                    ok = false;
                }
            }
            tc_commit(drain);
            volatile int no_abort = 0;
            mbar_wait(drain, 0, &no_abort);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue (warps 4..7)
        const int quad = warp & 3;
        const int key = quad * 32 + lane;                 // TMEM lane: key (S^T) or head dim (O^T)
        const uint32_t lane_t = tmem + ((uint32_t)(quad * 32) << 16);
        const float sl2 = P.scale_log2;
        float m[HQP], l[HQP];
#pragma unroll
        for (int h = 0; h < HQP; ++h) { m[h] = -CUDART_INF_F; l[h] = 0.f; }
        bool ok = true;
        for (int g = 0; ok; ++g) {
            const int s = g % NS, b = g & 1;
            // the tile's record, then its S^T (both waits decided together)
            bool w = mbar_wait(&kv_full[s], (uint32_t)(g / NS) & 1u, abort_flag);
            TileHdr h = {};
            if (w) {
                h = ti[s];
                if (!h.end) w = mbar_wait(&s_full[b], (uint32_t)(g >> 1) & 1u, abort_flag);
            }
            ok = bar_and(2, 128, w);
            if (!ok || h.end) break;
            tc_fence_after();
            float x[HQP];
#pragma unroll
            for (int c = 0; c < HQP; c += 16) {
                uint32_t v[16];
                tmem_ld_x16(lane_t + (uint32_t)(b * HQP + c), v);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 16; ++u) x[c + u] = __uint_as_float(v[u]);
            }
            const bool valid = key < h.nvalid;
#pragma unroll
            for (int hh = 0; hh < HQP; ++hh) x[hh] = valid ? x[hh] * sl2 : -CUDART_INF_F;
            float wmax[HQP];
            bool need = h.i == 0;
#pragma unroll
            for (int hh = 0; hh < HQP; ++hh) {
                wmax[hh] = warp_max(x[hh]);
                need |= wmax[hh] > m[hh] + 8.f;
            }
            if (bar_or(2, 128, need)) {
                // exact tile maximum of every head over the 128 key lanes
                if (lane == 0) {
#pragma unroll
                    for (int hh = 0; hh < HQP; ++hh) redmax[quad * HQP + hh] = wmax[hh];
                }
                bar_sync_n(3, 128);
                float f[HQP];
                bool resc = false;
#pragma unroll
                for (int hh = 0; hh < HQP; ++hh) {
                    const float tm = fmaxf(fmaxf(redmax[hh], redmax[HQP + hh]),
                                           fmaxf(redmax[2 * HQP + hh], redmax[3 * HQP + hh]));
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
                    ok = bar_and(2, 128, mbar_wait(&p_empty[(g - 1) & 1], (uint32_t)((g - 1) >> 1) & 1u, abort_flag));
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t ot = lane_t + (uint32_t)((2 + (h.j & 1)) * HQP);
#pragma unroll
                    for (int c = 0; c < HQP; c += 16) {
                        uint32_t o[16];
                        tmem_ld_x16(ot + (uint32_t)c, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int u = 0; u < 16; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * f[c + u]);
                        tmem_st16(ot + (uint32_t)c, o);
                    }
                    tmem_st_wait_all();
                }
            }
            // P buffer g % 2 is free once P V of tile g - 2 is done
            if (g >= 2) {
                ok = bar_and(2, 128, mbar_wait(&p_empty[b], ((uint32_t)(g >> 1) & 1u) ^ 1u, abort_flag));
                if (!ok) break;
            }
            // P^T (heads x keys, K-major SW128): key = this lane
            uint8_t *pb = sm + C::kOffP + b * C::kP;
            const int khalf = key >> 6, kc = key & 63;
#pragma unroll
            for (int hh = 0; hh < HQP; ++hh) {
                const float pv = ex2f(x[hh] - m[hh]);
                l[hh] += pv;
                const __nv_bfloat16 bv = __float2bfloat16_rn(pv);
                *reinterpret_cast<__nv_bfloat16 *>(pb + khalf * C::kQHalf + hh * 128 +
                                                   ((((kc >> 3) ^ (hh & 7)) << 4) | ((kc & 7) << 1))) = bv;
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[b]);
            if (h.last) {
                // ---- epilogue of query h.t: O^T / l
                ok = bar_and(2, 128, mbar_wait(&o_full[h.j & 1], (uint32_t)(h.j >> 1) & 1u, abort_flag));
                if (!ok) break;
                tc_fence_after();
                float L[HQP];
#pragma unroll
                for (int hh = 0; hh < HQP; ++hh) {
                    float v = l[hh];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    L[hh] = v;
                }
                if (lane == 0) {
#pragma unroll
                    for (int hh = 0; hh < HQP; ++hh) redsum[quad * HQP + hh] = L[hh];
                }
                bar_sync_n(3, 128);
#pragma unroll
                for (int hh = 0; hh < HQP; ++hh)
                    L[hh] = (redsum[hh] + redsum[HQP + hh]) + (redsum[2 * HQP + hh] + redsum[3 * HQP + hh]);
                const uint32_t ot = lane_t + (uint32_t)((2 + (h.j & 1)) * HQP);
                uint16_t *orow = P.out + (int64_t)h.t * P.Hq * D;
#pragma unroll
                for (int c = 0; c < HQP; c += 16) {
                    uint32_t o[16];
                    tmem_ld_x16(ot + (uint32_t)c, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int hh = c + u;
                        if (hh < P.Hq) {
                            const float inv = L[hh] > 0.f ? 1.f / L[hh] : 0.f;
                            const __nv_bfloat16 ob = __float2bfloat16_rn(__uint_as_float(o[u]) * inv);
                            orow[(int64_t)hh * D + key] = *reinterpret_cast<const uint16_t *>(&ob);
                        }
                    }
                }
                if (P.lse && quad == 0) {
#pragma unroll
                    for (int hh = 0; hh < HQP; ++hh)
                        if (lane == hh && hh < P.Hq)
                            P.lse[(int64_t)h.t * P.Hq + hh] =
                                (L[hh] > 0.f ? m[hh] + __log2f(L[hh]) : -CUDART_INF_F) * 0.69314718055994531f;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&o_empty[h.j & 1]);
            }
        }
    }
    // Once every role is past its last TMEM access, warp 8 frees TMEM.
    tc_fence_before();
    bar_sync_n(1, kGThreads);
    if (warp == 8) {
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
