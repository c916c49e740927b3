// attention.cu -- stage 3: exact softmax attention over the selected keys.
//
//   S(t) = {s in TopK(t) : s <= p - W}  U  {max(0, p-W+1) .. p}
//   O[t,h] = sum_{s in S(t)} softmax_s(q[t,h] . k[s] * scale) v[s]
//
// ("A Guide to Sparse Attention in Large Models", section 2: masked
// attention with Mask[i,j] = 1 iff j in S(i); section 4.2: index-based
// implementation computes only on the selected subset.)  All query heads of a
// token share S(t) and the single KV head.
//
// One CTA (4 warps) owns one query (prefill) or one chunk of one sequence's
// selection (decode, split-K).  It walks its key list in chunks of 64: the
// selected K and V rows are gathered with 16-byte cp.async into an XOR-
// swizzled, double-buffered shared-memory tile, then each warp computes
// S = Q K^T and O += P V on the tensor cores with m16n8k16 (M = 16 heads,
// the natural tile when only 16 heads share a gathered row) and a flash-style
// online softmax in fp32 (exp2 domain).  When a CTA has fewer than 4 head
// tiles, its warps split the chunk's keys and merge their softmax states in
// shared memory at the end.  Decode CTAs write normalised partial outputs
// and their log-sum-exp to the workspace; decode_merge_kernel combines them.
#include <math_constants.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

constexpr int kAttnThreads = 128;
constexpr int kChunk = 64;           // keys per pipeline stage
#ifndef SA_ATTN_STAGES
#define SA_ATTN_STAGES 2
#endif
constexpr int kStages = SA_ATTN_STAGES;   // gathered K/V chunks in flight + 1
constexpr int kDecodeSplit = 128;    // keys per CTA on the split-K decode path
constexpr int kMaxDecodeCluster = 16; // CTAs per sequence on the cluster decode path
// kernel modes: one query per CTA; decode split-K through a workspace; decode
// with one thread-block cluster per sequence merging through shared memory
constexpr int kPrefill = 0, kDecodeSplitK = 1, kDecodeCluster = 2;

struct AttnParams {
    const uint16_t *q, *k, *v;
    const int32_t *topk;
    int K, W, Hq;
    float scale_log2;                 // scale * log2(e)
    int T, S;                         // prefill
    const int32_t *page_table;        // decode
    int max_pages, pool_pages, S_max;
    const int32_t *seq_lens;
    int B, n_splits;
    int list_cap;                     // entries of the per-CTA key list in shared memory
    uint16_t *out;
    float *lse;
    float *ws_o, *ws_lse;
    int *dev_status;
};

// byte offset of 16-byte chunk c of row r in a swizzled tile of ROWB-byte rows
template <int ROWB>
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)(r * ROWB + ((c ^ (r & 7)) << 4));
}

template <int D, int HT, int MODE>
__global__ void __launch_bounds__(kAttnThreads) sparse_attn_kernel(AttnParams P) {
    constexpr bool DECODE = MODE != kPrefill;
    constexpr int KSPLIT = 4 / HT;          // warps sharing one head tile
    constexpr int KPW = kChunk / KSPLIT;    // keys per warp per chunk
    constexpr int ROWB = D * 2;
    constexpr int NCH = D / 8;              // 16-byte chunks per row
    constexpr int TILE = kChunk * ROWB;
    constexpr int NT = KPW / 8;             // S n-tiles per warp
    constexpr int DT = D / 8;               // O n-tiles

    extern __shared__ __align__(128) uint8_t sm[];
    uint8_t *sK = sm;                        // [2][64][D]
    uint8_t *sV = sm + kStages * TILE;       // [kStages][64][D]
    uint8_t *sQ = sm + 2 * kStages * TILE;   // [HT*16][D]
    int32_t *s_rows = reinterpret_cast<int32_t *>(sQ + HT * 16 * ROWB);   // [list_cap] cache rows, -1 = none
    __shared__ int s_ntop;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ht = warp / KSPLIT, ks = warp % KSPLIT;

    // ---- which query, which keys
    int b = 0, p, lo, hi;
    const int32_t *trow;
    const uint16_t *qrow;
    if (DECODE) {
        b = blockIdx.y;
        p = P.seq_lens[b] - 1;
        if (p >= P.S_max) {   // longer than the cache can hold
            if (blockIdx.x == 0 && threadIdx.x == 0) report(P.dev_status, SA_DEV_INDEX);
            p = P.S_max - 1;
        }
        trow = P.topk + (int64_t)b * P.K;
        qrow = P.q + (int64_t)b * P.Hq * D;
    } else {
        const int t = P.T - 1 - blockIdx.x;   // heavy (late) queries first
        b = t;
        p = P.S - P.T + t;
        trow = P.topk + (int64_t)t * P.K;
        qrow = P.q + (int64_t)t * P.Hq * D;
    }
    if (tid == 0) s_ntop = 0;
    __syncthreads();
    {
        int cnt = 0;
        bool bad_idx = false, bad_ord = false;
        auto check = [&](int i, int e, int prev) {
            if (e >= 0 && e <= p - P.W) ++cnt;
            if (e > p) bad_idx = true;
            if (e >= 0 && i > 0 && !(prev >= 0 && prev < e)) bad_ord = true;
        };
        if ((P.K & 3) == 0 && (reinterpret_cast<uintptr_t>(P.topk) & 15u) == 0) {
            // 16-byte loads, four per thread in flight at once (one L2 round trip
            // for a 2048-entry row instead of one per entry)
            const int nv = P.K >> 2;
            for (int base = 0; base < nv; base += 4 * kAttnThreads) {
                int4 v[4];
                int pv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int idx = base + u * kAttnThreads + tid;
                    v[u] = idx < nv ? __ldg(reinterpret_cast<const int4 *>(trow) + idx) : make_int4(-1, -1, -1, -1);
                    pv[u] = (idx < nv && idx > 0) ? __ldg(trow + 4 * idx - 1) : -1;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int idx = base + u * kAttnThreads + tid;
                    if (idx < nv) {
                        const int i = 4 * idx;
                        check(i, v[u].x, pv[u]);
                        check(i + 1, v[u].y, v[u].x);
                        check(i + 2, v[u].z, v[u].y);
                        check(i + 3, v[u].w, v[u].z);
                    }
                }
            }
        } else {
            for (int i = tid; i < P.K; i += kAttnThreads) check(i, trow[i], i > 0 ? trow[i - 1] : -1);
        }
        if (bad_idx) report(P.dev_status, SA_DEV_INDEX);
        if (bad_ord) report(P.dev_status, SA_DEV_ORDER);
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        if (lane == 0) atomicAdd(&s_ntop, cnt);
    }
    __syncthreads();
    const int n_top = s_ntop;
    const int w0 = max(0, p - P.W + 1);
    const int n = (p >= 0) ? n_top + (p - w0 + 1) : 0;
    if (MODE == kDecodeCluster) {      // CTA `rank` of the cluster takes an equal slice
        const int G = (int)cluster_size(), per = (n + G - 1) / G;
        lo = (int)cluster_rank() * per;
        hi = min(n, lo + per);
    } else if (MODE == kDecodeSplitK) {
        lo = blockIdx.x * kDecodeSplit;
        hi = min(n, lo + kDecodeSplit);
    } else {
        lo = 0;
        hi = n;
    }
    const int nchunks = hi > lo ? (hi - lo + kChunk - 1) / kChunk : 0;

    // ---- this CTA's key list as cache rows, built once in shared memory
    // (entry i < n_top is a top-K position, the rest is the window)
    const int n_list = hi > lo ? hi - lo : 0;
    // (two entries per thread at a time, their loads -- and then their page
    // lookups -- in flight together)
    for (int j0 = 0; j0 < nchunks * kChunk; j0 += 2 * kAttnThreads) {
        int sv[2];
        bool in[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = j0 + u * kAttnThreads + tid, i = lo + j;
            in[u] = j < nchunks * kChunk && i < hi;
            sv[u] = in[u] ? ((i < n_top) ? __ldg(trow + i) : w0 + (i - n_top)) : -1;
        }
        int pid[2] = {0, 0};
#pragma unroll
        for (int u = 0; u < 2; ++u)
            if (DECODE && P.page_table && in[u] && sv[u] >= 0 && sv[u] <= p)
                pid[u] = __ldg(P.page_table + (int64_t)b * P.max_pages + (sv[u] >> 6));
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = j0 + u * kAttnThreads + tid;
            if (j >= nchunks * kChunk) continue;
            int32_t row = -1;
            if (in[u]) {
                const int s = sv[u];
                if (s < 0 || s > p) {
                    report(P.dev_status, SA_DEV_INDEX);
                } else if (DECODE && P.page_table) {
                    if (pid[u] < 0 || pid[u] >= P.pool_pages) report(P.dev_status, SA_DEV_INDEX);
                    else row = pid[u] * 64 + (s & 63);
                } else {
                    row = DECODE ? b * P.S_max + s : s;
                }
            }
            s_rows[j] = row;
        }
    }
    (void)n_list;
    __syncthreads();

    // ---- gather: NCH consecutive lanes copy one key's row, so a warp
    // instruction reads whole rows (full 32-byte sectors) from L2/HBM
    auto gather = [&](int c, int buf) {
        uint8_t *dk = sK + buf * TILE, *dv = sV + buf * TILE;
#pragma unroll
        for (int it = 0; it < kChunk * NCH / kAttnThreads; ++it) {
            const int g = it * kAttnThreads + tid;
            const int key = g / NCH, ch = g % NCH;
            const int64_t row = s_rows[c * kChunk + key];
            const uint32_t off = swz<ROWB>(key, ch);
            if (row >= 0) {
                cp_async16(dk + off, P.k + row * D + ch * 8);
                cp_async16(dv + off, P.v + row * D + ch * 8);
            } else {
                *reinterpret_cast<uint4 *>(dk + off) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(dv + off) = make_uint4(0, 0, 0, 0);
            }
        }
    };

    // ---- Q tile (rows >= Hq are zero), then the first gathers
    for (int idx = tid; idx < HT * 16 * NCH; idx += kAttnThreads) {
        const int r = idx / NCH, ch = idx % NCH;
        const uint32_t off = swz<ROWB>(r, ch);
        if (r < P.Hq) cp_async16(sQ + off, qrow + (int64_t)r * D + ch * 8);
        else *reinterpret_cast<uint4 *>(sQ + off) = make_uint4(0, 0, 0, 0);
    }
    cp_async_commit();                        // group 0: Q
#pragma unroll
    for (int c = 0; c < kStages - 1; ++c) {   // groups 1 .. kStages-1: the first chunks
        if (c < nchunks) gather(c, c);
        cp_async_commit();
    }

    float acc[DT][4];
#pragma unroll
    for (int j = 0; j < DT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
    uint32_t qf[D / 16][4];

    cp_async_wait<kStages - 1>();             // Q has landed; chunks may still be in flight
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int r = ht * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        ldmatrix_x4(qf[kk], sQ + swz<ROWB>(r, kk * 2 + (lane >> 4)));
    }

    for (int c = 0; c < nchunks; ++c) {
        const int buf = c % kStages;
        if (c + kStages - 1 < nchunks) gather(c + kStages - 1, (c + kStages - 1) % kStages);
        cp_async_commit();
        cp_async_wait<kStages - 1>();
        __syncthreads();

        const uint8_t *tk = sK + buf * TILE, *tv = sV + buf * TILE;
        const int kbase = ks * KPW;
        // S = Q K^T over this warp's KPW keys
        float s[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int ng = 0; ng < NT / 2; ++ng) {
                uint32_t bf[4];
                const int key = kbase + ng * 16 + 8 * (lane >> 4) + (lane & 7);
                ldmatrix_x4(bf, tk + swz<ROWB>(key, kk * 2 + ((lane >> 3) & 1)));
                const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
                mma_bf16_16816(s[2 * ng], qf[kk], b0);
                mma_bf16_16816(s[2 * ng + 1], qf[kk], b1);
            }
        }
        // mask, scale, online softmax (rows g = lane/4 and g + 8)
        float mx0 = -CUDART_INF_F, mx1 = -CUDART_INF_F;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int key = kbase + j * 8 + 2 * (lane & 3);
            const bool v0 = s_rows[c * kChunk + key] >= 0, v1 = s_rows[c * kChunk + key + 1] >= 0;
            s[j][0] = v0 ? s[j][0] * P.scale_log2 : -CUDART_INF_F;
            s[j][1] = v1 ? s[j][1] * P.scale_log2 : -CUDART_INF_F;
            s[j][2] = v0 ? s[j][2] * P.scale_log2 : -CUDART_INF_F;
            s[j][3] = v1 ? s[j][3] * P.scale_log2 : -CUDART_INF_F;
            mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
            mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float base0 = (mn0 == -CUDART_INF_F) ? 0.f : mn0;
        const float base1 = (mn1 == -CUDART_INF_F) ? 0.f : mn1;
        const float corr0 = exp2f(m0 - base0), corr1 = exp2f(m1 - base1);
        m0 = mn0;
        m1 = mn1;
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            s[j][0] = exp2f(s[j][0] - base0);
            s[j][1] = exp2f(s[j][1] - base0);
            s[j][2] = exp2f(s[j][2] - base1);
            s[j][3] = exp2f(s[j][3] - base1);
            rs0 += s[j][0] + s[j][1];
            rs1 += s[j][2] + s[j][3];
        }
        l0 = l0 * corr0 + rs0;
        l1 = l1 * corr1 + rs1;
#pragma unroll
        for (int j = 0; j < DT; ++j) {
            acc[j][0] *= corr0; acc[j][1] *= corr0;
            acc[j][2] *= corr1; acc[j][3] *= corr1;
        }
        // O += P V
#pragma unroll
        for (int kk = 0; kk < KPW / 16; ++kk) {
            const uint32_t a[4] = {pack_bf16(s[2 * kk][0], s[2 * kk][1]), pack_bf16(s[2 * kk][2], s[2 * kk][3]),
                                   pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]),
                                   pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3])};
            const int key = kbase + kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
            for (int dn = 0; dn < DT / 2; ++dn) {
                uint32_t bf[4];
                ldmatrix_x4_trans(bf, tv + swz<ROWB>(key, dn * 2 + (lane >> 4)));
                const uint32_t b0[2] = {bf[0], bf[1]}, b1[2] = {bf[2], bf[3]};
                mma_bf16_16816(acc[2 * dn], a, b0);
                mma_bf16_16816(acc[2 * dn + 1], a, b1);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

    // ---- final softmax state of each head row (quad-reduce the row sums)
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    __syncthreads();   // every warp is done with the K/V tiles, which are reused below
    // cluster path: this CTA's normalised partial output and log2-sum-exp,
    // kept in shared memory (after the reduction area) for the other CTAs
    float *part_o = reinterpret_cast<float *>(sm + 4 * 16 * D * 4 + 4 * 4 * 16 * 4);   // [HT*16][D]
    float *part_lse = part_o + HT * 16 * D;                                             // [HT*16]
    // write row h's normalised output at dims (col, col+1) and, once, its lse
    auto emit2 = [&](int h, int col, float o0, float o1, bool with_lse, float lse2) {
        if (h >= P.Hq) return;
        if (MODE == kDecodeCluster) {
            *reinterpret_cast<float2 *>(&part_o[h * D + col]) = make_float2(o0, o1);
            if (with_lse) part_lse[h] = lse2;
        } else if (MODE == kDecodeSplitK) {
            const int64_t slot = ((int64_t)b * P.n_splits + blockIdx.x) * P.Hq + h;
            *reinterpret_cast<float2 *>(&P.ws_o[slot * D + col]) = make_float2(o0, o1);
            if (with_lse) P.ws_lse[slot] = lse2;
        } else {
            const int64_t orow = (int64_t)b * P.Hq + h;
            *reinterpret_cast<uint32_t *>(&P.out[orow * D + col]) = pack_bf16(o0, o1);
            if (with_lse && P.lse) P.lse[orow] = lse2 * 0.69314718055994531f;
        }
    };
    if (KSPLIT == 1) {
        // this warp alone holds its 16 heads: normalise in registers
        const int g = lane >> 2;
        const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
        const float lse0 = l0 > 0.f ? m0 + __log2f(l0) : -CUDART_INF_F;
        const float lse1 = l1 > 0.f ? m1 + __log2f(l1) : -CUDART_INF_F;
#pragma unroll
        for (int j = 0; j < DT; ++j) {
            const int col = j * 8 + 2 * (lane & 3);
            emit2(ht * 16 + g, col, acc[j][0] * inv0, acc[j][1] * inv0, j == 0 && (lane & 3) == 0, lse0);
            emit2(ht * 16 + g + 8, col, acc[j][2] * inv1, acc[j][3] * inv1, j == 0 && (lane & 3) == 0, lse1);
        }
    } else {
        // KSPLIT warps hold partial states of the same heads: combine them in
        // shared memory with per-row weights computed once
        float *red_acc = reinterpret_cast<float *>(sm);   // [4 warps][16][D]
        float *red_m = red_acc + 4 * 16 * D;               // [4][16]
        float *red_l = red_m + 4 * 16;                     // [4][16]
        float *row_w = red_l + 4 * 16;                     // [HT*16][KSPLIT] merge weights / L
        float *row_lse = row_w + 4 * 16;                   // [HT*16]
        const int g = lane >> 2;
        float *ra = red_acc + warp * 16 * D;
#pragma unroll
        for (int j = 0; j < DT; ++j) {
            const int col = j * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2 *>(&ra[g * D + col]) = make_float2(acc[j][0], acc[j][1]);
            *reinterpret_cast<float2 *>(&ra[(g + 8) * D + col]) = make_float2(acc[j][2], acc[j][3]);
        }
        if ((lane & 3) == 0) {
            red_m[warp * 16 + g] = m0; red_m[warp * 16 + g + 8] = m1;
            red_l[warp * 16 + g] = l0; red_l[warp * 16 + g + 8] = l1;
        }
        __syncthreads();
        if (tid < HT * 16) {
            const int rt = tid >> 4, rr = tid & 15;
            float mstar = -CUDART_INF_F;
#pragma unroll
            for (int k2 = 0; k2 < KSPLIT; ++k2) mstar = fmaxf(mstar, red_m[(rt * KSPLIT + k2) * 16 + rr]);
            const float mb = (mstar == -CUDART_INF_F) ? 0.f : mstar;
            float f[KSPLIT], L = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < KSPLIT; ++k2) {
                f[k2] = exp2f(red_m[(rt * KSPLIT + k2) * 16 + rr] - mb);
                L += red_l[(rt * KSPLIT + k2) * 16 + rr] * f[k2];
            }
            const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
            for (int k2 = 0; k2 < KSPLIT; ++k2) row_w[tid * KSPLIT + k2] = f[k2] * inv;
            row_lse[tid] = L > 0.f ? mb + __log2f(L) : -CUDART_INF_F;
        }
        __syncthreads();
        for (int idx = tid; idx < HT * 16 * D / 2; idx += kAttnThreads) {
            const int r = idx / (D / 2), col = 2 * (idx % (D / 2));
            const int rt = r >> 4, rr = r & 15;
            float o0 = 0.f, o1 = 0.f;
#pragma unroll
            for (int k2 = 0; k2 < KSPLIT; ++k2) {
                const float wgt = row_w[r * KSPLIT + k2];
                const float2 v = *reinterpret_cast<const float2 *>(&red_acc[((rt * KSPLIT + k2) * 16 + rr) * D + col]);
                o0 = fmaf(wgt, v.x, o0);
                o1 = fmaf(wgt, v.y, o1);
            }
            emit2(r, col, o0, o1, col == 0, row_lse[r]);
        }
    }
    if (MODE == kDecodeCluster) {
        // merge the G partial states of this sequence through distributed
        // shared memory: CTA `rank` produces heads [rank*hpr, rank*hpr + hpr).
        // The G log-sum-exps of those heads are staged locally first; the
        // partial outputs are then read with all G loads in flight.
        __shared__ float s_wt[kMaxDecodeCluster * 8];   // [hpr <= 8][G] weights
        __shared__ float s_inv[8], s_lse[8];
        cluster_sync();
        const int G = (int)cluster_size(), rank = (int)cluster_rank();
        const int hpr = (P.Hq + G - 1) / G;
        if (tid < hpr * G) {
            const int hh = tid / G, c = tid % G, h = rank * hpr + hh;
            s_wt[hh * kMaxDecodeCluster + c] =
                h < P.Hq ? __uint_as_float(dsmem_ld_u32(&part_lse[h], (uint32_t)c)) : -CUDART_INF_F;
        }
        __syncthreads();
        if (tid < hpr) {
            float M = -CUDART_INF_F;
            for (int c = 0; c < G; ++c) M = fmaxf(M, s_wt[tid * kMaxDecodeCluster + c]);
            const float mb = (M == -CUDART_INF_F) ? 0.f : M;
            float L = 0.f;
            for (int c = 0; c < G; ++c) {
                const float f = exp2f(s_wt[tid * kMaxDecodeCluster + c] - mb);
                s_wt[tid * kMaxDecodeCluster + c] = f;
                L += f;
            }
            s_inv[tid] = L > 0.f ? 1.f / L : 0.f;
            s_lse[tid] = L > 0.f ? mb + __log2f(L) : -CUDART_INF_F;
        }
        __syncthreads();
        for (int idx = tid; idx < hpr * D; idx += kAttnThreads) {
            const int hh = idx / D, h = rank * hpr + hh, dim = idx % D;
            if (h >= P.Hq) continue;
            float v[kMaxDecodeCluster];
#pragma unroll
            for (int c = 0; c < kMaxDecodeCluster; ++c)
                v[c] = c < G ? __uint_as_float(dsmem_ld_u32(&part_o[h * D + dim], (uint32_t)c)) : 0.f;
            float o = 0.f;
#pragma unroll
            for (int c = 0; c < kMaxDecodeCluster; ++c)
                if (c < G) o += s_wt[hh * kMaxDecodeCluster + c] * v[c];
            const int64_t orow = (int64_t)b * P.Hq + h;
            const __nv_bfloat16 ob = __float2bfloat16_rn(o * s_inv[hh]);
            P.out[orow * D + dim] = *reinterpret_cast<const uint16_t *>(&ob);
            if (dim == 0 && P.lse) P.lse[orow] = s_lse[hh] * 0.69314718055994531f;
        }
        cluster_sync();   // the other CTAs may still read this CTA's partials
    }
}

// Combine the decode splits of (sequence b, head h): O = sum_i O_i 2^(lse_i - M) / sum_i 2^(lse_i - M).
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(AttnParams P) {
    const int b = blockIdx.x, h = blockIdx.y, dim = threadIdx.x;
    const int64_t base = (int64_t)b * P.n_splits * P.Hq + h;
    float M = -CUDART_INF_F;
    for (int i = 0; i < P.n_splits; ++i) M = fmaxf(M, P.ws_lse[base + (int64_t)i * P.Hq]);
    const float mb = (M == -CUDART_INF_F) ? 0.f : M;
    float L = 0.f, o = 0.f;
    for (int i = 0; i < P.n_splits; ++i) {
        const int64_t slot = base + (int64_t)i * P.Hq;
        const float f = exp2f(P.ws_lse[slot] - mb);
        L += f;
        o += f * P.ws_o[slot * D + dim];
    }
    const float res = L > 0.f ? o / L : 0.f;
    const __nv_bfloat16 ob = __float2bfloat16_rn(res);
    P.out[((int64_t)b * P.Hq + h) * D + dim] = *reinterpret_cast<const uint16_t *>(&ob);
    if (dim == 0 && P.lse) P.lse[(int64_t)b * P.Hq + h] = (L > 0.f ? mb + __log2f(L) : -CUDART_INF_F) * 0.69314718055994531f;
}

template <int D, int HT, int MODE>
static sa_status launch_attn(const AttnParams &p, dim3 grid, int cluster, cudaStream_t st) {
    constexpr int TILE = kChunk * D * 2;
    size_t smem = 2 * kStages * TILE + HT * 16 * D * 2 + (size_t)p.list_cap * 4;
    if (MODE == kDecodeCluster) {   // the partials live after the reduction area
        const size_t need = 4 * 16 * D * 4 + 4 * 4 * 16 * 4 + (size_t)HT * 16 * (D + 1) * 4;
        smem = smem > need ? smem : need;
    }
    auto kern = sparse_attn_kernel<D, HT, MODE>;
    if (prepare_kernel<sparse_attn_kernel<D, HT, MODE>>(smem, cluster > 8) != cudaSuccess) return SA_ERR_CUDA;
    if (cluster <= 1) {
        kern<<<grid, kAttnThreads, smem, st>>>(p);
        return cuda_ok(cudaGetLastError());
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_ok(cudaLaunchKernelEx(&cfg, kern, p));
}

template <int MODE>
static sa_status launch_attn_shape(const AttnParams &p, int d, dim3 grid, int cluster, cudaStream_t st) {
    const int ht = (p.Hq + 15) / 16;
    if (d == 128) {
        if (ht == 1) return launch_attn<128, 1, MODE>(p, grid, cluster, st);
        if (ht == 2) return launch_attn<128, 2, MODE>(p, grid, cluster, st);
        if (ht <= 4) return launch_attn<128, 4, MODE>(p, grid, cluster, st);
    } else if (d == 64) {
        if (ht == 1) return launch_attn<64, 1, MODE>(p, grid, cluster, st);
        if (ht == 2) return launch_attn<64, 2, MODE>(p, grid, cluster, st);
        if (ht <= 4) return launch_attn<64, 4, MODE>(p, grid, cluster, st);
    }
    return SA_ERR_UNSUPPORTED;
}

static AttnParams base_params(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *topk, int K,
                              int W, int Hq, int d, float scale, uint16_t *out, float *lse, int *dev_status) {
    AttnParams p = {};
    p.q = q; p.k = k; p.v = v; p.topk = topk; p.K = K; p.W = W; p.Hq = Hq;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.out = out; p.lse = lse; p.dev_status = dev_status;
    return p;
}

sa_status launch_prefill(const PrefillArgs &a, cudaStream_t st) {
    if (a.T == 0) return SA_OK;
    // Dense selections (each query keeps a large share of its causal keys):
    // stream contiguous K/V tiles once per group of queries through masked
    // tensor-core tiles instead of gathering every query's rows.
    if (a.workspace && prefill_tc_supported(a) && a.workspace_bytes >= prefill_tc_workspace_bytes(a.T, a.S)) {
        const sa_status s = launch_prefill_tc(a, st);
        if (s != SA_ERR_UNSUPPORTED) return s;   // else the gathered path below
    }
    // Sparse selections: gather each query's rows onto tcgen05 tiles
    if (prefill_gather_supported(a)) return launch_prefill_gather(a, st);
    AttnParams p = base_params(a.q, a.k, a.v, a.topk, a.K, a.W, a.Hq, a.d, a.scale, a.out, a.lse, a.dev_status);
    p.T = a.T;
    p.S = a.S;
    p.list_cap = (a.K + a.W + kChunk - 1) / kChunk * kChunk;
    return launch_attn_shape<kPrefill>(p, a.d, dim3((unsigned)a.T), 1, st);
}

static int decode_splits(int K, int W) { return (K + W + kDecodeSplit - 1) / kDecodeSplit; }

size_t decode_workspace_bytes(int B, int Hq, int d, int K, int W) {
    const size_t slots = (size_t)B * decode_splits(K, W) * Hq;
    const size_t o_bytes = ((slots * d * 4) + 255) & ~size_t(255);
    return o_bytes + ((slots * 4 + 255) & ~size_t(255));
}

sa_status launch_decode(const DecodeArgs &a, cudaStream_t st) {
    if (a.B == 0) return SA_OK;
    AttnParams p = base_params(a.q, a.k, a.v, a.topk, a.K, a.W, a.Hq, a.d, a.scale, a.out, a.lse, a.dev_status);
    p.page_table = a.page_table; p.max_pages = a.max_pages; p.pool_pages = a.pool_pages; p.S_max = a.S_max;
    p.seq_lens = a.seq_lens; p.B = a.B;
    // Fast path: one cluster of G CTAs per sequence, each taking about
    // (K + W) / G keys, merged through distributed shared memory.
    // (at least ceil(Hq / 8) CTAs: the merge gives each CTA at most 8 heads)
    const int G = std::min(kMaxDecodeCluster, std::max({1, (a.K + a.W + kDecodeSplit - 1) / kDecodeSplit,
                                                        (a.Hq + 7) / 8}));
    const int per_cta = (a.K + a.W + G - 1) / G;
    if (!a.force_split_k && per_cta <= 1024) {
        p.list_cap = (per_cta + kChunk - 1) / kChunk * kChunk;
        return launch_attn_shape<kDecodeCluster>(p, a.d, dim3((unsigned)G, (unsigned)a.B), G, st);
    }
    p.n_splits = decode_splits(a.K, a.W);
    p.list_cap = kDecodeSplit;
    const size_t slots = (size_t)a.B * p.n_splits * a.Hq;
    p.ws_o = reinterpret_cast<float *>(a.workspace);
    p.ws_lse = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(a.workspace) +
                                         (((slots * a.d * 4) + 255) & ~size_t(255)));
    sa_status s = launch_attn_shape<kDecodeSplitK>(p, a.d, dim3((unsigned)p.n_splits, (unsigned)a.B), 1, st);
    if (s != SA_OK) return s;
    const dim3 mg((unsigned)a.B, (unsigned)a.Hq);
    if (a.d == 128) decode_merge_kernel<128><<<mg, 128, 0, st>>>(p);
    else decode_merge_kernel<64><<<mg, 64, 0, st>>>(p);
    return cuda_ok(cudaGetLastError());
}

}  // namespace sa
