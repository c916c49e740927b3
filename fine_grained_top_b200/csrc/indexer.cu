// indexer.cu -- stage 1: lightweight-indexer scores on the 5th-generation
// tensor cores.
//
//   I[t,s] = sum_j w[t,j] * ReLU(qI[t,j] . kI[s])
//
// ("Sparse Attention for Long-Context LLM Inference", section "Where Sparse
// Attention Is Actually Sparse": a lightweight indexer scores history
// positions and outputs candidate indices, without positional encoding;
// "Sparse Attention in 2026", "The designs that shipped": the lightning
// indexer is a small few-head low-precision scorer.)
//
// Tile mapping: keys on M, (query, head) pairs on N.  qI is stored
// [rows, H_I, D_I], so QT consecutive queries x H_I heads are QT*H_I
// consecutive rows of D_I elements: one K-major B operand.  One tile:
//     D[s, (t,j)] = kI[s] . qI[t,j]        M = 128 keys, N = 256 (or 16),
// accumulated in fp32 in TMEM.  The epilogue thread owning TMEM lane s reads
// the H_I adjacent columns of query t, applies ReLU and the weights w[t,:],
// and writes scores[t, s]; a warp writes 32 consecutive floats per query.
//
// The operands are bf16 (tcgen05.mma kind::f16) or e4m3 bytes (kind::f8f6f4,
// "Sparse Attention in 2026", "The designs that shipped": the shipped
// indexer runs in FP8).  Either way the tile machinery only sees rows of RB
// bytes (RB = 2*D_I or D_I) and K-steps of 32 bytes (16 bf16 or 32 e4m3).
//
// Warp roles (persistent CTAs, one per SM):
//   warp 0     TMA producer (one elected lane) + TMEM allocator
//   warp 1     MMA issuer (one elected lane)
//   warps 2..  epilogue teams: for the 256-column prefill tile, 2 item groups
//              (alternate items, one TMEM accumulator each) x 2 column groups;
//              for the 16-column decode tile, 4 item groups x 8 accumulators
//              (several items drain at once)
// All roles classify the CTA's items 32 at a time (one item per lane) and
// walk the same sequence of non-empty items; the producer resolves the page
// ids of 32 items in parallel, off the TMA issue path.
// Shared-memory ring of STAGES {A = 128 keys, B = N query-head rows} tiles,
// filled by TMA with the 128B (RB = 128) or 64B (RB = 64) swizzle that the
// UMMA K-major descriptors expect.
#include <cudaTypedefs.h>

#include "internal.h"
#include "ptx.cuh"

namespace sa {

struct IdxKernelArgs {
    const uint16_t *w;
    const int32_t *page_table;
    const int32_t *n_valid;
    float *scores;
    int64_t ld;
    int *dev_status;
    int max_pages, pool_pages;
    int B, T, S;
    int QT, QTN, KT;   // queries per tile, query tiles per batch, key tiles per batch
    int n_items;
};

// RB: bytes per qI / kI row (64 or 128).  PAIR: 64-byte e4m3 keys are loaded
// two to a 128-byte row (the TMA engine's cost is per row, not per byte), so
// an item covers 256 keys: A row r holds keys 2r and 2r+1 in its two halves.
template <int N, int RB, bool PAIR = false>
struct IdxCfg {
    static_assert(!PAIR || (RB == 64 && N == 16), "paired rows serve the 64-byte decode tile");
    static constexpr int kKeys = PAIR ? 256 : 128;            // keys per item
    static constexpr int kKeysPerRow = PAIR ? 2 : 1;
    static constexpr int kARowBytes = RB * kKeysPerRow;       // 128 rows of A per item
    static constexpr int kBoxRows = 64 / kKeysPerRow;         // one TMA box = 64 keys (one cache page)
    static constexpr int kBoxes = kKeys / 64;
    static constexpr int kABytes = 128 * kARowBytes;
    static constexpr int kBoxBytes = kABytes / kBoxes;
    static constexpr int kBBytes = N * RB;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kStages = (N == 256) ? 4 : 8;
    // Epilogue teams: CG column groups split one item's queries; IG item
    // groups take alternate items so that several accumulators drain at once.
    static constexpr int kCG = (N == 256) ? 2 : 1;
    static constexpr int kIG = (N == 256) ? 2 : 4;
    static constexpr int kAcc = (N == 256) ? 2 : 8;           // TMEM accumulators (multiple of kIG)
    static constexpr int kAccCols = N * kKeysPerRow;           // PAIR: even keys, then odd keys
    static constexpr int kEpiWarps = 4 * kCG * kIG;
    static constexpr int kThreads = (2 + kEpiWarps) * 32;
    static constexpr int kCols = kAcc * kAccCols;
    static constexpr uint32_t kTmemCols = (kCols <= 32) ? 32 : (kCols <= 64) ? 64 : (kCols <= 128) ? 128
                                        : (kCols <= 256) ? 256 : 512;
    // UMMA K-major operands: 8-row core group stride and layout (2 = 128B,
    // 4 = 64B swizzle), for A (keys) and B (query-head rows)
    static constexpr uint32_t kSboA = 8 * kARowBytes, kLayoutA = (kARowBytes == 128) ? 2 : 4;
    static constexpr uint32_t kSboB = 8 * RB, kLayoutB = (RB == 128) ? 2 : 4;
    static constexpr int kGroupCols = N / kCG;                 // TMEM columns per epilogue warp
    static constexpr size_t kWStage = (size_t)kEpiWarps * kGroupCols * 8;   // w (fp32) + n_valid per warp
    static constexpr size_t kSmemUsed = 1024 + (size_t)kStages * kStageBytes + 1024 + kWStage;
    // at least 116 KB so that exactly one persistent CTA (and one TMEM
    // allocation) lands on each SM
    static constexpr size_t kSmem = kSmemUsed > 118784 ? kSmemUsed : 118784;
    static_assert(kAcc % kIG == 0, "item groups must own whole accumulators");
};

// One work item: query tile qt of batch b against key tile kt (kKeys keys).
struct ItemInfo {
    int b, qt, kt, ext;   // ext: the tile's key extent (largest n_valid of its queries)
};

// Work of the CTA's item `i` (rectangle item blockIdx.x + i * gridDim.x),
// evaluated by one lane.  Every role classifies items the same way, 32 at a
// time, so all roles walk the same sequence of non-empty items.
__device__ __forceinline__ bool item_at(const IdxKernelArgs &a, int i, ItemInfo &it) {
    const long long item = (long long)blockIdx.x + (long long)i * gridDim.x;
    if (item >= a.n_items) return false;
    const int per_b = a.QTN * a.KT;
    it.b = (int)(item / per_b);
    const int rem = (int)(item - (long long)it.b * per_b);
    it.qt = rem / a.KT;
    it.kt = rem - it.qt * a.KT;
    const int t0 = it.qt * a.QT, t1 = min(t0 + a.QT, a.T);
    int ext;
    if (a.n_valid == nullptr) {
        ext = a.S - a.T + t1;   // causal: the tile's last query
    } else {
        ext = 0;
        for (int t = t0; t < t1; ++t) ext = max(ext, __ldg(a.n_valid + (int64_t)it.b * a.T + t));
        ext = min(ext, a.S);
    }
    it.ext = ext;
    return true;
}

template <int N, int RB, int H_I, bool F8, bool PAIR>
__global__ void __launch_bounds__(IdxCfg<N, RB, PAIR>::kThreads, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                      IdxKernelArgs a) {
    using C = IdxCfg<N, RB, PAIR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stage_base = smem;
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + C::kStages * C::kStageBytes);
    uint64_t *empty_bar = full_bar + C::kStages;
    uint64_t *tfull_bar = empty_bar + C::kStages;   // [kAcc]
    uint64_t *tempty_bar = tfull_bar + C::kAcc;     // [kAcc]
    uint64_t *drain_bar = tempty_bar + C::kAcc;     // [1]
    uint32_t *tmem_base_slot = reinterpret_cast<uint32_t *>(drain_bar + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_slot + 1);
    float *w_stage = reinterpret_cast<float *>(smem + C::kStages * C::kStageBytes + 1024);
    int *nv_stage = reinterpret_cast<int *>(w_stage + C::kEpiWarps * C::kGroupCols);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
        for (int i = 0; i < C::kAcc; ++i) { mbar_init(&tfull_bar[i], 1); mbar_init(&tempty_bar[i], 4 * C::kCG); }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&map_k);
        tma_prefetch_desc(&map_q);
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        for (int base = 0; ok; base += 32) {
            ItemInfo it;
            const bool in = item_at(a, base + lane, it);
            const bool valid = in && it.kt * C::kKeys < it.ext;
            // the 64-key boxes of this lane's item: rows of the key map, or -1 (skip)
            int rows[C::kBoxes];
#pragma unroll
            for (int i = 0; i < C::kBoxes; ++i) {
                const int s0 = it.kt * C::kKeys + i * 64;
                int row = -1;
                if (valid && s0 < it.ext) {
                    if (a.page_table) {
                        const int pid = __ldg(a.page_table + (int64_t)it.b * a.max_pages + (s0 >> 6));
                        if (pid < 0 || pid >= a.pool_pages) report(a.dev_status, SA_DEV_INDEX);
                        else row = pid * C::kBoxRows;
                    } else {
                        row = (it.b * a.S + s0) / C::kKeysPerRow;   // even for PAIR (S even)
                    }
                }
                rows[i] = row;
            }
            if (__ballot_sync(0xffffffffu, in) == 0) break;
            uint32_t vmask = __ballot_sync(0xffffffffu, valid);
            while (vmask) {
                const int j = __ffs(vmask) - 1;
                vmask &= vmask - 1;
                const int qrow = __shfl_sync(0xffffffffu, (it.b * a.T + it.qt * a.QT) * H_I, j);
                int r[C::kBoxes];
                uint32_t nbox = 0;
#pragma unroll
                for (int i = 0; i < C::kBoxes; ++i) {
                    r[i] = __shfl_sync(0xffffffffu, rows[i], j);
                    nbox += r[i] >= 0;
                }
                if (lane == 0) {
                    ok = mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag);
                    if (ok) {
                        uint8_t *sa_ = stage_base + stage * C::kStageBytes;
                        mbar_arrive_expect_tx(&full_bar[stage], C::kBBytes + nbox * C::kBoxBytes);
                        tma_load_2d(sa_ + C::kABytes, &map_q, 0, qrow, &full_bar[stage]);
#pragma unroll
                        for (int i = 0; i < C::kBoxes; ++i)
                            if (r[i] >= 0) tma_load_2d(sa_ + i * C::kBoxBytes, &map_k, 0, r[i], &full_bar[stage]);
                        ++issued;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
            }
        }
        // drain: wait (bounded) for this CTA's last loads to land before teardown
        if (lane == 0 && *abort_flag) {
            int s = stage;
            uint32_t p = phase;
            for (int i = 0; i < min(issued, C::kStages); ++i) {
                if (--s < 0) { s = C::kStages - 1; p ^= 1u; }
                volatile int no_abort = 0;
                mbar_wait(&full_bar[s], p, &no_abort);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = F8 ? idesc_e4m3_f32(128, N) : idesc_bf16_f32(128, N);
        int stage = 0;
        uint32_t phase = 0;
        int c = 0;   // non-empty items so far
        bool ok = true, any = false;
        for (int base = 0; ok; base += 32) {
            ItemInfo it;
            const bool in = item_at(a, base + lane, it);
            const bool valid = in && it.kt * C::kKeys < it.ext;
            if (__ballot_sync(0xffffffffu, in) == 0) break;
            const int nvalid = __popc(__ballot_sync(0xffffffffu, valid));
            for (int k = 0; k < nvalid; ++k, ++c) {
                const int acc = c % C::kAcc;
                const uint32_t acc_phase = (uint32_t)(c / C::kAcc) & 1u;
                if (lane == 0) {
                    ok = mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag) &&
                         mbar_wait(&full_bar[stage], phase, abort_flag);
                    if (ok) {
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(stage_base + stage * C::kStageBytes);
                        const uint32_t b_addr = a_addr + C::kABytes;
                        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * C::kAccCols);
                        // PAIR: the even keys sit in bytes 0..63 of each A row,
                        // the odd keys in bytes 64..127; one accumulator each
#pragma unroll
                        for (int h = 0; h < C::kKeysPerRow; ++h) {
#pragma unroll
                            for (int kk = 0; kk < RB / 32; ++kk) {
                                const uint64_t da = smem_desc(a_addr + h * RB + kk * 32, C::kSboA, C::kLayoutA);
                                const uint64_t db = smem_desc(b_addr + kk * 32, C::kSboB, C::kLayoutB);
                                const uint32_t d = d_tmem + (uint32_t)(h * N);
                                if constexpr (F8) tc_mma_f8(d, da, db, idesc, kk > 0 ? 1u : 0u);
                                else tc_mma_f16(d, da, db, idesc, kk > 0 ? 1u : 0u);
                            }
                        }
                        tc_commit(&empty_bar[stage]);
                        tc_commit(&tfull_bar[acc]);
                        any = true;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
            }
        }
        if (lane == 0 && any) {   // all issued MMAs complete before TMEM is released
            tc_commit(drain_bar);
            volatile int no_abort = 0;
            mbar_wait(drain_bar, 0, &no_abort);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Warp ew = (item group ig, column group cg, lane quadrant quad): it
        // owns TMEM lanes quad*32.. (keys) and the columns of query group cg
        // (kGroupCols = q_per_grp queries x H_I heads) of every kIG-th item.
        const int ew = warp - 2;
        const int quad = warp & 3;               // the TMEM lane quadrant a warp may access is warp % 4
        const int cg = (ew >> 2) % C::kCG, ig = (ew >> 2) / C::kCG;
        constexpr int QPL = 16 / H_I;            // queries per 16-column TMEM load
        constexpr int NLD = C::kGroupCols / 16;  // TMEM loads per item
        constexpr int BATCH = NLD < 4 ? NLD : 4;
        constexpr int QPG = C::kGroupCols / H_I; // queries per group
        constexpr int WREGS = (C::kGroupCols + 31) / 32;
        constexpr int NVREGS = (QPG + 31) / 32;
        const int q_lo = cg * QPG;
        float *ws = w_stage + ew * C::kGroupCols;
        int *nvs = nv_stage + ew * C::kGroupCols;
        int c = 0;
        bool ok = true;
        for (int base = 0; ok; base += 32) {
            ItemInfo mine;
            const bool in = item_at(a, base + lane, mine);
            const bool valid = in && mine.kt * C::kKeys < mine.ext;
            if (__ballot_sync(0xffffffffu, in) == 0) break;
            uint32_t vmask = __ballot_sync(0xffffffffu, valid);
            for (; vmask; ++c) {
                const int j = __ffs(vmask) - 1;
                vmask &= vmask - 1;
                if (c % C::kIG != ig) continue;
                const int b = __shfl_sync(0xffffffffu, mine.b, j);
                const int qt = __shfl_sync(0xffffffffu, mine.qt, j);
                const int kt = __shfl_sync(0xffffffffu, mine.kt, j);
                const int acc = c % C::kAcc;
                const uint32_t acc_phase = (uint32_t)(c / C::kAcc) & 1u;
                // this group's weights and row lengths, fetched before the wait
                const int t_base = qt * a.QT + q_lo;
                const int nq = max(0, min(QPG, a.T - t_base));
                const int64_t row0 = (int64_t)b * a.T + t_base;
                float wr[WREGS];
                int nvr[NVREGS];
#pragma unroll
                for (int k = 0; k < WREGS; ++k) {
                    const int i = lane + 32 * k;
                    wr[k] = (i < nq * H_I) ? __uint_as_float((uint32_t)__ldg(a.w + row0 * H_I + i) << 16) : 0.f;
                }
#pragma unroll
                for (int k = 0; k < NVREGS; ++k) {
                    const int i = lane + 32 * k;
                    int nv = 0;
                    if (i < nq) {
                        nv = a.n_valid ? __ldg(a.n_valid + row0 + i) : a.S - a.T + t_base + i + 1;
                        if (nv < 0 || nv > a.S) {   // never write outside the row
                            report(a.dev_status, SA_DEV_INDEX);
                            nv = nv < 0 ? 0 : a.S;
                        }
                    }
                    nvr[k] = nv;
                }
                ok = __all_sync(0xffffffffu, mbar_wait(&tfull_bar[acc], acc_phase, abort_flag));
                if (!ok) break;
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < WREGS; ++k)
                    if (lane + 32 * k < C::kGroupCols) ws[lane + 32 * k] = wr[k];
#pragma unroll
                for (int k = 0; k < NVREGS; ++k)
                    if (lane + 32 * k < QPG) nvs[lane + 32 * k] = nvr[k];
                __syncwarp();
                constexpr int KPR = C::kKeysPerRow;
                const int s = kt * C::kKeys + (quad * 32 + lane) * KPR;   // PAIR: keys s and s + 1
                const uint32_t t_cols = tmem_base + ((uint32_t)(quad * 32) << 16) +
                                        (uint32_t)(acc * C::kAccCols + cg * C::kGroupCols);
                float *op = a.scores + row0 * a.ld + s;
                const bool causal = a.n_valid == nullptr;
                const int causal_end = a.S - a.T + t_base + 1;   // row length of query q: causal_end + q
#pragma unroll
                for (int l0 = 0; l0 < NLD; l0 += BATCH) {
                    uint32_t v[BATCH][KPR][16];
#pragma unroll
                    for (int bb = 0; bb < BATCH; ++bb)
#pragma unroll
                        for (int h = 0; h < KPR; ++h)
                            tmem_ld_x16(t_cols + (uint32_t)(h * N + (l0 + bb) * 16), v[bb][h]);
                    tmem_ld_wait();
#pragma unroll
                    for (int bb = 0; bb < BATCH; ++bb) {
#pragma unroll
                        for (int qq = 0; qq < QPL; ++qq) {
                            const int q = (l0 + bb) * QPL + qq;
                            if (q < nq) {
                                float wv[H_I];
                                if constexpr (H_I >= 4) {
#pragma unroll
                                    for (int j4 = 0; j4 < H_I; j4 += 4) {
                                        const float4 w4 = *reinterpret_cast<const float4 *>(ws + q * H_I + j4);
                                        wv[j4] = w4.x; wv[j4 + 1] = w4.y; wv[j4 + 2] = w4.z; wv[j4 + 3] = w4.w;
                                    }
                                } else {
#pragma unroll
                                    for (int j1 = 0; j1 < H_I; ++j1) wv[j1] = ws[q * H_I + j1];
                                }
                                float sc[KPR];
#pragma unroll
                                for (int h = 0; h < KPR; ++h) {
                                    sc[h] = 0.f;
#pragma unroll
                                    for (int j1 = 0; j1 < H_I; ++j1)
                                        sc[h] = fmaf(wv[j1], fmaxf(__uint_as_float(v[bb][h][qq * H_I + j1]), 0.f), sc[h]);
                                }
                                // causal rows (no n_valid) end at their own position
                                const int lim = causal ? causal_end + q : nvs[q];
                                if constexpr (KPR == 2) {
                                    if (s + 1 < lim && (reinterpret_cast<uintptr_t>(op) & 7u) == 0) {
                                        *reinterpret_cast<float2 *>(op) = make_float2(sc[0], sc[1]);
                                    } else {
                                        if (s < lim) op[0] = sc[0];
                                        if (s + 1 < lim) op[1] = sc[1];
                                    }
                                } else {
                                    if (s < lim) *op = sc[0];
                                }
                            }
                            op += a.ld;
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty_bar[acc]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) report(a.dev_status, SA_DEV_TIMEOUT);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// rows x RB bytes (bf16 or e4m3 elements), row-major; box = box_rows whole
// rows with the swizzle matching RB.
static bool make_map(CUtensorMap *m, const void *base, uint64_t rows, int RB, bool f8, int box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    const int elems = f8 ? RB : RB / 2;
    cuuint64_t dims[2] = {(cuuint64_t)elems, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)RB};
    cuuint32_t box[2] = {(cuuint32_t)elems, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = (RB == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUtensorMapDataType dt = f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int N, int RB, int H_I, bool F8, bool PAIR>
static sa_status launch_tc(const IndexerArgs &a, cudaStream_t st) {
    using C = IdxCfg<N, RB, PAIR>;
    IdxKernelArgs k;
    k.w = a.w; k.page_table = a.page_table; k.n_valid = a.n_valid; k.scores = a.scores; k.ld = a.ld;
    k.dev_status = a.dev_status; k.max_pages = a.max_pages; k.pool_pages = a.pool_pages;
    k.B = a.B; k.T = a.T; k.S = a.S;
    k.QT = N / H_I;
    k.QTN = (a.T + k.QT - 1) / k.QT;
    k.KT = (a.S + C::kKeys - 1) / C::kKeys;
    const long long items = (long long)a.B * k.QTN * k.KT;
    if (items > 0x7fffffffLL) return SA_ERR_UNSUPPORTED;
    k.n_items = (int)items;
    if (k.n_items == 0) return SA_OK;

    CUtensorMap mk, mq;
    const uint64_t k_rows = a.page_table ? (uint64_t)a.pool_pages * a.page_size : (uint64_t)a.B * a.S;
    // PAIR: the key cache viewed as rows of two keys (k_rows is even: S even, or 64-key pages)
    if (!make_map(&mk, a.kI, k_rows / C::kKeysPerRow, C::kARowBytes, F8, C::kBoxRows)) return SA_ERR_CUDA;
    if (!make_map(&mq, a.qI, (uint64_t)a.B * a.T * H_I, RB, F8, N)) return SA_ERR_CUDA;

    auto kern = indexer_tc_kernel<N, RB, H_I, F8, PAIR>;
    if (prepare_kernel<indexer_tc_kernel<N, RB, H_I, F8, PAIR>>(C::kSmem, false) != cudaSuccess) return SA_ERR_CUDA;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = k.n_items < sms ? k.n_items : sms;
    kern<<<grid, C::kThreads, C::kSmem, st>>>(mk, mq, k);
    return cuda_ok(cudaGetLastError());
}

template <int N, int RB, bool F8, bool PAIR = false>
static sa_status launch_tc_h(const IndexerArgs &a, cudaStream_t st) {
    switch (a.H_I) {
        case 1: return launch_tc<N, RB, 1, F8, PAIR>(a, st);
        case 2: return launch_tc<N, RB, 2, F8, PAIR>(a, st);
        case 4: return launch_tc<N, RB, 4, F8, PAIR>(a, st);
        case 8: return launch_tc<N, RB, 8, F8, PAIR>(a, st);
    }
    return SA_ERR_UNSUPPORTED;
}

template <int RB, bool F8>
static sa_status launch_tc_n(const IndexerArgs &a, cudaStream_t st) {
    const bool small = a.T * a.H_I <= 16;   // decode: a handful of queries per sequence
    if (!small) return launch_tc_h<256, RB, F8>(a, st);
    // 64-byte e4m3 keys, two to a TMA row, when rows pair up: 64-key pages, or an even S
    if constexpr (F8 && RB == 64)
        if (a.page_table || a.S % 2 == 0) return launch_tc_h<16, 64, true, true>(a, st);
    return launch_tc_h<16, RB, F8>(a, st);
}

sa_status launch_indexer(const IndexerArgs &a, cudaStream_t st) {
    const int rb = a.fp8 ? a.D_I : 2 * a.D_I;
    if (rb == 128) return a.fp8 ? launch_tc_n<128, true>(a, st) : launch_tc_n<128, false>(a, st);
    if (rb == 64) return a.fp8 ? launch_tc_n<64, true>(a, st) : launch_tc_n<64, false>(a, st);
    return SA_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------------------
// bf16 -> e4m3 (OCP FP8: 4 exponent bits with bias 7, 3 mantissa bits, no
// infinities, S.1111.111 is NaN).  The hardware conversion rounds to nearest
// even and, with .satfinite, clamps finite overflow and infinities to +-448;
// NaN stays NaN.  Eight elements per thread: one 16-byte load, one 8-byte
// store; the elements past the last whole group of 8 (or all of them when
// the buffers are not aligned for that) go one per thread.
// ------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3_pair(uint32_t bf16x2) {
    const float lo = __uint_as_float(bf16x2 << 16), hi = __uint_as_float(bf16x2 & 0xFFFF0000u);
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));   // hi -> upper byte
    return r;
}

__global__ void __launch_bounds__(256) convert_e4m3_kernel(const uint16_t *src, uint8_t *dst, int64_t n,
                                                           int64_t n_vec) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (int64_t i = i0; i < n_vec; i += stride) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(src) + i);
        uint2 o;
        o.x = e4m3_pair(u.x) | (e4m3_pair(u.y) << 16);
        o.y = e4m3_pair(u.z) | (e4m3_pair(u.w) << 16);
        reinterpret_cast<uint2 *>(dst)[i] = o;
    }
    for (int64_t i = n_vec * 8 + i0; i < n; i += stride) dst[i] = (uint8_t)(e4m3_pair(src[i]) & 0xFFu);
}

sa_status launch_convert_e4m3(const uint16_t *src, uint8_t *dst, int64_t n, cudaStream_t st) {
    const bool vec = (reinterpret_cast<uintptr_t>(src) & 15u) == 0 && (reinterpret_cast<uintptr_t>(dst) & 7u) == 0;
    const int64_t n_vec = vec ? n / 8 : 0;
    const int64_t work = n_vec + (n - n_vec * 8);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (work + 255) / 256, cap = (int64_t)sms * 8;
    const int grid = (int)(want < cap ? want : cap);
    convert_e4m3_kernel<<<grid, 256, 0, st>>>(src, dst, n, n_vec);
    return cuda_ok(cudaGetLastError());
}

// ------------------------------------------------------------------------
// Fine pass over explicit candidates: one warp per query row, candidates
// strided over lanes.  qI[t] and w[t] are staged in shared memory; each lane
// reads its candidate's key row (D_I bf16) with 16-byte loads.  fp32 sums.
// ------------------------------------------------------------------------
template <int D_I, int H_I>
__global__ void __launch_bounds__(256) indexer_cand_kernel(CandArgs a) {
    constexpr int WPB = 8;
    __shared__ float qs[WPB][H_I][D_I];
    __shared__ float ws[WPB][H_I];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * WPB + warp;
    if (t >= a.T) return;
    for (int i = lane; i < H_I * D_I; i += 32)
        qs[warp][i / D_I][i % D_I] = __uint_as_float((uint32_t)a.qI[(int64_t)t * H_I * D_I + i] << 16);
    if (lane < H_I) ws[warp][lane] = __uint_as_float((uint32_t)a.w[(int64_t)t * H_I + lane] << 16);
    __syncwarp();
    int nc = a.n_cand[t];
    if (nc < 0 || nc > a.ld_cand) { if (lane == 0) report(a.dev_status, SA_DEV_INDEX); nc = nc < 0 ? 0 : (int)a.ld_cand; }
    const int32_t *cr = a.cand + (int64_t)t * a.ld_cand;
    float *out = a.scores + (int64_t)t * a.ld;
    for (int i = lane; i < nc; i += 32) {
        const int s = cr[i];
        if (s < 0 || s >= a.S) { report(a.dev_status, SA_DEV_INDEX); continue; }
        const uint4 *kr = reinterpret_cast<const uint4 *>(a.kI + (int64_t)s * D_I);
        float key[D_I];
#pragma unroll
        for (int c = 0; c < D_I / 8; ++c) {
            const uint4 u = __ldg(kr + c);
            const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                key[c * 8 + 2 * e] = __uint_as_float(wds[e] << 16);
                key[c * 8 + 2 * e + 1] = __uint_as_float(wds[e] & 0xFFFF0000u);
            }
        }
        float sc = 0.f;
#pragma unroll
        for (int j = 0; j < H_I; ++j) {
            float dot = 0.f;
#pragma unroll
            for (int c = 0; c < D_I; ++c) dot = fmaf(qs[warp][j][c], key[c], dot);
            sc = fmaf(ws[warp][j], fmaxf(dot, 0.f), sc);
        }
        out[i] = sc;
    }
}

template <int D_I>
static sa_status launch_cand_h(const CandArgs &a, cudaStream_t st) {
    const dim3 grid((a.T + 7) / 8);
    switch (a.H_I) {
        case 1: indexer_cand_kernel<D_I, 1><<<grid, 256, 0, st>>>(a); break;
        case 2: indexer_cand_kernel<D_I, 2><<<grid, 256, 0, st>>>(a); break;
        case 4: indexer_cand_kernel<D_I, 4><<<grid, 256, 0, st>>>(a); break;
        case 8: indexer_cand_kernel<D_I, 8><<<grid, 256, 0, st>>>(a); break;
        default: return SA_ERR_UNSUPPORTED;
    }
    return cuda_ok(cudaGetLastError());
}

sa_status launch_indexer_candidates(const CandArgs &a, cudaStream_t st) {
    if (a.T == 0) return SA_OK;
    if (a.D_I == 64) return launch_cand_h<64>(a, st);
    if (a.D_I == 32) return launch_cand_h<32>(a, st);
    return SA_ERR_UNSUPPORTED;
}

}  // namespace sa
