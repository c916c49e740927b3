// gather_ceiling.cu -- the rate at which one B200 moves randomly chosen
// 256-byte rows (one K or V row of the sparse attention, d = 128 bf16) from L2
// into shared memory with 16-byte cp.async, or into registers with 16-byte
// loads.  The sparse prefill attention of the two-stage 64K workload gathers
// about 82 GB of such rows per step from a 32 MB K+V set that L2 holds, so
// this ceiling, not HBM, bounds its time.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -o gather_ceiling gather_ceiling.cu
//   ./gather_ceiling
//
// Each "query" gathers 2560 keys (K + W of the workload); row indices come
// from a hash (no index reads).  Three row sets: 65536 rows (32 MB of K+V,
// L2-resident) in random and in sequential order, and 2M rows (1 GB, HBM).
// Each line prints the bytes moved per second; the stage shapes cover the
// depths and CTA counts a kernel can afford in shared memory.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include <vector>

#define CK(x) do { cudaError_t e = (x); if (e != cudaSuccess) { printf("CUDA %s at %d\n", cudaGetErrorString(e), __LINE__); return 1; } } while (0)

__device__ __forceinline__ uint32_t hash32(uint32_t x) {
    x ^= x >> 16; x *= 0x7feb352dU; x ^= x >> 15; x *= 0x846ca68bU; x ^= x >> 16; return x;
}
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void cp16(void *s, const void *g) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(smem_u32(s)), "l"(g) : "memory");
}
__device__ __forceinline__ void commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void waitg() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }

constexpr int D = 128;          // bf16 per row -> 256 B
constexpr int NCH = D / 8;      // 16-byte chunks per row
constexpr int KEYS = 2560;      // keys per query

// row of key i of query q: random (mode 0) or sequential (mode 1)
__device__ __forceinline__ uint32_t row_of(int mode, uint32_t q, uint32_t i, uint32_t mask) {
    return mode == 0 ? (hash32(q * 4096u + i) & mask) : ((q * KEYS + i) & mask);
}

// cp.async ring: CKEYS keys per stage (K and V rows), STAGES stages, THREADS threads.
template <int CKEYS, int STAGES, int THREADS>
__global__ void __launch_bounds__(THREADS) gather_cpasync(const uint16_t *K, const uint16_t *V, uint32_t mask,
                                                         int Q, int mode, uint32_t *sink) {
    extern __shared__ __align__(128) uint8_t sm[];
    constexpr int TILE = CKEYS * D * 2;
    const int tid = threadIdx.x;
    const int chunks_per_q = KEYS / CKEYS;
    // this CTA's global chunk stream: queries blockIdx.x, +gridDim.x, ...
    const int my_q = (Q - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const int total = my_q * chunks_per_q;
    auto issue = [&](int g) {
        const int qq = (int)blockIdx.x + (g / chunks_per_q) * (int)gridDim.x;
        const int c = g % chunks_per_q;
        uint8_t *dk = sm + (g % STAGES) * 2 * TILE, *dv = dk + TILE;
#pragma unroll
        for (int it = 0; it < CKEYS * NCH / THREADS; ++it) {
            const int idx = it * THREADS + tid, key = idx / NCH, ch = idx % NCH;
            const uint32_t row = row_of(mode, (uint32_t)qq, (uint32_t)(c * CKEYS + key), mask);
            const uint32_t off = key * (D * 2) + ((ch ^ (key & 7)) << 4);
            cp16(dk + off, K + (size_t)row * D + ch * 8);
            cp16(dv + off, V + (size_t)row * D + ch * 8);
        }
    };
    for (int g = 0; g < STAGES - 1; ++g) { if (g < total) issue(g); commit(); }
    uint32_t acc = 0;
    for (int g = 0; g < total; ++g) {
        if (g + STAGES - 1 < total) issue(g + STAGES - 1);
        commit();
        waitg<STAGES - 1>();
        __syncthreads();
        const uint8_t *dk = sm + (g % STAGES) * 2 * TILE;
        acc ^= *reinterpret_cast<const uint32_t *>(dk + (tid * 16) % (2 * TILE));
        __syncthreads();
    }
    waitg<0>();
    if (acc == 0x12345678u) sink[blockIdx.x] = acc;
}

// register loads: each thread keeps UNR 16-byte loads in flight
template <int UNR, int THREADS>
__global__ void __launch_bounds__(THREADS) gather_ldg(const uint16_t *K, const uint16_t *V, uint32_t mask, int Q,
                                                     int mode, uint32_t *sink) {
    const int tid = threadIdx.x;
    uint32_t acc = 0;
    // one "item" = one key's K and V rows = 2*NCH 16-byte loads; a warp covers 1 key x 2 arrays per instruction pair (16 lanes/row)
    const long long total_keys = (long long)Q * KEYS;
    const long long step = (long long)gridDim.x * (THREADS / NCH);
    long long k0 = (long long)blockIdx.x * (THREADS / NCH) + tid / NCH;
    const int ch = tid % NCH;
    for (; k0 < total_keys; k0 += step * UNR) {
        uint4 a[UNR], b[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const long long kk = k0 + u * step;
            if (kk < total_keys) {
                const uint32_t q = (uint32_t)(kk / KEYS), i = (uint32_t)(kk % KEYS);
                const uint32_t row = row_of(mode, q, i, mask);
                a[u] = __ldcg(reinterpret_cast<const uint4 *>(K + (size_t)row * D + ch * 8));
                b[u] = __ldcg(reinterpret_cast<const uint4 *>(V + (size_t)row * D + ch * 8));
            } else {
                a[u] = b[u] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) acc ^= a[u].x ^ a[u].w ^ b[u].y ^ b[u].z;
    }
    if (acc == 0x12345678u) sink[blockIdx.x] = acc;
}

template <class F>
float time_it(F f, int reps) {
    cudaEvent_t a, b;
    cudaEventCreate(&a); cudaEventCreate(&b);
    f();
    cudaDeviceSynchronize();
    cudaEventRecord(a);
    for (int r = 0; r < reps; ++r) f();
    cudaEventRecord(b);
    cudaEventSynchronize(b);
    float ms; cudaEventElapsedTime(&ms, a, b);
    return ms / reps;
}

template <int CKEYS, int STAGES, int THREADS>
int run_cp(const uint16_t *K, const uint16_t *V, uint32_t mask, int Q, int mode, uint32_t *sink, int sms, const char *tag) {
    auto kern = gather_cpasync<CKEYS, STAGES, THREADS>;
    const int smem = STAGES * 2 * CKEYS * D * 2;
    CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    int per = 0;
    CK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kern, THREADS, smem));
    const int grid = sms * per;
    float ms = time_it([&] { kern<<<grid, THREADS, smem>>>(K, V, mask, Q, mode, sink); }, 5);
    CK(cudaGetLastError());
    const double bytes = (double)Q * KEYS * 2 * D * 2;
    printf("%-8s cp.async  keys/stage %3d stages %d threads %3d ctas/SM %d  smem %6d  %8.3f ms  %7.0f GB/s\n", tag,
           CKEYS, STAGES, THREADS, per, smem, ms, bytes / ms / 1e6);
    return 0;
}

template <int UNR, int THREADS>
int run_ldg(const uint16_t *K, const uint16_t *V, uint32_t mask, int Q, int mode, uint32_t *sink, int sms, const char *tag) {
    auto kern = gather_ldg<UNR, THREADS>;
    int per = 0;
    CK(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kern, THREADS, 0));
    const int grid = sms * per;
    float ms = time_it([&] { kern<<<grid, THREADS>>>(K, V, mask, Q, mode, sink); }, 5);
    CK(cudaGetLastError());
    const double bytes = (double)Q * KEYS * 2 * D * 2;
    printf("%-8s ldg.v4    unroll %d threads %3d ctas/SM %d  %8.3f ms  %7.0f GB/s\n", tag, UNR, THREADS, per, ms,
           bytes / ms / 1e6);
    return 0;
}

int main() {
    int sms = 0;
    CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0));
    // two key sets: 65536 rows (32 MB of K+V, L2-resident) and 2M rows (1 GB, HBM)
    const size_t big_rows = 1u << 21;
    uint16_t *K, *V;
    uint32_t *sink;
    CK(cudaMalloc(&K, big_rows * D * 2));
    CK(cudaMalloc(&V, big_rows * D * 2));
    CK(cudaMalloc(&sink, 4096 * 4));
    CK(cudaMemset(K, 1, big_rows * D * 2));
    CK(cudaMemset(V, 2, big_rows * D * 2));
    const int Q = 8192;   // queries per launch: 8192 * 2560 keys * 512 B = 10.7 GB gathered
    struct { uint32_t mask; int mode; const char *tag; } cases[] = {
        {65535u, 0, "L2-rand"}, {65535u, 1, "L2-seq"}, {(uint32_t)big_rows - 1, 0, "HBM-rand"}};
    for (auto &c : cases) {
        run_cp<64, 2, 128>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_cp<64, 3, 128>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_cp<64, 4, 128>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_cp<64, 6, 128>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_cp<32, 4, 128>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_cp<32, 6, 128>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_cp<64, 3, 256>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_cp<128, 3, 256>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_ldg<2, 256>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_ldg<4, 256>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_ldg<8, 256>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
        run_ldg<4, 512>(K, V, c.mask, Q, c.mode, sink, sms, c.tag);
    }
    CK(cudaDeviceSynchronize());
    printf("done\n");
    return 0;
}
