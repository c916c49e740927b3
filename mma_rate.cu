// mma_rate.cu -- tcgen05.mma issue rate on one B200 SM: one thread issues
// groups of 8 MMAs (M = 128, K = 16 bf16 -> fp32) with precomputed
// descriptors over shared-memory operands holding arbitrary bits, and the
// cycles per instruction are printed for several N, K-major and MN-major A,
// and A from TMEM.  The gathered prefill attention issues 16 such MMAs (N = 16)
// per 128-key tile; this gives their cost.
//
//   nvcc -gencode arch=compute_100a,code=sm_100a -O3 -std=c++17 -o mma_rate mma_rate.cu && ./mma_rate
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
#include "fine_grained_top_b200/csrc/ptx.cuh"
using namespace sa;

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t id) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, 1, 0;"
                 " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d), "l"(a), "l"(b), "r"(id) : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t id) {
    asm volatile("{ .reg .pred p; setp.ne.b32 p, 1, 0;"
                 " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(d), "r"(a), "l"(b), "r"(id) : "memory");
}

template <int N, int NACC, bool TS, bool AMN = false>
__global__ void __launch_bounds__(128, 1) k_mma(int groups, long long *out) {
    extern __shared__ __align__(1024) uint8_t sm_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)sm_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t bar2;
    __shared__ uint32_t tslot;
    __shared__ int abortf;
    if (threadIdx.x == 0) { mbar_init(&bar2, 1); abortf = 0; fence_mbar_init(); }
    if (threadIdx.x < 32) { tmem_alloc(&tslot, 512); tmem_relinquish(); }
    tc_fence_before(); __syncthreads(); tc_fence_after();
    uint32_t tm = tslot;
    if (threadIdx.x == 0) {
        constexpr uint32_t id = idesc_bf16_f32(128, N) | (AMN ? (1u << 15) : 0u);
        uint64_t ad = smem_desc(smem_u32(sm), 1024, 2);
        if (AMN) {
            const uint32_t addr = smem_u32(sm);
            ad = 0; ad |= (uint64_t)((addr >> 4) & 0x3FFF); ad |= (uint64_t)((16384 >> 4) & 0x3FFF) << 16;
            ad |= (uint64_t)((1024 >> 4) & 0x3FFF) << 32; ad |= (uint64_t)1 << 46; ad |= (uint64_t)2 << 61;
        }
        const uint64_t bd = smem_desc(smem_u32(sm + 32768), 1024, 2);
        long long t0 = clock64();
        for (int g = 0; g < groups; ++g) {
#pragma unroll
            for (int j = 0; j < NACC; ++j) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4);
                    if (TS) mma_ts(tm + (uint32_t)(j * (256 / NACC)), tm + 384u + (uint32_t)(kk * 8), bd + off, id);
                    else if (AMN) mma_ss(tm + (uint32_t)(j * (256 / NACC)), ad + (uint64_t)((kk * 2048) >> 4), bd + off, id);
                    else mma_ss(tm + (uint32_t)(j * (256 / NACC)), ad + off, bd + off, id);
                }
            }
        }
        long long t1 = clock64();
        tc_commit(&bar2);
        bool ok = mbar_wait(&bar2, 0u, &abortf);
        long long t2 = clock64();
        if (blockIdx.x == 0) { out[0] = t1 - t0; out[1] = t2 - t0; out[2] = ok; }
    }
    tc_fence_before(); __syncthreads();
    if (threadIdx.x < 32) { tc_fence_after(); tmem_dealloc(tm, 512); }
}

template <int N, int NACC, bool TS, bool AMN = false>
void run(const char *name, long long *d) {
    long long h[3];
    cudaFuncSetAttribute(k_mma<N, NACC, TS, AMN>, cudaFuncAttributeMaxDynamicSharedMemorySize, 100000);
    const int groups = 64;
    for (int rep = 0; rep < 2; ++rep) {
        k_mma<N, NACC, TS, AMN><<<148, 128, 100000>>>(groups, d);
        cudaError_t err = cudaDeviceSynchronize();
        cudaMemcpy(h, d, 24, cudaMemcpyDeviceToHost);
        const double n = groups * NACC * 8.0;
        if (rep) printf("%-22s issue %6.1f cyc/mma  done %6.1f cyc/mma (nominal %d)  ok=%lld %s\n", name, h[0] / n, h[1] / n, N / 2, h[2], cudaGetErrorString(err));
    }
}

int main() {
    long long *d; cudaMalloc(&d, 64);
    run<128, 1, false>("SS N=128 1 acc", d);
    run<128, 2, false>("SS N=128 2 acc", d);
    run<64, 1, false>("SS N=64 1 acc", d);
    run<64, 4, false>("SS N=64 4 acc", d);
    run<256, 1, false>("SS N=256 1 acc", d);
    run<128, 1, true>("TS N=128 1 acc", d);
    run<128, 2, true>("TS N=128 2 acc", d);
    run<16, 1, false>("SS N=16 1 acc", d);
    run<16, 4, false>("SS N=16 4 acc", d);
    run<32, 1, false>("SS N=32 1 acc", d);
    run<16, 1, false, true>("SS N=16 A-MN 1 acc", d);
    run<16, 4, false, true>("SS N=16 A-MN 4 acc", d);
    run<32, 1, false, true>("SS N=32 A-MN 1 acc", d);
    return 0;
}
