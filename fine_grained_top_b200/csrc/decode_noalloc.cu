// decode_noalloc.cu -- sparse-attention decode without a caller workspace.
//
// sa_sparse_attn_decode keeps the partial results of its split-K chunks in a
// workspace that the caller allocates.  Some callers cannot do that: a
// plugin inside a serving engine that has reserved the device memory for its
// own KV-cache pool and hands plugins only input and output pointers; a C
// caller with no device allocator of its own; a latency-critical loop where
// cudaMalloc / cudaFree, which can synchronise the device, must not appear.
// For them, sa_sparse_attn_decode_noalloc runs the same decode kernels on a
// fixed scratch array that lives in this file as a device variable.
//
// Costs and limits:
//   * every GPU that loads this library holds the array
//     (SA_DECODE_NOALLOC_SCRATCH_BYTES = 16 MiB) until the process exits;
//   * a call whose partial results would not fit is rejected with
//     SA_ERR_WORKSPACE before anything is enqueued;
//   * every call on a device uses the same array, so calls that overlap on the
//     GPU (two streams, two host threads) race with each other and must be
//     serialised by the caller;
//   * the array keeps the last call's contents; nothing has to start at zero,
//     because the merge kernel reads only slots that the split kernel of the
//     same call has written first.
// The first call on a device looks up the array's device address (once per
// device, with that device current); make that first call before any stream
// capture.  The address is cached per device index for the life of the
// process.  cudaDeviceReset unloads the device's copy of the library's module,
// which leaves the cached address stale: a process that resets a device must
// not call this entry point on that device afterwards.  Nothing here calls
// cudaMalloc, cudaFree or an allocating routine.
#include <mutex>

#include "../../include/sa.h"
#include "internal.h"

namespace sa {

// In host code this name is only a host-side stand-in for the array, not a
// device address: the kernels must be given the address that
// cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_decode_scratch[SA_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
sa_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) {
            // clear the runtime's last-error slot, so that the failure is not
            // reported again by an unrelated later call
            (void)cudaGetLastError();
            return SA_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return SA_OK;
}
}  // namespace

}  // namespace sa

using namespace sa;


extern "C" sa_status sa_sparse_attn_decode_noalloc(const sa_bf16 *q, const sa_bf16 *k_cache,
                                                   const sa_bf16 *v_cache, const int32_t *page_table,
                                                   int max_pages, int pool_pages, int page_size, int S_max,
                                                   const int32_t *seq_lens, const int32_t *topk, int K, int W,
                                                   int B, int Hq, int d, float scale, sa_bf16 *out, float *lse,
                                                   int *dev_status, sa_stream stream) {
    const sa_status chk = check_decode_args(q, k_cache, v_cache, page_table, max_pages, pool_pages, page_size,
                                            S_max, seq_lens, topk, K, W, B, Hq, d, out);
    if (chk != SA_OK || B == 0) return chk;
    if (decode_workspace_bytes(B, Hq, d, K, W) > (size_t)SA_DECODE_NOALLOC_SCRATCH_BYTES)
        return SA_ERR_WORKSPACE;   // the partial results would not fit in the fixed array
    try {
        void *scratch = nullptr;
        const sa_status s = scratch_address(&scratch);
        if (s != SA_OK) return s;
        DecodeArgs a;
        a.q = q; a.k = k_cache; a.v = v_cache; a.page_table = page_table; a.max_pages = max_pages;
        a.pool_pages = pool_pages; a.page_size = page_size; a.S_max = page_table ? max_pages * 64 : S_max;
        a.seq_lens = seq_lens; a.topk = topk; a.K = K; a.W = W; a.B = B; a.Hq = Hq; a.d = d; a.scale = scale;
        a.out = out; a.lse = lse; a.workspace = scratch; a.dev_status = dev_status;
        a.force_split_k = true;   // the split-K kernels, with their partials in the fixed array
        return launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
    } catch (...) {
        return SA_ERR_CUDA;
    }
}
