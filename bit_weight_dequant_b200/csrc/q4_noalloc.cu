// q4_noalloc.cu -- the fused GEMM entry point for callers that cannot
// allocate device memory.
//
// q4_gemm_skinny needs a small scratch workspace (partial sums of weight
// tiles shared between thread blocks, one counter per tile, an error word)
// that its caller allocates.  Some callers cannot: code that runs while a
// stream is being captured into a CUDA graph (where cudaMalloc is not
// allowed), real-time or safety-constrained runtimes that forbid device
// allocations after start-up, and plugin hosts whose allocator hands no
// memory to third-party code.  q4_gemm_skinny_noalloc serves them with a
// fixed scratch array compiled into this library instead.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/q4.h"
#include "q4_internal.h"
#include "q4_plan.cuh"

namespace q4 {

// The built-in scratch: every GPU that loads the library holds it until the
// process exits.  Zero-initialised when the module is loaded.
static constexpr size_t kNoAllocBytes = (size_t)Q4_NOALLOC_WORKSPACE_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_ws[kNoAllocBytes];

// Device address of g_noalloc_ws, looked up once per device with that device
// current (in host code the symbol itself is only a host-side stand-in).
static void* noalloc_address(int* status) {
    static constexpr int kMaxDev = 64;
    static void* addr[kMaxDev] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        cudaGetLastError();
        *status = Q4_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_ws) != cudaSuccess || !p) {
            cudaGetLastError();
            *status = Q4_ERR_CUDA;
            return nullptr;
        }
        addr[dev] = p;
    }
    *status = Q4_OK;
    return addr[dev];
}

}  // namespace q4

extern "C" int q4_gemm_skinny_noalloc(const void* A, const uint8_t* Wpacked, const float* absmax, const float* code,
                                      int M, int N, int K, int blocksize, int act_dtype, void* out, void* stream) {
    size_t need = 0;
    int rc = q4_gemm_workspace_size(M, N, K, blocksize, act_dtype, &need);
    if (rc != Q4_OK) return rc;
    if (need > q4::kNoAllocBytes) return Q4_ERR_WORKSPACE;  // more scratch than the built-in array holds
    if (M == 0 || N == 0 || need == 0)
        return q4_gemm_skinny(A, Wpacked, absmax, code, M, N, K, blocksize, act_dtype, out, nullptr, 0, stream);
    void* ws = q4::noalloc_address(&rc);
    if (rc != Q4_OK) return rc;
    // The array keeps the previous call's contents.  Clear what must start
    // at zero -- the 256-byte header with the error word, and the tile
    // counters after the partial-sum slots -- with cudaMemsetAsync (which
    // allocates nothing); the slots are written before they are read.  A
    // kernel whose workspace is the header alone (the row-split kernel) only
    // ever writes the error word, which this entry does not report, so it
    // gets no memset: each one costs 3-4 us of stream time in a graph.
    cudaStream_t st = (cudaStream_t)stream;
    if (need > 256) {
        int sms = 0;
        if (q4::device_sm_count(&sms) != 0) return Q4_ERR_CUDA;
        const size_t counters = 256 + (size_t)sms * 2 * q4::kMaxSlotBytes;
        if (cudaMemsetAsync(ws, 0, 256, st) != cudaSuccess ||
            (need > counters &&
             cudaMemsetAsync(static_cast<char*>(ws) + counters, 0, need - counters, st) != cudaSuccess)) {
            cudaGetLastError();
            return Q4_ERR_CUDA;
        }
    }
    return q4_gemm_skinny(A, Wpacked, absmax, code, M, N, K, blocksize, act_dtype, out, ws, need, stream);
}
