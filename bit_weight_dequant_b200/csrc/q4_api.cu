// q4_api.cu -- extern "C" entry points of libq4 (declared in include/q4.h):
// argument validation, the M- and shape-keyed launch table, workspace sizing
// and error reporting.  Every function validates before it enqueues anything
// and returns a q4_status; a failed launch drains the runtime's last error.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "../../include/q4.h"
#include "q4_internal.h"
#include "q4_plan.cuh"

namespace q4 {

static constexpr int kMaxDevices = 64;

int device_sm_count(int* sms) {
    static std::atomic<int> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 1;
    }
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v <= 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
            cudaGetLastError();
            return 1;
        }
        cache[dev].store(v, std::memory_order_relaxed);
    }
    *sms = v;
    return 0;
}

cudaError_t ensure_smem_attr(const void* kernel, size_t bytes) {
    static std::mutex mu;
    static std::unordered_map<const void*, uint64_t> done;  // kernel -> bitmask of devices
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    uint64_t& mask = done[kernel];
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
    if (bit && (mask & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) mask |= bit;
    return e;
}

static bool is_pow2_blocksize(int bs) { return bs >= 32 && bs <= 4096 && (bs & (bs - 1)) == 0; }

static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Host-side fault injection for tests: Q4_TEST_FAIL_LAUNCH set to a
// non-empty value other than "0" makes every entry point report Q4_ERR_CUDA
// instead of launching (nothing reaches the GPU).
static bool injected_failure() {
    const char* v = std::getenv("Q4_TEST_FAIL_LAUNCH");
    return v && v[0] && std::strcmp(v, "0") != 0;
}

// Test hook for the row-split kernel: Q4_TEST_SKIP_STAGE=<i> makes each
// CTA's producer leave stage i unloaded, with short wait limits, so the
// kernel's bounded waits run out and it reports error word 1 (no GPU fault:
// every wait is bounded, every copy that was issued is waited for).
static int injected_stage_skip() {
    const char* v = std::getenv("Q4_TEST_SKIP_STAGE");
    if (!v || !v[0]) return -1;
    const int i = std::atoi(v);
    return i >= 0 ? i : -1;
}

static int from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return Q4_OK;
    cudaGetLastError();  // drain: leave no error of ours pending
    return Q4_ERR_CUDA;
}

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace layout: [header: error word, 256 B][partial slots: sms x 2 x
// kMaxSlotBytes][counters: one int per tile].  The counters sit at an offset
// that depends only on the SM count, so scratch written by a call of one
// shape never lands on another shape's counters; each call returns the
// counters it used to zero.
static constexpr size_t kWsHeader = 256;
static size_t ws_counter_offset(int sms) { return kWsHeader + (size_t)sms * 2 * kMaxSlotBytes; }

// With fewer tiles than SMs, one CTA per tile (every tile whole, no
// cross-CTA fix-up at the end) beats spreading the units over every SM when
// what the idle SMs would have streamed costs less time than the fix-up
// saves.  Fitted to B200 measurements: the fix-up (publish, count, read back)
// costs about 3 us at the end of a launch, and an SM streams about 34 KB/us
// in the main loop.  Examples: K8192/N8192 (128 tiles, ~10 % faster), K5120/
// N5120 (80 tiles, ~13 %), but not K28672/N8192 (128 tiles of 0.9 MB each).
static bool data_parallel_pays(int tiles, int sms, int64_t weights) {
    const double bytes = (double)weights * 0.5625;                // codes + absmax at blocksize 64
    const double idle_us = (double)(sms - tiles) * bytes / ((double)tiles * sms * 34400.0);
    return idle_us < 3.0;
}

// Row-split kernel (loader 7) or stream-K kernel (loader 2) for M <= 16,
// fitted to B200 measurements of both on the five benchmark configurations
// (back-to-back launches over distinct weight copies).  The row-split kernel
// has no cross-CTA fix-up, which is what dominates small and medium layers
// (K5120/N5120: 7.3 vs 8.2 us; K10240/N320: 5.9 vs 11.2 us; 4096^2: 6.1 vs
// 6.5 us; K8192/N10240: 13.5 vs 14.7 us), and a chain of layers runs best on
// one kernel throughout (the 70B-class decode step: 82.6 us on the row-split
// kernel, 84.8 us on stream-K, 86.7 us mixing them per layer).  The
// stream-K kernel stays where the row-split kernel's tiles hold few k-stages
// and every CTA has many of them (K2560/N248320: 67 vs 96 us), and for
// M >= 8 on layers of 2^26 weights or more (K17408/N5120 at M = 16: 21 vs
// 26 us).
static bool rows_kernel_pays(int M, int N, int K, int sms) {
    const int64_t tiles = ((int64_t)N + 63) / 64, weights = (int64_t)N * K;
    if (K < 4096 && tiles > 4 * (int64_t)sms) return false;
    if (M >= 8 && weights >= ((int64_t)1 << 26)) return false;
    return true;
}

// Validates a GEMM request.  Returns Q4_OK and fills `ch` with the launch
// table's choice (with `ov` applied) and the problem's unit counts.
static int gemm_choose(int M, int N, int K, int blocksize, int act_dtype, int num_sms, const q4_gemm_plan_t* ov,
                       GemmChoice* ch, int* tiles, int64_t* units, size_t* ws_bytes, int* sms_out) {
    if (M < 0 || N < 0 || K < 0) return Q4_ERR_INVALID_ARG;
    if (!is_pow2_blocksize(blocksize)) return Q4_ERR_INVALID_ARG;
    if (act_dtype != Q4_BF16 && act_dtype != Q4_FP16 && act_dtype != Q4_FP32) return Q4_ERR_INVALID_ARG;
    if (ov && (ov->math > 3 || ov->l2_prefetch > 256 || ov->loader > 7 || ov->pdl > 2)) return Q4_ERR_INVALID_ARG;
    if (M > 128 || K % blocksize != 0) return Q4_ERR_UNSUPPORTED;
    GemmChoice c{};
    if (act_dtype == Q4_FP32 || (ov && ov->math == 2)) {
        // The CUDA-core kernel (M <= 16), units of R rows x 512 k split over
        // every warp of the grid: fp32 activations always; bf16 / fp16 on
        // request (math = 2), widened exactly to fp32 on load.
        if (M > 16) return Q4_ERR_UNSUPPORTED;
        if (ov && ((ov->math > 0 && ov->math != 2) || ov->loader > 1)) return Q4_ERR_UNSUPPORTED;
        const SimtShape sh = simt_shape(M);
        if (ov && ov->warps > 0 && ov->warps != sh.warps) return Q4_ERR_UNSUPPORTED;
        c.math = 2;
        c.sub_block = 512;
        c.m_pad = sh.m_pad;
        c.rows_per_tile = sh.rows;
        c.warps = sh.warps;
        c.loader = 1;
        c.depth = 2;  // units in flight per warp
        c.l2pf = 0;
        c.pdl = (ov && ov->pdl > 0) ? ov->pdl : 0;
        const int64_t t64 = N > 0 ? ((int64_t)N + sh.rows - 1) / sh.rows : 0;
        const int64_t u = t64 * (((int64_t)K + 511) / 512);
        if (u >= ((int64_t)1 << 31) || K >= (1 << 29)) return Q4_ERR_UNSUPPORTED;  // 32-bit row offsets
        int sms = num_sms;
        if (sms <= 0 && device_sm_count(&sms) != 0) return Q4_ERR_CUDA;
        if (ov && ov->ctas > sms) return Q4_ERR_INVALID_ARG;
        int64_t g = (ov && ov->ctas > 0) ? ov->ctas : sms;
        const int64_t need_ctas = (u + sh.warps - 1) / sh.warps;  // at least one unit per warp where possible
        if (g > need_ctas) g = need_ctas;
        if (g < 1) g = 1;
        c.ctas = (int)g;
        *ch = c;
        *tiles = (int)t64;
        *units = u;
        *sms_out = sms;
        // Pieces of row groups go to the fixed partial region (at most
        // 2 x 128 floats per warp-slot pair and 8 KiB per SM); one counter
        // per row group sits at the fixed counter offset.
        *ws_bytes = u > 1 ? ws_counter_offset(sms) + align_up((size_t)t64 * sizeof(int), 256) : 0;
        return Q4_OK;
    }
    // 17 <= M <= 32 runs on the mma.sync kernel with 32-row tiles and 2-unit
    // stages when its TMA rules hold (and no override asks for tcgen05).
    const bool want_umma = ov && (ov->math == 3 || ov->loader == 6);
    // 33 <= M <= 64 under the same rules: row chunks of 32 on the mma.sync
    // kernels, one launch each (every chunk streams the weights again).
    // Measured faster than the tcgen05 kernel on every shape of the M sweep
    // at these M; M > 64 stays on tcgen05.
    if (M > 32 && M <= 64 && !want_umma && blocksize >= 64 && (K / blocksize) % 4 == 0 &&
        (int64_t)N * (K / 64) > 1) {
        GemmChoice first{}, rest{};
        int t1 = 0, t2 = 0, s1 = 0, s2 = 0;
        int64_t u1 = 0, u2 = 0;
        size_t w1 = 0, w2 = 0;
        int rc = gemm_choose(32, N, K, blocksize, act_dtype, num_sms, ov, &first, &t1, &u1, &w1, &s1);
        if (rc == Q4_OK) rc = gemm_choose(M - 32, N, K, blocksize, act_dtype, num_sms, ov, &rest, &t2, &u2, &w2, &s2);
        if (rc != Q4_OK) return rc;
        first.chunk_rows = 32;
        *ch = first;
        *tiles = t1;
        *units = u1;
        *ws_bytes = w1 > w2 ? w1 : w2;  // the chunks run one after another on one workspace
        *sms_out = s1;
        return Q4_OK;
    }
    const bool mma32 = M > 16 && M <= 32 && !want_umma && blocksize >= 64 && (K / blocksize) % 4 == 0 &&
                       (int64_t)N * (K / 64) > 1;
    if ((M > 16 && !mma32) || want_umma) {
        // Tensor-memory kernel (tcgen05): 128-row tiles, 64-k units, 4-unit
        // stages whose absmax box is 4 floats per row.
        if (blocksize < 64 || K % 256 != 0 || (K / blocksize) % 4 != 0) return Q4_ERR_UNSUPPORTED;
        if (ov && ov->loader > 0 && ov->loader != 6) return Q4_ERR_UNSUPPORTED;  // another kernel's loader
        c.math = 3;
        c.sub_block = 64;
        c.m_pad = M <= 32 ? 32 : M <= 64 ? 64 : 128;
        c.rows_per_tile = 128;
        c.loader = 6;
        c.warps = umma_warps();
        c.depth = 0;  // stages: as many as shared memory holds (set at launch)
        c.l2pf = 0;
        c.pdl = (ov && ov->pdl > 0) ? 1 : 0;  // activations and weights are read after the dependency wait
        const int64_t t64 = N > 0 ? ((int64_t)N + 127) / 128 : 0;
        if (t64 * (K / 64) >= (int64_t)kMaxUnits) return Q4_ERR_UNSUPPORTED;
        int sms = num_sms;
        if (sms <= 0 && device_sm_count(&sms) != 0) return Q4_ERR_CUDA;
        if (ov && ov->ctas > sms) return Q4_ERR_INVALID_ARG;
        const int t = (int)t64;
        const int64_t u = t64 * (K / 64);
        int64_t g = (ov && ov->ctas > 0) ? ov->ctas : sms;
        if (g > u) g = u;
        if (g < 1) g = 1;
        c.ctas = (int)g;
        *ch = c;
        *tiles = t;
        *units = u;
        *sms_out = sms;
        // counters at the fixed offset, then two partial slots (m_pad x 128 fp32) per CTA
        *ws_bytes = u > 1 ? ws_counter_offset(sms) + align_up((size_t)t * sizeof(int), 256) +
                                (size_t)c.ctas * 2 * umma_slot_bytes(c.m_pad)
                          : 0;
        return Q4_OK;
    }
    c.math = 1;
    c.sub_block = blocksize < 64 ? blocksize : 64;
    c.m_pad = M <= 8 ? 8 : M <= 16 ? 16 : 32;
    c.rows_per_tile = M <= 16 ? 64 : 32;
    // The TMA stage ring needs 64-k units and absmax rows that are whole
    // multiples of 16 bytes (a tensor-map stride rule); the pointer itself
    // must also be 16-byte aligned, which the caller checks at launch.
    const bool tma_ok = c.sub_block == 64 && (K / blocksize) % 4 == 0 && (int64_t)N * (K / 64) > 1;
    int sms_hint = num_sms;
    if (sms_hint <= 0 && device_sm_count(&sms_hint) != 0) sms_hint = 148;  // the choice only; the launch re-queries
    // The row-split kernel also takes blocksize 32 (two absmax per 64-k unit,
    // an 8-float box per stage): K a multiple of its 256-k stage.
    const bool rows_ok = tma_ok || (blocksize == 32 && K % 256 == 0 && (int64_t)N * (K / 64) > 1);
    c.loader = mma32 ? 3 : (rows_ok && rows_kernel_pays(M, N, K, sms_hint)) ? 7 : !tma_ok ? 1 : 2;
    if (ov && ov->loader > 0) c.loader = ov->loader;
    if (c.loader == 7 ? !rows_ok : (c.loader >= 2 && !tma_ok)) return Q4_ERR_UNSUPPORTED;
    if (c.loader == 7) {
        // Row-split kernel: 8-row groups of W split over the CTAs, one shared
        // stage ring per CTA, no cross-CTA combine (workspace: the error word).
        if (M > 32 || (M > 16 && !tma_ok)) return Q4_ERR_UNSUPPORTED;
        c.sub_block = 64;  // 64-k units at every blocksize (two absmax per unit at blocksize 32)
        c.rows_per_tile = 64;
        c.warps = rows_warps();
        c.depth = (ov && ov->depth > 0) ? ov->depth : 1;  // stage order: 1 round robin, 2 contiguous per warp
        if (c.depth > 2) return Q4_ERR_UNSUPPORTED;
        c.l2pf = (ov && ov->l2_prefetch > 1) ? ov->l2_prefetch : 0;
        c.pdl = (ov && ov->pdl > 0) ? ov->pdl : 0;
        if (ov && ov->warps > 0 && ov->warps != c.warps) return Q4_ERR_UNSUPPORTED;
        if (ov && ov->math > 0 && ov->math != 1) return Q4_ERR_UNSUPPORTED;
        if (!gemm_variant_exists(act_dtype, c)) return Q4_ERR_UNSUPPORTED;
        int sms = num_sms;
        if (sms <= 0 && device_sm_count(&sms) != 0) return Q4_ERR_CUDA;
        if (ov && ov->ctas > sms) return Q4_ERR_INVALID_ARG;
        const int64_t groups = N > 0 ? ((int64_t)N + 7) / 8 : 0;
        int64_t g = (ov && ov->ctas > 0) ? ov->ctas : sms;
        if (g > groups) g = groups;
        if (g < 1) g = 1;
        c.ctas = (int)g;
        *ch = c;
        *tiles = N > 0 ? (N + 63) / 64 : 0;
        *units = (int64_t)*tiles * (K / 64);
        *sms_out = sms;
        *ws_bytes = kWsHeader;  // the error word only
        return Q4_OK;
    }
    if (mma32) {
        // 32-row tiles: 2-unit stages (64-byte rows), six per warp
        c.warps = 8;
        c.depth = 6;
        c.l2pf = 0;
    } else if (c.loader == 2) {
        c.warps = 8;
        c.depth = 2;
        c.l2pf = 0;
    } else if (c.loader == 3) {
        c.warps = c.m_pad == 8 ? 16 : 8;
        c.depth = c.m_pad == 8 ? 2 : 4;
        c.l2pf = 0;
    } else if (c.loader == 4) {
        c.warps = 8;
        c.depth = 2;
        c.l2pf = 0;
    } else if (c.loader == 5) {
        c.warps = 16;
        c.depth = 2;
        c.l2pf = 0;
    } else {
        c.warps = c.m_pad == 8 ? 16 : 8;
        c.depth = 1;
        c.l2pf = 128;
    }
    c.pdl = 0;
    if (ov) {
        if (ov->math > 0) c.math = ov->math;
        if (ov->pdl > 0) c.pdl = c.loader == 1 ? 1 : ov->pdl;  // the direct kernel reads nothing early
        if (ov->warps > 0) c.warps = ov->warps;
        if (ov->depth > 0) c.depth = ov->depth;
        if (ov->l2_prefetch > 0) c.l2pf = ov->l2_prefetch == 1 ? 0 : ov->l2_prefetch;
    }
    if (c.math != 1 || !gemm_variant_exists(act_dtype, c)) return Q4_ERR_UNSUPPORTED;
    if ((int64_t)(N > 0 ? (N + c.rows_per_tile - 1) / c.rows_per_tile : 0) * (K / c.sub_block) >= (int64_t)kMaxUnits)
        return Q4_ERR_UNSUPPORTED;  // more than 2^23 work units (> 2^35 weights)
    int sms = num_sms;
    if (sms <= 0 && device_sm_count(&sms) != 0) return Q4_ERR_CUDA;
    if (ov && ov->ctas > sms) return Q4_ERR_INVALID_ARG;
    const int t = N > 0 ? (N + c.rows_per_tile - 1) / c.rows_per_tile : 0;
    const int64_t u = (int64_t)t * (K / c.sub_block);
    int64_t g = (ov && ov->ctas > 0) ? ov->ctas : sms;
    if (!(ov && ov->ctas > 0) && t >= 1 && t < sms && data_parallel_pays(t, sms, (int64_t)N * K)) g = t;
    if (g > u) g = u;  // every CTA owns at least one unit
    if (g < 1) g = 1;
    c.ctas = (int)g;
    *ch = c;
    *tiles = t;
    *units = u;
    *sms_out = sms;
    // A problem of one unit never splits a tile, so it needs no workspace.
    *ws_bytes = u > 1 ? ws_counter_offset(sms) + align_up((size_t)t * sizeof(int), 256) : 0;
    return Q4_OK;
}

}  // namespace q4

using namespace q4;

extern "C" {

const char* q4_status_string(int status) {
    switch (status) {
        case Q4_OK: return "Q4_OK";
        case Q4_ERR_INVALID_ARG: return "Q4_ERR_INVALID_ARG: null pointer, negative size, bad blocksize or dtype";
        case Q4_ERR_UNSUPPORTED: return "Q4_ERR_UNSUPPORTED: valid request outside this library's fused path";
        case Q4_ERR_MISALIGNED: return "Q4_ERR_MISALIGNED: pointer misses its required alignment";
        case Q4_ERR_CUDA: return "Q4_ERR_CUDA: CUDA call or kernel launch failed";
        case Q4_ERR_WORKSPACE: return "Q4_ERR_WORKSPACE: GEMM workspace missing or too small";
        default: return "unknown q4 status";
    }
}

int q4_quantize_blockwise_ex(const void* W, int w_dtype, int64_t n, int blocksize, const float* code,
                             uint8_t* packed, float* absmax, void* stream) {
    if (n < 0 || !is_pow2_blocksize(blocksize)) return Q4_ERR_INVALID_ARG;
    if (w_dtype != Q4_BF16 && w_dtype != Q4_FP16 && w_dtype != Q4_FP32) return Q4_ERR_INVALID_ARG;
    if (n == 0) return Q4_OK;  // empty input: pointers may be NULL
    if (!W || !code || !packed || !absmax) return Q4_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(code, 4) || !aligned(absmax, 4)) return Q4_ERR_MISALIGNED;
    if (injected_failure()) return Q4_ERR_CUDA;
    return from_cuda(quantize_launch(W, w_dtype, n, blocksize, code, packed, absmax, (cudaStream_t)stream));
}

int q4_quantize_blockwise(const float* W, int64_t n, int blocksize, const float* code, uint8_t* packed,
                          float* absmax, void* stream) {
    return q4_quantize_blockwise_ex(W, Q4_FP32, n, blocksize, code, packed, absmax, stream);
}

int q4_dequantize_blockwise(const uint8_t* packed, const float* absmax, const float* code, int64_t n,
                            int blocksize, int out_dtype, void* out, void* stream) {
    if (n < 0 || !is_pow2_blocksize(blocksize)) return Q4_ERR_INVALID_ARG;
    if (out_dtype != Q4_BF16 && out_dtype != Q4_FP16 && out_dtype != Q4_FP32) return Q4_ERR_INVALID_ARG;
    if (n == 0) return Q4_OK;  // empty input: pointers may be NULL
    if (!packed || !absmax || !code || !out) return Q4_ERR_INVALID_ARG;
    if (!aligned(packed, 16) || !aligned(out, 16) || !aligned(absmax, 4) || !aligned(code, 4))
        return Q4_ERR_MISALIGNED;
    if (injected_failure()) return Q4_ERR_CUDA;
    return from_cuda(dequantize_launch(packed, absmax, code, n, blocksize, out_dtype, out, (cudaStream_t)stream));
}

int q4_gemm_plan(int M, int N, int K, int blocksize, int act_dtype, int num_sms, q4_gemm_plan_t* plan) {
    if (!plan) return Q4_ERR_INVALID_ARG;
    GemmChoice ch;
    int tiles = 0, sms = 0;
    int64_t units = 0;
    size_t ws = 0;
    const int rc = gemm_choose(M, N, K, blocksize, act_dtype, num_sms, nullptr, &ch, &tiles, &units, &ws, &sms);
    if (rc != Q4_OK) return rc;
    plan->math = ch.math;
    plan->sub_block = ch.sub_block;
    plan->m_pad = ch.m_pad;
    plan->rows_per_tile = ch.rows_per_tile;
    plan->warps = ch.warps;
    plan->ctas = ch.ctas;
    plan->depth = ch.depth;
    plan->l2_prefetch = ch.l2pf == 0 ? 1 : ch.l2pf;
    plan->loader = ch.loader;
    plan->pdl = ch.pdl;
    plan->tiles = tiles;
    plan->units = units;
    plan->smem_bytes = ch.math == 2 ? simt_smem_bytes() : gemm_smem_bytes(act_dtype, ch);
    plan->workspace_bytes = ws;
    return Q4_OK;
}

int q4_gemm_workspace_size(int M, int N, int K, int blocksize, int act_dtype, size_t* bytes) {
    if (!bytes) return Q4_ERR_INVALID_ARG;
    GemmChoice ch;
    int tiles = 0, sms = 0;
    int64_t units = 0;
    return gemm_choose(M, N, K, blocksize, act_dtype, 0, nullptr, &ch, &tiles, &units, bytes, &sms);
}

int q4_gemm_workspace_size_ex(int M, int N, int K, int blocksize, int act_dtype, const q4_gemm_plan_t* overrides,
                              size_t* bytes) {
    if (!bytes) return Q4_ERR_INVALID_ARG;
    GemmChoice ch;
    int tiles = 0, sms = 0;
    int64_t units = 0;
    return gemm_choose(M, N, K, blocksize, act_dtype, 0, overrides, &ch, &tiles, &units, bytes, &sms);
}

// The fused GEMM behind every entry point; `bias` may be nullptr.
static int gemm_entry(const void* A, const uint8_t* Wpacked, const float* absmax, const float* code, const void* bias,
                      int M, int N, int K, int blocksize, int act_dtype, void* out, void* workspace,
                      size_t workspace_bytes, void* stream, const q4_gemm_plan_t* overrides) {
    // Pointers to empty arrays may be NULL; everything else must be given.
    if (M > 0 && N > 0 && (!out || (K > 0 && (!A || !Wpacked || !absmax || !code)))) return Q4_ERR_INVALID_ARG;
    GemmChoice ch;
    int tiles = 0, sms = 0;
    int64_t units = 0;
    size_t need = 0;
    int rc = gemm_choose(M, N, K, blocksize, act_dtype, 0, overrides, &ch, &tiles, &units, &need, &sms);
    if (rc != Q4_OK) return rc;
    if (M == 0 || N == 0) return Q4_OK;
    if (!aligned(out, 16) || (K > 0 && (!aligned(A, 16) || !aligned(Wpacked, 16) || !aligned(absmax, 4) ||
                                         !aligned(code, 4))) ||
        (bias && !aligned(bias, act_dtype == Q4_FP32 ? 4 : 2)))
        return Q4_ERR_MISALIGNED;
    if (need > 0 && (!workspace || workspace_bytes < need)) return Q4_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 16)) return Q4_ERR_MISALIGNED;
    if (ch.chunk_rows > 0) {
        // Row chunks: each is a call of its own (its own launch-table entry,
        // alignment fallback included) on the rows of A and out it covers,
        // one after another on the caller's stream and workspace.
        const size_t esize = act_dtype == Q4_FP32 ? 4 : 2;
        for (int r0 = 0; r0 < M; r0 += ch.chunk_rows) {
            const int mc = M - r0 < ch.chunk_rows ? M - r0 : ch.chunk_rows;
            rc = gemm_entry(static_cast<const char*>(A) + (size_t)r0 * K * esize, Wpacked, absmax, code, bias, mc, N,
                            K, blocksize, act_dtype, static_cast<char*>(out) + (size_t)r0 * N * esize, workspace,
                            workspace_bytes, stream, overrides);
            if (rc != Q4_OK) return rc;
        }
        return Q4_OK;
    }
    if (ch.math == 3 && !aligned(absmax, 16)) return Q4_ERR_MISALIGNED;  // tensor-map base
    if (ch.math != 3 && ch.loader >= 2 && !aligned(absmax, 16)) {  // the tensor map needs a 16-byte aligned base
        if (overrides && overrides->loader >= 2) return Q4_ERR_MISALIGNED;
        GemmChoice fb;
        q4_gemm_plan_t ov1{};
        if (overrides) ov1 = *overrides;
        ov1.loader = 1;
        ov1.warps = ov1.depth = ov1.l2_prefetch = 0;  // keep ctas and pdl
        rc = gemm_choose(M, N, K, blocksize, act_dtype, 0, &ov1, &fb, &tiles, &units, &need, &sms);
        if (rc != Q4_OK) return rc;
        ch = fb;
    }
    if (injected_failure()) return Q4_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    if (K == 0) {  // empty contraction: every row is the bias, or +0 (all-zero bits in every dtype)
        const size_t esize = act_dtype == Q4_FP32 ? 4 : 2;
        if (!bias) return from_cuda(cudaMemsetAsync(out, 0, (size_t)M * N * esize, st));
        for (int m = 0; m < M; ++m) {
            cudaError_t e = cudaMemcpyAsync(static_cast<char*>(out) + (size_t)m * N * esize, bias, (size_t)N * esize,
                                            cudaMemcpyDeviceToDevice, st);
            if (e != cudaSuccess) return from_cuda(e);
        }
        return Q4_OK;
    }
    GemmParams p{};
    p.A = A;
    p.Wp = Wpacked;
    p.absmax = absmax;
    p.code = code;
    p.out = out;
    p.bias = bias;
    p.error = static_cast<int*>(workspace);
    p.partials = workspace ? reinterpret_cast<float*>(static_cast<char*>(workspace) + kWsHeader) : nullptr;
    p.counters = workspace ? reinterpret_cast<int*>(static_cast<char*>(workspace) + ws_counter_offset(sms)) : nullptr;
    p.M = M;
    p.N = N;
    p.K = K;
    p.kb_per_tile = K / ch.sub_block;
    int sh = 0;
    while ((ch.sub_block << sh) < blocksize) ++sh;
    p.am_shift = sh;
    p.am_per_row = K / blocksize;
    p.pdl = ch.pdl;
    p.tiles = tiles;
    p.ctas = ch.ctas;
    p.units = (uint32_t)units;
    if (ch.math == 2) {
        int lbs = 0;
        while ((1 << lbs) < blocksize) ++lbs;
        return from_cuda(simt_launch(simt_shape(M), ch.ctas, p, lbs, act_dtype, st));
    }
    if (ch.loader == 7) {
        RowsParams rp{};
        rp.A = A;
        rp.out = out;
        rp.bias = bias;
        rp.code = code;
        rp.error = static_cast<int*>(workspace);
        rp.M = M;
        rp.N = N;
        rp.K = K;
        rp.am_shift = sh;
        rp.groups = (N + 7) / 8;
        rp.ctas = ch.ctas;
        rp.pdl = ch.pdl;
        rp.l2_ahead = ch.l2pf;
        rp.contig = ch.depth == 2 ? 1 : 0;
        rp.wait_limit = kWaitLimit;
        rp.skip_stage = -1;
        if (const int skip = injected_stage_skip(); skip >= 0) {
            rp.skip_stage = skip;
            rp.wait_limit = 1u << 14;  // run out within microseconds
        }
        int smem = 0, dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return from_cuda(cudaGetLastError());
        return from_cuda(rows_launch(act_dtype, ch.m_pad, rp, Wpacked, absmax, K / blocksize, smem, st));
    }
    if (ch.math == 3) {
        if (workspace)
            p.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + ws_counter_offset(sms) +
                                                  align_up((size_t)tiles * sizeof(int), 256));
        int smem = 0, dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return from_cuda(cudaGetLastError());
        return from_cuda(umma_launch(act_dtype, ch.m_pad, p, smem, st));
    }
    return from_cuda(gemm_launch(ch, act_dtype, p, st));
}

int q4_gemm_skinny_ex(const void* A, const uint8_t* Wpacked, const float* absmax, const float* code, int M, int N,
                      int K, int blocksize, int act_dtype, void* out, void* workspace, size_t workspace_bytes,
                      void* stream, const q4_gemm_plan_t* overrides) {
    return gemm_entry(A, Wpacked, absmax, code, nullptr, M, N, K, blocksize, act_dtype, out, workspace,
                      workspace_bytes, stream, overrides);
}

int q4_gemm_skinny(const void* A, const uint8_t* Wpacked, const float* absmax, const float* code, int M, int N,
                   int K, int blocksize, int act_dtype, void* out, void* workspace, size_t workspace_bytes,
                   void* stream) {
    return gemm_entry(A, Wpacked, absmax, code, nullptr, M, N, K, blocksize, act_dtype, out, workspace,
                      workspace_bytes, stream, nullptr);
}

int q4_gemm_skinny_bias(const void* A, const uint8_t* Wpacked, const float* absmax, const float* code,
                        const void* bias, int M, int N, int K, int blocksize, int act_dtype, void* out,
                        void* workspace, size_t workspace_bytes, void* stream, const q4_gemm_plan_t* overrides) {
    if (M > 0 && N > 0 && !bias) return Q4_ERR_INVALID_ARG;
    return gemm_entry(A, Wpacked, absmax, code, bias, M, N, K, blocksize, act_dtype, out, workspace,
                      workspace_bytes, stream, overrides);
}

int q4_gemm_route(int M, int N, int K, int blocksize, int act_dtype, int* route) {
    if (!route) return Q4_ERR_INVALID_ARG;
    GemmChoice ch;
    int tiles = 0, sms = 0;
    int64_t units = 0;
    size_t ws = 0;
    // Any positive SM count: the choice of path does not depend on it, and a
    // host-only query must not touch the device.
    const int rc = gemm_choose(M, N, K, blocksize, act_dtype, 148, nullptr, &ch, &tiles, &units, &ws, &sms);
    if (rc == Q4_ERR_UNSUPPORTED) {
        *route = Q4_ROUTE_SPLIT;
        return Q4_OK;
    }
    if (rc != Q4_OK) return rc;
    if (M <= 16 || (ch.math == 1 && ch.chunk_rows == 0)) {  // M <= 16, and 17 <= M <= 32 on the 32-row kernel
        *route = Q4_ROUTE_FUSED;
        return Q4_OK;
    }
    // 33 <= M <= 64 (row chunks on the mma.sync kernels) and the tensor-memory
    // kernel: fused only on layers of 2^26 weights or more
    *route = (M <= 64 && (int64_t)N * K >= ((int64_t)1 << 26)) ? Q4_ROUTE_FUSED : Q4_ROUTE_SPLIT;
    return Q4_OK;
}

// The exported partition functions compute with 64-bit integers; the kernels
// use the 32-bit forms of the same formulas, which agree whenever
// total * parts < 2^32 (the launcher enforces units < 2^23, parts <= 512).
int64_t q4_partition_start(int64_t total, int parts, int part) {
    if (total < 0 || parts <= 0 || part < 0 || part > parts) return -1;
    if (total < (int64_t)kMaxUnits && parts <= 512) return part_start((uint32_t)total, (uint32_t)parts, (uint32_t)part);
    return part_start64(total, parts, part);
}

int q4_partition_owner(int64_t total, int parts, int64_t u) {
    if (total <= 0 || parts <= 0 || u < 0 || u >= total) return -1;
    if (total < (int64_t)kMaxUnits && parts <= 512) return (int)part_owner((uint32_t)total, (uint32_t)parts, (uint32_t)u);
    return part_owner64(total, parts, u);
}

}  // extern "C"
