// q4_quant.cu -- blockwise 4-bit quantize and dequantize kernels.
//
// Dequantize is the building block of the split "dequantize + GEMM" path
// that bitsandbytes PR #1920 ("Fused path support for M > 1") compares the
// fused kernel against; quantize produces the packed format the fused
// kernel reads.  Both are memory-bound streams; both must match the
// definition exactly (codes and absmax equal, dequantized values bit-equal),
// so every floating-point step is an explicitly rounded intrinsic.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "q4_device.cuh"
#include "q4_internal.h"

namespace q4 {

// Index of the nearest code: argmin_j |x - code[j]| on binary32
// differences, lowest j on ties (strict "<" while scanning upward).
__device__ __forceinline__ int nearest_code(float x, const float (&c)[16]) {
    int best = 0;
    float bd = fabsf(__fsub_rn(x, c[0]));
#pragma unroll
    for (int j = 1; j < 16; ++j) {
        const float d = fabsf(__fsub_rn(x, c[j]));
        if (d < bd) {
            bd = d;
            best = j;
        }
    }
    return best;
}

// Weights arrive as fp32, bf16 or fp16; every element is widened to fp32
// exactly, so the quantizer's arithmetic (and result) does not depend on the
// input type.
template <typename TW>
struct WeightIn;
template <>
struct WeightIn<float> {
    __device__ __forceinline__ static float get(const float* p, int64_t i) { return __ldg(p + i); }
    // 16 consecutive elements from a 16-byte aligned address
    __device__ __forceinline__ static void get16(const float* p, float (&f)[16]) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const uint4 u = ldg_stream_v4(p + 4 * v);
            f[4 * v] = __uint_as_float(u.x);
            f[4 * v + 1] = __uint_as_float(u.y);
            f[4 * v + 2] = __uint_as_float(u.z);
            f[4 * v + 3] = __uint_as_float(u.w);
        }
    }
};
template <typename H, float (*TO_F)(H)>
struct WeightIn16 {
    __device__ __forceinline__ static float get(const H* p, int64_t i) {
        const unsigned short b = __ldg(reinterpret_cast<const unsigned short*>(p) + i);
        return TO_F(*reinterpret_cast<const H*>(&b));
    }
    __device__ __forceinline__ static void get16(const H* p, float (&f)[16]) {
#pragma unroll
        for (int v = 0; v < 2; ++v) {
            const uint4 u = ldg_stream_v4(p + 8 * v);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const unsigned short lo = (unsigned short)(w[k] & 0xFFFFu), hi = (unsigned short)(w[k] >> 16);
                f[8 * v + 2 * k] = TO_F(*reinterpret_cast<const H*>(&lo));
                f[8 * v + 2 * k + 1] = TO_F(*reinterpret_cast<const H*>(&hi));
            }
        }
    }
};
__device__ __forceinline__ float bf16_to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float f16_to_f(__half v) { return __half2float(v); }
template <>
struct WeightIn<__nv_bfloat16> : WeightIn16<__nv_bfloat16, bf16_to_f> {};
template <>
struct WeightIn<__half> : WeightIn16<__half, f16_to_f> {};

// One warp per block of `bs` elements (grid-stride over the blocks from
// `b0`).  Pairs of elements map to one output byte (even element -> high
// nibble); blocks start at even indices because bs is even, so pairs never
// straddle blocks.  Serves any blocksize and the ragged end of the input.
template <typename TW>
__device__ __forceinline__ void quantize_blocks_per_warp(const TW* __restrict__ W, int64_t n, int bs_shift,
                                                         const float (&c)[16], uint8_t* __restrict__ packed,
                                                         float* __restrict__ absmax, int64_t b0, int64_t nblocks) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t b = b0 + (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5); b < nblocks; b += nwarps) {
        const int64_t lo = b << bs_shift;
        const int64_t rem = n - lo;
        const int cnt = rem < ((int64_t)1 << bs_shift) ? (int)rem : (1 << bs_shift);
        const TW* wb = W + lo;
        float amax = 0.f;
        for (int i = lane; i < cnt; i += 32) amax = fmaxf(amax, fabsf(WeightIn<TW>::get(wb, i)));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) absmax[b] = amax;
        for (int p = lane; 2 * p < cnt; p += 32) {
            const bool has1 = 2 * p + 1 < cnt;
            const float w0 = WeightIn<TW>::get(wb, 2 * p);
            const float w1 = has1 ? WeightIn<TW>::get(wb, 2 * p + 1) : 0.f;
            const int i0 = nearest_code(amax > 0.f ? __fdiv_rn(w0, amax) : 0.f, c);
            const int i1 = has1 ? nearest_code(amax > 0.f ? __fdiv_rn(w1, amax) : 0.f, c) : 0;
            packed[(lo >> 1) + p] = (uint8_t)((i0 << 4) | i1);
        }
    }
}

template <typename TW>
__global__ void __launch_bounds__(256) q4_quantize_kernel(const TW* __restrict__ W, int64_t n, int bs_shift,
                                                          const float* __restrict__ code,
                                                          uint8_t* __restrict__ packed,
                                                          float* __restrict__ absmax, int64_t nblocks) {
    float c[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) c[j] = __ldg(code + j);
    quantize_blocks_per_warp<TW>(W, n, bs_shift, c, packed, absmax, 0, nblocks);
}

// Blocksizes 32..512: a warp takes 512-element chunks, each lane 16
// consecutive elements (vector loads, one 8-byte packed store; a warp writes
// 256 contiguous bytes).  The bs/16 lanes of a block reduce its absmax with
// shuffles; 16 independent elements per lane keep the division and the
// 16-way search in flight.  Elements after the last whole chunk (whole blocks,
// since 512 is a multiple of bs) go through the per-warp form.
template <typename TW>
__global__ void __launch_bounds__(256) q4_quantize_lanes_kernel(const TW* __restrict__ W, int64_t n, int bs_shift,
                                                                const float* __restrict__ code,
                                                                uint8_t* __restrict__ packed,
                                                                float* __restrict__ absmax, int64_t nblocks) {
    float c[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) c[j] = __ldg(code + j);
    const int lane = threadIdx.x & 31;
    const int group = 1 << (bs_shift - 4);  // lanes per block: 2 .. 32
    const int64_t nchunks = n >> 9;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; q < nchunks; q += nwarps) {
        const int64_t e0 = (q << 9) + 16 * lane;
        float f[16];
        WeightIn<TW>::get16(W + e0, f);
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
        for (int off = 1; off < group; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if ((lane & (group - 1)) == 0) absmax[e0 >> bs_shift] = amax;
        uint32_t word[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint32_t idx = (uint32_t)nearest_code(amax > 0.f ? __fdiv_rn(f[e], amax) : 0.f, c);
            // byte e/2 of the lane's 8 output bytes; even element in the high nibble
            word[e >> 3] |= idx << (8 * ((e >> 1) & 3) + ((e & 1) ? 0 : 4));
        }
        *reinterpret_cast<uint2*>(packed + (e0 >> 1)) = make_uint2(word[0], word[1]);
    }
    quantize_blocks_per_warp<TW>(W, n, bs_shift, c, packed, absmax, (nchunks << 9) >> bs_shift, nblocks);
}

template <int OUT>
struct DequantOut;

template <>
struct DequantOut<0> {  // bf16
    __device__ __forceinline__ static uint32_t pair(float a, float b) { return Act<__nv_bfloat16>::pack(a, b); }
    __device__ __forceinline__ static void one(void* out, int64_t i, float v) {
        static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
    }
};

template <>
struct DequantOut<1> {  // fp16
    __device__ __forceinline__ static uint32_t pair(float a, float b) { return Act<__half>::pack(a, b); }
    __device__ __forceinline__ static void one(void* out, int64_t i, float v) {
        static_cast<__half*>(out)[i] = __float2half_rn(v);
    }
};

// Writes dominate (2 or 4 output bytes per 0.5 input byte), so every store
// is a contiguous 16-byte piece of a warp-wide run: a warp takes 1024-element
// chunks, and in quarter w lane t dequantizes elements 256w + 8t .. +8 from
// the 4 packed bytes at 128w + 4t (one 128-byte load per quarter, 512 or
// 1024 contiguous output bytes per store instruction).  An 8-element run
// never straddles an absmax block because blocksize is a multiple of 32.
// Elements past the last whole chunk go 32 per thread, then one per thread.
template <int OUT>
__global__ void __launch_bounds__(256) q4_dequant_kernel(const uint8_t* __restrict__ packed,
                                                         const float* __restrict__ absmax,
                                                         const float* __restrict__ code, int64_t n, int bs_shift,
                                                         void* __restrict__ out) {
    __shared__ float sc[16];  // 16 entries in 16 banks: lookups never conflict
    if (threadIdx.x < 16) sc[threadIdx.x] = code[threadIdx.x];
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
    const int64_t nwchunks = n >> 10;
    for (int64_t q = tid >> 5; q < nwchunks; q += nthreads >> 5) {
        uint32_t words[4];
        float am[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            words[w] = ldg_stream_u32(packed + (q << 9) + 128 * w + 4 * lane);
            am[w] = __ldg(absmax + (((q << 10) + 256 * w + 8 * lane) >> bs_shift));
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int64_t e0 = (q << 10) + 256 * w + 8 * lane;  // first of this lane's 8 elements
            if constexpr (OUT == 2) {
                float f[8];
#pragma unroll
                for (int by = 0; by < 4; ++by) {
                    const uint32_t b = (words[w] >> (8 * by)) & 0xFFu;
                    f[2 * by] = __fmul_rn(sc[b >> 4], am[w]);
                    f[2 * by + 1] = __fmul_rn(sc[b & 15u], am[w]);
                }
                float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + e0);
                o[0] = make_float4(f[0], f[1], f[2], f[3]);
                o[1] = make_float4(f[4], f[5], f[6], f[7]);
            } else {
                uint32_t r[4];
#pragma unroll
                for (int by = 0; by < 4; ++by) {
                    const uint32_t b = (words[w] >> (8 * by)) & 0xFFu;
                    r[by] = DequantOut<OUT>::pair(__fmul_rn(sc[b >> 4], am[w]), __fmul_rn(sc[b & 15u], am[w]));
                }
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + e0) = make_uint4(r[0], r[1], r[2], r[3]);
            }
        }
    }
    // Whole 32-element chunks after the last 1024-element chunk.
    const int64_t c0 = nwchunks << 5, nchunks = n >> 5;
    const int64_t t0 = tid;
    const int64_t stride = nthreads;
    for (int64_t q = c0 + t0; q < nchunks; q += stride) {
        const uint4 v = ldg_stream_v4(packed + 16 * q);
        const float am = __ldg(absmax + ((q << 5) >> bs_shift));
        const uint32_t words[4] = {v.x, v.y, v.z, v.w};
        if constexpr (OUT == 2) {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + (q << 5));
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                float f[8];
#pragma unroll
                for (int by = 0; by < 4; ++by) {
                    const uint32_t b = (words[w] >> (8 * by)) & 0xFFu;
                    f[2 * by] = __fmul_rn(sc[b >> 4], am);
                    f[2 * by + 1] = __fmul_rn(sc[b & 15u], am);
                }
                o[2 * w] = make_float4(f[0], f[1], f[2], f[3]);
                o[2 * w + 1] = make_float4(f[4], f[5], f[6], f[7]);
            }
        } else {
            uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + (q << 5));
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t r[4];
#pragma unroll
                for (int by = 0; by < 4; ++by) {
                    const uint32_t b = (words[w] >> (8 * by)) & 0xFFu;
                    r[by] = DequantOut<OUT>::pair(__fmul_rn(sc[b >> 4], am), __fmul_rn(sc[b & 15u], am));
                }
                o[w] = make_uint4(r[0], r[1], r[2], r[3]);
            }
        }
    }
    // Ragged tail (n % 32 elements): one element per thread.
    for (int64_t i = (nchunks << 5) + t0; i < n; i += stride) {
        const uint32_t byte = packed[i >> 1];
        const uint32_t idx = (i & 1) ? (byte & 15u) : (byte >> 4);
        const float v = __fmul_rn(sc[idx], __ldg(absmax + (i >> bs_shift)));
        if constexpr (OUT == 2)
            static_cast<float*>(out)[i] = v;
        else
            DequantOut<OUT>::one(out, i, v);
    }
}

static int log2_exact(int v) {
    int s = 0;
    while ((1 << s) < v) ++s;
    return s;
}

static int grid_for(int64_t work_items, int threads, int per_sm) {
    int sms = 148;
    device_sm_count(&sms);
    int64_t blocks = (work_items + threads - 1) / threads;
    const int64_t cap = (int64_t)sms * per_sm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

cudaError_t quantize_launch(const void* W, int w_dtype, int64_t n, int blocksize, const float* code,
                            uint8_t* packed, float* absmax, cudaStream_t stream) {
    const int64_t nblocks = (n + blocksize - 1) / blocksize;
    const int threads = 256;
    const int sh = log2_exact(blocksize);
    // The lane-per-16-elements form needs bs <= 512 and an 8-byte aligned
    // packed array (its stores are 8 bytes wide).
    const bool lanes = blocksize <= 512 && (reinterpret_cast<uintptr_t>(packed) & 7u) == 0;
    // one warp per 512-element chunk (plus the tail's blocks), or per block
    const int64_t warps = lanes ? (n >> 9) + (512 >> sh) : nblocks;
    const int grid = grid_for(warps * 32, threads, 8);
#define Q4_QUANT(TW)                                                                                              \
    do {                                                                                                          \
        if (lanes)                                                                                                \
            q4_quantize_lanes_kernel<TW><<<grid, threads, 0, stream>>>(static_cast<const TW*>(W), n, sh, code,  \
                                                                       packed, absmax, nblocks);                 \
        else                                                                                                      \
            q4_quantize_kernel<TW><<<grid, threads, 0, stream>>>(static_cast<const TW*>(W), n, sh, code, packed, \
                                                                 absmax, nblocks);                               \
    } while (0)
    if (w_dtype == 0)
        Q4_QUANT(__nv_bfloat16);
    else if (w_dtype == 1)
        Q4_QUANT(__half);
    else
        Q4_QUANT(float);
#undef Q4_QUANT
    return cudaGetLastError();
}

cudaError_t dequantize_launch(const uint8_t* packed, const float* absmax, const float* code, int64_t n,
                              int blocksize, int out_dtype, void* out, cudaStream_t stream) {
    const int threads = 256;
    const int64_t items = (n >> 5) > 0 ? (n >> 5) : 1;
    const int grid = grid_for(items, threads, 8);
    const int sh = log2_exact(blocksize);
    if (out_dtype == 0)
        q4_dequant_kernel<0><<<grid, threads, 0, stream>>>(packed, absmax, code, n, sh, out);
    else if (out_dtype == 1)
        q4_dequant_kernel<1><<<grid, threads, 0, stream>>>(packed, absmax, code, n, sh, out);
    else
        q4_dequant_kernel<2><<<grid, threads, 0, stream>>>(packed, absmax, code, n, sh, out);
    return cudaGetLastError();
}

}  // namespace q4
