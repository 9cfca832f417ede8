// q4_simt.cu -- fused blockwise 4-bit dequantize + skinny GEMM on the CUDA
// cores, for sm_100a:
//
//     out[m, n] = [bias[n]] + sum_k A[m, k] * code[idx(n, k)] * absmax(n, k)
//     M <= 16; A / out / bias fp32, or bf16 / fp16.
//
// The maintainer's reply in bitsandbytes PR #1920 ("[ROCm] Optimize
// kgemm_4bit_inference_naive ...") describes the replacement kernels: a SIMT
// kernel for the smallest batches and tensor-core (MMA) versions past them,
// the SIMT kernel also taking fp32, all accumulating in fp32.  This is the
// SIMT kernel.  Every product is an fp32 FMA of the activation (16-bit
// activations widened exactly) with the exact fp32 code value; nothing is
// rounded to 16 bits before the single rounding of the output.  For 16-bit
// activations the launch table keeps the tensor-core kernels (measured
// faster at every M); this kernel serves them on request (math = 2).
//
// Design for B200:
//  * HBM-bound at M = 1 (0.5625 B per weight at blocksize 64), so the code
//    bytes stream through registers with coalesced 4-byte loads per lane and
//    row (128 B per warp instruction), the next unit in flight while one is
//    computed.  (Deeper register rings with fewer warps measured slower: the
//    loop is bound by instruction latency, which more warps hide better.)
//  * Dequantization is one shared-memory lookup per packed BYTE: a 256-row
//    table maps a byte to the float2 (code[hi], code[lo]).  Each 256-B row
//    holds 16 copies of the pair, one per bank pair, so a half-warp's 64-bit
//    lookups never conflict; the table sits on a 64 KiB boundary of the
//    shared window, so one byte-permute turns a packed word into the lookup
//    address (table base | byte << 8 | copy << 3).
//  * A lane covers 8 consecutive k of a row in each 256-k group: the 8
//    weights lie in one absmax block (blocksize >= 32), so the block scale is
//    applied once per 8 products (acc += absmax * t).
//  * Work units of R rows x 512 k are split evenly over all warps of the grid
//    (stream-K at warp granularity): every warp streams the same number of
//    weight bytes to within one unit.  A row group cut by a warp boundary is
//    combined deterministically through the GEMM workspace: each piece is
//    published with a release add on the group's counter, and the last
//    arriver sums the pieces in warp order.  No thread ever waits on another.
#include <cuda_runtime.h>
#include <stdint.h>

#include "q4_device.cuh"
#include "q4_internal.h"
#include "q4_plan.cuh"

namespace q4 {
namespace simt {

static constexpr int kUnitK = 512;                    // k-width of a work unit (two 256-k groups)
static constexpr uint32_t kTableBytes = 256u * 256u;  // 256 rows of 256 B (lower 128 B used)
// Dynamic shared memory: the device's opt-in maximum (the table on a 64 KiB
// boundary, the warps' copy rings below and above it).
static int max_smem() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return v;
}

struct Params {
    const void* A;         // [M, K] activations: fp32, or bf16/fp16 (widened exactly to fp32 on load)
    const uint8_t* Wp;     // [N, K/2]
    const float* absmax;   // [N * K / blocksize]
    const float* code;     // [16]
    void* out;             // [M, N] in the activation type
    const void* bias;      // [N] in the activation type, or nullptr
    float* partials;       // [warps][2][R * MP]
    int* counters;         // [row groups], zero between calls
    int M, N, K;
    int lbs;               // log2(blocksize)
    int ku;                // units per row group: ceil(K / 512)
    int row_groups;
    int pdl;               // 0, 1: wait before any global access; 2: code/weights/absmax first
    uint32_t units;        // row_groups * ku
    uint32_t warps;        // grid warps
    int narrow;            // units * warps < 2^32: the partition in 32-bit arithmetic
    int a32;               // A is 32-byte aligned: 256-bit activation loads
    int* error;            // workspace error word (set to 2 when shared memory is short), or nullptr
};

// First unit of part `p` when `total` units are split into `parts` ranges,
// and the part owning unit `u` (the formulas of q4_partition_start/_owner).
// `narrow`: total * parts < 2^32, so 32-bit arithmetic is exact.
__host__ __device__ __forceinline__ uint32_t wpart_start(uint32_t total, uint32_t parts, uint32_t p, bool narrow) {
    return narrow ? (total * p) / parts : (uint32_t)(((uint64_t)total * p) / parts);
}
__host__ __device__ __forceinline__ uint32_t wpart_owner(uint32_t total, uint32_t parts, uint32_t u, bool narrow) {
    return narrow ? ((u + 1) * parts - 1) / total : (uint32_t)((((uint64_t)u + 1) * parts - 1) / total);
}

// The loads below read data that no thread writes while the kernel runs (the
// table is complete before the first lookup), so they are plain asm the
// compiler may schedule freely.  Float pairs travel as 64-bit registers
// (first value in the low half), the operand form of fma.rn.f32x2.
__device__ __forceinline__ uint64_t lds_pair(uint32_t addr) {
    uint64_t v;
    asm("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(addr));
    return v;
}

// Four consecutive floats as two pairs (16-byte aligned).
__device__ __forceinline__ void ldg_pairs(const float* p, uint64_t& lo, uint64_t& hi) {
    asm("ld.global.nc.v2.b64 {%0, %1}, [%2];" : "=l"(lo), "=l"(hi) : "l"(p));
}

// Eight consecutive floats as four pairs in one 256-bit load (32-byte aligned).
__device__ __forceinline__ void ldg_pairs8(const float* p, uint64_t (&v)[4]) {
    asm("ld.global.nc.v4.b64 {%0, %1, %2, %3}, [%4];" : "=l"(v[0]), "=l"(v[1]), "=l"(v[2]), "=l"(v[3]) : "l"(p));
}

__device__ __forceinline__ uint32_t ldg_code_word(const uint8_t* p) {
    uint32_t v;
    asm("ld.global.nc.L1::no_allocate.b32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ float ldg_scale(const float* p) {
    float v;
    asm("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// An opaque copy of `v`: values derived from it cannot be computed before
// this point of the program (an ordering fence for the plain-asm loads).
template <typename V>
__device__ __forceinline__ void launder(V& v) {
    static_assert(sizeof(V) == 4 || sizeof(V) == 8, "32- or 64-bit values");
    if constexpr (sizeof(V) == 8)
        asm volatile("" : "+l"(v)::"memory");
    else
        asm volatile("" : "+r"(v)::"memory");
}

// d = a * b on both halves, each rounded once.
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// d = a * b + c on both halves, each an fp32 FMA rounded once.
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ float lo_f32(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi_f32(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }

// Byte BYTE of `word` -> the table pair (code[hi nibble], code[lo nibble]) of
// that byte, from this lane's copy.
template <int BYTE>
__device__ __forceinline__ uint64_t pair_of(uint32_t word, uint32_t lane8) {
    // result bytes: [0] = lane8.b0 (copy * 8), [1] = word.b<BYTE>, [2..3] = table base >> 16
    return lds_pair(prmt<0x7604u | (BYTE << 4)>(word, lane8));
}

// Asynchronous copies into the warp's shared-memory ring (the copy bytes
// beyond src_size are zero-filled, so rows past N and k past K read nothing).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_size) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_size) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t src_size) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_size) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Ring slot of one unit: R rows x 256 B of packed codes (row r, group q at
// r * 256 + q * 128), then R rows x 16 floats of absmax (the unit's blocks,
// 512 / blocksize of them, at least 1).
template <int R>
struct Slot {
    static constexpr uint32_t CODES = (uint32_t)R * 256u;
    static constexpr uint32_t BYTES = CODES + (uint32_t)R * 64u;
};

static constexpr int kErrNoRoom = 2;

// Activation types: fp32 as given; bf16 / fp16 widened exactly to fp32
// (four pairs from one 16-byte load), the output rounded once to the type.
template <typename TA>
struct ActIO;
template <>
struct ActIO<float> {
    __device__ __forceinline__ static float widen(float v) { return v; }
    __device__ __forceinline__ static float narrow(float v) { return v; }
};
template <>
struct ActIO<__nv_bfloat16> {
    __device__ __forceinline__ static float widen(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ __forceinline__ static __nv_bfloat16 narrow(float v) { return __float2bfloat16_rn(v); }
    // packed pair (first value in the low half) -> the float pair, exactly
    __device__ __forceinline__ static uint64_t pair(uint32_t w) {
        return (uint64_t)(w << 16) | ((uint64_t)(w & 0xFFFF0000u) << 32);
    }
};
template <>
struct ActIO<__half> {
    __device__ __forceinline__ static float widen(__half v) { return __half2float(v); }
    __device__ __forceinline__ static __half narrow(float v) { return __float2half_rn(v); }
    __device__ __forceinline__ static uint64_t pair(uint32_t w) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
        return (uint64_t)__float_as_uint(f.x) | ((uint64_t)__float_as_uint(f.y) << 32);
    }
};

template <typename TA, int MP, int R, int NW, int D>
__global__ void __launch_bounds__(NW * 32, 1) q4_gemm_f32_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t sbase = smem_addr(smem);
    const uint32_t table = (sbase + 0xFFFFu) & ~0xFFFFu;  // 64 KiB aligned (the host reserves the padding)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t lane8 = table | ((uint32_t)(lane & 15) << 3);
    const uint8_t* Wp = p.Wp;
    const float* absmax = p.absmax;
    const TA* Aact = static_cast<const TA*>(p.A);

    if (p.pdl != 2) griddep_wait();
    // The loads are plain asm the compiler may move: each one takes its
    // address from a value laundered after the point it must follow.
    launder(Wp);
    launder(absmax);
    // Table: row b = 16 copies of (code[b >> 4], code[b & 15]); the pair is
    // gathered by shuffles from one global load per thread.
    {
        const float cv = __ldg(p.code + (lane & 15));
        for (int e = tid; e < 256 * 8; e += NW * 32) {
            const int b = e >> 3;
            const float hi = __shfl_sync(0xffffffffu, cv, b >> 4);
            const float lo = __shfl_sync(0xffffffffu, cv, b & 15);
            sts_v4(table + (uint32_t)b * 256u + (uint32_t)(e & 7) * 16u, __float_as_uint(hi), __float_as_uint(lo),
                   __float_as_uint(hi), __float_as_uint(lo));
        }
    }

    // Ring slots: NW * D of them, below and above the table.
    using SL = Slot<R>;
    const uint32_t send = sbase + dynamic_smem_size();
    const uint32_t a0s = sbase, b0s = table + kTableBytes;
    const uint32_t na = (table - a0s) / SL::BYTES;
    const uint32_t nb = send > b0s ? (send - b0s) / SL::BYTES : 0u;
    if (na + nb < (uint32_t)(NW * D)) {  // uniform over the CTA: the host sized the launch wrongly
        if (tid == 0 && p.error) atomicExch(p.error, kErrNoRoom);
        return;
    }
    auto slot_addr = [&](int idx) -> uint32_t {
        return (uint32_t)idx < na ? a0s + (uint32_t)idx * SL::BYTES : b0s + ((uint32_t)idx - na) * SL::BYTES;
    };

    const uint32_t gw = blockIdx.x * NW + warp;
    const bool narrow = p.narrow != 0;
    auto start_of = [&](uint32_t w) { return wpart_start(p.units, p.warps, w, narrow); };
    const uint32_t ws = start_of(gw), we = start_of(gw + 1);
    const size_t row_bytes = (size_t)p.K >> 1;
    const int am_row = p.K >> p.lbs;

    // Position of a unit: row group and unit column inside it.
    struct Cursor {
        uint32_t rg;
        int kc;
    };
    auto advance = [&](Cursor& c) {
        if (++c.kc == p.ku) {
            c.kc = 0;
            ++c.rg;
        }
    };
    Cursor lc{0u, 0}, cc{0u, 0};
    if (ws < we) {
        lc.rg = cc.rg = ws / (uint32_t)p.ku;
        lc.kc = cc.kc = (int)(ws - lc.rg * (uint32_t)p.ku);
    }

    // Copies the packed words and absmax of the unit at `c` into ring slot
    // `st` and commits them as one group (an empty group past the range).
    const int lnab = p.lbs < 9 ? 9 - p.lbs : 0;  // log2 of the absmax values per row and unit (512 / bs, at least 1)
    const int nab = 1 << lnab;
    auto issue = [&](bool valid, const Cursor& c, uint32_t st) {
        if (valid) {
            const int n0 = (int)c.rg * R;
            const int k0 = c.kc * kUnitK;
            // codes: R x 256 B = R x 16 chunks of 16 B; lane l copies chunks l, l + 32, ...
            // (rows lane / 16 + 2 i, bytes 16 (lane % 16) of the row's 256)
            const int r0 = lane >> 4, cb = (lane & 15) * 16;
            const bool kok = k0 + 2 * cb < p.K;   // the chunk's 32 k lie inside the row (K % 32 == 0)
            const uint8_t* wsrc = Wp + (size_t)(n0 + r0) * row_bytes + (k0 >> 1) + cb;
            const uint32_t wdst = st + (uint32_t)(r0 * 256 + cb);
#pragma unroll
            for (int i = 0; i < R / 2; ++i) {
                const bool ok = kok && (n0 + r0 + 2 * i < p.N);
                // R rows of K/2 bytes stay below 2^32 bytes (K < 2^29): 32-bit row offsets
                cp_async16(wdst + (uint32_t)(512 * i), ok ? wsrc + (uint32_t)(2 * i) * (uint32_t)row_bytes : Wp,
                           ok ? 16u : 0u);
            }
            // absmax: R rows x nab values; lane l copies values l, l + 32, ...
            for (int v = lane; v < R * nab; v += 32) {
                const int r = v >> lnab, j = v & (nab - 1);
                const int kb = k0 + (j << p.lbs);       // first k of block j of the unit
                const bool ok = (n0 + r < p.N) && (kb < p.K);
                const float* src = ok ? absmax + (size_t)(n0 + r) * am_row + (kb >> p.lbs) : absmax;
                cp_async4(st + SL::CODES + (uint32_t)(r * 64 + 4 * j), src, ok ? 4u : 0u);
            }
        }
        cp_async_commit();
    };

    // Units ws .. we-1 go through slots warp * D + (u - ws) % D; D - 1 are
    // copied ahead of the one being computed.
    const int slot0 = warp * D;
#pragma unroll
    for (int i = 0; i < D - 1; ++i) {
        issue(ws + i < we, lc, slot_addr(slot0 + i));
        if (ws + i < we) advance(lc);
    }
    __syncthreads();  // the table is complete
    launder(lane8);   // every lookup address derives from lane8: none moves above the barrier
    // Activations, outputs and the workspace may belong to the preceding
    // grid: touch them only after the dependency wait.
    if (p.pdl == 2) griddep_wait();
    launder(Aact);  // activations only after the dependency wait
    griddep_launch_dependents();
    if (ws >= we) {
        cp_async_wait<0>();
        return;
    }

    float acc[R][MP];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MP; ++m) acc[r][m] = 0.f;

    // acc += this lane's share of the unit at `c`: per 256-k group, 8
    // consecutive k of every row, scaled once by that block's absmax.
    auto compute = [&](const Cursor& c, uint32_t st) {
        const int k0 = c.kc * kUnitK;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int kq = k0 + 256 * q + 8 * lane;
            if (kq >= p.K) continue;  // only in the last unit of a row, K % 512 != 0
            // The 8 activations of every row m: pairs (k, k+1), (k+2, k+3), ...
            uint64_t a[MP][4];
#pragma unroll
            for (int m = 0; m < MP; ++m) {
                if (m < p.M) {
                    const TA* src = Aact + (size_t)m * p.K + kq;
                    if constexpr (sizeof(TA) == 2) {
                        const uint4 v = ldg_v4(src);  // 8 values, 16-byte aligned (K % 32 == 0, A 16-byte aligned)
                        a[m][0] = ActIO<TA>::pair(v.x);
                        a[m][1] = ActIO<TA>::pair(v.y);
                        a[m][2] = ActIO<TA>::pair(v.z);
                        a[m][3] = ActIO<TA>::pair(v.w);
                    } else if (p.a32) {
                        ldg_pairs8(reinterpret_cast<const float*>(src), a[m]);
                    } else {
                        ldg_pairs(reinterpret_cast<const float*>(src), a[m][0], a[m][1]);
                        ldg_pairs(reinterpret_cast<const float*>(src) + 4, a[m][2], a[m][3]);
                    }
                } else {
                    a[m][0] = a[m][1] = a[m][2] = a[m][3] = 0ull;
                }
            }
            // this lane's word of every row, and the absmax of the block it lies in
            uint32_t wq[R];
            float amq[R];
            const uint32_t aj = (uint32_t)((256 * q + 8 * lane) >> p.lbs);  // block index inside the unit
#pragma unroll
            for (int r = 0; r < R; ++r) {
                wq[r] = lds_u32(st + (uint32_t)(r * 256 + q * 128 + 4 * lane));
                amq[r] = lds_f32(st + SL::CODES + (uint32_t)(r * 64) + 4u * aj);
            }
            // Two running sums per (row, m): even and odd k of the pairs.
            uint64_t t[R][MP];
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // byte j of the word: k = kq + 2j, kq + 2j + 1
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const uint64_t cp = j == 0   ? pair_of<0>(wq[r], lane8)
                                        : j == 1 ? pair_of<1>(wq[r], lane8)
                                        : j == 2 ? pair_of<2>(wq[r], lane8)
                                                 : pair_of<3>(wq[r], lane8);
#pragma unroll
                    for (int m = 0; m < MP; ++m) t[r][m] = j == 0 ? mul2(a[m][0], cp) : fma2(a[m][j], cp, t[r][m]);
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int m = 0; m < MP; ++m) {
                    acc[r][m] = fmaf(amq[r], lo_f32(t[r][m]), acc[r][m]);
                    acc[r][m] = fmaf(amq[r], hi_f32(t[r][m]), acc[r][m]);
                }
        }
    };

    // Output element e = m * R + r of row group rg (lane e % 32 writes it).
    auto store = [&](uint32_t rg, int e, float v) {
        const int r = e % R, m = e / R;
        const int n = (int)rg * R + r;
        if (n < p.N && m < p.M) {
            const TA* bias = static_cast<const TA*>(p.bias);
            static_cast<TA*>(p.out)[(size_t)m * p.N + n] = ActIO<TA>::narrow(bias ? v + ActIO<TA>::widen(bias[n]) : v);
        }
    };
    constexpr int RM = R * MP;

    // Closes row group `rg` after this warp's last unit of it.
    auto finish = [&](uint32_t rg) {
        // Sum over lanes; the butterfly leaves the same total in every lane
        // (each step adds the same two values, in either order).
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MP; ++m) {
                float v = acc[r][m];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                acc[r][m] = v;
            }
        const uint32_t g0 = rg * (uint32_t)p.ku, g1 = g0 + (uint32_t)p.ku;
        if (ws <= g0 && we >= g1) {  // the whole group is this warp's
#pragma unroll
            for (int e = 0; e < RM; ++e)
                if ((e & 31) == lane) store(rg, e, acc[e % R][e / R]);
        } else {
            // Publish this warp's piece (slot 0: the group is the range's
            // first; 1: its last) and count it in.
            const uint32_t slot = ws >= g0 ? 0u : 1u;
            float* mine = p.partials + ((size_t)gw * 2 + slot) * RM;
#pragma unroll
            for (int e = 0; e < RM; ++e)
                if ((e & 31) == lane) mine[e] = acc[e % R][e / R];
            __syncwarp();
            int prev = 0;
            if (lane == 0) prev = atom_add_acq_rel_gpu(p.counters + rg, 1);
            prev = __shfl_sync(0xffffffffu, prev, 0);
            __syncwarp();
            // Contributors: the warps whose ranges meet the group.  With more
            // warps than units some ranges are empty; they own no unit and
            // publish nothing.
            const uint32_t cf = wpart_owner(p.units, p.warps, g0, narrow);
            const uint32_t cl = wpart_owner(p.units, p.warps, g1 - 1, narrow);
            uint32_t pieces = 0;
            for (uint32_t c = cf, c0 = start_of(cf); c <= cl; ++c) {
                const uint32_t c1 = start_of(c + 1);
                pieces += c0 != c1 ? 1u : 0u;
                c0 = c1;
            }
            if ((uint32_t)prev + 1u == pieces) {  // last to arrive: sum the pieces in warp order
                // lane e (and e + 32) sums output element e over the pieces
                float v0 = 0.f, v1 = 0.f;
                for (uint32_t c = cf, c0 = start_of(cf); c <= cl; ++c) {
                    const uint32_t c1 = start_of(c + 1);
                    if (c0 != c1) {
                        const float* src = p.partials + ((size_t)c * 2 + (c0 >= g0 ? 0u : 1u)) * RM;
                        if (lane < RM) v0 += ldg_cg_f32(src + lane);
                        if (RM > 32 && lane + 32 < RM) v1 += ldg_cg_f32(src + lane + 32);
                    }
                    c0 = c1;
                }
                if (lane < RM) store(rg, lane, v0);
                if (RM > 32 && lane + 32 < RM) store(rg, lane + 32, v1);
                if (lane == 0) p.counters[rg] = 0;  // back to zero for the next call
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int m = 0; m < MP; ++m) acc[r][m] = 0.f;
    };
    auto step = [&](uint32_t st, bool last_of_range) {
        compute(cc, st);
        if (cc.kc == p.ku - 1 || last_of_range) finish(cc.rg);
        advance(cc);
    };

    for (uint32_t u = ws; u < we; ++u) {
        const int i = (int)(u - ws);
        cp_async_wait<D - 2>();  // this unit's group is complete (one group is committed per unit)
        __syncwarp();            // and visible to every lane (lanes read words other lanes copied)
        issue(u + D - 1 < we, lc, slot_addr(slot0 + (i + D - 1) % D));  // refills the slot computed last
        if (u + D - 1 < we) advance(lc);
        step(slot_addr(slot0 + i % D), u + 1 == we);
    }
    cp_async_wait<0>();
}

// Compiled variants: MP = padded M, R = rows per unit, NW = warps per CTA,
// D = register buffers per warp.
template <typename TA, int MP, int R, int NW, int D>
static cudaError_t launch_variant(const Params& p, int ctas, cudaStream_t stream) {
    auto kern = q4_gemm_f32_kernel<TA, MP, R, NW, D>;
    const int smem = max_smem();
    if (smem <= 0) return cudaErrorInvalidValue;
    cudaError_t e = ensure_smem_attr((const void*)kern, (size_t)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(NW * 32);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace simt

// Launch-table shape of the fp32 kernel for a padded M.
SimtShape simt_shape(int M) {
    if (M <= 1) return {1, 8, 16};
    if (M <= 2) return {2, 8, 8};
    if (M <= 4) return {4, 8, 8};
    if (M <= 8) return {8, 4, 8};
    return {16, 2, 8};
}

size_t simt_smem_bytes() { return (size_t)simt::max_smem(); }

template <typename TA>
static cudaError_t simt_launch_t(const SimtShape& sh, int ctas, const simt::Params& p, cudaStream_t stream) {
    switch (sh.m_pad) {
        case 1: return simt::launch_variant<TA, 1, 8, 16, 4>(p, ctas, stream);
        case 2: return simt::launch_variant<TA, 2, 8, 8, 4>(p, ctas, stream);
        case 4: return simt::launch_variant<TA, 4, 8, 8, 4>(p, ctas, stream);
        case 8: return simt::launch_variant<TA, 8, 4, 8, 4>(p, ctas, stream);
        case 16: return simt::launch_variant<TA, 16, 2, 8, 4>(p, ctas, stream);
        default: return cudaErrorInvalidConfiguration;
    }
}

cudaError_t simt_launch(const SimtShape& sh, int ctas, const GemmParams& g, int log2_bs, int act_dtype,
                        cudaStream_t stream) {
    simt::Params p{};
    p.A = g.A;
    p.Wp = g.Wp;
    p.absmax = g.absmax;
    p.code = g.code;
    p.out = g.out;
    p.bias = g.bias;
    p.partials = g.partials;
    p.counters = g.counters;
    p.M = g.M;
    p.N = g.N;
    p.K = g.K;
    p.lbs = log2_bs;
    p.ku = (g.K + simt::kUnitK - 1) / simt::kUnitK;
    p.row_groups = (g.N + sh.rows - 1) / sh.rows;
    p.pdl = g.pdl;
    p.units = (uint32_t)((uint64_t)p.row_groups * (uint64_t)p.ku);
    p.warps = (uint32_t)ctas * (uint32_t)sh.warps;
    p.narrow = (uint64_t)p.units * p.warps < ((uint64_t)1 << 32) ? 1 : 0;
    p.a32 = (reinterpret_cast<uintptr_t>(g.A) & 31u) == 0 ? 1 : 0;
    p.error = g.error;
    if (act_dtype == 0) return simt_launch_t<__nv_bfloat16>(sh, ctas, p, stream);
    if (act_dtype == 1) return simt_launch_t<__half>(sh, ctas, p, stream);
    return simt_launch_t<float>(sh, ctas, p, stream);
}

}  // namespace q4
