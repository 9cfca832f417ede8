// q4_device.cuh -- small device-side helpers shared by the libq4 kernels:
// cache-hinted global loads, shared-memory access by 32-bit window address,
// byte permutes, 16-bit float packing and the m16n8k16 tensor-core MMA.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "q4_plan.cuh"

namespace q4 {

// ---------------------------------------------------------------------------
// Global loads.  Weights and absmax are read exactly once per call: stream
// them past L1 (no_allocate) through the read-only path.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint2 ldg_stream_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

// Same, with an L2 fetch-size hint: the L2 brings in the whole 128/256-byte
// span around the 8 bytes requested (the following units of the same rows).
template <int L2PF>
__device__ __forceinline__ uint2 ldg_stream_v2_pf(const void* p) {
    uint2 v;
    if constexpr (L2PF == 256)
        asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v2.u32 {%0, %1}, [%2];"
                     : "=r"(v.x), "=r"(v.y)
                     : "l"(p));
    else if constexpr (L2PF == 128)
        asm volatile("ld.global.nc.L1::no_allocate.L2::128B.v2.u32 {%0, %1}, [%2];"
                     : "=r"(v.x), "=r"(v.y)
                     : "l"(p));
    else
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

template <int L2PF>
__device__ __forceinline__ uint32_t ldg_stream_u32_pf(const void* p) {
    uint32_t v;
    if constexpr (L2PF == 256)
        asm volatile("ld.global.nc.L1::no_allocate.L2::256B.u32 %0, [%1];" : "=r"(v) : "l"(p));
    else if constexpr (L2PF == 128)
        asm volatile("ld.global.nc.L1::no_allocate.L2::128B.u32 %0, [%1];" : "=r"(v) : "l"(p));
    else
        asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

template <int L2PF>
__device__ __forceinline__ float ldg_stream_f32_pf(const float* p) {
    float v;
    if constexpr (L2PF == 256)
        asm volatile("ld.global.nc.L1::no_allocate.L2::256B.f32 %0, [%1];" : "=f"(v) : "l"(p));
    else if constexpr (L2PF == 128)
        asm volatile("ld.global.nc.L1::no_allocate.L2::128B.f32 %0, [%1];" : "=f"(v) : "l"(p));
    else
        asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_stream_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ float ldg_stream_f32(const float* p) {
    float v;
    asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Activations are re-read by several warps of an SM: keep them in L1.
__device__ __forceinline__ uint4 ldg_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// gpu-scope atomic add with acquire-release semantics: publishes this
// thread's (and, by cumulativity, its warp's synchronised) earlier writes and
// observes the writes published by earlier adds to the same counter.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
    int old;
    asm volatile("atom.add.acq_rel.gpu.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// L2-coherent load (bypasses L1): for data other CTAs wrote in this launch.
__device__ __forceinline__ float ldg_cg_f32(const float* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// Shared memory by 32-bit shared-window address.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v));
}

__device__ __forceinline__ void sts_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d));
}

__device__ __forceinline__ void sts_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ float2 lds_f32x2(uint32_t addr) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// Four 8x8 matrices of 16-bit elements (here: 8 rows x 16 bytes of packed
// codes each); lane l supplies the row address of row l%8 of matrix l/8 and
// receives, from every matrix j, bytes [4(l%4), 4(l%4)+4) of row l/4.
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& d0, uint32_t& d1, uint32_t& d2, uint32_t& d3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(d0), "=r"(d1), "=r"(d2), "=r"(d3)
                 : "r"(addr));
}

// ---------------------------------------------------------------------------
// mbarrier + TMA (bulk tensor copies, no multicast).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Barrier among `nthreads` threads (a multiple of 32) on hardware barrier `id` (1..15).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// try_wait that may suspend the thread for up to `ns` nanoseconds while the
// phase is incomplete (it returns as soon as the phase completes), so a
// waiting warp does not spin on the issue slots the working warps need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Every wait on an mbarrier is bounded (kWaitLimit polls by default, see
// q4_plan.cuh).
__device__ __forceinline__ bool wait_stage(uint32_t bar, uint32_t parity, uint32_t limit = kWaitLimit) {
    for (uint32_t it = 0; it < limit; ++it)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(tmap), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Same copy with an L2 eviction-priority hint (a policy from l2_evict_first).
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const void* tmap, int x, int y, uint32_t bar,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(tmap), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

// Hint that the box at {x, y} of a tensor map will soon be read: the L2
// fetches it from DRAM now (no shared memory, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_l2_2d(const void* tmap, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(tmap), "r"(x), "r"(y)
                 : "memory");
}

// Starts fetching a tensor map (a kernel parameter) into the descriptor
// cache, so that the first copy through it does not wait for that fetch.
__device__ __forceinline__ void prefetch_tensormap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// L2 policy for data read exactly once: its lines are the first candidates
// for eviction, so they do not push out data that is read again.
__device__ __forceinline__ uint64_t l2_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Programmatic dependent launch: block until the grids this one depends on
// have completed and their writes are visible (a no-op without the launch
// attribute); allow the next dependent grid to begin launching.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t dynamic_smem_size() {
    uint32_t v;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(v));
    return v;
}

// ---------------------------------------------------------------------------
// Byte permute: result byte i = byte sel_i of the 8-byte value {hi:lo}.
// ---------------------------------------------------------------------------
template <uint32_t SEL>
__device__ __forceinline__ uint32_t prmt(uint32_t lo, uint32_t hi) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(lo), "r"(hi), "n"(SEL));
    return r;
}

// CTA-scope atomic add on a shared-memory word with acquire-release
// semantics (publishes this thread's earlier shared writes, observes the
// writes published by earlier adds).
__device__ __forceinline__ int atom_add_acq_rel_cta_smem(uint32_t addr, int v) {
    int old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.s32 %0, [%1], %2;" : "=r"(old) : "r"(addr), "r"(v) : "memory");
    return old;
}

// CTA-scope release add on a shared-memory word (no return value).
__device__ __forceinline__ void red_add_release_cta_smem(uint32_t addr, uint32_t v) {
    asm volatile("red.release.cta.shared::cta.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Polls a shared-memory counter (acquire loads) until it reaches `target`;
// false after `limit` polls.
__device__ __forceinline__ bool wait_count_at_least(uint32_t addr, uint32_t target, uint32_t limit) {
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t v;
        asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
        if (v >= target) return true;
    }
    return false;
}

// ---------------------------------------------------------------------------
// 16-bit activation types.
// ---------------------------------------------------------------------------
template <typename T>
struct Act;

template <>
struct Act<__nv_bfloat16> {
    // Two floats -> packed pair, each rounded to nearest even; `first` in the
    // low 16 bits.
    __device__ __forceinline__ static uint32_t pack(float first, float second) {
        __nv_bfloat162 h = __floats2bfloat162_rn(first, second);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ __forceinline__ static __nv_bfloat16 from_float(float v) { return __float2bfloat16_rn(v); }
};

// Operand format code of a 16-bit type in a tcgen05 instruction descriptor.
template <typename T>
struct Act16Format;
template <>
struct Act16Format<__nv_bfloat16> {
    static constexpr uint32_t value = 1;
};
template <>
struct Act16Format<__half> {
    static constexpr uint32_t value = 0;
};

template <>
struct Act<__half> {
    __device__ __forceinline__ static uint32_t pack(float first, float second) {
        __half2 h = __floats2half2_rn(first, second);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ __forceinline__ static __half from_float(float v) { return __float2half_rn(v); }
};

// ---------------------------------------------------------------------------
// D = A(16x16, row) * B(16x8, col) + C, fp32 accumulate.
// Fragment ownership (g = lane/4, t = lane%4):
//   a0: A[g][2t..2t+1]   a1: A[g+8][2t..2t+1]   a2: A[g][2t+8..2t+9]   a3: A[g+8][2t+8..2t+9]
//   b0: B[2t..2t+1][g]   b1: B[2t+8..2t+9][g]
//   d0,d1: D[g][2t..2t+1]   d2,d3: D[g+8][2t..2t+1]
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1, const float (&c)[4]);

template <>
__device__ __forceinline__ void mma16816<__nv_bfloat16>(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                        uint32_t a3, uint32_t b0, uint32_t b1,
                                                        const float (&c)[4]) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

template <>
__device__ __forceinline__ void mma16816<__half>(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                 uint32_t a3, uint32_t b0, uint32_t b1, const float (&c)[4]) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]),
          "f"(c[3]));
}

// ---------------------------------------------------------------------------
// Byte-pair code table in shared memory.
//
// Row b (256 bytes) holds 32 copies, one per bank, of the packed pair
// (code[b >> 4], code[b & 15]) in the activation type -- the first (even)
// element in the low half -- i.e. exactly one MMA A-fragment register for a
// packed byte.  Only the lower 128 bytes of a row are the table; the upper
// halves are free scratch.  The table sits on a 64 KiB boundary of the
// shared window, so ONE byte permute builds a lookup address
// (table base | byte << 8 | lane << 2) from a packed word, and a warp-wide
// lookup never has a bank conflict.
// ---------------------------------------------------------------------------
static constexpr uint32_t kLutBytes = 256u * 256u;

// One lookup: byte BYTE of `word` -> packed (code[hi], code[lo]).  `lane4` =
// table base | lane << 2.
template <int BYTE>
__device__ __forceinline__ uint32_t lut_pair(uint32_t word, uint32_t lane4) {
    // result bytes: [0] = lane4.b0 (lane*4), [1] = word.b<BYTE>, [2..3] = lane4.b2..b3 (table base >> 16)
    return lds_u32(prmt<0x7604u | (BYTE << 4)>(word, lane4));
}

// Builds the table.  `cv` is code[lane & 15] in every lane; the pair is
// gathered by shuffles, so the table costs one global load per thread.
// nthreads is a multiple of 32 that divides the 2048 row pieces evenly per
// warp (the shuffles need whole warps).
template <typename T>
__device__ __forceinline__ void build_lut(uint32_t lut, float cv, int tid, int nthreads) {
    for (int e = tid; e < 256 * 8; e += nthreads) {
        const int b = e >> 3;
        const float hi = __shfl_sync(0xffffffffu, cv, b >> 4);
        const float lo = __shfl_sync(0xffffffffu, cv, b & 15);
        const uint32_t v = Act<T>::pack(hi, lo);
        sts_v4(lut + (uint32_t)b * 256u + (uint32_t)(e & 7) * 16u, v, v, v, v);
    }
}

}  // namespace q4
