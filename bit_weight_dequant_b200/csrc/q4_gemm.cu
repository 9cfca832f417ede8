// q4_gemm.cu -- fused blockwise 4-bit dequantize + skinny GEMM for sm_100a.
//
//     out[m, n] = sum_k A[m, k] * code[idx(n, k)] * absmax(n, k),  M <= 16
//
// bitsandbytes PR #1920 ("[ROCm] Optimize kgemm_4bit_inference_naive ...",
// "Technical details" and "Fused path support for M > 1") describes this
// operation: a fused dequantize + matmul over packed 4-bit weights with a
// 16-entry code table, used for the vector case and small multi-row M.  Its
// kernels are written for AMD/consumer parts; this one is designed for B200:
//
//  * The path is HBM-bound (0.5625 B per weight at blocksize 64).  At B200's
//    ~6.5 TB/s the SMs must retire ~40 weights per clock each, which leaves
//    about 3 thread-instructions per weight -- too few for a per-element
//    lookup + convert + FMA (or a warp-shuffle / constant-memory LUT).
//  * So the multiply-add runs on the tensor cores (mma.sync m16n8k16, fp32
//    accumulate), with the matrix roles swapped: 16 weight rows form the MMA
//    "M" side and the (padded) activation rows the 8-wide "N" side.  Even at
//    M = 1 this costs one MMA per 256 weights.
//  * Dequantization is one shared-memory lookup per packed BYTE: a 256-entry
//    table maps a byte straight to the packed 16-bit pair (code[hi], code[lo])
//    in the activation type, i.e. directly to one A-fragment register.  The
//    table is replicated once per bank (32 copies, 256-B rows, 64 KiB) so a
//    warp-wide lookup never has a bank conflict, and it is placed on a 64 KiB
//    boundary of the shared window so that ONE byte-permute builds the full
//    shared address (table base | byte << 8 | lane << 2) from the packed word.
//  * The contraction order inside an MMA is free, so every lane loads its
//    weights as one contiguous 8-byte run of a row (16 k values) and the
//    activation fragment is gathered with the same k permutation.  Each MMA
//    step stays inside one absmax block; the block scale is applied once per
//    block in fp32 (acc += absmax * partial), not per weight.
//  * Load balance: a persistent grid of <= #SM CTAs splits the work units
//    (64 rows x 64 k) evenly (see q4_plan.cuh); tiles cut between warps are
//    combined in shared memory, tiles cut between CTAs through a small
//    workspace by the last CTA to arrive -- no spinning, deterministic order.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "q4_device.cuh"
#include "q4_internal.h"
#include "q4_plan.cuh"

namespace q4 {

// Registers of one work unit for one lane (loaded one unit ahead).
template <class S>
struct Unit {
    uint32_t w[S::TW][2][S::SB / 32];  // packed weights: rows g and g+8 of each 16-row tile
    uint32_t a[S::NJ][S::SB / 8];      // activations of row 8j+g, this lane's k run
    float am[S::TW][2];                // absmax of those rows for this k block
};

template <typename T, class S>
__device__ __forceinline__ void load_unit(Unit<S>& u, const GemmParams& p, int tile, int kb, int g, int tq) {
    const size_t row_bytes = (size_t)(p.K >> 1);
    const int kbyte = kb * (S::SB / 2) + tq * (S::SB / 8);
    const int am_col = kb >> p.am_shift;
#pragma unroll
    for (int i = 0; i < S::TW; ++i) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int n = min(tile * S::TR + 16 * i + g + 8 * r, p.N - 1);  // rows past N: clamp, never stored
            const uint8_t* wp = p.Wp + (size_t)n * row_bytes + kbyte;
            if constexpr (S::SB == 64) {
                const uint2 v = ldg_stream_v2_pf<S::L2PF>(wp);
                u.w[i][r][0] = v.x;
                u.w[i][r][1] = v.y;
            } else {
                u.w[i][r][0] = ldg_stream_u32_pf<S::L2PF>(wp);
            }
            u.am[i][r] = ldg_stream_f32_pf<S::L2PF>(p.absmax + (size_t)n * p.am_per_row + am_col);
        }
    }
    const T* A = static_cast<const T*>(p.A);
#pragma unroll
    for (int j = 0; j < S::NJ; ++j) {
        const int m = 8 * j + g;
        if (m < p.M) {
            const T* ap = A + (size_t)m * p.K + kb * S::SB + tq * (S::SB / 4);
#pragma unroll
            for (int q = 0; q < S::SB / 32; ++q) {
                const uint4 v = ldg_v4(ap + 8 * q);
                u.a[j][4 * q + 0] = v.x;
                u.a[j][4 * q + 1] = v.y;
                u.a[j][4 * q + 2] = v.z;
                u.a[j][4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int q = 0; q < S::SB / 8; ++q) u.a[j][q] = 0u;
        }
    }
}

template <typename T, class S>
__device__ __forceinline__ void mma_unit(float (&acc)[S::TW][S::NJ][4], const Unit<S>& u, uint32_t lane4) {
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < S::TW; ++i) {
        float t[S::NJ][4];
#pragma unroll
        for (int s = 0; s < S::SB / 16; ++s) {
            // step s consumes bytes 2s, 2s+1 of each row's 8-byte run:
            //   byte 2s   -> k = 4s, 4s+1 -> MMA k slots 2t, 2t+1     (a0 row g, a1 row g+8)
            //   byte 2s+1 -> k = 4s+2, 4s+3 -> MMA k slots 2t+8, 2t+9 (a2 row g, a3 row g+8)
            const uint32_t wg = u.w[i][0][s >> 1];
            const uint32_t wg8 = u.w[i][1][s >> 1];
            uint32_t a0, a1, a2, a3;
            if ((s & 1) == 0) {
                a0 = lut_pair<0>(wg, lane4);
                a2 = lut_pair<1>(wg, lane4);
                a1 = lut_pair<0>(wg8, lane4);
                a3 = lut_pair<1>(wg8, lane4);
            } else {
                a0 = lut_pair<2>(wg, lane4);
                a2 = lut_pair<3>(wg, lane4);
                a1 = lut_pair<2>(wg8, lane4);
                a3 = lut_pair<3>(wg8, lane4);
            }
#pragma unroll
            for (int j = 0; j < S::NJ; ++j) {
                if (s == 0)
                    mma16816<T>(t[j], a0, a1, a2, a3, u.a[j][0], u.a[j][1], zero);
                else
                    mma16816<T>(t[j], a0, a1, a2, a3, u.a[j][2 * s], u.a[j][2 * s + 1], t[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < S::NJ; ++j) {
            acc[i][j][0] = fmaf(u.am[i][0], t[j][0], acc[i][j][0]);
            acc[i][j][1] = fmaf(u.am[i][0], t[j][1], acc[i][j][1]);
            acc[i][j][2] = fmaf(u.am[i][1], t[j][2], acc[i][j][2]);
            acc[i][j][3] = fmaf(u.am[i][1], t[j][3], acc[i][j][3]);
        }
    }
}

template <typename T, class S>
__device__ __forceinline__ void store_tile(const float (&v)[S::TW][S::NJ][4], const GemmParams& p, int tile, int g,
                                           int tq) {
    T* out = static_cast<T*>(p.out);
    const T* bias = static_cast<const T*>(p.bias);
#pragma unroll
    for (int i = 0; i < S::TW; ++i)
#pragma unroll
        for (int j = 0; j < S::NJ; ++j)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int n = tile * S::TR + 16 * i + g + ((r & 2) ? 8 : 0);
                const int m = 8 * j + 2 * tq + (r & 1);
                if (n < p.N && m < p.M) {
                    const float b = bias ? static_cast<float>(bias[n]) : 0.f;  // exact widening
                    out[(size_t)m * p.N + n] = Act<T>::from_float(v[i][j][r] + b);
                }
            }
}

template <class S>
__device__ __forceinline__ void zero_acc(float (&v)[S::TW][S::NJ][4]) {
#pragma unroll
    for (int i = 0; i < S::TW; ++i)
#pragma unroll
        for (int j = 0; j < S::NJ; ++j)
#pragma unroll
            for (int r = 0; r < 4; ++r) v[i][j][r] = 0.f;
}

// Slot layout: [slot][reg][lane] floats, reg = (i * NJ + j) * 4 + r.
template <class S>
__device__ __forceinline__ void store_slot(const float (&v)[S::TW][S::NJ][4], uint32_t slots, int slot, int lane) {
#pragma unroll
    for (int i = 0; i < S::TW; ++i)
#pragma unroll
        for (int j = 0; j < S::NJ; ++j)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int reg = (i * S::NJ + j) * 4 + r;
                sts_f32(slots + (uint32_t)((slot * S::SLOT_FLOATS + reg * 32 + lane) * 4), v[i][j][r]);
            }
}

template <class S>
__device__ __forceinline__ void add_slot(float (&v)[S::TW][S::NJ][4], uint32_t slots, int slot, int lane) {
#pragma unroll
    for (int i = 0; i < S::TW; ++i)
#pragma unroll
        for (int j = 0; j < S::NJ; ++j)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int reg = (i * S::NJ + j) * 4 + r;
                v[i][j][r] += lds_f32(slots + (uint32_t)((slot * S::SLOT_FLOATS + reg * 32 + lane) * 4));
            }
}

// Per-warp cursor over its unit range.
struct Cursor {
    int tile, kb;
    bool from_start;   // this warp owns the current tile from its first unit
    bool first_tile;   // the current tile is the first one this warp touches
};

// After a unit: close the tile if it (or the warp's range) ends here.
template <typename T, class S>
__device__ __forceinline__ void finish_unit(float (&acc)[S::TW][S::NJ][4], Cursor& c, bool range_end,
                                            const GemmParams& p, uint32_t slots, int warp, int lane, int g,
                                            int tq) {
    const bool tile_end = (c.kb == p.kb_per_tile - 1);
    if (tile_end || range_end) {
        if (c.from_start && tile_end)
            store_tile<T, S>(acc, p, c.tile, g, tq);  // whole tile computed by this warp alone
        else
            store_slot<S>(acc, slots, warp * 2 + (c.first_tile ? 0 : 1), lane);
        zero_acc<S>(acc);
        c.first_tile = false;
    }
    if (++c.kb == p.kb_per_tile) {
        c.kb = 0;
        ++c.tile;
        c.from_start = true;
    }
}

__device__ __forceinline__ void advance(int& tile, int& kb, int kb_per_tile) {
    if (++kb == kb_per_tile) {
        kb = 0;
        ++tile;
    }
}

// Combines the tiles that warps or CTAs share (after a __syncthreads that
// makes every warp's slots visible): a tile cut only between warps of this
// CTA is summed in warp order from shared memory and stored; a tile cut
// between CTAs is published to the workspace, and the last CTA to arrive
// sums all partials in CTA order and stores the tile.
template <typename T, class S>
__device__ __forceinline__ void combine_tiles(const GemmParams& p, uint32_t slots, uint32_t cs, uint32_t ce, int warp,
                                              int lane, int g, int tq) {
    const uint32_t uc = ce - cs, kbt = (uint32_t)p.kb_per_tile;
    const int ta = (int)(cs / kbt);
    const int tb = (int)((ce - 1) / kbt);
    for (int t = ta + warp; t <= tb; t += S::NW) {
        const uint32_t t0 = (uint32_t)t * kbt, t1 = t0 + kbt;
        const uint32_t lo = t0 > cs ? t0 : cs, hi = t1 < ce ? t1 : ce;
        const int wlo = (int)part_owner(uc, S::NW, lo - cs), whi = (int)part_owner(uc, S::NW, hi - 1 - cs);
        const bool inside = (lo == t0) && (hi == t1);
        if (inside && wlo == whi) continue;  // already stored by its only warp
        float sum[S::TW][S::NJ][4];
        zero_acc<S>(sum);
        for (int w = wlo; w <= whi; ++w) {
            const uint32_t w0 = cs + part_start(uc, S::NW, w), w1 = cs + part_start(uc, S::NW, w + 1);
            if (w1 == w0) continue;  // empty warp range
            add_slot<S>(sum, slots, w * 2 + ((w0 >= t0) ? 0 : 1), lane);  // w0 >= t0: tile t is w's first
        }
        if (inside) {
            store_tile<T, S>(sum, p, t, g, tq);
            continue;
        }
        // The tile crosses this CTA's range: publish the partial, and let the
        // last CTA to arrive add all partials in CTA order and store the tile.
        float* mine = p.partials + ((size_t)blockIdx.x * 2 + (t == ta ? 0 : 1)) * S::SLOT_FLOATS;
#pragma unroll
        for (int i = 0; i < S::TW; ++i)
#pragma unroll
            for (int j = 0; j < S::NJ; ++j)
#pragma unroll
                for (int r = 0; r < 4; ++r) mine[((i * S::NJ + j) * 4 + r) * 32 + lane] = sum[i][j][r];
        // Release the warp's partial and count it in; the add also acquires
        // the partials the other CTAs released before it.
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atom_add_acq_rel_gpu(p.counters + t, 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        __syncwarp();  // the other lanes read the partials after lane 0's acquire
        const int cf = (int)part_owner(p.units, p.ctas, t0), cl = (int)part_owner(p.units, p.ctas, t1 - 1);
        if (prev != cl - cf) continue;
        zero_acc<S>(sum);
        for (int cta = cf; cta <= cl; ++cta) {
            const int which = (part_start(p.units, p.ctas, cta) >= t0) ? 0 : 1;  // tile t is the CTA's first
            const float* src = p.partials + ((size_t)cta * 2 + which) * S::SLOT_FLOATS;
#pragma unroll
            for (int i = 0; i < S::TW; ++i)
#pragma unroll
                for (int j = 0; j < S::NJ; ++j)
#pragma unroll
                    for (int r = 0; r < 4; ++r) sum[i][j][r] += ldg_cg_f32(src + ((i * S::NJ + j) * 4 + r) * 32 + lane);
        }
        store_tile<T, S>(sum, p, t, g, tq);
        if (lane == 0) p.counters[t] = 0;  // return the counter to zero for the next call
    }
}

template <typename T, class S>
__global__ void __launch_bounds__(S::NW * 32, 1) q4_gemm_mma_kernel(const GemmParams p) {
    griddep_wait();  // no overlap with a preceding grid in this kernel
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t sbase = smem_addr(smem);
    const uint32_t lut = (sbase + 0xFFFFu) & ~0xFFFFu;  // 64 KiB aligned (host reserves the padding)
    const uint32_t slots = (lut - sbase >= S::SLOT_BYTES) ? sbase : lut + S::LUT_BYTES;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;

    build_lut<T>(lut, __ldg(p.code + (lane & 15)), tid, S::NW * 32);
    __syncthreads();

    const uint32_t cs = part_start(p.units, p.ctas, blockIdx.x);
    const uint32_t ce = part_start(p.units, p.ctas, blockIdx.x + 1);
    const uint32_t uc = ce - cs;
    const uint32_t ws = cs + part_start(uc, S::NW, warp);
    const uint32_t we = cs + part_start(uc, S::NW, warp + 1);
    const uint32_t lane4 = lut | ((uint32_t)lane << 2);
    const int nunits = (int)(we - ws);

    if (nunits > 0) {
        float acc[S::TW][S::NJ][4];
        zero_acc<S>(acc);
        Cursor c;
        c.tile = (int)(ws / (uint32_t)p.kb_per_tile);
        c.kb = (int)(ws - (uint32_t)c.tile * (uint32_t)p.kb_per_tile);
        c.from_start = (c.kb == 0);
        c.first_tile = true;
        // Ring of DEPTH + 1 unit buffers: the loads of DEPTH units are in
        // flight while one unit is computed.
        constexpr int R = S::DEPTH + 1;
        int lt = c.tile, lk = c.kb;  // load cursor
        Unit<S> buf[R];
#pragma unroll
        for (int d = 0; d < S::DEPTH; ++d) {
            if (d < nunits) {
                load_unit<T, S>(buf[d], p, lt, lk, g, tq);
                advance(lt, lk, p.kb_per_tile);
            }
        }
        for (int i = 0; i < nunits; i += R) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                if (i + r < nunits) {
                    if (i + r + S::DEPTH < nunits) {
                        load_unit<T, S>(buf[(r + S::DEPTH) % R], p, lt, lk, g, tq);
                        advance(lt, lk, p.kb_per_tile);
                    }
                    mma_unit<T, S>(acc, buf[r], lane4);
                    finish_unit<T, S>(acc, c, i + r + 1 == nunits, p, slots, warp, lane, g, tq);
                }
            }
        }
    }
    __syncthreads();
    if (uc <= 0) return;

    combine_tiles<T, S>(p, slots, cs, ce, warp, lane, g, tq);
}

// ===========================================================================
// TMA-staged variant.
//
// The direct-load kernel above gives every lane its fragment bytes straight
// from global memory; each warp-wide load then touches 8 rows (8 lines) and
// each absmax load 8 lines for 32 useful bytes, and those L1 wavefronts --
// not DRAM -- limit it.  Here each warp streams its unit range through its
// own ring of shared-memory stages filled by the Tensor Memory Accelerator:
//   * weights: a 64-row box of UPS units (UPS x 32 bytes per row) per stage,
//     stored with the matching 64/128-byte swizzle so ldmatrix reads it
//     without bank conflicts;
//   * absmax: the 64-row x 4-float box that covers the stage's blocks.
// A stage's mbarrier completes when both boxes have landed; the warp's lane
// 0 issues the copy for stage k + D once stage k has been consumed.  Warps
// keep little state (the first partial tile is parked in the unused upper
// half of the LUT rows), so 16 warps fit and hide each other's latency.
// Every wait is bounded: on time-out the kernel records an error word in the
// workspace, stops issuing, drains its copies (also bounded) and returns
// normally (its outputs are then not valid).
// ===========================================================================
template <int UPS, int TR = 64>
struct StageGeom {
    static constexpr uint32_t ROW_BYTES = 32u * UPS;                   // 64 or 128
    static constexpr uint32_t WEIGHT_BYTES = (uint32_t)TR * ROW_BYTES; // TR rows of the stage's codes
    static constexpr uint32_t ABSMAX_BYTES = (uint32_t)TR * 4u * 4u;   // TR rows x 4 floats
    static constexpr uint32_t COPY_BYTES = WEIGHT_BYTES + ABSMAX_BYTES;  // what the two copies deliver
    static constexpr uint32_t BYTES = (COPY_BYTES + 1023u) & ~1023u;   // stage stride: swizzled boxes start 1 KiB aligned
    // physical address of 16-byte chunk `chunk` of box row `row` (TMA swizzle)
    __device__ __forceinline__ static uint32_t chunk_addr(uint32_t base, int row, int chunk) {
        if constexpr (UPS == 4)
            return base + (uint32_t)row * 128u + (uint32_t)((chunk ^ (row & 7)) << 4);
        else
            return base + (uint32_t)row * 64u + (uint32_t)((chunk ^ ((row >> 1) & 3)) << 4);
    }
};

struct StageCursor {
    int tile, kb, left;  // next unit to put in a stage; units of the range still unassigned
};

// Next stage of a warp's unit range: units [kb, kb + n) of `tile`, all in
// the same UPS-unit window [kb0, kb0 + UPS) and the same tile.
template <int UPS>
__device__ __forceinline__ void next_stage(StageCursor& c, int kb_per_tile, int& tile, int& kb0, int& kb, int& n) {
    tile = c.tile;
    kb = c.kb;
    kb0 = kb & ~(UPS - 1);
    int end = kb0 + UPS;
    if (end > kb_per_tile) end = kb_per_tile;
    n = end - kb;
    if (n > c.left) n = c.left;
    c.left -= n;
    c.kb += n;
    if (c.kb == kb_per_tile) {
        c.kb = 0;
        ++c.tile;
    }
}

// The first partial tile of a warp waits for the combine in the upper half
// of LUT rows warp*SLOT_REGS .. +SLOT_REGS (the lookups only use each row's
// lower 128 bytes).
template <class S>
__device__ __forceinline__ uint32_t parked_addr(uint32_t lut, int warp, int reg, int lane) {
    return lut + (uint32_t)(warp * S::SLOT_REGS + reg) * 256u + 128u + (uint32_t)lane * 4u;
}

// Closes a tile in the TMA kernel: a whole tile is stored, the warp's first
// partial tile is parked, a last partial tile stays in `acc`.
template <typename T, class S>
__device__ __forceinline__ void finish_unit_tma(float (&acc)[S::TW][S::NJ][4], bool& has_first, bool& has_last,
                                                Cursor& c, bool range_end, const GemmParams& p, uint32_t lut,
                                                int warp, int lane, int g, int tq) {
    const bool tile_end = (c.kb == p.kb_per_tile - 1);
    if (tile_end || range_end) {
        if (c.from_start && tile_end) {
            store_tile<T, S>(acc, p, c.tile, g, tq);  // whole tile computed by this warp alone
            zero_acc<S>(acc);
        } else if (c.first_tile) {
#pragma unroll
            for (int i = 0; i < S::TW; ++i)
#pragma unroll
                for (int j = 0; j < S::NJ; ++j)
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        sts_f32(parked_addr<S>(lut, warp, (i * S::NJ + j) * 4 + r, lane), acc[i][j][r]);
            has_first = true;
            zero_acc<S>(acc);
        } else {
            has_last = true;  // the range ends inside this tile: acc is the slot-1 partial
        }
        c.first_tile = false;
    }
    if (++c.kb == p.kb_per_tile) {
        c.kb = 0;
        ++c.tile;
        c.from_start = true;
    }
}

template <typename T, class S, int UPS, bool BS64>
__global__ void __launch_bounds__(S::NW * 32, 1)
    q4_gemm_tma_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_a,
                       const GemmParams p) {
    using G = StageGeom<UPS, S::TR>;
    static_assert(S::NW * S::SLOT_REGS <= 256, "parked partial tiles must fit in the LUT rows");
    extern __shared__ __align__(16) uint8_t smem_ring[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
    constexpr int D = S::DEPTH;  // stages per warp

    // Shared-memory layout (decided at run time from the window base): the
    // 64 KiB LUT on a 64 KiB boundary; barriers and stages in the space
    // below and above it.
    const uint32_t sbase = smem_addr(smem_ring);
    const uint32_t send = sbase + dynamic_smem_size();
    const uint32_t lut = (sbase + 0xFFFFu) & ~0xFFFFu;
    const uint32_t nbar_bytes = (uint32_t)S::NW * D * 8u;
    uint32_t bars, a0, b0 = lut + S::LUT_BYTES;
    if (lut - sbase >= nbar_bytes) {
        bars = sbase;
        a0 = (sbase + nbar_bytes + 1023u) & ~1023u;
    } else {
        bars = b0;
        b0 = (b0 + nbar_bytes + 1023u) & ~1023u;
        a0 = lut;
    }
    const uint32_t na = a0 < lut ? (lut - a0) / G::BYTES : 0u;
    const uint32_t nb = b0 < send ? (send - b0) / G::BYTES : 0u;
    const bool room = (lut + S::LUT_BYTES <= send) && (na + nb >= (uint32_t)(S::NW * D)) &&
                      ((send > b0 && send - b0 >= S::SLOT_BYTES) || (lut > a0 && lut - a0 >= S::SLOT_BYTES));
    if (!room) {  // uniform over the CTA: the host sized the launch wrongly
        if (tid == 0) atomicExch(p.error, kErrNoRoom);
        return;
    }
    const uint32_t slots = (send > b0 && send - b0 >= S::SLOT_BYTES) ? b0 : a0;
    auto stage_addr = [&](int idx) -> uint32_t {
        return (uint32_t)idx < na ? a0 + (uint32_t)idx * G::BYTES : b0 + ((uint32_t)idx - na) * G::BYTES;
    };

    if (p.pdl != 2) griddep_wait();
    const float cv = __ldg(p.code + (lane & 15));  // the table build's one global load, issued early
    if (lane == 0) {  // each warp's own stage barriers; only this warp uses them
        for (int d = 0; d < D; ++d) mbar_init(bars + (uint32_t)(warp * D + d) * 8u, 1);
        mbar_init_fence();
    }
    __syncwarp();

    const uint32_t cs = part_start(p.units, p.ctas, blockIdx.x);
    const uint32_t ce = part_start(p.units, p.ctas, blockIdx.x + 1);
    const uint32_t uc = ce - cs;
    const uint32_t ws = cs + part_start(uc, S::NW, warp);
    const uint32_t we = cs + part_start(uc, S::NW, warp + 1);
    const uint32_t lane4 = lut | ((uint32_t)lane << 2);
    const int nunits = (int)(we - ws);

    float acc[S::TW][S::NJ][4];
    bool has_first = false, has_last = false;
    zero_acc<S>(acc);
    Cursor c;
    c.tile = nunits > 0 ? (int)(ws / (uint32_t)p.kb_per_tile) : 0;
    c.kb = nunits > 0 ? (int)(ws - (uint32_t)c.tile * (uint32_t)p.kb_per_tile) : 0;
    c.from_start = (c.kb == 0);
    c.first_tile = true;
    StageCursor ld{c.tile, c.kb, nunits}, cm{c.tile, c.kb, nunits};
    int issued = 0, consumed = 0;
    const uint64_t stream_once = l2_evict_first();  // weights are read once; absmax lines are reused
    auto issue = [&](int k) {  // lane 0: stage k into ring slot k % D
        int tile, kb0, kb, n;
        next_stage<UPS>(ld, p.kb_per_tile, tile, kb0, kb, n);
        const uint32_t st = stage_addr(warp * D + k % D);
        const uint32_t bar = bars + (uint32_t)(warp * D + k % D) * 8u;
        if (lane == 0) {
            mbar_expect_tx(bar, G::COPY_BYTES);
            tma_load_2d_hint(st, &tmap_w, kb0 * 32, tile * S::TR, bar, stream_once);
            tma_load_2d(st + G::WEIGHT_BYTES, &tmap_a, (kb0 >> p.am_shift) & ~3, tile * S::TR, bar);
        }
    };
    // Start the first copies before anything else; the table is built while
    // they are in flight.
    for (; issued < D && ld.left > 0; ++issued) issue(issued);
    build_lut<T>(lut, cv, tid, S::NW * 32);
    __syncthreads();
    // Activations, outputs and the workspace may belong to the preceding
    // grid: touch them only after the dependency wait.
    if (p.pdl == 2) griddep_wait();
    griddep_launch_dependents();

    if (nunits > 0) {
        // ldmatrix row address pieces: lane l feeds row l%8 of matrix l/8.
        const int lm_q = lane >> 3, lm_r = lane & 7;
        const T* Aact = static_cast<const T*>(p.A);
        bool ok = true;

        // Activations of the current stage's UPS-unit window.  Windows are
        // UPS-aligned and tiles hold a multiple of UPS units, so a window
        // never reaches past K.  As soon as a unit is computed its registers
        // are refilled with the same unit of the next stage's window, so the
        // loads have most of a stage to land.
        uint32_t aw[UPS][S::NJ][2][4];
        auto load_unit = [&](int kbu, uint32_t(&dst)[S::NJ][2][4]) {
#pragma unroll
            for (int jj = 0; jj < S::NJ; ++jj) {
                const int m = 8 * jj + g;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    if (m < p.M) {
                        const uint4 v = ldg_v4(Aact + (size_t)m * p.K + kbu * S::SB + 32 * ch + 8 * tq);
                        dst[jj][ch][0] = v.x;
                        dst[jj][ch][1] = v.y;
                        dst[jj][ch][2] = v.z;
                        dst[jj][ch][3] = v.w;
                    } else {
                        dst[jj][ch][0] = dst[jj][ch][1] = dst[jj][ch][2] = dst[jj][ch][3] = 0u;
                    }
                }
            }
        };
        auto load_window = [&](int kbw) {
#pragma unroll
            for (int j = 0; j < UPS; ++j) load_unit(kbw + j, aw[j]);
        };
        load_window(c.kb & ~(UPS - 1));

        // One 64-row x 64-k unit (window position j) of the stage at `st`,
        // scaled by the per-row absmax (ag: rows 16i+g, ag8: rows 16i+8+g).
        auto unit_rows = [&](uint32_t st, int j, int i, float ag, float ag8) {
            const float zero[4] = {0.f, 0.f, 0.f, 0.f};
            // rows 16i + 8(q&1) + r, chunk 2j + (q>>1)
            uint32_t d[4];
            ldmatrix_x4(G::chunk_addr(st, 16 * i + 8 * (lm_q & 1) + lm_r, 2 * j + (lm_q >> 1)), d[0], d[1], d[2], d[3]);
            // q[x][b]: table pair of byte b of word d[x]
            uint32_t q[4][4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                q[x][0] = lut_pair<0>(d[x], lane4);
                q[x][1] = lut_pair<1>(d[x], lane4);
                q[x][2] = lut_pair<2>(d[x], lane4);
                q[x][3] = lut_pair<3>(d[x], lane4);
            }
            float t[S::NJ][4];
            // steps 0..3: (d0,d1) bytes 0/1, 2/3, then (d2,d3) bytes 0/1, 2/3
#pragma unroll
            for (int jj = 0; jj < S::NJ; ++jj)
                mma16816<T>(t[jj], q[0][0], q[1][0], q[0][1], q[1][1], aw[j][jj][0][0], aw[j][jj][0][1], zero);
#pragma unroll
            for (int jj = 0; jj < S::NJ; ++jj)
                mma16816<T>(t[jj], q[0][2], q[1][2], q[0][3], q[1][3], aw[j][jj][0][2], aw[j][jj][0][3], t[jj]);
#pragma unroll
            for (int jj = 0; jj < S::NJ; ++jj)
                mma16816<T>(t[jj], q[2][0], q[3][0], q[2][1], q[3][1], aw[j][jj][1][0], aw[j][jj][1][1], t[jj]);
#pragma unroll
            for (int jj = 0; jj < S::NJ; ++jj)
                mma16816<T>(t[jj], q[2][2], q[3][2], q[2][3], q[3][3], aw[j][jj][1][2], aw[j][jj][1][3], t[jj]);
#pragma unroll
            for (int jj = 0; jj < S::NJ; ++jj) {
                acc[i][jj][0] = fmaf(ag, t[jj][0], acc[i][jj][0]);
                acc[i][jj][1] = fmaf(ag, t[jj][1], acc[i][jj][1]);
                acc[i][jj][2] = fmaf(ag8, t[jj][2], acc[i][jj][2]);
                acc[i][jj][3] = fmaf(ag8, t[jj][3], acc[i][jj][3]);
            }
        };
        // With 4-unit stages and one absmax per unit, a row's 4-float absmax
        // box is exactly the stage's 4 units: one 16-byte read per row.
        constexpr bool kAmRow = (UPS == 4) && BS64;

        while (cm.left > 0) {
            int tile, kb0, kb, n;
            next_stage<UPS>(cm, p.kb_per_tile, tile, kb0, kb, n);
            const int kbn = cm.kb & ~(UPS - 1);  // next stage's window (when cm.left > 0)
            const int slot = consumed % D;
            const uint32_t st = stage_addr(warp * D + slot);
            const uint32_t bar = bars + (uint32_t)(warp * D + slot) * 8u;
            if (!wait_stage(bar, (uint32_t)(consumed / D) & 1u)) {
                ok = false;
                break;
            }
            const int x0 = (kb0 >> p.am_shift) & ~3;
            const uint32_t am_stage = st + G::WEIGHT_BYTES;
            float am[S::TW][2][4];
            if constexpr (kAmRow) {
#pragma unroll
                for (int i = 0; i < S::TW; ++i)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint4 v = lds_v4(am_stage + (uint32_t)(16 * i + 8 * h + g) * 16u);
                        am[i][h][0] = __uint_as_float(v.x);
                        am[i][h][1] = __uint_as_float(v.y);
                        am[i][h][2] = __uint_as_float(v.z);
                        am[i][h][3] = __uint_as_float(v.w);
                    }
            }
            auto unit_all_rows = [&](int j) {
                // absmax column of this unit inside the stage's 4-float box
                const int col = BS64 ? (kb0 + j - x0) : (((kb0 + j) >> p.am_shift) - x0);
                const uint32_t am_base = am_stage + (uint32_t)col * 4u;
#pragma unroll
                for (int i = 0; i < S::TW; ++i) {
                    if constexpr (kAmRow)
                        unit_rows(st, j, i, am[i][0][j], am[i][1][j]);
                    else
                        unit_rows(st, j, i, lds_f32(am_base + (uint32_t)(16 * i + g) * 16u),
                                  lds_f32(am_base + (uint32_t)(16 * i + 8 + g) * 16u));
                }
            };
            if (n == UPS) {
                // Whole stage inside one tile and the range: no tile can end
                // before its last unit, so the units run back to back.
#pragma unroll
                for (int j = 0; j < UPS; ++j) {
                    unit_all_rows(j);
                    if (cm.left > 0) load_unit(kbn + j, aw[j]);
                }
                c.kb += UPS - 1;
                finish_unit_tma<T, S>(acc, has_first, has_last, c, cm.left == 0, p, lut, warp, lane, g, tq);
            } else {
#pragma unroll
                for (int j = 0; j < UPS; ++j) {
                    if (kb0 + j < kb || kb0 + j >= kb + n) continue;
                    unit_all_rows(j);
                    finish_unit_tma<T, S>(acc, has_first, has_last, c, cm.left == 0 && kb0 + j + 1 == kb + n, p, lut,
                                          warp, lane, g, tq);
                }
                if (cm.left > 0) load_window(kbn);  // first or last stage of a range only
            }
            ++consumed;
            // Hand the slot back to the copy engine: order this warp's reads
            // of it before the next asynchronous write into it.
            fence_proxy_async_smem();
            __syncwarp();
            if (ld.left > 0) issue(issued++);
        }
        if (!ok) {
            if (lane == 0) atomicExch(p.error, kErrWaitTimeout);
            // drain the copies still in flight into this warp's stages
            for (int k = consumed; k < issued; ++k)
                wait_stage(bars + (uint32_t)(warp * D + k % D) * 8u, (uint32_t)(k / D) & 1u);
        }
    }
    __syncthreads();  // every warp is out of the stage ring: the slots may reuse it
    if (has_first) {
        float first[S::TW][S::NJ][4];
#pragma unroll
        for (int i = 0; i < S::TW; ++i)
#pragma unroll
            for (int j = 0; j < S::NJ; ++j)
#pragma unroll
                for (int r = 0; r < 4; ++r) first[i][j][r] = lds_f32(parked_addr<S>(lut, warp, (i * S::NJ + j) * 4 + r, lane));
        store_slot<S>(first, slots, warp * 2, lane);
    }
    if (has_last) store_slot<S>(acc, slots, warp * 2 + 1, lane);
    __syncthreads();
    if (uc <= 0) return;
    combine_tiles<T, S>(p, slots, cs, ce, warp, lane, g, tq);
}


// ===========================================================================
// Warp-specialised variant.
//
// Issuing a TMA copy can block the issuing thread while the SM's copy engine
// works through earlier boxes (it walks them row by row), so in the kernel
// above every consumer warp stalls behind its own lane 0 during the initial
// burst.  Here one producer warp issues all copies -- its lane w feeds
// consumer warp w's ring -- and consumers hand each stage back through an
// "empty" mbarrier.  Stages are 64 rows x 128 bytes (4 units), halving the
// copy engine's row requests per byte compared with 64-byte rows.
// ===========================================================================
template <typename T, class S, int UPS, bool BS64>
__global__ void __launch_bounds__((S::NW + 1) * 32, 1)
    q4_gemm_ws_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_a,
                      const GemmParams p) {
    using G = StageGeom<UPS, S::TR>;
    static_assert(S::NW * S::SLOT_REGS <= 256, "parked partial tiles must fit in the LUT rows");
    static_assert(S::NW <= 32, "one producer lane per consumer warp");
    constexpr int NC = S::NW;     // consumer warps
    constexpr int D = S::DEPTH;   // stages per consumer
    extern __shared__ __align__(16) uint8_t smem_ws[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
    const bool producer = (warp == NC);

    // Layout: 64 KiB LUT on a 64 KiB boundary; full/empty barriers and the
    // stages below and above it.
    const uint32_t sbase = smem_addr(smem_ws);
    const uint32_t send = sbase + dynamic_smem_size();
    const uint32_t lut = (sbase + 0xFFFFu) & ~0xFFFFu;
    const uint32_t nbar_bytes = (uint32_t)NC * D * 16u;
    uint32_t bars, a0, b0 = lut + S::LUT_BYTES;
    if (lut - sbase >= nbar_bytes) {
        bars = sbase;
        a0 = (sbase + nbar_bytes + 1023u) & ~1023u;
    } else {
        bars = b0;
        b0 = (b0 + nbar_bytes + 1023u) & ~1023u;
        a0 = lut;
    }
    const uint32_t na = a0 < lut ? (lut - a0) / G::BYTES : 0u;
    const uint32_t nb = b0 < send ? (send - b0) / G::BYTES : 0u;
    const bool room = (lut + S::LUT_BYTES <= send) && (na + nb >= (uint32_t)(NC * D)) &&
                      ((send > b0 && send - b0 >= S::SLOT_BYTES) || (lut > a0 && lut - a0 >= S::SLOT_BYTES));
    if (!room) {
        if (tid == 0) atomicExch(p.error, kErrNoRoom);
        return;
    }
    const uint32_t slots = (send > b0 && send - b0 >= S::SLOT_BYTES) ? b0 : a0;
    auto stage_addr = [&](int idx) -> uint32_t {
        return (uint32_t)idx < na ? a0 + (uint32_t)idx * G::BYTES : b0 + ((uint32_t)idx - na) * G::BYTES;
    };
    auto full_bar = [&](int w, int d) -> uint32_t { return bars + (uint32_t)(w * D + d) * 8u; };
    auto empty_bar = [&](int w, int d) -> uint32_t { return bars + (uint32_t)(NC * D + w * D + d) * 8u; };

    if (p.pdl != 2) griddep_wait();
    if (producer && lane < NC) {
        for (int d = 0; d < D; ++d) {
            mbar_init(full_bar(lane, d), 1);
            mbar_init(empty_bar(lane, d), 1);
        }
        mbar_init_fence();
    }
    __syncthreads();

    const uint32_t cs = part_start(p.units, p.ctas, blockIdx.x);
    const uint32_t ce = part_start(p.units, p.ctas, blockIdx.x + 1);
    const uint32_t uc = ce - cs;
    float acc[S::TW][S::NJ][4];
    bool has_first = false, has_last = false;
    zero_acc<S>(acc);

    if (producer) {
        // Lane w streams consumer w's unit range into its ring.
        if (lane < NC) {
            const uint64_t stream_once = l2_evict_first();
            const uint32_t ws = cs + part_start(uc, NC, lane), we = cs + part_start(uc, NC, lane + 1);
            const int nunits = (int)(we - ws);
            const int tile0 = nunits > 0 ? (int)(ws / (uint32_t)p.kb_per_tile) : 0;
            StageCursor ld{tile0, nunits > 0 ? (int)(ws - (uint32_t)tile0 * (uint32_t)p.kb_per_tile) : 0, nunits};
            for (int k = 0; ld.left > 0; ++k) {
                const int slot = k % D;
                if (k >= D && !wait_stage(empty_bar(lane, slot), (uint32_t)(k / D - 1) & 1u)) {
                    if (p.pdl == 2) griddep_wait();
                    atomicExch(p.error, kErrWaitTimeout);
                    break;
                }
                int tile, kb0, kb, n;
                next_stage<UPS>(ld, p.kb_per_tile, tile, kb0, kb, n);
                const uint32_t st = stage_addr(lane * D + slot);
                mbar_expect_tx(full_bar(lane, slot), G::COPY_BYTES);
                tma_load_2d_hint(st, &tmap_w, kb0 * 32, tile * S::TR, full_bar(lane, slot), stream_once);
                tma_load_2d(st + G::WEIGHT_BYTES, &tmap_a, (kb0 >> p.am_shift) & ~3, tile * S::TR, full_bar(lane, slot));
            }
        }
    } else {
        build_lut<T>(lut, __ldg(p.code + (lane & 15)), tid, NC * 32);
        named_bar_sync(1, NC * 32);
        if (p.pdl == 2) griddep_wait();
        griddep_launch_dependents();
        const uint32_t ws = cs + part_start(uc, NC, warp), we = cs + part_start(uc, NC, warp + 1);
        const int nunits = (int)(we - ws);
        const uint32_t lane4 = lut | ((uint32_t)lane << 2);
        if (nunits > 0) {
            Cursor c;
            c.tile = (int)(ws / (uint32_t)p.kb_per_tile);
            c.kb = (int)(ws - (uint32_t)c.tile * (uint32_t)p.kb_per_tile);
            c.from_start = (c.kb == 0);
            c.first_tile = true;
            StageCursor cm{c.tile, c.kb, nunits};
            const int lm_q = lane >> 3, lm_r = lane & 7;
            const T* Aact = static_cast<const T*>(p.A);
            bool ok = true;
            int consumed = 0;
            uint32_t bw[S::NJ][2][4], bwn[S::NJ][2][4];
            auto load_act = [&](int kunit, uint32_t(&dst)[S::NJ][2][4]) {
#pragma unroll
                for (int jj = 0; jj < S::NJ; ++jj) {
                    const int m = 8 * jj + g;
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch) {
                        if (m < p.M) {
                            const uint4 v = ldg_v4(Aact + (size_t)m * p.K + kunit + 32 * ch + 8 * tq);
                            dst[jj][ch][0] = v.x;
                            dst[jj][ch][1] = v.y;
                            dst[jj][ch][2] = v.z;
                            dst[jj][ch][3] = v.w;
                        } else {
                            dst[jj][ch][0] = dst[jj][ch][1] = dst[jj][ch][2] = dst[jj][ch][3] = 0u;
                        }
                    }
                }
            };
            load_act(c.kb * S::SB, bw);
            while (cm.left > 0) {
                int tile, kb0, kb, n;
                next_stage<UPS>(cm, p.kb_per_tile, tile, kb0, kb, n);
                const int slot = consumed % D;
                const uint32_t st = stage_addr(warp * D + slot);
                if (!wait_stage(full_bar(warp, slot), (uint32_t)(consumed / D) & 1u)) {
                    ok = false;
                    break;
                }
                const int x0 = (kb0 >> p.am_shift) & ~3;
#pragma unroll
                for (int j = 0; j < UPS; ++j) {
                    if (kb0 + j < kb || kb0 + j >= kb + n) continue;
                    if (kb0 + j + 1 < kb + n)
                        load_act((kb0 + j + 1) * S::SB, bwn);
                    else if (cm.left > 0)
                        load_act(cm.kb * S::SB, bwn);
                    const int col = BS64 ? (kb0 + j - x0) : (((kb0 + j) >> p.am_shift) - x0);
                    const uint32_t am_base = st + G::WEIGHT_BYTES + (uint32_t)col * 4u;
                    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int i = 0; i < S::TW; ++i) {
                        uint32_t d0, d1, d2, d3;
                        ldmatrix_x4(G::chunk_addr(st, 16 * i + 8 * (lm_q & 1) + lm_r, 2 * j + (lm_q >> 1)), d0, d1, d2,
                                    d3);
                        const float ag = lds_f32(am_base + (uint32_t)(16 * i + g) * 16u);
                        const float ag8 = lds_f32(am_base + (uint32_t)(16 * i + 8 + g) * 16u);
                        float t[S::NJ][4];
                        uint32_t a0, a1, a2, a3;
                        a0 = lut_pair<0>(d0, lane4); a2 = lut_pair<1>(d0, lane4);
                        a1 = lut_pair<0>(d1, lane4); a3 = lut_pair<1>(d1, lane4);
#pragma unroll
                        for (int jj = 0; jj < S::NJ; ++jj) mma16816<T>(t[jj], a0, a1, a2, a3, bw[jj][0][0], bw[jj][0][1], zero);
                        a0 = lut_pair<2>(d0, lane4); a2 = lut_pair<3>(d0, lane4);
                        a1 = lut_pair<2>(d1, lane4); a3 = lut_pair<3>(d1, lane4);
#pragma unroll
                        for (int jj = 0; jj < S::NJ; ++jj) mma16816<T>(t[jj], a0, a1, a2, a3, bw[jj][0][2], bw[jj][0][3], t[jj]);
                        a0 = lut_pair<0>(d2, lane4); a2 = lut_pair<1>(d2, lane4);
                        a1 = lut_pair<0>(d3, lane4); a3 = lut_pair<1>(d3, lane4);
#pragma unroll
                        for (int jj = 0; jj < S::NJ; ++jj) mma16816<T>(t[jj], a0, a1, a2, a3, bw[jj][1][0], bw[jj][1][1], t[jj]);
                        a0 = lut_pair<2>(d2, lane4); a2 = lut_pair<3>(d2, lane4);
                        a1 = lut_pair<2>(d3, lane4); a3 = lut_pair<3>(d3, lane4);
#pragma unroll
                        for (int jj = 0; jj < S::NJ; ++jj) mma16816<T>(t[jj], a0, a1, a2, a3, bw[jj][1][2], bw[jj][1][3], t[jj]);
#pragma unroll
                        for (int jj = 0; jj < S::NJ; ++jj) {
                            acc[i][jj][0] = fmaf(ag, t[jj][0], acc[i][jj][0]);
                            acc[i][jj][1] = fmaf(ag, t[jj][1], acc[i][jj][1]);
                            acc[i][jj][2] = fmaf(ag8, t[jj][2], acc[i][jj][2]);
                            acc[i][jj][3] = fmaf(ag8, t[jj][3], acc[i][jj][3]);
                        }
                    }
                    finish_unit_tma<T, S>(acc, has_first, has_last, c, cm.left == 0 && kb0 + j + 1 == kb + n, p, lut,
                                          warp, lane, g, tq);
#pragma unroll
                    for (int jj = 0; jj < S::NJ; ++jj)
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch)
#pragma unroll
                            for (int w = 0; w < 4; ++w) bw[jj][ch][w] = bwn[jj][ch][w];
                }
                // hand the stage back to the producer
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(warp, slot));
                ++consumed;
            }
            if (!ok) {
                if (lane == 0) atomicExch(p.error, kErrWaitTimeout);
                for (int k = 0; k < D; ++k)  // drain whatever the producer may still have in flight
                    wait_stage(full_bar(warp, (consumed + k) % D), (uint32_t)((consumed + k) / D) & 1u);
            }
        }
    }
    __syncthreads();  // every warp is out of the stage ring: the slots may reuse it
    if (!producer) {
        if (has_first) {
            float first[S::TW][S::NJ][4];
#pragma unroll
            for (int i = 0; i < S::TW; ++i)
#pragma unroll
                for (int j = 0; j < S::NJ; ++j)
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        first[i][j][r] = lds_f32(parked_addr<S>(lut, warp, (i * S::NJ + j) * 4 + r, lane));
            store_slot<S>(first, slots, warp * 2, lane);
        }
        if (has_last) store_slot<S>(acc, slots, warp * 2 + 1, lane);
    }
    __syncthreads();
    if (uc <= 0 || producer) return;
    combine_tiles<T, S>(p, slots, cs, ce, warp, lane, g, tq);
}

// ---------------------------------------------------------------------------
// Host launchers: the table of compiled variants.
// ---------------------------------------------------------------------------
template <typename T, class S>
static cudaError_t launch_mma(const GemmParams& p, cudaStream_t stream) {
    auto kern = q4_gemm_mma_kernel<T, S>;
    cudaError_t e = ensure_smem_attr((const void*)kern, S::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.ctas);
    cfg.blockDim = dim3(S::NW * 32);
    cfg.dynamicSmemBytes = S::SMEM_BYTES;
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

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda; the driver is already loaded by the runtime).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        else
            cudaGetLastError();
    });
    return fn;
}

// Weights: [N rows][K/2 bytes], box `rows` rows x (32 * UPS) bytes, 64/128-byte swizzle.
// Absmax: [N rows][K/bs floats], box `rows` rows x 4 floats.
static cudaError_t make_tensor_maps(const GemmParams& p, int ups, int rows, CUtensorMap* tw, CUtensorMap* ta) {
    auto enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint32_t estride[2] = {1, 1};
    const cuuint64_t wdim[2] = {(cuuint64_t)(p.K / 2), (cuuint64_t)p.N};
    const cuuint64_t wstride[1] = {(cuuint64_t)(p.K / 2)};
    const cuuint32_t wbox[2] = {(cuuint32_t)(32 * ups), (cuuint32_t)rows};
    if (enc(tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p.Wp), wdim, wstride, wbox, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, ups == 4 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            // no promotion past the box: a wider L2 fill would take the next
            // stage's bytes, which at a warp boundary belong to another warp
            // that reads them much later (by then evicted, so read twice)
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const cuuint64_t adim[2] = {(cuuint64_t)p.am_per_row, (cuuint64_t)p.N};
    const cuuint64_t astride[1] = {(cuuint64_t)p.am_per_row * 4};
    const cuuint32_t abox[2] = {4, (cuuint32_t)rows};
    if (enc(ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p.absmax), adim, astride, abox, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    return cudaSuccess;
}

static int max_dynamic_smem() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return v;
}

template <typename T, class S, int UPS>
static cudaError_t launch_tma(const GemmParams& p, cudaStream_t stream) {
    CUtensorMap tw, ta;
    cudaError_t e = make_tensor_maps(p, UPS, S::TR, &tw, &ta);
    if (e != cudaSuccess) return e;
    const int smem = max_dynamic_smem();  // the kernel lays out LUT, barriers and stages itself
    if (smem <= 0) return cudaErrorInvalidValue;
    auto kern = p.am_shift == 0 ? q4_gemm_tma_kernel<T, S, UPS, true> : q4_gemm_tma_kernel<T, S, UPS, false>;
    if ((e = ensure_smem_attr((const void*)kern, (size_t)smem)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.ctas);
    cfg.blockDim = dim3(S::NW * 32);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, tw, ta, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename T, class S, int UPS>
static cudaError_t launch_ws(const GemmParams& p, cudaStream_t stream) {
    CUtensorMap tw, ta;
    cudaError_t e = make_tensor_maps(p, UPS, S::TR, &tw, &ta);
    if (e != cudaSuccess) return e;
    const int smem = max_dynamic_smem();
    if (smem <= 0) return cudaErrorInvalidValue;
    auto kern = p.am_shift == 0 ? q4_gemm_ws_kernel<T, S, UPS, true> : q4_gemm_ws_kernel<T, S, UPS, false>;
    if ((e = ensure_smem_attr((const void*)kern, (size_t)smem)) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.ctas);
    cfg.blockDim = dim3((S::NW + 1) * 32);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, tw, ta, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

struct Variant {
    int act, loader, sub_block, m_pad, warps, depth, l2pf;
    size_t smem;
    cudaError_t (*launch)(const GemmParams&, cudaStream_t);
};

// Per-lane global loads (loader 1): the depth is the register ring, l2pf the L2 fetch hint.
#define Q4_VARIANT(ACT, T, SB, MP, NW, D, PF)                                                  \
    Variant {                                                                                 \
        ACT, 1, SB, MP, NW, D, PF, GemmShape<SB, MP, 4, NW, D, PF>::SMEM_BYTES,               \
            &launch_mma<T, GemmShape<SB, MP, 4, NW, D, PF>>                                   \
    }
// TMA stage rings: loader 2 = 4-unit (128-byte) stages, loader 3 = 2-unit
// (64-byte) stages; the depth is the number of stages per warp.
#define Q4_TMA_VARIANT(ACT, T, MP, NW, D)                                                      \
    Variant {                                                                                 \
        ACT, 2, 64, MP, NW, D, 0, 0, &launch_tma<T, GemmShape<64, MP, 4, NW, D, 0>, 4>         \
    }
// loader 3 with 32-row tiles (two 16-row MMA tiles per unit): 17 <= M <= 32
#define Q4_TMA2_R32_VARIANT(ACT, T, MP, NW, D)                                                 \
    Variant {                                                                                 \
        ACT, 3, 64, MP, NW, D, 0, 0, &launch_tma<T, GemmShape<64, MP, 2, NW, D, 0>, 2>         \
    }
#define Q4_TMA2_VARIANT(ACT, T, MP, NW, D)                                                     \
    Variant {                                                                                 \
        ACT, 3, 64, MP, NW, D, 0, 0, &launch_tma<T, GemmShape<64, MP, 4, NW, D, 0>, 2>         \
    }

// Warp-specialised rings: loader 4 = 4-unit stages, loader 5 = 2-unit stages;
// `warps` counts the consumer warps (plus one producer warp).
#define Q4_WS_VARIANT(ACT, T, MP, NW, D)                                                       \
    Variant {                                                                                 \
        ACT, 4, 64, MP, NW, D, 0, 0, &launch_ws<T, GemmShape<64, MP, 4, NW, D, 0>, 4>          \
    }
#define Q4_WS2_VARIANT(ACT, T, MP, NW, D)                                                      \
    Variant {                                                                                 \
        ACT, 5, 64, MP, NW, D, 0, 0, &launch_ws<T, GemmShape<64, MP, 4, NW, D, 0>, 2>          \
    }

#define Q4_VARIANTS_FOR(ACT, T)                                                                \
    Q4_VARIANT(ACT, T, 64, 8, 16, 1, 128), Q4_VARIANT(ACT, T, 64, 8, 8, 2, 128),               \
        Q4_VARIANT(ACT, T, 64, 16, 8, 1, 128), Q4_VARIANT(ACT, T, 32, 8, 16, 1, 128),         \
        Q4_VARIANT(ACT, T, 32, 16, 8, 1, 128), Q4_TMA_VARIANT(ACT, T, 8, 8, 2),               \
        Q4_TMA_VARIANT(ACT, T, 16, 8, 2), Q4_TMA2_VARIANT(ACT, T, 8, 16, 2),                  \
        Q4_TMA2_VARIANT(ACT, T, 16, 8, 4), Q4_WS_VARIANT(ACT, T, 8, 8, 2), Q4_WS_VARIANT(ACT, T, 16, 8, 2), \
        Q4_TMA2_R32_VARIANT(ACT, T, 32, 8, 6)

static const Variant kVariants[] = {
    Q4_VARIANTS_FOR(0, __nv_bfloat16),
    Q4_VARIANTS_FOR(1, __half),
    // measurement-only variants of the main M<=8, blocksize-64, bf16 case
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 16, 1, 0),
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 16, 1, 256),
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 8, 2, 0),
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 8, 1, 128),
    Q4_TMA_VARIANT(0, __nv_bfloat16, 8, 16, 1),
    Q4_TMA_VARIANT(0, __nv_bfloat16, 8, 12, 1),
    Q4_TMA2_VARIANT(0, __nv_bfloat16, 8, 8, 4),
    Q4_TMA2_VARIANT(0, __nv_bfloat16, 8, 12, 2),
    Q4_TMA2_VARIANT(0, __nv_bfloat16, 8, 16, 1),
    Q4_WS_VARIANT(0, __nv_bfloat16, 8, 16, 1),
    Q4_WS_VARIANT(0, __nv_bfloat16, 8, 12, 1),
    Q4_WS2_VARIANT(0, __nv_bfloat16, 8, 16, 2),
    Q4_WS2_VARIANT(0, __nv_bfloat16, 8, 8, 4),
};

static const Variant* find_variant(int act, const GemmChoice& ch) {
    for (const Variant& v : kVariants)
        if (v.act == act && v.loader == ch.loader && v.sub_block == ch.sub_block && v.m_pad == ch.m_pad &&
            v.warps == ch.warps && v.depth == ch.depth && (ch.loader >= 2 || v.l2pf == ch.l2pf))
            return &v;
    return nullptr;
}

// Loader 7 is the row-split kernel (q4_rows.cu): bf16/fp16, 64-k units,
// one, two or four n8 column tiles, the stage ring sized from shared memory.
static bool rows_variant(int act_dtype, const GemmChoice& ch) {
    return ch.loader == 7 && (act_dtype == 0 || act_dtype == 1) && ch.sub_block == 64 &&
           (ch.m_pad == 8 || ch.m_pad == 16 || ch.m_pad == 32) && ch.warps == rows_warps();
}

bool gemm_variant_exists(int act_dtype, const GemmChoice& ch) {
    return rows_variant(act_dtype, ch) || find_variant(act_dtype, ch) != nullptr;
}

size_t gemm_smem_bytes(int act_dtype, const GemmChoice& ch) {
    if (rows_variant(act_dtype, ch)) return (size_t)max_dynamic_smem();
    const Variant* v = find_variant(act_dtype, ch);
    if (!v) return 0;
    return v->loader >= 2 ? (size_t)max_dynamic_smem() : v->smem;
}

cudaError_t gemm_launch(const GemmChoice& ch, int act_dtype, const GemmParams& p, cudaStream_t stream) {
    const Variant* v = find_variant(act_dtype, ch);
    if (!v) return cudaErrorInvalidConfiguration;
    return v->launch(p, stream);
}

size_t gemm_slot_floats(int m_pad) { return (size_t)4 * (m_pad / 8) * 4 * 32; }

}  // namespace q4
