// q4_rows.cu -- row-split fused dequantize + skinny GEMM for sm_100a, M <= 16
// (the launch table's default there), and up to 32 on request.
//
//     out[m, n] = sum_k A[m, k] * code[idx(n, k)] * absmax(n, k)
//
// The operation of bitsandbytes PR #1920 ("[ROCm] Optimize
// kgemm_4bit_inference_naive ...", "Technical details" and "Fused path
// support for M > 1"), with the same inner step as the stream-K kernel in
// q4_gemm.cu (byte-pair table lookups feeding mma.sync m16n8k16 with the
// matrix roles swapped, fp32 absmax applied once per 64-k block, or per
// 32-k half at blocksize 32), organised so that a launch carries no
// cross-CTA work at all:
//
//  * Rows, not units, are split over the CTAs.  CTA c owns a contiguous run
//    of whole weight rows (8-row groups; the larger shares go to the lowest
//    block indices, which the hardware places first), so every output
//    element is finished inside one CTA: no partial sums in global memory,
//    no counters, no last-arriver fix-up at the end of the launch.  The
//    shares differ by at most one 8-row group.
//  * A CTA's rows form tiles of nearly equal height (the larger heights
//    first; at most 72 rows with one MMA column tile, 64 with two or with
//    contiguous ranges, 56 at blocksize 32, 32 with four column tiles).  A
//    stage is one tile's rows x 256 k of packed codes (128-byte swizzle)
//    plus its absmax box: one TMA box each, one tensor-map pair per height.
//  * The stages stream through one ring of D = 16 mbarrier-guarded slots.
//    Round robin (the default): warp w computes stages w, w + 8, w + 16, ...
//    from slots w and w + 8, and after copying a stage into registers (code
//    fragments and absmax) refills the slot with the stage 16 further on,
//    which is its own again -- no producer warp, no "slot free" barriers,
//    every slot is prefetch depth.  Each warp's first two copies are issued
//    by its own lanes right after they set up its slots' barriers.
//  * The stages of a tile run in a loop instantiated for the tile's shape
//    (16-row MMA tiles, half last tile), dispatched once per tile: each
//    stage is one straight-line block in which the four units' lookup and
//    MMA chains interleave; rows past a half tile do no lookups.
//  * Each warp sums its stages of a tile in registers; when it leaves the
//    tile it parks the partial tile in shared memory (the lookup table's
//    free row halves), and the last warp to do so adds the parked partials
//    in stage order (deterministic) and stores the tile.  An exact count of
//    reduced tiles guards the reuse of the parking space (two buffers with
//    contiguous ranges, one with round robin).
//  * Under programmatic dependent launch (mode 2) the weights are static:
//    the ring's first fill (and, optionally, an L2 prefetch of the stages
//    after it) goes out before the dependency wait, and the table is built
//    meanwhile.  Activations and outputs are touched only after the wait.
//  * Every wait is bounded; on time-out the kernel sets the workspace error
//    word, waits (bounded) for the copies it issued and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstring>
#include <type_traits>

#include "q4_device.cuh"
#include "q4_internal.h"
#include "q4_plan.cuh"

namespace q4 {
namespace rows {

constexpr int kW = 8;                // warps per CTA
constexpr int kThreads = kW * 32;
constexpr uint32_t kBarBytes = 512;  // mbarriers and small words at the start of the window

// Absmax granularity of a kernel instance: one block per stage or more
// (blocksize >= 128), one per 64-k unit (blocksize 64), two per unit
// (blocksize 32).
enum : int { kAmShared = 0, kAm64 = 1, kAm32 = 2 };

// Compile-time shape of the kernel for NJ n8 column tiles (M <= 8 or 16),
// stage order (CONTIG: each warp streams a contiguous range of stages;
// else round robin) and absmax granularity AMK.
template <int NJ, bool CONTIG, int AMK>
struct Geo {
    // Tallest tile.  Round robin with one column tile: 72 rows (a CTA of
    // 8q + 1 groups then needs no short tiles).  Contiguous ranges keep
    // several tiles open at once and need two parking buffers: 64 rows.
    // Blocksize 32 doubles the absmax box: 56 rows keep 16 slots in the
    // window.  Four column tiles (17 <= M <= 32): 32 rows, so that the
    // partial tiles (32 registers a warp) still fit the parking space.
    static constexpr int MAX_ROWS = NJ == 4 ? 32 : AMK == kAm32 ? 56 : (NJ == 1 && !CONTIG) ? 72 : 64;
    static constexpr int MT_MAX = (MAX_ROWS + 15) / 16;       // 16-row MMA tiles per stage, at most
    static constexpr uint32_t AMW = AMK == kAm32 ? 32u : 16u; // absmax bytes per row and stage (8 or 4 floats)
    static constexpr uint32_t CODE_BYTES = MAX_ROWS * 128u;   // a stage's codes: rows x 128 B (4 units of 64 k)
    static constexpr uint32_t AM_BYTES = MAX_ROWS * AMW;      // its absmax box
    // With 72-row tiles the codes (9 KiB, 1 KiB aligned for the swizzle) and
    // the absmax boxes live in separate rings, and the barriers in spare
    // table rows; otherwise a slot holds both (padded to 1 KiB: 9 KiB) and
    // the barriers sit at the start of the window.
    static constexpr bool SPLIT = MAX_ROWS == 72;
    static constexpr uint32_t SLOT = (CODE_BYTES + AM_BYTES + 1023u) & ~1023u;
    static constexpr int REGS = MT_MAX * 4 * NJ;              // a warp's partial tile: registers per lane
    // Ring depth: a compile-time constant, so that slot and phase of a stage
    // are a mask and a shift.
    static constexpr int D = 16;
    static constexpr int R = D / kW;                          // slots per warp with contiguous ranges
    // Parking buffers for partial tiles, in the table's free upper row
    // halves (256 rows of 128 B); with the split layout, rows PARK_ROWS and
    // PARK_ROWS + 1 hold the barriers and small words.
    static constexpr int NB = CONTIG ? 2 : 1;
    static constexpr int PARK_ROWS = NB * kW * REGS;
    static_assert(PARK_ROWS + (SPLIT ? 2 : 0) <= 256, "parking buffers must fit the table's free halves");
    static_assert(!SPLIT || D * 8 <= 128, "the full barriers fill one spare row");
    static_assert(2 * (MAX_ROWS / 8) + 2 <= 32 && kRowsMaxMaps <= 4, "map_bits holds a 2-bit pair index per h / 8");
};

// Tensor-map pair of tile height h.
__device__ __forceinline__ int map_index(const RowsParams& p, int h) { return (int)((p.map_bits >> (2 * (h >> 3))) & 3u); }

// Position of stage i in the CTA's work: tile `tile` (rows [y, y + h) of the
// CTA's rows), k-stage `s` (columns [256 s, 256 s + 256)).
struct Stage {
    int tile, s, y, h;
};

// The CTA's share and the order of its stages (identical in every thread):
// ng 8-row groups in T = ceil(ng / gmax) tiles, the first `extra` tiles one
// group taller; tile-major, k-stages in order.
struct Plan {
    int row0;  // first weight row of the CTA
    int T, S;  // tiles, k-stages per tile
    int base, extra;
    int n_total;

    __device__ __forceinline__ void init(const RowsParams& p, int cta, int gmax) {
        const int q = p.groups / p.ctas, r = p.groups - q * p.ctas;
        const int g0 = cta < r ? cta * (q + 1) : r * (q + 1) + (cta - r) * q;
        const int ng = q + (cta < r ? 1 : 0);
        row0 = 8 * g0;
        T = (ng + gmax - 1) / gmax;
        base = ng / T;
        extra = ng - base * T;
        S = p.K >> 8;
        n_total = T * S;
    }
    __device__ __forceinline__ int tile_rows(int t) const { return 8 * (base + (t < extra ? 1 : 0)); }
    __device__ __forceinline__ int tile_y(int t) const { return 8 * (t * base + min(t, extra)); }
};

// A warp's position in the stage sequence, advanced by `stride` stages at
// a time without divisions.
struct Cur {
    int i, t, s;
    __device__ __forceinline__ void init(const Plan& pl, int i0) {
        i = i0;
        t = i0 / pl.S;
        s = i0 - t * pl.S;
    }
    __device__ __forceinline__ void step(const Plan& pl, int stride) {
        i += stride;
        s += stride;
        while (s >= pl.S) {
            s -= pl.S;
            ++t;
        }
    }
    __device__ __forceinline__ Stage stage(const Plan& pl) const {
        Stage st;
        st.tile = t;
        st.s = s;
        st.h = pl.tile_rows(t);
        st.y = pl.tile_y(t);
        return st;
    }
};

// Parking slot of register `r` of warp `w`'s partial tile in buffer `b`:
// the upper (free) half of table row (b W + w) REGS + r, lane-major.
template <class G>
__device__ __forceinline__ uint32_t park_addr(uint32_t lut, int b, int w, int r, int lane) {
    constexpr int REGS = G::REGS;
    return lut + (uint32_t)((b * kW + w) * REGS + r) * 256u + 128u + (uint32_t)lane * 4u;
}

// Tensor maps of the launch: per box height h (8 .. 72 rows), one map of
// the packed codes (h rows x 128 bytes, 128-byte swizzle) and one of the
// absmax (h rows x 4 floats); map_index(p, h) selects the pair.
struct RowsMaps {
    CUtensorMap w[kRowsMaxMaps];
    CUtensorMap a[kRowsMaxMaps];
};

template <typename T, int NJ, int AMK, bool CONTIG>
__global__ void __launch_bounds__(kThreads, 1)
    q4_gemm_rows_kernel(const __grid_constant__ RowsParams p, const __grid_constant__ RowsMaps maps) {
    using G = Geo<NJ, CONTIG, AMK>;
    constexpr int D = G::D, MTM = G::MT_MAX, NB = G::NB;
    extern __shared__ __align__(16) uint8_t smem_rows[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
    // Long-latency first touches go out first: the tensor maps (read by the
    // first copies; every slot holds a valid map, so no parameter has to
    // arrive before the prefetch) and the code table (read by the table
    // build).
    if (tid < kRowsMaxMaps) {
        prefetch_tensormap(&maps.w[tid]);
        prefetch_tensormap(&maps.a[tid]);
    }
    const float cv = __ldg(p.code + (lane & 15));

    // Shared-memory layout (from the window base, decided at run time):
    // barriers and small words; ring slots below the 64 KiB-aligned table;
    // the table (its upper row halves hold the parking buffers); ring slots
    // above it.
    const uint32_t sbase = smem_addr(smem_rows);
    const uint32_t send = sbase + dynamic_smem_size();
    const uint32_t lut = (sbase + 0xFFFFu) & ~0xFFFFu;
    uint32_t bars, words, a0, b0, na, nb, am_a = 0, am_b = 0, nam_a = 0;
    bool room;
    if constexpr (G::SPLIT) {
        // barriers and words in the spare table rows; codes slots (1 KiB
        // aligned) below the table, then above it; absmax boxes in what is
        // left of the two regions.
        bars = lut + (uint32_t)G::PARK_ROWS * 256u + 128u;
        words = bars + 256u;
        a0 = (sbase + 1023u) & ~1023u;
        b0 = lut + kLutBytes;
        na = a0 < lut ? min((lut - a0) / G::CODE_BYTES, (uint32_t)D) : 0u;
        nb = (uint32_t)D - na;
        am_a = a0 + na * G::CODE_BYTES;
        nam_a = am_a < lut ? (lut - am_a) / G::AM_BYTES : 0u;
        am_b = b0 + nb * G::CODE_BYTES;
        room = am_b <= send && nam_a + (send - am_b) / G::AM_BYTES >= (uint32_t)D;
    } else {
        // barriers below the table when there is room there, else right
        // after it; code + absmax slots below and above the table.
        const bool bars_low = lut >= sbase + kBarBytes;
        bars = bars_low ? sbase : lut + kLutBytes;
        words = bars + (uint32_t)D * 8u;
        a0 = bars_low ? (sbase + kBarBytes + 1023u) & ~1023u : lut;
        b0 = bars_low ? lut + kLutBytes : lut + kLutBytes + 1024u;
        na = a0 < lut ? (lut - a0) / G::SLOT : 0u;
        nb = (send > b0) ? (send - b0) / G::SLOT : 0u;
        room = b0 <= send && na + nb >= (uint32_t)D;
    }
    if (!room) {  // the host sized the launch wrongly
        if (tid == 0 && p.error) atomicExch(p.error, kErrNoRoom);
        return;
    }
    auto slot_addr = [&](int k) -> uint32_t {  // the codes of ring slot k
        constexpr uint32_t stride = G::SPLIT ? G::CODE_BYTES : G::SLOT;
        return (uint32_t)k < na ? a0 + (uint32_t)k * stride : b0 + ((uint32_t)k - na) * stride;
    };
    auto am_addr = [&](int k) -> uint32_t {  // the absmax box of ring slot k
        if constexpr (G::SPLIT)
            return (uint32_t)k < nam_a ? am_a + (uint32_t)k * G::AM_BYTES : am_b + ((uint32_t)k - nam_a) * G::AM_BYTES;
        else
            return slot_addr(k) + G::CODE_BYTES;
    };
    auto full_bar = [&](int k) -> uint32_t { return bars + (uint32_t)k * 8u; };
    const uint32_t reduced = words;                                   // [2] ints: tiles reduced per parking buffer
    const uint32_t counters = reduced + 8u;                           // [2] ints: parked partials per buffer
    const uint32_t last_issued = counters + 8u;                       // [D] ints: phase + 1 of the newest copy per slot
    const uint32_t failed = last_issued + 4u * (uint32_t)D;           // int: a wait of this CTA ran out

    if (p.pdl == 1) griddep_wait();

    Plan pl;
    pl.init(p, blockIdx.x, G::MAX_ROWS / 8);
    const uint64_t once = l2_evict_first();  // the codes are read exactly once

    // This warp's stages.  Round robin (the default): stages warp, warp + W,
    // ... through the shared ring, slot i % D.  Contiguous: the warp's own
    // balanced range [ws, we) through its own R slots.
    constexpr bool rr = !CONTIG;
    const int ws = rr ? warp : (int)(((uint32_t)pl.n_total * (uint32_t)warp) / kW);
    const int we = rr ? pl.n_total : (int)(((uint32_t)pl.n_total * (uint32_t)(warp + 1)) / kW);
    const int stride = rr ? kW : 1, ahead = rr ? D : G::R;
    auto slot_of = [&](int i) -> int { return rr ? (i & (D - 1)) : warp * G::R + ((i - ws) & (G::R - 1)); };
    auto phase_of = [&](int i) -> uint32_t {
        return rr ? (uint32_t)(i / D) & 1u : (uint32_t)((i - ws) / G::R) & 1u;
    };

    // Lane 0 of the calling warp loads stage i (at `st`) into its ring slot.
    auto issue = [&](int i, const Stage& st) {
        if (i == p.skip_stage) return;  // test hook: this stage's barrier never completes
        const int k = slot_of(i), mi = map_index(p, st.h);
        const uint32_t dst = slot_addr(k);
        const int y = pl.row0 + st.y;
        sts_u32(last_issued + 4u * (uint32_t)k, phase_of(i) + 1u);
        mbar_expect_tx(full_bar(k), (uint32_t)st.h * (128u + G::AMW));
        tma_load_2d_hint(dst, &maps.w[mi], st.s * 128, y, full_bar(k), once);
        tma_load_2d(am_addr(k), &maps.a[mi], AMK == kAm32 ? st.s * 8 : ((st.s * 4) >> p.am_shift) & ~3, y,
                    full_bar(k));
    };
    // The ring's first fill.  The weights are static, so under dependent
    // launch mode 2 these copies (and the optional L2 prefetch of the stages
    // after them) overlap the previous kernel.  Every slot belongs to one
    // warp (round robin: slots w and w + W; contiguous: the warp's R slots),
    // so lane j of each warp sets up its j-th slot and loads the warp's j-th
    // stage into it at once, with no CTA-wide barrier in between; the
    // barrier after the table build publishes the rest.
    {
        const int i = ws + lane * stride;
        if (lane < (rr ? D / kW : G::R)) {
            const int k = rr ? warp + kW * lane : warp * G::R + lane;  // = slot_of(i)
            mbar_init(full_bar(k), 1);
            sts_u32(last_issued + 4u * (uint32_t)k, 0u);
            mbar_init_fence();
            if (i < we && i < (rr ? D : we)) {
                Cur c;
                c.init(pl, i);
                issue(i, c.stage(pl));
            }
        }
        if (tid == 0) {
            sts_u32(reduced, 0u);
            sts_u32(reduced + 4u, 0u);
            sts_u32(counters, 0u);
            sts_u32(counters + 4u, 0u);
            sts_u32(failed, 0u);
        }
        griddep_launch_dependents();
        if (warp == 0 && lane == 0 && p.l2_ahead > 0) {
            const int end = min(pl.n_total, D + p.l2_ahead);
            for (int j = D; j < end; ++j) {
                Cur c;
                c.init(pl, j);
                const Stage sj = c.stage(pl);
                tma_prefetch_l2_2d(&maps.w[map_index(p, sj.h)], sj.s * 128, pl.row0 + sj.y);
            }
        }
    }
    __syncwarp();

    build_lut<T>(lut, cv, tid, kW * 32);
    __syncthreads();
    if (p.pdl == 2) griddep_wait();  // activations and outputs may belong to the preceding grid

    const uint32_t lane4 = lut | ((uint32_t)lane << 2);
    const int lm_q = lane >> 3, lm_r = lane & 7;
    const T* Aact = static_cast<const T*>(p.A);
    T* out = static_cast<T*>(p.out);
    const T* bias = static_cast<const T*>(p.bias);

    // Activations of AU units of this warp's stages (NJ column tiles x two
    // 16-byte runs each), refilled unit by unit with the unit AU further
    // on: the whole stage ahead with one column tile; half a stage with two
    // (or at blocksize 32), whose registers would otherwise crowd out the
    // accumulators (spills).
    constexpr int AU = (NJ == 1 && AMK != kAm32) ? 4 : 2;
    uint32_t aw[AU][NJ][2][4];
    auto load_unit = [&](int kbu, uint32_t(&dst)[NJ][2][4]) {
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj) {
            const int m = 8 * jj + g;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                if (m < p.M) {
                    const uint4 v = ldg_v4(Aact + (size_t)m * p.K + kbu * 64 + 32 * ch + 8 * tq);
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

    float acc[MTM][NJ][4];
#pragma unroll
    for (int i = 0; i < MTM; ++i)
#pragma unroll
        for (int jj = 0; jj < NJ; ++jj)
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[i][jj][r] = 0.f;

    // The warps holding a partial of tile t, in stage order: the span
    // [w_first, w_first + n) modulo W.  Round robin: every warp of the span.
    // Contiguous: the warps whose (non-empty) ranges meet the tile's stages.
    auto tile_warps = [&](int t, int& w_first, int& n) {
        const int f = t * pl.S, l = f + pl.S - 1;
        if (rr) {
            w_first = f & (kW - 1);
            n = min(kW, pl.S);
        } else {
            w_first = (int)part_owner((uint32_t)pl.n_total, kW, (uint32_t)f);
            n = (int)part_owner((uint32_t)pl.n_total, kW, (uint32_t)l) - w_first + 1;
        }
    };
    auto holds_partial = [&](int w) -> bool {  // (within a tile's span)
        return rr || part_start((uint32_t)pl.n_total, kW, (uint32_t)w) !=
                         part_start((uint32_t)pl.n_total, kW, (uint32_t)(w + 1));
    };

    // Leaves tile t: park the partial, and if this warp is the last of the
    // tile's contributors, add all parked partials in stage order and store.
    auto flush = [&](int t) -> bool {
        const int b = NB == 1 ? 0 : (t & 1);
        // The buffer's previous tile (t - NB) must have been reduced: an
        // exact count, since a warp that holds no part of the tiles between
        // may arrive here several reductions ahead (a phase parity would
        // alias).
        if (t >= NB && !wait_count_at_least(reduced + 4u * (uint32_t)b, (uint32_t)(t / NB), p.wait_limit))
            return false;
#pragma unroll
        for (int i = 0; i < MTM; ++i)
#pragma unroll
            for (int jj = 0; jj < NJ; ++jj)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    sts_f32(park_addr<G>(lut, b, warp, (i * NJ + jj) * 4 + r, lane), acc[i][jj][r]);
                    acc[i][jj][r] = 0.f;
                }
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atom_add_acq_rel_cta_smem(counters + 4u * (uint32_t)b, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        __syncwarp();  // the other lanes read after lane 0's acquire
        int w0, span, nc = 0;
        tile_warps(t, w0, span);
        for (int c = 0; c < span; ++c) nc += holds_partial((w0 + c) & (kW - 1)) ? 1 : 0;
        if (old != nc - 1) return true;
        float sum[MTM][NJ][4];
#pragma unroll
        for (int i = 0; i < MTM; ++i)
#pragma unroll
            for (int jj = 0; jj < NJ; ++jj)
#pragma unroll
                for (int r = 0; r < 4; ++r) sum[i][jj][r] = 0.f;
        for (int c = 0; c < span; ++c) {
            const int w = (w0 + c) & (kW - 1);
            if (!holds_partial(w)) continue;
#pragma unroll
            for (int i = 0; i < MTM; ++i)
#pragma unroll
                for (int jj = 0; jj < NJ; ++jj)
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        sum[i][jj][r] += lds_f32(park_addr<G>(lut, b, w, (i * NJ + jj) * 4 + r, lane));
        }
        const int rows_t = pl.tile_rows(t), y_t = pl.tile_y(t);
#pragma unroll
        for (int i = 0; i < MTM; ++i)
#pragma unroll
            for (int jj = 0; jj < NJ; ++jj)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int rt = 16 * i + g + ((r & 2) ? 8 : 0);
                    const int n = pl.row0 + y_t + rt;
                    const int m = 8 * jj + 2 * tq + (r & 1);
                    if (rt < rows_t && n < p.N && m < p.M) {
                        const float bv = bias ? static_cast<float>(bias[n]) : 0.f;  // exact widening
                        out[(size_t)m * p.N + n] = Act<T>::from_float(sum[i][jj][r] + bv);
                    }
                }
        __syncwarp();
        if (lane == 0) {
            sts_u32(counters + 4u * (uint32_t)b, 0u);
            red_add_release_cta_smem(reduced + 4u * (uint32_t)b, 1u);  // the buffer may be refilled
        }
        return true;
    };

    bool ok = true;
    Cur cc, ci;  // the stage this warp computes next, and the one it loads into the slot it frees
    cc.init(pl, ws);
    ci.init(pl, ws + ahead);

    // This warp's stages of one tile (MT 16-row MMA tiles, the last of them
    // half when HALF), starting at cc: one tight loop per tile shape.  The
    // dispatch on the shape happens once per tile, outside the loop, so the
    // loop body stays one straight-line block in which the four units'
    // lookup and MMA chains interleave.
    auto run_tile = [&](auto mt_c, auto half_c) -> bool {
        constexpr int MT = decltype(mt_c)::value;
        constexpr bool HALF = decltype(half_c)::value;
        const int tile = cc.t;
        while (true) {
            const int i = cc.i, k = slot_of(i);
            const int s_cur = cc.s;
            const uint32_t st_addr = slot_addr(k);
            if (!wait_stage(full_bar(k), phase_of(i), p.wait_limit)) return false;
            cc.step(pl, stride);
            const bool more = cc.i < we;
            const int s_nxt = more ? cc.s : s_cur;
            const uint32_t am_st = am_addr(k);
            [[maybe_unused]] float am[MT][2][4];  // absmax of rows 16 ia + g (+ 8 hh), the stage's 4 units (unused at blocksize 32)
#pragma unroll
            for (int ia = 0; ia < MT; ++ia)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    if constexpr (AMK == kAm32) {
                        // two per unit: loaded unit by unit below
                    } else if constexpr (AMK == kAm64) {
                        const uint4 v = lds_v4(am_st + (uint32_t)(16 * ia + 8 * hh + g) * 16u);
                        am[ia][hh][0] = __uint_as_float(v.x);
                        am[ia][hh][1] = __uint_as_float(v.y);
                        am[ia][hh][2] = __uint_as_float(v.z);
                        am[ia][hh][3] = __uint_as_float(v.w);
                    } else {
                        const int x0 = ((s_cur * 4) >> p.am_shift) & ~3;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int col = ((s_cur * 4 + j) >> p.am_shift) - x0;
                            am[ia][hh][j] = lds_f32(am_st + (uint32_t)((16 * ia + 8 * hh + g) * 16 + col * 4));
                        }
                    }
                }
            const float zero[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
                for (int ia = 0; ia < MT; ++ia) {
                    // d[0 / 1]: rows g / g + 8 of the MMA tile, bytes 4 tq ..
                    // 4 tq + 3 of the unit (k = 8 tq .. 8 tq + 7); d[2 / 3] the
                    // same rows 32 k further.  Rows past a half tile look
                    // nothing up.
                    uint32_t d[4];
                    const int row = 16 * ia + 8 * (lm_q & 1) + lm_r, chunk = 2 * j + (lm_q >> 1);
                    ldmatrix_x4(st_addr + (uint32_t)row * 128u + (uint32_t)((chunk ^ (row & 7)) << 4), d[0], d[1], d[2],
                                d[3]);
                    uint32_t q[4][4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        if (HALF && ia == MT - 1 && (x & 1)) {
                            q[x][0] = q[x][1] = q[x][2] = q[x][3] = 0u;
                        } else {
                            q[x][0] = lut_pair<0>(d[x], lane4);
                            q[x][1] = lut_pair<1>(d[x], lane4);
                            q[x][2] = lut_pair<2>(d[x], lane4);
                            q[x][3] = lut_pair<3>(d[x], lane4);
                        }
                    }
                    if constexpr (AMK == kAm32) {
                        // Blocksize 32: the first two MMAs cover k 0..31 of the
                        // unit, the last two k 32..63; each half is scaled by
                        // its own block's absmax.
                        float2 a2[2];
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh)
                            a2[hh] = lds_f32x2(am_st + (uint32_t)(16 * ia + 8 * hh + g) * G::AMW + (uint32_t)j * 8u);
                        float tl[NJ][4], th[NJ][4];
#pragma unroll
                        for (int jj = 0; jj < NJ; ++jj) {
                            mma16816<T>(tl[jj], q[0][0], q[1][0], q[0][1], q[1][1], aw[j % AU][jj][0][0],
                                        aw[j % AU][jj][0][1], zero);
                            mma16816<T>(th[jj], q[2][0], q[3][0], q[2][1], q[3][1], aw[j % AU][jj][1][0],
                                        aw[j % AU][jj][1][1], zero);
                        }
#pragma unroll
                        for (int jj = 0; jj < NJ; ++jj) {
                            mma16816<T>(tl[jj], q[0][2], q[1][2], q[0][3], q[1][3], aw[j % AU][jj][0][2],
                                        aw[j % AU][jj][0][3], tl[jj]);
                            mma16816<T>(th[jj], q[2][2], q[3][2], q[2][3], q[3][3], aw[j % AU][jj][1][2],
                                        aw[j % AU][jj][1][3], th[jj]);
                        }
#pragma unroll
                        for (int jj = 0; jj < NJ; ++jj) {
                            acc[ia][jj][0] = fmaf(a2[0].x, tl[jj][0], acc[ia][jj][0]);
                            acc[ia][jj][1] = fmaf(a2[0].x, tl[jj][1], acc[ia][jj][1]);
                            acc[ia][jj][2] = fmaf(a2[1].x, tl[jj][2], acc[ia][jj][2]);
                            acc[ia][jj][3] = fmaf(a2[1].x, tl[jj][3], acc[ia][jj][3]);
                            acc[ia][jj][0] = fmaf(a2[0].y, th[jj][0], acc[ia][jj][0]);
                            acc[ia][jj][1] = fmaf(a2[0].y, th[jj][1], acc[ia][jj][1]);
                            acc[ia][jj][2] = fmaf(a2[1].y, th[jj][2], acc[ia][jj][2]);
                            acc[ia][jj][3] = fmaf(a2[1].y, th[jj][3], acc[ia][jj][3]);
                        }
                    } else {
                        float t[NJ][4];
#pragma unroll
                        for (int jj = 0; jj < NJ; ++jj)
                            mma16816<T>(t[jj], q[0][0], q[1][0], q[0][1], q[1][1], aw[j % AU][jj][0][0],
                                        aw[j % AU][jj][0][1], zero);
#pragma unroll
                        for (int jj = 0; jj < NJ; ++jj)
                            mma16816<T>(t[jj], q[0][2], q[1][2], q[0][3], q[1][3], aw[j % AU][jj][0][2],
                                        aw[j % AU][jj][0][3], t[jj]);
#pragma unroll
                        for (int jj = 0; jj < NJ; ++jj)
                            mma16816<T>(t[jj], q[2][0], q[3][0], q[2][1], q[3][1], aw[j % AU][jj][1][0],
                                        aw[j % AU][jj][1][1], t[jj]);
#pragma unroll
                        for (int jj = 0; jj < NJ; ++jj)
                            mma16816<T>(t[jj], q[2][2], q[3][2], q[2][3], q[3][3], aw[j % AU][jj][1][2],
                                        aw[j % AU][jj][1][3], t[jj]);
#pragma unroll
                        for (int jj = 0; jj < NJ; ++jj) {
                            acc[ia][jj][0] = fmaf(am[ia][0][j], t[jj][0], acc[ia][jj][0]);
                            acc[ia][jj][1] = fmaf(am[ia][0][j], t[jj][1], acc[ia][jj][1]);
                            acc[ia][jj][2] = fmaf(am[ia][1][j], t[jj][2], acc[ia][jj][2]);
                            acc[ia][jj][3] = fmaf(am[ia][1][j], t[jj][3], acc[ia][jj][3]);
                        }
                    }
                }
                // The unit AU further on, in this stage or the next (the
                // warp's own stage again at the end).
                load_unit(j + AU < 4 ? 4 * s_cur + j + AU : 4 * s_nxt + j + AU - 4, aw[j % AU]);
            }
            // Refill the slot with the warp's stage `ahead` further on: order
            // this warp's reads of the slot before the asynchronous write.
            fence_proxy_async_smem();
            __syncwarp();
            if (ci.i < we) {
                if (lane == 0) issue(ci.i, ci.stage(pl));
                ci.step(pl, stride);
            }
            __syncwarp();
            if (!more || cc.t != tile) return true;
        }
    };

    if (cc.i < we) {
#pragma unroll
        for (int j = 0; j < AU; ++j) load_unit(4 * cc.s + j, aw[j]);
        using F = std::false_type;
        using Tr = std::true_type;
        while (cc.i < we) {
            const int tile = cc.t;
            bool fine;
            switch (pl.tile_rows(tile) >> 3) {  // rows / 8
                case 1: fine = run_tile(std::integral_constant<int, 1>{}, Tr{}); break;
                case 2: fine = run_tile(std::integral_constant<int, 1>{}, F{}); break;
                case 3: fine = run_tile(std::integral_constant<int, 2>{}, Tr{}); break;
                case 4: fine = run_tile(std::integral_constant<int, 2>{}, F{}); break;
                case 5: fine = run_tile(std::integral_constant<int, 3>{}, Tr{}); break;
                case 6: fine = run_tile(std::integral_constant<int, 3>{}, F{}); break;
                case 7: fine = run_tile(std::integral_constant<int, 4>{}, Tr{}); break;
                case 8: fine = run_tile(std::integral_constant<int, 4>{}, F{}); break;
                default:
                    if constexpr (MTM >= 5) {
                        fine = run_tile(std::integral_constant<int, 5>{}, Tr{});  // 72 rows
                    } else {
                        fine = false;
                    }
                    break;
            }
            if (!fine || !flush(tile)) {
                ok = false;
                break;
            }
        }
    }
    if (!ok && lane == 0) {
        if (p.error) atomicExch(p.error, kErrWaitTimeout);
        sts_u32(failed, 1u);
    }
    __syncthreads();
    if (tid == 0 && lds_u32(failed)) {
        // A wait ran out and stages may have been left unread: let every
        // copy still in flight land before the CTA leaves (bounded).
        for (int k = 0; k < D; ++k) {
            const uint32_t ph = lds_u32(last_issued + 4u * (uint32_t)k);
            if (ph) wait_stage(full_bar(k), ph - 1u);
        }
    }
}

// Weights [N rows][K/2 bytes]: boxes of h rows x 128 bytes, 128-byte
// swizzle.  Absmax [N rows][K/bs floats]: boxes of h rows x `am_box` floats
// (4; 8 at blocksize 32).  One pair per distinct tile height of the launch
// (heights[] in rows).
static cudaError_t make_maps(const RowsParams& p, const uint8_t* Wp, const float* absmax, int am_per_row, int am_box,
                             const int* heights, int nh, RowsMaps* m) {
    auto enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const cuuint32_t es[2] = {1, 1};
    const cuuint64_t wdim[2] = {(cuuint64_t)(p.K / 2), (cuuint64_t)p.N};
    const cuuint64_t wstr[1] = {(cuuint64_t)(p.K / 2)};
    const cuuint64_t adim[2] = {(cuuint64_t)am_per_row, (cuuint64_t)p.N};
    const cuuint64_t astr[1] = {(cuuint64_t)am_per_row * 4};
    for (int v = 0; v < nh; ++v) {
        const cuuint32_t rows = (cuuint32_t)heights[v];
        const cuuint32_t wbox[2] = {128, rows};
        if (enc(&m->w[v], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(Wp), wdim, wstr, wbox, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        const cuuint32_t abox[2] = {(cuuint32_t)am_box, rows};
        if (enc(&m->a[v], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(absmax), adim, astr, abox, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    return cudaSuccess;
}

// Distinct tile heights of a launch (the device's Plan, replayed for the
// two group counts a CTA can have), and the map index of each height.
static int stage_heights(const RowsParams& p, int gmax, int* heights, uint32_t* map_bits) {
    int nh = 0;
    *map_bits = 0;
    auto add = [&](int h) {
        for (int v = 0; v < nh; ++v)
            if (heights[v] == h) return;
        *map_bits |= (uint32_t)nh << (2 * (h >> 3));
        heights[nh++] = h;
    };
    const int q = p.groups / p.ctas, r = p.groups - q * p.ctas;
    for (int ng = q; ng <= q + (r ? 1 : 0); ++ng) {
        if (ng <= 0) continue;
        const int T = (ng + gmax - 1) / gmax, base = ng / T, extra = ng - base * T;
        add(8 * base);
        if (extra) add(8 * (base + 1));
    }
    return nh;
}

template <typename T, int NJ, int AMK, bool CONTIG>
static cudaError_t launch_t(const RowsMaps& m, const RowsParams& p, int smem, cudaStream_t stream) {
    auto kern = q4_gemm_rows_kernel<T, NJ, AMK, CONTIG>;
    cudaError_t e = ensure_smem_attr((const void*)kern, (size_t)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, p, m);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace rows

int rows_warps() { return rows::kW; }

// The kernel instance for an activation type and absmax granularity:
// one column tile (round robin or contiguous ranges) or two.
template <typename T, int AMK>
static cudaError_t launch_for(int m_pad, const rows::RowsMaps& m, const RowsParams& p, int smem, cudaStream_t stream) {
    using namespace rows;
    if (m_pad == 32) {
        if constexpr (AMK != kAm32) return launch_t<T, 4, AMK, false>(m, p, smem, stream);
        return cudaErrorInvalidValue;  // M > 16 needs blocksize >= 64
    }
    if (m_pad != 8) return launch_t<T, 2, AMK, false>(m, p, smem, stream);
    if constexpr (AMK != kAm32) {
        if (p.contig) return launch_t<T, 1, AMK, true>(m, p, smem, stream);
    }
    return launch_t<T, 1, AMK, false>(m, p, smem, stream);
}

template <typename T>
static cudaError_t launch_am(int amk, int m_pad, const rows::RowsMaps& m, const RowsParams& p, int smem,
                             cudaStream_t stream) {
    using namespace rows;
    if (amk == kAm32) return launch_for<T, kAm32>(m_pad, m, p, smem, stream);
    if (amk == kAm64) return launch_for<T, kAm64>(m_pad, m, p, smem, stream);
    return launch_for<T, kAmShared>(m_pad, m, p, smem, stream);
}

cudaError_t rows_launch(int act_dtype, int m_pad, const RowsParams& p0, const uint8_t* Wp, const float* absmax,
                        int am_per_row, int smem, cudaStream_t stream) {
    using namespace rows;
    RowsParams p = p0;
    // blocksize = K / am_per_row: 32, 64, or larger (am_shift = log2(bs / 64))
    const int amk = (int64_t)am_per_row * 32 == p.K ? kAm32 : p.am_shift == 0 ? kAm64 : kAmShared;
    // Two or four column tiles or blocksize 32: round robin only (the
    // partial tiles fill the parking space; blocksize 32 has no contiguous
    // instance).
    if (m_pad != 8 || amk == kAm32) p.contig = 0;
    int heights[kRowsMaxMaps];
    const int max_rows = m_pad == 32     ? Geo<4, false, kAm64>::MAX_ROWS
                         : amk == kAm32 ? Geo<1, false, kAm32>::MAX_ROWS
                         : (m_pad == 8 && !p.contig) ? Geo<1, false, kAm64>::MAX_ROWS
                                                     : Geo<1, true, kAm64>::MAX_ROWS;
    const int nh = stage_heights(p, max_rows / 8, heights, &p.map_bits);
    RowsMaps m;
    memset(&m, 0, sizeof(m));
    cudaError_t e = make_maps(p, Wp, absmax, am_per_row, amk == kAm32 ? 8 : 4, heights, nh, &m);
    if (e != cudaSuccess) return e;
    for (int v = nh; v < kRowsMaxMaps; ++v) {  // unused slots repeat a valid map (the kernel prefetches all)
        m.w[v] = m.w[0];
        m.a[v] = m.a[0];
    }
    return act_dtype == 0 ? launch_am<__nv_bfloat16>(amk, m_pad, m, p, smem, stream)
                          : launch_am<__half>(amk, m_pad, m, p, smem, stream);
}

}  // namespace q4
