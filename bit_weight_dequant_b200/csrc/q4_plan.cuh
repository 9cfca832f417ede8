// q4_plan.cuh -- work decomposition of the fused dequantize + skinny GEMM.
//
// The weight matrix W[N,K] is cut into work units of `rows_per_tile` rows by
// `sub_block` columns (one absmax block, or a part of one).  Units are
// numbered tile-major: unit u covers tile u / kb_per_tile, column block
// u % kb_per_tile.  A persistent grid of `ctas` CTAs splits the unit range
// into equal contiguous ranges (stream-K style), and each CTA splits its
// range again over its warps.  A tile cut by a warp boundary is combined in
// shared memory; a tile cut by a CTA boundary is combined through a small
// global workspace by whichever CTA arrives last.  Every SM gets the same
// number of weight bytes to within one unit, whatever N and K are.
#pragma once

#include <stdint.h>

namespace q4 {

// First unit of part p when `total` units are split into `parts` ranges.
// 32-bit arithmetic (the kernels' hot path): the launcher guarantees
// total * parts < 2^32.
__host__ __device__ __forceinline__ uint32_t part_start(uint32_t total, uint32_t parts, uint32_t p) {
    return (total * p) / parts;
}

// The unique part p with part_start(p) <= u < part_start(p + 1).
// part_start(p) <= u  <=>  total*p < (u+1)*parts  <=>  p <= ((u+1)*parts - 1) / total.
__host__ __device__ __forceinline__ uint32_t part_owner(uint32_t total, uint32_t parts, uint32_t u) {
    return ((u + 1) * parts - 1) / total;
}

// The same two functions without the range limit (host-side reference).
inline int64_t part_start64(int64_t total, int parts, int p) { return (total * (int64_t)p) / parts; }
inline int part_owner64(int64_t total, int parts, int64_t u) { return (int)(((u + 1) * (int64_t)parts - 1) / total); }

// Every wait on an mbarrier is bounded: after kWaitLimit polls the kernel
// records an error word in the workspace, drains what it started (also
// bounded) and returns; its outputs are then not valid.
static constexpr uint32_t kWaitLimit = 1u << 20;  // try_wait polls before giving up
static constexpr int kErrWaitTimeout = 1;         // a bounded wait ran out
static constexpr int kErrNoRoom = 2;              // the launch gave too little shared memory

// Largest unit count the kernels accept (keeps total * parts below 2^32 for
// up to 512 parts).
static constexpr uint32_t kMaxUnits = (1u << 23);

// Compile-time shape of one GEMM kernel variant.
template <int SB_, int MPAD_, int TW_, int NW_, int DEPTH_, int L2PF_>
struct GemmShape {
    static constexpr int SB = SB_;      // k-width of a unit (32 or 64)
    static constexpr int MPAD = MPAD_;  // M padded to 8 or 16 (MMA columns)
    static constexpr int NJ = MPAD_ / 8;
    static constexpr int TW = TW_;      // 16-row MMA tiles per unit
    static constexpr int TR = 16 * TW_; // rows per unit
    static constexpr int NW = NW_;      // warps per CTA
    static constexpr int DEPTH = DEPTH_;  // units in flight ahead of the one being computed
    static constexpr int L2PF = L2PF_;    // L2 fetch-size hint for weight loads (0, 128, 256 bytes)
    static constexpr int SLOT_REGS = TW_ * NJ * 4;     // accumulator registers per lane
    static constexpr int SLOT_FLOATS = SLOT_REGS * 32; // one warp's partial tile
    static constexpr uint32_t LUT_BYTES = 256u * 256u; // 256 byte values x 32 lanes x 4 B, 256-B rows
    static constexpr uint32_t SLOT_BYTES = (uint32_t)NW_ * 2u * SLOT_FLOATS * 4u;
    // Dynamic shared memory: up to 64 KiB of padding so the LUT starts on a
    // 64 KiB boundary of the shared window, the LUT, and the warp slots.
    static constexpr uint32_t SMEM_BYTES = 65536u + LUT_BYTES + SLOT_BYTES;
};

// Largest partial-sum slot of any variant (TW = 4, MPAD = 16): the GEMM
// workspace reserves this much per slot so its counters sit at an offset
// that depends only on the device's SM count.
static constexpr size_t kMaxSlotBytes = 4 * 2 * 4 * 32 * 4;

// Runtime parameters of one GEMM launch.
struct GemmParams {
    const void* A;
    const uint8_t* Wp;
    const float* absmax;
    const float* code;
    void* out;
    const void* bias;  // [N] activation type, or nullptr: added in fp32 before the rounding
    float* partials;   // [ctas][2][SLOT_FLOATS]
    int* counters;     // [tiles], zero between calls
    int* error;        // workspace error word (0 = ok); set when a bounded wait gives up
    int pdl;           // 0: plain launch; 1: dependent launch, every global access after the
                       // dependency wait; 2: code/weights/absmax read before that wait
    int M, N, K;
    int kb_per_tile;   // K / SB
    int am_shift;      // log2(blocksize / SB): absmax column of unit column kb = kb >> am_shift
    int am_per_row;    // K / blocksize
    int tiles;
    int ctas;
    uint32_t units;    // < kMaxUnits
};

// Most distinct tile heights (tensor-map pairs) of one row-split launch:
// two for each of the two group counts a CTA can have.
static constexpr int kRowsMaxMaps = 4;

// Runtime parameters of one launch of the row-split kernel (q4_rows.cu):
// CTA c owns a contiguous run of 8-row groups of W and finishes its outputs
// itself (no workspace besides the error word).
struct RowsParams {
    // What the prologue reads comes first, so that it shares the first
    // cache lines of the parameter block.
    int groups;        // ceil(N / 8)
    int ctas;          // <= groups
    int K;
    int am_shift;      // log2(blocksize / 64)
    int pdl;           // dependent launch mode (0, 1, 2), as in GemmParams
    int l2_ahead;      // stages the producer asks the L2 to fetch beyond the first ring fill
    int skip_stage;    // test hook: this stage index is never loaded (-1: none)
    int contig;        // 1: each warp streams a contiguous range of stages (0: round robin)
    uint32_t map_bits; // tensor-map pair of tile height h (8 .. 72 rows): bits 2 (h / 8) .. 2 (h / 8) + 1,
                       // filled by the launcher (a uniform word, not an indexed array)
    uint32_t wait_limit;  // polls before a wait on a stage or a parking buffer gives up
    int M, N;
    const void* A;
    void* out;
    const void* bias;  // [N] activation type, or nullptr
    const float* code;
    int* error;        // workspace error word, or nullptr
};

}  // namespace q4
