// q4_umma.cu -- the fused 4-bit dequantize + GEMM for 17 <= M <= 128 on the
// fifth-generation tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// Above M = 16 the contraction stops being a skinny afterthought of the
// weight stream: at M = 128 a weight byte feeds 256 multiply-adds, which at
// B200's HBM rate is the tensor cores' whole dense bf16 budget.  The method
// is the same as the M <= 16 kernel's (bitsandbytes PR #1920, "Fused path
// support for M > 1": dequantize in registers, multiply without writing the
// dequantized matrix to memory); the machinery is Blackwell's:
//
//   warp 0       TMA producer: per stage, 128 weight rows x 256 k of packed
//                codes, their absmax, and the activations of the stage's four
//                64-k units (MP rows, zero-filled past M), all into one
//                shared-memory stage; completion on an mbarrier.
//   warp 1       allocates tensor memory; one lane issues the MMAs:
//                D[128 rows, MP] += A[128 rows, 16 k] . B[16 k, MP] with A
//                (the dequantized weights) read from tensor memory and B (the
//                activations) from shared memory, and commits each group to
//                mbarriers that release the A buffer, the stage and, at the
//                end of a tile, the accumulator.
//   warps 2..9   two warpgroups taking alternate units, one thread per
//                weight row.  Per 64-k unit the thread builds the 16 products
//                bf16_rn(code[j] *_fp32 absmax) of its row -- exactly the
//                values the standalone dequantizer writes, one rounding -- as
//                byte-plane tables in registers, turns its 32 packed bytes
//                into 32 bf16 pairs with byte permutes, and stores them into
//                a tensor-memory A buffer (tcgen05.st); at the end of a tile
//                segment it reads its accumulator row back (tcgen05.ld) and
//                stores, or publishes a partial.
//
// The one rounding matters: a weight rounded three times (a table of codes
// already rounded to bf16, times a bf16 absmax, rounded again) can be 1.2 %
// off, and a row of equal codes under one absmax adds those errors with one
// sign, past the 1e-2 * sum|a w| bound.
//
// Work is split stream-K over units of 128 rows x 64 k like the M <= 16
// kernel: a CTA's contiguous unit range may start and end inside tiles; such
// tiles are summed through the workspace by the last CTA to arrive, in CTA
// order (deterministic).  Every wait is bounded: a wait that runs out sets
// the workspace error word, the CTA drains what it started and frees its
// tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

#include "q4_device.cuh"
#include "q4_internal.h"
#include "q4_plan.cuh"

namespace q4 {
namespace umma {

constexpr int kRows = 128;                  // weight rows per tile = MMA M
constexpr int kUps = 4;                     // 64-k units per stage
constexpr uint32_t kWBytes = kRows * 128;   // packed codes of a stage (128 rows x 128 B)
constexpr uint32_t kAmBytes = kRows * 16;   // absmax of a stage (128 rows x 4 floats)
constexpr uint32_t kTmemCols = 512;         // the whole tensor memory (one CTA per SM)
constexpr uint32_t kColD0 = 0, kColD1 = 128, kColA = 256;  // A buffer b at kColA + 32 b
constexpr int kNA = 8;                                       // A buffers (64-k units in flight)
// Bounded waits: each try may sleep up to kWaitSleepNs; at most kWaitTries
// tries (about two seconds) before the wait gives up.
constexpr uint32_t kWaitSleepNs = 50000;
constexpr uint32_t kWaitTries = 40000;
constexpr int kErrWaitTimeout = 1;
constexpr int kNWG = 2;                      // dequantizing warpgroups (unit u goes to u % kNWG)
constexpr int kThreads = 64 + 128 * kNWG;    // producer, MMA issuer, the dequantizing warpgroups

template <int MP>
struct Geo {
    static constexpr uint32_t XBYTES = (uint32_t)MP * 128u;  // one unit's activations (MP rows x 128 B)
    static constexpr uint32_t X0 = kWBytes + kAmBytes;       // 18 KiB: 1024-aligned
    static constexpr uint32_t STAGE = X0 + kUps * XBYTES;     // multiple of 1024
    static_assert(STAGE % 1024 == 0 && X0 % 1024 == 0, "swizzled boxes need 1024-byte alignment");
};

// ---------------------------------------------------------------------------
// tcgen05 wrappers (PTX ISA, "Tensor Core 5th Generation Family Instructions").
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
                 : "memory");
}
// D[tmem] (+)= A[tmem] . B[smem descriptor], kind::f16 (bf16 or fp16 in, fp32 accumulate)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       bool accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),
        "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]),
        "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Instruction descriptor, kind::f16: fp32 accumulate, A and B of the
// activation type, both K-major, M = 128, N = MP.
template <typename T>
__host__ __device__ constexpr uint32_t idesc_f16(int n) {
    const uint32_t fmt = Act16Format<T>::value;  // 0 = fp16, 1 = bf16
    return (1u << 4)                             // D format: fp32
           | (fmt << 7) | (fmt << 10)            // A, B formats
           | ((uint32_t)(n >> 3) << 17)          // N / 8
           | ((uint32_t)(kRows >> 4) << 24);     // M / 16
}

// Shared-memory descriptor of a K-major operand in the 128-byte swizzled
// layout that TMA writes: rows of 128 B, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)1 << 16;                           // leading byte offset (unused in this layout)
    d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                           // descriptor version
    d |= (uint64_t)2 << 61;                           // 128-byte swizzle
    return d;
}

__device__ __forceinline__ bool wait_parity(uint32_t bar, uint32_t parity) {
    for (uint32_t it = 0; it < kWaitTries; ++it)
        if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    return false;
}

// Byte planes of the row's 16 scaled codes: tl[k] / th[k] hold the low /
// high bytes of values 4k .. 4k+3.
template <typename T>
__device__ __forceinline__ void scaled_tables(const float (&c)[16], float am, uint32_t (&tl)[4], uint32_t (&th)[4]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t p0 = Act<T>::pack(__fmul_rn(c[4 * k], am), __fmul_rn(c[4 * k + 1], am));
        const uint32_t p1 = Act<T>::pack(__fmul_rn(c[4 * k + 2], am), __fmul_rn(c[4 * k + 3], am));
        tl[k] = prmt<0x6420u>(p0, p1);
        th[k] = prmt<0x7531u>(p0, p1);
    }
}

__device__ __forceinline__ uint32_t prmt_r(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// The four packed pairs of word w: byte q -> (value[hi nibble] in the low
// half, value[lo nibble] in the high half), i.e. k = 2q then 2q + 1.
__device__ __forceinline__ void word_pairs(uint32_t w, const uint32_t (&tl)[4], const uint32_t (&th)[4],
                                           uint32_t* out) {
    const uint32_t idx = w & 0x77777777u;          // index inside an 8-entry half
    const uint32_t half = (w >> 1) & 0x44444444u;  // bit 3 of each nibble as +4 in a selector
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h ? idx >> 16 : idx;
        const uint32_t pick = (h ? half >> 16 : half) | 0x3210u;
        const uint32_t l = prmt_r(prmt_r(tl[0], tl[1], sel), prmt_r(tl[2], tl[3], sel), pick);
        const uint32_t u = prmt_r(prmt_r(th[0], th[1], sel), prmt_r(th[2], th[3], sel), pick);
        // l / u bytes follow the nibbles lo0 hi0 lo1 hi1 of this half-word
        out[2 * h] = prmt<0x4051u>(l, u);
        out[2 * h + 1] = prmt<0x6273u>(l, u);
    }
}

struct Seq {  // walk of a CTA's unit range in stages of <= kUps units of one tile
    int tile, kb, left;
};
__device__ __forceinline__ void next_stage(Seq& s, int kbt, int& tile, int& kb0, int& kb, int& n) {
    tile = s.tile;
    kb = s.kb;
    kb0 = kb & ~(kUps - 1);
    int end = kb0 + kUps;
    if (end > kbt) end = kbt;
    n = end - kb;
    if (n > s.left) n = s.left;
    s.left -= n;
    s.kb += n;
    if (s.kb == kbt) {
        s.kb = 0;
        ++s.tile;
    }
}

template <typename T, int MP>
__global__ void __launch_bounds__(kThreads, 1)
    q4_gemm_umma_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_a,
                        const __grid_constant__ CUtensorMap tmap_x, const GemmParams p, int nstages) {
    using G = Geo<MP>;
    extern __shared__ __align__(16) uint8_t smem_umma[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t sraw = smem_addr(smem_umma);
    const uint32_t base = (sraw + 1023u) & ~1023u;
    const int S = nstages;
    // barriers and the tensor-memory address after the stages
    const uint32_t bars = base + (uint32_t)S * G::STAGE;
    auto full = [&](int s) { return bars + 8u * (uint32_t)s; };
    auto sfree = [&](int s) { return bars + 8u * (uint32_t)(S + s); };
    const uint32_t aready = bars + 8u * (uint32_t)(2 * S), afree = aready + 8u * kNA;  // [kNA] each
    const uint32_t dready = afree + 8u * kNA, dfree = dready + 16u;                    // [2] each
    const uint32_t drain = dfree + 16u;                                                // MMA drain on error
    const uint32_t tslot = drain + 8u;                                                 // tensor-memory base
    // Cross-CTA epilogue handshakes: a CTA has at most two tiles it shares
    // with other CTAs (its first and its last), and two warpgroups may
    // run those epilogues at the same time, so each gets its own pair of
    // barriers and its own broadcast word, each used once per launch.
    const uint32_t ctl = tslot + 8u;      // [2] words
    const uint32_t epi1 = tslot + 16u;    // [2] barriers
    const uint32_t epi2 = tslot + 32u;    // [2] barriers

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full(s), 1);
            mbar_init(sfree(s), 1);
        }
        for (int b = 0; b < kNA; ++b) {
            mbar_init(aready + 8u * b, 4);
            mbar_init(afree + 8u * b, 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(dready + 8u * b, 1);
            mbar_init(dfree + 8u * b, 4);
        }
        mbar_init(drain, 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(epi1 + 8u * x, 4);
            mbar_init(epi2 + 8u * x, 1);
        }
        mbar_init_fence();
    }
    if (warp == 1) {
        tmem_alloc(tslot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = lds_u32(tslot);
    // Activations, outputs and the workspace may belong to the preceding
    // grid, and every stage carries activations: wait before any access.
    griddep_wait();
    griddep_launch_dependents();

    const uint32_t cs = part_start(p.units, p.ctas, blockIdx.x);
    const uint32_t ce = part_start(p.units, p.ctas, blockIdx.x + 1);
    const int nunits = (int)(ce - cs);
    const int kbt = p.kb_per_tile;
    const int tile0 = nunits > 0 ? (int)(cs / (uint32_t)kbt) : 0;
    const int kb00 = nunits > 0 ? (int)(cs - (uint32_t)tile0 * (uint32_t)kbt) : 0;
    bool ok = true;

    if (warp == 0) {
        // ---------------- producer ----------------
        if (lane == 0 && nunits > 0) {
            Seq q{tile0, kb00, nunits};
            int issued = 0;
            for (; q.left > 0; ++issued) {
                int tile, kb0, kb, n;
                next_stage(q, kbt, tile, kb0, kb, n);
                const int slot = issued % S;
                if (issued >= S && !wait_parity(sfree(slot), (uint32_t)(issued / S - 1) & 1u)) {
                    ok = false;
                    break;
                }
                const uint32_t st = base + (uint32_t)slot * G::STAGE;
                mbar_expect_tx(full(slot), G::STAGE);
                tma_load_2d(st, &tmap_w, kb0 * 32, tile * kRows, full(slot));
                tma_load_2d(st + kWBytes, &tmap_a, (kb0 >> p.am_shift) & ~3, tile * kRows, full(slot));
#pragma unroll
                for (int j = 0; j < kUps; ++j)
                    tma_load_2d(st + G::X0 + (uint32_t)j * G::XBYTES, &tmap_x, (kb0 + j) * 64, 0, full(slot));
            }
            if (!ok) {
                atomicExch(p.error, kErrWaitTimeout);
                // drain: every stage issued so far completes or times out
                for (int k = (issued > S ? issued - S : 0); k < issued; ++k)
                    wait_parity(full(k % S), (uint32_t)(k / S) & 1u);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && nunits > 0) {
            Seq q{tile0, kb00, nunits};
            const uint32_t idesc = idesc_f16<T>(MP);
            int stage = 0, u = 0, seg = 0;
            int cur_tile = -1;
            for (; q.left > 0 && ok; ++stage) {
                int tile, kb0, kb, n;
                next_stage(q, kbt, tile, kb0, kb, n);
                const int slot = stage % S;
                if (!wait_parity(full(slot), (uint32_t)(stage / S) & 1u)) {
                    ok = false;
                    break;
                }
                const uint32_t st = base + (uint32_t)slot * G::STAGE;
                for (int j = kb - kb0; j < kb - kb0 + n; ++j, ++u) {
                    const int b = u % kNA;
                    const bool seg_start = (tile != cur_tile);
                    if (seg_start) {
                        cur_tile = tile;
                        if (seg >= 2 && !wait_parity(dfree + 8u * (seg & 1), (uint32_t)((seg >> 1) - 1) & 1u)) {
                            ok = false;
                            break;
                        }
                    }
                    if (!wait_parity(aready + 8u * b, (uint32_t)(u / kNA) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t dcol = (seg & 1) ? kColD1 : kColD0;
                    const uint32_t acol = kColA + 32u * (uint32_t)b;
                    // B descriptor of this unit's activations; each 16-k step
                    // advances the start address by 32 bytes (2 in its units)
                    const uint64_t xd = smem_desc_sw128(st + G::X0 + (uint32_t)j * G::XBYTES);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        mma_ts(tbase + dcol, tbase + acol + 8u * k4, xd + 2u * (uint32_t)k4, idesc,
                               !(seg_start && k4 == 0));
                    tc_commit(afree + 8u * b);
                    const bool seg_end = (kb0 + j + 1 == kbt) || (q.left == 0 && j == kb - kb0 + n - 1);
                    if (seg_end) {
                        tc_commit(dready + 8u * (seg & 1));
                        ++seg;
                        cur_tile = -1;
                    }
                }
                if (!ok) break;
                tc_commit(sfree(slot));
            }
            if (!ok) {
                atomicExch(p.error, kErrWaitTimeout);
                tc_commit(drain);  // tracks every MMA issued so far
                wait_parity(drain, 0);
            }
        }
    } else {
        // ---------------- dequantize + epilogue (one thread per weight row) ----------------
        const int row = 32 * (warp & 3) + lane;             // this warp's tensor-memory lane quarter
        const uint32_t lane_bits = (uint32_t)(32 * (warp & 3)) << 16;
        const int wg = (warp - 2) >> 2;                      // warpgroup: takes the units u with u % kNWG == wg
        const int ew = (warp - 2) & 3;                       // warp within the warpgroup
        float c[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) c[j] = __ldg(p.code + j);
        const T* bias = static_cast<const T*>(p.bias);
        T* out = static_cast<T*>(p.out);
        if (nunits > 0) {
            Seq q{tile0, kb00, nunits};
            int stage = 0, u = 0, seg = 0, xsegs = 0;
            bool first_seg = true;
            for (; q.left > 0 && ok; ++stage) {
                int tile, kb0, kb, n;
                next_stage(q, kbt, tile, kb0, kb, n);
                const int slot = stage % S;
                // Wait for the stage only if this warpgroup has a unit in it
                // (a one-unit stage at a range edge may belong to the other
                // one); a wait on a stage it never reads could alias a later
                // fill of the same slot.
                const bool mine = n >= kNWG || (wg - u % kNWG + kNWG) % kNWG < n;
                if (mine && !wait_parity(full(slot), (uint32_t)(stage / S) & 1u)) {
                    ok = false;
                    break;
                }
                const uint32_t st = base + (uint32_t)slot * G::STAGE;
                uint4 amv = make_uint4(0u, 0u, 0u, 0u);
                if (mine) amv = lds_v4(st + kWBytes + (uint32_t)row * 16u);
                const float amr[4] = {__uint_as_float(amv.x), __uint_as_float(amv.y), __uint_as_float(amv.z),
                                      __uint_as_float(amv.w)};
                const int x0 = (kb0 >> p.am_shift) & ~3;
                for (int j = kb - kb0; j < kb - kb0 + n; ++j, ++u) {
                    const bool seg_end = (kb0 + j + 1 == kbt) || (q.left == 0 && j == kb - kb0 + n - 1);
                    if (u % kNWG != wg) {
                        // another warpgroup's unit: only keep the segment bookkeeping
                        if (seg_end) {
                            const uint32_t t0s = (uint32_t)tile * (uint32_t)kbt;
                            if (!((t0s >= cs) && (t0s + (uint32_t)kbt <= ce))) ++xsegs;
                            ++seg;
                            first_seg = false;
                        }
                        continue;
                    }
                    const int b = u % kNA;
                    if (u >= kNA && !wait_parity(afree + 8u * b, (uint32_t)(u / kNA - 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int col = ((kb0 + j) >> p.am_shift) - x0;
                    const float am = col == 0 ? amr[0] : col == 1 ? amr[1] : col == 2 ? amr[2] : amr[3];
                    uint32_t tl[4], th[4];
                    scaled_tables<T>(c, am, tl, th);
                    // the row's 32 packed bytes of unit j: 16-byte chunks 2j, 2j+1 (128-byte swizzle)
                    const uint32_t rb = st + (uint32_t)row * 128u;
                    const uint4 w0 = lds_v4(rb + (uint32_t)(((2 * j) ^ (row & 7)) << 4));
                    const uint4 w1 = lds_v4(rb + (uint32_t)(((2 * j + 1) ^ (row & 7)) << 4));
                    const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                    uint32_t v[32];
#pragma unroll
                    for (int i = 0; i < 8; ++i) word_pairs(words[i], tl, th, v + 4 * i);
                    tmem_st32(tbase + lane_bits + kColA + 32u * (uint32_t)b, v);
                    tmem_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(aready + 8u * b);
                    if (!seg_end) continue;
                    // ---- epilogue of tile `tile` ----
                    if (!wait_parity(dready + 8u * (seg & 1), (uint32_t)(seg >> 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t dcol = (seg & 1) ? kColD1 : kColD0;
                    const uint32_t t0u = (uint32_t)tile * (uint32_t)kbt;
                    const bool whole = (t0u >= cs) && (t0u + (uint32_t)kbt <= ce);
                    const int n_out = tile * kRows + row;
                    float* slotp = nullptr;
                    if (!whole)
                        slotp = reinterpret_cast<float*>(reinterpret_cast<char*>(p.partials)) +
                                ((size_t)blockIdx.x * 2 + (first_seg ? 0 : 1)) * (size_t)(MP * kRows);
                    const float bn = (bias && n_out < p.N) ? static_cast<float>(bias[n_out]) : 0.f;
                    const int m16 = (p.M + 15) & ~15;  // partial columns that carry real rows
#pragma unroll 1
                    for (int c32 = 0; c32 < MP / 32; ++c32) {
                        uint32_t r[32];
                        tmem_ld32(tbase + lane_bits + dcol + 32u * c32, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            const int m = 32 * c32 + e;
                            if (whole) {
                                if (m < p.M && n_out < p.N)
                                    out[(size_t)m * p.N + n_out] = Act<T>::from_float(__uint_as_float(r[e]) + bn);
                            } else if (m < m16) {
                                slotp[(size_t)m * kRows + row] = __uint_as_float(r[e]);
                            }
                        }
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(dfree + 8u * (seg & 1));
                    ++seg;
                    first_seg = false;
                    if (whole) continue;
                    // Cross-CTA tile: count this CTA's partial in; the last
                    // CTA to arrive adds all partials in CTA order.  The four
                    // warps meet on mbarriers (bounded waits), never on a
                    // barrier that a warp which gave up could leave hanging.
                    __threadfence();
                    __syncwarp();
                    const uint32_t e1 = epi1 + 8u * (uint32_t)xsegs, e2 = epi2 + 8u * (uint32_t)xsegs;
                    const uint32_t cw = ctl + 4u * (uint32_t)xsegs;
                    if (lane == 0) mbar_arrive(e1);
                    const int cf = (int)part_owner(p.units, p.ctas, t0u);
                    const int cl = (int)part_owner(p.units, p.ctas, t0u + (uint32_t)kbt - 1);
                    if (ew == 0 && lane == 0) {
                        bool last = false;
                        if (wait_parity(e1, 0u)) {
                            const int prev = atom_add_acq_rel_gpu(p.counters + tile, 1);
                            last = (prev == cl - cf);
                            if (last) p.counters[tile] = 0;  // every contributor has counted in: reset for the next call
                        } else {
                            ok = false;
                        }
                        sts_u32(cw, last ? 1u : 0u);
                        mbar_arrive(e2);
                    }
                    if (!wait_parity(e2, 0u)) ok = false;
                    ++xsegs;
                    if (!ok) break;
                    if (lds_u32(cw) == 0u) continue;
                    // Up to kFan contributors' values are loaded together before
                    // they are added in CTA order; more (small ranges) go in
                    // further rounds of the same order.
                    constexpr int kFan = 4;
#pragma unroll 1
                    for (int m0 = 0; m0 < m16; m0 += 16) {
                        float sum[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) sum[e] = 0.f;
                        for (int c0 = cf; c0 <= cl; c0 += kFan) {
                            float v[kFan][16];
#pragma unroll
                            for (int f = 0; f < kFan; ++f) {
                                const int cta = c0 + f;
                                if (cta <= cl) {
                                    const int which = (part_start(p.units, p.ctas, cta) >= t0u) ? 0 : 1;
                                    const float* src = reinterpret_cast<const float*>(p.partials) +
                                                       ((size_t)cta * 2 + which) * (size_t)(MP * kRows) +
                                                       (size_t)m0 * kRows + row;
#pragma unroll
                                    for (int e = 0; e < 16; ++e) v[f][e] = ldg_cg_f32(src + (size_t)e * kRows);
                                }
                            }
#pragma unroll
                            for (int f = 0; f < kFan; ++f)
                                if (c0 + f <= cl) {
#pragma unroll
                                    for (int e = 0; e < 16; ++e) sum[e] += v[f][e];
                                }
                        }
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            if (m0 + e < p.M && n_out < p.N)
                                out[(size_t)(m0 + e) * p.N + n_out] = Act<T>::from_float(sum[e] + bn);
                    }
                    // Every contributor has published and this was the last
                    // read: return the slots to zero.  They lie past this
                    // shape's tile counters, where another shape's counters
                    // may live, and counters must start at zero.
                    for (int cta = cf; cta <= cl; ++cta) {
                        const int which = (part_start(p.units, p.ctas, cta) >= t0u) ? 0 : 1;
                        float* src = reinterpret_cast<float*>(p.partials) + ((size_t)cta * 2 + which) * (size_t)(MP * kRows);
                        for (int m = 0; m < m16; ++m) src[(size_t)m * kRows + row] = 0.f;
                    }
                }
            }
            if (!ok) atomicExch(p.error, kErrWaitTimeout);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

static PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        cudaGetLastError();
    });
    return fn;
}

template <typename T, int MP>
static cudaError_t launch(const GemmParams& p, int smem, cudaStream_t stream) {
    auto enc = encoder();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap tw, ta, tx;
    const cuuint32_t es[2] = {1, 1};
    const cuuint64_t wdim[2] = {(cuuint64_t)(p.K / 2), (cuuint64_t)p.N};
    const cuuint64_t wstr[1] = {(cuuint64_t)(p.K / 2)};
    const cuuint32_t wbox[2] = {128, (cuuint32_t)kRows};
    if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p.Wp), wdim, wstr, wbox, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const cuuint64_t adim[2] = {(cuuint64_t)p.am_per_row, (cuuint64_t)p.N};
    const cuuint64_t astr[1] = {(cuuint64_t)p.am_per_row * 4};
    const cuuint32_t abox[2] = {4, (cuuint32_t)kRows};
    if (enc(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p.absmax), adim, astr, abox, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const cuuint64_t xdim[2] = {(cuuint64_t)p.K, (cuuint64_t)p.M};
    const cuuint64_t xstr[1] = {(cuuint64_t)p.K * 2};
    const cuuint32_t xbox[2] = {64, (cuuint32_t)MP};
    if (enc(&tx, sizeof(T) == 2 && Act16Format<T>::value == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
            2, const_cast<void*>(p.A), xdim, xstr, xbox, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int nstages = umma_stages(MP, smem);
    if (nstages < 2) return cudaErrorInvalidValue;
    auto kern = q4_gemm_umma_kernel<T, MP>;
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
    e = cudaLaunchKernelEx(&cfg, kern, tw, ta, tx, p, nstages);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace umma

int umma_stages(int mp, int smem_bytes) {
    const int stage = (int)(umma::kWBytes + umma::kAmBytes) + umma::kUps * mp * 128;
    // 1 KiB alignment slack + barriers, tensor-memory slot and handshake words (< 512 B)
    int s = (smem_bytes - 1024 - 512) / stage;
    if (s > 6) s = 6;
    return s;
}

size_t umma_slot_bytes(int mp) { return (size_t)mp * umma::kRows * 4; }

int umma_warps() { return umma::kThreads / 32; }

cudaError_t umma_launch(int act_dtype, int mp, const GemmParams& p, int smem, cudaStream_t stream) {
    if (act_dtype == 0) {
        if (mp == 32) return umma::launch<__nv_bfloat16, 32>(p, smem, stream);
        if (mp == 64) return umma::launch<__nv_bfloat16, 64>(p, smem, stream);
        if (mp == 128) return umma::launch<__nv_bfloat16, 128>(p, smem, stream);
    } else {
        if (mp == 32) return umma::launch<__half, 32>(p, smem, stream);
        if (mp == 64) return umma::launch<__half, 64>(p, smem, stream);
        if (mp == 128) return umma::launch<__half, 128>(p, smem, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace q4
