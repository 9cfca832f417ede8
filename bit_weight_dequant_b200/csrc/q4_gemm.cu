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
#include <cuda_runtime.h>

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

// One table lookup: byte BYTE of `word` -> packed (code[hi], code[lo]).
template <int BYTE>
__device__ __forceinline__ uint32_t lut_pair(uint32_t word, uint32_t lane4) {
    // result bytes: [0] = lane4.b0 (lane*4), [1] = word.b<BYTE>, [2..3] = lane4.b2..b3 (table base >> 16)
    return lds_u32(prmt<0x7604u | (BYTE << 4)>(word, lane4));
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
#pragma unroll
    for (int i = 0; i < S::TW; ++i)
#pragma unroll
        for (int j = 0; j < S::NJ; ++j)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int n = tile * S::TR + 16 * i + g + ((r & 2) ? 8 : 0);
                const int m = 8 * j + 2 * tq + (r & 1);
                if (n < p.N && m < p.M) out[(size_t)m * p.N + n] = Act<T>::from_float(v[i][j][r]);
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

template <typename T, class S>
__global__ void __launch_bounds__(S::NW * 32, 1) q4_gemm_mma_kernel(const GemmParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t sbase = smem_addr(smem);
    const uint32_t lut = (sbase + 0xFFFFu) & ~0xFFFFu;  // 64 KiB aligned (host reserves the padding)
    const uint32_t slots = (lut - sbase >= S::SLOT_BYTES) ? sbase : lut + S::LUT_BYTES;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;

    // Table row b (256 B): 32 copies (one per bank) of the pair (code[b>>4], code[b&15]) as T.
    for (int e = tid; e < 256 * 8; e += S::NW * 32) {
        const int b = e >> 3;
        const uint32_t v = Act<T>::pack(__ldg(p.code + (b >> 4)), __ldg(p.code + (b & 15)));
        sts_v4(lut + (uint32_t)b * 256u + (uint32_t)(e & 7) * 16u, v, v, v, v);
    }
    __syncthreads();

    const int64_t cs = part_start(p.units, p.ctas, blockIdx.x);
    const int64_t ce = part_start(p.units, p.ctas, blockIdx.x + 1);
    const int64_t uc = ce - cs;
    const int64_t ws = cs + part_start(uc, S::NW, warp);
    const int64_t we = cs + part_start(uc, S::NW, warp + 1);
    const uint32_t lane4 = lut | ((uint32_t)lane << 2);
    const int nunits = (int)(we - ws);

    if (nunits > 0) {
        float acc[S::TW][S::NJ][4];
        zero_acc<S>(acc);
        Cursor c;
        c.tile = (int)(ws / p.kb_per_tile);
        c.kb = (int)(ws - (int64_t)c.tile * p.kb_per_tile);
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

    // Combine the tiles that warps or CTAs share.
    const int ta = (int)(cs / p.kb_per_tile);
    const int tb = (int)((ce - 1) / p.kb_per_tile);
    for (int t = ta + warp; t <= tb; t += S::NW) {
        const int64_t t0 = (int64_t)t * p.kb_per_tile, t1 = t0 + p.kb_per_tile;
        const int64_t lo = t0 > cs ? t0 : cs, hi = t1 < ce ? t1 : ce;
        const int wlo = part_owner(uc, S::NW, lo - cs), whi = part_owner(uc, S::NW, hi - 1 - cs);
        const bool inside = (lo == t0) && (hi == t1);
        if (inside && wlo == whi) continue;  // already stored by its only warp
        float sum[S::TW][S::NJ][4];
        zero_acc<S>(sum);
        for (int w = wlo; w <= whi; ++w) {
            const int64_t w0 = cs + part_start(uc, S::NW, w), w1 = cs + part_start(uc, S::NW, w + 1);
            if (w1 == w0) continue;  // empty warp range
            add_slot<S>(sum, slots, w * 2 + ((w0 / p.kb_per_tile == t) ? 0 : 1), lane);
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
        __threadfence();
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atomicAdd(p.counters + t, 1);
        prev = __shfl_sync(0xffffffffu, prev, 0);
        const int cf = part_owner(p.units, p.ctas, t0), cl = part_owner(p.units, p.ctas, t1 - 1);
        if (prev != cl - cf) continue;
        __threadfence();
        zero_acc<S>(sum);
        for (int cta = cf; cta <= cl; ++cta) {
            const int which = (part_start(p.units, p.ctas, cta) / p.kb_per_tile == t) ? 0 : 1;
            const float* src = p.partials + ((size_t)cta * 2 + which) * S::SLOT_FLOATS;
#pragma unroll
            for (int i = 0; i < S::TW; ++i)
#pragma unroll
                for (int j = 0; j < S::NJ; ++j)
#pragma unroll
                    for (int r = 0; r < 4; ++r) sum[i][j][r] += ldg_cg_f32(src + ((i * S::NJ + j) * 4 + r) * 32 + lane);
        }
        store_tile<T, S>(sum, p, t, g, tq);
        if (lane == 0) p.counters[t] = 0;  // leave the workspace zero-filled
    }
}

// ---------------------------------------------------------------------------
// Host launchers: the table of compiled variants.
// ---------------------------------------------------------------------------
template <typename T, class S>
static cudaError_t launch_mma(const GemmParams& p, cudaStream_t stream) {
    auto kern = q4_gemm_mma_kernel<T, S>;
    cudaError_t e = ensure_smem_attr((const void*)kern, S::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<p.ctas, S::NW * 32, S::SMEM_BYTES, stream>>>(p);
    return cudaGetLastError();
}

struct Variant {
    int act, sub_block, m_pad, warps, depth, l2pf;
    size_t smem;
    cudaError_t (*launch)(const GemmParams&, cudaStream_t);
};

#define Q4_VARIANT(ACT, T, SB, MP, NW, D, PF)                                                  \
    Variant {                                                                                 \
        ACT, SB, MP, NW, D, PF, GemmShape<SB, MP, 4, NW, D, PF>::SMEM_BYTES,                  \
            &launch_mma<T, GemmShape<SB, MP, 4, NW, D, PF>>                                   \
    }

#define Q4_VARIANTS_FOR(ACT, T)                                                                \
    Q4_VARIANT(ACT, T, 64, 8, 16, 1, 128), Q4_VARIANT(ACT, T, 64, 8, 8, 2, 128),               \
        Q4_VARIANT(ACT, T, 64, 16, 8, 1, 128), Q4_VARIANT(ACT, T, 32, 8, 16, 1, 128),         \
        Q4_VARIANT(ACT, T, 32, 16, 8, 1, 128)

static const Variant kVariants[] = {
    Q4_VARIANTS_FOR(0, __nv_bfloat16),
    Q4_VARIANTS_FOR(1, __half),
    // measurement-only variants of the main M<=8, blocksize-64, bf16 case
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 16, 1, 0),
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 16, 1, 256),
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 16, 2, 128),
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 8, 1, 128),
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 8, 2, 0),
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 8, 2, 256),
    Q4_VARIANT(0, __nv_bfloat16, 64, 8, 8, 3, 128),
    Q4_VARIANT(0, __nv_bfloat16, 64, 16, 8, 2, 128),
};

static const Variant* find_variant(int act, const GemmChoice& ch) {
    for (const Variant& v : kVariants)
        if (v.act == act && v.sub_block == ch.sub_block && v.m_pad == ch.m_pad && v.warps == ch.warps &&
            v.depth == ch.depth && v.l2pf == ch.l2pf)
            return &v;
    return nullptr;
}

bool gemm_variant_exists(int act_dtype, const GemmChoice& ch) { return find_variant(act_dtype, ch) != nullptr; }

size_t gemm_smem_bytes(int act_dtype, const GemmChoice& ch) {
    const Variant* v = find_variant(act_dtype, ch);
    return v ? v->smem : 0;
}

cudaError_t gemm_launch(const GemmChoice& ch, int act_dtype, const GemmParams& p, cudaStream_t stream) {
    const Variant* v = find_variant(act_dtype, ch);
    if (!v) return cudaErrorInvalidConfiguration;
    return v->launch(p, stream);
}

size_t gemm_slot_floats(int m_pad) { return (size_t)4 * (m_pad / 8) * 4 * 32; }

}  // namespace q4
