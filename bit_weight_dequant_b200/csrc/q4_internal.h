// q4_internal.h -- declarations shared by the libq4 translation units
// (launchers, launch-table choice, per-device attribute cache).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "q4_plan.cuh"

namespace q4 {

// One launch-table decision for the GEMM.
struct GemmChoice {
    int math;       // 1 = tensor-core mma.sync, 2 = CUDA-core FMA, 3 = tcgen05 with tensor memory
    int sub_block;  // 32 or 64
    int m_pad;      // 8 or 16
    int warps;      // warps per CTA
    int ctas;       // persistent CTAs
    int rows_per_tile;
    int depth;      // units (loader 1) or stages (loader 2) in flight per warp
    int l2pf;       // L2 fetch-size hint on weight loads: 0 (none), 128, 256 (loader 1)
    int loader;     // 1 = per-lane global loads, 2/3 = TMA stage ring of 4/2-unit stages, 6 = tcgen05 kernel
    int pdl;        // programmatic dependent launch mode (0, 1, 2)
    int chunk_rows; // > 0: the call runs as ceil(M / chunk_rows) launches of at most chunk_rows
                    // activation rows each (this entry describes the first)
};

// Sets cudaFuncAttributeMaxDynamicSharedMemorySize once per (kernel, device).
cudaError_t ensure_smem_attr(const void* kernel, size_t bytes);

cudaError_t gemm_launch(const GemmChoice& ch, int act_dtype, const GemmParams& p, cudaStream_t stream);
bool gemm_variant_exists(int act_dtype, const GemmChoice& ch);
size_t gemm_smem_bytes(int act_dtype, const GemmChoice& ch);
size_t gemm_slot_floats(int m_pad);

// Tensor-memory (tcgen05) GEMM for 17 <= M <= 128 (q4_umma.cu).
cudaError_t umma_launch(int act_dtype, int m_pad, const GemmParams& p, int smem_bytes, cudaStream_t stream);
int umma_stages(int m_pad, int smem_bytes);
int umma_warps();  // warps per CTA: producer, MMA issuer, dequantizing warpgroups
size_t umma_slot_bytes(int m_pad);

// fp32-activation GEMM on the CUDA cores, M <= 16 (q4_simt.cu): padded M,
// rows per work unit (units are 512 k wide) and warps per CTA.
struct SimtShape {
    int m_pad, rows, warps;
};
SimtShape simt_shape(int M);
size_t simt_smem_bytes();
// act_dtype: 0 bf16, 1 fp16 (widened exactly to fp32 on load), 2 fp32.
cudaError_t simt_launch(const SimtShape& sh, int ctas, const GemmParams& p, int log2_bs, int act_dtype,
                        cudaStream_t stream);

// Row-split kernel for M <= 16 with 16-bit activations (q4_rows.cu).
// act_dtype 0 = bf16, 1 = fp16; m_pad 8 or 16; smem = dynamic shared memory
// to launch with (the kernel sizes its stage ring from it).
cudaError_t rows_launch(int act_dtype, int m_pad, const RowsParams& p, const uint8_t* Wp, const float* absmax,
                        int am_per_row, int smem, cudaStream_t stream);
int rows_warps();  // warps per CTA

// cuTensorMapEncodeTiled through the runtime's driver entry point, or
// nullptr when the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

cudaError_t quantize_launch(const void* W, int w_dtype, int64_t n, int blocksize, const float* code,
                            uint8_t* packed, float* absmax, cudaStream_t stream);
cudaError_t dequantize_launch(const uint8_t* packed, const float* absmax, const float* code, int64_t n,
                              int blocksize, int out_dtype, void* out, cudaStream_t stream);

int device_sm_count(int* sms);  // current device; returns 0 on success

}  // namespace q4
