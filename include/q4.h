/*
 * q4.h -- C ABI of libq4: blockwise 4-bit weight quantization,
 * dequantization and the fused dequantize + skinny matmul
 *     C[M,N] = A[M,K] . dequant(W)[N,K]^T,   1 <= M <= 128,
 * the decode-time hot path of a 4-bit quantized linear layer (M <= 16;
 * 17..128 on the larger-batch kernels), hand-written for NVIDIA B200
 * (sm_100a).
 *
 * Source of the method: bitsandbytes PR #1920, "[ROCm] Optimize
 * kgemm_4bit_inference_naive for ROCm, use it for batch sizes other than 1":
 *   - "Technical details / Kernel optimization": the fused dequantize +
 *     matmul kernel streams packed 4-bit weights and dequantizes them on the
 *     fly;
 *   - "Fused path support for M > 1": the op receives the real number of
 *     activation rows M and runs the fused kernel for small M > 1 instead of
 *     only the vector case; split dequantize + GEMM takes over past a
 *     GPU-specific crossover;
 *   - the maintainer's reply: weights index a 16-entry "NF4/FP4 dtype LUT",
 *     blocksize 64 is the default and other blocksizes are supported,
 *     accumulation is fp32, only the torch inference ("TN") layout W[N,K]
 *     is supported, activations fp16/bf16 (fp32 for the SIMT kernel).
 *
 * Data format (the pages print no byte layout; this is the plainest
 * reading they support):
 *   - W is row-major [N, K], flattened to n = N*K elements;
 *   - absmax: one fp32 per contiguous block of `blocksize` flattened
 *     elements (ceil(n / blocksize) values); the last block may be short;
 *   - packed: ceil(n / 2) bytes, two 4-bit codes per byte, the HIGH nibble
 *     holds the even element;
 *   - code: 16 fp32 values (the lookup table), caller supplied.
 *   - a weight is w[i] = code[idx[i]] * absmax[i / blocksize] (fp32).
 *
 * Conventions for every entry point:
 *   - All pointers are caller-owned DEVICE memory unless stated otherwise;
 *     the library allocates nothing and keeps no state besides a per-device
 *     cache of kernel attributes.  Pointers to empty arrays may be NULL.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream); calls are
 *     asynchronous on it.  Argument errors are reported synchronously by
 *     the return value before anything is enqueued.
 *   - Return value: a q4_status.  A launch failure returns Q4_ERR_CUDA after
 *     draining the runtime's last-error state, so no error the library
 *     caused is left pending for the caller.  Kernels never trap and never
 *     wait on other kernels.
 *   - Q4_ERR_UNSUPPORTED means "valid request this library does not run";
 *     it is the caller's cue to use a split dequantize + dense GEMM path.
 */
#ifndef Q4_H_
#define Q4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    Q4_OK = 0,
    Q4_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad blocksize or dtype */
    Q4_ERR_UNSUPPORTED = 2, /* M > 128, K % blocksize != 0, fp32 with M > 16,   */
                            /* a shape or override no compiled kernel takes     */
    Q4_ERR_MISALIGNED = 3,  /* a pointer misses the alignment stated below      */
    Q4_ERR_CUDA = 4,        /* a CUDA call or kernel launch failed              */
    Q4_ERR_WORKSPACE = 5    /* GEMM workspace missing or smaller than required  */
} q4_status;

typedef enum { Q4_BF16 = 0, Q4_FP16 = 1, Q4_FP32 = 2 } q4_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* q4_status_string(int status);

/*
 * Blockwise 4-bit quantization (inverse of the dequantize step the fused
 * kernel performs; the pages quantize offline).
 *   W       fp32 [n], 16-byte aligned
 *   n       number of elements, >= 0 (0 is a no-op)
 *   blocksize  power of two in [32, 4096]
 *   code    fp32 [16], 4-byte aligned; any values (a strict table order is
 *           not required)
 *   packed  uint8 [ceil(n/2)] output; for odd n the final low nibble is 0
 *   absmax  fp32 [ceil(n/blocksize)] output, 4-byte aligned
 * Per block: absmax = max|w| (exact); x = w / absmax, one correctly rounded
 * fp32 division (x = 0 for an all-zero block); idx = argmin_j |x - code[j]|
 * on fp32 differences, ties to the lowest j.  Non-finite W is undefined.
 */
int q4_quantize_blockwise(const float* W, int64_t n, int blocksize, const float* code,
                          uint8_t* packed, float* absmax, void* stream);

/*
 * The same quantization with the weights given as bf16, fp16 or fp32
 * (w_dtype: Q4_BF16, Q4_FP16, Q4_FP32; anything else -> Q4_ERR_INVALID_ARG).
 * Each element is widened to fp32 exactly, so the result equals
 * q4_quantize_blockwise on the widened values.  W is 16-byte aligned; every
 * other argument as above.
 */
int q4_quantize_blockwise_ex(const void* W, int w_dtype, int64_t n, int blocksize, const float* code,
                             uint8_t* packed, float* absmax, void* stream);

/*
 * Blockwise 4-bit dequantization (the building block of the split path of
 * PR #1920, "split dequantize + GEMM").
 *   packed  uint8 [ceil(n/2)], 16-byte aligned
 *   absmax  fp32 [ceil(n/blocksize)], 4-byte aligned
 *   code    fp32 [16], 4-byte aligned
 *   n, blocksize  as for quantize
 *   out_dtype  Q4_BF16, Q4_FP16 or Q4_FP32
 *   out     [n] elements of out_dtype, 16-byte aligned
 * out[i] = round_to_nearest_even_out_dtype(code[idx_i] * absmax[i/blocksize])
 * with the product formed once in fp32 (bit-exact, -0.0 kept).
 */
int q4_dequantize_blockwise(const uint8_t* packed, const float* absmax, const float* code,
                            int64_t n, int blocksize, int out_dtype, void* out, void* stream);

/*
 * Bytes of device workspace q4_gemm_skinny needs for this problem on the
 * CURRENT device (host-only query; never enqueues work).  Writes 0 when no
 * workspace is needed.  Same argument rules as q4_gemm_skinny.
 */
int q4_gemm_workspace_size(int M, int N, int K, int blocksize, int act_dtype, size_t* bytes);

/*
 * Fused dequantize + skinny matmul (PR #1920's kgemm_4bit_inference_naive
 * generalised to M > 1, "Fused path support for M > 1"):
 *     out[m, n] = round_rn_act( sum_k A[m,k] * code[idx(n,k)] * absmax(n,k) )
 * accumulated in fp32.  bf16/fp16 on the mma.sync kernels (M <= 32): codes
 * enter the tensor-core contraction rounded to the activation dtype T and the
 * per-block absmax scale is applied in fp32; on the tcgen05 kernel the
 * weights enter as T_rn(code *_fp32 absmax).  Either way each weight is
 * rounded once (at most 2^-8 relative for bf16, 2^-11 for fp16).
 * fp32 (the reply's SIMT kernel, which also takes fp32 inputs):
 * every product is an fp32 FMA with the exact fp32 code, scaled in fp32;
 * bf16/fp16 run on that kernel on request (override math = 2), widened
 * exactly to fp32 on load.
 *   A        [M, K] act_dtype, row-major contiguous, 16-byte aligned
 *   Wpacked  uint8 [N*K/2] (rows of K/2 bytes), 16-byte aligned
 *   absmax   fp32 [N*K/blocksize], 4-byte aligned
 *   code     fp32 [16], 4-byte aligned
 *   M        0 is a no-op.  bf16/fp16: 1..16 on the mma.sync kernels
 *            (the row-split kernel by default, the stream-K kernel on
 *            head-like layers and for M >= 8 on layers of >= 2^26 weights);
 *            17..32 on the mma.sync kernel with 32-row tiles when
 *            blocksize >= 64 and (K / blocksize) % 4 == 0, and 33..64 under
 *            the same rules as ceil(M / 32) launches of at most 32 rows each
 *            on the stream (every launch streams the weights again; the
 *            plan describes the first); otherwise (and for 65..128) on the
 *            tcgen05 (tensor-memory) kernel, which
 *            needs blocksize >= 64, K % 256 == 0, (K / blocksize) % 4 == 0
 *            (else Q4_ERR_UNSUPPORTED) and a 16-byte aligned absmax (else
 *            Q4_ERR_MISALIGNED).  fp32: 1..16.  Larger M ->
 *            Q4_ERR_UNSUPPORTED (the caller's cue for dequantize + GEMM).
 *   N, K     >= 0; K % blocksize == 0 (else Q4_ERR_UNSUPPORTED); N = 0 is
 *            a no-op; K = 0 writes zeros
 *   blocksize  power of two in [32, 4096]
 *   act_dtype  Q4_BF16, Q4_FP16 or Q4_FP32
 *   out      [M, N] act_dtype, row-major, 16-byte aligned
 *   workspace  device scratch of at least q4_gemm_workspace_size() bytes,
 *            16-byte aligned, ZERO-FILLED before its first use.  Layout: a
 *            256-byte header whose first int32 is an error word, a
 *            fixed-size region of partial sums (scratch), then one counter
 *            per weight tile (every call returns the counters it used to
 *            zero), so one workspace serves every problem size on a device.
 *            Some kernels need the header alone (q4_gemm_workspace_size
 *            then returns 256).
 *            The error word stays 0 unless a kernel gave up a bounded wait
 *            for its own asynchronous copies (1; outputs of that call are
 *            not valid) or found too little shared memory (2); the caller
 *            may read and clear it.  Calls that share a workspace must not
 *            overlap on the GPU (use one per stream).
 * The result is deterministic: partial sums are combined in a fixed order.
 */
int q4_gemm_skinny(const void* A, const uint8_t* Wpacked, const float* absmax, const float* code,
                   int M, int N, int K, int blocksize, int act_dtype, void* out, void* workspace,
                   size_t workspace_bytes, void* stream);

/*
 * q4_gemm_skinny for callers that cannot allocate device memory (code that
 * runs while a stream is captured into a CUDA graph, runtimes that forbid
 * device allocations after start-up, plugin hosts that hand out no memory).
 * The paper has no counterpart: it exists for such callers only.
 *
 * Same arguments and results as q4_gemm_skinny, without the workspace: the
 * scratch is a fixed array of Q4_NOALLOC_WORKSPACE_BYTES compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.  No call allocates or frees memory (no cudaMalloc, no cudaFree,
 * no allocating library routine).
 *   - A problem whose workspace (q4_gemm_workspace_size) exceeds that size
 *     returns Q4_ERR_WORKSPACE and enqueues nothing.
 *   - The first call on a device looks the array's device address up once,
 *     with that device current (cudaGetSymbolAddress); make that first call
 *     before capturing a stream into a CUDA graph.
 *   - Every call shares the one array and clears its error word and tile
 *     counters with cudaMemsetAsync on `stream` before the kernel (not when
 *     the kernel's workspace is the 256-byte header alone); calls that
 *     overlap on the GPU (other streams, other threads) race on it.
 *   - The array's error word (see q4_gemm_skinny) is not reported: a call
 *     whose kernel gave up a bounded wait returns Q4_OK with outputs that
 *     are not valid, and the next call clears the word.  Callers that must
 *     see such failures use q4_gemm_skinny with their own workspace.
 *   - The cached address belongs to the CUDA context that was current at
 *     the first call; after cudaDeviceReset on that device, do not call
 *     this entry again in the same process.
 */
#define Q4_NOALLOC_WORKSPACE_BYTES (2u << 20) /* 2 MiB */

int q4_gemm_skinny_noalloc(const void* A, const uint8_t* Wpacked, const float* absmax,
                           const float* code, int M, int N, int K, int blocksize, int act_dtype,
                           void* out, void* stream);

/* Launch-table entry chosen for a GEMM problem (host-only, for reporting and
 * tests).  `num_sms` <= 0 means "the current device's SM count". */
typedef struct {
    int math;          /* 1 = tensor-core (mma.sync m16n8k16), 2 = CUDA-core FMA  */
                       /* (fp32 activations; bf16/fp16 on request, M <= 16),     */
                       /* 3 = tcgen05 with tensor memory                         */
    int sub_block;     /* k-width of one work unit: min(blocksize, 64); 512 for  */
                       /* math 2                                                 */
    int m_pad;         /* M padded to the MMA column count: 8, 16, 32 (math 1), */
                       /* 32/64/128 (math 3), 1/2/4/8/16 (math 2)                */
    int rows_per_tile; /* weight rows per work unit (32 for 17 <= M <= 32 on      */
                       /* math 1, 64 below, 128 for math 3, R for math 2)        */
    int warps;         /* warps per CTA                                           */
    int ctas;          /* persistent CTAs (<= SM count, <= number of units)       */
    int depth;         /* work units each warp has in flight ahead of its compute */
                       /* (loader 7: stage order, 1 round robin over the warps,  */
                       /* 2 a contiguous range of stages per warp)               */
    int l2_prefetch;   /* L2 fetch-size hint on weight loads: 1 none, 128, 256 B  */
                       /* (loader 7: 0 none, else stages fetched into L2 ahead   */
                       /* of the shared-memory ring)                             */
    int loader;        /* 1 = per-lane global loads; TMA shared-memory ring with  */
                       /* 2 = 4-unit (128-byte) or 3 = 2-unit (64-byte) stages,  */
                       /* units split over CTAs (stream-K); 7 = row-split: 8-row */
                       /* groups of W split over the CTAs, every output finished */
                       /* inside one CTA (the default at M <= 16 where it        */
                       /* measured faster; blocksize 32 with K % 256 == 0 too;   */
                       /* 17 <= M <= 32 on request, blocksize >= 64)             */
    int pdl;           /* programmatic dependent launch: 0 off; 1 on, the kernel  */
                       /* touches global memory only after the preceding grid    */
                       /* completed; 2 on, and code/Wpacked/absmax may be read   */
                       /* before that (they must not be written by the grid that */
                       /* precedes the call on the stream, e.g. static weights)  */
    int tiles;         /* ceil(N / rows_per_tile)                                 */
    int64_t units;     /* tiles * (K / sub_block)                                 */
    size_t smem_bytes; /* dynamic shared memory per CTA                           */
    size_t workspace_bytes;
} q4_gemm_plan_t;

int q4_gemm_plan(int M, int N, int K, int blocksize, int act_dtype, int num_sms,
                 q4_gemm_plan_t* plan);

/*
 * Same as q4_gemm_skinny with explicit launch-table overrides, used to
 * measure the choices the table makes and to opt into programmatic
 * dependent launch.  `overrides` may be NULL; in it, math, warps, ctas,
 * depth, l2_prefetch, loader and pdl override the table when > 0 (all
 * other fields are ignored).  A combination that was not compiled returns
 * Q4_ERR_UNSUPPORTED; ctas above the SM count returns Q4_ERR_INVALID_ARG.
 * Overrides that select another kernel (math = 3 below M = 33) change the
 * workspace layout: size the workspace with q4_gemm_workspace_size_ex.
 */
/* q4_gemm_workspace_size for a call with launch-table overrides (NULL: the
 * same as q4_gemm_workspace_size).  Host-only. */
int q4_gemm_workspace_size_ex(int M, int N, int K, int blocksize, int act_dtype, const q4_gemm_plan_t* overrides,
                              size_t* bytes);

int q4_gemm_skinny_ex(const void* A, const uint8_t* Wpacked, const float* absmax,
                      const float* code, int M, int N, int K, int blocksize, int act_dtype,
                      void* out, void* workspace, size_t workspace_bytes, void* stream,
                      const q4_gemm_plan_t* overrides);

/*
 * The layer with a bias, fused into the epilogue (the planned gemm_4bit op of
 * bitsandbytes PR #1920, "Technical details", takes an optional bias):
 *     out[m, n] = round_rn_act( bias[n] + sum_k A[m,k] * dequant(W)[n,k] )
 * the bias added in fp32 to the fp32 sum before the single rounding.
 *   bias       [N] act_dtype, aligned to its element size (2 or 4 bytes),
 *              not NULL when M, N > 0 (use
 *              q4_gemm_skinny for no bias); with K = 0 every output row is
 *              the bias.
 *   overrides  as for q4_gemm_skinny_ex (NULL: the launch table decides).
 * Every other argument, result and error as q4_gemm_skinny.
 */
int q4_gemm_skinny_bias(const void* A, const uint8_t* Wpacked, const float* absmax, const float* code,
                        const void* bias, int M, int N, int K, int blocksize, int act_dtype, void* out,
                        void* workspace, size_t workspace_bytes, void* stream, const q4_gemm_plan_t* overrides);

/*
 * Fused-vs-split routing (host-only; no GPU work, no device query).  The
 * maintainer's reply in PR #1920 describes heuristics that route each layer
 * to dequantize + matmul or to one of the fused kernels by problem size.
 * This is that choice for this library on B200:
 *   *route = Q4_ROUTE_FUSED  call q4_gemm_skinny (measured faster), or
 *          = Q4_ROUTE_SPLIT  dequantize (q4_dequantize_blockwise) and run a
 *                            dense GEMM: the fused kernels do not take the
 *                            problem, or are measured slower on it.
 * The rule, fitted to measurements on B200:
 *   - M <= 16 (bf16, fp16, fp32): fused (2.5-4.9x faster than the split
 *     path for bf16, 1.4-7.7x for fp32);
 *   - 17 <= M <= 32, bf16/fp16, blocksize >= 64 and (K / blocksize) % 4 == 0:
 *     fused, on the mma.sync kernel with 32-row tiles (parity on 15-24 MB
 *     layers, 1.9x faster on a 50 MB one);
 *   - 33 <= M <= 64, bf16/fp16, with at least 2^26 weights (N*K): fused (row
 *     chunks of 32 on the mma.sync kernels, or the tcgen05 kernel, beat the
 *     split path there; below it the split path is faster);
 *   - everything else the fused entry rejects (M > 128, fp32 with M > 16,
 *     the tcgen05 kernel's shape rules) or loses on: split.
 * Argument errors as q4_gemm_skinny (Q4_ERR_INVALID_ARG); route NULL ->
 * Q4_ERR_INVALID_ARG.
 */
typedef enum { Q4_ROUTE_FUSED = 0, Q4_ROUTE_SPLIT = 1 } q4_route;
int q4_gemm_route(int M, int N, int K, int blocksize, int act_dtype, int* route);

/*
 * Work partition used by the GEMM (host-callable so it can be checked
 * without a GPU): `total` units split into `parts` contiguous ranges,
 * part p owning [q4_partition_start(total, parts, p),
 *                q4_partition_start(total, parts, p + 1)).
 * q4_partition_owner returns the part owning unit u (0 <= u < total).
 */
int64_t q4_partition_start(int64_t total, int parts, int part);
int q4_partition_owner(int64_t total, int parts, int64_t u);

#ifdef __cplusplus
}
#endif

#endif /* Q4_H_ */
