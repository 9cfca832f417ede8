"""q4_linear: each layer on the path q4_gemm_route recommends (the fused
kernel, or dequantize + cuBLAS GEMM), against the oracle within
1e-2 * sum_k |a w| + ulp(y).  The maintainer's reply in bitsandbytes PR
#1920 describes routing between dequantize + matmul and the fused kernels by
problem size."""
import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs
from parity import ORACLE_ACT, TORCH_ACT, bits_of, check_gemm, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("act", ["bf16", "fp16"])
@pytest.mark.parametrize("M,N,K,with_bias", [(4, 300, 1024, False), (128, 300, 1024, False), (200, 190, 512, True),
                                             (33, 257, 2048, True), (16, 64, 4096, True)])
def test_linear_matches_oracle(cuda_device, act, M, N, K, with_bias):
    dev = cuda_device
    code = inputs.code_normal_quantile()
    W = inputs.weights(N, K, 600 + M)
    packed, absmax = oracle.quantize(W, 64, code)
    A = inputs.activations(M, K, TORCH_ACT[act], 600 + M)
    bias = inputs.activations(1, N, TORCH_ACT[act], 601 + M).reshape(N) if with_bias else None
    y, S = oracle.gemm(bits_of(A), ORACLE_ACT[act], packed, absmax, code, M, N, K, 64,
                       bias_bits=bits_of(bias) if with_bias else None)
    out = q4.q4_linear(A.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(absmax).to(dev),
                       torch.from_numpy(code).to(dev), N, K, 64, bias=bias.to(dev) if with_bias else None)
    torch.cuda.synchronize(dev)
    route = q4.q4_gemm_route(M, N, K, 64, TORCH_ACT[act])
    assert route == (q4.Q4_ROUTE_FUSED if M <= 16 else q4.Q4_ROUTE_SPLIT)
    check_gemm(bits_of(out), y, S, act, f"linear {act} M{M} N{N} K{K} route {route}")


@pytest.mark.parametrize("M", [32, 64])
def test_linear_fused_tcgen05_route_sampled(cuda_device, M):
    """A large layer on the fused route (M = 32: the 32-row mma.sync kernel;
    M = 64: two row chunks of 32 on it, >= 2^26 weights), checked on sampled weight
    rows against the oracle."""
    dev = cuda_device
    N, K = 5120, 17408
    assert q4.q4_gemm_route(M, N, K, 64, torch.bfloat16) == q4.Q4_ROUTE_FUSED
    code = inputs.code_normal_quantile()
    code_d = torch.from_numpy(code).to(dev)
    Wd = inputs.weights_device(N, K, 700 + M, dev)
    packed, absmax = q4.q4_quantize_blockwise(Wd.reshape(-1), 64, code_d)
    rows = sample_rows(N, extra=24, seed=M)
    Wr = Wd[torch.from_numpy(rows).to(dev)].cpu().numpy()
    del Wd
    A = inputs.activations(M, K, torch.bfloat16, 700 + M)
    out = q4.q4_linear(A.to(dev), packed, absmax, code_d, N, K, 64)
    p_ref, a_ref = oracle.quantize(Wr, 64, code)
    y, S = oracle.gemm(bits_of(A), oracle.BF16, p_ref, a_ref, code, M, rows.size, K, 64)
    check_gemm(bits_of(out[:, torch.from_numpy(rows).to(dev)]), y, S, "bf16", f"linear tcgen05 M{M}")


def test_linear_fp32_routes(cuda_device):
    """fp32 activations: fused up to M = 16, split (fp32 dequantize + fp32
    GEMM) beyond; both against the oracle's fp32-activation layer."""
    dev = cuda_device
    code = inputs.code_uniform()
    N, K = 96, 1024
    W = inputs.weights(N, K, 800)
    packed, absmax = oracle.quantize(W, 64, code)
    for M in (3, 16, 40):
        A = inputs.activations_fp32(M, K, 800 + M)
        y, S = oracle.gemm_f32(A, packed, absmax, code, M, N, K, 64)
        out = q4.q4_linear(torch.from_numpy(A).to(dev), torch.from_numpy(packed).to(dev),
                           torch.from_numpy(absmax).to(dev), torch.from_numpy(code).to(dev), N, K, 64)
        got = out.cpu().numpy().astype(np.float64)
        tol = 1e-2 * S + oracle.ulp(y, oracle.FP32).reshape(y.shape)
        assert np.all(np.abs(got - y) <= tol), M
        assert q4.q4_gemm_route(M, N, K, 64, torch.float32) == (q4.Q4_ROUTE_FUSED if M <= 16 else q4.Q4_ROUTE_SPLIT)
