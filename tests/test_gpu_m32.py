"""GPU parity of 17 <= M <= 32 on the mma.sync kernel with 32-row tiles
(two 16-row MMA tiles per unit, 2-unit TMA stages, activations padded to 32
MMA columns): every output element within 1e-2 * sum_k |a w| + ulp(y) of the
oracle.  The operation is the fused path of bitsandbytes PR #1920 ("Fused
path support for M > 1"); the maintainer's reply notes MMA kernels win at
M = 32 and beyond."""
import pytest
import torch

from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200.inputs import Case
from parity import run_case

pytestmark = pytest.mark.gpu


def _plan(M, N, K, bs=64):
    return q4.q4_gemm_plan(M, N, K, bs)


@pytest.mark.parametrize("M", [17, 20, 24, 31, 32])
@pytest.mark.parametrize("N,K", [(32, 256), (300, 1024), (513, 2048), (1000, 512), (65, 4096)])
def test_m32_bf16(cuda_device, M, N, K):
    p = _plan(M, N, K)
    assert p["math"] == 1 and p["loader"] == 3 and p["m_pad"] == 32 and p["rows_per_tile"] == 32
    run_case(Case(M, N, K), seed=8000 + M * 3 + N + K, device=cuda_device, check_quantizer=False)


@pytest.mark.parametrize("M", [17, 32])
@pytest.mark.parametrize("act,table", [("fp16", "normal"), ("bf16", "uniform"), ("bf16", "fp4"), ("fp16", "fp4")])
def test_m32_dtypes_tables(cuda_device, M, act, table):
    run_case(Case(M, 384, 1536, act=act, table=table), seed=8100 + M, device=cuda_device, check_quantizer=False)


@pytest.mark.parametrize("M", [19, 32])
@pytest.mark.parametrize("bs", [128, 256, 1024])
def test_m32_blocksizes(cuda_device, M, bs):
    run_case(Case(M, 256, 4096, blocksize=bs), seed=8200 + bs + M, device=cuda_device, check_quantizer=False)


@pytest.mark.parametrize("ctas", [1, 2, 3, 7, 33, 148])
def test_m32_partitions(cuda_device, ctas):
    """Tiles cut between warps and CTAs (shared-memory and workspace fix-ups) at every CTA count."""
    run_case(Case(25, 640, 2048), seed=8300 + ctas, device=cuda_device, check_quantizer=False, ctas=ctas)


def test_m32_outliers_and_bias(cuda_device):
    run_case(Case(32, 256, 2048, outliers=True), seed=8500, device=cuda_device, check_quantizer=False)
    import numpy as np
    import oracle
    from bit_weight_dequant_b200 import inputs
    from parity import bits_of, check_gemm
    M, N, K = 29, 333, 2048
    code = inputs.code_normal_quantile()
    W = inputs.weights(N, K, 8600)
    packed, absmax = oracle.quantize(W, 64, code)
    A = inputs.activations(M, K, torch.bfloat16, 8600)
    bias = inputs.activations(1, N, torch.bfloat16, 8601).reshape(N)
    y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, 64, bias_bits=bits_of(bias))
    dev = cuda_device
    out = q4.q4_gemm_skinny(A.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(absmax).to(dev),
                            torch.from_numpy(code).to(dev), N, K, 64, bias=bias.to(dev))
    check_gemm(bits_of(out), y, S, "bf16", "m32 bias")


def test_m32_deterministic(cuda_device):
    import numpy as np
    import oracle
    from bit_weight_dequant_b200 import inputs
    M, N, K = 32, 700, 4096
    code = inputs.code_normal_quantile()
    W = inputs.weights(N, K, 8700)
    packed, absmax = oracle.quantize(W, 64, code)
    A = inputs.activations(M, K, torch.bfloat16, 8700).to(cuda_device)
    args = (A, torch.from_numpy(packed).to(cuda_device), torch.from_numpy(absmax).to(cuda_device),
            torch.from_numpy(inputs.code_normal_quantile()).to(cuda_device), N, K, 64)
    a = q4.q4_gemm_skinny(*args, ctas=37).clone()
    b = q4.q4_gemm_skinny(*args, ctas=37).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("M", [33, 40, 48, 49, 63, 64])
@pytest.mark.parametrize("N,K,act", [(300, 1024, "bf16"), (513, 2048, "fp16"), (1000, 512, "bf16"),
                                     (65, 4096, "bf16")])
def test_row_chunks_33_to_64(cuda_device, M, N, K, act):
    """33 <= M <= 64: row chunks of 32 on the mma.sync kernels (the last
    chunk of M - 32 rows on its own kernel: the row-split kernel for up to 16
    rows, the 32-row kernel above), one after another on one workspace."""
    p = _plan(M, N, K)
    assert p["math"] == 1 and p["loader"] == 3 and p["m_pad"] == 32
    run_case(Case(M, N, K, act=act), seed=8600 + M * 3 + N + K, device=cuda_device, check_quantizer=False)


def test_row_chunks_bias_and_partitions(cuda_device):
    import oracle
    from bit_weight_dequant_b200 import inputs
    from parity import bits_of, check_gemm
    M, N, K = 57, 700, 2048
    code = inputs.code_normal_quantile()
    packed, absmax = oracle.quantize(inputs.weights(N, K, 8700), 64, code)
    A = inputs.activations(M, K, torch.bfloat16, 8701)
    bias = inputs.activations(1, N, torch.bfloat16, 8702).reshape(N)
    y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, 64, bias_bits=bits_of(bias))
    dev = cuda_device
    P, C = torch.from_numpy(packed).to(dev), torch.from_numpy(code).to(dev)
    Am = torch.from_numpy(absmax).to(dev)
    for kw in ({}, {"ctas": 5}, {"pdl": 2}):
        out = q4.q4_gemm_skinny(A.to(dev), P, Am, C, N, K, 64, bias=bias.to(dev), **kw)
        torch.cuda.synchronize()
        check_gemm(bits_of(out), y, S, "bf16", f"row chunks M57 {kw}")
