"""The bias epilogue (q4_gemm_skinny_bias) against the oracle's layer with a
bias: out = round(bias + A . dequant(W)^T), every element within
1e-2 * sum_k |a w| + ulp(y).  The planned gemm_4bit op of bitsandbytes
PR #1920 ("Technical details") takes an optional bias."""
import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs
from parity import ORACLE_ACT, TORCH_ACT, bits_of, check_gemm

pytestmark = pytest.mark.gpu


def _problem(M, N, K, act, seed, table="normal"):
    code = inputs.CODE_TABLES[table]()
    W = inputs.weights(N, K, seed)
    packed, absmax = oracle.quantize(W, 64, code)
    A = inputs.activations(M, K, TORCH_ACT[act], seed)
    bias = inputs.activations(1, N, TORCH_ACT[act], seed + 1).reshape(N)
    return code, packed, absmax, A, bias


@pytest.mark.parametrize("act", ["bf16", "fp16"])
@pytest.mark.parametrize("M,N,K", [(1, 300, 1024), (5, 513, 2048), (16, 190, 1024), (3, 64, 64)])
@pytest.mark.parametrize("launch", [{}, {"loader": 1}, {"loader": 3}, {"loader": 1, "ctas": 7}, {"ctas": 5}])
def test_bias_matches_oracle(cuda_device, act, M, N, K, launch):
    if launch.get("loader", 0) >= 2 and (K // 64) % 4:
        pytest.skip("the TMA loaders need (K / blocksize) % 4 == 0")
    code, packed, absmax, A, bias = _problem(M, N, K, act, 900 + M + N)
    y, S = oracle.gemm(bits_of(A), ORACLE_ACT[act], packed, absmax, code, M, N, K, 64, bias_bits=bits_of(bias))
    dev = cuda_device
    out = q4.q4_gemm_skinny(A.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(absmax).to(dev),
                            torch.from_numpy(code).to(dev), N, K, 64, bias=bias.to(dev), **launch)
    check_gemm(bits_of(out), y, S, act, f"bias {act} M{M} N{N} K{K} {launch}")


def test_bias_applied_once_with_cut_tiles(cuda_device):
    """All weights zero (absmax 0): the output is the bias itself, bit for bit,
    also when every tile is summed from partials of several CTAs."""
    M, N, K = 4, 200, 2048
    code, packed, absmax, A, bias = _problem(M, N, K, "bf16", 11)
    dev = cuda_device
    for launch in ({}, {"ctas": 37}, {"loader": 1, "ctas": 64}):
        out = q4.q4_gemm_skinny(A.to(dev), torch.from_numpy(packed).to(dev),
                                torch.zeros(absmax.size, dtype=torch.float32, device=dev),
                                torch.from_numpy(code).to(dev), N, K, 64, bias=bias.to(dev), **launch)
        assert torch.equal(out.cpu().view(torch.int16), bias.expand(M, N).view(torch.int16)), launch


def test_bias_with_empty_contraction(cuda_device):
    M, N = 3, 77
    bias = inputs.activations(1, N, torch.bfloat16, 5).reshape(N).to(cuda_device)
    A = torch.zeros((M, 0), dtype=torch.bfloat16, device=cuda_device)
    empty_u8 = torch.zeros(0, dtype=torch.uint8, device=cuda_device)
    empty_f = torch.zeros(0, dtype=torch.float32, device=cuda_device)
    code = torch.from_numpy(inputs.code_normal_quantile()).to(cuda_device)
    out = q4.q4_gemm_skinny(A, empty_u8, empty_f, code, N, 0, 64, bias=bias)
    assert torch.equal(out.view(torch.int16), bias.expand(M, N).view(torch.int16))


def test_misaligned_bias_rejected(cuda_device):
    M, N, K = 1, 64, 128
    code, packed, absmax, A, bias = _problem(M, N, K, "bf16", 3)
    dev = cuda_device
    buf = torch.zeros(N + 1, dtype=torch.uint8, device=dev)
    odd = torch.zeros(2 * N + 2, dtype=torch.uint8, device=dev)[1:2 * N + 1].view(torch.uint8)
    L = q4.lib()
    Ad, P, Am, C = A.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(absmax).to(dev), torch.from_numpy(code).to(dev)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = q4.Workspace(dev).get(q4.q4_gemm_workspace_size(M, N, K, 64, torch.bfloat16) or 16)
    rc = L.q4_gemm_skinny_bias(Ad.data_ptr(), P.data_ptr(), Am.data_ptr(), C.data_ptr(), odd.data_ptr(), M, N, K, 64,
                               q4.Q4_BF16, out.data_ptr(), ws.data_ptr(), ws.numel(),
                               torch.cuda.current_stream().cuda_stream, None)
    assert rc == q4.Q4_ERR_MISALIGNED
    del buf
