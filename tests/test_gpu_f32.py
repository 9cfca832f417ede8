"""fp32 activations (the maintainer's reply in bitsandbytes PR #1920: the SIMT
kernel takes fp32 as well as fp16/bf16 inputs, all accumulating in fp32)
against the oracle's fp32-activation layer.

Two bounds per output element:
  * the contract: |gpu - y| <= 1e-2 * S + ulp_fp32(y), S = sum_k |a w|;
  * fp32 arithmetic: every product is an fp32 FMA with the exact code value,
    so the error is that of an fp32 sum, |gpu - y| <= d * 2^-24 * S + ulp(y)
    with d bounding the rounding depth of any term.  The kernel rounds each
    term at most 8 times in its block piece, K/256 times along a lane's
    running sum, 5 times across lanes and once per warp piece it is combined
    with; the oracle's own fp32 weight adds one.  d = 32 + K/128 covers that
    with a factor 2 on the K term.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs
from parity import check_f32, sample_rows

pytestmark = pytest.mark.gpu

def _problem(M, N, K, bs, seed, table="normal", outliers=False):
    code = inputs.CODE_TABLES[table]()
    W = inputs.weights(N, K, seed, outliers)
    packed, absmax = oracle.quantize(W, bs, code)
    A = inputs.activations_fp32(M, K, seed)
    return code, packed, absmax, A


def _run(dev, code, packed, absmax, A, N, K, bs, bias=None, **launch):
    return q4.q4_gemm_skinny(torch.from_numpy(A).to(dev), torch.from_numpy(packed).to(dev),
                             torch.from_numpy(absmax).to(dev), torch.from_numpy(code).to(dev), N, K, bs,
                             bias=None if bias is None else torch.from_numpy(bias).to(dev), **launch)


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 12, 16])
@pytest.mark.parametrize("N,K", [(300, 1024), (513, 2560), (61, 1088), (1, 32), (190, 320)])
def test_f32_matches_oracle(cuda_device, M, N, K):
    bs = 32 if K % 64 else 64
    code, packed, absmax, A = _problem(M, N, K, bs, 4000 + 7 * M + N)
    y, S = oracle.gemm_f32(A, packed, absmax, code, M, N, K, bs)
    out = _run(cuda_device, code, packed, absmax, A, N, K, bs)
    torch.cuda.synchronize(cuda_device)
    assert out.dtype == torch.float32 and tuple(out.shape) == (M, N)
    check_f32(out, y, S, K, f"f32 M{M} N{N} K{K}")


@pytest.mark.parametrize("bs", [32, 64, 128, 256, 1024, 4096])
@pytest.mark.parametrize("table", ["uniform", "normal", "fp4"])
def test_f32_blocksizes_and_tables(cuda_device, bs, table):
    M, N, K = 3, 77, 4096
    code, packed, absmax, A = _problem(M, N, K, bs, 4100 + bs, table, outliers=(bs == 64))
    y, S = oracle.gemm_f32(A, packed, absmax, code, M, N, K, bs)
    out = _run(cuda_device, code, packed, absmax, A, N, K, bs)
    check_f32(out, y, S, K, f"f32 bs{bs} {table}")


@pytest.mark.parametrize("M,N,K,ctas", [(1, 64, 16384, 0), (4, 24, 32768, 0), (2, 1000, 4096, 3), (16, 130, 8192, 5),
                                        (1, 4096, 4096, 148), (8, 9, 65536, 0)])
def test_f32_row_groups_split_over_warps(cuda_device, M, N, K, ctas):
    """Long rows with few row groups: each group is summed from the pieces of
    many warps (and CTAs) through the workspace, in warp order."""
    code, packed, absmax, A = _problem(M, N, K, 64, 4200 + N)
    y, S = oracle.gemm_f32(A, packed, absmax, code, M, N, K, 64)
    ws = q4.Workspace(cuda_device)
    launch = {"ctas": ctas} if ctas else {}
    outs = [_run(cuda_device, code, packed, absmax, A, N, K, 64, workspace=ws, **launch) for _ in range(2)]
    torch.cuda.synchronize(cuda_device)
    check_f32(outs[0], y, S, K, f"f32 split M{M} N{N} K{K} ctas{ctas}")
    assert torch.equal(outs[0].view(torch.int32), outs[1].view(torch.int32)), "not deterministic"
    tiles = q4.q4_gemm_plan(M, N, K, 64, torch.float32)["tiles"]
    off = q4.workspace_counter_offset(cuda_device)
    assert int(ws.buf[off:off + 4 * tiles].view(torch.int32).abs().sum()) == 0, "row-group counters not zero"


def test_f32_bias(cuda_device):
    M, N, K = 5, 333, 2048
    code, packed, absmax, A = _problem(M, N, K, 64, 4300)
    bias = inputs.activations_fp32(1, N, 4301).reshape(N)
    y, S = oracle.gemm_f32(A, packed, absmax, code, M, N, K, 64, bias=bias)
    for launch in ({}, {"ctas": 3}):
        out = _run(cuda_device, code, packed, absmax, A, N, K, 64, bias=bias, **launch)
        check_f32(out, y, S, K, f"f32 bias {launch}")
    # zero weights: the bias itself, bit for bit
    out0 = q4.q4_gemm_skinny(torch.from_numpy(A).to(cuda_device), torch.from_numpy(packed).to(cuda_device),
                             torch.zeros(absmax.size, dtype=torch.float32, device=cuda_device),
                             torch.from_numpy(code).to(cuda_device), N, K, 64,
                             bias=torch.from_numpy(bias).to(cuda_device), ctas=7)
    assert torch.equal(out0.cpu(), torch.from_numpy(bias).expand(M, N))


def test_f32_empty_and_degenerate(cuda_device):
    dev = cuda_device
    code = torch.from_numpy(inputs.code_normal_quantile()).to(dev)
    empty_u8 = torch.zeros(0, dtype=torch.uint8, device=dev)
    empty_f = torch.zeros(0, dtype=torch.float32, device=dev)
    out = q4.q4_gemm_skinny(torch.zeros((3, 0), dtype=torch.float32, device=dev), empty_u8, empty_f, code, 9, 0, 64)
    assert torch.equal(out.cpu(), torch.zeros(3, 9))
    bias = torch.arange(9, dtype=torch.float32, device=dev) - 4.5
    out = q4.q4_gemm_skinny(torch.zeros((2, 0), dtype=torch.float32, device=dev), empty_u8, empty_f, code, 9, 0, 64,
                            bias=bias)
    assert torch.equal(out, bias.expand(2, 9))
    # one-hot rows pick single dequantized weights exactly
    N, K = 40, 256
    cnp, packed, absmax, _ = _problem(1, N, K, 32, 4400)
    A = np.zeros((4, K), dtype=np.float32)
    for m, k in enumerate((0, 31, 32, 255)):
        A[m, k] = 1.0
    y, _ = oracle.gemm_f32(A, packed, absmax, cnp, 4, N, K, 32)
    out = _run(dev, cnp, packed, absmax, A, N, K, 32)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), y)


def test_f32_unsupported_and_misaligned(cuda_device):
    dev = cuda_device
    L = q4.lib()
    p = lambda n: torch.zeros(n, dtype=torch.uint8, device=dev)
    A, W, am, code, out = p(4096 * 17 * 4), p(64 * 2048), p(4096), p(64), p(64 * 17 * 4)
    ws = q4.Workspace(dev).get(1 << 21)
    st = torch.cuda.current_stream().cuda_stream
    args = (A.data_ptr(), W.data_ptr(), am.data_ptr(), code.data_ptr())
    assert L.q4_gemm_skinny(*args, 17, 64, 4096, 64, q4.Q4_FP32, out.data_ptr(), ws.data_ptr(), ws.numel(),
                            st) == q4.Q4_ERR_UNSUPPORTED
    odd_bias = p(64 * 4 + 4)[2:].data_ptr()
    assert L.q4_gemm_skinny_bias(*args, odd_bias, 1, 64, 4096, 64, q4.Q4_FP32, out.data_ptr(), ws.data_ptr(),
                                 ws.numel(), st, None) == q4.Q4_ERR_MISALIGNED
    for ov in (q4.overrides(math=1), q4.overrides(math=3), q4.overrides(loader=2), q4.overrides(warps=3)):
        assert L.q4_gemm_skinny_ex(*args, 1, 64, 4096, 64, q4.Q4_FP32, out.data_ptr(), ws.data_ptr(), ws.numel(),
                                   st, ov) == q4.Q4_ERR_UNSUPPORTED


@pytest.mark.parametrize("M,N,K", [(1, 28672, 8192), (1, 8192, 28672), (4, 10240, 8192), (16, 5120, 17408)])
def test_f32_full_size_sampled(cuda_device, M, N, K):
    """Full-size layers in the default launch: sampled weight rows against
    the oracle (W drawn on the device by the seeded generator)."""
    dev = cuda_device
    seed = 4500 + M
    code = inputs.code_normal_quantile()
    code_d = torch.from_numpy(code).to(dev)
    W = inputs.weights_device(N, K, seed, dev)
    packed, absmax = q4.q4_quantize_blockwise(W.reshape(-1), 64, code_d)
    rows = sample_rows(N, seed=seed)
    rows_d = torch.from_numpy(rows).to(dev)
    Wr = W[rows_d].cpu().numpy()
    del W
    A = inputs.activations_fp32(M, K, seed)
    out = q4.q4_gemm_skinny(torch.from_numpy(A).to(dev), packed, absmax, code_d, N, K, 64)
    p_ref, a_ref = oracle.quantize(Wr, 64, code)
    y, S = oracle.gemm_f32(A, p_ref, a_ref, code, M, rows.size, K, 64)
    check_f32(out[:, rows_d], y, S, K, f"f32 full M{M} N{N} K{K}")


@pytest.mark.parametrize("act", ["bf16", "fp16"])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 7, 16])
@pytest.mark.parametrize("N,K,bs", [(300, 1024, 64), (513, 2560, 64), (61, 1088, 32), (190, 4096, 256)])
def test_simt_16bit_activations(cuda_device, act, M, N, K, bs):
    """The same kernel on bf16 / fp16 activations (override math = 2): the
    activations are widened exactly, every product is an fp32 FMA and the
    output is rounded once to the activation type."""
    from parity import run_case
    run_case(inputs.Case(M, N, K, blocksize=bs, act=act), seed=4700 + M + N, device=cuda_device,
             check_quantizer=False, math=2)


@pytest.mark.parametrize("ctas", [1, 3, 37])
def test_simt_16bit_split_groups_and_bias(cuda_device, ctas):
    """Row groups cut by warp boundaries and the bias epilogue, bf16."""
    M, N, K, bs = 3, 700, 3072, 64
    code, packed, absmax, _ = _problem(M, N, K, bs, 4800 + ctas)
    A = inputs.activations(M, K, torch.bfloat16, 4801 + ctas)
    bias = inputs.activations(1, N, torch.bfloat16, 4802).reshape(N)
    dev = cuda_device
    out = q4.q4_gemm_skinny(A.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(absmax).to(dev),
                            torch.from_numpy(code).to(dev), N, K, bs, bias=bias.to(dev), math=2, ctas=ctas)
    torch.cuda.synchronize(dev)
    from parity import bits_of, check_gemm
    y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, bs, bias_bits=bits_of(bias))
    check_gemm(bits_of(out), y, S, "bf16", f"simt bf16 bias ctas {ctas}")
