"""GPU parity of the fused dequantize + skinny GEMM against the oracle at
sizes the oracle finishes quickly: every output element must satisfy
|gpu - y| <= 1e-2 * sum_k |a w| + ulp(y).  The operation is the fused path of
bitsandbytes PR #1920 ("Fused path support for M > 1")."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs
from bit_weight_dequant_b200.inputs import Case
from parity import TORCH_ACT, bits_of, check_gemm, run_case

pytestmark = pytest.mark.gpu

SHAPES = [(1, 64), (12, 2560), (64, 64), (65, 128), (100, 320), (513, 1024), (320, 1280), (257, 4096), (130, 192)]


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 8, 9, 12, 16])
@pytest.mark.parametrize("N,K", SHAPES)
def test_gemm_bf16_normal(cuda_device, M, N, K):
    run_case(Case(M, N, K), seed=1000 + M * 7 + N + K, device=cuda_device)


@pytest.mark.parametrize("M", [1, 4, 13])
@pytest.mark.parametrize("bs", [32, 128, 256, 1024])
def test_gemm_blocksizes(cuda_device, M, bs):
    run_case(Case(M, 200, 2048, blocksize=bs), seed=2000 + bs + M, device=cuda_device)


@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("act,table", [("fp16", "normal"), ("bf16", "uniform"), ("fp16", "uniform"), ("bf16", "fp4"),
                                       ("fp16", "fp4")])
def test_gemm_dtypes_tables(cuda_device, M, act, table):
    run_case(Case(M, 300, 1536, act=act, table=table), seed=3000 + M, device=cuda_device)


@pytest.mark.parametrize("M", [1, 8])
def test_gemm_outliers(cuda_device, M):
    run_case(Case(M, 256, 2048, outliers=True), seed=4000 + M, device=cuda_device)


# Launch-table overrides on the direct-load kernel: tiles cut between CTAs
# (global fix-up) and between warps (shared-memory combine), empty warp
# ranges, single CTA.
@pytest.mark.parametrize("ctas", [1, 2, 3, 7, 64, 148])
@pytest.mark.parametrize("warps", [8, 16])
@pytest.mark.parametrize("M", [1, 6])
def test_gemm_partition_overrides(cuda_device, ctas, warps, M):
    run_case(Case(M, 257, 1280), seed=5000 + ctas, device=cuda_device, check_quantizer=False, ctas=ctas, warps=warps,
             loader=1)


@pytest.mark.parametrize("ctas", [1, 5, 33])
@pytest.mark.parametrize("M", [9, 16])
def test_gemm_partition_overrides_m16(cuda_device, ctas, M):
    run_case(Case(M, 190, 960), seed=6000 + ctas, device=cuda_device, check_quantizer=False, ctas=ctas, warps=8,
             loader=1)


def _problem(device, M=3, N=300, K=1024, bs=64, seed=7):
    code = inputs.code_normal_quantile()
    W = inputs.weights(N, K, seed)
    packed, absmax = oracle.quantize(W, bs, code)
    A = inputs.activations(M, K, torch.bfloat16, seed).to(device)
    return (A, torch.from_numpy(packed).to(device), torch.from_numpy(absmax).to(device),
            torch.from_numpy(code).to(device), N, K, bs)


@pytest.mark.parametrize("loader", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("N,K,ctas", [(300, 1024, 5), (64, 4096, 20), (200, 2048, 7)])
def test_deterministic_and_counters_left_zero(cuda_device, loader, N, K, ctas):
    """Repeated calls agree bit for bit, match the oracle and leave every tile
    counter at zero: tiles cut between 2, 3 or 20 CTAs."""
    A, P, Am, C, N, K, bs = _problem(cuda_device, N=N, K=K)
    ws = q4.Workspace(cuda_device)
    outs = [q4.q4_gemm_skinny(A, P, Am, C, N, K, bs, workspace=ws, ctas=ctas, loader=loader) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    assert q4.workspace_error(ws) == 0
    off = q4.workspace_counter_offset(cuda_device)
    assert ws.buf.numel() > off and int(ws.buf[off:].count_nonzero()) == 0
    y, S = oracle.gemm(bits_of(A.cpu()), oracle.BF16, P.cpu().numpy(), Am.cpu().numpy(), C.cpu().numpy(), A.shape[0], N, K, bs)
    check_gemm(bits_of(outs[0].cpu()), y, S, "bf16", f"loader {loader} ctas {ctas}")


@pytest.mark.parametrize("order", [0, 1])
def test_one_workspace_serves_shapes_in_any_order(cuda_device, order):
    """Scratch left by a call of one shape must not disturb the next shape."""
    ws = q4.Workspace(cuda_device)
    shapes = [(2, 4000, 2560), (3, 300, 1024), (1, 9000, 640)]
    if order:
        shapes = shapes[::-1]
    for M, N, K in shapes:
        code = inputs.code_normal_quantile()
        W = inputs.weights(N, K, N + K)
        packed, absmax = oracle.quantize(W, 64, code)
        A = inputs.activations(M, K, torch.bfloat16, N)
        y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, 64)
        out = q4.q4_gemm_skinny(A.to(cuda_device), torch.from_numpy(packed).to(cuda_device),
                                torch.from_numpy(absmax).to(cuda_device), torch.from_numpy(code).to(cuda_device),
                                N, K, 64, workspace=ws)
        torch.cuda.synchronize()
        check_gemm(bits_of(out), y, S, "bf16", label=f"M{M} N{N} K{K}")


@pytest.mark.parametrize("depth,l2pf,warps", [(1, 1, 16), (1, 256, 16), (1, 128, 16), (2, 128, 8), (2, 1, 8)])
def test_direct_load_variants(cuda_device, depth, l2pf, warps):
    run_case(Case(1, 700, 2048), seed=7000 + depth, device=cuda_device, check_quantizer=False, depth=depth,
             l2_prefetch=l2pf, warps=warps, loader=1)
    run_case(Case(1, 190, 640), seed=7100 + depth, device=cuda_device, check_quantizer=False, depth=depth,
             l2_prefetch=l2pf, warps=warps, ctas=5, loader=1)


@pytest.mark.parametrize("loader,warps,depth", [(2, 8, 2), (2, 16, 1), (2, 12, 1), (3, 16, 2), (3, 8, 4), (3, 12, 2),
                                                (3, 16, 1), (4, 8, 2), (4, 16, 1), (4, 12, 1), (5, 16, 2), (5, 8, 4)])
def test_tma_ring_variants(cuda_device, loader, warps, depth):
    run_case(Case(1, 700, 2048), seed=7200 + warps, device=cuda_device, check_quantizer=False, depth=depth,
             warps=warps, loader=loader)
    run_case(Case(3, 190, 768), seed=7300 + warps, device=cuda_device, check_quantizer=False, depth=depth,
             warps=warps, ctas=5, loader=loader)


@pytest.mark.parametrize("M", [1, 7, 8, 9, 16])
@pytest.mark.parametrize("N,K,bs", [(1, 256, 64), (64, 256, 64), (100, 1280, 64), (513, 1024, 128), (300, 4096, 256),
                                    (257, 3072, 64), (70, 512, 128)])
@pytest.mark.parametrize("loader", [2, 3, 4])
def test_tma_ring_shapes(cuda_device, M, N, K, bs, loader):
    run_case(Case(M, N, K, blocksize=bs), seed=7400 + M + N, device=cuda_device, check_quantizer=False, loader=loader)


@pytest.mark.parametrize("ctas", [1, 2, 3, 7, 33, 148])
@pytest.mark.parametrize("loader", [2, 3, 4, 5])
def test_tma_ring_partitions(cuda_device, ctas, loader):
    run_case(Case(2, 257, 1280), seed=7500 + ctas, device=cuda_device, check_quantizer=False, loader=loader, ctas=ctas)


def test_tma_error_word_stays_zero(cuda_device):
    ws = q4.Workspace(cuda_device)
    A, P, Am, C, N, K, bs = _problem(cuda_device)
    for loader in (2, 3, 4, 5, 7):
        q4.q4_gemm_skinny(A, P, Am, C, N, K, bs, workspace=ws, loader=loader)
    torch.cuda.synchronize()
    assert q4.workspace_error(ws) == 0


def test_empty_and_degenerate(cuda_device):
    A, P, Am, C, N, K, bs = _problem(cuda_device)
    out = q4.q4_gemm_skinny(A[:0], P, Am, C, N, K, bs)          # M = 0
    assert out.shape == (0, N)
    out = q4.q4_gemm_skinny(A, P, Am, C, 0, K, bs)             # N = 0
    assert out.shape == (A.shape[0], 0)
    z = torch.empty((A.shape[0], 0), dtype=A.dtype, device=cuda_device)
    out = torch.full((A.shape[0], N), 7.0, dtype=A.dtype, device=cuda_device)
    q4.q4_gemm_skinny(z, P, Am, C, N, 0, bs, out=out)          # K = 0 -> zeros
    torch.cuda.synchronize()
    assert int(out.count_nonzero()) == 0


def test_error_paths_leave_no_sticky_error(cuda_device, monkeypatch):
    A, P, Am, C, N, K, bs = _problem(cuda_device)
    ref = q4.q4_gemm_skinny(A, P, Am, C, N, K, bs)
    Amis = torch.zeros(A.numel() + 1, dtype=A.dtype, device=cuda_device)[1:].view_as(A)
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_gemm_skinny(Amis, P, Am, C, N, K, bs)
    assert e.value.status == q4.Q4_ERR_MISALIGNED
    L = q4.lib()
    out = torch.empty_like(ref)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    need = q4.q4_gemm_workspace_size(A.shape[0], N, K, bs, A.dtype)
    if need:
        assert L.q4_gemm_skinny(ptr(A), ptr(P), ptr(Am), ptr(C), A.shape[0], N, K, bs, 0, ptr(out), None, 0,
                                None) == q4.Q4_ERR_WORKSPACE
    monkeypatch.setenv("Q4_TEST_FAIL_LAUNCH", "1")
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_gemm_skinny(A, P, Am, C, N, K, bs)
    assert e.value.status == q4.Q4_ERR_CUDA
    monkeypatch.delenv("Q4_TEST_FAIL_LAUNCH")
    again = q4.q4_gemm_skinny(A, P, Am, C, N, K, bs)
    torch.cuda.synchronize()
    assert torch.equal(again.view(torch.int16), ref.view(torch.int16))


def test_one_hot_activation_selects_dequantized_column(cuda_device):
    """A = e_k: out[0, n] = w[n, k] up to the kernel's rounding of the code to
    bf16 before the MMA (relative 2^-8, bf16's unit roundoff) and the final bf16 rounding, i.e.
    within one bf16 ulp of the oracle's bf16(w[n, k])."""
    M, N, K, bs = 1, 300, 1024, 64
    code = inputs.code_normal_quantile()
    packed, absmax = oracle.quantize(inputs.weights(N, K, 7), bs, code)
    want_all = oracle.decode(oracle.dequantize(packed, absmax, code, N * K, bs, oracle.BF16), oracle.BF16)
    want_all = want_all.reshape(N, K)
    P, Am, C = (torch.from_numpy(x).to(cuda_device) for x in (packed, absmax, code))
    for k in (0, 17, 64, K - 1):
        e = torch.zeros((1, K), dtype=torch.bfloat16, device=cuda_device)
        e[0, k] = 1.0
        out = q4.q4_gemm_skinny(e, P, Am, C, N, K, bs)
        want = want_all[:, k]
        got = out[0].to(torch.float64).cpu().numpy()
        assert np.all(np.abs(got - want) <= oracle.ulp(want, oracle.BF16)), k


@pytest.mark.parametrize("pdl", [1, 2])
@pytest.mark.parametrize("loader", [1, 3, 4, 7])
def test_dependent_launch_chain(cuda_device, pdl, loader):
    """A chain where each GEMM reads the previous GEMM's output as its
    activations: with programmatic dependent launch the second kernel may
    start early, but must read its activations only after the first one
    finished.  The result must equal the chain run without it, bit for bit."""
    dims = [2048, 1536, 2560, 1024]                  # K of step i = N of step i-1
    code = inputs.code_normal_quantile()
    C = torch.from_numpy(code).to(cuda_device)
    layers = []
    for i in range(len(dims) - 1):
        K, N = dims[i], dims[i + 1]
        packed, absmax = oracle.quantize(inputs.weights(N, K, 900 + i), 64, code)
        layers.append((torch.from_numpy(packed).to(cuda_device), torch.from_numpy(absmax).to(cuda_device), N, K))
    A0 = inputs.activations(4, dims[0], torch.bfloat16, 901).to(cuda_device)

    def chain(**launch):
        x = A0
        for (P, Am, N, K) in layers:
            x = q4.q4_gemm_skinny(x, P, Am, C, N, K, 64, loader=loader, **launch)
        return x

    ref = chain()
    torch.cuda.synchronize()
    for _ in range(3):
        got = chain(pdl=pdl)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_q4layer_matches_gemm_and_follows_in_place_activations(cuda_device):
    """Q4Layer (the bound, one-C-call form of q4_gemm_skinny) gives the same
    bits as q4_gemm_skinny and reads whatever its activation buffer holds."""
    dev = cuda_device
    M, N, K = 3, 300, 2048
    code = torch.from_numpy(inputs.code_normal_quantile()).to(dev)
    W = inputs.weights_device(N, K, 55, dev)
    packed, absmax = q4.q4_quantize_blockwise(W.reshape(-1), 64, code)
    A = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    bias = inputs.activations(1, N, torch.bfloat16, 57).reshape(N).to(dev)
    layer = q4.Q4Layer(packed, absmax, code, N, K, 64, A)
    layer_b = q4.Q4Layer(packed, absmax, code, N, K, 64, A, bias=bias, pdl=2)
    for seed in (1, 2):
        A.copy_(inputs.activations(M, K, torch.bfloat16, seed).to(dev))
        want = q4.q4_gemm_skinny(A, packed, absmax, code, N, K, 64)
        want_b = q4.q4_gemm_skinny(A, packed, absmax, code, N, K, 64, bias=bias)
        got, got_b = layer().clone(), layer_b().clone()
        torch.cuda.synchronize(dev)
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), seed
        assert torch.equal(got_b.view(torch.int16), want_b.view(torch.int16)), seed
