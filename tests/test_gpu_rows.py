"""GPU parity of the row-split fused kernel (launch-table loader 7, the
default for M <= 16 with 16-bit activations when blocksize >= 64 and
(K / blocksize) % 4 == 0, or blocksize 32 and K % 256 == 0) against the
oracle: every output element within
|gpu - y| <= 1e-2 * sum_k |a w| + ulp(y).

The kernel splits 8-row groups of W over the CTAs and finishes every output
inside one CTA; the cases below cover the shapes of that split (one CTA,
CTAs with one group, ragged last groups past N, groups that leave partial
64-row tiles), tiles of every height up to 72 rows, the L2 prefetch ahead of the stage
ring, every blocksize from 32 to 4096, fp16,
the code tables, the bias epilogue, dependent-launch chains, determinism,
and a bounded wait that is made to run out.  The operation is the fused path
of bitsandbytes PR #1920 ("Fused path support for M > 1")."""
import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs
from bit_weight_dequant_b200.inputs import Case
from parity import bits_of, check_gemm, run_case

pytestmark = pytest.mark.gpu

SHAPES = [(8, 256), (12, 2560), (100, 1280), (257, 4096), (513, 1024), (1000, 2048), (1190, 768), (3000, 512),
          (200, 16384)]


@pytest.mark.parametrize("M", [1, 3, 8, 9, 16])
@pytest.mark.parametrize("N,K", SHAPES)
def test_rows_shapes(cuda_device, M, N, K):
    run_case(Case(M, N, K), seed=11000 + 7 * M + N + K, device=cuda_device, check_quantizer=False, loader=7)


@pytest.mark.parametrize("M", [1, 16, 32])
@pytest.mark.parametrize("N,K", [(1, 256), (3, 512), (7, 768), (5, 256), (9, 256)])
def test_rows_tiny_layers(cuda_device, M, N, K):
    """Fewer rows than one 8-row group and fewer k-stages than warps: one CTA,
    one short tile, most warps idle."""
    run_case(Case(M, N, K), seed=12400 + 31 * M + N + K, device=cuda_device, check_quantizer=False, loader=7)


@pytest.mark.parametrize("ctas", [1, 2, 3, 7, 33, 148])
@pytest.mark.parametrize("M", [1, 5, 12])
def test_rows_partitions(cuda_device, ctas, M):
    """Explicit CTA counts: more groups per CTA than one 64-row tile holds,
    the larger shares first, partial last tiles of 8 .. 56 rows."""
    run_case(Case(M, 1100, 1536), seed=11100 + ctas + M, device=cuda_device, check_quantizer=False, loader=7,
             ctas=ctas)


@pytest.mark.parametrize("ng", [1, 2, 3, 8, 9, 10, 11, 17, 18, 19, 25, 36])
@pytest.mark.parametrize("M", [1, 9])
def test_rows_tile_heights(cuda_device, ng, M):
    """CTAs of ng and ng + 1 8-row groups: tiles of 8 .. 72 rows (64 with
    M > 8), taller tiles first, half 16-row MMA tiles, ragged N."""
    ctas = 3
    N = 8 * ng * ctas + 8 * (ctas - 1) - 3  # two CTAs get ng + 1 groups, the last group is ragged
    run_case(Case(M, N, 768), seed=11200 + ng + M, device=cuda_device, check_quantizer=False, loader=7, ctas=ctas)


@pytest.mark.parametrize("ctas", [1, 3, 33, 148])
@pytest.mark.parametrize("N,K", [(1100, 1536), (300, 256), (40, 1024), (5000, 768), (24, 2048)])
def test_rows_contiguous_warp_ranges(cuda_device, ctas, N, K):
    """Stage order 2 (depth override): each warp streams its own contiguous
    range through its own ring slots; tiles shared by warps are combined in
    shared memory, including CTAs with fewer stages than warps."""
    if ctas > (N + 7) // 8:
        pytest.skip("more CTAs than 8-row groups")
    run_case(Case(3, N, K), seed=11250 + ctas + N, device=cuda_device, check_quantizer=False, loader=7, depth=2,
             ctas=ctas)


@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("M", [2, 12])
@pytest.mark.parametrize("K,ctas", [(256, 1), (512, 1), (768, 2), (1536, 1), (256, 5)])
def test_rows_many_short_tiles(cuda_device, order, M, K, ctas):
    """Tiles of fewer k-stages than warps, many tiles per CTA: warps hold no
    part of some tiles and reach a parking buffer several reductions ahead
    of others (one buffer with two column tiles, two with one)."""
    run_case(Case(M, 1100, K), seed=11260 + K + M + ctas, device=cuda_device, check_quantizer=False, loader=7,
             depth=order, ctas=ctas)


@pytest.mark.parametrize("ahead", [2, 16, 200])
def test_rows_l2_prefetch(cuda_device, ahead):
    run_case(Case(1, 5000, 4096), seed=11300 + ahead, device=cuda_device, check_quantizer=False, loader=7,
             l2_prefetch=ahead)


@pytest.mark.parametrize("M", [1, 6, 16])
@pytest.mark.parametrize("bs,K", [(32, 1280), (32, 4096), (64, 1280), (128, 1536), (256, 4096), (512, 2048),
                                  (1024, 8192), (4096, 16384)])
def test_rows_blocksizes(cuda_device, M, bs, K):
    run_case(Case(M, 333, K, blocksize=bs), seed=11400 + bs + M, device=cuda_device, check_quantizer=False,
             loader=7)


@pytest.mark.parametrize("M", [1, 9])
@pytest.mark.parametrize("ctas,depth", [(1, 0), (3, 0), (37, 2), (148, 0)])
@pytest.mark.parametrize("N", [300, 1003])
def test_rows_blocksize32(cuda_device, M, ctas, depth, N):
    """Blocksize 32: two absmax per 64-k unit (8-float boxes per stage, tiles
    of at most 56 rows), each half of the unit's MMAs scaled by its own
    block; a request for contiguous ranges falls back to round robin."""
    if ctas > (N + 7) // 8:
        pytest.skip("more CTAs than 8-row groups")
    kw = {"ctas": ctas}
    if depth:
        kw["depth"] = depth
    run_case(Case(M, N, 2560, blocksize=32, outliers=(N == 1003)), seed=11450 + M + ctas + N, device=cuda_device,
             check_quantizer=False, loader=7, **kw)


@pytest.mark.parametrize("M", [1, 4, 11])
@pytest.mark.parametrize("act,table", [("fp16", "normal"), ("bf16", "uniform"), ("fp16", "fp4"), ("bf16", "fp4")])
def test_rows_dtypes_tables(cuda_device, M, act, table):
    run_case(Case(M, 777, 2304, act=act, table=table), seed=11500 + M, device=cuda_device, check_quantizer=False,
             loader=7)


@pytest.mark.parametrize("M", [1, 8, 16])
def test_rows_outliers(cuda_device, M):
    run_case(Case(M, 1500, 1024, outliers=True), seed=11600 + M, device=cuda_device, check_quantizer=False,
             loader=7)


def _layer(device, N, K, seed, bs=64):
    code = inputs.code_normal_quantile()
    packed, absmax = oracle.quantize(inputs.weights(N, K, seed), bs, code)
    return (torch.from_numpy(packed).to(device), torch.from_numpy(absmax).to(device),
            torch.from_numpy(code).to(device), packed, absmax, code)


@pytest.mark.parametrize("M,N", [(1, 1000), (7, 3001), (16, 96)])
def test_rows_bias(cuda_device, M, N):
    K, bs = 1024, 64
    P, Am, C, packed, absmax, code = _layer(cuda_device, N, K, 11700 + N)
    A = inputs.activations(M, K, torch.bfloat16, 11701)
    bias = inputs.activations(1, N, torch.bfloat16, 11702).reshape(N)
    out = q4.q4_gemm_skinny(A.to(cuda_device), P, Am, C, N, K, bs, bias=bias.to(cuda_device), loader=7)
    torch.cuda.synchronize()
    y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, bs, bias_bits=bits_of(bias))
    check_gemm(bits_of(out), y, S, "bf16", "rows bias")


@pytest.mark.parametrize("N,K,ctas", [(300, 1024, 5), (64, 4096, 20), (2000, 2048, 148), (1000, 2560, 0)])
def test_rows_deterministic_and_error_word_zero(cuda_device, N, K, ctas):
    P, Am, C, packed, absmax, code = _layer(cuda_device, N, K, 11800 + N)
    A = inputs.activations(3, K, torch.bfloat16, 11801).to(cuda_device)
    ws = q4.Workspace(cuda_device)
    kw = {"ctas": ctas} if ctas else {}
    outs = [q4.q4_gemm_skinny(A, P, Am, C, N, K, 64, workspace=ws, loader=7, **kw) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    assert q4.workspace_error(ws) == 0
    y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, 3, N, K, 64)
    check_gemm(bits_of(outs[0]), y, S, "bf16", "rows determinism")


@pytest.mark.parametrize("pdl", [1, 2])
def test_rows_dependent_launch_chain(cuda_device, pdl):
    """Each GEMM reads the previous one's output: under programmatic dependent
    launch the next kernel streams its weights early but must read its
    activations only after the previous grid finished (bit-equal results)."""
    dims = [2048, 1536, 2560, 1024, 4096]
    layers = [_layer(cuda_device, dims[i + 1], dims[i], 11900 + i)[:3] for i in range(len(dims) - 1)]
    A0 = inputs.activations(2, dims[0], torch.bfloat16, 11901).to(cuda_device)

    def chain(**launch):
        x = A0
        for (P, Am, C), N, K in zip(layers, dims[1:], dims[:-1]):
            x = q4.q4_gemm_skinny(x, P, Am, C, N, K, 64, loader=7, **launch)
        return x

    ref = chain()
    torch.cuda.synchronize()
    for _ in range(3):
        got = chain(pdl=pdl, l2_prefetch=8 if pdl == 2 else 0)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_rows_agrees_with_stream_k_kernel(cuda_device):
    """The row-split and stream-K kernels sum in different orders; both stay
    within the tolerance of the oracle on the same inputs."""
    M, N, K = 4, 2900, 3072
    P, Am, C, packed, absmax, code = _layer(cuda_device, N, K, 12000)
    A = inputs.activations(M, K, torch.bfloat16, 12001)
    y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, 64)
    for loader in (2, 7):
        out = q4.q4_gemm_skinny(A.to(cuda_device), P, Am, C, N, K, 64, loader=loader)
        torch.cuda.synchronize()
        check_gemm(bits_of(out), y, S, "bf16", f"loader {loader}")


@pytest.mark.parametrize("skip", [0, 3, 7])
def test_rows_bounded_wait_runs_out(cuda_device, monkeypatch, skip):
    """A stage that is never loaded (test hook Q4_TEST_SKIP_STAGE, which also
    shortens the wait limits): the consumer's bounded wait on it runs out, the
    kernel sets error word 1 and returns without faulting; after
    Workspace.reset() the next call is correct again."""
    M, N, K = 2, 3000, 2048
    P, Am, C, packed, absmax, code = _layer(cuda_device, N, K, 12100)
    A = inputs.activations(M, K, torch.bfloat16, 12101).to(cuda_device)
    ws = q4.Workspace(cuda_device)
    monkeypatch.setenv("Q4_TEST_SKIP_STAGE", str(skip))
    q4.q4_gemm_skinny(A, P, Am, C, N, K, 64, workspace=ws, loader=7)
    torch.cuda.synchronize()
    assert q4.workspace_error(ws) == 1
    monkeypatch.delenv("Q4_TEST_SKIP_STAGE")
    ws.reset()
    out = q4.q4_gemm_skinny(A, P, Am, C, N, K, 64, workspace=ws, loader=7)
    torch.cuda.synchronize()
    assert q4.workspace_error(ws) == 0
    y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, 64)
    check_gemm(bits_of(out), y, S, "bf16", "after the time-out")


@pytest.mark.parametrize("M", [17, 24, 32])
@pytest.mark.parametrize("N,K,act", [(300, 1024, "bf16"), (1000, 2560, "fp16"), (77, 4096, "bf16"), (4100, 768, "bf16")])
def test_rows_four_column_tiles(cuda_device, M, N, K, act):
    """17 <= M <= 32 on the row-split kernel (four n8 column tiles, tiles of
    at most 32 rows, half a stage of activations in flight)."""
    run_case(Case(M, N, K, act=act), seed=12200 + M + N, device=cuda_device, check_quantizer=False, loader=7)


def test_rows_four_column_tiles_bias_and_partitions(cuda_device):
    M, N, K = 29, 1500, 2048
    P, Am, C, packed, absmax, code = _layer(cuda_device, N, K, 12300)
    A = inputs.activations(M, K, torch.bfloat16, 12301)
    bias = inputs.activations(1, N, torch.bfloat16, 12302).reshape(N)
    y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, 64, bias_bits=bits_of(bias))
    for ctas in (1, 7, 148):
        out = q4.q4_gemm_skinny(A.to(cuda_device), P, Am, C, N, K, 64, bias=bias.to(cuda_device), loader=7, ctas=ctas)
        torch.cuda.synchronize()
        check_gemm(bits_of(out), y, S, "bf16", f"rows M29 bias ctas {ctas}")
