"""GPU parity of the tensor-memory (tcgen05) kernel that serves 65 <= M <= 128
(and M <= 64 on request, math=3; the launch table sends 17 <= M <= 64 to the
mma.sync kernels, in row chunks of 32 above M = 32, where their TMA rules
hold): every output element within
1e-2 * sum_k |a w| + ulp(y) of the oracle.  The weights enter the MMA as
bf16_rn(code * absmax) (fp16 for fp16 activations), i.e. exactly the values
the standalone dequantizer writes; the fp32 accumulation follows.  The
operation is the fused path of bitsandbytes PR #1920 ("Fused path support
for M > 1") at larger M."""
import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs
from bit_weight_dequant_b200.inputs import Case
from parity import ORACLE_ACT, TORCH_ACT, bits_of, check_gemm, run_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M", [17, 24, 32, 33, 48, 64, 65, 96, 127, 128])
@pytest.mark.parametrize("N,K", [(128, 256), (300, 1024), (513, 2048), (1000, 512)])
def test_tcgen05_bf16(cuda_device, M, N, K):
    run_case(Case(M, N, K), seed=7000 + M * 3 + N + K, device=cuda_device, check_quantizer=False,
             **({"math": 3} if M <= 64 else {}))


@pytest.mark.parametrize("M", [20, 64, 128])
@pytest.mark.parametrize("act,table", [("fp16", "normal"), ("bf16", "uniform"), ("bf16", "fp4"), ("fp16", "fp4")])
def test_tcgen05_dtypes_tables(cuda_device, M, act, table):
    run_case(Case(M, 384, 1536, act=act, table=table), seed=7100 + M, device=cuda_device, check_quantizer=False,
             **({"math": 3} if M <= 64 else {}))


@pytest.mark.parametrize("M", [40, 128])
@pytest.mark.parametrize("bs", [128, 256, 1024])
def test_tcgen05_blocksizes(cuda_device, M, bs):
    run_case(Case(M, 256, 4096, blocksize=bs), seed=7200 + bs + M, device=cuda_device, check_quantizer=False,
             **({"math": 3} if M <= 64 else {}))


@pytest.mark.parametrize("ctas", [1, 2, 3, 7, 33, 148])
@pytest.mark.parametrize("M", [18, 100])
def test_tcgen05_partitions(cuda_device, ctas, M):
    """Tiles cut between CTAs (workspace fix-up) at every CTA count."""
    run_case(Case(M, 640, 2048), seed=7300 + ctas, device=cuda_device, check_quantizer=False, ctas=ctas,
             **({"math": 3} if M <= 64 else {}))


@pytest.mark.parametrize("M", [1, 5, 16])
def test_tcgen05_small_m_on_request(cuda_device, M):
    run_case(Case(M, 512, 1024), seed=7400 + M, device=cuda_device, check_quantizer=False, math=3)


def test_tcgen05_outliers(cuda_device):
    run_case(Case(64, 256, 2048, outliers=True), seed=7500, device=cuda_device, check_quantizer=False, math=3)


@pytest.mark.parametrize("ctas", [5, 37])
def test_tcgen05_deterministic_and_counters_left_zero(cuda_device, ctas):
    M, N, K = 48, 700, 2048
    code = inputs.code_normal_quantile()
    W = inputs.weights(N, K, 9)
    packed, absmax = oracle.quantize(W, 64, code)
    A = inputs.activations(M, K, torch.bfloat16, 9).to(cuda_device)
    P, Am, C = (torch.from_numpy(x).to(cuda_device) for x in (packed, absmax, code))
    ws = q4.Workspace(cuda_device)
    outs = [q4.q4_gemm_skinny(A, P, Am, C, N, K, 64, workspace=ws, ctas=ctas, math=3) for _ in range(3)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    assert q4.workspace_error(ws) == 0
    off = q4.workspace_counter_offset(cuda_device)
    assert int(ws.buf[off:].count_nonzero()) == 0, "counters and partial slots must return to zero"
    y, S = oracle.gemm(bits_of(A.cpu()), oracle.BF16, packed, absmax, code, M, N, K, 64)
    check_gemm(bits_of(outs[0].cpu()), y, S, "bf16", "tcgen05 determinism")


@pytest.mark.parametrize("act", ["bf16", "fp16"])
@pytest.mark.parametrize("launch", [{"math": 3}, {"ctas": 9, "math": 3}])
def test_tcgen05_bias(cuda_device, act, launch):
    M, N, K = 50, 300, 1024
    code = inputs.code_normal_quantile()
    W = inputs.weights(N, K, 21)
    packed, absmax = oracle.quantize(W, 64, code)
    A = inputs.activations(M, K, TORCH_ACT[act], 21)
    bias = inputs.activations(1, N, TORCH_ACT[act], 22).reshape(N)
    y, S = oracle.gemm(bits_of(A), ORACLE_ACT[act], packed, absmax, code, M, N, K, 64, bias_bits=bits_of(bias))
    dev = cuda_device
    out = q4.q4_gemm_skinny(A.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(absmax).to(dev),
                            torch.from_numpy(code).to(dev), N, K, 64, bias=bias.to(dev), **launch)
    check_gemm(bits_of(out), y, S, act, f"tcgen05 bias {act} {launch}")


def test_tcgen05_requirements(cuda_device):
    """M > 16 outside the kernel's layout rules is reported, not run."""
    dev = cuda_device
    A = torch.zeros((32, 4160), dtype=torch.bfloat16, device=dev)
    P = torch.zeros(64 * 4160 // 2, dtype=torch.uint8, device=dev)
    Am = torch.zeros(64 * 4160 // 64, dtype=torch.float32, device=dev)
    C = torch.from_numpy(inputs.code_normal_quantile()).to(dev)
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_gemm_skinny(A, P, Am, C, 64, 4160, 64)        # K % 256 != 0
    assert e.value.status == q4.Q4_ERR_UNSUPPORTED
    A2 = torch.zeros((129, 256), dtype=torch.bfloat16, device=dev)
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_gemm_skinny(A2, P[:64 * 128], Am[:256], C, 64, 256, 64)
    assert e.value.status == q4.Q4_ERR_UNSUPPORTED


def test_tcgen05_then_small_m_share_a_workspace(cuda_device):
    """A tensor-memory call leaves nothing behind that a later call of another
    shape (whose counters may lie where the first call's slots were) could
    misread."""
    ws = q4.Workspace(cuda_device)
    for M, N, K in [(48, 300, 1024), (1, 10240, 1024), (64, 1000, 2048), (3, 20000, 512)]:
        code = inputs.code_normal_quantile()
        W = inputs.weights(N, K, N + M)
        packed, absmax = oracle.quantize(W, 64, code)
        A = inputs.activations(M, K, torch.bfloat16, N)
        y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, 64)
        out = q4.q4_gemm_skinny(A.to(cuda_device), torch.from_numpy(packed).to(cuda_device),
                                torch.from_numpy(absmax).to(cuda_device), torch.from_numpy(code).to(cuda_device),
                                N, K, 64, workspace=ws, ctas=17, **({"math": 3} if M > 16 else {}))
        check_gemm(bits_of(out.cpu()), y, S, "bf16", f"shared workspace M{M} N{N}")


@pytest.mark.parametrize("M", [16, 64])
def test_equal_codes_under_one_absmax(cuda_device, M):
    """Rows whose blocks hold one +1 code and 4095 copies of code 1/15 of the
    uniform table, all-positive activations: the weights' rounding errors
    share their sign, so the output error is the per-weight error itself.
    The fused kernels round each weight once (at most 2^-8 for bf16) and stay
    inside 1e-2 * S; a weight rounded three times (code and absmax each
    rounded to bf16, then their product) is 1.01 % off at these absmax
    values and would not.  M = 16 runs the mma.sync kernel, M = 64 the
    tcgen05 kernel."""
    dev = cuda_device
    code = inputs.code_uniform()
    base = np.float32(0.03308130428195)
    am = np.array([base * np.float32(2.0 ** k) * np.float32(f) for k in range(-3, 5) for f in (1.0, 1.0001)],
                  dtype=np.float32)
    K, bs = 16384, 4096
    W = inputs.weights_equal_codes(am, K, bs, float(code[8]))
    N = W.shape[0]
    packed, absmax = oracle.quantize(W, bs, code)
    codes = np.stack([packed >> 4, packed & 15], -1).reshape(N, K)
    assert np.array_equal(absmax, np.repeat(am, K // bs)) and (codes[:, ::bs] == 15).all()
    assert (np.delete(codes, np.s_[::bs], axis=1) == 8).all()
    A = torch.ones((M, K), dtype=torch.bfloat16)
    y, S = oracle.gemm(bits_of(A), ORACLE_ACT["bf16"], packed, absmax, code, M, N, K, bs)
    out = q4.q4_gemm_skinny(A.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(absmax).to(dev),
                            torch.from_numpy(code).to(dev), N, K, bs, **({"math": 3} if M > 16 else {}))
    torch.cuda.synchronize(dev)
    check_gemm(bits_of(out), y, S, "bf16", f"equal codes M{M}")
