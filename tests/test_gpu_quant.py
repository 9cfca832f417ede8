"""GPU parity of blockwise quantize / dequantize against the oracle: codes,
absmax and dequantized values must be bit-identical (the operation is the
quantize/dequantize half of bitsandbytes PR #1920's fused 4-bit path)."""
import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs

pytestmark = pytest.mark.gpu

SIZES = [(1, 32), (2, 64), (31, 64), (64, 64), (4097, 64), (777, 32), (100003, 128), (3 * 65536 + 5, 256),
         (12345, 4096), ((1 << 20) + 1, 64)]


def _weights(n, bs, seed, outliers):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal(n) * 0.02).astype(np.float32)
    if outliers:
        w[rng.random(n) < 0.01] *= 20
    if n >= 3 * bs:
        w[bs:2 * bs] = 0.0                                   # an all-zero block
    return w


@pytest.mark.parametrize("table", ["normal", "uniform", "fp4"])
@pytest.mark.parametrize("n,bs", SIZES)
@pytest.mark.parametrize("outliers", [False, True])
def test_quantize_bit_exact(cuda_device, table, n, bs, outliers):
    code = inputs.CODE_TABLES[table]()
    w = _weights(n, bs, n * 31 + bs, outliers)
    p_ref, a_ref = oracle.quantize(w, bs, code)
    p, a = q4.q4_quantize_blockwise(torch.from_numpy(w).to(cuda_device), bs, torch.from_numpy(code).to(cuda_device))
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))


def test_quantize_exact_code_points_and_ties(cuda_device):
    """Values exactly on codes and exactly between two codes (ties -> lower index)."""
    code = inputs.code_uniform()
    mids = ((code[:-1].astype(np.float64) + code[1:]) / 2).astype(np.float32)
    w = np.concatenate([code, mids, -mids, np.zeros(2, np.float32)]).astype(np.float32)   # 48 values
    w = np.concatenate([w[:32], np.zeros(32, np.float32), w[32:], np.zeros(48, np.float32)])
    assert w.size == 128
    w[63] = 1.0   # each 64-block has absmax 1 -> x = w
    w[127] = 1.0
    p_ref, a_ref = oracle.quantize(w, 64, code)
    p, a = q4.q4_quantize_blockwise(torch.from_numpy(w).to(cuda_device), 64, torch.from_numpy(code).to(cuda_device))
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(a.cpu().numpy(), a_ref)


@pytest.mark.parametrize("out", ["bf16", "fp16", "fp32"])
@pytest.mark.parametrize("n,bs", SIZES)
def test_dequantize_bit_exact(cuda_device, out, n, bs):
    dt = {"bf16": oracle.BF16, "fp16": oracle.FP16, "fp32": oracle.FP32}[out]
    tdt = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[out]
    code = inputs.code_normal_quantile()
    rng = np.random.default_rng(n + bs)
    packed = rng.integers(0, 256, (n + 1) // 2, dtype=np.uint8)
    nb = (n + bs - 1) // bs
    absmax = np.exp2(rng.uniform(-30, 18, nb)).astype(np.float32)   # subnormal fp16 .. fp16 overflow
    absmax[::7] = 0.0
    ref = oracle.dequantize(packed, absmax, code, n, bs, dt)
    got = q4.q4_dequantize_blockwise(torch.from_numpy(packed).to(cuda_device), torch.from_numpy(absmax).to(cuda_device),
                                     torch.from_numpy(code).to(cuda_device), n, bs, tdt)
    g = got.cpu()
    g = g.view(torch.int32).numpy().view(np.uint32) if out == "fp32" else g.view(torch.int16).numpy().view(np.uint16)
    r = ref.view(np.uint32) if out == "fp32" else ref
    assert np.array_equal(g, r)


def test_roundtrip_quantize_dequantize(cuda_device):
    code = inputs.code_normal_quantile()
    w = _weights(4096 * 64 + 10, 64, 7, True)
    wd = torch.from_numpy(w).to(cuda_device)
    cd = torch.from_numpy(code).to(cuda_device)
    p, a = q4.q4_quantize_blockwise(wd, 64, cd)
    got = q4.q4_dequantize_blockwise(p, a, cd, w.size, 64, torch.bfloat16)
    p_ref, a_ref = oracle.quantize(w, 64, code)
    ref = oracle.dequantize(p_ref, a_ref, code, w.size, 64, oracle.BF16)
    assert np.array_equal(got.cpu().view(torch.int16).numpy().view(np.uint16), ref)


def test_empty_input_is_noop(cuda_device):
    cd = torch.from_numpy(inputs.code_normal_quantile()).to(cuda_device)
    p, a = q4.q4_quantize_blockwise(torch.zeros(0, device=cuda_device), 64, cd)
    assert p.numel() == 0 and a.numel() == 0
    out = q4.q4_dequantize_blockwise(p, a, cd, 0, 64, torch.bfloat16)
    assert out.numel() == 0


def test_misaligned_pointer_rejected(cuda_device):
    cd = torch.from_numpy(inputs.code_normal_quantile()).to(cuda_device)
    w = torch.zeros(1025, device=cuda_device)[1:]
    with pytest.raises(q4.Q4Error) as e:
        q4.q4_quantize_blockwise(w, 64, cd)
    assert e.value.status == q4.Q4_ERR_MISALIGNED


@pytest.mark.parametrize("wdt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("n,bs", [(4097, 64), (100003, 128), (65536 * 3 + 5, 512), (12345, 4096), (1 << 20, 32)])
def test_quantize_16bit_weights_bit_exact(cuda_device, wdt, n, bs):
    """bf16 / fp16 weights: the result equals the oracle on the exactly widened fp32 values."""
    code = inputs.code_normal_quantile()
    w16 = torch.from_numpy(_weights(n, bs, n + bs, True)).to(wdt)
    p_ref, a_ref = oracle.quantize(w16.float().numpy(), bs, code)
    p, a = q4.q4_quantize_blockwise(w16.to(cuda_device), bs, torch.from_numpy(code).to(cuda_device))
    assert np.array_equal(p.cpu().numpy(), p_ref)
    assert np.array_equal(a.cpu().numpy().view(np.uint32), a_ref.view(np.uint32))


@pytest.mark.parametrize("bs", [64, 256])
def test_quantize_unaligned_packed_output(cuda_device, bs):
    """A packed array that is not 8-byte aligned takes the per-warp form; same bytes."""
    n = 3 * 4096 + 96
    code = inputs.code_uniform()
    w = _weights(n, bs, 5, False)
    p_ref, a_ref = oracle.quantize(w, bs, code)
    raw = torch.zeros((n + 1) // 2 + 16, dtype=torch.uint8, device=cuda_device)
    packed = raw[3:3 + (n + 1) // 2]
    absmax = torch.zeros((n + bs - 1) // bs, dtype=torch.float32, device=cuda_device)
    wd, cd = torch.from_numpy(w).to(cuda_device), torch.from_numpy(code).to(cuda_device)
    rc = q4.lib().q4_quantize_blockwise(wd.data_ptr(), n, bs, cd.data_ptr(), packed.data_ptr(), absmax.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)
    assert rc == q4.Q4_OK
    assert np.array_equal(packed.cpu().numpy(), p_ref)
    assert np.array_equal(absmax.cpu().numpy(), a_ref)
    assert int(raw[:3].count_nonzero()) == 0 and int(raw[3 + (n + 1) // 2:].count_nonzero()) == 0
