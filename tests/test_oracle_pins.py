"""Pins for the CPU oracle, independent of the oracle itself.

Each test checks the oracle against something the method or the
mathematics fixes: hand-worked examples (tests/golden), brute force with a
different implementation (numpy, vectorised), closed forms, invariants of
blockwise absmax quantization, and library conversions (numpy binary16,
torch bfloat16) for the IEEE roundings.  The method is the fused blockwise
4-bit dequantize + matmul of bitsandbytes PR #1920 ("[ROCm] Optimize
kgemm_4bit_inference_naive ...", "Technical details", "Fused path support
for M > 1").
"""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import inputs
from conftest import read_golden

TABLES = {"uniform": inputs.code_uniform(), "normal": inputs.code_normal_quantile(), "fp4": inputs.code_fp4_e2m1()}


# ---------------------------------------------------------------------------
# independent helpers (numpy / torch), NOT the oracle's code
# ---------------------------------------------------------------------------

def np_unpack(packed: np.ndarray, n: int) -> np.ndarray:
    hi = (packed >> 4) & 0xF
    lo = packed & 0xF
    idx = np.empty(2 * packed.size, dtype=np.int64)
    idx[0::2] = hi
    idx[1::2] = lo
    return idx[:n]


def np_weights(packed, absmax, code, n, bs) -> np.ndarray:
    idx = np_unpack(packed, n)
    blk = np.arange(n) // bs
    return (code[idx].astype(np.float32) * absmax[blk].astype(np.float32)).astype(np.float32)


def torch_bf16_bits(x32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def torch_bf16_values(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def np_fp16_bits(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):       # overflow to +-inf is part of what is checked
        return np.asarray(x).astype(np.float16).view(np.uint16)


# ---------------------------------------------------------------------------
# hand-worked examples
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fixture", ["hand_uniform_bs4.txt", "hand_normal_bs8.txt"])
def test_hand_worked_examples(fixture):
    g = read_golden(fixture)
    code = TABLES[g["table"][0]]
    bs = int(g["blocksize"][0])
    w = np.array([float(v) for v in g["w"]], dtype=np.float32)
    packed, absmax = oracle.quantize(w, bs, code)
    assert [int(v, 16) for v in g["packed"]] == packed.tolist()
    assert list(np_unpack(packed, w.size)) == [int(v) for v in g["idx"]]
    assert absmax.tolist() == [np.float32(float(v)) for v in g["absmax"]]
    if "dequant_bf16" in g:
        deq = oracle.dequantize(packed, absmax, code, w.size, bs, oracle.BF16)
        assert deq.tolist() == [int(v, 16) for v in g["dequant_bf16"]]
    a = np.array([int(v, 16) for v in g["a_bf16"]], dtype=np.uint16)
    y, S = oracle.gemm(a, oracle.BF16, packed, absmax, code, 1, 1, w.size, bs)
    yv, ytol = float(g["y"][0]), float(g["y"][1])
    assert abs(y[0, 0] - yv) <= ytol
    if "S" in g:
        assert abs(S[0, 0] - float(g["S"][0])) <= float(g["S"][1])


# ---------------------------------------------------------------------------
# code tables (inputs, checked against closed forms / scipy)
# ---------------------------------------------------------------------------

def test_uniform_table_closed_form():
    c = inputs.code_uniform()
    from fractions import Fraction
    for i in range(16):
        assert c[i] == np.float32(float(Fraction(2 * i - 15, 15)))
    assert c[0] == -1 and c[15] == 1 and 0 not in c


def test_normal_table_against_scipy():
    from scipy.stats import norm
    c = inputs.code_normal_quantile()
    eps = 1 / 32
    top = norm.ppf(1 - eps)
    pos = [norm.ppf(0.5 + j * (0.5 - eps) / 8) / top for j in range(1, 9)]
    neg = [-norm.ppf(0.5 + j * (0.5 - eps) / 7) / top for j in range(1, 8)]
    ref = np.array(sorted(neg + [0.0] + pos), dtype=np.float32)
    np.testing.assert_allclose(c, ref, rtol=0, atol=2e-7)
    assert c[0] == -1 and c[15] == 1 and c[7] == 0
    assert np.all(np.diff(c) > 0)
    assert (c > 0).sum() == 8 and (c < 0).sum() == 7


def test_fp4_table_is_the_e2m1_format():
    """Rebuild the table from binary16 bit patterns (a different route: the
    E2M1 fields moved into an IEEE half and decoded by numpy)."""
    c = inputs.code_fp4_e2m1()
    for i in range(16):
        s, e, m = i >> 3, (i >> 1) & 3, i & 1
        if e == 0 and m == 0:
            bits = s << 15                                   # +-0
        elif e == 0:
            bits = (s << 15) | ((15 - 1) << 10)              # subnormal 0.5 = 2^-1
        else:
            bits = (s << 15) | ((e - 1 + 15) << 10) | (m << 9)
        half = np.array([bits], dtype=np.uint16).view(np.float16)[0]
        want = np.float32(np.float64(half) / 6.0)
        assert c[i] == want and np.signbit(c[i]) == bool(s), i
    assert sorted(set(np.round(np.abs(c).astype(np.float64) * 6, 6))) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert c[7] == 1 and c[15] == -1


# ---------------------------------------------------------------------------
# quantize: brute force and invariants
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("table", ["uniform", "normal", "fp4"])
@pytest.mark.parametrize("n,bs", [(1, 32), (31, 32), (64, 64), (1001, 64), (777, 128), (2049, 256),
                                  (300, 4096)])
def test_quantize_brute_force(table, n, bs):
    code = TABLES[table]
    rng = np.random.default_rng(n * 7 + bs)
    w = (rng.standard_normal(n) * 0.02).astype(np.float32)
    packed, absmax = oracle.quantize(w, bs, code)
    nb = (n + bs - 1) // bs
    assert packed.size == (n + 1) // 2 and absmax.size == nb
    # absmax is the exact block maximum of |w|
    for b in range(nb):
        assert absmax[b] == np.max(np.abs(w[b * bs:(b + 1) * bs]))
    idx = np_unpack(packed, n)
    if n % 2:
        assert packed[-1] & 0xF == 0, "odd n pads the final low nibble with 0"
    x = (w / absmax[np.arange(n) // bs]).astype(np.float32)
    d = np.abs(x[:, None] - code[None, :]).astype(np.float32)   # [n, 16] fp32 distances
    dmin = d.min(axis=1)
    assert np.all(d[np.arange(n), idx] == dmin), "a strictly nearer code exists"
    first = np.argmax(d == dmin[:, None], axis=1)
    assert np.all(idx == first), "ties must go to the lowest index"


@pytest.mark.parametrize("table", ["uniform", "normal", "fp4"])
def test_quantize_error_bound_and_extremes(table):
    code = TABLES[table]
    bs = 64
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(64 * 50) * 0.02).astype(np.float32)
    w[64 * 3:64 * 4] = 0.0                       # an all-zero block
    w[64 * 7 + 5] *= 20                          # an outlier
    packed, absmax = oracle.quantize(w, bs, code)
    wq = np_weights(packed, absmax, code, w.size, bs).astype(np.float64)
    gap = float(np.max(np.diff(np.sort(code.astype(np.float64)))))   # largest gap between adjacent levels
    am = absmax[np.arange(w.size) // bs].astype(np.float64)
    err = np.abs(wq - w.astype(np.float64))
    assert np.all(err <= am * gap / 2 * (1 + 1e-6) + 1e-30)
    assert absmax[3] == 0 and np.all(wq[64 * 3:64 * 4] == 0)
    for b in range(50):                           # the absmax element maps to +-1 exactly
        blk = w[b * bs:(b + 1) * bs]
        if absmax[b] == 0:
            continue
        j = int(np.argmax(np.abs(blk)))
        i = np_unpack(packed, w.size)[b * bs + j]
        assert code[i] == (1.0 if blk[j] > 0 else -1.0)


def test_quantize_power_of_two_scaling():
    code = TABLES["normal"]
    rng = np.random.default_rng(9)
    w = (rng.standard_normal(4096) * 0.02).astype(np.float32)
    p0, a0 = oracle.quantize(w, 64, code)
    for k in (-3, 5):
        p1, a1 = oracle.quantize((w * np.float32(2.0 ** k)).astype(np.float32), 64, code)
        assert np.array_equal(p0, p1)
        assert np.array_equal(a1, (a0 * np.float32(2.0 ** k)).astype(np.float32))


def test_quantize_exact_code_points():
    code = TABLES["normal"]
    absmax = np.float32(0.75)
    order = np.array([15, 0, 3, 9, 7, 12, 1, 14, 2, 10, 5, 13, 4, 11, 6, 8])
    w = (code[order] * absmax).astype(np.float32)
    packed, am = oracle.quantize(w, 16, code)
    assert am[0] == absmax
    assert list(np_unpack(packed, 16)) == list(order)


def test_quantize_rejects_nonfinite():
    w = np.array([0.1, np.nan, 0.2, 0.3], dtype=np.float32)
    with pytest.raises(ValueError):
        oracle.quantize(w, 4, TABLES["normal"])


# ---------------------------------------------------------------------------
# dequantize vs library conversions
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("table", ["uniform", "normal", "fp4"])
@pytest.mark.parametrize("bs", [32, 64, 256])
def test_dequantize_matches_library_rounding(table, bs):
    code = TABLES[table]
    rng = np.random.default_rng(bs)
    n = 3 * bs + 17
    packed = rng.integers(0, 256, (n + 1) // 2, dtype=np.uint8)
    # absmax spanning fp16 subnormals, normals and fp16 overflow
    absmax = np.exp2(rng.uniform(-30, 20, (n + bs - 1) // bs)).astype(np.float32)
    absmax[0] = 0.0
    wv = np_weights(packed, absmax, code, n, bs)
    d32 = oracle.dequantize(packed, absmax, code, n, bs, oracle.FP32)
    assert np.array_equal(d32.view(np.uint32), wv.view(np.uint32))
    assert np.array_equal(oracle.dequantize(packed, absmax, code, n, bs, oracle.BF16), torch_bf16_bits(wv))
    assert np.array_equal(oracle.dequantize(packed, absmax, code, n, bs, oracle.FP16), np_fp16_bits(wv))


def test_dequantize_negative_zero_kept():
    code = TABLES["normal"]
    packed = np.array([0x0F], dtype=np.uint8)      # idx 0 (-1) and 15 (+1)
    absmax = np.array([0.0], dtype=np.float32)
    out = oracle.dequantize(packed, absmax, code, 2, 64, oracle.BF16)
    assert out.tolist() == [0x8000, 0x0000]


# ---------------------------------------------------------------------------
# roundings and ulp
# ---------------------------------------------------------------------------

def test_round_fp16_vs_numpy():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(20000) * np.exp2(rng.uniform(-28, 17, 20000)),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 2.0 ** -24, 2.0 ** -25,
                  3 * 2.0 ** -26, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 1e-9]),
    ])
    assert np.array_equal(oracle.round_to(x, oracle.FP16), np_fp16_bits(x))


def test_round_bf16_vs_torch_and_ties():
    rng = np.random.default_rng(12)
    x32 = (rng.standard_normal(20000) * np.exp2(rng.uniform(-130, 120, 20000))).astype(np.float32)
    x32 = np.concatenate([x32, np.array([0.0, 1e-45, 3e38, -3.4e38], dtype=np.float32)])
    # binary32 inputs: torch's float->bfloat16 is one RNE rounding
    assert np.array_equal(oracle.round_to(x32.astype(np.float64), oracle.BF16), torch_bf16_bits(x32))
    # binary64 inputs that are not binary32: exact ties and just-above-tie values, by hand
    cases = {1 + 2.0 ** -8: 0x3F80,                # tie -> even (1.0)
             1 + 2.0 ** -8 + 2.0 ** -40: 0x3F81,   # just above the tie -> up
             1 + 3 * 2.0 ** -8: 0x3F82,            # tie between 0x3F81 and 0x3F82 -> even
             -(2 - 2.0 ** -8): -0.0}               # rounds up to -2.0
    got = oracle.round_to(np.array(list(cases)), oracle.BF16)
    assert got[:3].tolist() == [0x3F80, 0x3F81, 0x3F82]
    assert got[3] == 0xC000


def test_decode_roundtrip():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    fin = (bits & 0x7C00) != 0x7C00
    v16 = oracle.decode(bits, oracle.FP16)
    assert np.array_equal(v16[fin], bits[fin].view(np.float16).astype(np.float64))
    finb = (bits & 0x7F80) != 0x7F80
    vb = oracle.decode(bits, oracle.BF16)
    assert np.array_equal(vb[finb], torch_bf16_values(bits)[finb])


def test_ulp_closed_forms():
    y = np.array([1.0, 1.5, 2.0, -3.0, 0.0, 2.0 ** -130, 65504.0, 2.0 ** -20])
    ub = oracle.ulp(y, oracle.BF16)
    assert ub.tolist() == [2.0 ** -7, 2.0 ** -7, 2.0 ** -6, 2.0 ** -6, 2.0 ** -133, 2.0 ** -133,
                           2.0 ** 8, 2.0 ** -27]
    uh = oracle.ulp(y, oracle.FP16)
    assert uh.tolist() == [2.0 ** -10, 2.0 ** -10, 2.0 ** -9, 2.0 ** -9, 2.0 ** -24, 2.0 ** -24,
                           32.0, 2.0 ** -24]


# ---------------------------------------------------------------------------
# GEMM: brute force, special cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("act", [oracle.BF16, oracle.FP16])
@pytest.mark.parametrize("M,N,K,bs", [(1, 1, 64, 64), (3, 7, 64, 32), (4, 9, 128, 64), (2, 5, 96, 32),
                                      (5, 3, 40, 16)])
def test_gemm_brute_force(act, M, N, K, bs):
    code = TABLES["normal"]
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    w = (rng.standard_normal(N * K) * 0.02).astype(np.float32)
    packed, absmax = oracle.quantize(w, bs, code)
    a32 = rng.standard_normal((M, K)).astype(np.float32)
    if act == oracle.BF16:
        abits = torch_bf16_bits(a32).reshape(M, K)
        a64 = torch_bf16_values(abits.reshape(-1)).reshape(M, K)
    else:
        abits = np_fp16_bits(a32).reshape(M, K)
        a64 = abits.view(np.float16).astype(np.float64)
    W64 = np_weights(packed, absmax, code, N * K, bs).astype(np.float64).reshape(N, K)
    y, S = oracle.gemm(abits, act, packed, absmax, code, M, N, K, bs)
    yref = a64 @ W64.T
    Sref = np.abs(a64) @ np.abs(W64).T
    assert y.shape == (M, N)
    np.testing.assert_allclose(y, yref, rtol=0, atol=1e-12 * (Sref.max() + 1))
    np.testing.assert_allclose(S, Sref, rtol=1e-12)


@pytest.mark.parametrize("act", [oracle.BF16, oracle.FP16])
def test_gemm_bias_against_numpy_and_zero_weights(act):
    """The bias epilogue: numpy fp64 matmul plus the decoded bias; with every
    absmax 0 the layer is the bias itself, exactly."""
    code = TABLES["normal"]
    M, N, K, bs = 3, 40, 128, 64
    rng = np.random.default_rng(77)
    w = (rng.standard_normal(N * K) * 0.02).astype(np.float32)
    packed, absmax = oracle.quantize(w, bs, code)
    a32 = rng.standard_normal((M, K)).astype(np.float32)
    b32 = rng.standard_normal(N).astype(np.float32)
    if act == oracle.BF16:
        abits, bbits = torch_bf16_bits(a32).reshape(M, K), torch_bf16_bits(b32)
        a64, b64 = torch_bf16_values(abits.reshape(-1)).reshape(M, K), torch_bf16_values(bbits)
    else:
        abits, bbits = np_fp16_bits(a32).reshape(M, K), np_fp16_bits(b32)
        a64, b64 = abits.view(np.float16).astype(np.float64), bbits.view(np.float16).astype(np.float64)
    W64 = np_weights(packed, absmax, code, N * K, bs).astype(np.float64).reshape(N, K)
    y, S = oracle.gemm(abits, act, packed, absmax, code, M, N, K, bs, bias_bits=bbits)
    np.testing.assert_allclose(y, a64 @ W64.T + b64[None, :], rtol=0, atol=1e-12 * (S.max() + 1))
    np.testing.assert_allclose(S, np.abs(a64) @ np.abs(W64).T, rtol=1e-12)
    y0, S0 = oracle.gemm(abits, act, packed, np.zeros_like(absmax), code, M, N, K, bs, bias_bits=bbits)
    assert np.array_equal(y0, np.broadcast_to(b64, (M, N))) and np.all(S0 == 0)


def test_gemm_all_codes_one_closed_form():
    code = TABLES["uniform"]
    M, N, K, bs = 2, 3, 128, 64
    packed = np.full(N * K // 2, 0xFF, dtype=np.uint8)       # every idx -> code[15] = 1
    absmax = np.array([0.5, 0.25, 2.0, 4.0, 0.125, 1.0], dtype=np.float32)
    abits = np.full((M, K), 0x3F80, dtype=np.uint16)           # a = 1
    abits[1, :] = 0x4000                                       # a = 2
    y, _ = oracle.gemm(abits, oracle.BF16, packed, absmax, code, M, N, K, bs)
    for m, a in enumerate((1.0, 2.0)):
        for n in range(N):
            assert y[m, n] == a * 64 * (absmax[2 * n] + absmax[2 * n + 1])


def test_gemm_one_hot_selects_a_weight():
    code = TABLES["normal"]
    N, K, bs = 6, 128, 64
    rng = np.random.default_rng(3)
    w = (rng.standard_normal(N * K) * 0.02).astype(np.float32)
    packed, absmax = oracle.quantize(w, bs, code)
    wq = np_weights(packed, absmax, code, N * K, bs).reshape(N, K)
    for k in (0, 63, 64, 127):
        abits = np.zeros((1, K), dtype=np.uint16)
        abits[0, k] = 0x3F80
        y, _ = oracle.gemm(abits, oracle.BF16, packed, absmax, code, 1, N, K, bs)
        assert np.array_equal(y[0], wq[:, k].astype(np.float64))


def test_gemm_zero_block_and_empty():
    code = TABLES["normal"]
    packed = np.zeros(64, dtype=np.uint8)
    absmax = np.zeros(2, dtype=np.float32)
    abits = np.full((1, 64), 0x3F80, dtype=np.uint16)
    y, S = oracle.gemm(abits, oracle.BF16, packed, absmax, code, 1, 2, 64, 64)
    assert np.all(y == 0) and np.all(S == 0)
    y0 = oracle.gemm(np.zeros(0, np.uint16), oracle.BF16, packed, absmax, code, 1, 2, 0, 64, want_s=False)
    assert np.all(y0 == 0)


def test_tolerance_formula():
    y = np.array([1.0, -3.0, 0.0])
    S = np.array([10.0, 3.0, 0.0])
    tol = oracle.gemm_tolerance(y, S, oracle.BF16)
    assert tol.tolist() == [0.1 + 2.0 ** -7, 0.03 + 2.0 ** -6, 2.0 ** -133]


# ---------------------------------------------------------------------------
# fp32 activations (the reply's SIMT kernel: fp32, fp16 and bf16 inputs)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K,bs", [(1, 1, 64, 64), (3, 7, 64, 32), (4, 9, 128, 64), (2, 5, 96, 32),
                                      (5, 3, 40, 8)])
def test_gemm_f32_brute_force(M, N, K, bs):
    """Full-mantissa fp32 activations: numpy fp64 matmul over the explicitly
    dequantized weights."""
    code = TABLES["normal"]
    rng = np.random.default_rng(9000 + M * 100 + N * 10 + K)
    w = (rng.standard_normal(N * K) * 0.02).astype(np.float32)
    packed, absmax = oracle.quantize(w, bs, code)
    a32 = rng.standard_normal((M, K)).astype(np.float32)
    a64 = a32.astype(np.float64)
    W64 = np_weights(packed, absmax, code, N * K, bs).astype(np.float64).reshape(N, K)
    y, S = oracle.gemm_f32(a32, packed, absmax, code, M, N, K, bs)
    np.testing.assert_allclose(y, a64 @ W64.T, rtol=0, atol=1e-12 * ((np.abs(a64) @ np.abs(W64).T).max() + 1))
    np.testing.assert_allclose(S, np.abs(a64) @ np.abs(W64).T, rtol=1e-12)


def test_gemm_f32_agrees_with_bf16_path_on_bf16_values():
    """Activations that bf16 holds exactly give the same fp64 sums through
    the fp32 entry as through the (separately pinned) bf16 entry."""
    code = TABLES["fp4"]
    M, N, K, bs = 3, 11, 256, 64
    rng = np.random.default_rng(31)
    w = (rng.standard_normal(N * K) * 0.02).astype(np.float32)
    packed, absmax = oracle.quantize(w, bs, code)
    abits = torch_bf16_bits(rng.standard_normal((M, K)).astype(np.float32)).reshape(M, K)
    a32 = torch_bf16_values(abits.reshape(-1)).astype(np.float32).reshape(M, K)
    y16, S16 = oracle.gemm(abits, oracle.BF16, packed, absmax, code, M, N, K, bs)
    y32, S32 = oracle.gemm_f32(a32, packed, absmax, code, M, N, K, bs)
    assert np.array_equal(y16, y32) and np.array_equal(S16, S32)


def test_gemm_f32_one_hot_and_bias():
    """One-hot rows select a dequantized weight exactly; the fp32 bias is
    added once, exactly, and with every absmax 0 the layer is the bias."""
    code = TABLES["normal"]
    N, K, bs = 6, 128, 32
    rng = np.random.default_rng(5)
    w = (rng.standard_normal(N * K) * 0.02).astype(np.float32)
    packed, absmax = oracle.quantize(w, bs, code)
    wq = np_weights(packed, absmax, code, N * K, bs).reshape(N, K)
    a = np.zeros((4, K), dtype=np.float32)
    ks = (0, 31, 32, 127)
    for m, k in enumerate(ks):
        a[m, k] = 1.0
    y, _ = oracle.gemm_f32(a, packed, absmax, code, 4, N, K, bs)
    for m, k in enumerate(ks):
        assert np.array_equal(y[m], wq[:, k].astype(np.float64))
    b = rng.standard_normal(N).astype(np.float32)
    yb, _ = oracle.gemm_f32(a, packed, absmax, code, 4, N, K, bs, bias=b)
    assert np.array_equal(yb, y + b.astype(np.float64)[None, :])
    y0, S0 = oracle.gemm_f32(a, packed, np.zeros_like(absmax), code, 4, N, K, bs, bias=b)
    assert np.array_equal(y0, np.broadcast_to(b.astype(np.float64), (4, N))) and np.all(S0 == 0)


def test_ulp_fp32_against_numpy_spacing():
    """The fp32 spacing is numpy's own ``spacing`` of the binary32 value
    (normal, subnormal and zero)."""
    rng = np.random.default_rng(2)
    y = np.concatenate([rng.standard_normal(200) * 10.0 ** rng.integers(-30, 30, 200),
                        [0.0, 1.0, -1.0, 2.0 ** -126, 2.0 ** -140, 3.0e38]]).astype(np.float32)
    want = np.abs(np.spacing(np.abs(y))).astype(np.float64)
    got = oracle.ulp(y.astype(np.float64), oracle.FP32)
    assert np.array_equal(got, want)
