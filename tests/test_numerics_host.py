"""Host checks of the weight arithmetic the fused kernels feed their MMAs
(no GPU), against the contract |gpu - y| <= 1e-2 * sum_k |a w| + ulp(y).

  * The mma.sync kernels (M <= 32) feed T(code) and apply the absmax in fp32
    to partial sums: one rounding to the activation type T per weight.
  * The tcgen05 kernel feeds T_rn(code *_fp32 absmax), the standalone
    dequantizer's value: one rounding as well.

One rounding to T costs at most its unit roundoff u, 2^-8 for bf16 (8
significant bits) and 2^-11 for fp16; errors of equal codes under one
absmax share their sign, so u itself must stay below 1e-2.  A cheaper
form that rounds three times -- a table of codes already in T, times the
absmax rounded to T, rounded again -- is shown here to exceed 1e-2 for
some (code, absmax) pairs, which is why no kernel uses it.

bf16 rounding is emulated by round-to-nearest-even on the fp32 bit
pattern, fp16 by numpy's conversion; the product of two bf16 (fp16)
values is exact in fp32.
"""
import numpy as np
import pytest

from bit_weight_dequant_b200 import inputs


def _bf16(x):
    """fp32 -> nearest bf16 (ties to even), returned as fp32."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def _fp16(x):
    return np.asarray(x, dtype=np.float32).astype(np.float16).astype(np.float32)


ROUND = {"bf16": (_bf16, 2.0 ** -8, (-12, 6)), "fp16": (_fp16, 2.0 ** -11, (-10, 10))}


def _grid(table, kind):
    code = inputs.CODE_TABLES[table]().astype(np.float32)
    lo, hi = ROUND[kind][2]  # fp16: absmax in the normal range and |w| <= 65504
    am = np.exp2(np.random.default_rng(20261202).uniform(lo, hi, 4096)).astype(np.float32)
    exact = code[None, :].astype(np.float64) * am[:, None].astype(np.float64)
    return code, am, exact


def _max_rel(fed, exact):
    nz = exact != 0
    return float((np.abs(fed.astype(np.float64) - exact)[nz] / np.abs(exact[nz])).max())


def test_bf16_rounding_helper_against_known_values():
    # 1 + 2^-8 lies halfway between bf16 neighbours 1 and 1 + 2^-7: ties to even -> 1
    assert _bf16(np.float32(1 + 2.0 ** -8)) == np.float32(1.0)
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: ties to even -> 1 + 2^-6
    assert _bf16(np.float32(1 + 3 * 2.0 ** -8)) == np.float32(1 + 2.0 ** -6)
    assert _bf16(np.float32(-0.1)) == np.float32(-0.10009765625)


@pytest.mark.parametrize("table", ["normal", "uniform", "fp4"])
@pytest.mark.parametrize("kind", ["bf16", "fp16"])
def test_one_rounding_stays_inside_the_contract(table, kind):
    rnd, u, _ = ROUND[kind]
    code, am, exact = _grid(table, kind)
    tcgen05 = rnd((code[None, :].astype(np.float32) * am[:, None]))  # T_rn(code *_fp32 absmax)
    mma = rnd(code)[None, :].astype(np.float64) * am[:, None]         # T(code), absmax applied in fp32
    # the fp32 product itself adds at most 2^-24 before the rounding to T
    assert _max_rel(tcgen05, exact) <= (1 + u) * (1 + 2.0 ** -24) - 1
    assert _max_rel(mma, exact) <= u
    assert u < 1e-2


def test_three_roundings_can_break_the_contract():
    rnd, u, _ = ROUND["bf16"]
    code, am, exact = _grid("uniform", "bf16")
    three = rnd(rnd(code)[None, :] * rnd(am)[:, None])
    worst = _max_rel(three, exact)
    assert worst > 1e-2  # a row of such weights under one absmax exceeds the bound
    assert worst <= (1 + u) ** 3 - 1


@pytest.mark.parametrize("table", ["normal", "uniform", "fp4"])
def test_two_roundings_fit_the_contract(table):
    """The table form that stays admissible: codes rounded to bf16 in the
    table, the absmax applied in fp32, one rounding of the product.  Two
    roundings: at most (1 + 2^-8)^2 - 1, about 0.78 %, below 1e-2."""
    rnd, u, _ = ROUND["bf16"]
    code, am, exact = _grid(table, "bf16")
    two = rnd(rnd(code)[None, :] * am[:, None])  # fp32 product of a bf16 code and the fp32 absmax
    # the fp32 product rounds once more before bf16: at most 2^-24 on top
    assert _max_rel(two, exact) <= (1 + u) ** 2 * (1 + 2.0 ** -24) - 1
    assert (1 + u) ** 2 - 1 < 1e-2
