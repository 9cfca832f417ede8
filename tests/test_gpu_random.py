"""Seeded random sweep over the operation's parameter space, each case
against the oracle: activation dtype (bf16, fp16, fp32), M (1 .. 128, the
kernels each entry routes to), N (ragged), K (a multiple of the blocksize,
ragged against every kernel's unit width), blocksize (32 .. 4096), code table
(uniform, normal-quantile, FP4), optional bias and outliers.  Cases the fused
entry does not take (Q4_ERR_UNSUPPORTED) go through q4_linear's split path
instead, so every drawn case is checked on some path of the library."""
import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs
from parity import ORACLE_ACT, TORCH_ACT, bits_of, check_f32, check_gemm

pytestmark = pytest.mark.gpu

TABLES = ("uniform", "normal", "fp4")


def _draw(i: int):
    rng = np.random.default_rng(31337 + i)
    act = ("bf16", "fp16", "fp32")[rng.integers(3)]
    bs = int(2 ** rng.integers(5, 13))                       # 32 .. 4096
    K = bs * int(rng.integers(1, max(2, 6144 // bs) + 1))
    N = int(rng.integers(1, 1500))
    M = int(rng.choice([1, 2, 3, 5, 8, 13, 16, 17, 31, 48, 64, 100, 128] if act != "fp32" else [1, 2, 3, 5, 8, 13, 16]))
    return dict(act=act, M=M, N=N, K=K, bs=bs, table=TABLES[rng.integers(3)], bias=bool(rng.integers(2)),
                outliers=bool(rng.integers(2)), seed=int(rng.integers(1 << 30)))


@pytest.mark.parametrize("i", range(100))
def test_random_case(cuda_device, i):
    c = _draw(i)
    dev = cuda_device
    M, N, K, bs, act = c["M"], c["N"], c["K"], c["bs"], c["act"]
    code = inputs.CODE_TABLES[c["table"]]()
    W = inputs.weights(N, K, c["seed"], c["outliers"])
    packed, absmax = oracle.quantize(W, bs, code)
    if act == "fp32":
        a = inputs.activations_fp32(M, K, c["seed"])
        A = torch.from_numpy(a)
        b = inputs.activations_fp32(1, N, c["seed"] + 1).reshape(N) if c["bias"] else None
        y, S = oracle.gemm_f32(a, packed, absmax, code, M, N, K, bs, bias=b)
        bias = torch.from_numpy(b).to(dev) if b is not None else None
    else:
        A = inputs.activations(M, K, TORCH_ACT[act], c["seed"])
        bt = inputs.activations(1, N, TORCH_ACT[act], c["seed"] + 1).reshape(N) if c["bias"] else None
        y, S = oracle.gemm(bits_of(A), ORACLE_ACT[act], packed, absmax, code, M, N, K, bs,
                           bias_bits=bits_of(bt) if bt is not None else None)
        bias = bt.to(dev) if bt is not None else None
    args = (A.to(dev), torch.from_numpy(packed).to(dev), torch.from_numpy(absmax).to(dev),
            torch.from_numpy(code).to(dev), N, K, bs)
    try:
        out = q4.q4_gemm_skinny(*args, bias=bias)
        path = "fused"
    except q4.Q4Error as e:
        assert e.status == q4.Q4_ERR_UNSUPPORTED, (c, e)
        assert q4.q4_gemm_route(M, N, K, bs, TORCH_ACT[act]) == q4.Q4_ROUTE_SPLIT, c
        out = q4.q4_linear(*args, bias=bias)
        path = "split"
    torch.cuda.synchronize(dev)
    label = f"random {i} {path} {c}"
    if act == "fp32":
        if path == "fused":
            check_f32(out, y, S, K, label)
        else:
            got = out.cpu().numpy().astype(np.float64)
            tol = 1e-2 * S + oracle.ulp(y, oracle.FP32).reshape(y.shape)
            assert np.all(np.abs(got - y) <= tol), label
    else:
        check_gemm(bits_of(out), y, S, act, label)
