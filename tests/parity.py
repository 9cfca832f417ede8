"""Helpers for GPU-vs-oracle parity checks (used by the -m gpu tests and
the smoke check).  Inputs come from bit_weight_dequant_b200.inputs; expected
values come only from the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs

TORCH_ACT = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}
ORACLE_ACT = {"bf16": oracle.BF16, "fp16": oracle.FP16}


def bits_of(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a bf16/fp16 tensor (any device)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def check_gemm(out_bits: np.ndarray, y: np.ndarray, S: np.ndarray, act: str, label: str = ""):
    """Assert |gpu - y| <= 1e-2 * S + ulp(y) element by element."""
    dt = ORACLE_ACT[act]
    got = oracle.decode(out_bits.reshape(-1), dt).reshape(y.shape)
    tol = oracle.gemm_tolerance(y, S, dt)
    err = np.abs(got - y)
    bad = ~(err <= tol)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{label}: {int(bad.sum())} of {bad.size} outputs out of tolerance; first at "
                             f"{tuple(i)}: gpu={got[tuple(i)]!r} oracle={y[tuple(i)]!r} tol={tol[tuple(i)]!r}")
    return float((err / np.maximum(tol, 1e-300)).max()) if err.size else 0.0


def check_f32(out: torch.Tensor, y: np.ndarray, S: np.ndarray, K: int, label: str = "") -> float:
    """fp32 outputs: within the contract bound 1e-2 * S + ulp_fp32(y) and
    within the fp32-arithmetic bound (32 + K/128) * 2^-24 * S + ulp(y) (the
    fp32 kernel rounds each term at most 8 times in its block piece, K/256
    times along a lane's running sum, 5 times across lanes and once per warp
    piece it is combined with; the oracle's fp32 weight adds one)."""
    got = out.detach().cpu().numpy().astype(np.float64).reshape(y.shape)
    u = oracle.ulp(y, oracle.FP32).reshape(y.shape)
    err = np.abs(got - y)
    worst = 0.0
    for name, tol in (("contract", 1e-2 * S + u), ("fp32", (32 + K / 128) * 2.0 ** -24 * S + u)):
        bad = ~(err <= tol)
        if bad.any():
            i = tuple(np.argwhere(bad)[0])
            raise AssertionError(f"{label}: {int(bad.sum())}/{bad.size} outputs outside the {name} bound; first "
                                 f"at {i}: gpu={got[i]!r} oracle={y[i]!r} tol={tol[i]!r}")
        if name == "contract" and err.size:
            worst = float((err / np.maximum(tol, 1e-300)).max())
    return worst


def _activations(case: inputs.Case, seed: int):
    """(A as a CPU tensor, the oracle's expected values and S) for a case."""
    if case.act == "fp32":
        a = inputs.activations_fp32(case.M, case.K, seed)
        return torch.from_numpy(a), a
    A = inputs.activations(case.M, case.K, TORCH_ACT[case.act], seed)
    return A, bits_of(A)


def _oracle_gemm(case: inputs.Case, a, packed, absmax, code, n_rows: int):
    if case.act == "fp32":
        return oracle.gemm_f32(a, packed, absmax, code, case.M, n_rows, case.K, case.blocksize)
    return oracle.gemm(a, ORACLE_ACT[case.act], packed, absmax, code, case.M, n_rows, case.K, case.blocksize)


def _check(case: inputs.Case, out: torch.Tensor, y, S, label: str) -> float:
    if case.act == "fp32":
        return check_f32(out, y, S, case.K, label)
    return check_gemm(bits_of(out), y, S, case.act, label=label)


def run_case(case: inputs.Case, seed: int, device, check_quantizer: bool = True, **launch) -> float:
    """Quantize with the oracle, run the GPU GEMM on the oracle's packed
    weights, compare every output against the oracle.  Returns the worst
    error as a fraction of the tolerance."""
    code = inputs.CODE_TABLES[case.table]()
    W = inputs.weights(case.N, case.K, seed, case.outliers)
    packed, absmax = oracle.quantize(W, case.blocksize, code)
    code_d = torch.from_numpy(code).to(device)
    if check_quantizer:
        gp, ga = q4.q4_quantize_blockwise(torch.from_numpy(W).to(device).reshape(-1), case.blocksize, code_d)
        assert np.array_equal(gp.cpu().numpy(), packed), "GPU codes differ from the oracle's"
        assert np.array_equal(ga.cpu().numpy().view(np.uint32), absmax.view(np.uint32)), "absmax differs"
    A, a_ref = _activations(case, seed)
    y, S = _oracle_gemm(case, a_ref, packed, absmax, code, case.N)
    out = q4.q4_gemm_skinny(A.to(device), torch.from_numpy(packed).to(device), torch.from_numpy(absmax).to(device),
                            code_d, case.N, case.K, case.blocksize, **launch)
    torch.cuda.synchronize(device)
    assert tuple(out.shape) == (case.M, case.N) and out.dtype == TORCH_ACT[case.act]
    return _check(case, out, y, S, str(case))


def sample_rows(N: int, extra: int = 40, seed: int = 0) -> np.ndarray:
    """Rows to check at full size: the first and last row of every 64-row
    tile and of the 8-row group after its first, both ends, the middle and a
    seeded random spread (about 1 row in 16)."""
    rows = {0, 1, N // 2, N - 2, N - 1, N - 65, N - 64}
    for r in range(0, N, 64):
        rows |= {r, r + 7, r + 8, r + 63}
    rng = np.random.default_rng(seed)
    rows |= set(rng.integers(0, N, extra).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N), dtype=np.int64)


def run_case_sampled(case: inputs.Case, seed: int, device, rows: np.ndarray | None = None) -> float:
    """Full-size run in the default launch configuration; W is drawn on the
    device by the seeded input generator, and the oracle checks the GPU's
    codes/absmax and outputs on sampled weight rows (all M rows of A)."""
    rows = sample_rows(case.N, seed=seed) if rows is None else rows
    code = inputs.CODE_TABLES[case.table]()
    code_d = torch.from_numpy(code).to(device)
    W = inputs.weights_device(case.N, case.K, seed, device, case.outliers)
    packed, absmax = q4.q4_quantize_blockwise(W.reshape(-1), case.blocksize, code_d)
    Wr = W[torch.from_numpy(rows).to(device)].cpu().numpy()
    del W
    A, a_ref = _activations(case, seed)
    out = q4.q4_gemm_skinny(A.to(device), packed, absmax, code_d, case.N, case.K, case.blocksize)
    torch.cuda.synchronize(device)
    p_ref, ab_ref = oracle.quantize(Wr, case.blocksize, code)
    rows_d = torch.from_numpy(rows).to(device)
    gp = packed.view(case.N, case.K // 2)[rows_d].cpu().numpy().reshape(-1)
    ga = absmax.view(case.N, case.K // case.blocksize)[rows_d].cpu().numpy().reshape(-1)
    assert np.array_equal(gp, p_ref), "GPU codes differ from the oracle's on sampled rows"
    assert np.array_equal(ga.view(np.uint32), ab_ref.view(np.uint32)), "absmax differs on sampled rows"
    y, S = _oracle_gemm(case, a_ref, p_ref, ab_ref, code, rows.size)
    return _check(case, out[:, rows_d], y, S, f"{case} rows={rows.size}")
