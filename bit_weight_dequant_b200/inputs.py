"""Seeded synthetic inputs and 16-entry code tables.

This module generates inputs only: it holds none of the quantize,
dequantize or matmul arithmetic, so the oracle and the CUDA path can both
take their inputs from it without sharing any of the method.

Workloads (the shapes of the pages' decode benchmarks):
  * bitsandbytes PR #1920, "kgemm_4bit_inference_naive benchmark" and the
    maintainer's RTX 4090 table: 4-bit blockwise weights, blocksize 64,
    llama3-70b-class shapes such as N=28672, K=8192;
  * the GPTQ decode-shape table of the vllm-rdna PR ("Decode-critical
    shapes"): K=5120/N=8192, K=5120/N=5120, K=17408/N=5120, batch 1..32;
  * the wvSplitK report (vLLM PR #40687): batch 5 for speculative decode;
  * the aiter tuning table (ROCm/aiter PR #6201): N=248320 / K=2560 heads,
    K=320, N=12 and N=513 shapes.
Activations are A ~ N(0, 1) drawn in fp32 and rounded to bf16/fp16; weights
are W ~ N(0, 0.02^2) in fp32 (optionally with 1% outliers x20).
"""
from __future__ import annotations

import statistics
from dataclasses import dataclass, field

import numpy as np
import torch

# ---------------------------------------------------------------------------
# Code tables (the pages name an "NF4/FP4 dtype LUT" but print no values).
# ---------------------------------------------------------------------------


def code_uniform() -> np.ndarray:
    """16 evenly spaced levels spanning exactly [-1, 1]: (2i - 15) / 15.

    The table does not contain 0; its largest gap is 2/15."""
    return np.array([(2.0 * i - 15.0) / 15.0 for i in range(16)], dtype=np.float64).astype(np.float32)


def code_normal_quantile(eps: float = 1.0 / 32.0) -> np.ndarray:
    """Normal-quantile ("NF4-like") table in [-1, 1] that contains 0.

    With 16 entries a table cannot be both symmetric and contain an exact 0,
    so it holds 8 positive levels, 7 negative levels and 0:
      pos_j = invPhi(1/2 + j (1/2 - eps) / 8) / invPhi(1 - eps),  j = 1..8
      neg_j = -invPhi(1/2 + j (1/2 - eps) / 7) / invPhi(1 - eps), j = 1..7
    computed in fp64, rounded once to fp32, sorted ascending.  Both ends are
    exactly -1 and +1."""
    nd = statistics.NormalDist()
    top = nd.inv_cdf(1.0 - eps)
    pos = [nd.inv_cdf(0.5 + j * (0.5 - eps) / 8.0) / top for j in range(1, 9)]
    neg = [-nd.inv_cdf(0.5 + j * (0.5 - eps) / 7.0) / top for j in range(1, 8)]
    vals = sorted(neg + [0.0] + pos)
    return np.array(vals, dtype=np.float64).astype(np.float32)


def code_fp4_e2m1() -> np.ndarray:
    """The 16 values of a 4-bit float (1 sign, 2 exponent, 1 mantissa bit,
    exponent bias 1), indexed by their bit pattern and divided by the
    largest magnitude, 6, so that the table spans [-1, 1].

    Code i has sign = bit 3, exponent e = bits 2..1, mantissa m = bit 0.
    Its magnitude is m/2 for e = 0 (zero and the one subnormal, 1/2) and
    2^(e-1) * (1 + m/2) otherwise, i.e. 0, 1/2, 1, 3/2, 2, 3, 4, 6.  The
    table is in bit order, not sorted, and code 8 is -0."""
    vals = []
    for i in range(16):
        s, e, m = i >> 3, (i >> 1) & 3, i & 1
        mag = m / 2.0 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
        vals.append((-mag if s else mag) / 6.0)
    return np.array(vals, dtype=np.float64).astype(np.float32)


CODE_TABLES = {"normal": code_normal_quantile, "uniform": code_uniform, "fp4": code_fp4_e2m1}

# ---------------------------------------------------------------------------
# Random inputs.
# ---------------------------------------------------------------------------

WEIGHT_SIGMA = 0.02
OUTLIER_RATE = 0.01
OUTLIER_SCALE = 20.0
ROWS_PER_CHUNK = 256  # W rows drawn per generator stream (lets a row subset be regenerated)


def seed_for(config_index: int, M: int) -> int:
    return 20261202 + 100 * config_index + M


def activations_fp32(M: int, K: int, seed: int) -> np.ndarray:
    """A ~ N(0, 1) in fp32, shape [M, K]."""
    return np.random.default_rng([seed, 0xA]).standard_normal((M, K), dtype=np.float32)


def activations(M: int, K: int, dtype: torch.dtype, seed: int) -> torch.Tensor:
    """A ~ N(0, 1) drawn in fp32 and rounded (RNE, torch's conversion) to
    ``dtype`` (bf16 or fp16; fp32 keeps the draws); a CPU tensor of shape [M, K]."""
    return torch.from_numpy(activations_fp32(M, K, seed)).to(dtype)


def weight_rows(K: int, seed: int, row0: int, row1: int, outliers: bool = False) -> np.ndarray:
    """Rows [row0, row1) of W ~ N(0, 0.02^2) (fp32, shape [row1-row0, K]).

    Rows are drawn in chunks of ROWS_PER_CHUNK from per-chunk streams, so any
    row range can be regenerated on its own.  With ``outliers`` an
    independent Bernoulli(0.01) mask (its own streams) multiplies the chosen
    elements by 20."""
    out = np.empty((row1 - row0, K), dtype=np.float32)
    c0, c1 = row0 // ROWS_PER_CHUNK, (row1 - 1) // ROWS_PER_CHUNK
    for c in range(c0, c1 + 1):
        base = c * ROWS_PER_CHUNK
        rng = np.random.default_rng([seed, 0xB, c])
        block = rng.standard_normal((ROWS_PER_CHUNK, K), dtype=np.float32) * np.float32(WEIGHT_SIGMA)
        if outliers:
            mrng = np.random.default_rng([seed + 1, 0xC, c])
            mask = mrng.random((ROWS_PER_CHUNK, K)) < OUTLIER_RATE
            block[mask] *= np.float32(OUTLIER_SCALE)
        lo, hi = max(row0, base), min(row1, base + ROWS_PER_CHUNK)
        out[lo - row0:hi - row0] = block[lo - base:hi - base]
    return out


def weights(N: int, K: int, seed: int, outliers: bool = False) -> np.ndarray:
    """Full W [N, K] fp32 (see ``weight_rows``)."""
    return weight_rows(K, seed, 0, N, outliers)


def weights_equal_codes(absmax_rows: np.ndarray, K: int, blocksize: int, value: float) -> np.ndarray:
    """Adversarial W [len(absmax_rows), K] fp32: in every block of row n the
    first element is absmax_rows[n] and the others are absmax_rows[n] * value
    (one fp32 product), so each block quantizes to one +1 code and
    blocksize - 1 copies of the code nearest `value`.  With non-negative
    activations every weight's rounding error then has the same sign."""
    am = np.asarray(absmax_rows, dtype=np.float32)
    W = np.repeat((am * np.float32(value))[:, None], K, axis=1).astype(np.float32)
    W[:, ::blocksize] = am[:, None]
    return W


def weights_device(N: int, K: int, seed: int, device, outliers: bool = False) -> torch.Tensor:
    """W ~ N(0, 0.02^2) drawn directly on a CUDA device with torch's seeded
    generator (for full-size runs where host generation is too slow).  Rows
    can be copied back to the host to feed the oracle."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * WEIGHT_SIGMA
    if outliers:
        g2 = torch.Generator(device=device)
        g2.manual_seed(seed + 1)
        mask = torch.rand((N, K), generator=g2, device=device) < OUTLIER_RATE
        w = torch.where(mask, w * OUTLIER_SCALE, w)
    return w


# ---------------------------------------------------------------------------
# Workload catalogue (shapes of the five benchmark configurations).
# ---------------------------------------------------------------------------


@dataclass(frozen=True)
class Case:
    """One GEMM problem: C[M,N] = A[M,K] . dequant(W)[N,K]^T."""
    M: int
    N: int
    K: int
    blocksize: int = 64
    act: str = "bf16"          # "bf16" | "fp16" | "fp32"
    table: str = "normal"      # "normal" | "uniform"
    outliers: bool = False
    tag: str = ""

    def algorithmic_bytes(self) -> int:
        """M*K*e + N*K/2 + 4*N*K/bs + M*N*e (activations, codes, absmax, out;
        e = 2 bytes for bf16/fp16 activations, 4 for fp32)."""
        nk = self.N * self.K
        e = 4 if self.act == "fp32" else 2
        return self.M * self.K * e + nk // 2 + 4 * ((nk + self.blocksize - 1) // self.blocksize) \
            + self.M * self.N * e


@dataclass
class Workload:
    name: str
    index: int
    cases: list = field(default_factory=list)


def workloads() -> dict:
    """The five configurations, each a list of Cases, and one profiling shape."""
    w = {}
    # 0: small square check case.
    w["square4096"] = Workload("M=1 K=4096 N=4096 bs64 bf16 normal-table", 0,
                               [Case(1, 4096, 4096, tag="sq4096")])
    # 1: 70B-class decode layer at M=1.
    w["decode70b"] = Workload(
        "M=1 decode shapes of a 70B-class layer (K8192/N10240, K8192/N28672, K28672/N8192, K8192/N8192), "
        "bs64 bf16 normal-table", 1,
        [Case(1, 10240, 8192, tag="qkv"), Case(1, 28672, 8192, tag="gate_up"),
         Case(1, 8192, 28672, tag="down"), Case(1, 8192, 8192, tag="o_proj")])
    # 2: M sweep on GPTQ-page decode shapes.
    sweep = []
    for (K, N) in ((5120, 5120), (5120, 8192), (17408, 5120)):
        for M in (1, 2, 4, 5, 8, 12, 16):
            sweep.append(Case(M, N, K, tag=f"K{K}N{N}M{M}"))
    w["msweep"] = Workload("M sweep 1,2,4,5,8,12,16 on K5120/N5120, K5120/N8192, K17408/N5120", 2, sweep)
    # 3: quantization variants at M=1 and M=4 on 4096x4096.
    var = []
    for M in (1, 4):
        for bs in (32, 128, 256):
            var.append(Case(M, 4096, 4096, blocksize=bs, tag=f"bs{bs}M{M}"))
        var.append(Case(M, 4096, 4096, act="fp16", tag=f"fp16M{M}"))
        var.append(Case(M, 4096, 4096, table="uniform", tag=f"uniformM{M}"))
        var.append(Case(M, 513, 4096, tag=f"N513M{M}"))
        var.append(Case(M, 4096, 4096, outliers=True, tag=f"outlierM{M}"))
    w["variants"] = Workload("quantization variants at M=1,4 on K4096/N4096", 3, var)
    # 4: extreme aspect ratios at M=1..8.
    ext = []
    for (K, N) in ((2560, 248320), (320, 10240), (10240, 320), (2560, 12)):
        for M in (1, 2, 4, 8):
            ext.append(Case(M, N, K, tag=f"K{K}N{N}M{M}"))
    w["aspect"] = Workload("extreme aspect ratios at M=1..8: K2560/N248320, K320/N10240, K10240/N320, "
                           "K2560/N12", 4, ext)
    # Beyond the five: the M sweep's shapes at 17 <= M <= 128 (the
    # tensor-memory kernel), for parity and for the fused-vs-split crossover.
    big = []
    for (K, N) in ((5120, 5120), (5120, 8192), (17408, 5120)):
        for M in (17, 32, 64, 128):
            big.append(Case(M, N, K, tag=f"K{K}N{N}M{M}"))
    w["mlarge"] = Workload("M 17,32,64,128 on K5120/N5120, K5120/N8192, K17408/N5120 (tcgen05 kernel)", 6, big)
    # Beyond the five: fp32 activations (the CUDA-core kernel) on the decode
    # shapes at M=1 and on the M sweep's shapes.
    w["decode70b_f32"] = Workload(
        "M=1 decode shapes of a 70B-class layer (K8192/N10240, K8192/N28672, K28672/N8192, K8192/N8192), "
        "bs64 fp32 activations, normal-table", 7,
        [Case(1, 10240, 8192, act="fp32", tag="qkv"), Case(1, 28672, 8192, act="fp32", tag="gate_up"),
         Case(1, 8192, 28672, act="fp32", tag="down"), Case(1, 8192, 8192, act="fp32", tag="o_proj")])
    f32 = []
    for (K, N) in ((5120, 5120), (17408, 5120)):
        for M in (1, 2, 4, 8, 16):
            f32.append(Case(M, N, K, act="fp32", tag=f"K{K}N{N}M{M}"))
    w["msweep_f32"] = Workload("fp32 activations, M 1,2,4,8,16 on K5120/N5120, K17408/N5120", 8, f32)
    w["longk_f32"] = Workload("M=1 K=131072 N=2048 bs64 fp32 activations (main-loop profiling shape)", 9,
                              [Case(1, 2048, 131072, act="fp32", tag="longk")])
    # Not one of the five: the decode gate_up shape at M = 1, 2, 4, for the
    # CUDA-core against tensor-core comparison.
    w["gate_up_m"] = Workload("M 1,2,4 on K8192/N28672 bs64 bf16 normal-table", 10,
                              [Case(M, 28672, 8192, tag=f"gate_upM{M}") for M in (1, 2, 4)])
    # Not one of the five: one long-K layer whose launch is almost all main
    # loop (start-up and tail are a few percent), for profiling the loop.
    w["longk"] = Workload("M=1 K=131072 N=8192 bs64 bf16 normal-table (main-loop profiling shape)", 5,
                          [Case(1, 8192, 131072, tag="longk")])
    return w
