"""CPU oracle for blockwise 4-bit quantize / dequantize / skinny matmul.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product library never does.
The arithmetic lives in ``q4_oracle.c`` (plain C loops, fp64 accumulation);
this module only marshals numpy arrays into it through ctypes.  It shares no
code with the CUDA library.

The method it follows is the fused 4-bit dequantize + matmul of bitsandbytes
PR #1920 ("[ROCm] Optimize kgemm_4bit_inference_naive ...", sections
"Technical details" and "Fused path support for M > 1"); the readings taken
where that page is silent are listed in the header of ``q4_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

BF16, FP16, FP32 = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

# Flags matter: no fast-math (IEEE binary32 / binary64 with subnormals) and no
# FMA contraction (every product and sum is rounded as written).
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to the source (gcc) if stale or missing."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *CFLAGS, "-o", _LIB_PATH, _SRC, "-lm"])
    return _LIB_PATH


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        ci = ctypes.c_int
        lib.oracle_quantize.argtypes = [P, i64, ci, P, P, P]
        lib.oracle_dequantize.argtypes = [P, P, P, i64, ci, ci, P]
        lib.oracle_gemm.argtypes = [P, ci, P, P, P, ci, ci, ci, ci, P, P]
        lib.oracle_gemm_bias.argtypes = [P, ci, P, P, P, P, ci, ci, ci, ci, P, P]
        lib.oracle_gemm_f32.argtypes = [P, P, P, P, P, ci, ci, ci, ci, P, P]
        lib.oracle_round.argtypes = [P, i64, ci, P]
        lib.oracle_decode.argtypes = [P, i64, ci, P]
        lib.oracle_ulp.argtypes = [P, i64, ci, P]
        for f in ("oracle_quantize", "oracle_dequantize", "oracle_gemm", "oracle_gemm_bias", "oracle_gemm_f32",
                  "oracle_round",
                  "oracle_decode", "oracle_ulp"):
            getattr(lib, f).restype = ci
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (status {rc})")


def quantize(w: np.ndarray, blocksize: int, code: np.ndarray):
    """Blockwise 4-bit quantization of a flattened fp32 array.

    Returns ``(packed uint8[ceil(n/2)], absmax float32[ceil(n/bs)])``."""
    w = np.ascontiguousarray(w, dtype=np.float32).reshape(-1)
    code = np.ascontiguousarray(code, dtype=np.float32)
    assert code.shape == (16,)
    n = w.size
    packed = np.zeros((n + 1) // 2, dtype=np.uint8)
    absmax = np.zeros((n + blocksize - 1) // blocksize, dtype=np.float32)
    _check(_load().oracle_quantize(_ptr(w), n, blocksize, _ptr(code), _ptr(packed), _ptr(absmax)), "quantize")
    return packed, absmax


def dequantize(packed: np.ndarray, absmax: np.ndarray, code: np.ndarray, n: int, blocksize: int,
               dtype: int) -> np.ndarray:
    """Dequantize to bf16/fp16 bit patterns (uint16) or fp32 values."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    code = np.ascontiguousarray(code, dtype=np.float32)
    out = np.zeros(n, dtype=np.float32 if dtype == FP32 else np.uint16)
    _check(_load().oracle_dequantize(_ptr(packed), _ptr(absmax), _ptr(code), n, blocksize, dtype, _ptr(out)),
           "dequantize")
    return out


def gemm(a_bits: np.ndarray, act_dtype: int, packed: np.ndarray, absmax: np.ndarray, code: np.ndarray,
         M: int, N: int, K: int, blocksize: int, want_s: bool = True, bias_bits: np.ndarray | None = None):
    """fp64 reference ``y[M,N]`` (unrounded) and ``S[M,N] = sum |a*w|``;
    with ``bias_bits`` (N bf16/fp16 patterns) the bias is added to y."""
    a_bits = np.ascontiguousarray(a_bits, dtype=np.uint16).reshape(-1)
    assert a_bits.size == M * K
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    code = np.ascontiguousarray(code, dtype=np.float32)
    y = np.zeros((M, N), dtype=np.float64)
    S = np.zeros((M, N), dtype=np.float64) if want_s else None
    if bias_bits is None:
        _check(_load().oracle_gemm(_ptr(a_bits), act_dtype, _ptr(packed), _ptr(absmax), _ptr(code), M, N, K,
                                   blocksize, _ptr(y), _ptr(S) if want_s else None), "gemm")
    else:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16).reshape(-1)
        assert bias_bits.size == N
        _check(_load().oracle_gemm_bias(_ptr(a_bits), act_dtype, _ptr(packed), _ptr(absmax), _ptr(code),
                                        _ptr(bias_bits), M, N, K, blocksize, _ptr(y),
                                        _ptr(S) if want_s else None), "gemm_bias")
    return (y, S) if want_s else y


def gemm_f32(a: np.ndarray, packed: np.ndarray, absmax: np.ndarray, code: np.ndarray, M: int, N: int, K: int,
             blocksize: int, want_s: bool = True, bias: np.ndarray | None = None):
    """fp64 reference ``y[M,N]`` and ``S[M,N] = sum |a*w|`` for fp32
    activations ``a[M,K]``; ``bias`` (N fp32 values) is added to y."""
    a = np.ascontiguousarray(a, dtype=np.float32).reshape(-1)
    assert a.size == M * K
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    code = np.ascontiguousarray(code, dtype=np.float32)
    if bias is not None:
        bias = np.ascontiguousarray(bias, dtype=np.float32).reshape(-1)
        assert bias.size == N
    y = np.zeros((M, N), dtype=np.float64)
    S = np.zeros((M, N), dtype=np.float64) if want_s else None
    _check(_load().oracle_gemm_f32(_ptr(a), _ptr(packed), _ptr(absmax), _ptr(code),
                                   _ptr(bias) if bias is not None else None, M, N, K, blocksize, _ptr(y),
                                   _ptr(S) if want_s else None), "gemm_f32")
    return (y, S) if want_s else y


def round_to(x: np.ndarray, dtype: int) -> np.ndarray:
    """Round doubles once (nearest-even) to bf16/fp16; returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float64).reshape(-1)
    out = np.zeros(x.size, dtype=np.uint16)
    _check(_load().oracle_round(_ptr(x), x.size, dtype, _ptr(out)), "round")
    return out


def decode(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Exact values (float64) of bf16/fp16 bit patterns."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16).reshape(-1)
    out = np.zeros(bits.size, dtype=np.float64)
    _check(_load().oracle_decode(_ptr(bits), bits.size, dtype, _ptr(out)), "decode")
    return out


def ulp(y: np.ndarray, dtype: int) -> np.ndarray:
    """Spacing of the bf16/fp16/fp32 format at |y| (subnormal spacing at 0)."""
    y = np.ascontiguousarray(y, dtype=np.float64).reshape(-1)
    out = np.zeros(y.size, dtype=np.float64)
    _check(_load().oracle_ulp(_ptr(y), y.size, dtype, _ptr(out)), "ulp")
    return out


def gemm_tolerance(y: np.ndarray, S: np.ndarray, dtype: int, rel: float = 1e-2) -> np.ndarray:
    """Acceptance bound ``rel * S + ulp(y)`` for a GEMM output element."""
    return rel * S + ulp(y, dtype).reshape(np.shape(y))
