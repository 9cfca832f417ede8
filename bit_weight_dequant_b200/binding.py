"""Thin ctypes binding over libq4.so (the C ABI of include/q4.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libq4.  PyTorch supplies device memory and the current stream.
The library must be built (``python -m bit_weight_dequant_b200.build``);
there is no fallback of any kind, a missing library raises.
"""
from __future__ import annotations

import ctypes
import functools
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libq4.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "q4.h")

Q4_OK, Q4_ERR_INVALID_ARG, Q4_ERR_UNSUPPORTED, Q4_ERR_MISALIGNED, Q4_ERR_CUDA, Q4_ERR_WORKSPACE = range(6)
Q4_BF16, Q4_FP16, Q4_FP32 = 0, 1, 2
Q4_ROUTE_FUSED, Q4_ROUTE_SPLIT = 0, 1

_TORCH_TO_Q4 = {torch.bfloat16: Q4_BF16, torch.float16: Q4_FP16, torch.float32: Q4_FP32}
_Q4_TO_TORCH = {v: k for k, v in _TORCH_TO_Q4.items()}


class Q4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class q4_gemm_plan_t(ctypes.Structure):
    _fields_ = [("math", ctypes.c_int), ("sub_block", ctypes.c_int), ("m_pad", ctypes.c_int),
                ("rows_per_tile", ctypes.c_int), ("warps", ctypes.c_int), ("ctas", ctypes.c_int),
                ("depth", ctypes.c_int), ("l2_prefetch", ctypes.c_int), ("loader", ctypes.c_int), ("pdl", ctypes.c_int),
                ("tiles", ctypes.c_int),
                ("units", ctypes.c_int64), ("smem_bytes", ctypes.c_size_t), ("workspace_bytes", ctypes.c_size_t)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libq4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libq4.so is not built ({LIB_PATH}); run `python -m bit_weight_dequant_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, ci, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.q4_status_string.argtypes = [ci]
        L.q4_status_string.restype = ctypes.c_char_p
        L.q4_quantize_blockwise.argtypes = [P, i64, ci, P, P, P, P]
        L.q4_quantize_blockwise_ex.argtypes = [P, ci, i64, ci, P, P, P, P]
        L.q4_dequantize_blockwise.argtypes = [P, P, P, i64, ci, ci, P, P]
        L.q4_gemm_workspace_size.argtypes = [ci, ci, ci, ci, ci, ctypes.POINTER(sz)]
        L.q4_gemm_workspace_size_ex.argtypes = [ci, ci, ci, ci, ci, ctypes.POINTER(q4_gemm_plan_t),
                                                ctypes.POINTER(sz)]
        L.q4_gemm_skinny.argtypes = [P, P, P, P, ci, ci, ci, ci, ci, P, P, sz, P]
        L.q4_gemm_skinny_ex.argtypes = [P, P, P, P, ci, ci, ci, ci, ci, P, P, sz, P, ctypes.POINTER(q4_gemm_plan_t)]
        L.q4_gemm_plan.argtypes = [ci, ci, ci, ci, ci, ci, ctypes.POINTER(q4_gemm_plan_t)]
        L.q4_gemm_skinny_noalloc.argtypes = [P, P, P, P, ci, ci, ci, ci, ci, P, P]
        L.q4_gemm_skinny_bias.argtypes = [P, P, P, P, P, ci, ci, ci, ci, ci, P, P, sz, P,
                                          ctypes.POINTER(q4_gemm_plan_t)]
        L.q4_gemm_route.argtypes = [ci, ci, ci, ci, ci, ctypes.POINTER(ci)]
        L.q4_partition_start.argtypes = [i64, ci, ci]
        L.q4_partition_start.restype = i64
        L.q4_partition_owner.argtypes = [i64, ci, i64]
        for f in ("q4_quantize_blockwise", "q4_quantize_blockwise_ex", "q4_dequantize_blockwise", "q4_gemm_workspace_size",
                  "q4_gemm_skinny", "q4_gemm_skinny_ex", "q4_gemm_plan", "q4_partition_owner",
                  "q4_gemm_skinny_noalloc", "q4_gemm_skinny_bias", "q4_gemm_route", "q4_gemm_workspace_size_ex"):
            getattr(L, f).restype = ci
        _lib = L
    return _lib


def declared_functions() -> list:
    """Names of the functions include/q4.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(q4_\w+)\s*\(", text)))


def status_string(status: int) -> str:
    return lib().q4_status_string(status).decode()


def _check(rc: int, what: str):
    if rc != Q4_OK:
        raise Q4Error(rc, what)


def _ptr(t):
    """Device address of a tensor as a plain int (ctypes converts it), or None."""
    return t.data_ptr() if t is not None else None


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def q4_quantize_blockwise(W: torch.Tensor, blocksize: int, code: torch.Tensor):
    """Quantize a CUDA fp32, bf16 or fp16 tensor blockwise; returns (packed uint8, absmax fp32)."""
    assert W.is_cuda and W.dtype in _TORCH_TO_Q4 and W.is_contiguous()
    n = W.numel()
    packed = torch.empty((n + 1) // 2, dtype=torch.uint8, device=W.device)
    absmax = torch.empty((n + blocksize - 1) // blocksize, dtype=torch.float32, device=W.device)
    rc = lib().q4_quantize_blockwise_ex(_ptr(W), _TORCH_TO_Q4[W.dtype], n, blocksize, _ptr(code), _ptr(packed),
                                        _ptr(absmax), _stream(W.device))
    _check(rc, "q4_quantize_blockwise")
    return packed, absmax


def q4_dequantize_blockwise(packed: torch.Tensor, absmax: torch.Tensor, code: torch.Tensor, n: int,
                            blocksize: int, out_dtype: torch.dtype = torch.bfloat16,
                            out: torch.Tensor | None = None) -> torch.Tensor:
    """Dequantize to bf16/fp16/fp32 (CUDA tensor of n elements)."""
    if out is None:
        out = torch.empty(n, dtype=out_dtype, device=packed.device)
    rc = lib().q4_dequantize_blockwise(_ptr(packed), _ptr(absmax), _ptr(code), n, blocksize,
                                       _TORCH_TO_Q4[out.dtype], _ptr(out), _stream(packed.device))
    _check(rc, "q4_dequantize_blockwise")
    return out


def q4_gemm_workspace_size(M: int, N: int, K: int, blocksize: int, act_dtype: torch.dtype, **launch) -> int:
    """Workspace bytes for a call (with the same launch-table overrides as
    the call, if any)."""
    return _workspace_bytes(M, N, K, blocksize, _TORCH_TO_Q4[act_dtype], tuple(sorted(launch.items())))


@functools.lru_cache(maxsize=4096)
def _workspace_bytes(M: int, N: int, K: int, blocksize: int, act: int, launch: tuple = ()) -> int:
    v = ctypes.c_size_t(0)
    ov = _overrides_ref(launch)[1] if launch else None
    _check(lib().q4_gemm_workspace_size_ex(M, N, K, blocksize, act, ov, ctypes.byref(v)), "q4_gemm_workspace_size")
    return v.value


def q4_gemm_plan(M: int, N: int, K: int, blocksize: int, act_dtype: torch.dtype = torch.bfloat16,
                 num_sms: int = 0) -> dict:
    pl = q4_gemm_plan_t()
    _check(lib().q4_gemm_plan(M, N, K, blocksize, _TORCH_TO_Q4[act_dtype], num_sms, ctypes.byref(pl)),
           "q4_gemm_plan")
    return {f: getattr(pl, f) for f, _ in q4_gemm_plan_t._fields_}


class Workspace:
    """Zero-filled device scratch for q4_gemm_skinny, grown on demand.

    Every successful call returns the workspace's tile counters (and the
    tensor-memory kernel's partial slots) to zero, so it is zero-filled once,
    at allocation, and again by ``reset()`` after a call that set the error
    word; one per stream."""

    def __init__(self, device):
        self.device = torch.device(device)
        self.buf = torch.zeros(0, dtype=torch.uint8, device=self.device)

    def reset(self):
        """Zero the whole workspace (needed after a call that set the error word)."""
        self.buf.zero_()

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 2 * self.buf.numel()), dtype=torch.uint8, device=self.device)
        return self.buf


_workspaces: dict = {}

MAX_SLOT_BYTES = 4096     # partial-sum slot of the largest variant (64 rows x 16 columns x fp32)


WORKSPACE_HEADER_BYTES = 256   # the first int32 is the error word


def workspace_counter_offset(device) -> int:
    """Byte offset of the per-tile counters inside a GEMM workspace (a
    256-byte header and two partial-sum slots per SM come first; see
    q4_gemm_skinny in q4.h)."""
    return WORKSPACE_HEADER_BYTES + torch.cuda.get_device_properties(device).multi_processor_count * 2 * MAX_SLOT_BYTES


def workspace_error(ws: "Workspace") -> int:
    """The workspace's error word (0 = no kernel gave up a bounded wait)."""
    return int(ws.buf[:4].view(torch.int32).item()) if ws.buf.numel() >= 4 else 0



def _default_workspace(device, stream: int) -> Workspace:
    key = (device, stream)
    ws = _workspaces.get(key)
    if ws is None:
        ws = _workspaces[key] = Workspace(device)
    return ws


def overrides(**kw) -> q4_gemm_plan_t | None:
    """Launch-table overrides (math, warps, ctas, depth, l2_prefetch, loader, pdl); None if empty."""
    kw = {k: v for k, v in kw.items() if v}
    if not kw:
        return None
    ov = q4_gemm_plan_t()
    for k, v in kw.items():
        setattr(ov, k, int(v))
    return ov


@functools.lru_cache(maxsize=256)
def _overrides_ref(items: tuple):
    """byref() of a cached, never-modified overrides struct (None if empty)."""
    ov = overrides(**dict(items))
    return (ov, ctypes.byref(ov)) if ov is not None else (None, None)


def q4_gemm_skinny(A: torch.Tensor, Wpacked: torch.Tensor, absmax: torch.Tensor, code: torch.Tensor, N: int,
                   K: int, blocksize: int, out: torch.Tensor | None = None, workspace: Workspace | None = None,
                   bias: torch.Tensor | None = None, **launch) -> torch.Tensor:
    """out[M, N] = A[M, K] . dequant(W)[N, K]^T (+ bias[N]) on the GPU (fused kernel).

    ``bias`` (N values of A's dtype) is added in the epilogue before the
    rounding (q4_gemm_skinny_bias).  ``launch`` may hold launch-table
    overrides (math, warps, ctas, depth, l2_prefetch, loader) for
    measurements, and ``pdl`` to opt into programmatic dependent launch (see
    q4.h); by default the table decides.  Argument marshalling only: the
    per-call work on the host is a few dictionary lookups and one C call."""
    M = A.shape[0] if A.dim() == 2 else 1
    if out is None:
        out = torch.empty((M, N), dtype=A.dtype, device=A.device)
    act = _TORCH_TO_Q4[A.dtype]
    items = tuple(sorted(launch.items())) if launch else ()
    nbytes = _workspace_bytes(M, N, K, blocksize, act, items)
    stream = torch.cuda.current_stream(A.device).cuda_stream
    ws = (workspace or _default_workspace(A.device, stream)).get(nbytes) if nbytes else None
    ov_ref = _overrides_ref(items)[1] if launch else None
    if bias is None:
        rc = lib().q4_gemm_skinny_ex(A.data_ptr(), Wpacked.data_ptr(), absmax.data_ptr(), code.data_ptr(), M, N, K,
                                     blocksize, act, out.data_ptr(), ws.data_ptr() if ws is not None else None,
                                     ws.numel() if ws is not None else 0, stream, ov_ref)
    else:
        assert bias.dtype == A.dtype and bias.numel() == N and bias.is_contiguous()
        rc = lib().q4_gemm_skinny_bias(A.data_ptr(), Wpacked.data_ptr(), absmax.data_ptr(), code.data_ptr(),
                                       bias.data_ptr(), M, N, K, blocksize, act, out.data_ptr(),
                                       ws.data_ptr() if ws is not None else None,
                                       ws.numel() if ws is not None else 0, stream, ov_ref)
    _check(rc, "q4_gemm_skinny")
    return out


def q4_gemm_skinny_noalloc(A: torch.Tensor, Wpacked: torch.Tensor, absmax: torch.Tensor, code: torch.Tensor, N: int,
                           K: int, blocksize: int, out: torch.Tensor | None = None) -> torch.Tensor:
    """q4_gemm_skinny on the library's built-in scratch array: no workspace
    is allocated, by this call or by the library (see q4.h)."""
    M = A.shape[0] if A.dim() == 2 else 1
    if out is None:
        out = torch.empty((M, N), dtype=A.dtype, device=A.device)
    rc = lib().q4_gemm_skinny_noalloc(_ptr(A), _ptr(Wpacked), _ptr(absmax), _ptr(code), M, N, K, blocksize,
                                      _TORCH_TO_Q4[A.dtype], _ptr(out), _stream(A.device))
    _check(rc, "q4_gemm_skinny_noalloc")
    return out


@functools.lru_cache(maxsize=1024)
def _route(M: int, N: int, K: int, blocksize: int, act: int) -> int:
    r = ctypes.c_int(-1)
    _check(lib().q4_gemm_route(M, N, K, blocksize, act, ctypes.byref(r)), "q4_gemm_route")
    return r.value


def q4_gemm_route(M: int, N: int, K: int, blocksize: int, act_dtype: torch.dtype = torch.bfloat16) -> int:
    """Q4_ROUTE_FUSED or Q4_ROUTE_SPLIT: the library's fused-vs-split choice (see q4.h)."""
    return _route(M, N, K, blocksize, _TORCH_TO_Q4[act_dtype])


def q4_linear(A: torch.Tensor, Wpacked: torch.Tensor, absmax: torch.Tensor, code: torch.Tensor, N: int, K: int,
              blocksize: int, bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
              workspace: Workspace | None = None) -> torch.Tensor:
    """out = A . dequant(W)^T (+ bias) on the path q4_gemm_route picks: the
    fused kernel, or this library's dequantize into a temporary dense matrix
    followed by a cuBLAS GEMM (torch.matmul / torch.addmm)."""
    M = A.shape[0] if A.dim() == 2 else 1
    if q4_gemm_route(M, N, K, blocksize, A.dtype) == Q4_ROUTE_FUSED:
        return q4_gemm_skinny(A, Wpacked, absmax, code, N, K, blocksize, out=out, workspace=workspace, bias=bias)
    W = q4_dequantize_blockwise(Wpacked, absmax, code, N * K, blocksize, out_dtype=A.dtype).view(N, K)
    A2 = A.view(M, K)
    if out is None:
        out = torch.empty((M, N), dtype=A.dtype, device=A.device)
    if bias is None:
        return torch.matmul(A2, W.t(), out=out)
    return torch.addmm(bias, A2, W.t(), out=out)


class Q4Layer:
    """A 4-bit linear layer bound once for repeated calls (a decode loop).

    Weights, code table, the activation buffer ``A`` [M, K], the output buffer,
    optional bias, workspace, stream and launch options are marshalled at
    construction.  Each call is then a single C call
    (``q4_gemm_skinny_ex`` / ``q4_gemm_skinny_bias``) with the prepared
    arguments.  It computes ``out = A . dequant(W)^T (+ bias)`` from whatever
    ``A`` holds at the time: write the next activations into ``A`` in place
    between calls."""

    def __init__(self, Wpacked: torch.Tensor, absmax: torch.Tensor, code: torch.Tensor, N: int, K: int,
                 blocksize: int, A: torch.Tensor, out: torch.Tensor | None = None, bias: torch.Tensor | None = None,
                 workspace: Workspace | None = None, stream: torch.cuda.Stream | None = None, **launch):
        M = A.shape[0] if A.dim() == 2 else 1
        act = _TORCH_TO_Q4[A.dtype]
        assert A.is_cuda and A.is_contiguous() and A.numel() == M * K
        self.A, self.Wpacked, self.absmax, self.code, self.bias = A, Wpacked, absmax, code, bias
        self.out = out if out is not None else torch.empty((M, N), dtype=A.dtype, device=A.device)
        assert self.out.dtype == A.dtype and self.out.numel() == M * N and self.out.is_contiguous()
        nbytes = _workspace_bytes(M, N, K, blocksize, act, tuple(sorted((k, v) for k, v in launch.items() if v)))
        self.workspace = workspace if workspace is not None else Workspace(A.device)
        ws = self.workspace.get(nbytes) if nbytes else None
        self.stream = stream if stream is not None else torch.cuda.current_stream(A.device)
        self._ov = overrides(**launch)
        P = ctypes.c_void_p
        head = (P(A.data_ptr()), P(Wpacked.data_ptr()), P(absmax.data_ptr()), P(code.data_ptr()))
        tail = (M, N, K, blocksize, act, P(self.out.data_ptr()), P(ws.data_ptr()) if ws is not None else None,
                ws.numel() if ws is not None else 0, P(self.stream.cuda_stream),
                ctypes.byref(self._ov) if self._ov is not None else None)
        if bias is None:
            self._fn, self._args = lib().q4_gemm_skinny_ex, head + tail
        else:
            assert bias.dtype == A.dtype and bias.numel() == N and bias.is_contiguous()
            self._fn, self._args = lib().q4_gemm_skinny_bias, head + (P(bias.data_ptr()),) + tail

    def __call__(self) -> torch.Tensor:
        rc = self._fn(*self._args)
        if rc != Q4_OK:
            raise Q4Error(rc, "q4_gemm_skinny")
        return self.out
