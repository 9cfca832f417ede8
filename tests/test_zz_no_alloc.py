"""The allocation-free GEMM entry point, q4_gemm_skinny_noalloc.

Some callers cannot allocate device memory -- code running while a stream is
captured into a CUDA graph, runtimes that forbid allocations after start-up,
plugin hosts with no allocator to offer -- so they cannot hand
q4_gemm_skinny its workspace.  This entry point uses a scratch array built
into the library instead.  The test calls it through the C ABI, twice in a
row (the second call finds the first call's leftovers in the shared array),
and checks each result against the regular entry point's on the same inputs,
within the tolerance the parity tests use.  It lives in a file of its own
that pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bit_weight_dequant_b200 import binding as q4
from bit_weight_dequant_b200 import inputs
from parity import bits_of

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


# (2, 40000, 2048) runs on the stream-K kernel, whose tile counters the entry
# point clears; the others need the 256-byte header alone.
@pytest.mark.parametrize("M,N,K", [(1, 1000, 4096), (5, 3000, 2560), (16, 700, 1024), (2, 40000, 2048)])
def test_noalloc_matches_regular_entry_point_twice(cuda_device, M, N, K):
    bs = 64
    code = inputs.code_normal_quantile()
    packed, absmax = oracle.quantize(inputs.weights(N, K, 4242 + N), bs, code)
    A = inputs.activations(M, K, torch.bfloat16, 4243).to(cuda_device)
    P, Am, C = (torch.from_numpy(x).to(cuda_device) for x in (packed, absmax, code))
    ref = q4.q4_gemm_skinny(A, P, Am, C, N, K, bs)
    y, S = oracle.gemm(bits_of(A), oracle.BF16, packed, absmax, code, M, N, K, bs)
    tol = oracle.gemm_tolerance(y, S, oracle.BF16)
    ref_v = oracle.decode(bits_of(ref).reshape(-1), oracle.BF16).reshape(M, N)
    L = q4.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    for call in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        rc = L.q4_gemm_skinny_noalloc(_ptr(A), _ptr(P), _ptr(Am), _ptr(C), M, N, K, bs, q4.Q4_BF16, _ptr(out),
                                      stream)
        assert rc == q4.Q4_OK, q4.status_string(rc)
        torch.cuda.synchronize()
        got = oracle.decode(bits_of(out).reshape(-1), oracle.BF16).reshape(M, N)
        assert np.all(np.abs(got - ref_v) <= tol), f"call {call}: differs from q4_gemm_skinny"
        assert np.all(np.abs(got - y) <= tol), f"call {call}: outside the oracle tolerance"


@pytest.mark.parametrize("M,N,K", [(1, 3000, 4096), (9, 700, 1024)])
def test_noalloc_fp32_activations_twice(cuda_device, M, N, K):
    """The CUDA-core kernel (fp32 activations) through the built-in array,
    whose row-group counters the entry point clears before each call."""
    bs = 64
    code = inputs.code_normal_quantile()
    packed, absmax = oracle.quantize(inputs.weights(N, K, 4343 + N), bs, code)
    a = inputs.activations_fp32(M, K, 4344)
    A = torch.from_numpy(a).to(cuda_device)
    P, Am, C = (torch.from_numpy(x).to(cuda_device) for x in (packed, absmax, code))
    y, S = oracle.gemm_f32(a, packed, absmax, code, M, N, K, bs)
    L = q4.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream(cuda_device).cuda_stream)
    for call in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.float32, device=cuda_device)
        rc = L.q4_gemm_skinny_noalloc(_ptr(A), _ptr(P), _ptr(Am), _ptr(C), M, N, K, bs, q4.Q4_FP32, _ptr(out),
                                      stream)
        assert rc == q4.Q4_OK, q4.status_string(rc)
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - y) <= 1e-2 * S + np.spacing(np.abs(y).astype(np.float32)).astype(np.float64)), \
            f"call {call}: outside the oracle tolerance"


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    # the workspace grows with the tile count: find an N whose need exceeds the array
    limit = 2 << 20
    N = 64
    while q4.q4_gemm_workspace_size(1, N, 64, 64, torch.bfloat16) <= limit:
        N *= 2
    L = q4.lib()
    dummy = torch.zeros(16, device=cuda_device)
    rc = L.q4_gemm_skinny_noalloc(_ptr(dummy), _ptr(dummy), _ptr(dummy), _ptr(dummy), 1, N, 64, 64, q4.Q4_BF16,
                                  _ptr(dummy), None)
    assert rc == q4.Q4_ERR_WORKSPACE
