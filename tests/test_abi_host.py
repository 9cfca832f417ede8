"""Host-only checks of libq4's C ABI (no GPU work is enqueued here).

* the library loads and exports every function include/q4.h declares;
* argument validation answers before any CUDA call;
* the launch table and the stream-K work partition keep their invariants.
"""
import ctypes
import os

import pytest

from bit_weight_dequant_b200 import binding as b
from bit_weight_dequant_b200 import inputs

pytestmark = pytest.mark.skipif(not os.path.exists(b.LIB_PATH), reason="libq4.so not built")


def test_exports_every_declared_symbol():
    names = b.declared_functions()
    assert {"q4_quantize_blockwise", "q4_dequantize_blockwise", "q4_gemm_skinny"} <= set(names)
    L = b.lib()
    for n in names:
        assert hasattr(L, n), f"libq4.so does not export {n}"


def test_status_strings():
    for s in range(6):
        assert b.status_string(s).startswith("Q4_")
    assert b.status_string(99) == "unknown q4 status"


ALIGNED = ctypes.c_void_p(1 << 20)      # never dereferenced: every call below returns before launching
MISALIGNED = ctypes.c_void_p((1 << 20) + 4)


def test_quantize_validation():
    L = b.lib()
    q = L.q4_quantize_blockwise
    assert q(None, 16, 64, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_ERR_INVALID_ARG
    assert q(ALIGNED, -1, 64, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_ERR_INVALID_ARG
    for bs in (0, 16, 48, 8192):
        assert q(ALIGNED, 16, bs, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_ERR_INVALID_ARG
    assert q(MISALIGNED, 16, 64, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_ERR_MISALIGNED
    assert q(ALIGNED, 0, 64, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_OK   # empty input: no-op
    qx = L.q4_quantize_blockwise_ex
    assert qx(ALIGNED, 7, 16, 64, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_ERR_INVALID_ARG   # unknown weight type
    assert qx(MISALIGNED, b.Q4_BF16, 16, 64, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_ERR_MISALIGNED
    assert qx(ALIGNED, b.Q4_FP16, 0, 64, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_OK


def test_dequantize_validation():
    d = b.lib().q4_dequantize_blockwise
    assert d(ALIGNED, ALIGNED, ALIGNED, 16, 64, 3, ALIGNED, None) == b.Q4_ERR_INVALID_ARG
    assert d(ALIGNED, ALIGNED, ALIGNED, 16, 64, 0, None, None) == b.Q4_ERR_INVALID_ARG
    assert d(MISALIGNED, ALIGNED, ALIGNED, 16, 64, 0, ALIGNED, None) == b.Q4_ERR_MISALIGNED
    assert d(ALIGNED, ALIGNED, ALIGNED, 16, 64, 0, MISALIGNED, None) == b.Q4_ERR_MISALIGNED
    assert d(ALIGNED, ALIGNED, ALIGNED, 0, 64, 1, ALIGNED, None) == b.Q4_OK


def test_injected_launch_failure_reports_cuda_error(monkeypatch):
    monkeypatch.setenv("Q4_TEST_FAIL_LAUNCH", "1")
    L = b.lib()
    assert L.q4_quantize_blockwise(ALIGNED, 16, 64, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_ERR_CUDA
    assert L.q4_dequantize_blockwise(ALIGNED, ALIGNED, ALIGNED, 16, 64, 0, ALIGNED, None) == b.Q4_ERR_CUDA
    monkeypatch.setenv("Q4_TEST_FAIL_LAUNCH", "0")
    assert L.q4_quantize_blockwise(ALIGNED, 0, 64, ALIGNED, ALIGNED, ALIGNED, None) == b.Q4_OK


def test_gemm_validation_before_cuda():
    g = b.lib().q4_gemm_skinny
    args = [ALIGNED] * 4
    # (M, N, K, bs, dtype) -> status; all decided before the device is queried
    cases = {(129, 64, 4096, 64, 0): b.Q4_ERR_UNSUPPORTED,
             (1, 64, 4000, 64, 0): b.Q4_ERR_UNSUPPORTED,
             (17, 64, 4096, 64, 2): b.Q4_ERR_UNSUPPORTED,   # fp32 activations: M <= 16
             (-1, 64, 4096, 64, 0): b.Q4_ERR_INVALID_ARG,
             (1, -5, 4096, 64, 0): b.Q4_ERR_INVALID_ARG,
             (1, 64, 4096, 96, 0): b.Q4_ERR_INVALID_ARG,
             (1, 64, 4096, 64, 7): b.Q4_ERR_INVALID_ARG}
    for (M, N, K, bs, dt), want in cases.items():
        assert g(*args, M, N, K, bs, dt, ALIGNED, None, 0, None) == want, (M, N, K, bs, dt)
    assert g(None, *args[1:], 1, 64, 4096, 64, 0, ALIGNED, None, 0, None) == b.Q4_ERR_INVALID_ARG
    bias = b.lib().q4_gemm_skinny_bias
    assert bias(*args, None, 1, 64, 4096, 64, 0, ALIGNED, None, 0, None, None) == b.Q4_ERR_INVALID_ARG  # no bias
    assert bias(*args, ALIGNED, 129, 64, 4096, 64, 0, ALIGNED, None, 0, None, None) == b.Q4_ERR_UNSUPPORTED
    ex = b.lib().q4_gemm_skinny_ex
    assert ex(*args, 1, 64, 4096, 64, 0, ALIGNED, None, 0, None, b.overrides(math=4)) == b.Q4_ERR_INVALID_ARG
    # the tensor-memory kernel (M > 16) needs blocksize >= 64 and K % 256 == 0
    assert ex(*args, 32, 64, 4096, 32, 0, ALIGNED, None, 0, None, None) == b.Q4_ERR_UNSUPPORTED
    assert ex(*args, 32, 64, 4160, 64, 0, ALIGNED, None, 0, None, None) == b.Q4_ERR_UNSUPPORTED
    assert ex(*args, 12, 64, 4096, 64, 0, ALIGNED, None, 0, None, b.overrides(warps=16)) == b.Q4_ERR_UNSUPPORTED
    assert ex(*args, 1, 64, 4096, 64, 0, ALIGNED, None, 0, None, b.overrides(depth=7, loader=2)) == b.Q4_ERR_UNSUPPORTED
    assert ex(*args, 12, 64, 4096, 64, 0, ALIGNED, None, 0, None, b.overrides(loader=8)) == b.Q4_ERR_INVALID_ARG
    # the row-split kernel (loader 7): M <= 32 (blocksize >= 64 past 16; 33..64 in row chunks), 64-k units (blocksize 32 only with
    # K % 256 == 0), its own warp count
    assert ex(*args, 65, 64, 4096, 64, 0, ALIGNED, None, 0, None, b.overrides(loader=7)) == b.Q4_ERR_UNSUPPORTED
    assert ex(*args, 20, 64, 4096, 32, 0, ALIGNED, None, 0, None, b.overrides(loader=7)) == b.Q4_ERR_UNSUPPORTED
    assert ex(*args, 4, 64, 4160, 32, 0, ALIGNED, None, 0, None, b.overrides(loader=7)) == b.Q4_ERR_UNSUPPORTED
    assert ex(*args, 4, 64, 4096, 32, 0, ALIGNED, None, 0, None, b.overrides(loader=7, depth=3)) == b.Q4_ERR_UNSUPPORTED
    assert ex(*args, 4, 64, 4096, 64, 0, ALIGNED, None, 0, None, b.overrides(loader=7, warps=9)) == b.Q4_ERR_UNSUPPORTED
    # the CUDA-core kernel takes 16-bit activations on request, M <= 16
    assert ex(*args, 17, 64, 4096, 64, 0, ALIGNED, None, 0, None, b.overrides(math=2)) == b.Q4_ERR_UNSUPPORTED
    assert ex(*args, 4, 64, 4096, 64, 1, ALIGNED, None, 0, None, b.overrides(math=2, loader=2)) == b.Q4_ERR_UNSUPPORTED


@pytest.mark.parametrize("M,N,K", [(17, 4096, 4096), (32, 300, 1024), (31, 8192, 28672)])
def test_launch_table_m32(M, N, K):
    """17 <= M <= 32: the mma.sync kernel with 32-row tiles and 2-unit stages."""
    p = b.q4_gemm_plan(M, N, K, 64, num_sms=148)
    assert p["math"] == 1 and p["loader"] == 3 and p["rows_per_tile"] == 32 and p["m_pad"] == 32
    assert p["warps"] == 8 and p["depth"] == 6 and p["sub_block"] == 64
    tiles = -(-N // 32)
    assert p["tiles"] == tiles and p["units"] == tiles * (K // 64)
    assert p["workspace_bytes"] == 256 + 148 * 2 * 4096 + -(-tiles * 4 // 256) * 256
    # bs = 32 or (K / bs) % 4 != 0: the tensor-memory kernel's rules decide
    assert b.q4_gemm_plan(24, 256, 4096, 128, num_sms=148)["math"] == 1
    with pytest.raises(b.Q4Error):
        b.q4_gemm_plan(24, 256, 4096, 32, num_sms=148)


@pytest.mark.parametrize("M,N,K", [(33, 4096, 4096), (48, 300, 1024), (64, 28672, 8192)])
def test_launch_table_row_chunks(M, N, K):
    """33 <= M <= 64: row chunks of 32 on the mma.sync kernels; the plan is
    the first chunk's (the 32-row kernel), the workspace the largest chunk's."""
    p = b.q4_gemm_plan(M, N, K, 64, num_sms=148)
    p32 = b.q4_gemm_plan(32, N, K, 64, num_sms=148)
    prest = b.q4_gemm_plan(M - 32, N, K, 64, num_sms=148)
    assert p["math"] == 1 and p["loader"] == 3 and p["m_pad"] == 32
    assert {k: p[k] for k in p if k != "workspace_bytes"} == {k: p32[k] for k in p32 if k != "workspace_bytes"}
    assert p["workspace_bytes"] == max(p32["workspace_bytes"], prest["workspace_bytes"])


@pytest.mark.parametrize("M,N,K", [(65, 4096, 4096), (96, 300, 1024), (128, 8192, 28672)])
def test_launch_table_tcgen05(M, N, K):
    p = b.q4_gemm_plan(M, N, K, 64, num_sms=148)
    assert p["math"] == 3 and p["loader"] == 6 and p["rows_per_tile"] == 128 and p["sub_block"] == 64
    assert p["warps"] == 10  # producer, MMA issuer, two dequantizing warpgroups
    assert p["m_pad"] == (32 if M <= 32 else 64 if M <= 64 else 128)
    tiles = -(-N // 128)
    assert p["tiles"] == tiles and p["units"] == tiles * (K // 64)
    assert 1 <= p["ctas"] <= min(148, p["units"])
    slots = p["ctas"] * 2 * p["m_pad"] * 128 * 4
    assert p["workspace_bytes"] == 256 + 148 * 2 * 4096 + -(-tiles * 4 // 256) * 256 + slots


@pytest.mark.parametrize("M,N,K,bs", [(1, 8192, 28672, 64), (2, 300, 1024, 32), (3, 61, 1088, 64),
                                      (5, 10240, 8192, 64), (12, 1, 32, 32), (16, 5120, 16384, 4096)])
def test_launch_table_f32(M, N, K, bs):
    """fp32 activations: the CUDA-core kernel, units of R rows x 512 k."""
    import torch
    p = b.q4_gemm_plan(M, N, K, bs, act_dtype=torch.float32, num_sms=148)
    mp = 1 if M == 1 else 2 if M == 2 else 4 if M <= 4 else 8 if M <= 8 else 16
    assert p["math"] == 2 and p["sub_block"] == 512 and p["m_pad"] == mp and p["loader"] == 1
    R = p["rows_per_tile"]
    assert p["tiles"] == -(-N // R) and p["units"] == p["tiles"] * -(-K // 512)
    assert 1 <= p["ctas"] <= 148 and (p["ctas"] - 1) * p["warps"] < p["units"]
    # the pieces of every warp fit the fixed partial region: 2 slots of R x MP floats
    assert p["ctas"] * p["warps"] * 2 * R * mp * 4 <= 148 * 2 * 4096
    want_ws = 0 if p["units"] == 1 else 256 + 148 * 2 * 4096 + -(-p["tiles"] * 4 // 256) * 256
    assert p["workspace_bytes"] == want_ws


@pytest.mark.parametrize("M,N,K,ctas", [(1, 64, 16384, 0), (4, 24, 32768, 0), (2, 1000, 4096, 3), (1, 8, 512, 0),
                                        (16, 130, 8192, 5), (8, 9, 65536, 0), (1, 8192, 28672, 0)])
def test_f32_piece_bookkeeping(M, N, K, ctas):
    """The fp32 kernel's row-group pieces, replayed on the host with the
    exported partition: each (warp, slot) holds at most one group's piece,
    and the warps the finaliser sums (the non-empty ranges meeting the group,
    slot 0 where the group is the range's first) are exactly the writers."""
    import torch
    L = b.lib()
    p = b.q4_gemm_plan(M, N, K, 64, act_dtype=torch.float32, num_sms=148)
    ku, U = -(-K // 512), p["units"]
    W = (min(ctas, p["ctas"]) if ctas else p["ctas"]) * p["warps"]
    start = [L.q4_partition_start(U, W, w) for w in range(W + 1)]
    used = {}
    for w in range(W):
        ws, we = start[w], start[w + 1]
        for g in range(ws // ku, (we - 1) // ku + 1) if ws < we else ():
            g0, g1 = g * ku, g * ku + ku
            if ws <= g0 and we >= g1:
                continue
            key = (w, 0 if ws >= g0 else 1)
            assert key not in used
            used[key] = g
    by_group = {}
    for key, g in used.items():
        by_group.setdefault(g, []).append(key)
    for g in range(p["tiles"]):
        g0, g1 = g * ku, g * ku + ku
        cf, cl = L.q4_partition_owner(U, W, g0), L.q4_partition_owner(U, W, g1 - 1)
        summed = [(c, 0 if start[c] >= g0 else 1) for c in range(cf, cl + 1) if start[c] != start[c + 1]]
        assert sorted(by_group.get(g, [])) == (summed if len(summed) > 1 else [])


@pytest.mark.parametrize("wl", list(inputs.workloads()))
def test_launch_table_invariants(wl):
    for c in inputs.workloads()[wl].cases:
        if c.M > 16 or c.act == "fp32":
            continue  # tensor-memory and fp32 tables: test_launch_table_tcgen05, test_launch_table_f32
        p = b.q4_gemm_plan(c.M, c.N, c.K, c.blocksize, num_sms=148)
        assert p["math"] == 1
        assert p["m_pad"] == (8 if c.M <= 8 else 16)
        assert p["tiles"] == -(-c.N // p["rows_per_tile"])
        assert p["units"] == p["tiles"] * (c.K // p["sub_block"])
        assert 1 <= p["ctas"] <= min(148, p["units"])
        assert p["smem_bytes"] <= 227 * 1024
        tma_ok = c.blocksize >= 64 and (c.K // c.blocksize) % 4 == 0 and c.N * (c.K // 64) > 1
        # the row-split kernel also takes blocksize 32 when K is a multiple of its 256-k stage
        rows_ok = tma_ok or (c.blocksize == 32 and c.K % 256 == 0 and c.N * (c.K // 64) > 1)
        tiles, weights = -(-c.N // 64), c.N * c.K
        rows = rows_ok and not (c.K < 4096 and tiles > 4 * 148) and not (c.M >= 8 and weights >= 2**26)
        assert p["loader"] == (7 if rows else 2 if tma_ok else 1), (wl, c)
        assert p["sub_block"] == (64 if rows else min(c.blocksize, 64))
        if rows:
            # row-split kernel: 8-row groups over at most one CTA per SM, the
            # workspace is the 256-byte error header alone
            assert p["ctas"] == min(148, -(-c.N // 8)) and p["warps"] == 8 and p["rows_per_tile"] == 64
            assert p["workspace_bytes"] == 256 and p["depth"] >= 0
            continue
        # workspace: 2 slots of 4 KiB per SM, then one int per tile (256-B granules)
        want_ws = 0 if p["units"] == 1 else 256 + 148 * 2 * 4096 + -(-p["tiles"] * 4 // 256) * 256
        assert p["workspace_bytes"] == want_ws
        assert p["depth"] >= 1 and p["l2_prefetch"] in (1, 128, 256)
        if tma_ok:
            assert p["warps"] == 8 and p["depth"] == 2  # stream-K TMA kernel


@pytest.mark.parametrize("total,parts", [(1, 1), (1, 16), (7, 3), (40, 148), (4096, 148), (57344, 148),
                                         (155200, 148), (13, 16), (1000003, 2368)])
def test_partition_invariants(total, parts):
    L = b.lib()
    starts = [L.q4_partition_start(total, parts, p) for p in range(parts + 1)]
    assert starts[0] == 0 and starts[-1] == total
    sizes = [starts[p + 1] - starts[p] for p in range(parts)]
    assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1, "ranges must be balanced to one unit"
    probe = sorted({0, total - 1, total // 2, total // 3} | set(s for s in starts if s < total) |
                   set(s - 1 for s in starts if 0 < s <= total))
    for u in probe:
        p = L.q4_partition_owner(total, parts, u)
        assert starts[p] <= u < starts[p + 1], (u, p)
    assert L.q4_partition_owner(total, parts, total) == -1


def test_route_table():
    """Fused-vs-split advice: fused at M <= 16 (any dtype), at 17 <= M <= 32
    on the 32-row mma.sync kernel, and for the tcgen05 kernel's M <= 64 on
    layers of >= 2^26 weights; split for the rest and for everything the
    fused entry rejects."""
    import torch
    F, S = b.Q4_ROUTE_FUSED, b.Q4_ROUTE_SPLIT
    cases = {(1, 8192, 8192, 64, torch.bfloat16): F, (16, 5120, 5120, 64, torch.float16): F,
             (8, 5120, 17408, 32, torch.float32): F, (16, 5120, 5120, 64, torch.float32): F,
             (17, 5120, 5120, 64, torch.float32): S,                       # fp32 stops at M = 16
             (32, 5120, 17408, 64, torch.bfloat16): F, (64, 5120, 17408, 64, torch.bfloat16): F,
             (65, 5120, 17408, 64, torch.bfloat16): S, (128, 5120, 17408, 64, torch.bfloat16): S,
             (32, 5120, 5120, 64, torch.bfloat16): F, (17, 8192, 5120, 64, torch.float16): F,  # 32-row mma.sync
             (48, 5120, 5120, 64, torch.bfloat16): S, (48, 8192, 5120, 64, torch.bfloat16): S,
             (48, 8192, 8192, 64, torch.bfloat16): F,                      # exactly 2^26 weights
             (32, 5120, 17408, 32, torch.bfloat16): S,                     # both need blocksize >= 64
             (129, 8192, 8192, 64, torch.bfloat16): S, (4, 64, 4000, 64, torch.bfloat16): S}
    for (M, N, K, bs, dt), want in cases.items():
        assert b.q4_gemm_route(M, N, K, bs, dt) == want, (M, N, K, bs, dt)
    r = ctypes.c_int(-1)
    L = b.lib()
    assert L.q4_gemm_route(1, 64, 4096, 96, 0, ctypes.byref(r)) == b.Q4_ERR_INVALID_ARG
    assert L.q4_gemm_route(1, 64, 4096, 64, 0, None) == b.Q4_ERR_INVALID_ARG
    assert L.q4_gemm_route(-1, 64, 4096, 64, 0, ctypes.byref(r)) == b.Q4_ERR_INVALID_ARG
