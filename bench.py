"""Benchmark of the fused 4-bit dequantize + skinny GEMM on B200.

One step = one decode pass through the four 4-bit linear layers of a
70B-class transformer block at M = 1 (K8192/N10240, K8192/N28672,
K28672/N8192, K8192/N8192; blocksize 64, bf16 activations, normal-quantile
code table).  Metric: effective HBM bandwidth
    (M*K*2 + N*K/2 + 4*N*K/bs + M*N*2 bytes) / time
summed over the step, and its fraction of the measured B200 peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload decode70b|square4096|msweep|variants|aspect]

For N > 1 it runs under torchrun, one process per GPU, each GPU running the
same step on its own replica of the weights (the path has no exchange step:
"replicas only", weak scaling); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_weight_dequant_b200 import binding as q4  # noqa: E402
from bit_weight_dequant_b200 import inputs  # noqa: E402

METRIC = "fused 4-bit dequant-GEMM effective HBM GB/s and % of B200 peak, per M=1..16"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
CHUNK_STEPS = 100          # steps per captured CUDA graph


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs: STREAM-style copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


def gemm_kernel_hash() -> str:
    """Hash of the GEMM kernels' source with line comments and blank lines
    removed: a comment edit does not invalidate counters taken on the code."""
    h = hashlib.sha256()
    for f in ("q4_gemm.cu", "q4_rows.cu", "q4_device.cuh", "q4_plan.cuh"):
        with open(os.path.join(ROOT, "bit_weight_dequant_b200", "csrc", f), encoding="utf-8") as fh:
            for line in fh:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def kernel_name(plan: dict) -> str:
    """The GEMM kernel a launch-table entry runs."""
    if plan["math"] == 2:
        return "q4_gemm_f32_kernel"
    if plan["math"] == 3:
        return "q4_gemm_umma_kernel"
    return {1: "q4_gemm_mma_kernel", 2: "q4_gemm_tma_kernel", 3: "q4_gemm_tma_kernel",
            7: "q4_gemm_rows_kernel"}.get(plan["loader"], "q4_gemm_ws_kernel")


def ncu_traffic(workload: str):
    """DRAM bytes per launch of the GEMM kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "gemm_dram_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        if d.get("kernel_hash") != gemm_kernel_hash():
            return None
        return d.get("bytes_per_launch", {}).get(workload)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"q4_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

TORCH_ACT = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}


class Layer:
    """One 4-bit linear layer resident on the device, with its C-ABI call
    arguments prepared once (the timed loop only makes the call)."""

    def __init__(self, case: inputs.Case, seed: int, device, pdl: int = 2, launch: dict | None = None):
        self.case = case
        dt = TORCH_ACT[case.act]
        code = inputs.CODE_TABLES[case.table]()
        self.code = torch.from_numpy(code).to(device)
        W = inputs.weights_device(case.N, case.K, seed, device, case.outliers)
        self.packed, self.absmax = q4.q4_quantize_blockwise(W.reshape(-1), case.blocksize, self.code)
        del W
        torch.cuda.empty_cache()  # the fp32 weights were transient: hand their memory back
        self.A_host = inputs.activations(case.M, case.K, dt, seed).pin_memory()
        self.A = self.A_host.to(device)
        self.out = torch.empty((case.M, case.N), dtype=dt, device=device)
        self.out_host = torch.empty((case.M, case.N), dtype=dt).pin_memory()
        self.launch_kw = {k: v for k, v in (launch or {}).items() if v}
        self.ws_bytes = q4.q4_gemm_workspace_size(case.M, case.N, case.K, case.blocksize, dt, **self.launch_kw)
        self.ws = torch.zeros(max(self.ws_bytes, 16), dtype=torch.uint8, device=device)
        self.act = {"bf16": q4.Q4_BF16, "fp16": q4.Q4_FP16, "fp32": q4.Q4_FP32}[case.act]
        self.plan = q4.q4_gemm_plan(case.M, case.N, case.K, case.blocksize, dt)
        self.plan.update({k: v for k, v in self.launch_kw.items() if k in ("math", "loader")})
        self.rebind(self.A, self.out)
        # Decode-time weights are static model parameters: let each GEMM's
        # prologue and first weight copies overlap the previous kernel.
        self.pdl = pdl
        self._ov = q4.overrides(pdl=pdl, **self.launch_kw)
        self.bytes = case.algorithmic_bytes()

    def rebind(self, A: torch.Tensor, out: torch.Tensor):
        """Point the layer at (possibly shared) activation and output buffers."""
        import ctypes
        P = ctypes.c_void_p
        self.A, self.out = A, out
        c = self.case
        self._args = (P(self.A.data_ptr()), P(self.packed.data_ptr()), P(self.absmax.data_ptr()),
                      P(self.code.data_ptr()), c.M, c.N, c.K, c.blocksize, self.act,
                      P(self.out.data_ptr()), P(self.ws.data_ptr()), self.ws.numel())

    def launch(self, stream_handle):
        import ctypes
        rc = q4.lib().q4_gemm_skinny_ex(*self._args, ctypes.c_void_p(stream_handle),
                                        ctypes.byref(self._ov) if self._ov is not None else None)
        if rc != 0:
            raise q4.Q4Error(rc, "q4_gemm_skinny_ex")



def split_time_est_us(case: inputs.Case, peak_gbs: float) -> float:
    """Time at the HBM peak of the split path: read the packed weights and
    absmax, write the dequantized weights in the activation type (2 or 4
    bytes), read them back in a dense GEMM, plus A and C once."""
    nk = case.N * case.K
    e = 4 if case.act == "fp32" else 2
    b = nk * (0.5 + 4.0 / case.blocksize) + e * nk + e * nk + e * case.M * case.K + e * case.M * case.N
    return b / (peak_gbs * 1e3)


def crossover_estimates(layers, per_shape, peak_gbs: float) -> list:
    """Per weight shape measured at several M: the smallest M at which the
    split path's HBM-peak time undercuts the measured fused time, taken
    from the measured points or, past them, from a line through the last two."""
    return crossover_from_points([(L.case, ps["us_serialized"]) for L, ps in zip(layers, per_shape)], peak_gbs)


def crossover_from_points(points, peak_gbs: float) -> list:
    """crossover_estimates over (case, measured fused us) pairs."""
    by_shape = {}
    for c, us in points:
        if c.act != "bf16" or c.table != "normal" or c.outliers:
            continue
        by_shape.setdefault((c.N, c.K, c.blocksize), []).append((c.M, us, c))
    res = []
    for (N, K, bs), pts in by_shape.items():
        pts.sort(key=lambda x: x[0])
        if len(pts) < 2:
            continue
        est = None
        for M, t, c in pts:
            if t > split_time_est_us(c, peak_gbs):
                est = {"M": M, "how": "measured point"}
                break
        if est is None:
            (m1, t1, c1), (m2, t2, c2) = pts[-2], pts[-1]
            s_fused = (t2 - t1) / (m2 - m1)
            a2, b2 = split_time_est_us(c2, peak_gbs), 2 * (K + N) / (peak_gbs * 1e3)
            if s_fused > b2:
                m_star = m2 + (a2 - t2) / (s_fused - b2)
                est = {"M": round(m_star, 1), "how": "extrapolated (line through the last two measured M)"}
            else:
                est = {"M": None, "how": "fused time grows no faster than the split estimate: no crossover"}
        res.append({"shape": f"K{K} N{N} bs{bs}", "M_measured": [p[0] for p in pts], **est})
    return res


def measure_split_path(layers, device, stream, reps: int = 20) -> list:
    """Device time of dequantize (this library) + cuBLAS bf16 GEMM per layer:
    each half captured as a CUDA graph of `reps` launches, timed by events
    around its replay."""
    out = []
    for L in layers:
        c = L.case
        dt = L.A.dtype
        W = torch.empty((c.N, c.K), dtype=dt, device=device)
        Y = torch.empty((c.M, c.N), dtype=dt, device=device)
        deq = lambda: q4.q4_dequantize_blockwise(L.packed, L.absmax, L.code, c.N * c.K, c.blocksize, out=W.view(-1))
        mm = lambda: torch.matmul(L.A, W.t(), out=Y)
        times = []
        for fn in (deq, mm):
            with torch.cuda.stream(stream):
                for _ in range(3):
                    fn()
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(reps):
                    fn()
            best = float("inf")
            for _ in range(3):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
                stream.synchronize()
                best = min(best, e0.elapsed_time(e1) * 1e3 / reps)
            times.append(best)
            del g
        del W, Y
        out.append({"tag": c.tag, "dequant_us": round(times[0], 2), "gemm_us": round(times[1], 2),
                    "us": round(times[0] + times[1], 2), "timing": f"CUDA graph of {reps} launches per half, best of 3"})
    return out


CONFIGS = ("square4096", "decode70b", "msweep", "variants", "aspect")


def copies_for(weight_bytes: int) -> int:
    """Distinct weight copies a back-to-back timing cycles through so that
    the bytes it reads exceed three times the L2: max(2, ceil(3 L2 / bytes)),
    at most 64 and at most about 6 GB in all."""
    need = max(2, -(-3 * L2_BYTES // max(1, weight_bytes)))
    return int(max(1, min(need, 64, (6 << 30) // max(1, weight_bytes))))


def time_case(c, seed: int, device, stream, reps: int = 3):
    """Device time per launch of back-to-back fused GEMMs for one case (CUDA
    graph, dependent launch mode 2) through the C ABI, cycling over distinct
    weight copies so that the weights come from HBM, not L2 (the copies read
    more than 3x the L2).  Returns (us, copies, weight bytes)."""
    import ctypes
    P = ctypes.c_void_p
    L = q4.lib()
    dt = TORCH_ACT[c.act]
    code = torch.from_numpy(inputs.CODE_TABLES[c.table]()).to(device)
    W = inputs.weights_device(c.N, c.K, seed, device, c.outliers)
    packed, absmax = q4.q4_quantize_blockwise(W.reshape(-1), c.blocksize, code)
    del W
    wbytes = packed.numel() + 4 * absmax.numel()
    n = copies_for(wbytes)
    copies = [(packed, absmax)] + [(packed.clone(), absmax.clone()) for _ in range(n - 1)]
    A = inputs.activations(c.M, c.K, dt, seed).to(device)
    out = torch.empty((c.M, c.N), dtype=dt, device=device)
    ws_bytes = q4.q4_gemm_workspace_size(c.M, c.N, c.K, c.blocksize, dt)
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=device)
    act = {"bf16": q4.Q4_BF16, "fp16": q4.Q4_FP16, "fp32": q4.Q4_FP32}[c.act]
    ov = q4.overrides(pdl=2)
    args = [(P(A.data_ptr()), P(pk.data_ptr()), P(am.data_ptr()), P(code.data_ptr()), c.M, c.N, c.K,
             c.blocksize, act, P(out.data_ptr()), P(ws.data_ptr()), ws.numel()) for pk, am in copies]
    R = max(20, n)

    def run(s):
        for r in range(R):
            rc = L.q4_gemm_skinny_ex(*args[r % n], P(s.cuda_stream), ctypes.byref(ov))
            if rc != 0:
                raise q4.Q4Error(rc, "q4_gemm_skinny_ex")

    with torch.cuda.stream(stream):
        run(stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        run(torch.cuda.current_stream())
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        best = min(best, e0.elapsed_time(e1) * 1e3 / R)
    del g, copies, packed, absmax
    torch.cuda.empty_cache()
    return best, n, wbytes


# The smallest layer the row-split kernel takes (one 8-row group, one
# 256-k stage): timed like every case, its per-launch time is the fixed cost
# of one link in a chain of dependent launches, the floor for tiny layers.
FLOOR_CASE = inputs.Case(1, 8, 256, tag="floor")


def measure_latency_floor(device, stream) -> dict:
    us, _, _ = time_case(FLOOR_CASE, 12345, device, stream)
    plan = q4.q4_gemm_plan(FLOOR_CASE.M, FLOOR_CASE.N, FLOOR_CASE.K, FLOOR_CASE.blocksize, torch.bfloat16)
    log(f"latency floor (M1 N8 K256): {us:.2f} us")
    return {"case": "M1 N8 K256 bs64 bf16", "us": round(us, 3), "kernel": kernel_name(plan),
            "how": "per-launch time of the smallest layer, timed like per_config: the fixed cost of one "
                   "dependent launch in a chain"}


def measure_configs(device, peak: float, stream, reps: int = 3) -> list:
    """Every case of the five configurations, one at a time (time_case)."""
    rows = []
    for name in CONFIGS:
        wl = inputs.workloads()[name]
        for i, c in enumerate(wl.cases):
            seed = inputs.seed_for(wl.index, c.M) + i
            dt = TORCH_ACT[c.act]
            best, n, wbytes = time_case(c, seed, device, stream, reps)
            plan = q4.q4_gemm_plan(c.M, c.N, c.K, c.blocksize, dt)
            b = c.algorithmic_bytes()
            gbs = b / (best * 1e-6) / 1e9
            e = 4 if c.act == "fp32" else 2
            rows.append({
                "config": name, "case": c.tag, "M": c.M, "N": c.N, "K": c.K, "blocksize": c.blocksize, "act": c.act,
                "table": c.table, "outliers": c.outliers, "us": round(best, 3), "GB/s": round(gbs, 1),
                "frac_of_peak": round(gbs / peak, 4), "bytes": b,
                "bf16_weight_roofline_us": round((c.M * c.K * e + 2 * c.N * c.K + c.M * c.N * e) / (peak * 1e3), 3),
                "t_split_est_us": round(split_time_est_us(c, peak), 3),
                "weight_copies": n, "l2": "from HBM" if n * wbytes > L2_BYTES else "fits L2 (not HBM-bound)",
                "kernel": kernel_name(plan), "loader": plan["loader"], "ctas": plan["ctas"]})
            log(f"per_config {name} {c.tag}: {best:.2f} us, {gbs:.0f} GB/s, {n} copies, {kernel_name(plan)}")
    return rows


def oracle_per_config(rows: list, seconds: float) -> None:
    """The oracle (as it stands) on a sample of each per_config case's
    weight rows, one thread and all of this process's cores (row slices on
    threads; the C oracle releases the GIL), scaled to the full layer."""
    import concurrent.futures as cf
    import oracle
    cores = len(os.sched_getaffinity(0))
    budget = seconds / max(1, len(rows))
    with cf.ThreadPoolExecutor(max_workers=cores) as pool:
        for r in rows:
            c = inputs.Case(r["M"], r["N"], r["K"], r["blocksize"], r["act"], r["table"], r["outliers"], r["case"])
            per_row = _oracle_time(c, 2, _oracle_sample(c, 2, 1)) / 2
            nrows = int(max(cores, min(c.N, 4096, budget / max(per_row, 1e-9))))
            prep = _oracle_sample(c, nrows, 1)
            t1 = _oracle_time(c, nrows, prep)
            a, packed, absmax, code = prep
            rb, ab = c.K // 2, c.K // c.blocksize
            bounds = [nrows * t // cores for t in range(cores + 1)]

            def part(t):
                lo, hi = bounds[t], bounds[t + 1]
                if hi <= lo:
                    return 0.0
                sub = (a, packed[lo * rb:hi * rb], absmax[lo * ab:hi * ab], code)
                return _oracle_time(c, hi - lo, sub)

            t0 = time.perf_counter()
            list(pool.map(part, range(cores)))
            tall = time.perf_counter() - t0
            r["oracle_us_1core"] = round(t1 / nrows * c.N * 1e6, 1)
            r["oracle_us_all_cores"] = round(tall / nrows * c.N * 1e6, 1)
            r["oracle_cores"] = cores
            r["oracle_sample_rows"] = nrows


def run_e2e(layers, device, steps: int, world: int) -> float:
    """Wall-clock seconds (max over ranks) for `steps` pipelined steps through
    Q4Layer, with every step's H2D and D2H copies."""
    comp = torch.cuda.current_stream(device)
    h2d_stream, d2h_stream = torch.cuda.Stream(device), torch.cuda.Stream(device)
    sets = []
    for _ in range(2):
        host_in, dev_in, host_out, dev_out, views = step_buffers(layers, device)
        pubs = [q4.Q4Layer(L.packed, L.absmax, L.code, L.case.N, L.case.K, L.case.blocksize, A, out=out,
                           stream=comp, pdl=L.pdl) for L, (A, out) in zip(layers, views)]
        sets.append((host_in, dev_in, host_out, dev_out, pubs))
    ev = {k: [torch.cuda.Event(), torch.cuda.Event()] for k in ("h2d", "comp", "d2h")}

    def step(i):
        b = i % 2
        host_in, dev_in, host_out, dev_out, pubs = sets[b]
        with torch.cuda.stream(h2d_stream):
            if i >= 2:
                h2d_stream.wait_event(ev["comp"][b])  # step i-2's kernels have read this set's inputs
            dev_in.copy_(host_in, non_blocking=True)
            ev["h2d"][b].record(h2d_stream)
        comp.wait_event(ev["h2d"][b])
        if i >= 2:
            comp.wait_event(ev["d2h"][b])  # step i-2's outputs are back on the host
        for pub in pubs:
            pub()
        ev["comp"][b].record(comp)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(ev["comp"][b])
            host_out.copy_(dev_out, non_blocking=True)
            ev["d2h"][b].record(d2h_stream)

    step(0)
    step(1)  # untimed pass through both sets
    torch.cuda.synchronize()
    barrier(world)
    t0 = time.perf_counter()
    for i in range(steps):
        step(i)
    torch.cuda.synchronize()
    return max_over_ranks(time.perf_counter() - t0, world, device)


def step_buffers(layers, device):
    """One pinned host buffer and one device buffer for all of a step's
    activations (16-byte aligned slots), likewise for the outputs, filled with
    the layers' activations.  Returns (host_in, dev_in, host_out, dev_out,
    [(A view, out view) per layer])."""
    def slots(sizes):
        offs, tot = [], 0
        for nb in sizes:
            offs.append(tot)
            tot += (nb + 15) // 16 * 16
        return offs, max(tot, 16)
    isz = [L.A_host.numel() * L.A_host.element_size() for L in layers]
    osz = [L.out.numel() * L.out.element_size() for L in layers]
    ioff, itot = slots(isz)
    ooff, otot = slots(osz)
    host_in = torch.zeros(itot, dtype=torch.uint8).pin_memory()
    dev_in = torch.zeros(itot, dtype=torch.uint8, device=device)
    host_out = torch.zeros(otot, dtype=torch.uint8).pin_memory()
    dev_out = torch.zeros(otot, dtype=torch.uint8, device=device)
    views = []
    for L, io, ni, oo, no in zip(layers, ioff, isz, ooff, osz):
        dt = L.A_host.dtype
        host_in[io:io + ni].view(dt).view(L.A_host.shape).copy_(L.A_host)
        A = dev_in[io:io + ni].view(dt).view(L.A_host.shape)
        A.copy_(L.A_host)
        views.append((A, dev_out[oo:oo + no].view(dt).view(L.out.shape)))
    return host_in, dev_in, host_out, dev_out, views


def bind_step_io(layers, device):
    """Place every layer's activations in one pinned host buffer mirrored by
    one device buffer, and likewise the outputs (16-byte aligned slots), so
    that a step moves all of its inputs with one H2D copy and all of its
    results with one D2H copy.  Returns (host_in, dev_in, host_out, dev_out)."""
    def slots(sizes):
        offs, tot = [], 0
        for nb in sizes:
            offs.append(tot)
            tot += (nb + 15) // 16 * 16
        return offs, max(tot, 16)
    isz = [L.A_host.numel() * L.A_host.element_size() for L in layers]
    osz = [L.out.numel() * L.out.element_size() for L in layers]
    ioff, itot = slots(isz)
    ooff, otot = slots(osz)
    host_in = torch.zeros(itot, dtype=torch.uint8).pin_memory()
    dev_in = torch.zeros(itot, dtype=torch.uint8, device=device)
    host_out = torch.zeros(otot, dtype=torch.uint8).pin_memory()
    dev_out = torch.zeros(otot, dtype=torch.uint8, device=device)
    for L, io, ni, oo, no in zip(layers, ioff, isz, ooff, osz):
        dt = L.A_host.dtype
        h = host_in[io:io + ni].view(dt).view(L.A_host.shape)
        h.copy_(L.A_host)
        L.A_host = h
        A = dev_in[io:io + ni].view(dt).view(h.shape)
        A.copy_(h)
        out = dev_out[oo:oo + no].view(dt).view(L.out.shape)
        L.out_host = host_out[oo:oo + no].view(dt).view(L.out.shape)
        L.rebind(A, out)
    return host_in, dev_in, host_out, dev_out


def run_ours(args, world, rank, local):
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    wl = inputs.workloads()[args.workload]
    peak, peak_src = hbm_peak()
    cases = [(i, c) for i, c in enumerate(wl.cases) if not args.only or c.tag in args.only.split(",")]
    if not cases:
        raise SystemExit(f"--only {args.only!r} matches no case of {args.workload}")
    launch = {"loader": args.loader, "depth": args.depth, "l2_prefetch": args.l2_ahead, "ctas": args.ctas,
              "math": args.math}
    layers = [Layer(c, inputs.seed_for(wl.index, c.M) + i, device, args.pdl, launch) for i, c in cases]
    host_in, dev_in, host_out, dev_out = bind_step_io(layers, device)
    torch.cuda.synchronize()
    step_bytes = sum(L.bytes for L in layers)
    stream = torch.cuda.Stream(device)

    # Warm-up (eager launches through the C ABI; sets kernel attributes).
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            for L in layers:
                L.launch(stream.cuda_stream)
    stream.synchronize()

    # Timed region: CUDA graphs of CHUNK steps of back-to-back GEMM launches
    # (no event nodes between kernels, so dependent launches can overlap).
    def capture(nsteps, per_kernel_events=False):
        g = torch.cuda.CUDAGraph()
        evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(nsteps * len(layers) + 1)] \
            if per_kernel_events else []
        with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
            s = torch.cuda.current_stream()
            if evs:
                evs[0].record(s)
            k = 1
            for _ in range(nsteps):
                for L in layers:
                    L.launch(s.cuda_stream)
                    if evs:
                        evs[k].record(s)
                    k += 1
        return g, evs

    chunk = min(CHUNK_STEPS, args.steps)
    g_main, _ = capture(chunk)
    nfull, rem = divmod(args.steps, chunk)
    g_rem, _ = capture(rem) if rem else (None, None)
    g_main.replay()           # graph warm-up (not timed)
    stream.synchronize()

    uuid = str(getattr(torch.cuda.get_device_properties(device), "uuid", ""))
    sampler = ClockSampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or str(local)))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    # The sampler needs a moment to start: keep the GPU on untimed replays of
    # the same graph meanwhile (about 0.3 s), so the timed steps do not start
    # from an idle GPU.
    sampler.start()
    t_warm = time.time()
    while time.time() - t_warm < 0.3:
        with torch.cuda.stream(stream):
            g_main.replay()
        stream.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(nfull):
            g_main.replay()
        if g_rem is not None:
            g_rem.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(world)
    ms_total = e0.elapsed_time(e1)
    ms_total = max_over_ranks(ms_total, world, device)
    ms_step = ms_total / args.steps
    value = world * step_bytes * args.steps / (ms_total * 1e-3) / 1e9
    # Every launch in the timed region is the GEMM kernel: its average launch
    # duration is the region's device time over the launches.
    launches = args.steps * len(layers)
    achieved = step_bytes * args.steps / (ms_total * 1e-3) / 1e9
    del g_main, g_rem

    # Per-shape breakdown (outside the timed region): one event after every
    # launch, which also serialises the kernels.
    g_b, ev_b = capture(min(chunk, 50), per_kernel_events=True)
    with torch.cuda.stream(stream):
        g_b.replay()
        g_b.replay()
    torch.cuda.synchronize()
    per = {L.case.tag: [] for L in layers}
    for k in range((len(ev_b) - 1)):
        per[layers[k % len(layers)].case.tag].append(ev_b[k].elapsed_time(ev_b[k + 1]))
    del g_b
    per_shape = []
    for L in layers:
        us = statistics.mean(per[L.case.tag]) * 1e3
        gbs = L.bytes / (us * 1e-6) / 1e9
        bf16_roof_us = (L.case.M * L.case.K * 2 + 2 * L.case.N * L.case.K + L.case.M * L.case.N * 2) / (peak * 1e3)
        per_shape.append({"shape": f"M{L.case.M} K{L.case.K} N{L.case.N} bs{L.case.blocksize}", "tag": L.case.tag,
                          "us_serialized": round(us, 3), "GB/s": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4),
                          "bytes": L.bytes, "bf16_weight_roofline_us": round(bf16_roof_us, 3),
                          "t_split_est_us": round(split_time_est_us(L.case, peak), 3),
                          "plan": {k: L.plan[k] for k in ("ctas", "warps", "depth", "loader", "m_pad", "units")}})

    # The split path the fused kernel competes with (opt-in): the library's
    # dequantize kernel into a bf16 weight matrix, then a cuBLAS bf16 GEMM.
    split_path = measure_split_path(layers, device, stream) if args.split_path else None


    # End to end through the public Python API: per step, one H2D copy of all
    # of the step's activations from pinned memory, the layer calls, one D2H
    # copy of all of its outputs.  Two buffer sets alternate between steps and
    # the copies run on their own streams, so that step i+1's inputs and step
    # i-1's outputs move while step i computes (event-ordered: a set is
    # refilled only after the kernels that read it, and its outputs are
    # overwritten only after they were copied back).
    e2e_steps = 0 if args.no_e2e else max(1, min(args.steps, 2000))
    e2e_value = None
    if e2e_steps:
        e2e_s = run_e2e(layers, device, e2e_steps, world)
        e2e_value = world * step_bytes * e2e_steps / e2e_s / 1e9
    h2d = host_in.numel()
    d2h = host_out.numel()

    # Every case of the five configurations, each timed from HBM (outside
    # the timed region; single-GPU runs).
    total_weight_bytes = sum(L.packed.numel() + 4 * L.absmax.numel() for L in layers)
    per_config = latency_floor = None
    if not args.no_per_config and world == 1:
        for L in layers:  # hand the step's weights back before the per-case layers are built
            L.packed = L.absmax = None
        torch.cuda.empty_cache()
        per_config = measure_configs(device, peak, stream)
        latency_floor = measure_latency_floor(device, stream)

    if rank != 0:
        return None
    cpu = cpu_baseline(wl, args.cpu_seconds) if (world == 1 and not args.no_cpu_baseline) else None
    if per_config is not None and not args.no_cpu_baseline:
        oracle_per_config(per_config, args.cpu_seconds)
    act_dtype = "+".join(sorted({ {"bf16": "bf16", "fp16": "f16", "fp32": "f32"}[L.case.act] for L in layers}))
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": act_dtype, "data": "synthetic",
        "config": {"workload": wl.name + (f" [only {args.only}]" if args.only else ""), "M": sorted({c.M for c in wl.cases}), "blocksize": 64,
                   "code_table": "normal-quantile", "activations": f"{act_dtype} ~N(0,1)", "weights": "N(0,0.02^2) fp32 -> 4-bit",
                   "l2": (f"inputs larger than L2: {total_weight_bytes / 1e6:.0f} MB of packed weights per step "
                          f"vs {L2_BYTES / 2**20:.0f} MiB L2, no flush" if total_weight_bytes * args.steps > 3 * L2_BYTES
                          and total_weight_bytes > L2_BYTES else
                          f"{total_weight_bytes / 1e6:.1f} MB of packed weights per step fit the "
                          f"{L2_BYTES / 2**20:.0f} MiB L2: this step's figure is L2-fed, not HBM-bound "
                          f"(per_config times every case from HBM)"),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "timing": f"CUDA graphs of {chunk} steps, CUDA events, device time",
                   "dependent_launch": args.pdl},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": ncu_traffic(args.workload),
                     "peak_source": peak_src, "kernel": "+".join(sorted({kernel_name(L.plan) for L in layers})),
                     "per_unit": "0.5 B per weight (codes) + 4/bs B (absmax) + A and C once",
                     "duration": "average launch = timed-region device time / launches (all launches are this kernel)"},
        "per_shape": per_shape,
        "crossover": crossover_estimates(layers, per_shape, peak) or (
            crossover_from_points([(inputs.Case(r["M"], r["N"], r["K"], r["blocksize"], r["act"], r["table"],
                                                r["outliers"]), r["us"]) for r in per_config
                                   if r["config"] == "msweep"], peak) if per_config else []),
        "per_config": per_config,
        "latency_floor": latency_floor,
        "split_path": split_path if args.split_path else None,
        "e2e": {"value": round(e2e_value, 2) if e2e_value else None, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "api": "bit_weight_dequant_b200.Q4Layer per layer (bound once; each call is one ctypes call into "
                       "the libq4 C ABI), wall clock; copies on their own streams, two buffer sets "
                       "alternating so a step's copies overlap the neighbouring steps' kernels"},
        "gpu_launches": launches,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    return line


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg and the reference arm)
# ---------------------------------------------------------------------------

SAMPLE_ROWS_MAX = 1024


def _oracle_sample(case: inputs.Case, rows: int, seed: int):
    """The first `rows` weight rows of a layer, quantized by the oracle, and
    its activations (bf16 bit patterns)."""
    import oracle
    code = inputs.CODE_TABLES[case.table]()
    W = inputs.weight_rows(case.K, seed, 0, rows, case.outliers)
    packed, absmax = oracle.quantize(W, case.blocksize, code)
    if case.act == "fp32":
        return (inputs.activations_fp32(case.M, case.K, seed), packed, absmax, code)
    A = inputs.activations(case.M, case.K, TORCH_ACT[case.act], seed)
    abits = A.view(torch.int16).numpy().view(np.uint16)
    return (abits, packed, absmax, code)


def _oracle_time(case, rows, prepared):
    import oracle
    a, packed, absmax, code = prepared
    t0 = time.perf_counter()
    if case.act == "fp32":
        oracle.gemm_f32(a, packed, absmax, code, case.M, rows, case.K, case.blocksize, want_s=False)
    else:
        oracle.gemm(a, oracle.BF16 if case.act == "bf16" else oracle.FP16, packed, absmax, code, case.M, rows,
                    case.K, case.blocksize, want_s=False)
    return time.perf_counter() - t0


def _oracle_parallel(case, rows, prepared, pool, cores) -> float:
    """Seconds for the oracle's GEMM over `rows` weight rows split into
    `cores` row slices run on threads (the C oracle releases the GIL)."""
    a, packed, absmax, code = prepared
    rb, ab = case.K // 2, case.K // case.blocksize
    bounds = [rows * t // cores for t in range(cores + 1)]

    def part(t):
        lo, hi = bounds[t], bounds[t + 1]
        return _oracle_time(case, hi - lo, (a, packed[lo * rb:hi * rb], absmax[lo * ab:hi * ab], code)) if hi > lo else 0.0

    t0 = time.perf_counter()
    list(pool.map(part, range(cores)))
    return time.perf_counter() - t0


def cpu_baseline(wl, seconds: float) -> dict:
    """The oracle's GEMM as it stands (plain C loops) on the first rows of
    each layer: on all of this process's cores (row slices on threads; the
    value) and on one thread, called repeatedly for about `seconds` in all."""
    import concurrent.futures as cf
    cores = len(os.sched_getaffinity(0))
    res = {}
    desc = []
    with cf.ThreadPoolExecutor(max_workers=cores) as pool:
        for mode, n_thr in (("1", 1), ("all", cores)):
            tot_bytes = tot_s = 0.0
            for i, c in enumerate(wl.cases):
                rows = min(c.N, SAMPLE_ROWS_MAX * n_thr)
                prep = _oracle_sample(c, rows, inputs.seed_for(wl.index, c.M) + i)
                spent, reps = 0.0, 0
                while reps == 0 or spent < seconds / 2 / len(wl.cases):
                    spent += _oracle_time(c, rows, prep) if n_thr == 1 else _oracle_parallel(c, rows, prep, pool, n_thr)
                    reps += 1
                tot_s += spent
                tot_bytes += reps * inputs.Case(c.M, rows, c.K, c.blocksize, act=c.act).algorithmic_bytes()
                if mode == "all":
                    desc.append(f"{reps}x {rows}/{c.N} rows of K{c.K}N{c.N}")
            res[mode] = tot_bytes / tot_s / 1e9
    return {"value": round(res["all"], 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "single_thread_value": round(res["1"], 4),
            "sample": "; ".join(desc) + f" per all-core run (M={wl.cases[0].M}; row slices on {cores} threads, "
                      f"and the same layers one thread at a time; about {seconds:.0f} s in all)"}


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle as it stands, each step a bounded
    sample of the same workload (the first rows of each layer), sized so the
    whole run takes about --reference-seconds."""
    if rank != 0:
        return None
    import concurrent.futures as cf
    wl = inputs.workloads()[args.workload]
    cores = len(os.sched_getaffinity(0))
    pool = cf.ThreadPoolExecutor(max_workers=cores)
    per_row = []
    for i, c in enumerate(wl.cases):
        prep = _oracle_sample(c, 2, inputs.seed_for(wl.index, c.M) + i)
        per_row.append(_oracle_time(c, 2, prep) / 2)
    step_s = args.reference_seconds / max(1, args.steps + args.warmup)
    rows = [int(max(cores, min(c.N, SAMPLE_ROWS_MAX * cores, cores * step_s / len(wl.cases) / max(pr, 1e-9))))
            for c, pr in zip(wl.cases, per_row)]
    preps = [_oracle_sample(c, r, inputs.seed_for(wl.index, c.M) + i) for i, (c, r) in enumerate(zip(wl.cases, rows))]
    for _ in range(args.warmup):
        for c, r, p in zip(wl.cases, rows, preps):
            _oracle_parallel(c, r, p, pool, cores)
    tot_s = 0.0
    for _ in range(args.steps):
        for c, r, p in zip(wl.cases, rows, preps):
            tot_s += _oracle_parallel(c, r, p, pool, cores)
    pool.shutdown()
    step_bytes = sum(inputs.Case(c.M, r, c.K, c.blocksize, act=c.act).algorithmic_bytes()
                     for c, r in zip(wl.cases, rows))
    value = step_bytes * args.steps / tot_s / 1e9
    sample = "; ".join(f"{r}/{c.N} rows of K{c.K}N{c.N}" for c, r in zip(wl.cases, rows))
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_s / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "parallelism": f"CPU oracle, row slices on {cores} threads"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample + " per step"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode70b", choices=list(inputs.workloads()))
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--no-per-config", action="store_true", help="skip timing every case of the five configurations")
    ap.add_argument("--only", default="", help="comma-separated case tags of the workload to run (profiling)")
    ap.add_argument("--split-path", action="store_true",
                    help="also time the split path (dequantize kernel + cuBLAS bf16 GEMM) per layer")
    ap.add_argument("--loader", type=int, default=0, help="launch-table override: GEMM loader (measurement)")
    ap.add_argument("--depth", type=int, default=0, help="launch-table override: depth (measurement)")
    ap.add_argument("--l2-ahead", type=int, default=0, help="launch-table override: l2_prefetch (measurement)")
    ap.add_argument("--ctas", type=int, default=0, help="launch-table override: CTAs (measurement)")
    ap.add_argument("--math", type=int, default=0, choices=[0, 1, 2, 3],
                    help="launch-table override: math (2: the CUDA-core kernel; measurement)")
    ap.add_argument("--pdl", type=int, default=2, choices=[0, 1, 2],
                    help="programmatic dependent launch mode for the GEMMs (2: static weights read early)")
    args = ap.parse_args()
    if args.warmup < 3:
        log("note: warm-up raised to 3 steps (minimum)")
        args.warmup = 3
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            line = run_reference(args, world, rank)
        else:
            line = run_ours(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
