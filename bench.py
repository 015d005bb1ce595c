"""Benchmark of the NVFP4 W4A16 linear layer on B200 (one JSON line on stdout).

One step = one pass of every kernel of the hot path over the 27B-class layer
(hidden 5120, MLP 17408), inputs resident in HBM:
  * quantize: nvfp4_amax + nvfp4_quantize of a BF16 [17408, 5120] N(0, 0.02) tensor
  * quantize_mse: the same with the micro-scale search (nvfp4_quantize_mse)
  * gemv:     batch-1 decode GEMV, NVFP4 W [17408, 5120] (headline: HBM GB/s)
  * gemm_m32: 32-user decode GEMM, X [32, 5120]
  * gemm_m512: 512-token prefill GEMM, X [512, 5120]
  * gemv_down: the MLP down projection W [5120, 17408], split-K decode GEMV
Each kernel row is a CUDA graph of several launches over rotating weight copies
(more bytes than the 126 MB L2 between two reads of one copy), timed with CUDA
events on the launching stream.  `value` is the decode GEMV's algorithmic HBM
throughput (weight nibbles + scales + x + y + g per launch / launch time), summed
over ranks; every other kernel is reported under "kernels".

--impl reference times the CPU oracle (test infrastructure) on the same
workload: a bounded sample of decode-GEMV rows per step on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

HIDDEN, MLP = 5120, 17408
METRIC = "NVFP4 W4A16 GEMV HBM GB/s (frac of peak); GEMM TFLOP/s at M=32/512"
WORKLOAD = "decode GEMV NVFP4 W [N=17408, K=5120] x BF16 [1, 5120] (27B-class MLP layer)"


def gemv_bytes(N: int, K: int) -> int:
    """Algorithmic bytes of one decode GEMV: nibbles + scales + x + y + g."""
    return N * K // 2 + N * K // 16 + 2 * K + 2 * N + 4


def gemm_bytes(M: int, N: int, K: int) -> int:
    return N * K // 2 + N * K // 16 + 2 * M * K + 2 * M * N + 4


def quantize_bytes(N: int, K: int) -> int:
    """amax pass (read W) + quantize pass (read W, write q and s)."""
    return 2 * (2 * N * K) + N * K // 2 + N * K // 16


def mx_gemv_bytes(N: int, K: int) -> int:
    """MXFP4 decode GEMV: nibbles + one UE8M0 byte per 32 + x + y (no tensor scale)."""
    return N * K // 2 + N * K // 32 + 2 * K + 2 * N


def mx_quantize_bytes(N: int, K: int) -> int:
    """One pass: read W, write q and s (the scales need no tensor amax)."""
    return 2 * N * K + N * K // 2 + N * K // 32


def w4a4_gemm_bytes(M: int, N: int, K: int) -> int:
    """W4A4 GEMM kernel alone: weight nibbles + scales, activation nibbles +
    scales, Y, g and x_amax."""
    return N * K // 2 + N * K // 16 + M * K // 2 + M * K // 16 + 2 * M * N + 8


MSE_WINDOW = 8                  # E4M3 codes either side of the round-to-nearest scale
MSE_FP64_OPS_PER_CANDIDATE = 64  # 16 elements x (multiply, subtract, square, add)

FP4_PER_BF16 = 4  # nominal dense FP4 / BF16 tensor throughput of B200 (9 / 2.25 PFLOP/s)

MOE = {"E": 128, "N": 1536, "K": 2048, "top": 8}  # synthetic MoE layer: stacked experts, top-8 routing, one token
MOE_T = 4  # tokens per call of the multi-token grouped row


def moe_bytes(n_problems: int, N: int, K: int) -> int:
    """Grouped decode GEMV: each problem's expert weights + x + y + ids and g."""
    return n_problems * (N * K // 2 + N * K // 16 + 2 * N + 8 + 4) + 2 * K


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# Sources each timed row's kernels are built from: a committed traffic figure
# counts only while these files are unchanged since the ncu capture.
_CSRC = "gemm_decode_nvfp4_b200/csrc/"
KERNEL_SOURCES = {
    "gemv": [_CSRC + "gemv.cu", _CSRC + "nvfp4_device.cuh", _CSRC + "sm100_ptx.cuh", _CSRC + "tc_host.h"],
    "quantize": [_CSRC + "quantize.cu", _CSRC + "nvfp4_quant.cuh", _CSRC + "nvfp4_device.cuh"],
    "quantize_mse": [_CSRC + "quantize.cu", _CSRC + "nvfp4_device.cuh"],
    "gemm_m32": [_CSRC + "gemm_small.cu", _CSRC + "gemm_tc.cu", _CSRC + "nvfp4_device.cuh", _CSRC + "sm100_ptx.cuh",
                 _CSRC + "tc_host.h"],
    "gemm_m512": [_CSRC + "gemm_tc.cu", _CSRC + "nvfp4_device.cuh", _CSRC + "sm100_ptx.cuh"],
    "mx_gemv": [_CSRC + "gemv.cu", _CSRC + "nvfp4_device.cuh", _CSRC + "sm100_ptx.cuh", _CSRC + "tc_host.h"],
    "mx_quantize": [_CSRC + "quantize.cu", _CSRC + "nvfp4_quant.cuh", _CSRC + "nvfp4_device.cuh"],
    "moe_gemv": [_CSRC + "gemv.cu", _CSRC + "nvfp4_device.cuh", _CSRC + "sm100_ptx.cuh", _CSRC + "tc_host.h"],
    "moe_gemv_t4": [_CSRC + "gemv.cu", _CSRC + "nvfp4_device.cuh", _CSRC + "sm100_ptx.cuh", _CSRC + "tc_host.h"],
    "gemv_down": [_CSRC + "gemv.cu", _CSRC + "nvfp4_device.cuh", _CSRC + "sm100_ptx.cuh", _CSRC + "tc_host.h"],
    "w4a4_m512": [_CSRC + "gemm_w4a4.cu", _CSRC + "nvfp4_quant.cuh", _CSRC + "nvfp4_device.cuh",
                  _CSRC + "sm100_ptx.cuh", _CSRC + "tc_host.h"],
    "w4a4_gemm": [_CSRC + "gemm_w4a4.cu", _CSRC + "nvfp4_quant.cuh", _CSRC + "nvfp4_device.cuh",
                  _CSRC + "sm100_ptx.cuh", _CSRC + "tc_host.h"],
    "w4a4_pair": [_CSRC + "gemm_w4a4.cu", _CSRC + "nvfp4_quant.cuh", _CSRC + "nvfp4_device.cuh",
                  _CSRC + "sm100_ptx.cuh", _CSRC + "tc_host.h"],
}


def traffic_from_profiles(row: str):
    """DRAM bytes (read + write) per call of a timed row from the committed ncu
    summary profiles/traffic.json, if it was taken on the current source of that
    row's kernels; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p) or row not in KERNEL_SOURCES:
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(row)
    if not e or e.get("source_hash") != kernel_source_hash(KERNEL_SOURCES[row]):
        return None
    return e.get("dram_bytes_per_call")


def dram_attested(traffic_bytes, us: float, hbm_gbs: float) -> dict:
    """GB/s and fraction of the HBM peak that a row's measured DRAM bytes per
    call (read + write, from ncu) give over its CUDA-event time; None without a
    current traffic figure."""
    if not traffic_bytes:
        return {"GB/s_dram": None, "frac_hbm_dram": None}
    gbs = traffic_bytes / (us * 1e-6) / 1e9
    return {"GB/s_dram": gbs, "frac_hbm_dram": gbs / hbm_gbs}


# ------------------------------------------------------------ ranks (replicas)

def max_over_ranks(values, world: int, device="cpu"):
    """Element-wise max of per-rank timings (the replicas run independently;
    the job ends when the slowest rank ends).  Every rank must call it."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(bytes_per_rank: float, max_ms: float, world: int) -> float:
    """Whole-job GB/s: the bytes all ranks processed over the slowest rank's time."""
    return bytes_per_rank * world / (max_ms * 1e-3) / 1e9


# ------------------------------------------------------------ clock sampler

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        load = [v for v in sm if mx and v >= 0.0]
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------- GPU arm

class _Skip(Exception):
    pass


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    import gemm_decode_nvfp4_b200 as nv
    import workloads

    dev = torch.device("cuda", local)
    peaks = load_peaks()
    stream = torch.cuda.Stream(device=dev)
    N, K = MLP, HIDDEN
    copies = args.copies

    # ---- inputs (seeded, synthetic), quantized on the GPU by the library itself
    w_layer = workloads.weight_bf16(workloads.CONFIGS["decode"]).to(dev)
    amax_buf = torch.zeros((1,), dtype=torch.float32, device=dev)
    q0, s0, g0 = nv.quantize_new(w_layer)
    del w_layer
    qs = [q0] + [q0.clone() for _ in range(copies - 1)]
    ss = [s0] + [s0.clone() for _ in range(copies - 1)]
    x1 = workloads.activations(1, K, 1).to(dev).reshape(-1)
    y1 = [torch.empty((N,), dtype=torch.bfloat16, device=dev) for _ in range(copies)]
    X32 = workloads.activations(32, K, 3).to(dev)
    Y32 = [torch.empty((32, N), dtype=torch.bfloat16, device=dev) for _ in range(copies)]
    X512 = workloads.activations(512, K, 4).to(dev)
    Y512 = torch.empty((512, N), dtype=torch.bfloat16, device=dev)
    ws32 = torch.empty((max(1, nv.gemm_workspace_size(32, N, K)),), dtype=torch.uint8, device=dev)
    ws512 = torch.empty((max(1, nv.gemm_workspace_size(512, N, K)),), dtype=torch.uint8, device=dev)
    wq_in = workloads.to_bf16(workloads.plain_weight_f32(N, K, 4)).to(dev)
    qq = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    sq = torch.empty((N, K // 16), dtype=torch.uint8, device=dev)
    gq = torch.empty((1,), dtype=torch.float32, device=dev)

    gemm_ok = args.only in ("all", "gemm_m32", "gemm_m512")
    gemm_err = f"not run (--only {args.only})"
    try:
        if not gemm_ok:
            raise _Skip()
        nv.gemm(X32, qs[0], ss[0], g0, Y32[0], workspace=ws32)
        nv.gemm(X512, qs[0], ss[0], g0, Y512, workspace=ws512)
        torch.cuda.synchronize()
    except _Skip:
        pass
    except nv.Nvfp4Error as e:
        gemm_ok = False
        gemm_err = str(e)

    rows = []  # (name, fn launching one graph's worth of work, launches per graph, kernels per launch)

    def gemv_all():  # weights are static model parameters: programmatic dependent launch
        for i in range(copies):
            nv.gemv(x1, qs[i], ss[i], g0, y1[i], static_weights=True)

    def gemv_ordered_all():  # same, every access waiting for the previous kernel
        for i in range(copies):
            nv.gemv(x1, qs[i], ss[i], g0, y1[i])

    # MXFP4 (UE8M0 scale per 32, no tensor scale) of the same layer, 8 copies
    mq0, ms0 = nv.mx_quantize_new(workloads.weight_bf16(workloads.CONFIGS["decode"]).to(dev))
    mqs = [mq0] + [mq0.clone() for _ in range(copies - 1)]
    mss = [ms0] + [ms0.clone() for _ in range(copies - 1)]
    mq_out = torch.empty_like(mq0)
    ms_out = torch.empty_like(ms0)

    def mx_gemv_all():
        for i in range(copies):
            nv.mx_gemv(x1, mqs[i], mss[i], y1[i], static_weights=True)

    def mx_quant_all():
        nv.mx_quantize(wq_in, mq_out, ms_out)

    # grouped MoE decode: 128 stacked experts [1536, 2048] (226 MB, more than L2),
    # 8 calls per graph, each routing one token to 8 different experts
    me, mn, mk, mtop = MOE["E"], MOE["N"], MOE["K"], MOE["top"]
    moe_w = workloads.to_bf16(workloads.plain_weight_f32(me * mn, mk, 7)).to(dev)
    moe_q, moe_s, _ = nv.quantize_new(moe_w)
    del moe_w
    moe_q = moe_q.reshape(me, mn, mk // 2)
    moe_s = moe_s.reshape(me, mn, mk // 16)
    moe_g = torch.full((me,), 0.004, dtype=torch.float32, device=dev)
    moe_x = workloads.activations(1, mk, 5).to(dev)
    route = torch.randperm(me, generator=torch.Generator().manual_seed(3))[: copies * mtop].reshape(copies, mtop)
    moe_ids = route.to(torch.int32).to(dev)
    moe_tok = torch.zeros((mtop,), dtype=torch.int32, device=dev)
    moe_y = torch.empty((mtop, mn), dtype=torch.bfloat16, device=dev)

    def moe_all():
        for i in range(copies):
            nv.gemv_grouped(moe_x, moe_q, moe_s, moe_g, moe_ids[i], moe_tok, moe_y)

    # the same layer with MOE_T tokens per call (each to its own top-8 experts):
    # one launch covers MOE_T * 8 problems, amortising the dependent-launch cost
    gen = torch.Generator().manual_seed(5)
    moe_ids_t = torch.stack([torch.cat([torch.randperm(me, generator=gen)[:mtop] for _ in range(MOE_T)])
                             for _ in range(copies)]).to(torch.int32).to(dev)
    moe_tok_t = torch.arange(MOE_T, dtype=torch.int32).repeat_interleave(mtop).to(dev)
    moe_x_t = workloads.activations(MOE_T, mk, 6).to(dev)
    moe_y_t = torch.empty((MOE_T * mtop, mn), dtype=torch.bfloat16, device=dev)

    def moe_t_all():
        for i in range(copies):
            nv.gemv_grouped(moe_x_t, moe_q, moe_s, moe_g, moe_ids_t[i], moe_tok_t, moe_y_t)

    # MLP down projection of the same layer, W [5120, 17408]: few rows, long K,
    # the split-K decode GEMV (the library's choice of split), 8 copies (400 MB)
    dcfg = workloads.CONFIGS["down"]
    dq0, ds0, dg0 = nv.quantize_new(workloads.weight_bf16(dcfg).to(dev))
    dqs = [dq0] + [dq0.clone() for _ in range(copies - 1)]
    dss = [ds0] + [ds0.clone() for _ in range(copies - 1)]
    xdown = workloads.activations(1, dcfg.K, dcfg.seed).to(dev).reshape(-1)
    ydown = [torch.empty((dcfg.N,), dtype=torch.bfloat16, device=dev) for _ in range(copies)]

    def gemv_down_all():
        for i in range(copies):
            nv.gemv(xdown, dqs[i], dss[i], dg0, ydown[i], static_weights=True)

    def quant_all():
        amax_buf.zero_()
        nv.amax(wq_in, amax_buf)
        nv.quantize(wq_in, qq, sq, gq, amax=amax_buf)

    def quant_mse_all():  # the same tensor, micro-scale search over +-8 E4M3 codes
        amax_buf.zero_()
        nv.amax(wq_in, amax_buf)
        nv.quantize_mse(wq_in, qq, sq, gq, amax=amax_buf, window=8)

    # W4A4 prefill (NVFP4 activations): the same 8 weight copies, scales
    # rearranged once for the block-scaled tensor cores
    w4_ok = args.only in ("all", "w4a4_m512", "w4a4_gemm", "w4a4_pair")
    if w4_ok:
        smmas = [nv.w4a4_prepare_weights(ss[i], K) for i in range(copies)]
        ws_w4 = torch.empty((nv.w4a4_workspace_size(512, K),), dtype=torch.uint8, device=dev)
        w4_amax = torch.empty((nv.AMAX_FLOATS,), dtype=torch.float32, device=dev)
        w4_qx, w4_sx = nv.w4a4_quantize_x(X512, w4_amax)
        Y512w = torch.empty((512, N), dtype=torch.bfloat16, device=dev)

        def w4a4_all():  # activation amax + quantize + GEMM per call
            for i in range(copies):
                nv.w4a4_linear(X512, qs[i], smmas[i], g0, Y512w, ws_w4, static_weights=True)

        def w4a4_gemm_all():  # the GEMM kernel alone on quantized activations
            for i in range(copies):
                nv.w4a4_gemm(w4_qx, w4_sx, w4_amax, qs[i], smmas[i], g0, Y512w, static_weights=True)

        def w4a4_pair_all():  # the same GEMM on tiles of 256 weight rows over pairs of SMs
            for i in range(copies):
                nv.w4a4_gemm(w4_qx, w4_sx, w4_amax, qs[i], smmas[i], g0, Y512w, static_weights=True, pair=True)

    rows.append(("quantize", quant_all, 1, 2))
    rows.append(("quantize_mse", quant_mse_all, 1, 2))
    rows.append(("mx_quantize", mx_quant_all, 1, 1))
    if gemm_ok:
        def m32_all():
            for i in range(copies):
                nv.gemm(X32, qs[i], ss[i], g0, Y32[i], workspace=ws32, static_weights=True)

        def m512_all():
            for i in range(copies):
                nv.gemm(X512, qs[i], ss[i], g0, Y512, workspace=ws512, static_weights=True)

        rows.append(("gemm_m512", m512_all, copies, 2))
    if w4_ok:
        rows.append(("w4a4_m512", w4a4_all, copies, 3))  # amax + quantize X + GEMM per call
        rows.append(("w4a4_gemm", w4a4_gemm_all, copies, 1))
        rows.append(("w4a4_pair", w4a4_pair_all, copies, 1))
    if gemm_ok:
        rows.append(("gemm_m32", m32_all, copies, 2))    # X prep + GEMM per call
    rows.append(("mx_gemv", mx_gemv_all, copies, 1))
    rows.append(("moe_gemv", moe_all, copies, 1))
    rows.append(("moe_gemv_t4", moe_t_all, copies, 1))
    rows.append(("gemv_down", gemv_down_all, copies, 1))
    rows.append(("gemv_ordered", gemv_ordered_all, copies, 1))
    rows.append(("gemv", gemv_all, copies, 1))
    if args.only != "all":  # profiling runs: keep only the named row (plus the headline GEMV)
        rows = [r for r in rows if r[0] in (args.only, "gemv")]

    graphs = {}
    with torch.cuda.stream(stream):
        for name, fn, _, _ in rows:  # eager warm-up (also compiles nothing: all AOT)
            fn()
    stream.synchronize()
    for name, fn, _, _ in rows:
        gph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gph, stream=stream):
            fn()
        graphs[name] = gph

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # The quantizer rows leave tens of MB of dirty q/s in L2 (written back only
    # when evicted): an untimed read of twice the L2 after each of them keeps the
    # next row from paying for that write-back.  The GEMV rows run after GEMVs
    # and are not preceded by a flush (a cold L2 and TLB slowed them).
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = torch.ones((2 * l2_bytes // 4,), dtype=torch.float32, device=dev)
    flush_out = torch.empty((), dtype=torch.float32, device=dev)
    flush_after = ("quantize", "quantize_mse", "mx_quantize")

    def l2_writeback():
        torch.sum(flush_buf, dim=0, out=flush_out)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            for name, *_ in rows:
                graphs[name].replay()
                if name in flush_after:
                    l2_writeback()
    stream.synchronize()

    evs = {name: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)] for name, *_ in rows}
    step_start = torch.cuda.Event(enable_timing=True)
    step_end = torch.cuda.Event(enable_timing=True)
    barrier()
    with ClockSampler(local) as clocks:
        with torch.cuda.stream(stream):
            step_start.record(stream)
            for it in range(args.steps):
                for name, *_ in rows:
                    a, b = evs[name][it]
                    a.record(stream)
                    graphs[name].replay()
                    b.record(stream)
                    if name in flush_after:
                        l2_writeback()
            step_end.record(stream)
        stream.synchronize()
        barrier()
    clk = clocks.summary()

    total_ms = step_start.elapsed_time(step_end)
    per_launch_ms = {}
    spread = {}
    for name, _, launches, _ in rows:
        per_step = [a.elapsed_time(b) / launches for a, b in evs[name]]
        per_launch_ms[name] = sum(per_step) / args.steps
        q = statistics.quantiles(per_step, n=10) if len(per_step) >= 2 else [per_step[0]] * 9
        spread[name] = {"p10_us": q[0] * 1e3, "median_us": statistics.median(per_step) * 1e3, "p90_us": q[-1] * 1e3}

    red = max_over_ranks([total_ms] + [per_launch_ms[n] for n, *_ in rows], world, dev)
    total_ms = red[0]
    for i, (n, *_) in enumerate(rows):
        per_launch_ms[n] = red[i + 1]

    hbm = peaks["hbm_gbs"]
    bf16_burst = peaks["bf16_tflops"]
    kernels = {}
    gb = gemv_bytes(N, K)
    gemv_gbs = gb / (per_launch_ms["gemv"] * 1e-3) / 1e9
    kernels["gemv"] = {"us": per_launch_ms["gemv"] * 1e3, "GB/s": gemv_gbs, "frac_hbm": gemv_gbs / hbm,
                       "bytes": gb, "weight_bytes_per_token": N * K // 2 + N * K // 16,
                       "launch": "static weights: programmatic dependent launch between back-to-back GEMVs"}
    if "gemv_ordered" in per_launch_ms:
        go = gb / (per_launch_ms["gemv_ordered"] * 1e-3) / 1e9
        kernels["gemv_ordered"] = {"us": per_launch_ms["gemv_ordered"] * 1e3, "GB/s": go, "frac_hbm": go / hbm,
                                   "launch": "no static-weights flag: all reads wait for the previous kernel"}
    if "quantize" in per_launch_ms:
        qb = quantize_bytes(N, K)
        qgbs = qb / (per_launch_ms["quantize"] * 1e-3) / 1e9
        kernels["quantize"] = {"us": per_launch_ms["quantize"] * 1e3, "GB/s": qgbs, "frac_hbm": qgbs / hbm,
                               "bytes": qb}
    if "mx_gemv" in per_launch_ms:
        mb = mx_gemv_bytes(N, K)
        mg = mb / (per_launch_ms["mx_gemv"] * 1e-3) / 1e9
        kernels["mx_gemv"] = {"us": per_launch_ms["mx_gemv"] * 1e3, "GB/s": mg, "frac_hbm": mg / hbm, "bytes": mb,
                              "weight_bytes_per_token": N * K // 2 + N * K // 32,
                              "format": "MXFP4: UE8M0 scale per 32, no tensor scale"}
    if "moe_gemv" in per_launch_ms:
        mb = moe_bytes(MOE["top"], MOE["N"], MOE["K"])
        mg = mb / (per_launch_ms["moe_gemv"] * 1e-3) / 1e9
        kernels["moe_gemv"] = {"us": per_launch_ms["moe_gemv"] * 1e3, "GB/s": mg, "frac_hbm": mg / hbm, "bytes": mb,
                               "workload": f"grouped decode GEMV: {MOE['top']} of {MOE['E']} stacked experts "
                                           f"[{MOE['N']}, {MOE['K']}], one token, synthetic routing"}
    if "quantize_mse" in per_launch_ms:
        qb = quantize_bytes(N, K)
        t_mse = per_launch_ms["quantize_mse"] * 1e3
        kernels["quantize_mse"] = {
            "us": t_mse, "GB/s": qb / (t_mse * 1e-6) / 1e9, "bytes": qb,
            "x_round_to_nearest": t_mse / kernels["quantize"]["us"] if "quantize" in kernels else None,
            "fp64_ops_per_block_max": MSE_FP64_OPS_PER_CANDIDATE * (2 * MSE_WINDOW + 1),
            "what": "amax + micro-scale search quantizer (E4M3 candidates within 8 codes, fp64 error): "
                    "FP64-bound; the pages report about 6x the round-to-nearest cost"}
    if "moe_gemv_t4" in per_launch_ms:
        P = MOE_T * MOE["top"]
        mb = moe_bytes(P, MOE["N"], MOE["K"]) + 2 * MOE["K"] * (MOE_T - 1)
        mg = mb / (per_launch_ms["moe_gemv_t4"] * 1e-3) / 1e9
        kernels["moe_gemv_t4"] = {"us": per_launch_ms["moe_gemv_t4"] * 1e3, "GB/s": mg, "frac_hbm": mg / hbm, "bytes": mb,
                                  "us_per_token": per_launch_ms["moe_gemv_t4"] * 1e3 / MOE_T,
                                  "workload": f"grouped decode GEMV: {MOE_T} tokens x top-{MOE['top']} of {MOE['E']} "
                                              f"stacked experts [{MOE['N']}, {MOE['K']}] = {P} problems per launch"}
    if "gemv_down" in per_launch_ms:
        db = gemv_bytes(dcfg.N, dcfg.K)
        dgbs = db / (per_launch_ms["gemv_down"] * 1e-3) / 1e9
        kernels["gemv_down"] = {"us": per_launch_ms["gemv_down"] * 1e3, "GB/s": dgbs, "frac_hbm": dgbs / hbm,
                                "bytes": db, "weight_bytes_per_token": dcfg.N * dcfg.K // 2 + dcfg.N * dcfg.K // 16,
                                "workload": f"down-projection decode GEMV W [{dcfg.N}, {dcfg.K}] x BF16 [1, {dcfg.K}]",
                                "launch": "split-K (library's choice), static weights, 8 copies per graph"}
    if "mx_quantize" in per_launch_ms:
        mb = mx_quantize_bytes(N, K)
        mq = mb / (per_launch_ms["mx_quantize"] * 1e-3) / 1e9
        kernels["mx_quantize"] = {"us": per_launch_ms["mx_quantize"] * 1e3, "GB/s": mq, "frac_hbm": mq / hbm,
                                  "bytes": mb}
    for name, M in (("gemm_m32", 32), ("gemm_m512", 512)):
        if name in per_launch_ms:
            t = per_launch_ms[name] * 1e-3
            fl = 2.0 * M * N * K
            byt = gemm_bytes(M, N, K)
            kernels[name] = {"us": t * 1e6, "TFLOP/s": fl / t / 1e12, "frac_bf16": fl / t / 1e12 / bf16_burst,
                             "GB/s": byt / t / 1e9, "frac_hbm": byt / t / 1e9 / hbm,
                             "weight_bytes_per_token": (N * K // 2 + N * K // 16) / M}
        elif not gemm_ok and args.only == "all":
            kernels[name] = {"unavailable": gemm_err}

    fp4_peak = bf16_burst * FP4_PER_BF16
    for name in ("w4a4_m512", "w4a4_gemm", "w4a4_pair"):
        if name in per_launch_ms:
            t = per_launch_ms[name] * 1e-3
            fl = 2.0 * 512 * N * K
            byt = gemm_bytes(512, N, K) if name == "w4a4_m512" else w4a4_gemm_bytes(512, N, K)
            kernels[name] = {"us": t * 1e6, "TFLOP/s": fl / t / 1e12, "frac_fp4": fl / t / 1e12 / fp4_peak,
                             "fp4_peak_tflops": fp4_peak,
                             "fp4_peak_source": f"{peaks['source']} bf16 x {FP4_PER_BF16} (nominal dense FP4/BF16)",
                             "GB/s": byt / t / 1e9, "frac_hbm": byt / t / 1e9 / hbm, "bytes": byt,
                             "what": ("activation amax + NVFP4 quantize of X + block-scaled FP4 GEMM"
                                      if name == "w4a4_m512" else "block-scaled FP4 GEMM on quantized X"
                                      + (", tiles of 256 weight rows on pairs of SMs" if name == "w4a4_pair" else ""))}

    # ---- end to end through the public API with host buffers (decode GEMV):
    # pinned x -> device, GEMV, y -> pinned host, every step.
    x_host = workloads.activations(1, K, 1).reshape(-1).pin_memory()
    y_host = torch.empty((N,), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x_host, device=dev)
    e2e_ms = []
    with torch.cuda.stream(stream):
        for it in range(args.warmup + args.steps):
            for i in range(copies):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                x_dev.copy_(x_host, non_blocking=True)
                nv.gemv(x_dev, qs[i], ss[i], g0, y1[i])
                y_host.copy_(y1[i], non_blocking=True)
                b.record(stream)
                b.synchronize()
                if it >= args.warmup:
                    e2e_ms.append(a.elapsed_time(b))
    e2e_t = max_over_ranks([statistics.mean(e2e_ms)], world, dev)[0]

    launches = 0
    for name, _, n_launch, n_kern in rows:
        launches += args.steps * n_launch * n_kern

    for name in kernels:
        if "us" in kernels[name]:
            kernels[name]["traffic"] = traffic_from_profiles(name)
            if name in spread:
                kernels[name]["spread"] = spread[name]
    for name in ("quantize", "mx_quantize"):
        # the quantizers' output is still in L2 when their events end: beside the
        # algorithmic fraction, the fraction that the DRAM bytes ncu measured for
        # the same row support
        if name in kernels:
            kernels[name].update(dram_attested(kernels[name]["traffic"], kernels[name]["us"], hbm))
    traffic = kernels["gemv"]["traffic"]
    out = None
    if rank == 0:
        out = {
            "metric": METRIC,
            "value": job_throughput(gb, per_launch_ms["gemv"], world),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "nvfp4 weights (e2m1 + e4m3 + f32), bf16 activations, f32 accumulate",
            "data": "synthetic (seeded numpy draws; no checkpoint)",
            "config": {"workload": WORKLOAD, "N": N, "K": K, "M": 1, "parallelism": f"replicas x{world}",
                       "l2": f"inputs larger than L2: {copies} rotating weight copies "
                             f"({copies * (N * K // 2 + N * K // 16) / 1e6:.0f} MB) per graph",
                       "row_order": "quantize, MSE quantize, MXFP4 quantize (each followed by an untimed read of 2 x L2 that writes back their dirty output), gemm M=512, W4A4 M=512 (step), W4A4 GEMM, gemm M=32, MXFP4 gemv, MoE gemv (1 and 4 tokens), down-projection gemv, gemv ordered, gemv static: each GEMV graph "
                                    "follows GEMVs, not the rows that leave tens of MB of dirty output in L2",
                       "step": "quantize [17408,5120] (NVFP4 round-to-nearest, NVFP4 micro-scale search, MXFP4) + gemm M=512 + W4A4 M=512 (quantize X + GEMM) + W4A4 GEMM + gemm M=32 + MXFP4 gemv + grouped MoE gemv (1 and 4 tokens) + down-projection gemv [5120, 17408] (split-K) + gemv M=1 (x2: ordered and static-weights)",
            "gemv_launch": "8 GEMVs per graph on 8 weight copies, programmatic dependent launch (static weights)"},
            "roofline": {"bound": "hbm", "achieved": gemv_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gemv_gbs / hbm, "traffic": traffic,
                         "peak_source": peaks["source"], "kernel": "gemv",
                         "algorithmic_bytes_per_launch": gb},
            "kernels": kernels,
            "e2e": {"value": job_throughput(gb, e2e_t, world), "unit": "GB/s",
                    "h2d_bytes_per_step": 2 * K, "d2h_bytes_per_step": 2 * N,
                    "what": "per step: pinned x H2D, nvfp4_gemv, y D2H (weights resident)"},
            "gpu_launches": launches,
            "clocks": clk,
        }
        if not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(args.cpu_rows)
        print(json.dumps(out), flush=True)

    for g in graphs.values():
        del g
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return out


# ------------------------------------------------------------ CPU oracle

def _oracle_gemv_sample(n_rows: int):
    import oracle
    import workloads
    cfg = workloads.CONFIGS["decode"]
    w = workloads.to_bf16(workloads.layer_weight_f32(cfg.N, cfg.K, cfg.seed)[:n_rows])
    q, s, g = oracle.quantize(w)
    x = workloads.activations(1, cfg.K, cfg.seed)
    return oracle, x, q, s, g


def cpu_baseline(n_rows: int):
    """The oracle's decode GEMV on a sample of rows of the decode workload,
    timed on this host's cores; bytes counted like the GPU's (per row)."""
    oracle, x, q, s, g = _oracle_gemv_sample(n_rows)
    oracle.linear(x, q[:8], s[:8], g)  # load + warm
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.linear(x, q, s, g)
        reps += 1
        if time.perf_counter() - t0 > 10.0:  # about 10 s of CPU work
            break
    dt = (time.perf_counter() - t0) / reps
    byt = gemv_bytes(n_rows, HIDDEN)
    return {"value": byt / dt / 1e9, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"decode GEMV rows 0..{n_rows - 1} of [17408, 5120] (fp64 oracle, {reps} reps)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    oracle, x, q, s, g = _oracle_gemv_sample(args.cpu_rows)
    for _ in range(args.warmup):
        oracle.linear(x, q, s, g)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.linear(x, q, s, g)
        ts.append(time.perf_counter() - t0)
    dt = sum(ts) / len(ts)
    byt = gemv_bytes(args.cpu_rows, HIDDEN)
    v = byt / dt / 1e9
    out = {
        "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic (seeded numpy draws)",
        "config": {"workload": WORKLOAD, "N": MLP, "K": HIDDEN, "M": 1, "sample_rows": args.cpu_rows},
        "impl": "reference",
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"decode GEMV rows 0..{args.cpu_rows - 1} of [17408, 5120] per step"},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(out), flush=True)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--copies", type=int, default=8, help="rotating weight copies per graph (L2 defeat)")
    ap.add_argument("--cpu-rows", type=int, default=17408)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default="all", choices=["all", "gemv", "gemv_ordered", "quantize", "quantize_mse", "gemm_m32",
                                                      "gemm_m512", "mx_gemv", "mx_quantize", "moe_gemv",
                                                      "gemv_down", "moe_gemv_t4", "w4a4_m512", "w4a4_gemm", "w4a4_pair"],
                    help="time only this row (and the headline GEMV): for profiling runs")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
