"""Benchmark of the NVFP4 linear-layer training step on B200.

One step = one pass of the whole hot path over one batch: quantize X (rows RNE +
RHT columns), W (16x16, both orientations), dY (rows SR + RHT columns SR), and the
fprop / dgrad / wgrad block-scaled FP4 GEMMs, on the 12B-class MLP up-projection
(tokens M=8192, hidden K=5120, FFN N=20480), synthetic seeded inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is device-timed whole-job TFLOP/s of the
three GEMMs per step time (inputs resident in HBM); `e2e` is the same metric with
the inputs copied from pinned host memory and the outputs read back every step.
N > 1 runs independent replicas (weak scaling): the step has no exchange.
`--impl reference` times the CPU oracle on a bounded sample of the same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 linear fprop+dgrad+wgrad TFLOPS and quantize GB/s, % of B200 roofline"
WORKLOAD = "12B-class MLP up-projection training step (fprop+dgrad+wgrad), M=8192 K=5120 N=20480"
M, K, N = 8192, 5120, 20480
FLOPS_PER_GEMM = 2.0 * M * K * N
FLOPS_PER_STEP = 3 * FLOPS_PER_GEMM
KERNELS_PER_STEP = 9  # 2 amax + 2 quantize (fprop), 1 + 1 (dgrad), 3 GEMMs
FP4_OVER_BF16 = 4.0   # nominal dense FP4 9 PFLOP/s over bf16 2.25 PFLOP/s
# DRAM bytes (read + write) of one launch of each GEMM of the step, from one-pass ncu
# captures of that launch; reported only while the GEMM source is the one that was
# captured.
GEMM_TRAFFIC = {"gemm_cu_sha256_16": "30f8c6ccc064eacd", "bytes": {
    "fprop": 87166208 + 296675584, "dgrad": 428784128 + 71357440, "wgrad": 118288128 + 178921984}}


def env_rank():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(
        os.environ.get("LOCAL_RANK", "0"))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while timing."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- ranks
def init_ranks(world, dev, backend="nccl", timeout_s=120):
    """Process group of the `world` ranks (none at world 1) and the two collective
    steps the bench takes: a barrier and the maximum of a float over ranks.  Every
    rank calls both in the same order; the short timeout turns a lost rank into an
    error instead of a hang."""
    import datetime

    import torch
    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        kw = {"device_id": dev} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        if world == 1:
            return float(v)
        t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return t.item()

    def finish():
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()

    return barrier, max_over_ranks, finish


def whole_job_tflops(world, flops_per_rank_step, ms_max):
    """Whole-job throughput: the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank_step / (ms_max * 1e-3) / 1e12


def bench_line(world, steps, warmup, ms, value, clocks, e2e, cpu, extra):
    """The JSON line rank 0 prints (weak scaling: every rank a full replica)."""
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world,
        "steps": steps, "warmup": max(warmup, 3), "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
        "data": "synthetic (seeded: X~N(0,1), W~N(0,0.02^2), dY~N(0,1e-3^2), bf16)",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "N": N,
                   "global_batch_tokens": M * world,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2 (629 MB bf16 inputs, ~1.6 GB touched per step)",
                   "recipe": "X,dY 1x16; W 16x16; SR on dY; 16-pt RHT on wgrad operands"},
        "gpu_launches": KERNELS_PER_STEP * steps,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    line.update(extra)
    return line


# --------------------------------------------------------------------------- ours
def run_ours(args, rank, world, local_rank):
    import torch

    from nvfp4_bit_quantized_amax_b200 import capi
    from nvfp4_bit_quantized_amax_b200 import synthetic as syn

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    barrier, max_over_ranks, finish = init_ranks(world, dev, "nccl")
    capi.load()
    stream = torch.cuda.current_stream()

    # synthetic inputs (seeded per rank: every replica its own batch)
    Xb, Wb, dYb = syn.mlp_inputs(M, K, N, seed=1000 * rank)

    def to_dev(b):
        return torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)

    X, W, dY = to_dev(Xb), to_dev(Wb), to_dev(dYb)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dW = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(capi.linear_workspace_bytes(M, K, N), dtype=torch.uint8, device=dev)
    signs = syn.rht_signs(rank)
    seed = 20260 + rank

    def step(x=X, w=W, dy=dY, y=Y, dx=dX, dw=dW):
        capi.nvfp4_linear_fprop(x, w, y, signs, ws)
        capi.nvfp4_linear_dgrad(dy, dx, seed, signs, ws)
        capi.nvfp4_linear_wgrad(None, dw, M, seed, signs, ws)

    def timed(fn, iters, warm):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(iters):
            fn()
        e.record(stream)
        e.synchronize()
        torch.cuda.synchronize()
        barrier()
        return s.elapsed_time(e) / iters

    # ---- the timed step (inputs resident in HBM; per-step working set ~1.6 GB >> L2)
    with ClockSampler(local_rank) as clk:
        ms = timed(step, args.steps, max(args.warmup, 3))
    ms = max_over_ranks(ms)
    assert capi.nvfp4_read_status(ws) == 0
    value = whole_job_tflops(world, FLOPS_PER_STEP, ms)

    out = {}
    # ---- the same step, its three C-ABI calls captured once as a CUDA graph and
    # replayed (the launch gaps between the calls' kernels go away); one rank only, so
    # that a capture failure cannot leave other ranks waiting in a collective
    def graph_step_ms():
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        g_ms = timed(graph.replay, args.steps, max(args.warmup, 3))
        del graph
        return g_ms

    if world > 1:
        out["step_graph"] = {"skipped": "measured on one GPU only"}
    else:
        try:
            g_ms = graph_step_ms()
            out["step_graph"] = {"ms_per_step": round(g_ms, 4),
                                 "value": round(whole_job_tflops(world, FLOPS_PER_STEP, g_ms), 2),
                                 "note": "the timed step's three C-ABI calls replayed as one CUDA graph"}
        except Exception as exc:  # reported, not fatal: the eager number stands
            out["step_graph"] = {"error": str(exc)[:200]}
    assert capi.nvfp4_read_status(ws) == 0
    out["in_step"] = in_step_breakdown(capi, syn, X, W, dY, Y, dX, dW, ws, signs, seed, stream,
                                       barrier, iters=max(5, min(20, args.steps)))
    # ---- per-kernel timing on the same stream (each launch alone, back to back); every
    # rank runs it (timed() holds barriers)
    iters = max(10, min(50, args.steps))
    ops = {w: capi.nvfp4_linear_operand(ws, M, K, N, w) for w in range(6)}
    lib = capi.load()

    def gemm(a, b, alpha, D, Mx, Nx, Kx):
        va, vb = ops[a], ops[b]
        return lambda: lib.nvfp4_gemm(va.data, va.scales, vb.data, vb.scales,
                                      va.tensor_scale, vb.tensor_scale, alpha, Mx, Nx, Kx,
                                      D.data_ptr(), None, None, stream.cuda_stream)

    g_ms = {
        "fprop": timed(gemm(capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0, Y, M, N, K), iters, 3),
        "dgrad": timed(gemm(capi.LIN_DY_ROW, capi.LIN_W_COL, 1.0, dX, M, K, N), iters, 3),
        "wgrad": timed(gemm(capi.LIN_DY_COL, capi.LIN_X_COL, 1.0 / 16, dW, N, K, M), iters, 3),
    }
    qws = torch.empty(capi.quantize_workspace_bytes(), dtype=torch.uint8, device=dev)

    def tview(w):
        v = ops[w]
        return (v.data, v.scales, v.tensor_scale)

    def quant(x, bm, rr, cr, rht, row_w, col_w):
        r = capi.Tensor(*tview(row_w), 0, 0) if row_w is not None else None
        c = capi.Tensor(*tview(col_w), 0, 0) if col_w is not None else None
        sgn = np.ascontiguousarray(signs)
        opts = capi.QuantizeOpts(bm, rr, cr, seed, int(rht), sgn.ctypes.data)
        import ctypes
        args_ = (ctypes.c_void_p(x.data_ptr()), x.shape[0], x.shape[1], ctypes.byref(opts),
                 ctypes.byref(r) if r is not None else None,
                 ctypes.byref(c) if c is not None else None,
                 ctypes.c_void_p(qws.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
        return lambda: lib.nvfp4_quantize_2d(*args_)

    q_ms = {
        "X_row+col_rht": (timed(quant(X, 0, 0, 0, True, capi.LIN_X_ROW, capi.LIN_X_COL), iters, 3), M * K),
        "W_16x16_both": (timed(quant(W, 1, 0, 0, False, capi.LIN_W_ROW, capi.LIN_W_COL), iters, 3), N * K),
        "dY_row_sr+col_rht_sr": (timed(quant(dY, 0, 1, 1, True, capi.LIN_DY_ROW, capi.LIN_DY_COL), iters, 3), M * N),
    }
    peaks, peak_kind = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    gemm_avg_ms = sum(g_ms.values()) / 3
    achieved = FLOPS_PER_GEMM / (gemm_avg_ms * 1e-3) / 1e12
    # dual-orientation quantize: amax read 2 B + quantize read 2 B + 2 x (0.5 + 1/16) B written
    q_bytes_per_el = 2.0 + 2.0 + 2 * (0.5 + 1.0 / 16)
    quant = {k: {"ms": round(v[0], 4),
                 "GB/s": round(q_bytes_per_el * v[1] / (v[0] * 1e-3) / 1e9, 1),
                 "frac_hbm": round(q_bytes_per_el * v[1] / (v[0] * 1e-3) / 1e9 / peaks["hbm_gbs"], 3)}
             for k, v in q_ms.items()}
    q_total_bytes = sum(q_bytes_per_el * v[1] for v in q_ms.values())
    q_total_ms = sum(v[0] for v in q_ms.values())
    traffic, traffic_by_gemm = args.traffic, None
    if traffic is None:
        import hashlib
        with open(os.path.join(ROOT, "nvfp4_bit_quantized_amax_b200", "csrc", "gemm.cu"), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] == GEMM_TRAFFIC["gemm_cu_sha256_16"]:
                traffic_by_gemm = GEMM_TRAFFIC["bytes"]
                traffic = round(sum(traffic_by_gemm.values()) / 3)
    out["roofline"] = {
        "bound": "tensor", "kernel": "gemm_nvf4_pair_kernel (fprop/dgrad/wgrad average)",
        "achieved": round(achieved, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
        "frac": round(achieved / fp4_peak, 4), "traffic": traffic,
        "traffic_by_gemm": traffic_by_gemm,
        "peak_source": f"derived from {peak_kind} peaks: FP4 = {FP4_OVER_BF16:g} x the bf16 burst "
                       f"{peaks['bf16_tflops']} TFLOP/s (nominal 9 / 2.25 PFLOP/s ratio); no FP4 "
                       f"peak is measured",
        "frac_of_spec_9pf": round(achieved / 9000.0, 4),
    }
    out["kernels"] = {
        "gemm_ms": {k: round(v, 4) for k, v in g_ms.items()},
        "gemm_tflops": {k: round(FLOPS_PER_GEMM / (v * 1e-3) / 1e12, 1) for k, v in g_ms.items()},
        "quantize": quant,
        "quantize_GB/s": round(q_total_bytes / (q_total_ms * 1e-3) / 1e9, 1),
        "quantize_frac_hbm": round(q_total_bytes / (q_total_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 3),
        "hbm_peak_GB/s": peaks["hbm_gbs"],
    }

    # ---- MXFP4, the comparison format: one-pass quantize of X and W, MX GEMM (fprop shape)
    xm = (torch.empty(M * K // 2, dtype=torch.uint8, device=dev),
          torch.empty(capi.mx_scale_bytes(M, K), dtype=torch.uint8, device=dev))
    wm = (torch.empty(N * K // 2, dtype=torch.uint8, device=dev),
          torch.empty(capi.mx_scale_bytes(N, K), dtype=torch.uint8, device=dev))
    iters_mx = max(10, min(50, args.steps))
    qx_ms = timed(lambda: capi.nvfp4_mx_quantize(X, *xm), iters_mx, 3)
    qw_ms = timed(lambda: capi.nvfp4_mx_quantize(W, *wm), iters_mx, 3)
    # the MX and the NVFP4 fprop GEMM timed alternately, three times each (best of
    # each), so that both meet the same clocks
    mx_fn = lambda: capi.nvfp4_mx_gemm(xm[0], xm[1], wm[0], wm[1], 1.0, M, N, K, D_bf16=Y)
    nv_fn = gemm(capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0, Y, M, N, K)
    g_mx, g_nv = float("inf"), float("inf")
    for _ in range(3):
        g_mx = min(g_mx, timed(mx_fn, iters_mx, 3))
        g_nv = min(g_nv, timed(nv_fn, iters_mx, 3))
    mx_bytes_per_el = 2.0 + 0.5 + 1.0 / 32   # one read, codes + E8M0 scales written
    out["kernels"]["mxfp4"] = {
        "quantize_X_ms": round(qx_ms, 4), "quantize_W_ms": round(qw_ms, 4),
        "quantize_GB/s": round(mx_bytes_per_el * (M * K + N * K) / ((qx_ms + qw_ms) * 1e-3) / 1e9, 1),
        "gemm_fprop_ms": round(g_mx, 4),
        "gemm_fprop_tflops": round(FLOPS_PER_GEMM / (g_mx * 1e-3) / 1e12, 1),
        "nvfp4_fprop_ms_alongside": round(g_nv, 4),
        "mx_over_nvfp4_fprop_time": round(g_mx / g_nv, 3),
        "note": "two-SM 256x256 tiles, block_scale.scale_vec::2X, UE8M0 per 32 elements"}

    # ---- the other workloads: the 256^3 outlier step, the 8192^2 quantize sweep and the
    # GEMM shape sweep
    if not args.no_sweeps:
        out["linear_256"] = bench_linear_256(capi, syn, dev, stream, timed)
        out["quant_sweep_8192"] = bench_quant_sweep(capi, syn, dev, stream, timed, peaks)
        out["gemm_sweep"] = bench_gemm_sweep(capi, syn, dev, stream, timed, fp4_peak)

    # ---- mixture-of-experts expert layer (64 experts, Zipf(1.1) top-4 routing)
    if not args.no_moe:
        out["moe"] = moe_step_bench(capi, syn, dev, stream, timed, max_over_ranks, world,
                                    iters=max(3, min(20, args.steps // 5)))

    # ---- end to end through the C ABI with host buffers (pinned), copies timed
    e2e = None
    if not args.no_e2e:
        hX = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).pin_memory()
        hW = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).pin_memory()
        hdY = torch.from_numpy(dYb.view(np.int16)).view(torch.bfloat16).pin_memory()
        hY = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        hdX = torch.empty((M, K), dtype=torch.bfloat16).pin_memory()
        hdW = torch.empty((N, K), dtype=torch.bfloat16).pin_memory()

        # Every step copies its inputs in from pinned host memory and its results
        # out.  Two device sets of inputs and outputs and three streams (copies in,
        # the step, copies out) let step i's copies overlap the neighbouring steps'
        # compute and copies, as a training loop that streams batches would.
        sets = [(X, W, dY, Y, dX, dW), tuple(torch.empty_like(t) for t in (X, W, dY, Y, dX, dW))]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_steps(n):
            for i in range(n):
                b = i % 2
                x, w, dy, y, dx, dw = sets[b]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_done[b])     # step i-2 is done reading this set
                    x.copy_(hX, non_blocking=True)
                    w.copy_(hW, non_blocking=True)
                    dy.copy_(hdY, non_blocking=True)
                    ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])        # step i-2's results are out
                step(x, w, dy, y, dx, dw)
                ev_done[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[b])
                    hY.copy_(y, non_blocking=True)
                    hdX.copy_(dx, non_blocking=True)
                    hdW.copy_(dw, non_blocking=True)
                    ev_out[b].record(s_out)

        def e2e_timed(n):
            e2e_steps(3)  # warm-up
            torch.cuda.synchronize()
            barrier()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            e2e_steps(n)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)
            t1.record(stream)
            t1.synchronize()
            torch.cuda.synchronize()
            barrier()
            return t0.elapsed_time(t1) / n

        e_iters = max(4, min(10, args.steps))
        e_ms = max_over_ranks(e2e_timed(e_iters))
        h2d = 2 * (M * K + N * K + M * N)
        e2e = {"value": round(whole_job_tflops(world, FLOPS_PER_STEP, e_ms), 2), "unit": "TFLOPS",
               "ms_per_step": round(e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h2d,
               "copies": "pinned host <-> device every step, copies in / step / copies out on three "
                         "streams with two device buffer sets (copies overlap neighbouring steps)"}
        del sets

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.cpu_seconds)

    finish()
    if rank != 0:
        return
    line = bench_line(world, args.steps, args.warmup, ms, value, clk.summary(), e2e, cpu, out)
    print(json.dumps(line), flush=True)


def in_step_breakdown(capi, syn, X, W, dY, Y, dX, dW, ws, signs, seed, stream, barrier, iters):
    """The step's own kernels, in the step's order, on the step's data, with a CUDA
    event between every C-ABI call: quantize X (rows + RHT columns), quantize W (16x16,
    both orientations), fprop GEMM, quantize dY (rows SR + RHT columns SR), dgrad GEMM,
    wgrad GEMM.  The parts add up to the step (plus event overhead), unlike the
    per-kernel figures below, which time each launch alone and back to back (its
    operands then partly stay in L2 between repeats)."""
    import ctypes

    import torch
    lib = capi.load()
    ops = {w: capi.nvfp4_linear_operand(ws, M, K, N, w) for w in range(6)}
    qws = torch.empty(capi.quantize_workspace_bytes(), dtype=torch.uint8, device=X.device)
    sgn = np.ascontiguousarray(signs)
    st = ctypes.c_void_p(stream.cuda_stream)

    def quant(x, bm, rr, cr, rht, row_w, col_w):
        v, c = ops[row_w], ops[col_w]
        r = capi.Tensor(v.data, v.scales, v.tensor_scale, 0, 0)
        cc = capi.Tensor(c.data, c.scales, c.tensor_scale, 0, 0)
        opts = capi.QuantizeOpts(bm, rr, cr, seed, int(rht), sgn.ctypes.data)
        return lambda: lib.nvfp4_quantize_2d(ctypes.c_void_p(x.data_ptr()), x.shape[0], x.shape[1],
                                             ctypes.byref(opts), ctypes.byref(r), ctypes.byref(cc),
                                             ctypes.c_void_p(qws.data_ptr()), st)

    def gemm(a, b, alpha, D, Mx, Nx, Kx):
        va, vb = ops[a], ops[b]
        return lambda: lib.nvfp4_gemm(va.data, va.scales, vb.data, vb.scales, va.tensor_scale,
                                      vb.tensor_scale, alpha, Mx, Nx, Kx, D.data_ptr(), None, None, st)

    parts = [("quantize_X", quant(X, 0, 0, 0, True, capi.LIN_X_ROW, capi.LIN_X_COL)),
             ("quantize_W", quant(W, 1, 0, 0, False, capi.LIN_W_ROW, capi.LIN_W_COL)),
             ("gemm_fprop", gemm(capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0, Y, M, N, K)),
             ("quantize_dY", quant(dY, 0, 1, 1, True, capi.LIN_DY_ROW, capi.LIN_DY_COL)),
             ("gemm_dgrad", gemm(capi.LIN_DY_ROW, capi.LIN_W_COL, 1.0, dX, M, K, N)),
             ("gemm_wgrad", gemm(capi.LIN_DY_COL, capi.LIN_X_COL, 1.0 / 16, dW, N, K, M))]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(parts) + 1)]
    tot = [0.0] * len(parts)
    for i in range(iters + 3):
        ev[0].record(stream)
        for j, (_, fn) in enumerate(parts):
            rc = fn()
            assert rc == 0, rc
            ev[j + 1].record(stream)
        ev[-1].synchronize()
        if i >= 3:
            for j in range(len(parts)):
                tot[j] += ev[j].elapsed_time(ev[j + 1])
    torch.cuda.synchronize()
    barrier()
    res = {name: round(t / iters, 4) for (name, _), t in zip(parts, tot)}
    res["sum_ms"] = round(sum(tot) / iters, 4)
    res["gemm_ms"] = round(sum(res[k] for k in ("gemm_fprop", "gemm_dgrad", "gemm_wgrad")), 4)
    res["quantize_ms"] = round(sum(res[k] for k in ("quantize_X", "quantize_W", "quantize_dY")), 4)
    return res


def bench_linear_256(capi, syn, dev, stream, timed, iters=200):
    """Linear layer M=K=N=256 with 1% x50 outliers (X, W, dY ~ N(0,1), seed 0): the
    whole step (quantize X, W, dY; fprop, dgrad, wgrad) in microseconds, launched
    eagerly through the C ABI and replayed as one CUDA graph of the same calls.
    Latency-bound (0.1 GFLOP, ~1 MB): no roofline fraction."""
    import torch
    M_, K_, N_ = 256, 256, 256
    Xb, Wb, dYb = syn.linear_small_inputs(0)

    def to_dev(b):
        return torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)

    X_, W_, dY_ = to_dev(Xb), to_dev(Wb), to_dev(dYb)
    Y_ = torch.empty((M_, N_), dtype=torch.bfloat16, device=dev)
    dX_ = torch.empty((M_, K_), dtype=torch.bfloat16, device=dev)
    dW_ = torch.empty((N_, K_), dtype=torch.bfloat16, device=dev)
    ws_ = torch.empty(capi.linear_workspace_bytes(M_, K_, N_), dtype=torch.uint8, device=dev)
    signs = syn.rht_signs(0)

    def step():
        capi.nvfp4_linear_fprop(X_, W_, Y_, signs, ws_)
        capi.nvfp4_linear_dgrad(dY_, dX_, 7, signs, ws_)
        capi.nvfp4_linear_wgrad(None, dW_, M_, 7, signs, ws_)

    eager_us = timed(step, iters, 10) * 1e3
    graph_us, graph_err = None, None
    try:
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        graph_us = timed(graph.replay, iters, 10) * 1e3
        del graph
    except Exception as exc:  # reported, not fatal: the eager number stands
        graph_err = str(exc)[:200]
    assert capi.nvfp4_read_status(ws_) == 0
    flops = 3 * 2.0 * M_ * K_ * N_
    return {"workload": "linear layer M=K=N=256, X/W/dY ~ N(0,1) with 1% of entries x50, "
                        "X,dY 1x16, W 16x16, SR on dY, RHT on the wgrad operands",
            "us_per_step_eager": round(eager_us, 2),
            "us_per_step_graph": None if graph_us is None else round(graph_us, 2),
            "graph_error": graph_err,
            "kernel_launches_per_step": 11,
            "tflops_eager": round(flops / (eager_us * 1e-6) / 1e12, 3),
            "bound": "latency (0.1 GFLOP and ~1 MB per step)"}


QUANT_BYTES_PER_EL = 2.0 + 2.0 + 0.5 + 1.0 / 16   # amax read + quantize read + codes + scales
QUANT_ONE_READ_BYTES_PER_EL = 2.0 + 0.5 + 1.0 / 16


def bench_quant_sweep(capi, syn, dev, stream, timed, peaks, n=8192, iters=20):
    """Quantize sweep on 8192 x 8192 bf16 tensors (Gaussian N(0,1), Student-t nu=3,
    Laplace(0,1), fixed seeds 0/1/2, drawn on the device): 1x16 and 16x16 blocks x RNE
    and SR through nvfp4_quantize (tensor amax pass + quantize pass), the RHT
    column orientation (1x16, RNE and SR) through nvfp4_quantize_2d, and the
    standalone 16-point RHT (both axes) through nvfp4_rht.  GB/s counts the
    algorithmic bytes: 4.5625 B/element per quantized orientation (the global amax
    precedes every scale, so the tensor is read twice); the one-read bound (2.5625
    B/element) is given beside it.  The 134 MB input is above the 126 MB L2."""
    import torch
    hbm = peaks["hbm_gbs"]
    el = n * n
    out = {"workload": f"quantize sweep, {n}x{n} bf16 per tensor",
           "bytes_per_element": QUANT_BYTES_PER_EL, "one_read_bytes_per_element": QUANT_ONE_READ_BYTES_PER_EL,
           "hbm_peak_GB/s": hbm, "modes": {}}
    packed = torch.empty(capi.packed_bytes(n, n), dtype=torch.uint8, device=dev)
    sf = torch.empty(capi.scale_bytes(n, n), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(capi.quantize_workspace_bytes(), dtype=torch.uint8, device=dev)
    signs = syn.rht_signs(0)
    worst = None
    for seed, dist in enumerate(("normal", "student_t", "laplace")):
        x = syn.device_bf16(dist, (n, n), seed, dev)
        torch.cuda.synchronize()
        modes = [(f"{dist}/1x16/rne", lambda: capi.nvfp4_quantize(x, 0, 0, 5, packed, sf, g, ws)),
                 (f"{dist}/1x16/sr", lambda: capi.nvfp4_quantize(x, 0, 1, 5, packed, sf, g, ws)),
                 (f"{dist}/16x16/rne", lambda: capi.nvfp4_quantize(x, 1, 0, 5, packed, sf, g, ws)),
                 (f"{dist}/16x16/sr", lambda: capi.nvfp4_quantize(x, 1, 1, 5, packed, sf, g, ws)),
                 (f"{dist}/rht_cols_1x16/rne", lambda: capi.nvfp4_quantize_2d(
                     x, 0, 0, 0, 5, True, signs, None, (packed, sf, g), ws)),
                 (f"{dist}/rht_cols_1x16/sr", lambda: capi.nvfp4_quantize_2d(
                     x, 0, 0, 1, 5, True, signs, None, (packed, sf, g), ws))]
        for name, fn in modes:
            ms = timed(fn, iters, 3)
            gbs = QUANT_BYTES_PER_EL * el / (ms * 1e-3) / 1e9
            out["modes"][name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                                  "one_read_GB/s": round(QUANT_ONE_READ_BYTES_PER_EL * el / (ms * 1e-3) / 1e9, 1)}
            worst = gbs if worst is None else min(worst, gbs)
        assert capi.nvfp4_read_status(ws) == 0
        if dist == "normal":
            y = torch.empty((n, n), dtype=torch.float32, device=dev)
            for axis in (0, 1):
                ms = timed(lambda: capi.nvfp4_rht(x, signs, 16, y, axis=axis), iters, 3)
                gbs = 6.0 * el / (ms * 1e-3) / 1e9   # 2 B read + 4 B (fp32) written
                out["modes"][f"standalone_rht_axis{axis}"] = {
                    "ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                    "bytes_per_element": 6.0}
            del y
        del x
    out["min_frac_hbm_quantize"] = round(worst / hbm, 3)
    return out


def bench_gemm_sweep(capi, syn, dev, stream, timed, fp4_peak, iters=10):
    """GEMM shape sweep: square M = N = K in {1024 .. 16384} with both operands
    quantized from N(0,1) bf16 (1x16 RNE), and the skinny wgrad shapes (reduction 32768
    tokens, N, K in {4096, 8192}) whose operands are the RHT column orientation of
    dY [32768, N] (SR) and X [32768, K].  Inputs are drawn on the device.  TFLOP/s =
    2 M N K per launch over its CUDA-event time, against the FP4 peak derived from
    the measured bf16 burst and against the 9 PFLOP/s dense FP4 specification."""
    import torch
    res = {"workload": "GEMM shape sweep (bf16 output)", "fp4_peak_tflops": round(fp4_peak, 1),
           "spec_fp4_tflops": 9000.0, "shapes": {}}
    ws = torch.empty(capi.quantize_workspace_bytes(), dtype=torch.uint8, device=dev)
    signs = syn.rht_signs(0)

    def opbufs(rows, cols):
        return (torch.empty(capi.packed_bytes(rows, cols), dtype=torch.uint8, device=dev),
                torch.empty(capi.scale_bytes(rows, cols), dtype=torch.uint8, device=dev),
                torch.empty(1, dtype=torch.float32, device=dev))

    def run(name, a, b, Mx, Nx, Kx, alpha):
        D = torch.empty((Mx, Nx), dtype=torch.bfloat16, device=dev)
        fn = lambda: capi.nvfp4_gemm(a[0], a[1], b[0], b[1], alpha, Mx, Nx, Kx, D_bf16=D,
                                     scale_a=a[2], scale_b=b[2])
        ms = timed(fn, iters, 3)
        tf = 2.0 * Mx * Nx * Kx / (ms * 1e-3) / 1e12
        res["shapes"][name] = {"M": Mx, "N": Nx, "K": Kx, "ms": round(ms, 4), "tflops": round(tf, 1),
                               "frac_fp4_peak": round(tf / fp4_peak, 3), "frac_spec_9pf": round(tf / 9000.0, 3)}

    for n in syn.GEMM_SQUARE:
        x = syn.device_bf16("normal", (n, n), 10 + n, dev)
        w = syn.device_bf16("normal", (n, n), 20 + n, dev)
        a, b = opbufs(n, n), opbufs(n, n)
        capi.nvfp4_quantize(x, 0, 0, 0, *a, ws)
        capi.nvfp4_quantize(w, 0, 0, 0, *b, ws)
        del x, w
        run(f"square_{n}", a, b, n, n, n, 1.0)
        del a, b
    red = 32768
    for (Nn, Kk) in syn.GEMM_SKINNY_WGRAD:
        dy = syn.device_bf16("normal", (red, Nn), 30 + Nn, dev)
        xx = syn.device_bf16("normal", (red, Kk), 40 + Kk, dev)
        a, b = opbufs(Nn, red), opbufs(Kk, red)
        capi.nvfp4_quantize_2d(dy, 0, 0, 1, 11, True, signs, None, a, ws)
        capi.nvfp4_quantize_2d(xx, 0, 0, 0, 0, True, signs, None, b, ws)
        del dy, xx
        run(f"wgrad_N{Nn}_K{Kk}_red{red}", a, b, Nn, Kk, red, 1.0 / 16)
        del a, b
    assert capi.nvfp4_read_status(ws) == 0
    big = [v["frac_fp4_peak"] for k, v in res["shapes"].items() if v["M"] * v["N"] * v["K"] >= 4096 ** 3]
    res["min_frac_fp4_peak_large"] = min(big) if big else None
    return res


def moe_step_bench(capi, syn, dev, stream, timed, max_over_ranks, world, iters):
    """Expert layer of the MoE config: gather routed token rows, NVFP4 fprop / dgrad /
    wgrad of all experts (grouped: one launch per kernel kind over all experts), and
    combine the routed input gradients.  Useful FLOPs count the routed tokens only
    (padding rows excluded).  The per-expert calls are timed beside it."""
    import torch
    s = syn.MOE
    E, K, N, T, k = s["experts"], s["hidden"], s["ffn"], s["tokens"], s["topk"]
    d = syn.moe_inputs(T, E, K, N, k, s["zipf_s"], seed=0, pad=128)
    rows = int(d["group_rows"].sum())

    def to_dev(b):
        return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(torch.bfloat16)

    x_tok = to_dev(d["X"])
    W = to_dev(d["W"].reshape(E * N, K)).view(E, N, K)
    dY = to_dev(d["dY"])
    row_src = torch.from_numpy(d["row_src"]).to(dev)
    slots = torch.from_numpy(d["slots"]).to(dev)
    X_perm = torch.empty((rows, K), dtype=torch.bfloat16, device=dev)
    Y = torch.empty((rows, N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((rows, K), dtype=torch.bfloat16, device=dev)
    dX_tok = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
    dW = torch.empty((E, N, K), dtype=torch.bfloat16, device=dev)
    gws = torch.empty(capi.moe_grouped_workspace_bytes(d["group_rows"], K, N), dtype=torch.uint8,
                      device=dev)
    signs = syn.rht_signs(0)

    def step():  # the routing gather is fused into the quantization of X
        capi.nvfp4_moe_grouped_fprop_gather(x_tok, row_src, W, Y, d["group_rows"], signs, gws)
        capi.nvfp4_moe_grouped_dgrad(dY, dX, d["group_rows"], 7, signs, gws)
        capi.nvfp4_moe_combine(dX, slots, dX_tok)
        capi.nvfp4_moe_grouped_wgrad(dW, d["group_rows"], gws)

    ms = max_over_ranks(timed(step, iters, 3))
    assert capi.nvfp4_read_status(gws) == 0
    pws = torch.empty(capi.moe_workspace_bytes(d["group_rows"], K, N), dtype=torch.uint8, device=dev)

    def step_per_expert():
        capi.nvfp4_moe_gather(x_tok, row_src, X_perm)
        capi.nvfp4_moe_linear_fprop(X_perm, W, Y, d["group_rows"], signs, pws)
        capi.nvfp4_moe_linear_dgrad(dY, dX, d["group_rows"], 7, signs, pws)
        capi.nvfp4_moe_combine(dX, slots, dX_tok)
        capi.nvfp4_moe_linear_wgrad(dW, d["group_rows"], 7, signs, pws)

    ms_pe = max_over_ranks(timed(step_per_expert, 3, 3))
    useful = 3 * 2.0 * T * k * K * N
    padded = 3 * 2.0 * rows * K * N
    return {"workload": "MoE expert layer: 64 experts, hidden 2048, FFN 1024, 16384 tokens, "
                        "top-4 of Zipf(1.1), expert segments padded to 128 rows; gather fused into "
                        "the quantization of X, grouped GEMMs on two-SM 256x256 tiles",
            "ms_per_step": round(ms, 4),
            "useful_tflops": round(world * useful / (ms * 1e-3) / 1e12, 1),
            "executed_tflops_incl_padding": round(world * padded / (ms * 1e-3) / 1e12, 1),
            "per_expert_calls_ms_per_step": round(ms_pe, 4),
            "routed_rows": T * k, "padded_rows": rows,
            "group_rows_max_min": [int(d["group_rows"].max()), int(d["group_rows"].min())]}


# --------------------------------------------------------------------------- oracle
def oracle_sample_step(Ms, Ks, Ns, nthreads=0):
    """The same step (same recipe, same distributions) on a reduced shape, run by the
    CPU oracle: six quantizations and three fp64 GEMMs.  Returns seconds."""
    from nvfp4_bit_quantized_amax_b200 import synthetic as syn
    from oracle import oracle as ora

    X, W, dY = syn.mlp_inputs(Ms, Ks, Ns, seed=0)
    s = syn.rht_signs(0)
    t0 = time.perf_counter()
    q = {}
    for name, x, orient, rht, bm, rnd in (("xr", X, 0, 0, 0, 0), ("xc", X, 1, 1, 0, 0),
                                          ("wr", W, 0, 0, 1, 0), ("wc", W, 1, 0, 1, 0),
                                          ("dr", dY, 0, 0, 0, 1), ("dc", dY, 1, 1, 0, 1)):
        p, sf, g, _ = ora.quantize(x, orient, rht, s, bm, rnd, 7, nthreads=nthreads)
        q[name] = (p, sf, float(g))
    for a, b, alpha in (("xr", "wr", 1.0), ("dr", "wc", 1.0), ("dc", "xc", 1.0 / 16)):
        pa, sa, ga = q[a]
        pb, sb, gb = q[b]
        ora.gemm(pa, sa, pb, sb, alpha * ga * gb, nthreads=nthreads)
    return time.perf_counter() - t0


ORACLE_SAMPLE = (256, 256, 512)  # M, K, N of the oracle's sample step (both CPU legs)


def cpu_baseline(budget_s=15.0):
    """The oracle on the host cores, on the same sample step as the reference arm:
    with every core (the reported value) and with one thread.  Each is repeated
    until about budget_s / 2 of CPU time has passed."""
    cores = os.cpu_count() or 1
    flops = 3 * 2.0 * ORACLE_SAMPLE[0] * ORACLE_SAMPLE[1] * ORACLE_SAMPLE[2]

    def per_step(nthreads):
        times = [oracle_sample_step(*ORACLE_SAMPLE, nthreads=nthreads)]
        while sum(times) < budget_s / 2 and len(times) < 50:
            times.append(oracle_sample_step(*ORACLE_SAMPLE, nthreads=nthreads))
        return sum(times) / len(times), len(times)

    t_all, n_all = per_step(0)
    t_one, n_one = per_step(1)
    return {"value": round(flops / t_all / 1e12, 6), "unit": "TFLOPS", "cores": cores,
            "kind": "oracle",
            "value_1_thread": round(flops / t_one / 1e12, 6),
            "sample": f"whole step (6 quantizations + 3 fp64 GEMMs) at M={ORACLE_SAMPLE[0]} "
                      f"K={ORACLE_SAMPLE[1]} N={ORACLE_SAMPLE[2]} instead of 8192/5120/20480, same "
                      f"recipe and distributions (the reference arm's sample); {t_all * 1e3:.0f} ms "
                      f"per step on {cores} threads ({n_all} steps), {t_one * 1e3:.0f} ms on 1 thread "
                      f"({n_one} steps)"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    cores = os.cpu_count() or 1
    shape = ORACLE_SAMPLE
    flops = 3 * 2.0 * shape[0] * shape[1] * shape[2]
    for _ in range(max(args.warmup, 3)):
        oracle_sample_step(*shape)
    times = [oracle_sample_step(*shape) for _ in range(args.steps)]
    per = sum(times) / len(times)
    value = flops / per / 1e12
    sample = (f"whole step at M={shape[0]} K={shape[1]} N={shape[2]} per timed step (same recipe "
              f"and distributions as the 8192/5120/20480 workload)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(per * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "N": N, "parallelism": "single"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_kernel(args):
    """Single-kernel mode for profilers: quantize synthetic bf16 inputs of the given
    shape, then launch one kernel `--steps` times.  --kernel gemm (M,N,K),
    quant-x / quant-w / quant-dy (rows,cols): the three fused quantize passes;
    moe-step: the grouped MoE expert-layer step (no shape)."""
    import torch

    from nvfp4_bit_quantized_amax_b200 import capi
    from nvfp4_bit_quantized_amax_b200 import synthetic as syn

    dev = torch.device("cuda", 0)
    dims = [int(v) for v in args.shape.split(",")]
    signs = syn.rht_signs(0)

    def to_dev(b):
        return torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)

    def operand(rows, cols, seed):
        x = to_dev(syn.normal_bf16((rows, cols), seed))
        op = (torch.empty(capi.packed_bytes(rows, cols), dtype=torch.uint8, device=dev),
              torch.empty(capi.scale_bytes(rows, cols), dtype=torch.uint8, device=dev),
              torch.empty(1, dtype=torch.float32, device=dev))
        ws = torch.empty(capi.quantize_workspace_bytes(), dtype=torch.uint8, device=dev)
        capi.nvfp4_quantize(x, 0, 0, 0, *op, ws)
        return op

    if args.kernel == "moe-step":
        s_ = syn.MOE
        E, K_, N_, T_, k_ = s_["experts"], s_["hidden"], s_["ffn"], s_["tokens"], s_["topk"]
        d = syn.moe_inputs(T_, E, K_, N_, k_, s_["zipf_s"], seed=0, pad=128)
        rows = int(d["group_rows"].sum())
        x_tok, dY = to_dev(d["X"]), to_dev(d["dY"])
        Wm = to_dev(d["W"].reshape(E * N_, K_)).view(E, N_, K_)
        row_src = torch.from_numpy(d["row_src"]).to(dev)
        slots = torch.from_numpy(d["slots"]).to(dev)
        X_perm = torch.empty((rows, K_), dtype=torch.bfloat16, device=dev)
        Y = torch.empty((rows, N_), dtype=torch.bfloat16, device=dev)
        dX = torch.empty((rows, K_), dtype=torch.bfloat16, device=dev)
        dX_tok = torch.empty((T_, K_), dtype=torch.bfloat16, device=dev)
        dW = torch.empty((E, N_, K_), dtype=torch.bfloat16, device=dev)
        gws = torch.empty(capi.moe_grouped_workspace_bytes(d["group_rows"], K_, N_), dtype=torch.uint8,
                          device=dev)

        def fn():
            capi.nvfp4_moe_grouped_fprop_gather(x_tok, row_src, Wm, Y, d["group_rows"], signs, gws)
            capi.nvfp4_moe_grouped_dgrad(dY, dX, d["group_rows"], 7, signs, gws)
            capi.nvfp4_moe_combine(dX, slots, dX_tok)
            capi.nvfp4_moe_grouped_wgrad(dW, d["group_rows"], gws)
    elif args.kernel == "gemm":
        Mk, Nk, Kk = dims
        a, b = operand(Mk, Kk, 1), operand(Nk, Kk, 2)
        D = torch.empty((Mk, Nk), dtype=torch.bfloat16, device=dev)
        fn = lambda: capi.nvfp4_gemm(a[0], a[1], b[0], b[1], 1.0, Mk, Nk, Kk, D_bf16=D,
                                     scale_a=a[2], scale_b=b[2])
    else:
        rows, cols = dims
        x = to_dev(syn.normal_bf16((rows, cols), 3))
        ws = torch.empty(capi.quantize_workspace_bytes(), dtype=torch.uint8, device=dev)

        def bufs(r, c):
            return (torch.empty(capi.packed_bytes(r, c), dtype=torch.uint8, device=dev),
                    torch.empty(capi.scale_bytes(r, c), dtype=torch.uint8, device=dev),
                    torch.empty(1, dtype=torch.float32, device=dev))
        ro, co = bufs(rows, cols), bufs(cols, rows)
        bm, rr, cr, rht = {"quant-x": (0, 0, 0, 1), "quant-w": (1, 0, 0, 0),
                           "quant-dy": (0, 1, 1, 1)}[args.kernel]
        fn = lambda: capi.nvfp4_quantize_2d(x, bm, rr, cr, 5, rht, signs, ro, co, ws)
    for _ in range(args.steps):
        fn()
    torch.cuda.synchronize()
    print(json.dumps({"kernel": args.kernel, "shape": dims, "launches": args.steps}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", default=None, choices=["gemm", "quant-x", "quant-w", "quant-dy", "moe-step"],
                    help="profiler mode: launch one kernel kind only")
    ap.add_argument("--shape", default="4096,8192,5120")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-moe", action="store_true")
    ap.add_argument("--no-sweeps", action="store_true",
                    help="skip the 256^3 step, the 8192^2 quantize sweep and the GEMM shape sweep")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per GEMM launch from an ncu capture of this kernel")
    args = ap.parse_args()
    rank, world, local_rank = env_rank()
    if args.kernel:
        run_kernel(args)
    elif args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
