#!/usr/bin/env python
"""Benchmark of the STQ1_0 decode GEMV (and MoE gate/up) on B200.

Default (N = 1) workload: decode GEMV on expert-shaped STQ1_0 matrices,
[4096, 7168] (fused gate+up of 2 x 2048 rows over hidden 7168), encoded by the
WLS / weighted-zero-placement encoder with importance from 512 synthetic
calibration vectors; bf16 activations, batch 1, fp32 accumulation.

One step = one decode pass over a stack of L = 64 distinct such matrices
(308 MB of packed weights, more than twice the 126 MB L2), i.e. 64 GEMV
launches replayed from a CUDA graph, the same activation vector each time.
``value`` = packed weight bytes streamed per second (GB/s) over the timed
steps.  Extra keys report the same GEMV at batch 2/4/8 and the MoE decode
gate/up workload (16 tokens, top-8 of 256 experts) in tokens/s.

Multi-GPU: every rank runs the same per-rank workload (weak scaling, no
collective on the data path); the time is the max over ranks.

``--impl reference`` times the CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = ("STQ1_0 GEMV packed-weight GB/s & % HBM roofline; MoE gate/up tokens/s (1×B200)")
N_ROWS, K_COLS = 4096, 7168
PACKED = N_ROWS * (K_COLS // 256) * 42          # 4,816,896 bytes per matrix
STACK = 64                                      # matrices per step
FP8_OVER_BF16 = 2.0                        # nominal dense fp8 / bf16 tensor rate on B200
HBM_NOMINAL_GBS = 8000.0


def measure_fp8_peak(torch, device, n=8192, reps=10):
    """Dense E4M3 tensor throughput on this GPU, TFLOP/s: best of `reps`
    torch._scaled_mm calls on n^3 (fp32 accumulation, bf16 output)."""
    a = torch.randn((n, n), device=device).to(torch.float8_e4m3fn)
    b = torch.randn((n, n), device=device).to(torch.float8_e4m3fn).t()   # column-major operand
    one = torch.ones((), dtype=torch.float32, device=device)
    for _ in range(3):
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    del a, b
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("bf16_tflops", 1672.0)), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------
# multi-rank aggregation (weak scaling: every rank runs the per-rank workload)
# ---------------------------------------------------------------------------


def max_over_ranks(ms: float, device=None) -> float:
    """The slowest rank's elapsed time (all ranks take part; no-op at world 1)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return world * units_per_rank / (ms * 1e-3)


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, sampled from a thread)
# ---------------------------------------------------------------------------


class ClockSampler:
    REASONS = {
        "hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index: int, period_s: float = 0.0):
        # period 0: sample back to back (each NVML query takes a while), so that
        # a timed region of a few milliseconds still gets several samples
        self.index, self.period = index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._first = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._first.set()
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
            self._first.wait(1.0)          # the sampler is running when the region starts
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# workload construction
# ---------------------------------------------------------------------------


def build_stack(torch, stq1, device):
    """L distinct encoded matrices on the device: the WLS-encoded decode matrix and
    copies whose block order is rotated (same statistics, distinct bytes)."""
    import workloads
    w, h, x = workloads.decode_gemv_inputs()
    packed = stq1.quantize_ref(w, h, mode="sherry", rounds=3)
    base = torch.from_numpy(packed).to(device)
    blocks = base.view(-1, 42)
    nblk = blocks.shape[0]
    stack = torch.empty((STACK, PACKED), dtype=torch.uint8, device=device)
    for i in range(STACK):
        shift = (i * 7919) % nblk
        stack[i].view(-1, 42).copy_(torch.roll(blocks, shifts=shift, dims=0))
    return packed, stack, x


def time_graph(torch, fn, steps, warmup, stream):
    """Captures one step into a CUDA graph, runs `warmup` replays, then times `steps`."""
    with torch.cuda.stream(stream):
        fn()                                  # configure kernels before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    return g


def run_gpu(args):
    import torch
    import torch.distributed as dist
    import sub_bit_sparse_b200 as stq1

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    hbm_peak, bf16_peak, peak_kind = _peaks()

    packed, stack, x_bits = build_stack(torch, stq1, device)
    xs = torch.from_numpy(x_bits.view(np.int16)).to(device).view(torch.bfloat16)   # [8, K]
    y_all = torch.empty((STACK, 8, N_ROWS), dtype=torch.float32, device=device)
    ws = stq1.workspace(max(stq1.LIB.stq1_gemv_workspace(N_ROWS, K_COLS, b) for b in (1, 2, 4, 8)), device)

    def make_step(b):
        # a chain of GEMVs over known matrices: each call also brings the next
        # matrix into L2 (stq1_gemv_prefetch)
        xb = xs[:b].contiguous()
        def step():
            for i in range(STACK):
                stq1.gemv(stack[i], xb, N_ROWS, K_COLS, out=y_all[i, :b], ws=ws, prefetch=stack[(i + 1) % STACK])
        return step

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(g, steps):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(steps):
                g.replay()
            end.record(stream)
        torch.cuda.synchronize()
        ms = start.elapsed_time(end)
        barrier()
        return max_over_ranks(ms, device)

    # --- headline: batch 1 ---
    g1 = time_graph(torch, make_step(1), args.steps, args.warmup, stream)
    with ClockSampler(local) as clk:
        ms = timed(g1, args.steps)
    ms_step = ms / args.steps
    launch_ms = ms_step / STACK
    bytes_step = STACK * PACKED
    value = whole_job_rate(bytes_step * args.steps, world, ms) / 1e9
    achieved = PACKED / (launch_ms * 1e-3) / 1e9

    # --- the same GEMV at larger batches ---
    batches = {}
    for b in (2, 4, 8):
        gb = time_graph(torch, make_step(b), max(1, args.steps // 4), 3, stream)
        msb = timed(gb, max(1, args.steps // 4)) / max(1, args.steps // 4)
        batches[str(b)] = {"gbs": round(bytes_step / (msb * 1e-3) / 1e9, 1),
                           "ms_per_step": round(msb, 4)}
        del gb

    # --- MoE decode gate/up (16 tokens, top-8 of 256 experts) ---
    moe = run_moe(torch, stq1, device, stream, args, world, timed)

    # --- a whole routed MoE feed-forward layer at decode ---
    try:
        ffn = run_moe_ffn(torch, stq1, device, stream, args, world, timed)
    except Exception as exc:  # reported, never hidden
        ffn = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    # --- MoE prefill gate/up on the tensor-core tile path (4096 tokens) ---
    try:
        prefill = run_prefill(torch, stq1, device, stream, args, world, timed, bf16_peak)
    except Exception as exc:  # reported, never hidden
        prefill = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    # --- encoders (GPU and host) ---
    try:
        encoder = run_encoder(torch, stq1, device, stream)
    except Exception as exc:  # reported, never hidden
        encoder = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    # --- mixed-precision allocation: layer scoring on the tensor cores ---
    try:
        mix = run_mix(torch, stq1, device, stream, args, world, timed, bf16_peak, hbm_peak)
    except Exception as exc:  # reported, never hidden
        mix = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    # --- crossover between the kernels on [18432, 7168], batches 1 .. 1024 ---
    try:
        xover = crossover(torch, stq1, device, stream, (1, 4, 16, 64, 256, 1024), reps_cap=1024)
    except Exception as exc:  # reported, never hidden
        xover = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    # --- end to end through the public API with host buffers ---
    e2e = run_e2e(torch, stq1, device, stream, stack, xs, ws, args, world, barrier)

    # --- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only) ---
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(packed, x_bits, seconds=args.cpu_seconds)

    traffic = kernel_traffic("lut_gemv_kernel<1>")
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": bench_config(world),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": traffic,
                     "peak_kind": peak_kind, "frac_of_nominal_8tbs": round(achieved / HBM_NOMINAL_GBS, 4),
                     "kernel": "lut_gemv_kernel<1>", "algorithmic_bytes_per_launch": PACKED},
        "gemv_batches": batches,
        "moe_decode": moe,
        "moe_prefill": prefill,
        "moe_ffn_decode": ffn,
        "encoder": encoder,
        "mix_allocation": mix,
        "crossover": xover,
        "e2e": e2e,
        "gpu_launches": args.steps * STACK,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g1
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_moe(torch, stq1, device, stream, args, world, timed):
    import workloads
    E, n, k = 256, N_ROWS, K_COLS
    eb = PACKED
    flat = _random_expert_bank(torch, device, E, 2024)
    x, ids, wts = workloads.moe_decode_inputs()
    xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    idd = torch.from_numpy(ids).to(device)
    wd = torch.from_numpy(wts).to(device)
    y = torch.empty((16, 8, n), dtype=torch.float32, device=device)
    ws = stq1.workspace(stq1.LIB.stq1_moe_workspace(16, 8, E, n, k, 0), device, kind="moe")

    def step():
        stq1.moe_gateup(flat, xd, idd, wd, n, k, E, out=y, ws=ws)

    steps = max(1, args.steps // 8)
    gm = time_graph(torch, step, steps, 3, stream)
    ms = timed(gm, steps) / steps
    uniq = len(np.unique(ids))
    del gm
    return {"tokens_per_s": round(world * 16 / (ms * 1e-3), 1), "ms_per_call": round(ms, 4),
            "unique_experts": int(uniq), "expert_bytes_read": int(uniq * eb),
            "gbs": round(uniq * eb / (ms * 1e-3) / 1e9, 1),
            "config": "256 experts x [4096, 7168] STQ1_0, 16 tokens, Zipf(1.1) top-8, unweighted"}


def _random_expert_bank(torch, device, E, seed, packed=None, d_mean=0.058):
    """E random but valid STQ1_0 matrices (default [4096, 7168]) on the device:
    uniform code bytes, fp16 scales near d_mean (0.058 = the amax of 256
    N(0, 0.02^2) weights)."""
    packed = PACKED if packed is None else packed
    flat = torch.empty(E * packed, dtype=torch.uint8, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    flat.copy_(torch.randint(0, 256, (E * packed,), dtype=torch.uint8, device=device, generator=g))
    blk = flat.view(-1, 42)
    d = (d_mean * (1 + 0.1 * torch.randn(blk.shape[0], device=device, generator=g))).to(torch.float16)
    blk[:, 0:2].copy_(d.view(torch.uint8).view(-1, 2))
    return flat


def run_moe_ffn(torch, stq1, device, stream, args, world, timed):
    """A routed MoE feed-forward layer at decode: 16 tokens, top-8 of 256 experts,
    gate/up [4096, 7168] -> SwiGLU -> down [7168, 2048] -> combine."""
    import workloads
    E, n, hidden = 256, N_ROWS, K_COLS
    gu = _random_expert_bank(torch, device, E, 2024)
    down_packed = hidden * (n // 2) // 256 * 42
    dn = _random_expert_bank(torch, device, E, 2025, packed=down_packed, d_mean=0.004)
    x, ids, wts = workloads.moe_decode_inputs()
    xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    idd = torch.from_numpy(ids).to(device)
    wd = torch.from_numpy(wts).to(device)
    out = torch.empty((16, hidden), dtype=torch.float32, device=device)
    ws = stq1.workspace(stq1.LIB.stq1_moe_ffn_workspace(16, 8, E, n, hidden, 0), device, kind="ffn")

    def step():
        stq1.moe_ffn(gu, dn, xd, idd, wd, n, hidden, E, out=out, ws=ws)

    steps = max(1, args.steps // 8)
    gm = time_graph(torch, step, steps, 3, stream)
    ms = timed(gm, steps) / steps
    uniq = len(np.unique(ids))
    del gm
    return {"tokens_per_s": round(world * 16 / (ms * 1e-3), 1), "ms_per_call": round(ms, 4),
            "expert_bytes_read": int(uniq * (PACKED + down_packed)),
            "gbs": round(uniq * (PACKED + down_packed) / (ms * 1e-3) / 1e9, 1),
            "config": "256 experts, gate/up [4096, 7168] + down [7168, 2048] STQ1_0, 16 tokens, Zipf(1.1) "
                      "top-8, SwiGLU (bf16) and routing-weighted combine"}


def run_prefill(torch, stq1, device, stream, args, world, timed, bf16_peak):
    """MoE prefill gate/up: 4096 tokens x top-8 of 256 experts (32,768 pairs), on
    the bf16 tile path and on its fp8 variant.  The fp8 error is measured
    against the bf16 result (itself within 1e-3 * sum|W x| of the exact one)."""
    import workloads
    E, n, k = 256, N_ROWS, K_COLS
    flat = _random_expert_bank(torch, device, E, 4096)
    x, ids, _ = workloads.moe_prefill_inputs()
    xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    idd = torch.from_numpy(ids).to(device)
    flops = 2.0 * 4096 * 8 * n * k
    out = {}
    ys = {}
    try:
        fp8_peak, fp8_kind = measure_fp8_peak(torch, device), "measured in this run (torch._scaled_mm E4M3 8192^3)"
    except Exception as exc:  # reported, never hidden
        fp8_peak, fp8_kind = bf16_peak * FP8_OVER_BF16, f"measured bf16 x 2 (nominal ratio; fp8 probe failed: {exc})"[:200]
    for name, flags, peak in (("bf16", 0, bf16_peak), ("fp8", stq1.MOE_FP8, fp8_peak)):
        y = torch.empty((4096, 8, n), dtype=torch.float32, device=device)
        ws = stq1.workspace(stq1.LIB.stq1_moe_workspace(4096, 8, E, n, k, flags), device, kind="moe")

        def step():
            stq1.moe_gateup(flat, xd, idd, None, n, k, E, flags=flags, out=y, ws=ws)

        steps = max(2, args.steps // 40)
        gp = time_graph(torch, step, steps, 3, stream)
        ms = timed(gp, steps) / steps
        del gp
        tflops = flops / (ms * 1e-3) / 1e12
        out[name] = {"tokens_per_s": round(world * 4096 / (ms * 1e-3), 1), "ms_per_call": round(ms, 4),
                     "tflops_dense_equiv": round(tflops, 1), "peak_tflops": round(peak, 1),
                     "tensor_frac": round(tflops / peak, 4)}
        ys[name] = y
        del ws
    d = (ys["fp8"] - ys["bf16"]).abs_()
    ref = ys["bf16"].abs()
    scale = float(ref.mean())
    out["fp8"]["error_vs_bf16"] = {
        "mean_abs_over_mean_abs_y": round(float(d.mean()) / scale, 6),
        "max_abs_over_mean_abs_y": round(float(d.max()) / scale, 6),
        "rel_l2": round(float(torch.linalg.vector_norm(d) / torch.linalg.vector_norm(ys["bf16"])), 6)}
    del ys, d, ref
    res = out["bf16"]
    res["bf16_peak_tflops"] = bf16_peak
    res["fp8"] = out["fp8"]
    res["fp8"]["peak_kind"] = fp8_kind
    res["config"] = ("256 experts x [4096, 7168] STQ1_0, 4096 tokens, Zipf(1.1) top-8 (32,768 pairs), "
                     "tcgen05 tiles, A = decoded +/-1 in TMEM (bf16, kind::f16; fp8: E4M3, kind::f8f6f4 with "
                     "per-token E4M3 activations), fp32 per-block scale")
    return res


def run_encoder(torch, stq1, device, stream):
    """Encoders on the decode matrix [4096, 7168]: GPU (stq1_quantize) and host
    (stq1_quantize_ref, all cores), weights per second; the GPU and host bytes
    are checked equal."""
    import workloads
    import time
    w, h, _ = workloads.decode_gemv_inputs()
    n, k = w.shape
    wd = torch.from_numpy(w).to(device)
    hd = torch.from_numpy(h).to(device)
    res = {}
    outs = {}
    for mode, hh in (("plain", None), ("sherry", hd)):
        with torch.cuda.stream(stream):
            o = stq1.quantize_gpu(wd, hh, mode=mode)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 5
            e0.record(stream)
            for _ in range(reps):
                stq1.quantize_gpu(wd, hh, mode=mode, out=o)
            e1.record(stream)
        torch.cuda.synchronize()
        res[f"gpu_{mode}_weights_per_s"] = round(n * k * reps / (e0.elapsed_time(e1) * 1e-3), 1)
        outs[mode] = o.cpu().numpy()
    t0 = time.perf_counter()
    host = stq1.quantize_ref(w, h, mode="sherry")
    res["host_sherry_weights_per_s"] = round(n * k / (time.perf_counter() - t0), 1)
    res["host_threads"] = os.cpu_count()
    res["gpu_equals_host"] = bool(np.array_equal(host, outs["sherry"]))
    res["config"] = "decode matrix [4096, 7168], Sherry 3 rounds with calibration importance; plain = amax"
    return res


MIX_LAYERS, MIX_N, MIX_K, MIX_CAL = 77, 4096, 7168, 512


def _mix_inputs(torch, device, n_layers, seed=2025):
    import workloads
    w = torch.empty((n_layers, MIX_N, MIX_K), dtype=torch.float32, device=device)
    x = torch.empty((n_layers, MIX_CAL, MIX_K), dtype=torch.bfloat16, device=device)
    for l in range(n_layers):
        wl, xl = workloads.mix_layer_torch(MIX_N, MIX_K, MIX_CAL, l, seed, device)
        w[l].copy_(wl)
        x[l].copy_(xl)
        del wl, xl
    return w, x


def _ranks(v):
    r = np.empty(len(v))
    r[np.argsort(v, kind="stable")] = np.arange(len(v))
    return r


def run_mix(torch, stq1, device, stream, args, world, timed, bf16_peak, hbm_peak):
    """Mixed-precision allocation study: 77 layers of one [4096, 7168] matrix
    each with 512 calibration rows; STQ1_0 (Sherry, 3 rounds) versus STQ2
    (importance-fitted, 3 rounds) for every layer, both scored under the full and the diagonal Hessian on the
    tensor cores, then the greedy per-byte allocation at the pages' split
    (29 layers low, 48 high)."""
    L, n, k, nc = MIX_LAYERS, MIX_N, MIX_K, MIX_CAL
    w, x = _mix_inputs(torch, device, L)
    with torch.cuda.stream(stream):
        h = stq1.hessian_diag(x)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        p_low = torch.cat([stq1.quantize_gpu(w[l], h[l], mode="sherry", rounds=3) for l in range(L)])
        e1.record(stream)
        p_high = torch.cat([stq1.stq2_quantize(w[l], h[l], rounds=3) for l in range(L)])
        e2 = torch.cuda.Event(enable_timing=True)
        e2.record(stream)
    torch.cuda.synchronize()
    enc_ms = e0.elapsed_time(e1)
    enc2_ms = e1.elapsed_time(e2)
    out_low = torch.empty((L, 2), dtype=torch.float64, device=device)
    out_high = torch.empty((L, 2), dtype=torch.float64, device=device)
    flops = 2.0 * L * n * k * nc
    res = {}
    for name, fmt, pk, o, bb in (("stq1_0", stq1.FMT_STQ1_0, p_low, out_low, 42),
                                 ("stq2", stq1.FMT_STQ2, p_high, out_high, 66)):
        def step():
            stq1.hessian_error(fmt, pk, w, x, h, out=o)
        steps = 5
        g = time_graph(torch, step, steps, 3, stream)
        ms = timed(g, steps) / steps
        del g
        nbytes = L * (n * k * 4 + n * k // 256 * bb + nc * k * 2 + k * 4)
        t_hbm, t_tc = nbytes / (hbm_peak * 1e9), flops / (bf16_peak * 1e12)
        res[name] = {"ms_per_call": round(ms, 4), "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                     "tflops": round(flops / (ms * 1e-3) / 1e12, 1),
                     "hbm_frac": round(nbytes / (ms * 1e-3) / 1e9 / hbm_peak, 4),
                     "tensor_frac": round(flops / (ms * 1e-3) / 1e12 / bf16_peak, 4),
                     "bound": "hbm" if t_hbm >= t_tc else "tensor",
                     "roofline_frac": round(max(t_hbm, t_tc) / (ms * 1e-3), 4),
                     "algorithmic_bytes": nbytes, "flops": flops}
    torch.cuda.synchronize()
    assert stq1.status() == 0
    el, eh = out_low.cpu().numpy(), out_high.cpu().numpy()
    b_low, b_high = float(n * k // 256 * 42), float(n * k // 256 * 66)
    bl, bh = np.full(L, b_low), np.full(L, b_high)
    budget = 29 * b_low + 48 * b_high
    import time
    t0 = time.perf_counter()
    pick_full = stq1.mix_allocate(el[:, 0], eh[:, 0], bl, bh, budget)
    alloc_ms = (time.perf_counter() - t0) * 1e3
    pick_diag = stq1.mix_allocate(el[:, 1], eh[:, 1], bl, bh, budget)
    gain_full = (el[:, 0] - eh[:, 0]) / (bh - bl)
    gain_diag = (el[:, 1] - eh[:, 1]) / (bh - bl)
    rf, rd = _ranks(gain_full), _ranks(gain_diag)
    spearman = float(np.corrcoef(rf, rd)[0, 1])
    sens_rank = float(np.corrcoef(_ranks(el[:, 0]), _ranks(el[:, 1]))[0, 1])

    def total(pick):
        return float(np.sum(np.where(pick, eh[:, 0], el[:, 0])))

    res.update({
        "layers": L, "layer_shape": [n, k], "calibration_rows": nc,
        "picked_high_full": int(pick_full.sum()), "picked_high_diag": int(pick_diag.sum()),
        "picks_differ": int(np.sum(pick_full != pick_diag)),
        "full_error_of_full_allocation": total(pick_full),
        "full_error_of_diag_allocation": total(pick_diag),
        "full_error_all_stq1_0": float(el[:, 0].sum()), "full_error_all_stq2": float(eh[:, 0].sum()),
        "spearman_gain_full_vs_diag": round(spearman, 4),
        "spearman_stq1_error_full_vs_diag": round(sens_rank, 4),
        "avg_bpw": round((29 * 1.3125 + 48 * 2.0625) / 77, 4),
        "sherry_encode_ms_all_layers": round(enc_ms, 2), "stq2_encode_ms_all_layers": round(enc2_ms, 2),
        "allocate_ms": round(alloc_ms, 3),
        "kernel": "hess_score_kernel", "peak_hbm_gbs": hbm_peak, "peak_bf16_tflops": bf16_peak,
        "config": "77 layers x [4096, 7168] fp32 weights, 512 bf16 calibration rows each (synthetic: "
                  "correlated channels, weights partly along the shared directions), all layers per call",
    })
    del w, x, p_low, p_high
    torch.cuda.empty_cache()
    return res


def crossover(torch, stq1, device, stream, batches, reps_cap=4096):
    """Crossover between the kernels on one [18432, 7168] matrix with the decode
    matrix's statistics: per batch, each forced path and the library's own
    choice, timed in a CUDA graph of launches over rotating copies larger than
    L2 (GB/s of packed weights and dense-equivalent TFLOP/s): the lookup-table
    kernel, the tensor-core decode kernel (mma.sync), the tcgen05 tile kernel
    and the library's own choice."""
    import workloads
    w, h, x = workloads.crossover_inputs()
    n, k = w.shape
    packed = stq1.quantize_ref(w, h, mode="sherry")
    pb = packed.size
    copies = max(2, (300 * 1024 * 1024) // pb + 1)          # rotate > 2 x L2
    wd = torch.from_numpy(packed).to(device)
    stack = torch.stack([torch.roll(wd.view(-1, 42), shifts=i * 7919, dims=0).reshape(-1) for i in range(copies)])
    del wd
    xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    y = torch.empty((max(batches), n), dtype=torch.float32, device=device)
    paths = (("table", stq1.PATH_TABLE), ("mma", stq1.PATH_MMA), ("tiles", stq1.PATH_TILES), ("auto", stq1.PATH_AUTO))
    need = 0
    try:
        for _, path in paths:                                 # each kernel's plan has its own split
            stq1.set_path(path)
            need = max([need] + [stq1.LIB.stq1_gemv_workspace(n, k, b) for b in batches])
    finally:
        stq1.set_path(stq1.PATH_AUTO)
    ws = stq1.workspace(need, device)
    rows = []
    try:
        for b in batches:
            row = {"batch": b}
            xb = xd[:b].contiguous()
            for name, path in paths:
                stq1.set_path(path)
                reps = max(2, min(copies, reps_cap // b))

                def step():
                    for i in range(reps):
                        stq1.gemv(stack[i % copies], xb, n, k, out=y[:b], ws=ws)

                g = time_graph(torch, step, 1, 3, stream)
                s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                with torch.cuda.stream(stream):
                    s0.record(stream)
                    g.replay()
                    s1.record(stream)
                torch.cuda.synchronize()
                ms = s0.elapsed_time(s1) / reps
                del g
                row[name] = {"us": round(ms * 1e3, 2), "gbs": round(pb / (ms * 1e-3) / 1e9, 1),
                             "tflops": round(2.0 * b * n * k / (ms * 1e-3) / 1e12, 2)}
            rows.append(row)
    finally:
        stq1.set_path(stq1.PATH_AUTO)
    faster = [r["batch"] for r in rows if r["tiles"]["us"] < min(r["table"]["us"], r["mma"]["us"])]
    del stack, y
    return {"matrix": [n, k], "packed_bytes": int(pb), "rows": rows,
            "tiles_faster_from_batch": min(faster) if faster else None,
            "config": "one [18432, 7168] STQ1_0 matrix (decode-matrix statistics, Sherry 3 rounds), bf16 batch "
                      "prefix of x [1024, 7168]; CUDA graph over rotating copies (> 2 x L2); table = lookup-table "
                      "kernel, mma = tensor-core decode kernel, tiles = tcgen05 tile kernel, auto = the library's "
                      "own choice"}


def run_sweep(args):
    """Crossover sweep: the stated batches 1, 4, 16, 64, 256, 1024 plus 2, 8 and
    32 around the crossover."""
    import torch
    import sub_bit_sparse_b200 as stq1
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    res = crossover(torch, stq1, device, stream, (1, 2, 4, 8, 16, 32, 64, 256, 1024))
    for row in res["rows"]:
        print(json.dumps(row), flush=True)
    print(json.dumps({"sweep": "crossover", **res}))


def run_e2e(torch, stq1, device, stream, stack, xs, ws, args, world, barrier):
    """Host buffers: per step copy x in from pinned memory, run the 64 GEMVs, read
    all outputs back to pinned memory.  `value` goes through the C-ABI entry point
    (stq1_gemv_prefetch) with the pointers ready, as a C caller makes the call;
    `python_api` is the same loop through the Python binding (`stq1.gemv`)."""
    xh = torch.empty((1, K_COLS), dtype=torch.bfloat16).pin_memory()
    xh.copy_(xs[:1].cpu())
    yh = torch.empty((STACK, 1, N_ROWS), dtype=torch.float32).pin_memory()
    xd = torch.empty((1, K_COLS), dtype=torch.bfloat16, device=device)
    yd = torch.empty((STACK, 1, N_ROWS), dtype=torch.float32, device=device)
    steps = max(20, args.steps // 2)

    # per-matrix views and pointers made once, as a decode loop over resident weights would
    mats, outs = list(stack.unbind(0)), list(yd.unbind(0))
    nxt = mats[1:] + mats[:1]
    import ctypes as C
    stq1.LIB.stq1_gemv_prefetch                   # loads the library (and checks its version)
    # the same symbol through a handle without declared argument types: the
    # arguments below are already ctypes objects of the C types, so no per-call
    # conversion runs
    call = C.CDLL(stq1.LIB_PATH).stq1_gemv_prefetch
    call.restype = C.c_int
    vp = C.c_void_p
    common = (vp(xd.data_ptr()),)
    tail = (C.c_int64(N_ROWS), C.c_int64(K_COLS), C.c_int(1), vp(ws.data_ptr()), C.c_size_t(ws.numel()))
    # argument tuples built once (ctypes objects of the declared types pass without conversion)
    argv = [(vp(w.data_ptr()),) + common + (vp(y.data_ptr()),) + tail + (vp(wn.data_ptr()), C.c_int64(PACKED),
                                                                           vp(stream.cuda_stream))
            for w, y, wn in zip(mats, outs, nxt)]

    def one_abi():
        xd.copy_(xh, non_blocking=True)
        for a in argv:
            rc = call(*a)
            if rc:
                raise RuntimeError(f"stq1_gemv_prefetch returned {rc}")
        yh.copy_(yd, non_blocking=True)

    def one_py():
        xd.copy_(xh, non_blocking=True)
        for w, y, wn in zip(mats, outs, nxt):
            stq1.gemv(w, xd, N_ROWS, K_COLS, out=y, ws=ws, prefetch=wn)
        yh.copy_(yd, non_blocking=True)

    def timed_loop(one):
        with torch.cuda.stream(stream):
            for _ in range(3):
                one()
        torch.cuda.synchronize()
        barrier()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(steps):
                one()
            end.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(start.elapsed_time(end), device)

    ms = timed_loop(one_abi)
    ms_py = timed_loop(one_py)
    rate = lambda t: round(whole_job_rate(STACK * PACKED * steps, world, t) / 1e9, 1)
    return {"value": rate(ms), "unit": "GB/s",
            "h2d_bytes_per_step": K_COLS * 2, "d2h_bytes_per_step": STACK * N_ROWS * 4,
            "steps": steps, "ms_per_step": round(ms / steps, 4), "route": "C ABI (stq1_gemv_prefetch)",
            "python_api": {"value": rate(ms_py), "ms_per_step": round(ms_py / steps, 4), "route": "stq1.gemv"}}


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------


def _blas_threads():
    """Threads the oracle's fp64 matmul runs on (the BLAS pool; the decode is one thread)."""
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return 1


def _oracle_sample(packed, x_bits, rows):
    import oracle
    rb = (K_COLS // 256) * 42
    sub = packed[: rows * rb]
    return oracle.gemv(sub, x_bits[:1], rows, K_COLS)


def cpu_baseline(packed, x_bits, seconds=10.0):
    """The oracle (decode + fp64 matmul) on row samples of the decode matrix."""
    rows = 256
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < seconds:
        _oracle_sample(packed, x_bits, rows)
        n += 1
    dt = time.perf_counter() - t0
    rb = (K_COLS // 256) * 42
    return {"value": round(n * rows * rb / dt / 1e9, 6), "unit": "GB/s", "cores": _blas_threads(),
            "host_cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{n} oracle GEMVs of {rows} x {K_COLS} rows of the WLS-encoded decode matrix, "
                      f"batch 1, {dt:.1f} s"}


def bench_config(world):
    """The workload both arms report (the reference arm times a bounded sample of it)."""
    return {
        "workload": "STQ1_0 decode GEMV, W [4096, 7168] WLS-encoded (1.3125 bpw), x bf16 batch 1, "
                    "fp32 accumulation; one step = 64 distinct matrices (308 MB packed)",
        "global_batch": 1, "l2": "inputs larger than L2 (64 x 4.8 MB packed matrices rotate)",
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        "launch": "CUDA graph of 64 GEMV launches per step; each launch prefetches the next matrix "
                  "of the chain into L2 (stq1_gemv_prefetch)",
    }


def run_reference(args):
    """The CPU oracle as the reference arm, on a bounded sample per step (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import workloads
    import oracle
    w, h, x = workloads.decode_gemv_inputs()
    rows = 32
    packed = oracle.encode_sherry(w[:rows], h, rounds=3)
    rb = (K_COLS // 256) * 42
    for _ in range(args.warmup):
        oracle.gemv(packed, x[:1], rows, K_COLS)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gemv(packed, x[:1], rows, K_COLS)
    dt = time.perf_counter() - t0
    value = args.steps * rows * rb / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": bench_config(int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": _blas_threads(),
                         "host_cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"each step: decode + fp64 GEMV of {rows} of the 4096 rows x {K_COLS} of the "
                                   "decode matrix, batch 1 (a bounded sample of the workload)"},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def kernel_source_digest():
    """SHA-256 over the table kernel's sources: a DRAM-traffic figure recorded
    for an older version of the kernel no longer applies."""
    h = hashlib.sha256()
    for rel in ("sub_bit_sparse_b200/csrc/gemv_lut.cuh", "sub_bit_sparse_b200/csrc/packed_copy.cuh",
                "sub_bit_sparse_b200/csrc/device_common.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def kernel_traffic(kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the ncu summary in
    profiles/traffic.json, or None when it was taken on other sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(kernel)
    if not ent or ent.get("source_sha256") != kernel_source_digest():
        return None
    return ent.get("dram_bytes_per_launch")


def profile_case(args):
    """Small launch sequence for ncu captures: the decode GEMV on 64 distinct
    [4096, 7168] matrices (308 MB, larger than L2), 32 launches, batch 1, each
    prefetching the next matrix as the bench's chain does (or the MoE decode
    call with --profile-case moe)."""
    import torch
    import sub_bit_sparse_b200 as stq1
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    if args.profile_case == "mix":
        # four layers (about 500 MB of weights, larger than L2), one scoring call each format
        w, x = _mix_inputs(torch, device, 4)
        h = stq1.hessian_diag(x)
        pk = torch.cat([stq1.quantize_gpu(w[l], h[l], mode="sherry", rounds=3) for l in range(4)])
        for _ in range(3):
            o = stq1.hessian_error(stq1.FMT_STQ1_0, pk, w, x, h)
        torch.cuda.synchronize()
        print("profile case done", o.cpu().numpy().tolist())
        return
    if args.profile_case == "encode":
        # two [4096, 7168] fp32 layers (235 MB, larger than L2) with importances;
        # launches alternate Sherry (3 rounds) and STQ2 (3 rounds), so the first
        # two captured launches are one of each, on a layer not read before
        g = torch.Generator(device=device)
        g.manual_seed(7)
        w = torch.randn((2, N_ROWS, K_COLS), device=device, generator=g) * 0.02
        h = torch.rand((K_COLS,), device=device, generator=g)
        clean = torch.empty(64 << 20, dtype=torch.float32, device=device)
        float(clean.sum())
        del clean
        outs = []
        for l in range(2):
            outs.append(stq1.quantize_gpu(w[l], h, mode="sherry", rounds=3))
            outs.append(stq1.stq2_quantize(w[1 - l], h, rounds=3))
        torch.cuda.synchronize()
        print("profile case done", [int(o.view(torch.int16).sum(dtype=torch.int64)) for o in outs])
        return
    if args.profile_case in ("moe", "prefill"):
        stream = torch.cuda.Stream(device)
        fn = run_moe if args.profile_case == "moe" else run_prefill
        extra = () if args.profile_case == "moe" else (1672.0,)
        out = fn(torch, stq1, device, stream, argparse.Namespace(steps=80), 1, lambda g, steps: 1.0, *extra)
        print(json.dumps(out))
        return
    _, stack, x_bits = build_stack(torch, stq1, device)
    xs = torch.from_numpy(x_bits.view(np.int16)).to(device).view(torch.bfloat16)
    y = torch.empty((1, N_ROWS), dtype=torch.float32, device=device)
    ws = stq1.workspace(stq1.LIB.stq1_gemv_workspace(N_ROWS, K_COLS, 1), device)
    # read a buffer larger than L2 first: the dirty lines left by building the
    # stack are written back here, not during the captured launches
    clean = torch.empty(64 << 20, dtype=torch.float32, device=device)
    float(clean.sum())
    del clean
    for i in range(32):
        stq1.gemv(stack[i % STACK], xs[:1], N_ROWS, K_COLS, out=y, ws=ws, prefetch=stack[(i + 1) % STACK])
    torch.cuda.synchronize()
    print("profile case done", float(y.abs().sum()))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", default=None, choices=["gemv", "moe", "prefill", "mix", "encode"])
    ap.add_argument("--sweep", action="store_true", help="crossover sweep (18432 x 7168, batch 1..1024)")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.profile_case:
        profile_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
