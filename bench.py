"""Benchmark of the SVDQuant W4A4 linear layer on B200.

One step = the whole hot path on one batch: smoothing + NVFP4 activation
quantisation + lora-down (one kernel), then the block-scaled 4-bit GEMM with
the lora-up and bias in its epilogue (one kernel), on the FLUX-shaped fused
QKV projection (M=4608 tokens, K=3072, N=9216, rank 32, NVFP4).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is effective TOPS (2*M*N*K dense-
equivalent operations per second, the low-rank flops not counted) summed
over all ranks; ranks run independent replicas (the layer has no exchange
step).  L2 is flushed before every timed step by reading a 256 MiB buffer (a read
leaves only clean lines, so the step pays no write-back of the flush),
outside the step's CUDA-event bracket.  `--impl reference` times the CPU oracle on the
host cores on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
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

WORKLOAD = "qkv"
SEED = 2


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, "fallback"


def _src_hash(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def _traffic(kernel_key, src):
    """dram bytes per launch from the committed ncu summary, or None if the
    kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel_key)
    if not d or d.get("src_sha") != _src_hash(src):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 20 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = str(gpu_index)
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "20", "-i", self.gpu], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def stop(self, t0, t1):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sel = [r for (ts, r) in self.rows if t0 - 0.05 <= ts <= t1 + 0.05] or [r for (_, r) in self.rows]
        if not sel:
            return None
        sm = [float(r[1]) for r in sel if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in sel for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": float(sel[0][2]),
                "reasons": reasons, "samples": len(sel)}


def _oracle_sample(li, rows, reps=1):
    """Times the oracle (as it stands) on `rows` rows: quantise + lora-down +
    fp64 forward.  Weight preparation is done first and not timed."""
    from oracle import svdq as V
    lam = V.smoothing_lambda(li.x, li.w)
    L1, L2 = V.lowrank_factors(li.w, lam, li.shape.rank)
    prep = V.prepare_weights(li.w, lam, L1, L2, li.bias)
    gx = V.act_global_scale(li.x, prep.inv_lam)
    xs = li.x[:rows]
    times = []
    for _ in range(reps):
        t = time.perf_counter()
        V.forward(xs, prep, gx)
        times.append(time.perf_counter() - t)
    return times


def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, li, rank, world):
    if rank != 0:
        return
    K, N = li.shape.K, li.shape.N
    rows = 128
    times = _oracle_sample(li, rows, reps=args.warmup + args.steps)[args.warmup:]
    t = sum(times) / len(times)
    value = 2.0 * rows * N * K / t / 1e12
    line = {
        "impl": "reference", "metric": "fused SVDQuant W4A4 linear effective TOPS", "value": value, "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD} M={li.shape.M} K={K} N={N} rank={li.shape.rank} nvfp4",
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": _cpu_threads(), "kind": "oracle",
                         "sample": f"{rows} of {li.shape.M} rows per step, numpy fp64 oracle"},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, li, rank, world, local_rank):
    import torch
    import synth
    from bit_diffusion_transformer_svdq_b200 import svdq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    svdq.load_library()
    M, K, N, r = li.shape.M, li.shape.K, li.shape.N, li.shape.rank
    stream = torch.cuda.current_stream()

    # ---- offline preparation (untimed): calibration, factorisation, weight prep
    X = torch.from_numpy(li.x_bits.view(np.int16)).to(dev)
    W = torch.from_numpy(li.w).to(dev)
    bias = torch.from_numpy(li.bias_bits.view(np.int16)).to(dev)
    lam = torch.empty(K, dtype=torch.float32, device=dev)
    scratch = torch.empty(2 * K, dtype=torch.float32, device=dev)
    svdq.svdq_smoothing_lambda(X, W, lam, scratch)
    # the offline factoriser: rank-r factors of W_til^T by the library's
    # GPU subspace iteration from a seeded start block
    L1 = torch.empty((r, K), dtype=torch.int16, device=dev)
    L2 = torch.empty((N, r), dtype=torch.int16, device=dev)
    omega = torch.from_numpy(synth.svd_start_block(N, r + 16, SEED)).to(dev)
    lr_ws = svdq.alloc_workspace(None, 0, dev, nbytes=svdq.svdq_lowrank_workspace_bytes(N, K))
    svdq.svdq_lowrank_factors(W, lam, r, omega, L1, L2, lr_ws)
    del lr_ws, omega
    w = svdq.prepare_layer(W, lam, L1, L2, bias, r)
    gx_t = torch.empty(1, dtype=torch.float32, device=dev)
    svdq.svdq_act_global_scale(w, X, gx_t)
    gx = float(gx_t.item())
    del W

    ws = svdq.alloc_workspace(w, M, dev)
    qx = ws
    sx_off = (M * K // 2 + 1023) // 1024 * 1024
    sx = ws[sx_off:]
    la_off = sx_off + (svdq.svdq_act_scale_bytes(w, M) + 1023) // 1024 * 1024
    la = ws[la_off:]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    pro = None
    if args.qkv_prologue:  # the fused attention prologue: seeded QK-norm weights and rotary tables
        nq, nk, cs, sn = synth.qkv_prologue_inputs(M, 128, SEED)
        pro_t = [torch.from_numpy(a).to(dev) for a in (nq, nk, cs.T.copy(), sn.T.copy())]
        pro = svdq.make_qkv_prologue(N // 384, *pro_t, eps=1e-6)

    def gemm():
        if pro is None:
            svdq.svdq_w4a4_gemm_lora_up(w, qx, sx, gx, la, M, Y, svdq.SVDQ_OUT_BF16, stream)
        else:
            svdq.svdq_w4a4_gemm_lora_up_qkv(w, qx, sx, gx, la, M, pro, Y, svdq.SVDQ_OUT_BF16, stream)

    def step():
        svdq.svdq_quantize_act_lora_down(w, X, M, gx, qx, sx, la, stream)
        gemm()

    for _ in range(args.warmup):
        flush.sum()
        step()
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(w) == 0

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    time.sleep(0.1)
    _barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.sum()
        e0, e1, e2 = ev[i]
        e0.record(stream)
        svdq.svdq_quantize_act_lora_down(w, X, M, gx, qx, sx, la, stream)
        e1.record(stream)
        gemm()
        e2.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    t_wall1 = time.time()
    clocks = sampler.stop(t_wall0, t_wall1)
    assert svdq.svdq_device_status(w) == 0

    t_q = [a.elapsed_time(b) for a, b, _ in ev]
    t_g = [b.elapsed_time(c) for _, b, c in ev]
    t_step_ms = sum(a.elapsed_time(c) for a, _, c in ev) / args.steps
    t_step_ms = _allreduce_max(t_step_ms, world, dev)
    flops = 2.0 * M * N * K
    value = _job_tops(flops, t_step_ms, world)

    # ---- end to end through the C ABI with host buffers: H2D X, forward, D2H Y
    X_h = torch.from_numpy(li.x_bits.view(np.int16)).pin_memory()
    Y_h = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    X_d = torch.empty_like(X)
    ws2 = svdq.alloc_workspace(w, M, dev)
    e2e_steps = max(3, min(args.steps, 20))
    def forward():
        if pro is None:
            svdq.svdq_linear_forward(w, X_d, M, gx, Y, ws2, ws2.numel(), svdq.SVDQ_OUT_BF16, stream)
        else:
            svdq.svdq_linear_forward_qkv(w, X_d, M, gx, pro, Y, ws2, ws2.numel(), svdq.SVDQ_OUT_BF16, stream)

    for _ in range(2):
        X_d.copy_(X_h, non_blocking=True)
        forward()
        Y_h.copy_(Y, non_blocking=True)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(e2e_steps):
        X_d.copy_(X_h, non_blocking=True)
        forward()
        Y_h.copy_(Y, non_blocking=True)
    s1.record(stream)
    torch.cuda.synchronize()
    t_e2e_ms = _allreduce_max(s0.elapsed_time(s1) / e2e_steps, world, dev)

    peaks, peak_kind = _peaks()
    fp4_peak = peaks["bf16_tflops"] * 4.0  # nominal dense FP4 / BF16 ratio (9 / 2.25)
    tg = statistics.mean(t_g) * 1e-3
    tq = statistics.mean(t_q) * 1e-3
    gemm_tflops = flops / tg / 1e12
    q_bytes = M * K * 2 + M * K // 2 + M * K // 16 + M * w.view().rank_pad * 4
    q_gbs = q_bytes / tq / 1e9
    csrc = os.path.join(ROOT, "bit_diffusion_transformer_svdq_b200", "csrc")

    if rank == 0:
        line = {
            "metric": "fused SVDQuant W4A4 linear effective TOPS"
                      + (" (QKV projection with the fused attention prologue)" if pro is not None else ""),
            "value": value, "unit": "TOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
            "data": "synthetic",
            "config": {"workload": f"{WORKLOAD} M={M} K={K} N={N} rank={r} nvfp4 (FLUX fused QKV projection)",
                       "l2": "flushed (256 MiB read) before each step, outside the step's event bracket",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "tensor", "kernel": "gemm_nvfp4_kernel", "achieved": gemm_tflops, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": gemm_tflops / fp4_peak,
                         "traffic": _traffic("gemm_nvfp4", os.path.join(csrc, "gemm_nvfp4.cu")),
                         "peak_source": f"{peak_kind} bf16 burst {peaks['bf16_tflops']} TFLOP/s x 4 (nominal FP4:BF16)",
                         "us_per_launch": tg * 1e6},
            "roofline_quantize": {"bound": "hbm", "kernel": "quantize_lora_down_kernel", "achieved": q_gbs,
                                  "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": q_gbs / peaks["hbm_gbs"],
                                  "traffic": _traffic("quantize", os.path.join(csrc, "quantize.cu")),
                                  "algorithmic_bytes": q_bytes, "us_per_launch": tq * 1e6},
            "e2e": {"value": _job_tops(flops, t_e2e_ms, world), "unit": "TOPS",
                    "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2, "ms_per_step": t_e2e_ms},
            "gpu_launches": 2 * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            rows = 128
            times = _oracle_sample(li, rows, reps=2)
            t = min(times)
            line["cpu_baseline"] = {"value": 2.0 * rows * N * K / t / 1e12, "unit": "TOPS", "cores": _cpu_threads(),
                                    "kind": "oracle",
                                    "sample": f"{rows} of {M} rows (quantise + lora-down + fp64 forward), weights prepared untimed"}
        print(json.dumps(line), flush=True)


def run_stack(args, rank, world, local_rank):
    """One denoising step of a random-init stack of `--blocks` MMDiT-style
    blocks (QKV 3072->9216, out 3072->3072, MLP up 3072->12288, down
    12288->3072; M = 4608 tokens, rank 32, NVFP4): every linear through
    svdq_linear_forward, each with its own seeded weights, input and
    calibration (inputs are not chained: attention and norms are not part of
    the layer).  Weights and inputs are drawn on the GPU; preparation is
    untimed.  One L2 read-flush before each timed step.

    --scale static: each layer's calibrated tensor scale (svdq_linear_forward).
    --scale dynamic: every layer takes its scale from its own input on the
    device (svdq_linear_forward_dyn: an amax pass, the quantiser, the GEMM).
    --scale chain: dynamic, and the feed-forward is chained: the MLP up
    epilogue applies the GELU and max-reduces the down layer's amax, and the
    down layer quantises that output with it (no amax pass there)."""
    import torch
    import synth
    from bit_diffusion_transformer_svdq_b200 import svdq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    svdq.load_library()
    stream = torch.cuda.current_stream()
    M = synth.WORKLOADS["stack_qkv"].M
    layers = []
    lr_ws = svdq.alloc_workspace(None, 0, dev, nbytes=max(
        svdq.svdq_lowrank_workspace_bytes(synth.WORKLOADS[n].N, synth.WORKLOADS[n].K) for n in synth.STACK_LAYERS))
    for blk in range(args.blocks):
        for j, name in enumerate(synth.STACK_LAYERS):
            shp = synth.WORKLOADS[name]
            K, N, r = shp.K, shp.N, shp.rank
            g = torch.Generator(device=dev)
            g.manual_seed(synth.stack_seed(blk, j))
            W = torch.randn(N, K, generator=g, device=dev) * 0.02
            Xf = torch.randn(M, K, generator=g, device=dev)
            Xf[:, torch.randperm(K, generator=g, device=dev)[:4]] *= 50.0  # the outlier channels
            X = Xf.to(torch.bfloat16).view(torch.int16)
            b = (torch.randn(N, generator=g, device=dev) * 0.01).to(torch.bfloat16).view(torch.int16)
            lam = torch.empty(K, dtype=torch.float32, device=dev)
            scratch = torch.empty(2 * K, dtype=torch.float32, device=dev)
            svdq.svdq_smoothing_lambda(X, W, lam, scratch)
            L1 = torch.empty((r, K), dtype=torch.int16, device=dev)
            L2 = torch.empty((N, r), dtype=torch.int16, device=dev)
            omega = torch.randn(N, r + 16, generator=g, device=dev)
            svdq.svdq_lowrank_factors(W, lam, r, omega, L1, L2, lr_ws)
            w = svdq.prepare_layer(W, lam, L1, L2, b, r)
            gx_t = torch.empty(1, dtype=torch.float32, device=dev)
            svdq.svdq_act_global_scale(w, X, gx_t)
            layers.append((w, X, float(gx_t.item()), N, K))
            del W, Xf, omega
    torch.cuda.empty_cache()
    ws_bytes = max(svdq.svdq_workspace_bytes(w, M) for (w, _, _, _, _) in layers[:4])
    ws = svdq.alloc_workspace(layers[0][0], M, dev, nbytes=ws_bytes)
    Ys = {N: torch.empty((M, N), dtype=torch.bfloat16, device=dev) for (_, _, _, N, _) in layers[:4]}
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    words = torch.zeros(2, dtype=torch.float32, device=dev)
    epis = {}
    for i, (w, _, _, _, _) in enumerate(layers):
        if i % 4 == 2:  # MLP up: GELU, and the amax of the down layer that follows
            il = layers[i + 1][0].view().inv_lambda
            epis[i] = svdq.make_epilogue_next(svdq.SVDQ_ACT_GELU_TANH, il, words[1:])

    def step():
        if args.scale == "static":
            for (w, X, gx, N, _) in layers:
                svdq.svdq_linear_forward(w, X, M, gx, Ys[N], ws, ws.numel(), svdq.SVDQ_OUT_BF16, stream)
        elif args.scale == "dynamic":
            for (w, X, _, N, _) in layers:
                svdq.svdq_linear_forward_dyn(w, X, M, None, Ys[N], ws, ws.numel(), stream=stream)
        else:
            for i, (w, X, _, N, _) in enumerate(layers):
                if i % 4 == 3:  # MLP down on the up layer's output and amax
                    svdq.svdq_linear_forward_dyn(w, Ys[12288].view(torch.int16), M, words[1:], Ys[N], ws,
                                                 ws.numel(), stream=stream)
                else:
                    svdq.svdq_linear_forward_dyn(w, X, M, None, Ys[N], ws, ws.numel(), epi=epis.get(i),
                                                 stream=stream)

    for _ in range(args.warmup):
        flush.sum()
        step()
    torch.cuda.synchronize()
    assert all(svdq.svdq_device_status(w) == 0 for (w, _, _, _, _) in layers)
    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    time.sleep(0.1)
    _barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ts = []
    for _ in range(args.steps):
        flush.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        ts.append((e0, e1))
    torch.cuda.synchronize()
    _barrier(world)
    clocks = sampler.stop(t_wall0, time.time())
    assert all(svdq.svdq_device_status(w) == 0 for (w, _, _, _, _) in layers)
    t_ms = _allreduce_max(sum(a.elapsed_time(b) for a, b in ts) / len(ts), world, dev)
    flops = sum(2.0 * M * N * K for (_, _, _, N, K) in layers)
    # kernels per linear: quantiser + GEMM, plus the amax pass when the
    # scale is dynamic (not for the chained down layers)
    per_step = {"static": 2 * len(layers), "dynamic": 3 * len(layers),
                "chain": 3 * len(layers) - len(layers) // 4}[args.scale]
    if rank == 0:
        print(json.dumps({
            "metric": "fused SVDQuant W4A4 linear effective TOPS, one denoising step of the block stack",
            "value": _job_tops(flops, t_ms, world), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
            "config": {"workload": f"{args.blocks} blocks x 4 linears (QKV, out, MLP up, down), M={M}, rank 32, nvfp4",
                       "linears": len(layers), "tensor_scale": args.scale,
                       "l2": "flushed (256 MiB read) once before each step",
                       "parallelism": f"replicas x{world}"},
            "gpu_launches": per_step * args.steps, "clocks": clocks}), flush=True)


def run_awq(args, rank, world, local_rank):
    """The awq_w4a16 family on its FLUX workload: a double block's adaLN
    modulation (3072 -> 6 x 3072) for a batch of `--batch` images, seeded
    random weights and activation-aware channel scales, L2 read-flushed
    before every step.  Memory-bound: the roofline is the HBM copy rate
    against the weight codes + scales + X + Y bytes."""
    import torch
    import synth
    from bit_diffusion_transformer_svdq_b200 import svdq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    svdq.load_library()
    stream = torch.cuda.current_stream()
    li = synth.make_layer("awq", SEED, M=args.batch)
    M, K, N = li.shape.M, li.shape.K, li.shape.N
    W = torch.from_numpy(li.w).to(dev)
    alpha = torch.from_numpy(synth.awq_alpha(K, SEED)).to(dev)
    b = torch.from_numpy(li.bias_bits.view(np.int16)).to(dev)
    w = svdq.prepare_layer(W, alpha, None, None, b, 0, svdq.SVDQ_AWQ_W4A16)
    del W
    X = torch.from_numpy(li.x_bits.view(np.int16)).to(dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        flush.sum()
        svdq.svdq_awq_w4a16_forward(w, X, M, Y, svdq.SVDQ_OUT_BF16, stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                           else os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])
    sampler.start()
    time.sleep(0.1)
    _barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ev = []
    for _ in range(args.steps):
        flush.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        svdq.svdq_awq_w4a16_forward(w, X, M, Y, svdq.SVDQ_OUT_BF16, stream)
        e1.record(stream)
        ev.append((e0, e1))
    torch.cuda.synchronize()
    _barrier(world)
    clocks = sampler.stop(t_wall0, time.time())
    assert svdq.svdq_device_status(w) == 0
    t_ms = _allreduce_max(sum(a.elapsed_time(c) for a, c in ev) / len(ev), world, dev)
    nbytes = N * K // 2 + (K // 64) * N * 2 + M * K * 2 + M * N * 2 + K * 4 + N * 4
    peaks, peak_kind = _peaks()
    gbs = nbytes / (t_ms * 1e-3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "awq_w4a16 modulation projection, GB/s of weight + activation traffic",
            "value": world * gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int4 weights x fp32 (bf16 activations)", "data": "synthetic",
            "config": {"workload": f"awq adaLN modulation M={M} K={K} N={N} int4/64",
                       "l2": "flushed (256 MiB read) before each step", "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "kernel": "awq_gemv_kernel", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes": nbytes, "peak_source": f"{peak_kind} hbm_gbs"},
            "gpu_launches": args.steps, "clocks": clocks}), flush=True)


def _job_tops(ops_per_rank, t_ms_max, world):
    """Whole-job throughput of N independent replicas (weak scaling): every
    rank does the same work, and the job takes as long as its slowest rank."""
    return world * ops_per_rank / (t_ms_max * 1e-3) / 1e12


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _allreduce_max(v, world, dev):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rows", type=int, default=None, help="override M (smaller profiling cases only)")
    ap.add_argument("--workload", default="qkv", choices=["qkv", "stack", "awq"],
                    help="qkv: the single-layer bench line; stack: one denoising step of the block stack; "
                         "awq: the awq_w4a16 modulation projection")
    ap.add_argument("--batch", type=int, default=1, help="rows of the awq workload (images)")
    ap.add_argument("--blocks", type=int, default=57, help="blocks of the stack workload")
    ap.add_argument("--scale", default="static", choices=["static", "dynamic", "chain"],
                    help="activation tensor scale of the stack workload (see run_stack)")
    ap.add_argument("--qkv-prologue", action="store_true",
                    help="qkv workload: the GEMM also applies the QK-norm + rotary attention prologue")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    import synth
    if args.impl == "reference":
        if rank == 0:
            li = synth.make_layer(WORKLOAD, SEED)
            run_reference(args, li, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.workload in ("stack", "awq"):
        try:
            (run_stack if args.workload == "stack" else run_awq)(args, rank, world, local_rank)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    li = synth.make_layer(WORKLOAD, SEED, **({"M": args.rows} if args.rows else {}))
    try:
        run_ours(args, li, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
