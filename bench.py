"""Benchmark of the SVDQuant W4A4 linear layer on B200.

One step = the whole hot path over one batch, for every linear of the
workload: smoothing + 4-bit activation quantisation + lora-down (one
kernel), then the 4-bit GEMM with the lora-up and bias in its epilogue (one
kernel).  Workloads (--workload):

  mlp   (default) the FLUX-shaped MLP pair: up 4608 x 3072 -> 12288, then
        down 4608 x 12288 -> 3072 on a GELU(tanh) input, rank 32, NVFP4
  qkv   the FLUX-shaped fused QKV projection 4608 x 3072 -> 9216, rank 32,
        NVFP4 (--qkv-prologue adds the attention prologue to the GEMM)
  int4  the INT4 group-64 variant on a batch of four images:
        18432 x 3072 -> 3072, rank 32
  tiny  64 x 256 -> 256, rank 16, NVFP4 (launch-bound; microseconds only)
  stack one denoising step of the 57-block stack (run_stack)
  awq   the awq_w4a16 modulation projection (run_awq)

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload ...]

Prints one JSON line (rank 0).  `value` is effective TOPS (2*M*N*K dense-
equivalent operations per second over the step's linears, the low-rank
flops not counted) summed over all ranks; ranks run independent replicas
(the layer has no exchange step).  L2 is flushed before every timed step by
reading a 256 MiB buffer (a read leaves only clean lines, so the step pays
no write-back of the flush), outside the step's CUDA-event bracket;
`--flush-mib` sets its size (0 skips it: a warm-L2 diagnostic).
`--impl reference` times the CPU oracle on the host cores on a bounded row
sample of the same workload.
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

# workload -> (description, [(layer shape, seed), ...])
LAYER_WORKLOADS = {
    "mlp": ("FLUX MLP pair: up 4608x3072->12288 then down 4608x12288->3072 (GELU(tanh) input), rank 32, nvfp4",
            [("mlp_up", 2), ("mlp_down", 3)]),
    "qkv": ("FLUX fused QKV projection 4608x3072->9216, rank 32, nvfp4", [("qkv", 2)]),
    "int4": ("INT4 group-64, four images: 18432x3072->3072, rank 32", [("int4", 4)]),
    "tiny": ("tiny 64x256->256, rank 16, nvfp4", [("tiny", 1)]),
}
CPU_SAMPLE_ROWS = 128
METRIC = "fused SVDQuant W4A4 linear effective TOPS"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, "fallback"


def _src_hash(path):
    """Hash of a kernel's source file together with the shared device
    headers it includes (a change to either changes the kernel)."""
    h = hashlib.sha256()
    d = os.path.dirname(path)
    for f in (path, os.path.join(d, "ptx.cuh"), os.path.join(d, "internal.h")):
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def _traffic(key, src):
    """dram bytes per launch from the committed ncu summary, or None if the
    kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(key)
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
        """Starts sampling and returns once the first sample has arrived (at
        most 3 s), so that the timed region that follows is covered."""
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "20", "-i", self.gpu], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
            return
        t_end = time.time() + 3.0
        while not self.rows and time.time() < t_end:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [c.strip() for c in line.split(",")]))

    def stop(self, t0, t1):
        if not self.proc:
            return None
        t_end = time.time() + 0.5  # one sample past the timed region
        while not any(ts > t1 for ts, _ in self.rows) and time.time() < t_end:
            time.sleep(0.01)
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


def _sampler(local_rank):
    return ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ
                        else os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local_rank])


def _oracle_prepare(li):
    """Oracle weight preparation of one layer (untimed)."""
    from oracle import svdq as V
    lam = V.smoothing_lambda(li.x, li.w)
    L1, L2 = V.lowrank_factors(li.w, lam, li.shape.rank)
    prep = V.prepare_weights(li.w, lam, L1, L2, li.bias, li.shape.precision)
    gx = V.act_global_scale(li.x, prep.inv_lam) if li.shape.precision == "nvfp4" else None
    return prep, gx


def _oracle_step(lis, preps, rows):
    """One bounded-sample step of the oracle as it stands: quantise +
    lora-down + fp64 forward of `rows` rows of every layer.  Returns
    (seconds, operations counted like the GPU metric)."""
    from oracle import svdq as V
    t = time.perf_counter()
    ops = 0.0
    for li, (prep, gx) in zip(lis, preps):
        r = min(rows, li.shape.M)
        V.forward(li.x[:r], prep, gx)
        ops += 2.0 * r * li.shape.N * li.shape.K
    return time.perf_counter() - t, ops


def _cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def _layer_inputs(args):
    import synth
    desc, specs = LAYER_WORKLOADS[args.workload]
    over = {"M": args.rows} if args.rows else {}
    return desc, [synth.make_layer(name, seed, **over) for name, seed in specs]


def run_reference(args, rank, world):
    if rank != 0:
        return
    desc, lis = _layer_inputs(args)
    preps = [_oracle_prepare(li) for li in lis]
    res = [_oracle_step(lis, preps, CPU_SAMPLE_ROWS) for _ in range(args.warmup + args.steps)][args.warmup:]
    t = sum(r[0] for r in res) / len(res)
    value = res[0][1] / t / 1e12
    rows = min(CPU_SAMPLE_ROWS, lis[0].shape.M)
    sample = f"{rows} rows of each of the {len(lis)} linear(s) per step, numpy fp64 oracle, weights prepared untimed"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {desc}", "sample_rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": _cpu_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def _gpu_layer(svdq, li, dev, seed):
    """Offline preparation on the GPU (untimed): smoothing factor, the
    library's factoriser from a seeded start block, weight preparation and
    the calibrated activation tensor scale."""
    import torch
    import synth
    M, K, N, r = li.shape.M, li.shape.K, li.shape.N, li.shape.rank
    X = torch.from_numpy(li.x_bits.view(np.int16)).to(dev)
    W = torch.from_numpy(li.w).to(dev)
    bias = torch.from_numpy(li.bias_bits.view(np.int16)).to(dev)
    lam = torch.empty(K, dtype=torch.float32, device=dev)
    svdq.svdq_smoothing_lambda(X, W, lam, torch.empty(2 * K, dtype=torch.float32, device=dev))
    L1 = torch.empty((r, K), dtype=torch.int16, device=dev)
    L2 = torch.empty((N, r), dtype=torch.int16, device=dev)
    omega = torch.from_numpy(synth.svd_start_block(N, r + 16, seed)).to(dev)
    lr_ws = svdq.alloc_workspace(None, 0, dev, nbytes=svdq.svdq_lowrank_workspace_bytes(N, K))
    svdq.svdq_lowrank_factors(W, lam, r, omega, L1, L2, lr_ws)
    prec = svdq.SVDQ_INT4 if li.shape.precision == "int4" else svdq.SVDQ_NVFP4
    w = svdq.prepare_layer(W, lam, L1, L2, bias, r, prec)
    gx = 1.0
    if prec == svdq.SVDQ_NVFP4:
        g = torch.empty(1, dtype=torch.float32, device=dev)
        svdq.svdq_act_global_scale(w, X, g)
        gx = float(g.item())
    ws = svdq.alloc_workspace(w, M, dev)
    sx_off = (svdq.svdq_act_codes_bytes(w, M) + 1023) // 1024 * 1024
    la_off = sx_off + (svdq.svdq_act_scale_bytes(w, M) + 1023) // 1024 * 1024
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    act_scale_bytes = M * K // 16 if prec == svdq.SVDQ_NVFP4 else M * (K // 64) * 2
    q_bytes = M * K * 2 + M * K // 2 + act_scale_bytes + M * w.view().rank_pad * 4
    return dict(name=li.shape.name, w=w, X=X, gx=gx, M=M, K=K, N=N, prec=prec, qx=ws, sx=ws[sx_off:],
                la=ws[la_off:], Y=Y, flops=2.0 * M * N * K, q_bytes=q_bytes)


def run_layers(args, rank, world, local_rank):
    import torch
    from bit_diffusion_transformer_svdq_b200 import svdq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    svdq.load_library()
    stream = torch.cuda.current_stream()
    desc, lis = _layer_inputs(args)
    _, specs = LAYER_WORKLOADS[args.workload]
    layers = [_gpu_layer(svdq, li, dev, seed) for li, (_, seed) in zip(lis, specs)]
    flush = _make_flush(args, dev)
    pro = None
    if args.qkv_prologue:  # the fused attention prologue: seeded QK-norm weights and rotary tables
        if args.workload != "qkv":
            raise SystemExit("--qkv-prologue needs --workload qkv")
        import synth
        L = layers[0]
        nq, nk, cs, sn = synth.qkv_prologue_inputs(L["M"], 128, 2)
        pro_t = [torch.from_numpy(a).to(dev) for a in (nq, nk, cs.T.copy(), sn.T.copy())]
        pro = svdq.make_qkv_prologue(L["N"] // 384, *pro_t, eps=1e-6)

    def quantize(L):
        svdq.svdq_quantize_act_lora_down(L["w"], L["X"], L["M"], L["gx"], L["qx"], L["sx"], L["la"], stream)

    def gemm(L):
        if pro is None:
            svdq.svdq_w4a4_gemm_lora_up(L["w"], L["qx"], L["sx"], L["gx"], L["la"], L["M"], L["Y"],
                                        svdq.SVDQ_OUT_BF16, stream)
        else:
            svdq.svdq_w4a4_gemm_lora_up_qkv(L["w"], L["qx"], L["sx"], L["gx"], L["la"], L["M"], pro, L["Y"],
                                            svdq.SVDQ_OUT_BF16, stream)

    for _ in range(args.warmup):
        flush.sum()
        for L in layers:
            quantize(L)
            gemm(L)
    torch.cuda.synchronize()
    assert all(svdq.svdq_device_status(L["w"]) == 0 for L in layers)

    nl = len(layers)
    # The timed steps carry one event at each end only: an event recorded
    # between two kernels would stop the second from launching early
    # (programmatic dependent launch) and overlapping the first one's tail.
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    # per-kernel durations: as many steps again, with an event between kernels
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nl + 1)] for _ in range(args.steps)]
    sampler = _sampler(local_rank)
    sampler.start()
    _barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    for i in range(args.steps):
        flush.sum()
        ev_step[i][0].record(stream)
        for L in layers:
            quantize(L)
            gemm(L)
        ev_step[i][1].record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    for i in range(args.steps):
        flush.sum()
        ev[i][0].record(stream)
        for j, L in enumerate(layers):
            quantize(L)
            ev[i][2 * j + 1].record(stream)
            gemm(L)
            ev[i][2 * j + 2].record(stream)
    torch.cuda.synchronize()
    t_wall2 = time.time()
    clocks = sampler.stop(t_wall0, t_wall2)
    assert all(svdq.svdq_device_status(L["w"]) == 0 for L in layers)

    # per layer: mean quantiser and GEMM times (seconds) over the per-kernel steps
    tq = [statistics.mean(e[2 * j].elapsed_time(e[2 * j + 1]) for e in ev) * 1e-3 for j in range(nl)]
    tg = [statistics.mean(e[2 * j + 1].elapsed_time(e[2 * j + 2]) for e in ev) * 1e-3 for j in range(nl)]
    t_step_ms = _allreduce_max(statistics.mean(a.elapsed_time(b) for a, b in ev_step), world, dev)
    t_step_serial_ms = statistics.mean(e[0].elapsed_time(e[-1]) for e in ev)
    flops = sum(L["flops"] for L in layers)
    value = _job_tops(flops, t_step_ms, world)

    # ---- end to end through the C ABI with host buffers: H2D X, the layer
    # forward (svdq_linear_forward), D2H Y, for every linear of the step.
    # The copies in and out run on their own streams (the two directions use
    # separate copy engines) and overlap each other and the kernels; device
    # inputs and outputs are double-buffered, so that a step's copies may
    # proceed while the previous step computes.  Events order every reuse of
    # a buffer after the work that last read it.
    host = [(torch.from_numpy(li.x_bits.view(np.int16)).pin_memory(),
             torch.empty((L["M"], L["N"]), dtype=torch.bfloat16).pin_memory(),
             svdq.alloc_workspace(L["w"], L["M"], dev)) for li, L in zip(lis, layers)]
    nbuf = 2
    dbuf = [[(torch.empty_like(L["X"]), torch.empty_like(L["Y"])) for _ in range(nbuf)] for L in layers]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    evs = {key: [[torch.cuda.Event() for _ in range(nbuf)] for _ in layers]
           for key in ("x_ready", "x_free", "y_ready", "y_free")}

    def e2e_step(k):
        b = k % nbuf
        for j, ((X_h, Y_h, ws), L) in enumerate(zip(host, layers)):
            X_d, Y_d = dbuf[j][b]
            s_in.wait_event(evs["x_free"][j][b])  # the forward that last read X_d is done
            with torch.cuda.stream(s_in):
                X_d.copy_(X_h, non_blocking=True)
            evs["x_ready"][j][b].record(s_in)
            stream.wait_event(evs["x_ready"][j][b])
            stream.wait_event(evs["y_free"][j][b])  # the copy that last read Y_d is done
            if pro is None:
                svdq.svdq_linear_forward(L["w"], X_d, L["M"], L["gx"], Y_d, ws, ws.numel(), svdq.SVDQ_OUT_BF16,
                                         stream)
            else:
                svdq.svdq_linear_forward_qkv(L["w"], X_d, L["M"], L["gx"], pro, Y_d, ws, ws.numel(),
                                             svdq.SVDQ_OUT_BF16, stream)
            evs["x_free"][j][b].record(stream)
            evs["y_ready"][j][b].record(stream)
            s_out.wait_event(evs["y_ready"][j][b])
            with torch.cuda.stream(s_out):
                Y_h.copy_(Y_d, non_blocking=True)
            evs["y_free"][j][b].record(s_out)

    def e2e_join():  # the compute stream waits for every copy out
        for j in range(len(layers)):
            for b in range(nbuf):
                stream.wait_event(evs["y_free"][j][b])

    e2e_steps = max(3, min(args.steps, 20))
    for k in range(2):
        e2e_step(k)
    e2e_join()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    s_in.wait_event(s0)
    s_out.wait_event(s0)
    for k in range(e2e_steps):
        e2e_step(k)
    e2e_join()
    s1.record(stream)
    torch.cuda.synchronize()
    t_e2e_ms = _allreduce_max(s0.elapsed_time(s1) / e2e_steps, world, dev)

    peaks, peak_kind = _peaks()
    csrc = os.path.join(ROOT, "bit_diffusion_transformer_svdq_b200", "csrc")
    kernels = []
    for j, L in enumerate(layers):
        int4 = L["prec"] == svdq.SVDQ_INT4
        # nominal dense ratios to bf16: FP4 9 / 2.25 = 4, INT8 4.5 / 2.25 = 2
        peak = peaks["bf16_tflops"] * (2.0 if int4 else 4.0)
        gk = "gemm_int4_kernel" if int4 else "gemm_nvfp4_kernel"
        tkey = f"{'gemm_int4' if int4 else 'gemm_nvfp4'}/{L['name']}"
        kernels.append({"kernel": gk, "layer": L["name"], "bound": "tensor", "us_per_launch": tg[j] * 1e6,
                        "achieved": L["flops"] / tg[j] / 1e12, "peak": peak, "unit": "TFLOP/s",
                        "frac": L["flops"] / tg[j] / 1e12 / peak,
                        "peak_source": f"{peak_kind} bf16 burst {peaks['bf16_tflops']} TFLOP/s x "
                                       f"{2 if int4 else 4} (nominal {'INT8' if int4 else 'FP4'}:BF16)",
                        "traffic": _traffic(tkey, os.path.join(csrc, "gemm_int4.cu" if int4 else "gemm_nvfp4.cu"))})
        kernels.append({"kernel": "quantize_lora_down_kernel", "layer": L["name"], "bound": "hbm",
                        "us_per_launch": tq[j] * 1e6, "achieved": L["q_bytes"] / tq[j] / 1e9,
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": L["q_bytes"] / tq[j] / 1e9 / peaks["hbm_gbs"], "algorithmic_bytes": L["q_bytes"],
                        "traffic": _traffic(f"quantize/{L['name']}", os.path.join(csrc, "quantize.cu"))})
    gemms = [k for k in kernels if k["bound"] == "tensor"]
    quants = [k for k in kernels if k["bound"] == "hbm"]
    # the dominant kernel: the GEMM (every layer's launch of it, averaged)
    g_us = statistics.mean(k["us_per_launch"] for k in gemms)
    g_flops = statistics.mean(L["flops"] for L in layers)
    roof = {"bound": "tensor", "kernel": gemms[0]["kernel"], "achieved": g_flops / g_us / 1e6, "peak": gemms[0]["peak"],
            "unit": "TFLOP/s", "frac": g_flops / g_us / 1e6 / gemms[0]["peak"],
            "traffic": (statistics.mean(k["traffic"] for k in gemms) if all(k["traffic"] for k in gemms) else None),
            "peak_source": gemms[0]["peak_source"], "us_per_launch": g_us,
            "launches_per_step": len(gemms)}
    q_big = max(quants, key=lambda k: k["algorithmic_bytes"])  # the largest activation pass
    roof_q = {k: q_big[k] for k in ("bound", "kernel", "layer", "achieved", "peak", "unit", "frac", "traffic",
                                    "algorithmic_bytes", "us_per_launch")}

    if rank == 0:
        line = {
            "metric": METRIC + (" (QKV projection with the fused attention prologue)" if pro is not None else ""),
            "value": value, "unit": "TOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int4" if layers[0]["prec"] == svdq.SVDQ_INT4 else "nvfp4",
            "data": "synthetic",
            "config": {"workload": f"{args.workload}: {desc}",
                       "linears": [f"{L['name']} M={L['M']} K={L['K']} N={L['N']}" for L in layers],
                       "l2": _l2_note(args),
                       "parallelism": f"replicas x{world}"},
            "roofline": roof,
            "roofline_quantize": roof_q,
            "kernels": kernels,
            "kernel_timing": {"steps": args.steps, "ms_per_step": t_step_serial_ms,
                              "how": "per-kernel CUDA events in as many further steps, each kernel bracketed "
                                     "(which stops the programmatic-launch overlap the timed steps have)"},
            "e2e": {"value": _job_tops(flops, t_e2e_ms, world), "unit": "TOPS",
                    "h2d_bytes_per_step": sum(L["M"] * L["K"] * 2 for L in layers),
                    "d2h_bytes_per_step": sum(L["M"] * L["N"] * 2 for L in layers), "ms_per_step": t_e2e_ms,
                    "how": "svdq_linear_forward per linear; every step copies X in from pinned host memory and Y "
                           "out, on two copy streams overlapping each other and the kernels (double-buffered)"},
            "gpu_launches": 2 * nl * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            preps = [_oracle_prepare(li) for li in lis]
            res = [_oracle_step(lis, preps, CPU_SAMPLE_ROWS) for _ in range(2)]
            t, ops = min(res)
            line["cpu_baseline"] = {"value": ops / t / 1e12, "unit": "TOPS", "cores": _cpu_threads(),
                                    "kind": "oracle",
                                    "sample": f"{min(CPU_SAMPLE_ROWS, layers[0]['M'])} rows of each linear "
                                              "(quantise + lora-down + fp64 forward), weights prepared untimed"}
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
    flush = _make_flush(args, dev)

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
    sampler = _sampler(local_rank)
    sampler.start()
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
                       "l2": _l2_note(args, "once before each step"),
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
    li = synth.make_layer("awq", 2, M=args.batch)
    M, K, N = li.shape.M, li.shape.K, li.shape.N
    W = torch.from_numpy(li.w).to(dev)
    alpha = torch.from_numpy(synth.awq_alpha(K, 2)).to(dev)
    b = torch.from_numpy(li.bias_bits.view(np.int16)).to(dev)
    w = svdq.prepare_layer(W, alpha, None, None, b, 0, svdq.SVDQ_AWQ_W4A16)
    del W
    X = torch.from_numpy(li.x_bits.view(np.int16)).to(dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = _make_flush(args, dev)
    for _ in range(args.warmup):
        flush.sum()
        svdq.svdq_awq_w4a16_forward(w, X, M, Y, svdq.SVDQ_OUT_BF16, stream)
    torch.cuda.synchronize()
    sampler = _sampler(local_rank)
    sampler.start()
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
                       "l2": _l2_note(args, "before each step"), "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "kernel": "awq_gemv_kernel", "achieved": gbs, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes": nbytes, "peak_source": f"{peak_kind} hbm_gbs"},
            "gpu_launches": args.steps, "clocks": clocks}), flush=True)


class _NoFlush:
    def sum(self):
        return None


def _make_flush(args, dev):
    """The L2 read-flush run before every step: a buffer of --flush-mib MiB
    that is summed (0: no flush, a warm-L2 diagnostic only)."""
    import torch
    if args.flush_mib <= 0:
        return _NoFlush()
    return torch.ones(args.flush_mib << 18, dtype=torch.float32, device=dev)


def _l2_note(args, when="before each step, outside the step's event bracket"):
    if args.flush_mib <= 0:
        return "not flushed (warm-L2 diagnostic, not a bench value)"
    return f"flushed ({args.flush_mib} MiB read) {when}"


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
    ap.add_argument("--flush-mib", type=int, default=256,
                    help="MiB read before every step to flush the L2 (0: none, a warm-L2 diagnostic)")
    ap.add_argument("--rows", type=int, default=None, help="override M (smaller profiling cases only)")
    ap.add_argument("--workload", default="mlp", choices=["mlp", "qkv", "int4", "tiny", "stack", "awq"],
                    help="mlp (default): the FLUX MLP pair; qkv: the fused QKV projection; int4: the INT4 "
                         "batch of four images; tiny: the 64-row case; stack: one denoising step of the block "
                         "stack; awq: the awq_w4a16 modulation projection")
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
    if args.impl == "reference":
        if args.workload not in LAYER_WORKLOADS:
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable": f"the oracle arm covers the single-layer "
                                  f"workloads {sorted(LAYER_WORKLOADS)}, not {args.workload}"}), flush=True)
            return
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.workload == "stack":
            run_stack(args, rank, world, local_rank)
        elif args.workload == "awq":
            run_awq(args, rank, world, local_rank)
        else:
            run_layers(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
