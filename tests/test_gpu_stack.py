"""Parity of the whole 57-block denoising stack (4 linears per block: QKV
3072 -> 9216, out 3072 -> 3072, MLP up 3072 -> 12288, down 12288 -> 3072;
M = 4608 tokens, rank 32, NVFP4), every linear at full size with its own
seeded inputs: all weight parts and all activation codes and scales of all
rows bit-exact against the oracle, and Y of 64 seeded sampled rows per
linear through svdq_linear_forward within the bf16-output bar.

The oracle's work (factorisation, preparation, quantisation of every row)
dominates, so it runs in a pool of spawned worker processes while this
process checks the GPU side linear by linear."""
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

import synth
from tests import svdq_testlib as T

pytestmark = pytest.mark.gpu

REL_F = 2e-3
MAX_ABS = 1e-2
ROWS_PER_LINEAR = 64


@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def _workers():
    """One single-threaded oracle worker per host core (this process only
    checks bytes the GPU wrote while they work)."""
    n = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    return max(1, min(64, n)), 1


def _check_linear(svdq, e):
    ol = e["ol"]
    M, K = e["x_bits"].shape
    N = e["w"].shape[0]
    li = synth.LayerInputs(synth.WORKLOADS[e["name"]], 0, e["x_bits"], synth.f32_from_bf16_bits(e["x_bits"]),
                           e["w"], e["bias_bits"], e["bias"])
    w = T.gpu_prepare(svdq, li, ol)
    T.check_weights_exact(svdq, w, e["exp_w"])
    X, qx, sx, la = T.gpu_quantize(svdq, w, li.x_bits, float(ol.gx))
    T.check_act_exact(svdq, w, li.x, ol, qx, sx, la, e["exp_a"])
    ws = T.aligned_empty(svdq.svdq_workspace_bytes(w, M))
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    svdq.svdq_linear_forward(w, X, M, float(ol.gx), Y, ws, ws.numel(), 0)
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(w) == 0
    y = Y[torch.from_numpy(e["rows"]).cuda()].float().cpu().numpy()
    T.check_y(y, e["ref"], 0, REL_F, MAX_ABS)


def test_stack_all_blocks(svdq):
    blocks = int(os.environ.get("SVDQ_STACK_BLOCKS", synth.STACK_BLOCKS))
    n_workers, threads = _workers()
    jobs = [(b, j, ROWS_PER_LINEAR, threads) for b in range(blocks) for j in range(len(synth.STACK_LAYERS))]
    seen = set()
    # spawn: the workers must not inherit this process's CUDA state
    with mp.get_context("spawn").Pool(n_workers) as pool:
        for e in pool.imap_unordered(T.stack_linear_expected, jobs):
            try:
                _check_linear(svdq, e)
            except AssertionError as err:
                raise AssertionError(f"block {e['blk']} {e['name']}: {err}") from err
            seen.add((e["blk"], e["j"]))
    assert len(seen) == len(jobs)
