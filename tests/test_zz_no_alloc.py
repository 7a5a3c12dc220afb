"""The no-allocation forward (svdq_linear_forward_noalloc) against the
workspace forward (svdq_linear_forward), through the C ABI.

The no-allocation entry point serves callers that cannot allocate device
memory (a host framework that owns every allocation, a serving loop that
must never call cudaMalloc); its intermediates live in the library's own
static device scratch.  Two calls in a row with different inputs must each
match the workspace forward on the same inputs, so nothing left in the
shared scratch by one call leaks into the next.  This file is collected
last on purpose.
"""
import numpy as np
import pytest
import torch

import synth
from tests import svdq_testlib as T

pytestmark = pytest.mark.gpu

REL_F = 2e-3
MAX_ABS = 1e-2


@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def _close(y, ref):
    d = y.astype(np.float64) - ref.astype(np.float64)
    rms = np.sqrt(np.mean(ref.astype(np.float64) ** 2))
    rel_f = np.linalg.norm(d) / np.linalg.norm(ref.astype(np.float64))
    assert rel_f <= REL_F and np.abs(d).max() <= MAX_ABS * rms, (rel_f, np.abs(d).max() / rms)


def test_noalloc_forward_matches_workspace_forward_twice(svdq):
    li = synth.make_layer("qkv", 31, M=333, K=1024, N=768)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    M, N = li.shape.M, li.shape.N
    ws = T.aligned_empty(svdq.svdq_workspace_bytes(w, M))
    x2 = synth.make_layer("qkv", 32, M=M, K=1024, N=768).x_bits
    for x_bits in (li.x_bits, x2):
        X = T.dev_u16(x_bits)
        ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
        svdq.svdq_linear_forward(w, X, M, float(ol.gx), ref, ws, ws.numel(), svdq.SVDQ_OUT_F32)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        svdq.svdq_linear_forward_noalloc(w, X, M, float(ol.gx), y, svdq.SVDQ_OUT_F32)
        torch.cuda.synchronize()
        _close(y.cpu().numpy(), ref.cpu().numpy())
    assert svdq.svdq_device_status(w) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch(svdq):
    li = synth.make_layer("tiny", 3, K=3072, N=256, M=16)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    M = 9216  # codes + scales + lora_act need about 17 MB, more than the 16 MiB scratch
    X = torch.zeros((M, 3072), dtype=torch.int16, device="cuda")
    Y = torch.empty((M, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(svdq.SVDQError) as e:
        svdq.svdq_linear_forward_noalloc(w, X, M, float(ol.gx), Y)
    assert e.value.status == 7
