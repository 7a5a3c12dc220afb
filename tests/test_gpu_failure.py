"""Failure detection on the GPU without a GPU fault: a bounded wait that runs
out (on a barrier nothing arrives on) is reported to the host as
SVDQ_ERR_TIMEOUT, and the context stays usable for real work afterwards."""
import time

import numpy as np
import pytest
import torch

import synth
from oracle import svdq as V
from tests import svdq_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def test_bounded_wait_reports_timeout_and_context_survives(svdq):
    t0 = time.time()
    assert svdq.svdq_selftest_bounded_wait() == 6  # SVDQ_ERR_TIMEOUT
    assert 1.5 < time.time() - t0 < 60.0  # ended by its own 2 s limit
    # the same context still runs the layer, with a clean status
    li = synth.make_layer("tiny", 3)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    M, N = li.shape.M, li.shape.N
    X = T.dev_u16(li.x_bits)
    ws = T.aligned_empty(svdq.svdq_workspace_bytes(w, M))
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    svdq.svdq_linear_forward(w, X, M, float(ol.gx), Y, ws, ws.numel(), 1)
    assert svdq.svdq_device_status(w) == 0
    ref = V.forward(li.x, ol.prep, ol.gx)
    y = Y.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) <= 2e-3
