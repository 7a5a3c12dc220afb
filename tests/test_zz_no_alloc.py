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

@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def test_noalloc_forward_matches_workspace_forward_twice(svdq):
    """Two calls in a row, the second with fewer rows than the first, so that
    it runs over the first call's leftovers in the shared scratch: each must
    equal the workspace forward bit for bit (same kernels, same inputs), and
    the second call must leave device memory use unchanged."""
    K, N = 1024, 768
    li = synth.make_layer("qkv", 31, M=333, K=K, N=N)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    x2 = synth.make_layer("qkv", 32, M=200, K=K, N=N).x_bits
    for call, x_bits in enumerate((li.x_bits, x2)):
        M = x_bits.shape[0]
        ws = T.aligned_empty(svdq.svdq_workspace_bytes(w, M))
        X = T.dev_u16(x_bits)
        for out_dtype, dt in ((svdq.SVDQ_OUT_F32, torch.float32), (svdq.SVDQ_OUT_BF16, torch.bfloat16)):
            ref = torch.empty((M, N), dtype=dt, device="cuda")
            svdq.svdq_linear_forward(w, X, M, float(ol.gx), ref, ws, ws.numel(), out_dtype)
            y = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
            torch.cuda.synchronize()
            if call == 1:
                alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
            svdq.svdq_linear_forward_noalloc(w, X, M, float(ol.gx), y, out_dtype)
            torch.cuda.synchronize()
            if call == 1:
                assert torch.cuda.memory_allocated() == alloc0
                assert torch.cuda.mem_get_info()[0] == free0
            assert torch.equal(y, ref), (call, out_dtype)
    assert svdq.svdq_device_status(w) == 0


def test_noalloc_int4_matches_workspace_forward(svdq):
    """INT4 weights: the scratch also holds the E4M3 copy of the codes that
    the GEMM reads.  Two calls (the second with fewer rows, over the first's
    leftovers) equal the workspace forward bit for bit."""
    K, N = 576, 320  # an odd number of 64-groups, a ragged last column tile
    li = synth.make_layer("int4", 41, M=300, K=K, N=N)
    ol = T.oracle_layer(li, precision="int4")
    w = T.gpu_prepare(svdq, li, ol, "int4")
    x2 = synth.make_layer("int4", 42, M=130, K=K, N=N).x_bits
    for call, x_bits in enumerate((li.x_bits, x2)):
        M = x_bits.shape[0]
        ws = T.aligned_empty(svdq.svdq_workspace_bytes(w, M))
        X = T.dev_u16(x_bits)
        ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
        svdq.svdq_linear_forward(w, X, M, 1.0, ref, ws, ws.numel(), svdq.SVDQ_OUT_F32)
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        svdq.svdq_linear_forward_noalloc(w, X, M, 1.0, y, svdq.SVDQ_OUT_F32)
        torch.cuda.synchronize()
        assert torch.equal(y, ref), call
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


def test_noalloc_rejects_awq_weights_before_the_size_check(svdq):
    """awq_w4a16 weights have no activation quantisation: an argument error,
    whatever M, as in svdq_linear_forward."""
    li = synth.make_layer("awq", 5, M=4, K=256, N=256)
    W = T.dev_f32(li.w)
    w = svdq.prepare_layer(W, torch.ones(256, dtype=torch.float32, device="cuda"), None, None, T.dev_u16(li.bias_bits),
                           0, svdq.SVDQ_AWQ_W4A16)
    M = 1 << 20
    X = torch.zeros((16, 256), dtype=torch.int16, device="cuda")
    Y = torch.empty((16, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(svdq.SVDQError) as e:
        svdq.svdq_linear_forward_noalloc(w, X, M, 1.0, Y)
    assert e.value.status == 1
