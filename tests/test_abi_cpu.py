"""The C-ABI library loads without a GPU and exports every entry point that
include/svdq.h declares; host-only entry points behave as documented."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    hdr = open(os.path.join(ROOT, "include", "svdq.h")).read()
    return re.findall(r"^SVDQ_API [^;(]*?\b(svdq_\w+)\s*\(", hdr, re.M)


@pytest.fixture(scope="module")
def svdq():
    from bit_diffusion_transformer_svdq_b200 import build, svdq as mod
    build.build()
    mod.load_library()
    return mod


def test_every_declared_symbol_is_exported(svdq):
    names = _declared()
    assert len(names) >= 14
    lib = svdq.load_library()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(svdq._SIGS), set(names) - set(svdq._SIGS)


def _prototypes():
    """name -> number of parameters, from every SVDQ_API declaration."""
    hdr = open(os.path.join(ROOT, "include", "svdq.h")).read()
    out = {}
    for m in re.finditer(r"^SVDQ_API [^;(]*?\b(svdq_\w+)\s*\(([^;]*?)\)\s*;", hdr, re.M | re.S):
        params = " ".join(m.group(2).split())
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_bindings_match_the_header_prototypes(svdq):
    protos = _prototypes()
    assert set(protos) == set(_declared())
    for name, n in protos.items():
        assert len(svdq._SIGS[name][1]) == n, (name, n, len(svdq._SIGS[name][1]))


def test_status_strings(svdq):
    for code in range(8):
        assert svdq.svdq_status_string(code)
    assert "timed out" in svdq.svdq_status_string(6)


def test_weights_bytes_validates_the_descriptor(svdq):
    ok = svdq.make_desc(3072, 9216, 32)
    n = svdq.svdq_weights_bytes(ok)
    assert n >= 9216 * 3072 // 2 + 9216 * 3072 // 16
    assert svdq.svdq_weights_bytes(svdq.make_desc(100, 256, 16)) == 0  # K % 64
    assert svdq.svdq_weights_bytes(svdq.make_desc(256, 250, 16)) == 0  # N % 16
    assert svdq.svdq_weights_bytes(svdq.make_desc(256, 256, 12)) == 0  # rank % 8
    assert svdq.svdq_weights_bytes(svdq.make_desc(256, 256, 72)) == 0  # rank > 64
    bad = svdq.LayerDesc(256, 256, 16, 0, 64)  # nvfp4 with group 64
    assert svdq.svdq_weights_bytes(bad) == 0
    assert svdq.svdq_weights_bytes(svdq.make_desc(256, 256, 16, svdq.SVDQ_INT4)) > 0


def test_null_arguments_rejected_before_any_cuda_call(svdq):
    import ctypes
    lib = svdq.load_library()
    assert lib.svdq_quantize_act_lora_down(None, None, 4, 1.0, None, None, None, None) == 1
    assert lib.svdq_w4a4_gemm_lora_up(None, None, None, 1.0, None, 4, None, 0, None) == 1
    assert lib.svdq_linear_forward(None, None, 4, 1.0, None, 0, None, 0, None) == 1
    pro = svdq.QkvPrologue()
    assert lib.svdq_w4a4_gemm_lora_up_qkv(None, None, None, 1.0, None, 4, ctypes.byref(pro), None, 0, None) == 1
    assert lib.svdq_w4a4_gemm_lora_up_qkv(None, None, None, 1.0, None, 4, None, None, 0, None) == 1
    assert lib.svdq_linear_forward_qkv(None, None, 4, 1.0, ctypes.byref(pro), None, 0, None, 0, None) == 1
    # the dynamic-scale and chained entry points
    epi = svdq.EpilogueNext()
    assert lib.svdq_act_amax(None, None, 4, None, None) == 1
    assert lib.svdq_quantize_act_lora_down_dyn(None, None, 4, None, None, None, None, None) == 1
    assert lib.svdq_w4a4_gemm_lora_up_dyn(None, None, None, None, None, 4, None, ctypes.byref(epi), None, 0, None) == 1
    assert lib.svdq_linear_forward_dyn(None, None, 4, None, None, ctypes.byref(epi), None, 0, None, 0, None) == 1
    assert lib.svdq_awq_w4a16_forward(None, None, 1, None, 0, None) == 1
    out = ctypes.c_void_p()
    d = svdq.make_desc(256, 256, 16)
    assert lib.svdq_prepare_weights(ctypes.byref(d), None, None, None, None, None, None, 0, ctypes.byref(out), None) == 1
    assert lib.svdq_weights_get_view(None, None) == 1
