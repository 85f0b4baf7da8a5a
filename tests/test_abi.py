"""CPU checks of the C-ABI library: it builds for sm_100a, loads, exports every entry point
that include/apex_w4a4.h declares, and rejects bad arguments on the host before touching
the GPU.  No compute call runs here."""
import ctypes
import os
import re

import pytest

import group_quantized_w4a4_b200 as apex
from group_quantized_w4a4_b200 import build as apex_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "apex_w4a4.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(apex_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    apex_build.build()
    return apex.load_library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("apex_pack_weights_int4", "apex_quantize_act_int4", "apex_w4a4_gemm",
                 "apex_w4a4_gemm_workspace_size", "apex_w4a4_group_partials",
                 "apex_get_device_status", "apex_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert getattr(apex, name, None) is not None, f"binding lacks {name}"


def test_library_is_sm100a_only():
    assert apex_build.ARCH_FLAGS == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings(lib):
    for code in range(6):
        assert apex.apex_status_string(code)
    assert apex.apex_status_string(5) == "device pipeline wait timed out"


P = ctypes.c_void_p


def _gemm(lib, M, N, K, ga, gw, a=0x1000, sa=0x2000, w=0x3000, sw=0x4000, y=0x5000,
          ws=None, wsb=0):
    return lib.apex_w4a4_gemm(M, N, K, ga, gw, P(a), P(sa), P(w), P(sw), P(y),
                              P(ws) if ws else None, wsb, None)


def test_gemm_argument_errors_are_host_side(lib):
    assert _gemm(lib, 0, 8, 128, 128, 128) == apex.APEX_ERR_INVALID_ARG
    assert _gemm(lib, 4, -1, 128, 128, 128) == apex.APEX_ERR_INVALID_ARG
    assert _gemm(lib, 4, 8, 100, 128, 128) == apex.APEX_ERR_INVALID_ARG      # K % ga
    assert _gemm(lib, 4, 8, 256, 128, 96) == apex.APEX_ERR_INVALID_ARG       # K % gw
    assert _gemm(lib, 4, 8, 512, 256, 256) == apex.APEX_ERR_UNSUPPORTED      # ga != 128
    assert _gemm(lib, 4, 8, 192, 64, 192) == apex.APEX_ERR_UNSUPPORTED
    assert _gemm(lib, 4, 8, 256, 128, 128, a=0) == apex.APEX_ERR_INVALID_ARG  # null
    assert _gemm(lib, 4, 8, 256, 128, 128, a=0x1008) == apex.APEX_ERR_ALIGNMENT
    assert _gemm(lib, 4, 8, 256, 128, 128, w=0x3004) == apex.APEX_ERR_ALIGNMENT
    assert _gemm(lib, 4, 8, 256, 128, 128, y=0x5001) == apex.APEX_ERR_ALIGNMENT


def test_quantizer_argument_errors_are_host_side(lib):
    q = lib.apex_quantize_act_int4
    assert q(None, 4, 256, 128, P(0x1000), P(0x2000), None) == apex.APEX_ERR_INVALID_ARG
    assert q(P(0x1000), 4, 200, 128, P(0x2000), P(0x3000), None) == apex.APEX_ERR_INVALID_ARG
    assert q(P(0x1000), 4, 256, 64, P(0x2000), P(0x3000), None) == apex.APEX_ERR_INVALID_ARG
    assert q(P(0x1008), 4, 256, 128, P(0x2000), P(0x3000), None) == apex.APEX_ERR_ALIGNMENT
    pw = lib.apex_pack_weights_int4
    assert pw(P(0x1000), 0, 256, 128, P(0x2000), P(0x3000), None) == apex.APEX_ERR_INVALID_ARG
    assert pw(P(0x1000), 4, 256, 128, P(0x2002), P(0x3000), None) == apex.APEX_ERR_ALIGNMENT


def test_quantized_output_argument_errors_are_host_side(lib):
    def f(N=256, y=None, yq=0x6000, yqs=0x7000):
        return lib.apex_w4a4_gemm_quant(16, N, 256, 128, 128, P(0x1000), P(0x2000), P(0x3000),
                                        P(0x4000), P(y), P(yq), P(yqs), 0, None, 0, None)
    assert f(N=200) == apex.APEX_ERR_UNSUPPORTED          # output groups are whole tiles
    assert f(yq=None) == apex.APEX_ERR_INVALID_ARG
    assert f(yqs=None) == apex.APEX_ERR_INVALID_ARG
    assert f(yq=0x6008) == apex.APEX_ERR_ALIGNMENT        # written in 16-byte words
    assert f(yqs=0x7001) == apex.APEX_ERR_ALIGNMENT
    assert f(y=0x5001) == apex.APEX_ERR_ALIGNMENT


def test_partials_argument_errors(lib):
    f = lib.apex_w4a4_group_partials
    assert f(4, 8, 100, P(0x1000), P(0x2000), P(0x3000), None) == apex.APEX_ERR_INVALID_ARG
    assert f(4, 8, 256, P(0x1000), P(0x2000), None, None) == apex.APEX_ERR_INVALID_ARG
    assert f(4, 8, 256, P(0x1001), P(0x2000), P(0x3000), None) == apex.APEX_ERR_ALIGNMENT


def test_workspace_size_contract(lib):
    # invalid problems need no workspace; a decode-shaped problem uses split-K scratch
    assert lib.apex_w4a4_gemm_workspace_size(0, 8, 128, 128, 128) == 0
    n = lib.apex_w4a4_gemm_workspace_size(16, 8192, 8192, 128, 128)
    assert n == 0 or n >= 16 * 8192 * 4 * 2
    # a prefill-shaped problem has enough tiles to fill the GPU without splitting K
    assert lib.apex_w4a4_gemm_workspace_size(4096, 8192, 8192, 128, 128) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros((4, 256), dtype=torch.float16)
    with pytest.raises((ValueError, RuntimeError)):
        apex.quantize_act(x)


def test_fp8_path_argument_errors_are_host_side(lib):
    def g(M=16, N=256, K=256, ga=128, gw=128, a=0x1000, sa=0x2000, w=0x3000, sw=0x4000,
          y=0x5000):
        return lib.apex_w4a4_gemm_fp8(M, N, K, ga, gw, P(a), P(sa), P(w), P(sw), P(y), None)
    assert g(K=200) == apex.APEX_ERR_INVALID_ARG
    assert g(ga=64) == apex.APEX_ERR_UNSUPPORTED
    assert g(a=0) == apex.APEX_ERR_INVALID_ARG
    assert g(y=0) == apex.APEX_ERR_INVALID_ARG
    assert g(a=0x1008) == apex.APEX_ERR_ALIGNMENT       # TMA base: 16 bytes
    assert g(w=0x3004) == apex.APEX_ERR_ALIGNMENT
    assert g(sa=0x2001) == apex.APEX_ERR_ALIGNMENT

    def gq(N=256, y=None, yq=0x6000, yqs=0x7000):
        return lib.apex_w4a4_gemm_fp8_quant(16, N, 256, 128, 128, P(0x1000), P(0x2000),
                                            P(0x3000), P(0x4000), P(y), P(yq), P(yqs), None)
    assert gq(N=200) == apex.APEX_ERR_UNSUPPORTED
    assert gq(yq=None) == apex.APEX_ERR_INVALID_ARG
    assert gq(yq=0x6008) == apex.APEX_ERR_ALIGNMENT
    assert gq(y=0x5001) == apex.APEX_ERR_ALIGNMENT

    q = lib.apex_quantize_act_int4_fp8
    assert q(P(0x1000), 4, 256, 256, P(0x2000), P(0x3000), None) == apex.APEX_ERR_UNSUPPORTED
    assert q(P(0x1000), 4, 200, 128, P(0x2000), P(0x3000), None) == apex.APEX_ERR_INVALID_ARG
    assert q(P(0x1000), 4, 256, 128, P(0x2004), P(0x3000), None) == apex.APEX_ERR_ALIGNMENT
    pw = lib.apex_pack_weights_int4_fp8
    assert pw(P(0x1000), 4, 512, 96, P(0x2000), P(0x3000), None) == apex.APEX_ERR_INVALID_ARG
    u = lib.apex_unpack_int4_fp8
    assert u(P(0x1000), 4, 200, P(0x2000), None) == apex.APEX_ERR_INVALID_ARG    # K % 16
    assert u(P(0x1000), 4, 256, P(0x2008), None) == apex.APEX_ERR_ALIGNMENT
    pp = lib.apex_w4a4_group_partials_fp8
    assert pp(4, 8, 256, P(0x1000), P(0x2000), None, None) == apex.APEX_ERR_INVALID_ARG


def test_dual_path_argument_errors_are_host_side(lib):
    ch = P(0x8000)

    def dq(C=5, Cp=64, form=2, x=0x1000, xo=0x9000):
        return lib.apex_quantize_act_int4_dual(P(x), 4, 256, 128, ch, C, form, P(0x2000),
                                               P(0x3000), P(xo), Cp, None)
    assert dq(Cp=48) == apex.APEX_ERR_INVALID_ARG        # Cp % 64
    assert dq(C=65) == apex.APEX_ERR_INVALID_ARG         # C > Cp
    assert dq(C=0) == apex.APEX_ERR_INVALID_ARG
    assert dq(form=3) == apex.APEX_ERR_INVALID_ARG
    assert dq(x=0x1008) == apex.APEX_ERR_ALIGNMENT
    assert dq(xo=0x9008) == apex.APEX_ERR_ALIGNMENT
    gw = lib.apex_gather_weight_columns
    assert gw(P(0x1000), 8, 256, ch, 5, P(0x9000), 32, None) == apex.APEX_ERR_INVALID_ARG
    assert gw(P(0x1000), 8, 256, ch, 5, P(0x9008), 64, None) == apex.APEX_ERR_ALIGNMENT

    def dg(Cp=64, xo=0x9000):
        return lib.apex_w4a4_gemm_fp8_dual(16, 256, 256, 128, 128, P(0x1000), P(0x2000),
                                           P(0x3000), P(0x4000), P(xo), P(0xA000), Cp,
                                           P(0x5000), None)
    assert dg(Cp=0) == apex.APEX_ERR_INVALID_ARG
    assert dg(Cp=96) == apex.APEX_ERR_INVALID_ARG
    assert dg(Cp=512) == apex.APEX_ERR_INVALID_ARG       # more outlier channels than K
    assert dg(xo=0x9008) == apex.APEX_ERR_ALIGNMENT
