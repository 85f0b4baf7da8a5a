"""B200-native pure W4A4 group-quantized GEMM.

Python binding of the C ABI in include/apex_w4a4.h (libapex_w4a4.so, sm_100a).  Each
``apex_*`` function here has the name and arguments of the C entry point, with torch CUDA
tensors standing in for device pointers and a torch stream (default: the current one) for
the cudaStream_t.  The binding only marshals arguments: every step of the computation runs
in the library's CUDA kernels, and there is no CPU fallback -- without the built library
or a CUDA device the calls raise.

The operation ("APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute
Rebalancing", abstract): 4-bit activations and weights with one fp16 scale per 128-wide
K-group, exact INT4 products per group on the tensor cores, per-group dequantisation and
accumulation on the CUDA cores; the mixed-granularity mode uses coarser weight groups.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "ApexError", "load_library", "library_path",
    "apex_pack_weights_int4", "apex_quantize_act_int4", "apex_w4a4_gemm",
    "apex_w4a4_gemm_noalloc", "apex_quantize_act_int4_expanded", "apex_w4a4_gemm_expanded",
    "apex_w4a4_gemm_quant", "apex_w4a4_gemm_expanded_quant",
    "quantize_act_expanded",
    "apex_quantize_act_int4_fp8", "apex_pack_weights_int4_fp8", "apex_unpack_int4_fp8",
    "apex_w4a4_gemm_fp8", "apex_w4a4_group_partials_fp8", "quantize_act_fp8",
    "pack_weights_fp8", "gemm_fp8",
    "apex_gather_weight_columns", "apex_quantize_act_int4_dual", "apex_w4a4_gemm_fp8_dual",
    "apex_select_weight_group", "apex_w4a4_gemm_fp8_quant",
    "apex_w4a4_gemm_workspace_size", "apex_w4a4_group_partials", "apex_get_device_status",
    "apex_set_wait_limit_ns", "apex_status_string", "apex_debug_withhold_step",
    "apex_debug_trace_next_gemm", "apex_debug_gemm_plan", "apex_debug_partials_split",
    "pack_weights", "quantize_act", "gemm", "workspace",
]

APEX_OK = 0
APEX_ERR_INVALID_ARG = 1
APEX_ERR_UNSUPPORTED = 2
APEX_ERR_ALIGNMENT = 3
APEX_ERR_CUDA = 4
APEX_ERR_TIMEOUT = 5

APEX_FORM_PACKED = 0     # output forms of apex_quantize_act_int4_dual
APEX_FORM_EXPANDED = 1
APEX_FORM_FP8 = 2

_lock = threading.Lock()
_lib = None


class ApexError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = int(code)
        super().__init__(f"{where}: {apex_status_string(code)} (status {code})")


def library_path() -> str:
    from . import build as _b
    return _b.LIB_PATH


def load_library(build_if_missing: bool = True):
    """Load libapex_w4a4.so (building it with nvcc first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        from . import build as _b
        path = _b.LIB_PATH
        if build_if_missing and _b.is_stale():
            _b.build()
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library not built: {path} (run python -m "
                               "group_quantized_w4a4_b200.build)")
        lib = ctypes.CDLL(path)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        st = ctypes.c_int
        lib.apex_pack_weights_int4.argtypes = [P, I64, I64, I32, P, P, P]
        lib.apex_pack_weights_int4.restype = st
        lib.apex_quantize_act_int4.argtypes = [P, I64, I64, I32, P, P, P]
        lib.apex_quantize_act_int4.restype = st
        lib.apex_quantize_act_int4_expanded.argtypes = [P, I64, I64, I32, P, P, P]
        lib.apex_quantize_act_int4_expanded.restype = st
        lib.apex_w4a4_gemm_expanded.argtypes = [I64, I64, I64, I32, I32, P, P, P, P, P, P, SZ, P]
        lib.apex_w4a4_gemm_expanded.restype = st
        lib.apex_w4a4_gemm.argtypes = [I64, I64, I64, I32, I32, P, P, P, P, P, P, SZ, P]
        lib.apex_w4a4_gemm.restype = st
        for name in ("apex_w4a4_gemm_quant", "apex_w4a4_gemm_expanded_quant"):
            fn = getattr(lib, name)
            fn.argtypes = [I64, I64, I64, I32, I32, P, P, P, P, P, P, P, I32, P, SZ, P]
            fn.restype = st
        lib.apex_quantize_act_int4_fp8.argtypes = [P, I64, I64, I32, P, P, P]
        lib.apex_quantize_act_int4_fp8.restype = st
        lib.apex_pack_weights_int4_fp8.argtypes = [P, I64, I64, I32, P, P, P]
        lib.apex_pack_weights_int4_fp8.restype = st
        lib.apex_unpack_int4_fp8.argtypes = [P, I64, I64, P, P]
        lib.apex_unpack_int4_fp8.restype = st
        lib.apex_w4a4_gemm_fp8.argtypes = [I64, I64, I64, I32, I32, P, P, P, P, P, P]
        lib.apex_w4a4_gemm_fp8.restype = st
        lib.apex_w4a4_gemm_fp8_quant.argtypes = [I64, I64, I64, I32, I32, P, P, P, P, P, P, P,
                                                 P]
        lib.apex_w4a4_gemm_fp8_quant.restype = st
        lib.apex_w4a4_group_partials_fp8.argtypes = [I64, I64, I64, P, P, P, P]
        lib.apex_w4a4_group_partials_fp8.restype = st
        lib.apex_gather_weight_columns.argtypes = [P, I64, I64, P, I32, P, I32, P]
        lib.apex_gather_weight_columns.restype = st
        lib.apex_quantize_act_int4_dual.argtypes = [P, I64, I64, I32, P, I32, I32, P, P, P,
                                                    I32, P]
        lib.apex_quantize_act_int4_dual.restype = st
        lib.apex_w4a4_gemm_fp8_dual.argtypes = [I64, I64, I64, I32, I32, P, P, P, P, P, P, I32,
                                                P, P]
        lib.apex_w4a4_gemm_fp8_dual.restype = st
        lib.apex_w4a4_gemm_noalloc.argtypes = [I64, I64, I64, I32, I32, P, P, P, P, P, P]
        lib.apex_w4a4_gemm_noalloc.restype = st
        lib.apex_w4a4_gemm_workspace_size.argtypes = [I64, I64, I64, I32, I32]
        lib.apex_w4a4_gemm_workspace_size.restype = SZ
        lib.apex_w4a4_linear.argtypes = [I64, I64, I64, I32, I32, P, P, P, P, P, SZ, P]
        lib.apex_w4a4_linear.restype = st
        lib.apex_w4a4_linear_workspace_size.argtypes = [I64, I64, I64, I32, I32]
        lib.apex_w4a4_linear_workspace_size.restype = SZ
        lib.apex_w4a4_group_partials.argtypes = [I64, I64, I64, P, P, P, P]
        lib.apex_w4a4_group_partials.restype = st
        lib.apex_get_device_status.argtypes = [P]
        lib.apex_get_device_status.restype = st
        lib.apex_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.apex_set_wait_limit_ns.restype = None
        lib.apex_status_string.argtypes = [st]
        lib.apex_status_string.restype = ctypes.c_char_p
        lib.apex_select_weight_group.argtypes = [I64, I64, I64, ctypes.c_double,
                                                 ctypes.c_double]
        lib.apex_select_weight_group.restype = I32
        lib.apex_debug_withhold_step.argtypes = [I32]
        lib.apex_debug_withhold_step.restype = None
        lib.apex_debug_partials_split.argtypes = [I32]
        lib.apex_debug_partials_split.restype = None
        lib.apex_debug_trace_next_gemm.argtypes = [P, I32, I32]
        lib.apex_debug_trace_next_gemm.restype = None
        lib.apex_debug_gemm_plan.argtypes = [I64, I64, I64, I32, I32, P]
        lib.apex_debug_gemm_plan.restype = st
        _lib = lib
        return lib


# ------------------------------------------------------------------ marshalling helpers

def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor (device memory)")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(code: int, where: str):
    if code != APEX_OK:
        raise ApexError(code, where)


# ------------------------------------------------------------------ the C entry points

def apex_status_string(code: int) -> str:
    try:
        return load_library().apex_status_string(int(code)).decode()
    except Exception:  # the message of an error must not itself fail
        return f"status {code}"


def apex_pack_weights_int4(w_f16, N, K, group_w, w_packed_u8, w_scales_f16, stream=None):
    _check(load_library().apex_pack_weights_int4(_ptr(w_f16), N, K, group_w, _ptr(w_packed_u8),
                                                 _ptr(w_scales_f16), _stream(stream)),
           "apex_pack_weights_int4")


def apex_quantize_act_int4(x_f16, M, K, group_a, x_packed_u8, x_scales_f16, stream=None):
    _check(load_library().apex_quantize_act_int4(_ptr(x_f16), M, K, group_a, _ptr(x_packed_u8),
                                                 _ptr(x_scales_f16), _stream(stream)),
           "apex_quantize_act_int4")


def apex_w4a4_gemm(M, N, K, group_a, group_w, a_packed, a_scales, w_packed, w_scales, y_f16,
                   workspace=None, workspace_bytes=None, stream=None):
    if workspace is not None and workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().apex_w4a4_gemm(M, N, K, group_a, group_w, _ptr(a_packed),
                                         _ptr(a_scales), _ptr(w_packed), _ptr(w_scales),
                                         _ptr(y_f16), _ptr(workspace), workspace_bytes or 0,
                                         _stream(stream)),
           "apex_w4a4_gemm")


def apex_quantize_act_int4_expanded(x_f16, M, K, group_a, x_q8, x_scales_f16, stream=None):
    _check(load_library().apex_quantize_act_int4_expanded(_ptr(x_f16), M, K, group_a,
                                                          _ptr(x_q8), _ptr(x_scales_f16),
                                                          _stream(stream)),
           "apex_quantize_act_int4_expanded")


def _gemm_quant(name, M, N, K, group_a, group_w, a, a_scales, w_packed, w_scales, y_f16,
                yq, yq_scales, yq_expanded, workspace, workspace_bytes, stream):
    if workspace is not None and workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(getattr(load_library(), name)(M, N, K, group_a, group_w, _ptr(a), _ptr(a_scales),
                                         _ptr(w_packed), _ptr(w_scales), _ptr(y_f16),
                                         _ptr(yq), _ptr(yq_scales), 1 if yq_expanded else 0,
                                         _ptr(workspace), workspace_bytes or 0,
                                         _stream(stream)), name)


def apex_w4a4_gemm_quant(M, N, K, group_a, group_w, a_packed, a_scales, w_packed, w_scales,
                         y_f16, yq, yq_scales, yq_expanded=False, workspace=None,
                         workspace_bytes=None, stream=None):
    """The GEMM plus its output quantized as the next layer's activations (y_f16 may be
    None); see the C header."""
    _gemm_quant("apex_w4a4_gemm_quant", M, N, K, group_a, group_w, a_packed, a_scales,
                w_packed, w_scales, y_f16, yq, yq_scales, yq_expanded, workspace,
                workspace_bytes, stream)


def apex_w4a4_gemm_expanded_quant(M, N, K, group_a, group_w, a_q8, a_scales, w_packed,
                                  w_scales, y_f16, yq, yq_scales, yq_expanded=False,
                                  workspace=None, workspace_bytes=None, stream=None):
    """As apex_w4a4_gemm_quant, reading expanded activations."""
    _gemm_quant("apex_w4a4_gemm_expanded_quant", M, N, K, group_a, group_w, a_q8, a_scales,
                w_packed, w_scales, y_f16, yq, yq_scales, yq_expanded, workspace,
                workspace_bytes, stream)


def apex_w4a4_gemm_expanded(M, N, K, group_a, group_w, a_q8, a_scales, w_packed, w_scales,
                            y_f16, workspace=None, workspace_bytes=None, stream=None):
    if workspace is not None and workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().apex_w4a4_gemm_expanded(M, N, K, group_a, group_w, _ptr(a_q8),
                                                  _ptr(a_scales), _ptr(w_packed),
                                                  _ptr(w_scales), _ptr(y_f16), _ptr(workspace),
                                                  workspace_bytes or 0, _stream(stream)),
           "apex_w4a4_gemm_expanded")


def quantize_act_expanded(x, group_a: int = 128, stream=None):
    """fp16 [M, K] CUDA tensor -> (expanded int8 [M, K], scales fp16 [M, K/group_a])."""
    import torch
    M, K = x.shape
    q8 = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    scales = torch.empty((M, K // group_a), dtype=torch.float16, device=x.device)
    apex_quantize_act_int4_expanded(x, M, K, group_a, q8, scales, stream)
    return q8, scales


def apex_quantize_act_int4_fp8(x_f16, M, K, group_a, x_codes, x_scales_f16, stream=None):
    _check(load_library().apex_quantize_act_int4_fp8(_ptr(x_f16), M, K, group_a, _ptr(x_codes),
                                                     _ptr(x_scales_f16), _stream(stream)),
           "apex_quantize_act_int4_fp8")


def apex_pack_weights_int4_fp8(w_f16, N, K, group_w, w_codes, w_scales_f16, stream=None):
    _check(load_library().apex_pack_weights_int4_fp8(_ptr(w_f16), N, K, group_w, _ptr(w_codes),
                                                     _ptr(w_scales_f16), _stream(stream)),
           "apex_pack_weights_int4_fp8")


def apex_unpack_int4_fp8(packed, rows, K, codes, stream=None):
    _check(load_library().apex_unpack_int4_fp8(_ptr(packed), rows, K, _ptr(codes),
                                               _stream(stream)),
           "apex_unpack_int4_fp8")


def apex_w4a4_gemm_fp8(M, N, K, group_a, group_w, a_codes, a_scales, w_codes, w_scales, y_f16,
                       stream=None):
    _check(load_library().apex_w4a4_gemm_fp8(M, N, K, group_a, group_w, _ptr(a_codes),
                                             _ptr(a_scales), _ptr(w_codes), _ptr(w_scales),
                                             _ptr(y_f16), _stream(stream)),
           "apex_w4a4_gemm_fp8")


def apex_w4a4_gemm_fp8_quant(M, N, K, group_a, group_w, a_codes, a_scales, w_codes, w_scales,
                             y_f16, yq_codes, yq_scales, stream=None):
    """The E4M3-carrier GEMM plus its output quantized as the next layer's E4M3-coded
    activations (y_f16 may be None); see the C header."""
    _check(load_library().apex_w4a4_gemm_fp8_quant(M, N, K, group_a, group_w, _ptr(a_codes),
                                                   _ptr(a_scales), _ptr(w_codes),
                                                   _ptr(w_scales), _ptr(y_f16),
                                                   _ptr(yq_codes), _ptr(yq_scales),
                                                   _stream(stream)),
           "apex_w4a4_gemm_fp8_quant")


def apex_w4a4_group_partials_fp8(M, N, K, a_codes, w_codes, partials_i32, stream=None):
    _check(load_library().apex_w4a4_group_partials_fp8(M, N, K, _ptr(a_codes), _ptr(w_codes),
                                                       _ptr(partials_i32), _stream(stream)),
           "apex_w4a4_group_partials_fp8")


def quantize_act_fp8(x, group_a: int = 128, stream=None):
    """fp16 [M, K] CUDA tensor -> (E4M3 codes uint8 [M, K], scales fp16 [M, K/group_a])."""
    import torch
    M, K = x.shape
    codes = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    scales = torch.empty((M, K // group_a), dtype=torch.float16, device=x.device)
    apex_quantize_act_int4_fp8(x, M, K, group_a, codes, scales, stream)
    return codes, scales


def pack_weights_fp8(w, group_w: int = 128, stream=None):
    """fp16 [N, K] CUDA tensor -> (E4M3 codes uint8 [N, K], scales fp16 [N, K/group_w])."""
    import torch
    N, K = w.shape
    codes = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    scales = torch.empty((N, K // group_w), dtype=torch.float16, device=w.device)
    apex_pack_weights_int4_fp8(w, N, K, group_w, codes, scales, stream)
    return codes, scales


def gemm_fp8(a_codes, a_scales, w_codes, w_scales, group_a=128, group_w=128, out=None,
             stream=None):
    """Y = W4A4 GEMM of E4M3-coded operands -> fp16 [M, N]."""
    import torch
    M, K = a_codes.shape
    N = w_codes.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a_codes.device)
    apex_w4a4_gemm_fp8(M, N, K, group_a, group_w, a_codes, a_scales, w_codes, w_scales, out,
                       stream)
    return out


def apex_gather_weight_columns(w_f16, N, K, channels_i32, C, w_out_f16, Cp, stream=None):
    _check(load_library().apex_gather_weight_columns(_ptr(w_f16), N, K, _ptr(channels_i32), C,
                                                     _ptr(w_out_f16), Cp, _stream(stream)),
           "apex_gather_weight_columns")


def apex_quantize_act_int4_dual(x_f16, M, K, group_a, channels_i32, C, form, x_q, x_scales_f16,
                                x_out_f16, Cp, stream=None):
    _check(load_library().apex_quantize_act_int4_dual(_ptr(x_f16), M, K, group_a,
                                                      _ptr(channels_i32), C, int(form),
                                                      _ptr(x_q), _ptr(x_scales_f16),
                                                      _ptr(x_out_f16), Cp, _stream(stream)),
           "apex_quantize_act_int4_dual")


def apex_w4a4_gemm_fp8_dual(M, N, K, group_a, group_w, a_codes, a_scales, w_codes, w_scales,
                            x_out_f16, w_out_f16, Cp, y_f16, stream=None):
    _check(load_library().apex_w4a4_gemm_fp8_dual(M, N, K, group_a, group_w, _ptr(a_codes),
                                                  _ptr(a_scales), _ptr(w_codes),
                                                  _ptr(w_scales), _ptr(x_out_f16),
                                                  _ptr(w_out_f16), Cp, _ptr(y_f16),
                                                  _stream(stream)),
           "apex_w4a4_gemm_fp8_dual")


def apex_w4a4_gemm_noalloc(M, N, K, group_a, group_w, a_packed, a_scales, w_packed, w_scales,
                           y_f16, stream=None):
    """apex_w4a4_gemm without a workspace argument: for callers that may not allocate device
    memory at call time; the split-K scratch is a fixed array inside the library."""
    _check(load_library().apex_w4a4_gemm_noalloc(M, N, K, group_a, group_w, _ptr(a_packed),
                                                 _ptr(a_scales), _ptr(w_packed),
                                                 _ptr(w_scales), _ptr(y_f16), _stream(stream)),
           "apex_w4a4_gemm_noalloc")


def apex_w4a4_gemm_workspace_size(M, N, K, group_a, group_w) -> int:
    return int(load_library().apex_w4a4_gemm_workspace_size(M, N, K, group_a, group_w))


def apex_w4a4_linear(M, N, K, group_a, group_w, x_f16, w_packed, w_scales, y_f16,
                     workspace=None, workspace_bytes=None, stream=None):
    if workspace is not None and workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size()
    _check(load_library().apex_w4a4_linear(M, N, K, group_a, group_w, _ptr(x_f16),
                                           _ptr(w_packed), _ptr(w_scales), _ptr(y_f16),
                                           _ptr(workspace), workspace_bytes or 0,
                                           _stream(stream)),
           "apex_w4a4_linear")


def apex_w4a4_linear_workspace_size(M, N, K, group_a, group_w) -> int:
    return int(load_library().apex_w4a4_linear_workspace_size(M, N, K, group_a, group_w))


def apex_w4a4_group_partials(M, N, K, a_packed, w_packed, partials_i32, stream=None):
    _check(load_library().apex_w4a4_group_partials(M, N, K, _ptr(a_packed), _ptr(w_packed),
                                                   _ptr(partials_i32), _stream(stream)),
           "apex_w4a4_group_partials")


def apex_get_device_status(stream=None) -> int:
    return int(load_library().apex_get_device_status(_stream(stream)))


def apex_set_wait_limit_ns(ns: int):
    load_library().apex_set_wait_limit_ns(int(ns))


def apex_select_weight_group(M, N, K, rho, ridge_ops_per_byte) -> int:
    """Host only: 128 or K, see the C header (0 for invalid arguments)."""
    return int(load_library().apex_select_weight_group(int(M), int(N), int(K), float(rho),
                                                       float(ridge_ops_per_byte)))


def apex_debug_withhold_step(step: int):
    load_library().apex_debug_withhold_step(int(step))


def apex_debug_partials_split(on: bool):
    load_library().apex_debug_partials_split(1 if on else 0)


def apex_debug_trace_next_gemm(trace, ctas: int, steps: int):
    """trace: int64 CUDA tensor with at least ctas*16*steps elements (zeroed by the caller)."""
    if trace.numel() < ctas * 16 * steps:
        raise ValueError("trace buffer too small")
    load_library().apex_debug_trace_next_gemm(_ptr(trace), int(ctas), int(steps))


def apex_debug_gemm_plan(M: int, N: int, K: int, sms: int, with_workspace: bool = True) -> dict:
    """The work plan apex_w4a4_gemm would use on a GPU with `sms` SMs (host only)."""
    import ctypes
    out = (ctypes.c_int32 * 6)()
    _check(load_library().apex_debug_gemm_plan(int(M), int(N), int(K), int(sms),
                                               1 if with_workspace else 0, out),
           "apex_debug_gemm_plan")
    return dict(zip(("bt", "tiles", "stages", "ctas", "split_k", "cluster"), list(out)))


# ------------------------------------------------------------------ tensor conveniences

def quantize_act(x, group_a: int = 128, stream=None):
    """fp16 [M, K] CUDA tensor -> (packed uint8 [M, K/2], scales fp16 [M, K/group_a])."""
    import torch
    M, K = x.shape
    packed = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((M, K // group_a), dtype=torch.float16, device=x.device)
    apex_quantize_act_int4(x, M, K, group_a, packed, scales, stream)
    return packed, scales


def pack_weights(w, group_w: int = 128, stream=None):
    """fp16 [N, K] CUDA tensor -> (packed uint8 [N, K/2], scales fp16 [N, K/group_w])."""
    import torch
    N, K = w.shape
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    scales = torch.empty((N, K // group_w), dtype=torch.float16, device=w.device)
    apex_pack_weights_int4(w, N, K, group_w, packed, scales, stream)
    return packed, scales


def workspace(M, N, K, group_a=128, group_w=128, device="cuda", linear=False):
    """A zero-filled workspace of the size apex_w4a4_gemm (or, with linear=True,
    apex_w4a4_linear) uses for this problem (or None)."""
    import torch
    size_fn = apex_w4a4_linear_workspace_size if linear else apex_w4a4_gemm_workspace_size
    nbytes = size_fn(M, N, K, group_a, group_w)
    if nbytes == 0:
        return None
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def gemm(a_packed, a_scales, w_packed, w_scales, group_a=128, group_w=128, out=None,
         ws=None, stream=None):
    """Y = W4A4 GEMM of packed operands -> fp16 [M, N]."""
    import torch
    M = a_packed.shape[0]
    N = w_packed.shape[0]
    K = a_packed.shape[1] * 2
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=a_packed.device)
    apex_w4a4_gemm(M, N, K, group_a, group_w, a_packed, a_scales, w_packed, w_scales, out,
                   ws, None, stream)
    return out
