"""CPU oracle for the pure W4A4 group-quantized GEMM (test infrastructure).

TEST INFRASTRUCTURE, NOT PRODUCT CODE: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with ``group_quantized_w4a4_b200`` and never imports it.

The arithmetic lives in ``w4a4_oracle.c`` (plain C, int64 partials, fp64 output),
which follows "APEX4: Efficient Pure W4A4 LLM Inference via Intra-SM Compute
Rebalancing" (abstract: W4A4 with 128-wide groups, INT4 products dequantised per
group).  This module only compiles it with gcc and marshals numpy arrays.

Parity status per function (pins in ``tests/test_oracle_pins.py``):
  f32_to_f16        pinned (numpy float16 cast on edge cases and random values)
  quantize_pack     pinned (exact-rational re-derivation, tie table, round-trip bound)
  unpack            pinned (explicit byte formula, all 256 bytes)
  group_partials    pinned (numpy int64 matmul per group)
  gemm              pinned (fp64 brute force of dequantised operands, group=K closed
                    form, permutation invariance, power-of-two linearity)
  split_outlier_channels, gemm_dual
                    pinned (outlier-only inputs reduce to numpy's fp64 matmul; no
                    outlier channels reduce to gemm; the per-element error bound of the
                    dual path against the exact product; planted mistakes fail it)
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4a4_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libw4a4_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math) and return the .so path."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I32 = ctypes.c_int32
        lib.w4o_f32_to_f16.argtypes = [ctypes.c_float]
        lib.w4o_f32_to_f16.restype = ctypes.c_uint16
        lib.w4o_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.w4o_f16_to_f64.restype = ctypes.c_double
        lib.w4o_quantize_pack.argtypes = [P, I64, I64, I32, P, P]
        lib.w4o_quantize_pack.restype = ctypes.c_int
        lib.w4o_unpack.argtypes = [P, I64, I64, P]
        lib.w4o_unpack.restype = None
        lib.w4o_group_partials.argtypes = [P, P, I64, I64, I64, I32, I32, P, I64, P]
        lib.w4o_group_partials.restype = ctypes.c_int
        lib.w4o_gemm.argtypes = [P, P, P, P, I64, I64, I64, I32, I32, P, I64, P]
        lib.w4o_gemm.restype = ctypes.c_int
        lib.w4o_num_threads.argtypes = []
        lib.w4o_num_threads.restype = ctypes.c_int
        _lib = lib
        return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f16bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        return x.view(np.uint16)
    if x.dtype == np.uint16:
        return x
    raise TypeError("expected float16 values (or their uint16 bit patterns)")


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use on this host."""
    return int(_load().w4o_num_threads())


def f32_to_f16(values) -> np.ndarray:
    """Hand-written fp32 -> fp16 RNE conversion, element by element (uint16 bits)."""
    lib = _load()
    v = np.asarray(values, dtype=np.float32).ravel()
    return np.array([lib.w4o_f32_to_f16(float(t)) for t in v], dtype=np.uint16)


def quantize_pack(x: np.ndarray, group: int):
    """Per-row, per-group symmetric absmax int4 quantization and nibble packing.

    x: [rows, K] float16.  Returns (packed uint8 [rows, K/2], scales float16 [rows, K/group]).
    """
    xb = _f16bits(x)
    if xb.ndim != 2:
        raise ValueError("x must be 2-D")
    rows, K = xb.shape
    if K % group or K % 2 or group % 2:
        raise ValueError("K must be a multiple of the (even) group")
    packed = np.zeros((rows, K // 2), dtype=np.uint8)
    scales = np.zeros((rows, K // group), dtype=np.uint16)
    rc = _load().w4o_quantize_pack(_ptr(xb), rows, K, group, _ptr(packed), _ptr(scales))
    if rc:
        raise ValueError(f"oracle quantize_pack rejected the shape (rc={rc})")
    return packed, scales.view(np.float16)


def unpack(packed: np.ndarray, K: int) -> np.ndarray:
    """Packed nibbles [rows, K/2] -> signed int8 values [rows, K]."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    rows = packed.shape[0]
    q = np.zeros((rows, K), dtype=np.int8)
    _load().w4o_unpack(_ptr(packed), rows, K, _ptr(q))
    return q


def _check(ap, wp, M, N, K, ga, gw, sa=None, sw=None, rows=None):
    if ap.shape != (M, K // 2) or wp.shape != (N, K // 2):
        raise ValueError("packed operands must be [M, K/2] and [N, K/2]")
    if sa is not None and sa.shape != (M, K // ga):
        raise ValueError("activation scales must be [M, K/ga]")
    if sw is not None and sw.shape != (N, K // gw):
        raise ValueError("weight scales must be [N, K/gw]")
    if rows is not None and rows.size and (rows.min() < 0 or rows.max() >= M):
        raise ValueError("row index out of range")


def group_partials(ap, wp, M, N, K, ga, gw, rows=None) -> np.ndarray:
    """Exact per-group integer partials, int64 [K/min(ga,gw), len(rows) or M, N]."""
    ap = np.ascontiguousarray(ap, dtype=np.uint8)
    wp = np.ascontiguousarray(wp, dtype=np.uint8)
    _check(ap, wp, M, N, K, ga, gw,
           rows=None if rows is None else np.asarray(rows, dtype=np.int64))
    ge = min(ga, gw)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = M if r is None else r.size
    out = np.zeros((K // ge, nr, N), dtype=np.int64)
    rc = _load().w4o_group_partials(_ptr(ap), _ptr(wp), M, N, K, ga, gw,
                                    None if r is None else _ptr(r), nr, _ptr(out))
    if rc:
        raise ValueError(f"oracle group_partials failed (rc={rc})")
    return out


def gemm(ap, sa, wp, sw, M, N, K, ga, gw, rows=None) -> np.ndarray:
    """Y = sum_g P_g * sa * sw in fp64, [len(rows) or M, N]."""
    ap = np.ascontiguousarray(ap, dtype=np.uint8)
    wp = np.ascontiguousarray(wp, dtype=np.uint8)
    sab = _f16bits(sa)
    swb = _f16bits(sw)
    _check(ap, wp, M, N, K, ga, gw, sab, swb,
           None if rows is None else np.asarray(rows, dtype=np.int64))
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    nr = M if r is None else r.size
    y = np.zeros((nr, N), dtype=np.float64)
    rc = _load().w4o_gemm(_ptr(ap), _ptr(sab), _ptr(wp), _ptr(swb), M, N, K, ga, gw,
                          None if r is None else _ptr(r), nr, _ptr(y))
    if rc:
        raise ValueError(f"oracle gemm failed (rc={rc})")
    return y


def split_outlier_channels(x: np.ndarray, channels):
    """The activation split of the outlier dual path ("OSC: Hardware Efficient W4A4
    Quantization via Outlier Separation in Channel Dimension", abstract): a fixed set of
    input channels, the same for every token, is pulled out into a compact dense fp16
    tensor for the 16-bit branch, and the 4-bit path sees those channels as zeros.

    x: [rows, K] float16; channels: distinct indices in [0, K).
    Returns (x_in float16 [rows, K] with the channels zeroed, x_out float16
    [rows, len(channels)] holding them in the given order)."""
    x = np.ascontiguousarray(x)
    if x.dtype != np.float16 or x.ndim != 2:
        raise TypeError("x must be a 2-D float16 array")
    ch = np.asarray(channels, dtype=np.int64)
    if ch.size and (ch.min() < 0 or ch.max() >= x.shape[1] or np.unique(ch).size != ch.size):
        raise ValueError("channels must be distinct indices of x's columns")
    x_in = x.copy()
    x_in[:, ch] = 0
    return x_in, np.ascontiguousarray(x[:, ch])


def gemm_dual(ap, sa, wp, sw, x_out, w_out, M, N, K, ga, gw, rows=None) -> np.ndarray:
    """The dual-path output (OSC abstract): the W4A4 path on the quantized operands,
    Y4 = gemm(ap, sa, wp, sw, ...), plus the 16-bit branch over the outlier channels,
    x_out [M, C] . w_out [N, C]^T, the fp16 values multiplied exactly and summed in fp64
    (numpy matmul as the library step).  [len(rows) or M, N] float64."""
    y = gemm(ap, sa, wp, sw, M, N, K, ga, gw, rows)
    xo = np.asarray(x_out)
    wo = np.asarray(w_out)
    if xo.dtype != np.float16 or wo.dtype != np.float16:
        raise TypeError("the 16-bit branch operands must be float16")
    if xo.shape[0] != M or wo.shape[0] != N or xo.shape[1] != wo.shape[1]:
        raise ValueError("x_out must be [M, C] and w_out [N, C]")
    if rows is not None:
        xo = xo[np.asarray(rows, dtype=np.int64)]
    return y + xo.astype(np.float64) @ wo.astype(np.float64).T


def within_tolerance(y, y_ref, max_abs_ref=None):
    """Acceptance rule for an fp16 output against the fp64 oracle:
    |y - y_ref| <= 2^-10 |y_ref| + 1e-3 * max|y_ref| (max over the whole GEMM output).
    Returns (ok, worst excess ratio)."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    mx = float(np.max(np.abs(y_ref))) if max_abs_ref is None else float(max_abs_ref)
    bound = 2.0 ** -10 * np.abs(y_ref) + 1e-3 * mx
    err = np.abs(y - y_ref)
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0
    return bool(np.all(err <= bound)), ratio
