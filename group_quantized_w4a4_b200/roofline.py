"""Roofline arithmetic used by the benchmark.

The crossover model comes from "Why INT4 Weight-Only Quantization Doesn't Speed Up
Prefill" (section "Where does a weight-stationary GEMM stop being memory-bound?"):
a weight-stationary GEMM that reads each weight once and uses it for B token vectors
does 2*B FLOP per weight, so its intensity is 2*B / b FLOP per byte for b bytes per
weight; it turns compute-bound once that reaches the machine's ridge point
(dense FLOP/s divided by HBM byte/s).  Solving for B gives B* = ridge * b / 2.

For a W4A4 GEMM both operands are 0.5 byte per element; the full byte count
(activations, both scale tensors, fp16 output) is used for the bound below.
"""
from __future__ import annotations


def ridge_point(dense_ops_per_s: float, hbm_bytes_per_s: float) -> float:
    """Operations per byte at which compute time equals memory time."""
    return dense_ops_per_s / hbm_bytes_per_s


def crossover_tokens(dense_ops_per_s: float, hbm_bytes_per_s: float,
                     bytes_per_weight: float) -> float:
    """Concurrent tokens B at which a weight-stationary GEMM becomes compute-bound."""
    return ridge_point(dense_ops_per_s, hbm_bytes_per_s) * bytes_per_weight / 2.0


def bound_time_s(ops: float, nbytes: float, peak_ops_per_s: float,
                 hbm_bytes_per_s: float) -> tuple[float, str]:
    """Lower bound on a kernel's time and which resource sets it ("tensor" or "hbm")."""
    t_c = ops / peak_ops_per_s
    t_m = nbytes / hbm_bytes_per_s
    return (t_c, "tensor") if t_c >= t_m else (t_m, "hbm")
