"""Seeded synthetic inputs for the W4A4 GEMM workloads (no quantization arithmetic here).

This module only draws random fp16 matrices.  It is the one piece of code that both
the CUDA path (bench, GPU tests) and the CPU oracle (pins, parity references) consume;
it computes nothing of the method itself.

Distributions follow the workload descriptions of the W4A4-g128 benchmarks:
  * activations ~ N(0, 1)            ("normal")
  * activations ~ N(0, 1), 1% of the K channels (the same channels for every token,
    chosen once per seed) multiplied by 20  ("outlier"; token-persistent outlier
    channels as described in the OSC paper's abstract)
  * activations ~ Student-t(df=4) / sqrt(2)  ("student_t", unit variance)
  * weights ~ N(0, 0.02)
All values are drawn with numpy's PCG64 in float32 and rounded to fp16 (RNE).
Seeds: base seed s; activations use s*16+0, weights s*16+1, outlier pick s*16+2.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


def _rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(np.random.PCG64(seed))


def normal_f16(shape, std: float, seed: int) -> np.ndarray:
    x = _rng(seed).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x.astype(np.float16)


def student_t4_f16(shape, seed: int) -> np.ndarray:
    x = _rng(seed).standard_t(4.0, size=shape).astype(np.float32)
    x *= np.float32(1.0 / math.sqrt(2.0))
    return x.astype(np.float16)


def outlier_channels(K: int, seed: int, frac: float = 0.01) -> np.ndarray:
    n = int(math.ceil(frac * K))
    return np.sort(_rng(seed).choice(K, size=n, replace=False))


def activations(M: int, K: int, dist: str, seed: int) -> np.ndarray:
    """fp16 [M, K] activations for base seed `seed`."""
    if dist == "normal":
        return normal_f16((M, K), 1.0, seed * 16 + 0)
    if dist == "outlier":
        x = _rng(seed * 16 + 0).standard_normal(size=(M, K), dtype=np.float32)
        ch = outlier_channels(K, seed * 16 + 2)
        x[:, ch] *= np.float32(20.0)
        return x.astype(np.float16)
    if dist == "student_t":
        return student_t4_f16((M, K), seed * 16 + 0)
    raise ValueError(f"unknown activation distribution {dist!r}")


def weights(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    """fp16 [N, K] weights (PyTorch Linear layout) for base seed `seed`."""
    return normal_f16((N, K), std, seed * 16 + 1)


@dataclass(frozen=True)
class Gemm:
    """One W4A4 GEMM problem: Y[M,N] = A[M,K] . W[N,K]^T with K-groups ga / gw."""
    name: str
    M: int
    N: int
    K: int
    ga: int
    gw: int
    act: str
    seed: int

    @property
    def ops(self) -> float:
        return 2.0 * self.M * self.N * self.K

    def gemm_bytes(self, form: str = "packed") -> int:
        """Algorithmic HBM bytes of one GEMM call: A, W, fp16 scales, fp16 Y.  A is packed
        int4 plus scales ("packed") or one byte per element plus scales ("expanded");
        "fp8" has one byte per element for both A and W (E4M3 codes of the int4 values)."""
        M, N, K = self.M, self.N, self.K
        a = {"packed": M * K // 2 + 2 * M * (K // self.ga),
             "expanded": M * K + 2 * M * (K // self.ga),
             "fp8": M * K + 2 * M * (K // self.ga)}[form]
        w = N * K if form == "fp8" else N * K // 2     # fp8: one byte per weight
        return a + w + 2 * N * (K // self.gw) + 2 * M * N

    def quant_bytes(self, form: str = "packed") -> int:
        """Algorithmic HBM bytes of the online activation quantizer."""
        M, K = self.M, self.K
        return 2 * M * K + (M * K // 2 if form == "packed" else M * K) + 2 * M * (K // self.ga)


def workloads() -> dict:
    """The named W4A4 workloads (all fp16 inputs, g128 activations)."""
    w = {}
    w["tiny_m16_n256_k512"] = Gemm("tiny_m16_n256_k512", 16, 256, 512, 128, 128, "normal", 1000)
    w["decode_m16_n8192_k8192"] = Gemm("decode_m16_n8192_k8192", 16, 8192, 8192, 128, 128,
                                       "normal", 1001)
    w["prefill_m4096_n8192_k8192"] = Gemm("prefill_m4096_n8192_k8192", 4096, 8192, 8192,
                                          128, 128, "outlier", 1002)
    w["mlp_up_m2048_n28672_k8192"] = Gemm("mlp_up_m2048_n28672_k8192", 2048, 28672, 8192,
                                          128, 128, "student_t", 1003)
    w["mlp_down_m2048_n8192_k28672"] = Gemm("mlp_down_m2048_n8192_k28672", 2048, 8192, 28672,
                                            128, 128, "student_t", 10031)
    for gw in (128, 512, 8192):
        for M in (1, 16, 128, 1024, 4096):
            nm = f"sweep_m{M}_gw{gw}"
            w[nm] = Gemm(nm, M, 8192, 8192, 128, gw, "outlier", 1004)
    return w


def make(g: Gemm):
    """(A fp16 [M,K], W fp16 [N,K]) for a workload."""
    return activations(g.M, g.K, g.act, g.seed), weights(g.N, g.K, g.seed)
