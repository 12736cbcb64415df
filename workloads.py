"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the benchmark.

This module only draws random numbers and rounds them to bf16 input patterns. It holds
none of the coding or matmul arithmetic, so that both the oracle and the CUDA path can
take their inputs from it without sharing any of the method.

Workloads (sizes and value distributions of the pages' settings):
  * DYADIC_1: one 2048x2048 weight, N(0, 0.02^2) with 0.1% of the entries (exactly
    round(0.001*n*k) positions, drawn without replacement) multiplied by 20; one
    N(0, 1) activation vector of length 2048.
  * DECODE_SWEEP: a Llama-style 1B stack, hidden 2048, intermediate 5632, 24 layers of
    seven projections (q 2048x2048, k 256x2048, v 256x2048, o 2048x2048,
    gate 5632x2048, up 5632x2048, down 2048x5632), weights as in DYADIC_1; batch
    1/4/16 activations N(0, 1).
  * LLOYD_G32: 224 matrices 2048x2048, Laplace(0, 0.015) times a per-row factor drawn
    from U(0.5, 2).
  * PREFILL: weights (n, k) = (4096, 11008) and (11008, 4096) as in DYADIC_1;
    activations [m, k] N(0, 1), m in {16, 128, 512, 2048, 4096}.
  * LUT16: 8192x28672 weights, N(0, 0.01^2) or Student-t(4) * 0.01.

Seeds: workload i draws matrix j from numpy PCG64 seeded [1000 + i, j] and activation
set j from [2000 + i, j]. Values are drawn in float64, rounded to float32 and then to
bf16 (round to nearest even at each step).
"""
from __future__ import annotations

import numpy as np

# workload ids (seed offsets)
DYADIC_1, DECODE_SWEEP, LLOYD_G32, PREFILL, LUT16 = 1, 2, 3, 4, 5

HIDDEN, INTERMEDIATE, LAYERS = 2048, 5632, 24
KV_ROWS = 256
SWEEP_PROJ = [("q", HIDDEN, HIDDEN), ("k", KV_ROWS, HIDDEN), ("v", KV_ROWS, HIDDEN),
              ("o", HIDDEN, HIDDEN), ("gate", INTERMEDIATE, HIDDEN),
              ("up", INTERMEDIATE, HIDDEN), ("down", HIDDEN, INTERMEDIATE)]
PREFILL_SHAPES = [(4096, 11008), (11008, 4096)]
PREFILL_M = [16, 128, 512, 2048, 4096]
LUT16_SHAPE = (8192, 28672)


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float64 -> float32 -> bf16 bit patterns, round to nearest even at each step."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16).reshape(a.shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rng(workload: int, index: int, activations: bool = False) -> np.random.Generator:
    return np.random.default_rng([(2000 if activations else 1000) + workload, index])


def gaussian_outlier_weight(n: int, k: int, workload: int, index: int,
                            sigma: float = 0.02, outlier_frac: float = 0.001,
                            outlier_mult: float = 20.0) -> np.ndarray:
    """N(0, sigma^2) with exactly round(frac*n*k) entries (no replacement) scaled by mult."""
    g = rng(workload, index)
    w = g.normal(0.0, sigma, size=(n, k))
    n_out = int(round(outlier_frac * n * k))
    if n_out:
        pos = g.choice(n * k, size=n_out, replace=False)
        w.reshape(-1)[pos] *= outlier_mult
    return f64_to_bf16_bits(w)


def activations(m: int, k: int, workload: int, index: int = 0) -> np.ndarray:
    return f64_to_bf16_bits(rng(workload, index, activations=True).normal(0.0, 1.0, size=(m, k)))


def laplace_rowscaled_weight(n: int, k: int, workload: int = LLOYD_G32, index: int = 0,
                             b: float = 0.015) -> np.ndarray:
    g = rng(workload, index)
    w = g.laplace(0.0, b, size=(n, k))
    w *= g.uniform(0.5, 2.0, size=(n, 1))
    return f64_to_bf16_bits(w)


def lut16_weight(n: int, k: int, heavy_tail: bool, workload: int = LUT16, index: int = 0) -> np.ndarray:
    g = rng(workload, index + (1 if heavy_tail else 0))
    if heavy_tail:
        w = g.standard_t(4.0, size=(n, k)) * 0.01
    else:
        w = g.normal(0.0, 0.01, size=(n, k))
    return f64_to_bf16_bits(w)


def sweep_matrices(layers: int = LAYERS):
    """(layer, name, n, k, index) for the decode-sweep stack, in execution order."""
    out = []
    idx = 0
    for layer in range(layers):
        for name, n, k in SWEEP_PROJ:
            out.append((layer, name, n, k, idx))
            idx += 1
    return out


def sweep_weight_count(layers: int = LAYERS) -> int:
    return sum(n * k for _, _, n, k, _ in sweep_matrices(layers))
