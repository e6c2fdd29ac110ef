"""Seeded synthetic inputs for the W8A8 linear layer.

This module only draws random numbers and packs them as bf16 bit patterns.
It holds none of the layer's arithmetic (no absmax, no scales, no rounding to
int8, no products), so both the CUDA path and the CPU oracle can take their
inputs from it without sharing any of the method.

Recipe (one numpy ``PCG64`` stream per role, spawned from ``SeedSequence(seed)``
in a fixed order: X, outlier-column choice, outlier sign/magnitude, W, bias,
calibration batch):

* samples are drawn in float32 and rounded to bf16 round-to-nearest-even;
* "scaled xF" outlier columns multiply the column by F, "offset +-V" outlier
  columns add a per-column signed constant;
* the number of outlier columns for a fraction f of K is ``round(f*K)``,
  chosen with ``rng.choice(K, n, replace=False)`` and returned sorted.

The shapes and distributions follow the workloads of the pages:
"量化基础与INT8" (quantization-flow example: X [tokens, K], W [out, in]),
"从自动驾驶芯片到大语言模型INT8量化训练实战解析" §2.1 (activations ~ randn*0.1
with the first channels offset by +50), "SmoothQuant量化实战：W8A8推理部署与单节点
530B模型落地" §1.2 (a few channels tens of times larger than the rest) and
"LLM.int8()技术解析" §2.1 (about 0.1% outlier activations).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

PER_TENSOR = 0
PER_CHANNEL = 1

_ROLES = ("x", "cols", "mag", "w", "bias", "calib")


def f32_to_bf16_bits(a) -> np.ndarray:
    """Pack finite float32 values as bf16 bit patterns, round-to-nearest-even (format conversion only)."""
    u = np.array(np.asarray(a, dtype=np.float32), copy=True, order="C").view(np.uint32)
    lsb = u >> np.uint32(16)
    lsb &= np.uint32(1)
    u += np.uint32(0x7FFF)
    u += lsb
    u >>= np.uint32(16)
    return u.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint16))
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _streams(seed: int) -> dict:
    kids = np.random.SeedSequence(seed).spawn(len(_ROLES))
    return {r: np.random.Generator(np.random.PCG64(k)) for r, k in zip(_ROLES, kids)}


@dataclass
class Problem:
    """One W8A8 linear workload: X [M,K] and W [N,K] as bf16 bits (row-major, K contiguous)."""

    name: str
    X: np.ndarray
    W: np.ndarray
    bias: Optional[np.ndarray] = None
    calib: Optional[np.ndarray] = None  # calibration batch [Mc,K]; None => calibrate on X
    alpha: float = 0.5
    w_gran: int = PER_CHANNEL
    threshold: float = 6.0
    outlier_cols: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))

    @property
    def M(self) -> int:
        return self.X.shape[0]

    @property
    def N(self) -> int:
        return self.W.shape[0]

    @property
    def K(self) -> int:
        return self.X.shape[1]


def _normal(rng, shape, sigma):
    x = rng.standard_normal(shape, dtype=np.float32)
    x *= np.float32(sigma)
    return x


def _pick_cols(rng, K, n):
    if n <= 0:
        return np.zeros(0, np.int64)
    return np.sort(rng.choice(K, n, replace=False)).astype(np.int64)


def tiny(seed: int = 0) -> Problem:
    """X [16,256] ~N(0,0.1), channels 0-1 offset +50; W [256,256] ~N(0,0.02); per-tensor W."""
    g = _streams(seed)
    x = _normal(g["x"], (16, 256), 0.1)
    x[:, 0:2] += np.float32(50.0)
    w = _normal(g["w"], (256, 256), 0.02)
    return Problem("tiny_16x256x256", f32_to_bf16_bits(x), f32_to_bf16_bits(w), alpha=0.5,
                   w_gran=PER_TENSOR, threshold=6.0, outlier_cols=np.array([0, 1], np.int64))


def llama7b_mlp_up(seed: int = 0, M: int = 2048) -> Problem:
    """X [M,4096] ~N(0,1) with round(0.1% K) columns scaled x60; W [11008,4096] ~N(0,0.02)."""
    K, N = 4096, 11008
    g = _streams(seed)
    x = _normal(g["x"], (M, K), 1.0)
    cols = _pick_cols(g["cols"], K, int(round(0.001 * K)))
    x[:, cols] *= np.float32(60.0)
    w = _normal(g["w"], (N, K), 0.02)
    return Problem(f"llama7b_mlp_up_{M}x{N}x{K}", f32_to_bf16_bits(x), f32_to_bf16_bits(w),
                   alpha=0.5, w_gran=PER_CHANNEL, threshold=6.0, outlier_cols=cols)


def decode(M: int, seed: int = 0, K: int = 4096, N: int = 4096, calib_tokens: int = 512) -> Problem:
    """M tokens, X ~N(0,1) with 6 channels offset +-40 (sign per channel); W [N,K] ~N(0,0.02).

    The smoothing vector is calibrated on a separate batch of ``calib_tokens`` tokens of the
    same distribution (same outlier channels and signs)."""
    g = _streams(seed)
    cols = _pick_cols(g["cols"], K, 6)
    signs = np.where(g["mag"].random(len(cols)) < 0.5, -1.0, 1.0).astype(np.float32)
    x = _normal(g["x"], (M, K), 1.0)
    x[:, cols] += np.float32(40.0) * signs
    c = _normal(g["calib"], (calib_tokens, K), 1.0)
    c[:, cols] += np.float32(40.0) * signs
    w = _normal(g["w"], (N, K), 0.02)
    return Problem(f"decode_{M}x{N}x{K}", f32_to_bf16_bits(x), f32_to_bf16_bits(w),
                   calib=f32_to_bf16_bits(c), alpha=0.5, w_gran=PER_CHANNEL, outlier_cols=cols)


def llmint8_sweep(frac: float, seed: int = 0, M: int = 4096, K: int = 8192, N: int = 8192,
                  truncate: Optional[float] = 5.5) -> Problem:
    """X = 0.5*t(nu=3) [M,K] plus round(frac*K) columns offset by +-U(20,200); W ~N(0,0.015).

    With ``truncate`` set, base samples whose magnitude exceeds it are redrawn until none does,
    so that only the injected columns cross the 6.0 threshold; ``truncate=None`` keeps the
    literal heavy-tailed draw (nearly every column then crosses the threshold)."""
    g = _streams(seed)
    rx = g["x"]
    x = (np.float32(0.5) * rx.standard_t(3, size=(M, K))).astype(np.float32)
    if truncate is not None:
        bad = np.abs(x) > truncate
        while bad.any():
            x[bad] = (np.float32(0.5) * rx.standard_t(3, size=int(bad.sum()))).astype(np.float32)
            bad = np.abs(x) > truncate
    cols = _pick_cols(g["cols"], K, int(round(frac * K)))
    if len(cols):
        rm = g["mag"]
        mags = rm.uniform(20.0, 200.0, len(cols)).astype(np.float32)
        signs = np.where(rm.random(len(cols)) < 0.5, -1.0, 1.0).astype(np.float32)
        x[:, cols] += mags * signs
    w = _normal(g["w"], (N, K), 0.015)
    tag = "lit" if truncate is None else f"{frac:g}"
    return Problem(f"llmint8_{tag}_{M}x{N}x{K}", f32_to_bf16_bits(x), f32_to_bf16_bits(w),
                   alpha=0.5, w_gran=PER_CHANNEL, threshold=6.0, outlier_cols=cols)


def ffn70b(alpha: float = 0.5, seed: int = 0, M: int = 8192) -> Problem:
    """X [M,8192] ~N(0,1) with round(0.05% K) columns scaled x100; W [28672,8192] ~N(0,0.01);
    bias [28672] ~N(0,0.1)."""
    K, N = 8192, 28672
    g = _streams(seed)
    x = _normal(g["x"], (M, K), 1.0)
    cols = _pick_cols(g["cols"], K, int(round(0.0005 * K)))
    x[:, cols] *= np.float32(100.0)
    w = _normal(g["w"], (N, K), 0.01)
    b = _normal(g["bias"], (N,), 0.1)
    return Problem(f"ffn70b_a{alpha:g}_{M}x{N}x{K}", f32_to_bf16_bits(x), f32_to_bf16_bits(w),
                   bias=f32_to_bf16_bits(b), alpha=alpha, w_gran=PER_CHANNEL, outlier_cols=cols)


def random_problem(M: int, N: int, K: int, seed: int = 0, outliers: int = 2, offset: float = 30.0,
                   sigma_x: float = 1.0, sigma_w: float = 0.02, bias: bool = True,
                   w_gran: int = PER_CHANNEL, alpha: float = 0.5, threshold: float = 6.0) -> Problem:
    """Small ragged-shape problem with ``outliers`` columns offset by +-``offset``."""
    g = _streams(seed)
    x = _normal(g["x"], (M, K), sigma_x)
    cols = _pick_cols(g["cols"], K, min(outliers, K))
    if len(cols):
        signs = np.where(g["mag"].random(len(cols)) < 0.5, -1.0, 1.0).astype(np.float32)
        x[:, cols] += np.float32(offset) * signs
    w = _normal(g["w"], (N, K), sigma_w)
    b = f32_to_bf16_bits(_normal(g["bias"], (N,), 0.1)) if bias else None
    return Problem(f"random_{M}x{N}x{K}_s{seed}", f32_to_bf16_bits(x), f32_to_bf16_bits(w), bias=b,
                   alpha=alpha, w_gran=w_gran, threshold=threshold, outlier_cols=cols)


def workload(name: str, **kw) -> Problem:
    """Look a workload up by name: tiny, llama7b_mlp_up, decode, llmint8_sweep, ffn70b."""
    table = {"tiny": tiny, "llama7b_mlp_up": llama7b_mlp_up, "decode": decode,
             "llmint8_sweep": llmint8_sweep, "ffn70b": ffn70b}
    return table[name](**kw)
