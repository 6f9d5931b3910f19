"""Seeded synthetic inputs for the ARL2 layer (shared by the tests, the bench and smoke).

This module only draws random numbers and rounds them to bfloat16. It holds none
of the layer's arithmetic, so the CUDA path and the fp64 oracle can both take
their inputs from here without sharing any computation.

Recipe (the pages give no token counts or distributions; these are the chosen
synthetic stand-ins for their 480p autoregressive video workloads):
  * every tensor has its own stream ``SeedSequence([seed, config, frame, pass, tensor])``
    over numpy's PCG64;
  * values are drawn in float32 and rounded to bfloat16 round-to-nearest-even;
  * q, k, v ~ N(0, 1); phi weights ~ N(0, std 1/sqrt(d));
  * forget gate alpha = sigmoid(N(2, 0.5)), rate beta = sigmoid(N(0, 1)), kept fp32.
Pass ids 0..3 are the denoising passes of a frame, pass 4 is its clean pass.
"""
from __future__ import annotations

import numpy as np

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_ALPHA, TENSOR_BETA = 0, 1, 2, 3, 4
TENSOR_WQ, TENSOR_WK, TENSOR_WV, TENSOR_STATE = 5, 6, 7, 8
TENSOR_X, TENSOR_WA, TENSOR_WB = 9, 10, 11
CLEAN_PASS = 4
_WEIGHT_FRAME = 0xFFFF  # frame slot used for the per-layer phi weights


def rng(seed: int, config: int, frame: int, pass_: int, tensor: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, config, frame, pass_, tensor])))


def bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float64 exactly."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _sigmoid32(x: np.ndarray) -> np.ndarray:
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def qkv(seed: int, config: int, frame: int, pass_: int, B: int, T: int, H: int, d: int):
    """q, k, v of one pass as bfloat16 bit arrays of shape [B, T, H, d] (token-major)."""
    out = []
    for t in (TENSOR_Q, TENSOR_K, TENSOR_V):
        g = rng(seed, config, frame, pass_, t)
        out.append(bf16_bits(g.standard_normal((B, T, H, d), dtype=np.float32)))
    return tuple(out)


def gates(seed: int, config: int, frame: int, B: int, H: int, T: int):
    """alpha, beta of a frame's clean pass, float32 of shape [B, H, T]."""
    ga = rng(seed, config, frame, CLEAN_PASS, TENSOR_ALPHA)
    gb = rng(seed, config, frame, CLEAN_PASS, TENSOR_BETA)
    alpha = _sigmoid32(ga.normal(2.0, 0.5, size=(B, H, T)).astype(np.float32))
    beta = _sigmoid32(gb.standard_normal((B, H, T), dtype=np.float32))
    return alpha, beta


def feature_maps(seed: int, config: int, H: int, d: int):
    """phi_q, phi_k, phi_v weights as bfloat16 bits [H, d_in, d_out]; x' = x @ W[h]."""
    out = []
    for t in (TENSOR_WQ, TENSOR_WK, TENSOR_WV):
        g = rng(seed, config, _WEIGHT_FRAME, 0, t)
        w = g.standard_normal((H, d, d), dtype=np.float32) / np.float32(np.sqrt(d))
        out.append(bf16_bits(w.astype(np.float32)))
    return tuple(out)


def hidden(seed: int, config: int, frame: int, B: int, T: int, D: int) -> np.ndarray:
    """The clean pass's hidden states x ~ N(0, 1), bfloat16 bits [B, T, D] (D: model width)."""
    g = rng(seed, config, frame, CLEAN_PASS, TENSOR_X)
    return bf16_bits(g.standard_normal((B, T, D), dtype=np.float32))


def gate_weights(seed: int, config: int, H: int, D: int):
    """Gate projections for gates produced from x: Wa, Wb as bfloat16 bits [H, D] and biases
    ba, bb as float32 [H]. Wa ~ N(0, std 0.5/sqrt(D)) with ba = 2 and Wb ~ N(0, std 1/sqrt(D))
    with bb = 0, so that for x ~ N(0, 1) alpha = sigmoid(N(2, 0.5)) and beta = sigmoid(N(0, 1)),
    the same distributions as the gates drawn directly."""
    ga = rng(seed, config, _WEIGHT_FRAME, 0, TENSOR_WA)
    gb = rng(seed, config, _WEIGHT_FRAME, 0, TENSOR_WB)
    wa = ga.standard_normal((H, D), dtype=np.float32) * np.float32(0.5 / np.sqrt(D))
    wb = gb.standard_normal((H, D), dtype=np.float32) / np.float32(np.sqrt(D))
    return (bf16_bits(wa.astype(np.float32)), np.full(H, 2.0, np.float32),
            bf16_bits(wb.astype(np.float32)), np.zeros(H, np.float32))


def state(seed: int, config: int, B: int, H: int, d: int, scale: float = 1.0) -> np.ndarray:
    """A float32 state [B, H, d_k, d_v] ~ N(0, scale^2), for set_state tests."""
    g = rng(seed, config, _WEIGHT_FRAME, 1, TENSOR_STATE)
    return (g.standard_normal((B, H, d, d), dtype=np.float32) * np.float32(scale)).astype(np.float32)


# The workloads, by name. Shapes come from the configurations the layer is
# measured on; "frames" counts autoregressive frames, each with 4 denoising
# queries and one clean-pass commit.
WORKLOADS = {
    "tiny": dict(config=0, B=1, H=2, T=64, d=32, frames=4, queries=2),
    "480p": dict(config=1, B=1, H=12, T=1560, d=128, frames=21, queries=4),
    "stream240": dict(config=2, B=1, H=12, T=1560, d=128, frames=240, queries=4),
    "sweep": dict(config=3, B=(1, 4), H=12, T=(390, 1560, 3600), d=128, frames=21, queries=4),
    "kv_baseline": dict(config=4, B=1, H=12, T=1560, d=128, frames=(21, 60, 120), queries=4),
}
