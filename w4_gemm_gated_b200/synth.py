"""Seeded synthetic inputs for the W4A16 linear layer with a gated Error Compensator.

This module only draws random numbers and stores them on the input grids the
layer consumes (fp32 weights before quantisation, bf16 bit patterns for
activations and EC parameters).  It contains none of the layer's arithmetic:
no quantisation, packing, matmul, gate or low-rank product.  Both the CPU
oracle and the CUDA path take their inputs from here, so the two sides see
bit-identical inputs while sharing no compute code.

Distributions follow the workloads the SPEAR pages evaluate on (per-channel
W4 weights, activations with token-dependent outliers, see the gist.science
technical summary, section 1 "Enonce du probleme"): W ~ N(0, 0.02),
A, B ~ N(0, 0.01), w_g ~ N(0, 1/sqrt(K)), x ~ N(0, 1) with optional outlier
tokens or a heavy-tailed Student-t(3) component on a fixed 1 % of channels.

bf16 values are numpy ``uint16`` arrays holding the raw bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "LayerInputs",
    "make_layer",
    "tiny",
    "decode",
    "prefill",
    "sweep_point",
    "stack_layer_seed",
]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even), return bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    u = np.ascontiguousarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


@dataclass
class LayerInputs:
    """One layer's inputs.  Shapes: x M x K, W K x N (fp32, pre-quantisation),
    A K x r, B r x N, w_g K (all bf16 bit patterns), b_g a Python float."""

    M: int
    K: int
    N: int
    r: int
    x: np.ndarray
    W: np.ndarray
    A: np.ndarray | None
    B: np.ndarray | None
    w_g: np.ndarray | None
    b_g: float
    meta: dict = field(default_factory=dict)


def _activations(M: int, K: int, kind: str, rng: np.random.Generator,
                 force_outlier: bool) -> tuple[np.ndarray, dict]:
    x = rng.standard_normal((M, K), dtype=np.float32)
    meta: dict = {"x_kind": kind}
    if kind == "normal":
        pass
    elif kind == "outlier":
        # A fixed 1 % of input channels carries the outliers; each token is an
        # outlier token independently with probability 0.05 and has those
        # channels scaled by 10.
        n_ch = max(1, int(round(0.01 * K)))
        chans = np.sort(rng.choice(K, size=n_ch, replace=False))
        tok = rng.random(M) < 0.05
        if force_outlier and M > 0 and not tok.any():
            tok[rng.integers(M)] = True
        x[np.ix_(np.nonzero(tok)[0], chans)] *= 10.0
        meta.update(outlier_channels=chans, outlier_tokens=np.nonzero(tok)[0])
    elif kind == "t3":
        # A fixed 1 % of input channels receives an added Student-t(3) sample
        # (unit scale) for every token.
        n_ch = max(1, int(round(0.01 * K)))
        chans = np.sort(rng.choice(K, size=n_ch, replace=False))
        x[:, chans] += rng.standard_t(3, size=(M, n_ch)).astype(np.float32)
        meta.update(t3_channels=chans)
    else:
        raise ValueError(f"unknown activation kind {kind!r}")
    return f32_to_bf16_bits(x), meta


def make_layer(M: int, K: int, N: int, r: int, *, b_g: float = 0.0,
               x_kind: str = "normal", seed: int = 0,
               force_outlier: bool = False, w_std: float = 0.02,
               ec_std: float = 0.01) -> LayerInputs:
    """Draw one layer's inputs.  Every tensor has its own counter-derived stream
    (PCG64 seeded with ``[seed, tensor_id]``), so changing M does not change W."""
    W = _rng(seed, 1).standard_normal((K, N), dtype=np.float32) * np.float32(w_std)
    x, meta = _activations(M, K, x_kind, _rng(seed, 2), force_outlier)
    if r > 0:
        A = f32_to_bf16_bits(_rng(seed, 3).standard_normal((K, r), dtype=np.float32) * np.float32(ec_std))
        B = f32_to_bf16_bits(_rng(seed, 4).standard_normal((r, N), dtype=np.float32) * np.float32(ec_std))
        w_g = f32_to_bf16_bits(_rng(seed, 5).standard_normal(K, dtype=np.float32) * np.float32(1.0 / np.sqrt(K)))
    else:
        A = B = w_g = None
    meta.update(seed=seed)
    return LayerInputs(M, K, N, r, x, W, A, B, w_g, float(b_g), meta)


def tiny(seed: int = 0) -> LayerInputs:
    """Tiny single layer: M=16, K=N=512, r=16, b_g=0."""
    return make_layer(16, 512, 512, 16, b_g=0.0, x_kind="normal", seed=seed)


def decode(M: int, seed: int = 0, force_outlier: bool = False) -> LayerInputs:
    """Decode GEMV shape (7B-style MLP up-projection): K=4096, N=11008, r=64,
    b_g=-1, 5 % outlier tokens with 10x channels."""
    return make_layer(M, 4096, 11008, 64, b_g=-1.0, x_kind="outlier", seed=seed,
                      force_outlier=force_outlier)


def prefill(seed: int = 0, M: int = 2048) -> LayerInputs:
    """Prefill GEMM (attention o-projection shape): M=2048, K=N=4096, r=64,
    Student-t(3) component on 1 % of channels, b_g=-1."""
    return make_layer(M, 4096, 4096, 64, b_g=-1.0, x_kind="t3", seed=seed)


def sweep_point(M: int, K: int, N: int, r: int, seed: int = 0) -> LayerInputs:
    """One point of the fused-vs-unfused dispatch sweep (inputs as the prefill GEMM)."""
    return make_layer(M, K, N, r, b_g=-1.0, x_kind="t3", seed=seed)


def stack_layer_seed(seed: int, layer: int, proj: int) -> int:
    """Seed of projection ``proj`` (0..6 = q,k,v,o,gate,up,down) of decoder layer ``layer``."""
    return int(np.random.SeedSequence([seed, 1000 + layer, proj]).generate_state(1)[0])
