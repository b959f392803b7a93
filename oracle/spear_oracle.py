"""CPU oracle for the W4A16 linear layer with a per-token-gated Error Compensator.

TEST INFRASTRUCTURE.  This module is the plain, slow, obviously correct
reference that the CUDA library is checked against.  Only the test suite,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` may import it.  The product path never calls it, and it shares no
code with the CUDA library (it imports only numpy and the seeded input
generators, which hold no layer arithmetic).

What it computes (SPEAR, gist.science technical summary, section 2.1 A
"Compensateurs d'erreurs adaptatifs a l'entree": an EC projects x into a
low-rank space with A, applies an input-dependent gate and projects back with
B, on top of the quantised weight; abstract on fugumt.com: ECs "modulated by
per-token gates" on top of W4 per-channel weights), in the row-vector,
scalar-gate form this library implements:

    g_t = sigmoid(x_t . w_g + b_g)
    y_t = x_t . dequant(W4) + g_t * ((x_t . A) . B)

with x (M x K), W logically K x N stored per output channel, A (K x r),
B (r x N), w_g (K), b_g a scalar.  Everything is evaluated in float64 from
the exact values of the bf16 / fp16 inputs.

Readings where the pages are silent:
  * the pages' global strength alpha is 1 (folded into B);
  * quantiser: symmetric RTN; scale s = fp16_rne(max|w| / 7) computed in
    fp32, saturated to 65504; a scale that is 0 becomes 1.0 with all codes 0;
    codes q = clamp(rint_even(w / s), -7, 7) with the fp32 quotient;
  * stored code is offset binary u = q + 8;
  * the packed layout is the library's own (defined in ``pack_w4`` below and
    in the public header); the pages give none.

The pages' own gate form, W + alpha B diag(gamma(A x)) A with gamma a
bottleneck MLP, is ``linear_rank_gated`` below (per-rank gates).

Parity status: every function here is pinned by ``tests/test_oracle.py``
against hand-worked fixtures, closed forms, invariants or brute force.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_to_f64",
    "f32_to_bf16_bits_rne",
    "quantize_rtn",
    "pack_w4",
    "unpack_w4",
    "w4_nibble_address",
    "dequantize",
    "gate",
    "gate_mask_count",
    "linear",
    "linear_bruteforce",
    "prescale_B",
    "ec_pack",
    "TAU_DEFAULT",
]

TAU_DEFAULT = 0.1
FP16_MAX = 65504.0


# ----------------------------------------------------------------------------
# storage formats
# ----------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns as float64 (bf16 = top half of fp32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f32_to_bf16_bits_rne(v: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16, ties to even, by integer arithmetic on the
    IEEE bit pattern (finite inputs; NaN becomes the canonical quiet NaN)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    u = v.view(np.uint32).astype(np.uint64)
    keep = u >> 16
    low = u & 0xFFFF
    up = (low > 0x8000) | ((low == 0x8000) & ((keep & 1) == 1))
    out = (keep + up.astype(np.uint64)).astype(np.uint16)
    out[np.isnan(v)] = 0x7FC0
    return out


# ----------------------------------------------------------------------------
# a-0: symmetric round-to-nearest int4 quantiser (per channel, or per group of 128 k)
# ----------------------------------------------------------------------------

def _rtn_blocks(Wb: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """RTN over axis 0 of ``Wb`` (one block per remaining index), fp32 arithmetic.

    s = fp16_rne(max|w| / 7) (saturated to 65504; 0 -> 1.0 with codes 0),
    q = clamp(rint_even(w / s), -7, 7) with the IEEE fp32 quotient.
    """
    w32 = Wb.astype(np.float32)
    m = np.max(np.abs(w32), axis=0)
    with np.errstate(over="ignore"):
        s16 = (m / np.float32(7.0)).astype(np.float16)
    s16 = np.where(np.isfinite(s16), s16, np.float16(FP16_MAX)).astype(np.float16)
    zero = s16 == 0
    s16 = np.where(zero, np.float16(1.0), s16).astype(np.float16)
    q = np.clip(np.rint(w32 / s16.astype(np.float32)), -7, 7)
    q = np.where(zero, 0.0, q).astype(np.int8)
    return s16, q


def quantize_rtn(W: np.ndarray, group: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """Quantise W (K x N fp32) to int4 codes.

    SPEAR evaluates W4 per-channel RTN weights (gist.science technical summary,
    section 3.1: "RTN, per-channel"); the group-of-128 variant uses one scale
    per (128 consecutive k, output channel).

    Returns q (N x K int8, values in [-7, 7]) and scales s: float16 [N]
    (group 0) or float16 [K/128, N] (group 128).
    """
    W = np.asarray(W, dtype=np.float32)
    K, N = W.shape
    if group == 0:
        s, q = _rtn_blocks(W)                          # s [N], q K x N
        return np.ascontiguousarray(q.T), s
    if group != 128:
        raise ValueError("group must be 0 (per channel) or 128")
    if K % 128:
        raise ValueError("group-128 quantisation needs K % 128 == 0")
    G = K // 128
    s, q = _rtn_blocks(W.reshape(G, 128, N).transpose(1, 0, 2))   # s [G, N], q 128 x G x N
    q = q.transpose(1, 0, 2).reshape(K, N)
    return np.ascontiguousarray(q.T), s


# ----------------------------------------------------------------------------
# a-1: packed int4 layout
# ----------------------------------------------------------------------------
#
# The packed weight is a grid of 512-byte tiles, each holding 16 output
# channels x 64 input features.  Tile (p, t) (p = n // 16, t = k // 64) starts at
# byte (p * (K/64) + t) * 512.  Inside a tile, "lane" L = 0..31 owns bytes
# [16L, 16L + 16) as four little-endian 32-bit words w_s (s = 0..3) at byte
# 16L + 4s.  With rho = L // 4 and c = L % 4, nibble slot i = 0..7 of word s
# (bits 4i..4i+3) holds the code of
#       row  n = 16p + rho + 8 * (i & 1)
#       col  k = 64t + 16c + 4s + 2 * ((i & 3) >> 1) + (i >> 2)
# stored as u = q + 8.

def w4_nibble_address(n: int, k: int, K: int) -> tuple[int, int]:
    """(byte offset, nibble index 0 = low / 1 = high) of code (n, k), per the layout above."""
    p, rr = divmod(n, 16)
    t, kk = divmod(k, 64)
    c, rest = divmod(kk, 16)
    s, o = divmod(rest, 4)
    rho, half = rr % 8, rr // 8
    i = (2 * (o >> 1) + half) + 4 * (o & 1)
    lane = 4 * rho + c
    byte = (p * (K // 64) + t) * 512 + 16 * lane + 4 * s + (i >> 1)
    return byte, i & 1


def _layout_index(N: int, K: int) -> tuple[np.ndarray, np.ndarray]:
    """For every (n, k) the byte offset and nibble index of its code."""
    n = np.arange(N)[:, None]
    k = np.arange(K)[None, :]
    p, rr = n // 16, n % 16
    t, kk = k // 64, k % 64
    c, rest = kk // 16, kk % 16
    s, o = rest // 4, rest % 4
    rho, half = rr % 8, rr // 8
    i = (2 * (o >> 1) + half) + 4 * (o & 1)
    lane = 4 * rho + c
    byte = (p * (K // 64) + t) * 512 + 16 * lane + 4 * s + (i >> 1)
    return np.broadcast_to(byte, (N, K)), np.broadcast_to(i & 1, (N, K))


def pack_w4(q: np.ndarray) -> np.ndarray:
    """Pack codes q (N x K int8 in [-8, 7]) into the tiled layout; returns uint8 [N*K/2]."""
    q = np.asarray(q)
    N, K = q.shape
    if N % 16 or K % 64:
        raise ValueError("pack needs N % 16 == 0 and K % 64 == 0")
    if q.min(initial=0) < -8 or q.max(initial=0) > 7:
        raise ValueError("codes must lie in [-8, 7]")
    u = (q.astype(np.int16) + 8).astype(np.uint8)
    byte, nib = _layout_index(N, K)
    out = np.zeros(N * K // 2, dtype=np.uint8)
    lo = nib == 0
    out[byte[lo]] |= u[lo]
    out[byte[~lo]] |= (u[~lo] << 4).astype(np.uint8)
    return out


def unpack_w4(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    """Inverse of ``pack_w4``: uint8 [N*K/2] -> codes q (N x K int8)."""
    packed = np.asarray(packed, dtype=np.uint8).reshape(-1)
    if packed.size != N * K // 2:
        raise ValueError("packed size mismatch")
    byte, nib = _layout_index(N, K)
    v = packed[byte]
    u = np.where(nib == 0, v & 0xF, v >> 4)
    return (u.astype(np.int16) - 8).astype(np.int8)


# ----------------------------------------------------------------------------
# a-2 .. a-4: dequantise, gate, low-rank EC, combine
# ----------------------------------------------------------------------------

def dequantize(q: np.ndarray, s: np.ndarray, group: int = 0) -> np.ndarray:
    """Dense K x N float64 weight: W[k, n] = s[n] * q[n, k] (or s[k // 128, n] * q[n, k])."""
    qf = np.asarray(q, dtype=np.float64)            # N x K
    s64 = np.asarray(s, dtype=np.float16).astype(np.float64)
    if group == 0:
        return (qf * s64[:, None]).T
    N, K = qf.shape
    per_k = np.repeat(s64, 128, axis=0)[:K, :]        # K x N
    return qf.T * per_k


def gate(x_bits: np.ndarray, w_g_bits: np.ndarray, b_g: float) -> tuple[np.ndarray, np.ndarray]:
    """Per-token gate g_m = sigmoid(x_m . w_g + b_g); returns (g, logit) in float64.

    The per-token gate is the pages' input-dependent modulation of the EC
    (gist.science technical summary, section 2.1 A), here a scalar per token.
    """
    x = bf16_to_f64(x_bits)
    wg = bf16_to_f64(w_g_bits)
    logit = x @ wg + float(b_g)
    with np.errstate(over="ignore"):
        g = 1.0 / (1.0 + np.exp(-logit))
    return g, logit


def gate_mask_count(g: np.ndarray, tau: float = TAU_DEFAULT) -> int:
    """Number of tokens whose gate is below tau (tokens the EC barely corrects)."""
    return int(np.count_nonzero(np.asarray(g) < tau))


def linear(x_bits: np.ndarray, q: np.ndarray, s: np.ndarray, group: int,
           A_bits: np.ndarray | None, B_bits: np.ndarray | None,
           w_g_bits: np.ndarray | None, b_g: float) -> tuple[np.ndarray, np.ndarray | None]:
    """y = x . dequant(W4) + g * ((x . A) . B), all in float64.  Returns (y, g).

    With A, B or w_g None the EC is absent and y = x . dequant(W4), g = None.
    """
    x = bf16_to_f64(x_bits)
    Wd = dequantize(q, s, group)
    y = x @ Wd
    if A_bits is None or B_bits is None or w_g_bits is None:
        return y, None
    g, _ = gate(x_bits, w_g_bits, b_g)
    t = x @ bf16_to_f64(A_bits)
    y = y + g[:, None] * (t @ bf16_to_f64(B_bits))
    return y, g


def linear_bruteforce(x_bits, q, s, group, A_bits, B_bits, w_g_bits, b_g):
    """Element-by-element loops over the same definition (tiny inputs only)."""
    x = bf16_to_f64(x_bits)
    M, K = x.shape
    N = q.shape[0]
    s16 = np.asarray(s, dtype=np.float16)
    ec = A_bits is not None
    if ec:
        A = bf16_to_f64(A_bits)
        B = bf16_to_f64(B_bits)
        wg = bf16_to_f64(w_g_bits)
        r = A.shape[1]
    y = np.zeros((M, N))
    for m in range(M):
        if ec:
            lg = float(b_g)
            for k in range(K):
                lg += x[m, k] * wg[k]
            gm = 1.0 / (1.0 + math.exp(-lg)) if lg > -700 else 0.0
            t = [0.0] * r
            for j in range(r):
                for k in range(K):
                    t[j] += x[m, k] * A[k, j]
        for n in range(N):
            acc = 0.0
            for k in range(K):
                sc = float(s16[n]) if group == 0 else float(s16[k // 128, n])
                acc += x[m, k] * (sc * int(q[n, k]))
            if ec:
                e = 0.0
                for j in range(r):
                    e += t[j] * B[j, n]
                acc += gm * e
            y[m, n] = acc
    return y


# ----------------------------------------------------------------------------
# The pages' per-rank gate: gamma(t), a bottleneck MLP on t = x . A
# ----------------------------------------------------------------------------

def rank_gate(t: np.ndarray, W1: np.ndarray, b1: np.ndarray, W2: np.ndarray,
              b2: np.ndarray) -> np.ndarray:
    """gamma(t) = sigmoid(W2 . relu(W1 . t + b1) + b2), one row per token, float64.

    SPEAR, gist.science technical summary, section 2.1 A: the effective weight
    is W + alpha B diag(gamma(A x)) A with gamma "a bottleneck MLP" on the
    low-rank projection.  The pages name neither the layers nor the
    activation; this is the plainest reading: r -> h (ReLU) -> r (sigmoid, so
    every rank's gate lies in (0, 1) like the scalar gate).
    t: M x r; W1: h x r; b1: h; W2: r x h; b2: r (fp32 values, read exactly).
    """
    W1 = np.asarray(W1, dtype=np.float32).astype(np.float64)
    W2 = np.asarray(W2, dtype=np.float32).astype(np.float64)
    b1 = np.asarray(b1, dtype=np.float32).astype(np.float64)
    b2 = np.asarray(b2, dtype=np.float32).astype(np.float64)
    u = np.maximum(t @ W1.T + b1, 0.0)
    z = u @ W2.T + b2
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def linear_rank_gated(x_bits: np.ndarray, q: np.ndarray, s: np.ndarray, group: int,
                      A_bits: np.ndarray, B_bits: np.ndarray, W1: np.ndarray, b1: np.ndarray,
                      W2: np.ndarray, b2: np.ndarray, alpha: float
                      ) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """y = x . dequant(W4) + alpha * ((x . A) * gamma(x . A)) . B, float64.

    The row-vector form of W + alpha B diag(gamma(A x)) A (summary section
    2.1 A).  Returns (y, gamma, gate_mean) with gate_mean[m] the mean over the
    r ranks of gamma, the per-token gate this form reports (and compares with
    tau for the mask count).
    """
    x = bf16_to_f64(x_bits)
    y = x @ dequantize(q, s, group)
    t = x @ bf16_to_f64(A_bits)
    gam = rank_gate(t, W1, b1, W2, b2)
    y = y + float(alpha) * ((t * gam) @ bf16_to_f64(B_bits))
    return y, gam, gam.mean(axis=1)


def linear_rank_gated_bruteforce(x_bits, q, s, group, A_bits, B_bits, W1, b1, W2, b2, alpha):
    """Element-by-element loops over the same definition (tiny inputs only)."""
    x = bf16_to_f64(x_bits)
    A = bf16_to_f64(A_bits)
    B = bf16_to_f64(B_bits)
    W1 = np.asarray(W1, dtype=np.float32)
    W2 = np.asarray(W2, dtype=np.float32)
    b1 = np.asarray(b1, dtype=np.float32)
    b2 = np.asarray(b2, dtype=np.float32)
    s16 = np.asarray(s, dtype=np.float16)
    M, K = x.shape
    N = q.shape[0]
    r = A.shape[1]
    h = W1.shape[0]
    y = np.zeros((M, N))
    for m in range(M):
        t = [sum(x[m, k] * A[k, j] for k in range(K)) for j in range(r)]
        u = []
        for i in range(h):
            v = float(b1[i]) + sum(float(W1[i, j]) * t[j] for j in range(r))
            u.append(v if v > 0.0 else 0.0)
        gam = []
        for j in range(r):
            z = float(b2[j]) + sum(float(W2[j, i]) * u[i] for i in range(h))
            gam.append(1.0 / (1.0 + math.exp(-z)) if z > -700 else 0.0)
        for n in range(N):
            acc = 0.0
            for k in range(K):
                sc = float(s16[n]) if group == 0 else float(s16[k // 128, n])
                acc += x[m, k] * (sc * int(q[n, k]))
            e = 0.0
            for j in range(r):
                e += t[j] * gam[j] * B[j, n]
            y[m, n] = acc + float(alpha) * e
    return y


# ----------------------------------------------------------------------------
# EC operand preparation (what the library's EC pack step must produce)
# ----------------------------------------------------------------------------

def prescale_B(B_bits: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Fold the per-channel scale into B: B'[j, n] = bf16_rne(fp32(B[j, n] / s[n])).

    Lets a kernel accumulate x . q and (g t) . B' in one accumulator and apply
    s_n once at the end.  The quotient is the IEEE fp32 quotient of the two
    exact inputs, then rounded to bf16 ties-to-even (the library's precision
    for this step).
    """
    B32 = bf16_to_f64(B_bits).astype(np.float32)
    s32 = np.asarray(s, dtype=np.float16).astype(np.float32)
    return f32_to_bf16_bits_rne(B32 / s32[None, :])


def ec_pack(A_bits: np.ndarray, B_bits: np.ndarray, w_g_bits: np.ndarray,
            s: np.ndarray, group: int) -> tuple[np.ndarray, np.ndarray]:
    """EC operands in the library's layout.

    Returns (AgT, BpT): AgT is (r+1) x K bf16 = [A^T ; w_g] (the gate weight as
    one extra projection row), BpT is N x r bf16 = (B')^T with the per-channel
    fold B' = prescale_B(B, s) for group 0, or B^T unchanged for group 128.
    """
    AgT = np.concatenate([np.asarray(A_bits, dtype=np.uint16).T,
                          np.asarray(w_g_bits, dtype=np.uint16)[None, :]], axis=0)
    if group == 0:
        BpT = prescale_B(B_bits, s).T
    else:
        BpT = np.asarray(B_bits, dtype=np.uint16).T
    return np.ascontiguousarray(AgT), np.ascontiguousarray(BpT)
