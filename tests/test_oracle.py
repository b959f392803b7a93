"""Pins of the CPU oracle against things other than itself.

Each test checks the oracle against a hand-worked fixture, a closed form, an
invariant of the layer definition, a library routine, or a brute-force loop,
chosen so that a plausible slip (transposed W / A / B, wrong nibble, wrong
rounding, dropped gate or EC term) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import expit

from oracle import spear_oracle as O
from w4_gemm_gated_b200 import synth


def _read_rows(path):
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


# --------------------------------------------------------------------------
# quantiser
# --------------------------------------------------------------------------

def test_rtn_hand_worked_cases(golden_dir):
    for row in _read_rows(os.path.join(golden_dir, "rtn_quantizer_cases.txt")):
        name, ws, sbits, codes = [p.strip() for p in row.split("|")]
        w = np.array([float(v) for v in ws.split()], dtype=np.float32)
        q, s = O.quantize_rtn(w[:, None], group=0)
        assert int(s.view(np.uint16)[0]) == int(sbits, 16), name
        assert q[0].tolist() == [int(c) for c in codes.split()], name


def test_rtn_group128_uses_its_own_block():
    # group 0 holds max 0.7 (scale 0x2E66), group 1 max 1.4 (scale 0x3266)
    w = np.zeros((256, 1), dtype=np.float32)
    w[5, 0] = 0.7
    w[130, 0] = -1.4
    w[131, 0] = 0.2
    q, s = O.quantize_rtn(w, group=128)
    assert s.shape == (2, 1)
    assert s.view(np.uint16)[:, 0].tolist() == [0x2E66, 0x3266]
    assert q[0, 5] == 7 and q[0, 130] == -7 and q[0, 131] == 1
    assert np.count_nonzero(q) == 3


def test_rtn_is_identity_on_grid():
    # weights already on the int4 grid quantise back to exactly their codes
    rng = np.random.default_rng(3)
    N, K = 32, 128
    q0 = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    q0[:, 0] = 7                                    # max |q| = 7 in every channel
    s0 = (rng.random(N) * 0.1 + 0.01).astype(np.float16)
    W = (q0.astype(np.float32) * s0.astype(np.float32)[:, None]).T   # K x N, exact in fp32
    q, s = O.quantize_rtn(W, group=0)
    assert np.array_equal(s.view(np.uint16), s0.view(np.uint16))
    assert np.array_equal(q, q0)


def test_rtn_codes_bounded_and_error_within_half_step():
    L = synth.make_layer(1, 256, 64, 0, seed=5)
    q, s = O.quantize_rtn(L.W, group=0)
    assert q.min() >= -7 and q.max() <= 7
    err = np.abs(L.W.astype(np.float64) - q.T * s.astype(np.float64)[None, :])
    # rounding error at most half a step (plus the fp32 quotient's rounding)
    assert np.all(err <= 0.5 * s.astype(np.float64)[None, :] * (1 + 1e-6))


# --------------------------------------------------------------------------
# packed layout
# --------------------------------------------------------------------------

def test_layout_hand_worked_addresses(golden_dir):
    N, K = 32, 128
    for row in _read_rows(os.path.join(golden_dir, "w4_layout_addresses.txt")):
        n, k, byte, nib = (int(v) for v in row.split())
        assert O.w4_nibble_address(n, k, K) == (byte, nib), (n, k)
        q = np.zeros((N, K), dtype=np.int8)
        q[n, k] = 7                                 # u = 15, everything else u = 8
        packed = O.pack_w4(q)
        expect = np.full(N * K // 2, 0x88, dtype=np.uint8)
        expect[byte] = 0x8F if nib == 0 else 0xF8
        assert np.array_equal(packed, expect), (n, k)


def test_pack_unpack_roundtrip_all_codes():
    rng = np.random.default_rng(11)
    for N, K in [(16, 64), (48, 192), (128, 512)]:
        q = rng.integers(-8, 8, size=(N, K)).astype(np.int8)
        p = O.pack_w4(q)
        assert p.dtype == np.uint8 and p.size == N * K // 2
        assert np.array_equal(O.unpack_w4(p, N, K), q)
    # every byte value is reachable: the map is a bijection on bytes
    q = rng.integers(-8, 8, size=(64, 256)).astype(np.int8)
    p = O.pack_w4(q)
    assert np.array_equal(O.pack_w4(O.unpack_w4(p, 64, 256)), p)


def test_layout_tiles_are_contiguous_512_bytes():
    # all codes of tile (p, t) land in bytes [(p*K/64+t)*512, +512)
    N, K = 32, 128
    for p in range(N // 16):
        for t in range(K // 64):
            base = (p * (K // 64) + t) * 512
            for n in range(16 * p, 16 * p + 16):
                for k in range(64 * t, 64 * t + 64, 7):
                    b, _ = O.w4_nibble_address(n, k, K)
                    assert base <= b < base + 512


# --------------------------------------------------------------------------
# the layer
# --------------------------------------------------------------------------

def _small_layer(group, seed=0, M=3, K=128, N=16, r=2, b_g=0.25):
    L = synth.make_layer(M, K, N, r, b_g=b_g, seed=seed)
    q, s = O.quantize_rtn(L.W, group=group)
    return L, q, s


@pytest.mark.parametrize("group", [0, 128])
def test_linear_matches_bruteforce(group):
    L, q, s = _small_layer(group)
    y, g = O.linear(L.x, q, s, group, L.A, L.B, L.w_g, L.b_g)
    yb = O.linear_bruteforce(L.x, q, s, group, L.A, L.B, L.w_g, L.b_g)
    assert np.allclose(y, yb, rtol=1e-12, atol=1e-12)


def test_linear_matches_bruteforce_several_scale_groups():
    # K = 384 with group 128: three scale groups per channel, each from its own
    # block of 128 k, so a dequantiser that used one group's scale for another
    # (or the per-channel layout) disagrees with the loop
    L, q, s = _small_layer(128, seed=11, M=3, K=384, N=16, r=3, b_g=-0.5)
    assert s.shape == (3, 16)
    assert not np.array_equal(s[0], s[1]) and not np.array_equal(s[1], s[2])
    y, g = O.linear(L.x, q, s, 128, L.A, L.B, L.w_g, L.b_g)
    yb = O.linear_bruteforce(L.x, q, s, 128, L.A, L.B, L.w_g, L.b_g)
    assert np.allclose(y, yb, rtol=1e-12, atol=1e-12)


def test_one_hot_token_closed_form_several_scale_groups():
    # x = e_k with k in the second and third scale groups: y[n] picks the scale
    # of k's own group, s[k // 128, n]
    L, q, s = _small_layer(128, seed=12, M=1, K=384, N=16, r=2)
    A = O.bf16_to_f64(L.A)
    B = O.bf16_to_f64(L.B)
    wg = O.bf16_to_f64(L.w_g)
    s64 = s.astype(np.float64)
    for k in [128, 200, 255, 256, 383]:
        x = np.zeros((1, L.K), dtype=np.uint16)
        x[0, k] = 0x3F80                            # bf16 1.0
        y, g = O.linear(x, q, s, 128, L.A, L.B, L.w_g, L.b_g)
        gk = 1.0 / (1.0 + math.exp(-(wg[k] + L.b_g)))
        for n in range(L.N):
            ec = sum(A[k, j] * B[j, n] for j in range(L.r))
            assert y[0, n] == pytest.approx(s64[k // 128, n] * q[n, k] + gk * ec, rel=1e-13, abs=1e-15)


@pytest.mark.parametrize("group", [0, 128])
def test_one_hot_token_closed_form(group):
    # x = e_k: y[n] = s(k, n) * q[n, k] + sigmoid(w_g[k] + b_g) * sum_j A[k, j] B[j, n]
    L, q, s = _small_layer(group, seed=1, r=3)
    K, N = L.K, L.N
    A = O.bf16_to_f64(L.A)
    B = O.bf16_to_f64(L.B)
    wg = O.bf16_to_f64(L.w_g)
    s64 = s.astype(np.float64)
    for k in [0, 1, 77, 127]:
        x = np.zeros((1, K), dtype=np.uint16)
        x[0, k] = 0x3F80                            # bf16 1.0
        y, g = O.linear(x, q, s, group, L.A, L.B, L.w_g, L.b_g)
        gk = 1.0 / (1.0 + math.exp(-(wg[k] + L.b_g)))
        assert g[0] == pytest.approx(gk, rel=1e-15)
        for n in range(N):
            sc = s64[n] if group == 0 else s64[k // 128, n]
            ec = sum(A[k, j] * B[j, n] for j in range(L.r))
            assert y[0, n] == pytest.approx(sc * q[n, k] + gk * ec, rel=1e-13, abs=1e-15)


def test_all_ones_token_gives_scaled_column_sums():
    L, q, s = _small_layer(0, seed=2)
    x = np.full((1, L.K), 0x3F80, dtype=np.uint16)
    y, _ = O.linear(x, q, s, 0, None, None, None, 0.0)
    expect = s.astype(np.float64) * q.astype(np.int64).sum(axis=1)
    assert np.allclose(y[0], expect, rtol=1e-14)


def test_gate_off_gives_plain_w4_gemm():
    L, q, s = _small_layer(0, seed=4)
    y0, _ = O.linear(L.x, q, s, 0, None, None, None, 0.0)
    y_inf, g = O.linear(L.x, q, s, 0, L.A, L.B, L.w_g, -math.inf)
    assert np.all(g == 0.0)
    assert np.array_equal(y_inf, y0)


def test_zero_A_or_B_gives_plain_w4_gemm():
    L, q, s = _small_layer(0, seed=6)
    y0, _ = O.linear(L.x, q, s, 0, None, None, None, 0.0)
    zA = np.zeros_like(L.A)
    zB = np.zeros_like(L.B)
    yA, _ = O.linear(L.x, q, s, 0, zA, L.B, L.w_g, L.b_g)
    yB, _ = O.linear(L.x, q, s, 0, L.A, zB, L.w_g, L.b_g)
    assert np.array_equal(yA, y0) and np.array_equal(yB, y0)


def test_on_grid_weights_equal_dense_gemm():
    # W = s * q exactly: the W4 path equals a plain float64 GEMM with W
    rng = np.random.default_rng(8)
    M, N, K = 4, 32, 128
    q0 = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    q0[:, 3] = -7
    s0 = (rng.random(N) * 0.05 + 0.005).astype(np.float16)
    W = (q0.astype(np.float32) * s0.astype(np.float32)[:, None]).T
    q, s = O.quantize_rtn(W, 0)
    x = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    y, _ = O.linear(x, q, s, 0, None, None, None, 0.0)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    ref = xf @ W.astype(np.float64)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_ec_term_is_gated_per_token():
    # scaling b_g changes only the EC part, token by token, by the ratio of gates
    L, q, s = _small_layer(0, seed=9, M=5)
    y0, _ = O.linear(L.x, q, s, 0, None, None, None, 0.0)
    y1, g1 = O.linear(L.x, q, s, 0, L.A, L.B, L.w_g, 0.0)
    y2, g2 = O.linear(L.x, q, s, 0, L.A, L.B, L.w_g, 1.5)
    e1, e2 = y1 - y0, y2 - y0
    for m in range(L.M):
        assert np.allclose(e2[m] * g1[m], e1[m] * g2[m], rtol=1e-10, atol=1e-15)


def test_gate_is_logistic_function():
    rng = np.random.default_rng(12)
    K = 64
    x = synth.f32_to_bf16_bits(rng.standard_normal((50, K)).astype(np.float32))
    wg = synth.f32_to_bf16_bits((rng.standard_normal(K) * 0.3).astype(np.float32))
    g, logit = O.gate(x, wg, -0.7)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    wf = synth.bf16_bits_to_f32(wg).astype(np.float64)
    assert np.allclose(logit, xf @ wf - 0.7, rtol=1e-13)
    assert np.allclose(g, expit(logit), rtol=1e-14)
    z = np.zeros((1, K), dtype=np.uint16)
    g0, _ = O.gate(z, wg, 0.0)
    assert g0[0] == 0.5


def test_gate_mask_count_threshold():
    g = np.array([0.0, 0.05, 0.0999999, 0.1, 0.2, 1.0])
    assert O.gate_mask_count(g, 0.1) == 3
    assert O.gate_mask_count(g, 0.0) == 0


# --------------------------------------------------------------------------
# EC operand preparation
# --------------------------------------------------------------------------

def test_fold_hand_worked_cases(golden_dir):
    for row in _read_rows(os.path.join(golden_dir, "ec_fold_cases.txt")):
        b, sb, out = (int(v.strip(), 16) for v in row.split("|"))
        B = np.array([[b]], dtype=np.uint16)
        s = np.array([sb], dtype=np.uint16).view(np.float16)
        assert int(O.prescale_B(B, s)[0, 0]) == out, row


def test_bf16_rounding_ties_to_even():
    v = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 1.0 + 2.0 ** -8 + 2.0 ** -20],
                 dtype=np.float32)
    # exact ties go to the even neighbour, anything above a tie goes up
    assert O.f32_to_bf16_bits_rne(v).tolist() == [0x3F80, 0x3F82, 0xBF80, 0x3F81]


def test_ec_pack_layout():
    L, q, s = _small_layer(0, seed=10, r=4)
    AgT, BpT = O.ec_pack(L.A, L.B, L.w_g, s, 0)
    assert AgT.shape == (L.r + 1, L.K) and BpT.shape == (L.N, L.r)
    assert np.array_equal(AgT[:L.r], L.A.T) and np.array_equal(AgT[L.r], L.w_g)
    # the fold undoes the channel scale: B'[j, n] * s[n] ~ B[j, n] within bf16 rounding
    Bp = O.bf16_to_f64(BpT.T) * s.astype(np.float64)[None, :]
    assert np.allclose(Bp, O.bf16_to_f64(L.B), rtol=2 ** -8)
    _, BpT_g = O.ec_pack(L.A, L.B, L.w_g, s, 128)
    assert np.array_equal(BpT_g, L.B.T)


def test_fold_reproduces_layer_within_bf16():
    # y computed with the folded B' and a final scale equals the oracle within bf16 error
    L, q, s = _small_layer(0, seed=13, M=4, K=256, N=32, r=8)
    y, g = O.linear(L.x, q, s, 0, L.A, L.B, L.w_g, L.b_g)
    _, BpT = O.ec_pack(L.A, L.B, L.w_g, s, 0)
    x = O.bf16_to_f64(L.x)
    t = x @ O.bf16_to_f64(L.A)
    acc = x @ q.T.astype(np.float64) + (g[:, None] * t) @ O.bf16_to_f64(BpT.T)
    y2 = acc * s.astype(np.float64)[None, :]
    assert np.max(np.abs(y2 - y)) <= 1e-2 * np.max(np.abs(y))


def test_synthetic_configs_shapes_and_gate_fraction():
    L = synth.tiny()
    assert (L.M, L.K, L.N, L.r, L.b_g) == (16, 512, 512, 16, 0.0)
    D = synth.decode(16, force_outlier=True)
    assert len(D.meta["outlier_tokens"]) >= 1
    assert len(D.meta["outlier_channels"]) == 41
    g, _ = O.gate(D.x, D.w_g, D.b_g)
    assert g.shape == (16,) and np.all((g > 0) & (g < 1))


# --------------------------------------------------------------------------
# the pages' per-rank gate gamma(t) (bottleneck MLP on t = x . A)
# --------------------------------------------------------------------------

def _bits(v):
    return O.f32_to_bf16_bits_rne(np.asarray(v, dtype=np.float32))


def test_rank_gate_hand_worked():
    # q = 0 (no W term), x = e_0, A row 0 = (1, 2): t = (1, 2).  h = 1:
    # W1 . t + b1 = 0.5 - 2 + 2 = 0.5 -> relu 0.5; W2 . u + b2 = (1, -2);
    # gamma = (sigmoid(1), sigmoid(-2)); B = (1, 1)^T, alpha = 0.5:
    # y = 0.5 * (1 * sigmoid(1) + 2 * sigmoid(-2)).
    K, N, r = 64, 1, 2
    x = np.zeros((1, K), np.float32); x[0, 0] = 1.0
    A = np.zeros((K, r), np.float32); A[0] = (1.0, 2.0)
    B = np.ones((r, N), np.float32)
    q = np.zeros((N, K), np.int8)
    s = np.ones(N, np.float16)
    W1 = np.array([[0.5, -1.0]], np.float32); b1 = np.array([2.0], np.float32)
    W2 = np.array([[2.0], [-4.0]], np.float32); b2 = np.zeros(2, np.float32)
    y, gam, gm = O.linear_rank_gated(_bits(x), q, s, 0, _bits(A), _bits(B), W1, b1, W2, b2, 0.5)
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    assert y[0, 0] == pytest.approx(0.5 * (sig(1.0) + 2.0 * sig(-2.0)), rel=1e-15)
    assert gam[0] == pytest.approx([sig(1.0), sig(-2.0)], rel=1e-15)
    assert gm[0] == pytest.approx(0.5 * (sig(1.0) + sig(-2.0)), rel=1e-15)


def _rank_case(seed, M=3, K=128, N=16, r=16, h=8, group=0):
    rng = np.random.default_rng(seed)
    x = _bits(rng.standard_normal((M, K)))
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    q, s = O.quantize_rtn(W, group)
    A = _bits(rng.standard_normal((K, r)) * 0.05)
    B = _bits(rng.standard_normal((r, N)) * 0.05)
    W1 = (rng.standard_normal((h, r)) * 0.5).astype(np.float32)
    b1 = (rng.standard_normal(h) * 0.1).astype(np.float32)
    W2 = (rng.standard_normal((r, h)) * 0.5).astype(np.float32)
    b2 = (rng.standard_normal(r) * 0.5).astype(np.float32)
    return x, q, s, A, B, W1, b1, W2, b2


@pytest.mark.parametrize("group", [0, 128])
def test_rank_gated_matches_bruteforce(group):
    x, q, s, A, B, W1, b1, W2, b2 = _rank_case(11 + group, K=256, group=group)
    y, _, _ = O.linear_rank_gated(x, q, s, group, A, B, W1, b1, W2, b2, 0.75)
    yb = O.linear_rank_gated_bruteforce(x, q, s, group, A, B, W1, b1, W2, b2, 0.75)
    assert np.max(np.abs(y - yb)) <= 1e-12 * max(1.0, np.max(np.abs(yb)))


def test_rank_gate_constant_reduces_to_scalar_gate():
    # W1 = W2 = 0 and b2 = c on every rank: gamma = sigmoid(c) everywhere, which
    # is the scalar gate with w_g = 0 and b_g = c (alpha = 1)
    x, q, s, A, B, W1, b1, W2, b2 = _rank_case(21)
    r, h = W2.shape
    c = -0.7
    y, gam, gm = O.linear_rank_gated(x, q, s, 0, A, B, np.zeros_like(W1), b1, np.zeros_like(W2),
                                     np.full(r, c, np.float32), 1.0)
    wg = _bits(np.zeros(x.shape[1]))
    ys, g = O.linear(x, q, s, 0, A, B, wg, float(np.float32(c)))
    assert np.allclose(y, ys, rtol=1e-13, atol=1e-15)
    assert np.allclose(gm, g, rtol=1e-15)


def test_rank_gate_off_gives_pure_w4_gemm():
    x, q, s, A, B, W1, b1, W2, b2 = _rank_case(31)
    y0, _ = O.linear(x, q, s, 0, None, None, None, 0.0)
    ya, _, _ = O.linear_rank_gated(x, q, s, 0, A, B, W1, b1, W2, b2, 0.0)        # alpha = 0
    yb, gam, _ = O.linear_rank_gated(x, q, s, 0, A, B, W1, b1, W2,
                                     np.full(W2.shape[0], -1000.0, np.float32), 1.0)  # gamma -> 0
    assert np.array_equal(ya, y0)
    assert np.max(gam) < 1e-300
    assert np.allclose(yb, y0, rtol=0, atol=1e-250)


def test_rank_gate_relu_cuts_w1():
    # b1 far below zero: relu gives u = 0 whatever W1 is, so gamma = sigmoid(b2)
    x, q, s, A, B, W1, b1, W2, b2 = _rank_case(41)
    t = O.bf16_to_f64(x) @ O.bf16_to_f64(A)
    g1 = O.rank_gate(t, W1, np.full_like(b1, -1e6), W2, b2)
    g2 = O.rank_gate(t, 3.0 * W1 + 1.0, np.full_like(b1, -1e6), W2, b2)
    assert np.array_equal(g1, g2)
    assert np.allclose(g1, expit(b2.astype(np.float64))[None, :], rtol=1e-15)
