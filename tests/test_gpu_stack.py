"""Config-4 stack: the W4 linears at the stack's shapes (M = 256) against the
oracle, teacher-forced, and two decoder layers of the glue pipeline through the
library against the same pipeline in float64 on the oracle."""
import os
import sys

import numpy as np
import pytest
import torch

from oracle import spear_oracle as O
from w4_gemm_gated_b200 import synth

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402  (the stack glue lives in the benchmark harness)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4_gemm_gated_b200 import build
    build.build()
    from w4_gemm_gated_b200 import spear
    return spear


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _f64(t):
    return O.bf16_to_f64(t.cpu().view(torch.int16).numpy().view(np.uint16))


@pytest.mark.parametrize("proj", [0, 4, 6])  # q (4096x4096), gate (4096->11008), down (11008->4096)
@pytest.mark.parametrize("ec", [False, True])
def test_stack_linear_teacher_forced(S, proj, ec):
    K, N = bench.STACK_SHAPES[proj]
    L = synth.make_layer(256, K, N, 64 if ec else 0, b_g=-1.0, x_kind="normal",
                         seed=synth.stack_layer_seed(0, 0 if ec else 5, proj))
    layer = S.prepare_layer(torch.from_numpy(L.W).cuda(), 0, _bf16(L.A) if ec else None,
                            _bf16(L.B) if ec else None, _bf16(L.w_g) if ec else None, L.b_g)
    ws = S.make_workspace(layer, 256)
    y = S.forward(layer, _bf16(L.x), ws)
    torch.cuda.synchronize()
    assert S.read_status(ws) == S.OK
    q, s = O.quantize_rtn(L.W, 0)
    y_o, _ = O.linear(L.x, q, s, 0, L.A, L.B, L.w_g, L.b_g)
    assert np.max(np.abs(_f64(y) - y_o)) <= 1e-2 * np.max(np.abs(y_o))


def _oracle_stack(x, mats, eps=1e-6):
    """The glue of bench.stack_glue in float64 with the oracle's linear, rounding
    activations to bf16 where the library's pipeline does."""
    def bf(v):
        return O.bf16_to_f64(O.f32_to_bf16_bits_rne(v.astype(np.float32)))

    def rms(v):
        return bf(v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps))

    def lin(h, m):
        q, s, A, B, w_g, b_g = m
        hb = O.f32_to_bf16_bits_rne(h.astype(np.float32))
        y, _ = O.linear(hb, q, s, 0, A, B, w_g, b_g)
        return bf(y)

    for layer in mats:
        mq, mk, mv, mo, mg, mu, md = layer
        h = rms(x)
        v = lin(h, mv)
        x = bf(x + lin(v, mo))
        h2 = rms(x)
        g = lin(h2, mg)
        u = lin(h2, mu)
        x = bf(x + lin(bf(g / (1.0 + np.exp(-g)) * u), md))
    return x


def test_two_layer_pipeline_against_oracle(S):
    M = 8
    mats, layers = [], []
    for l, with_ec in ((0, True), (1, False)):
        row_m, row_l = [], []
        for proj, (K, N) in enumerate(bench.STACK_SHAPES):
            L = synth.make_layer(M, K, N, 64 if with_ec else 0, b_g=-1.0, seed=synth.stack_layer_seed(3, l, proj))
            q, s = O.quantize_rtn(L.W, 0)
            row_m.append((q, s, L.A, L.B, L.w_g, L.b_g))
            row_l.append(S.prepare_layer(torch.from_numpy(L.W).cuda(), 0, _bf16(L.A) if with_ec else None,
                                         _bf16(L.B) if with_ec else None, _bf16(L.w_g) if with_ec else None,
                                         L.b_g))
        mats.append(row_m)
        layers.append(row_l)
    x_bits = synth.make_layer(M, 4096, 16, 0, seed=11).x
    ws = torch.zeros(max(S.workspace_bytes(lay, M) for row in layers for lay in row), dtype=torch.uint8,
                     device="cuda")
    out = bench.stack_glue(S, layers, _bf16(x_bits), ws, n_layers=2)
    torch.cuda.synchronize()
    assert S.read_status(ws) == S.OK
    ref = _oracle_stack(O.bf16_to_f64(x_bits), mats)
    got = _f64(out)
    assert np.all(np.isfinite(got))
    # the oracle pipeline rounds to bf16 at the same points as the device glue,
    # so the per-linear bound holds across the 14 linears as well
    assert np.max(np.abs(got - ref)) <= 1e-2 * np.max(np.abs(ref))
