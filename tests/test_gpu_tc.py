"""GPU parity of the tensor-core (tcgen05) paths against the CPU oracle:
the fused kernel (EC inside the GEMM) and the unfused pair (EC-disabled GEMM,
then the standalone EC kernel), including ragged token counts, every EC rank,
group-wise scales, the model shapes of the dispatch sweep and the full
prefill workload."""
import math

import numpy as np
import pytest
import torch

from oracle import spear_oracle as O
from tests.test_gpu_parity import (GATE_TOL, assert_close, dev_bf16, host_bits, oracle_ref, prepared, run)
from w4_gemm_gated_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4_gemm_gated_b200 import build
    build.build()
    from w4_gemm_gated_b200 import spear
    return spear


def test_fused_tiny_config(S):
    L = synth.tiny()
    layer = prepared(S, L, 0)
    y, g, cnt, _ = run(S, layer, L.x, S.PATH_FUSED, gate=True)
    y_ref, g_ref, _, _ = oracle_ref(L, 0)
    assert_close(y, y_ref)
    assert np.max(np.abs(g.cpu().numpy() - g_ref)) <= GATE_TOL
    assert int(cnt.item()) == O.gate_mask_count(g_ref)


@pytest.mark.parametrize("M", [17, 100, 128, 129, 300])
def test_fused_ragged_tokens(S, M):
    L = synth.make_layer(M, 1024, 1024, 64, b_g=-0.5, x_kind="t3", seed=100 + M)
    layer = prepared(S, L, 0)
    y, g, _, _ = run(S, layer, L.x, S.PATH_FUSED, gate=True)
    y_ref, g_ref, _, _ = oracle_ref(L, 0)
    assert_close(y, y_ref)
    assert np.max(np.abs(g.cpu().numpy() - g_ref)) <= GATE_TOL


@pytest.mark.parametrize("r", [16, 32, 64, 128])
def test_fused_every_rank(S, r):
    L = synth.make_layer(200, 2048, 1024, r, b_g=0.2, seed=200 + r)
    layer = prepared(S, L, 0)
    y, _, _, _ = run(S, layer, L.x, S.PATH_FUSED)
    assert_close(y, oracle_ref(L, 0)[0])


@pytest.mark.parametrize("group", [0, 128])
def test_fused_and_unfused_group_scales(S, group):
    L = synth.make_layer(256, 4096, 1024, 64, b_g=-1.0, x_kind="t3", seed=300)
    layer = prepared(S, L, group)
    y_ref, g_ref, _, _ = oracle_ref(L, group)
    for path in (S.PATH_FUSED, S.PATH_UNFUSED):
        y, g, _, _ = run(S, layer, L.x, path, gate=True)
        assert_close(y, y_ref)
        assert np.max(np.abs(g.cpu().numpy() - g_ref)) <= GATE_TOL


@pytest.mark.parametrize("shape", [(4096, 4096), (4096, 14336), (14336, 4096)])
@pytest.mark.parametrize("M", [32, 512])
def test_sweep_shapes_fused_vs_oracle(S, shape, M):
    K, N = shape
    L = synth.sweep_point(M, K, N, 32, seed=7)
    layer = prepared(S, L, 0)
    y, _, _, _ = run(S, layer, L.x, S.PATH_FUSED)
    assert_close(y, oracle_ref(L, 0)[0])


def test_gate_off_equals_ec_disabled_tc(S):
    L = synth.make_layer(300, 2048, 2048, 64, b_g=0.5, seed=400)
    W = torch.from_numpy(L.W).cuda()
    plain = S.prepare_layer(W, 0, None, None, None, 0.0)
    y0, _, cnt0, _ = run(S, plain, L.x, S.PATH_FUSED, gate=True)
    assert int(cnt0.item()) == 300
    y1, g1, _, _ = run(S, prepared(S, L, 0, b_g=-math.inf), L.x, S.PATH_FUSED, gate=True)
    assert torch.equal(y1.float(), y0.float())
    assert torch.all(g1 == 0)
    assert_close(y0, O.linear(L.x, *O.quantize_rtn(L.W, 0), 0, None, None, None, 0.0)[0])


def test_decode_and_fused_agree_at_m16(S):
    L = synth.decode(16, force_outlier=True)
    L2 = synth.make_layer(16, 4096, 11008 - 11008 % 256, 64, b_g=-1.0, x_kind="outlier", seed=0,
                          force_outlier=True)
    layer = prepared(S, L2, 0)
    yd, _, _, _ = run(S, layer, L2.x, S.PATH_DECODE)
    yf, _, _, _ = run(S, layer, L2.x, S.PATH_FUSED)
    y_ref = oracle_ref(L2, 0)[0]
    assert_close(yd, y_ref)
    assert_close(yf, y_ref)
    del L


def test_prefill_config_full(S):
    # M=2048, K=N=4096, r=64, Student-t(3) channels, b_g=-1: every output element
    L = synth.prefill()
    layer = prepared(S, L, 0)
    y, g, cnt, _ = run(S, layer, L.x, S.PATH_FUSED, gate=True)
    y_ref, g_ref, _, _ = oracle_ref(L, 0)
    assert_close(y, y_ref)
    assert np.max(np.abs(g.cpu().numpy() - g_ref)) <= GATE_TOL
    yu, _, _, _ = run(S, layer, L.x, S.PATH_UNFUSED)
    assert_close(yu, y_ref)


def test_fused_is_deterministic(S):
    L = synth.make_layer(384, 2048, 2048, 64, seed=500)
    layer = prepared(S, L, 0)
    x = dev_bf16(L.x)
    ws = S.make_workspace(layer, 384)
    ys = [S.forward(layer, x, ws, path=S.PATH_FUSED).clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0].view(torch.int16), t.view(torch.int16)) for t in ys[1:])
    assert S.read_status(ws) == S.OK


def test_one_workspace_across_paths_and_sizes(S):
    # the same workspace serves every path and size in any order (its flags are
    # epoch-tagged per launch, so no call can see another call's state)
    L = synth.make_layer(640, 2048, 1024, 64, b_g=-0.3, seed=600)
    layer = prepared(S, L, 0)
    ws = S.make_workspace(layer, 640)
    q, s = O.quantize_rtn(L.W, 0)
    plain = S.Layer(layer.K, layer.N, 0, 0, layer.w_packed, layer.scales, None, None, 0.0)
    order = [(128, S.PATH_FUSED), (128, S.PATH_UNFUSED), (16, S.PATH_DECODE), (512, S.PATH_FUSED),
             (640, S.PATH_UNFUSED), (300, S.PATH_FUSED), (5, S.PATH_UNFUSED), (640, S.PATH_FUSED),
             (40, S.PATH_UNFUSED), (600, S.PATH_UNFUSED), (16, S.PATH_UNFUSED), (256, S.PATH_UNFUSED)]
    for it, (M, path) in enumerate(order):
        x = L.x[:M]
        if it % 3 == 2:
            # an EC-disabled layer on the same workspace in between
            S.forward(plain, dev_bf16(x), ws, path=S.PATH_FUSED)
        y = S.forward(layer, dev_bf16(x), ws, path=path)
        torch.cuda.synchronize()
        assert S.read_status(ws) == S.OK, (M, path)
        assert_close(y, O.linear(x, q, s, 0, L.A, L.B, L.w_g, L.b_g)[0])


@pytest.mark.parametrize("M,group,r", [(512, 0, 64), (600, 128, 32), (1000, 0, 128), (1300, 128, 16)])
def test_tall_tiles_ragged(S, M, group, r):
    """From M = 512 the kernel uses 256-token tiles (two accumulators); ragged
    M leaves a partial last block."""
    L = synth.make_layer(M, 2048, 1024, r, b_g=-0.3, x_kind="t3", seed=700 + M)
    layer = prepared(S, L, group)
    y_ref, g_ref, _, _ = oracle_ref(L, group)
    for path in (S.PATH_FUSED, S.PATH_UNFUSED):
        y, g, cnt, _ = run(S, layer, L.x, path, gate=True)
        assert_close(y, y_ref)
        assert np.max(np.abs(g.cpu().numpy() - g_ref)) <= GATE_TOL
