"""GPU parity of the semi-fused prefill path: the EC projection on a second
stream beside the EC-disabled GEMM, then the in-place EC update (SPEAR,
gist.science technical summary, section 2.2 A).  Checked against the CPU
oracle, bit for bit against the unfused path (the same EC launches after the
GEMM instead of beside it), and under CUDA-graph capture of the two-branch
DAG."""
import numpy as np
import pytest
import torch

from oracle import spear_oracle as O
from tests.test_gpu_parity import GATE_TOL, assert_close, dev_bf16, host_bits, oracle_ref, prepared, run
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


@pytest.mark.parametrize("M,r,group", [(1, 64, 0), (16, 32, 128), (17, 16, 0), (300, 64, 128), (1000, 128, 0)])
def test_semifused_vs_oracle(S, M, r, group):
    L = synth.make_layer(M, 2048, 1024, r, b_g=-0.5, x_kind="t3", seed=900 + M + r)
    layer = prepared(S, L, group)
    y, g, cnt, _ = run(S, layer, L.x, S.PATH_SEMIFUSED, gate=True)
    y_ref, g_ref, _, _ = oracle_ref(L, group)
    assert_close(y, y_ref)
    assert np.max(np.abs(g.cpu().numpy() - g_ref)) <= GATE_TOL
    # the mask count is an integer decided in fp32 on both sides: exact unless
    # a gate sits within rounding of tau
    near = np.abs(g_ref - O.TAU_DEFAULT) <= GATE_TOL
    assert int(cnt.item()) == int(np.sum(g.cpu().numpy() < np.float32(O.TAU_DEFAULT)))
    assert abs(int(cnt.item()) - O.gate_mask_count(g_ref)) <= int(near.sum())


@pytest.mark.parametrize("group", [0, 128])
def test_semifused_bitwise_equals_unfused(S, group):
    L = synth.make_layer(257, 4096, 2048, 64, b_g=0.3, x_kind="t3", seed=950)
    layer = prepared(S, L, group)
    y1, g1, c1, _ = run(S, layer, L.x, S.PATH_UNFUSED, gate=True)
    y2, g2, c2, _ = run(S, layer, L.x, S.PATH_SEMIFUSED, gate=True)
    assert np.array_equal(host_bits(y1), host_bits(y2))
    assert torch.equal(g1, g2)
    assert int(c1.item()) == int(c2.item())


def test_semifused_graph_capture_replays(S):
    """Capturing the caller's stream captures the fork / join: the replayed
    graph recomputes the layer for new inputs written into the same buffers."""
    M, K, N, r = 384, 2048, 2048, 64
    L1 = synth.make_layer(M, K, N, r, b_g=0.0, seed=960)
    L2 = synth.make_layer(M, K, N, r, b_g=0.0, seed=961)
    L2.W, L2.A, L2.B, L2.w_g = L1.W, L1.A, L1.B, L1.w_g   # same layer, new tokens
    layer = prepared(S, L1, 0)
    x = dev_bf16(L1.x)
    ws = S.make_workspace(layer, M)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(M, dtype=torch.float32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        S.forward(layer, x, ws, y=y, gate_out=g, mask_count=cnt, path=S.PATH_SEMIFUSED, stream=s)  # warm-up
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        S.forward(layer, x, ws, y=y, gate_out=g, mask_count=cnt, path=S.PATH_SEMIFUSED, stream=s)
    for Li in (L2, L1, L2):
        x.copy_(dev_bf16(Li.x))
        y.zero_()
        graph.replay()
        torch.cuda.synchronize()
        y_ref, g_ref, _, _ = oracle_ref(Li, 0)
        assert_close(y, y_ref)
        assert np.max(np.abs(g.cpu().numpy() - g_ref)) <= GATE_TOL
    assert S.read_status(ws) == S.OK
    del graph


def test_semifused_ec_off_layer_is_plain_gemm(S):
    L = synth.make_layer(200, 1024, 1024, 0, seed=970)
    layer = prepared(S, L, 0)
    y1, _, _, _ = run(S, layer, L.x, S.PATH_FUSED)
    y2, _, _, _ = run(S, layer, L.x, S.PATH_SEMIFUSED)
    assert np.array_equal(host_bits(y1), host_bits(y2))
