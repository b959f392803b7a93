"""GPU parity of the pages' per-rank gate (SPEAR, gist.science technical
summary, section 2.1 A): y = x . dequant(W4) + alpha * ((x . A) * gamma) . B
with gamma = sigmoid(W2 relu(W1 (x . A) + b1) + b2), on every path that
carries it (decode kernel, tensor-core kernel, unfused and semi-fused EC),
against the CPU oracle.  The reported gate is the mean of gamma."""
import numpy as np
import pytest
import torch

from oracle import spear_oracle as O
from tests.test_gpu_parity import GATE_TOL, assert_close, dev_bf16, prepared
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


def _gate_params(r, h, seed):
    rng = np.random.default_rng(seed)
    W1 = (rng.standard_normal((h, r)) / np.sqrt(r)).astype(np.float32) * 4.0
    b1 = (rng.standard_normal(h) * 0.2).astype(np.float32)
    W2 = (rng.standard_normal((r, h)) / np.sqrt(h)).astype(np.float32) * 2.0
    b2 = (rng.standard_normal(r) * 1.0 - 0.5).astype(np.float32)
    return W1, b1, W2, b2


def _case(S, M, K, N, r, h, group, seed, alpha=0.8):
    L = synth.make_layer(M, K, N, r, b_g=0.0, x_kind="t3", seed=seed)
    L.w_g = O.f32_to_bf16_bits_rne(np.zeros(K, np.float32))   # unused by the rank gate
    W1, b1, W2, b2 = _gate_params(r, h, seed + 1)
    base = prepared(S, L, group)
    layer = S.with_rank_gate(base, torch.from_numpy(W1), torch.from_numpy(b1), torch.from_numpy(W2),
                             torch.from_numpy(b2), alpha)
    q, s = O.quantize_rtn(L.W, group)
    y_ref, gam, gmean = O.linear_rank_gated(L.x, q, s, group, L.A, L.B, W1, b1, W2, b2, alpha)
    return L, layer, y_ref, gmean


def _run(S, layer, x_bits, path, M_max=None):
    x = dev_bf16(x_bits)
    M = x.shape[0]
    ws = S.make_workspace(layer, M_max or max(M, 16))
    g = torch.zeros(M, dtype=torch.float32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = S.forward(layer, x, ws, gate_out=g, mask_count=cnt, path=path)
    torch.cuda.synchronize()
    assert S.read_status(ws) == S.OK
    return y, g.cpu().numpy(), int(cnt.item())


def _check_gate(g, gmean, cnt):
    assert np.max(np.abs(g - gmean)) <= GATE_TOL
    # the count is decided in fp32 on the device: it must equal the count of the
    # gates it reported, and the oracle's up to gates within rounding of tau
    assert cnt == int(np.sum(g < np.float32(O.TAU_DEFAULT)))
    near = int(np.sum(np.abs(gmean - O.TAU_DEFAULT) <= GATE_TOL))
    assert abs(cnt - int(np.sum(gmean < O.TAU_DEFAULT))) <= near


@pytest.mark.parametrize("M,r,h,group", [(1, 64, 16, 0), (5, 16, 8, 0), (16, 128, 32, 128), (16, 32, 16, 0)])
def test_rank_gate_decode(S, M, r, h, group):
    L, layer, y_ref, gmean = _case(S, M, 4096, 2048, r, h, group, seed=1000 + M + r)
    y, g, cnt = _run(S, layer, L.x, S.PATH_DECODE)
    assert_close(y, y_ref)
    _check_gate(g, gmean, cnt)


@pytest.mark.parametrize("M,r,h,group", [(17, 64, 16, 0), (200, 16, 8, 128), (300, 128, 32, 0)])
def test_rank_gate_fused(S, M, r, h, group):
    L, layer, y_ref, gmean = _case(S, M, 2048, 1024, r, h, group, seed=2000 + M + r)
    y, g, cnt = _run(S, layer, L.x, S.PATH_FUSED)
    assert_close(y, y_ref)
    _check_gate(g, gmean, cnt)


@pytest.mark.parametrize("path", ["unfused", "semifused"])
@pytest.mark.parametrize("M,r,h,group", [(8, 64, 16, 0), (100, 32, 32, 128), (257, 128, 8, 0)])
def test_rank_gate_separate_ec(S, path, M, r, h, group):
    L, layer, y_ref, gmean = _case(S, M, 2048, 1024, r, h, group, seed=3000 + M + r)
    y, g, cnt = _run(S, layer, L.x, S.PATH_UNFUSED if path == "unfused" else S.PATH_SEMIFUSED)
    assert_close(y, y_ref)
    _check_gate(g, gmean, cnt)


def test_rank_gate_full_decode_shape(S):
    """Config 2's shape (K=4096, N=11008, r=64) at M = 1, 4, 16 with the rank gate."""
    for M in (1, 4, 16):
        L, layer, y_ref, gmean = _case(S, M, 4096, 11008, 64, 16, 0, seed=4000 + M)
        y, g, cnt = _run(S, layer, L.x, S.PATH_DECODE)
        assert_close(y, y_ref)
        _check_gate(g, gmean, cnt)


def test_rank_gate_constant_matches_scalar_gate(S):
    """W1 = W2 = 0 and b2 = c: every rank's gate is sigmoid(c), which is the
    scalar gate with w_g = 0 and b_g = c: the two layer forms agree on the GPU."""
    M, K, N, r, h = 16, 2048, 1024, 64, 16
    L = synth.make_layer(M, K, N, r, b_g=0.0, seed=5000)
    L.w_g = O.f32_to_bf16_bits_rne(np.zeros(K, np.float32))
    c = -0.4
    scalar = prepared(S, L, 0, b_g=c)
    rank = S.with_rank_gate(scalar, torch.zeros(h, r), torch.zeros(h), torch.zeros(r, h), torch.full((r,), c), 1.0)
    for path in (S.PATH_DECODE, S.PATH_FUSED, S.PATH_UNFUSED):
        y1, g1, _ = _run(S, scalar, L.x, path)
        y2, g2, _ = _run(S, rank, L.x, path)
        assert np.max(np.abs(g1 - g2)) <= 1e-6
        d = (y1.float() - y2.float()).abs().max().item()
        assert d <= 1e-2 * y1.float().abs().max().item() * 0.1, (path, d)
