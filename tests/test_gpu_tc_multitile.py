"""GPU parity of the tensor-core paths when the grid holds far more output
tiles than there are SMs, so that every CTA of the persistent kernel runs a
second and later tile (the reused accumulator, the next-tile prefetch and
the per-tile scale staging), against the CPU oracle.

Shapes are the dispatch sweep's large points (K, N) = (4096, 14336) at
M = 2048 with r = 128 and group-128 scales (456 tiles), and (4096, 4096) at
M = 8192 with r = 32 (544 tiles), plus the pages' per-rank gate at M = 4096.
The oracle runs on a seeded sample of whole rows: the first and last row of
every 128-token block and two more drawn at random from it, so every output
tile (a token block times a channel block) is compared on whole rows, every
channel, within the bound max|y - y_ref| <= 1e-2 max|y_ref| over the sample."""
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


def sample_rows(M, seed):
    rng = np.random.default_rng(seed)
    rows = set()
    for b0 in range(0, M, 128):
        b1 = min(M, b0 + 128)
        rows.update({b0, b1 - 1})
        rows.update(int(v) for v in rng.integers(b0, b1, size=2))
    return np.array(sorted(rows))


def run_rows(S, layer, x_bits, path, rows):
    x = dev_bf16(x_bits)
    M = x.shape[0]
    ws = S.make_workspace(layer, M)
    g = torch.zeros(M, dtype=torch.float32, device="cuda")
    y = S.forward(layer, x, ws, gate_out=g, path=path)
    torch.cuda.synchronize()
    assert S.read_status(ws) == S.OK
    idx = torch.from_numpy(rows).cuda()
    return y.index_select(0, idx), g.cpu().numpy()[rows]


def tiles(M, N, tm=256):
    return ((M + tm - 1) // tm) * (N // 256)


@pytest.mark.parametrize("M,K,N,r,group", [(2048, 4096, 14336, 128, 128), (8192, 4096, 4096, 32, 0)])
def test_more_tiles_than_sms_scalar_gate(S, M, K, N, r, group):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert tiles(M, N) > 2 * sms
    L = synth.sweep_point(M, K, N, r, seed=31)
    layer = prepared(S, L, group)
    rows = sample_rows(M, seed=M + N)
    q, s = O.quantize_rtn(L.W, group)
    y_ref, g_ref = O.linear(L.x[rows], q, s, group, L.A, L.B, L.w_g, L.b_g)
    for path in (S.PATH_FUSED, S.PATH_UNFUSED, S.PATH_SEMIFUSED):
        y, g = run_rows(S, layer, L.x, path, rows)
        assert_close(y, y_ref)
        assert np.max(np.abs(g - g_ref)) <= GATE_TOL, path


def test_more_tiles_than_sms_rank_gate(S):
    M, K, N, r, h = 4096, 4096, 4096, 64, 32
    L = synth.make_layer(M, K, N, r, b_g=0.0, x_kind="t3", seed=41)
    L.w_g = O.f32_to_bf16_bits_rne(np.zeros(K, np.float32))   # unused by the rank gate
    rng = np.random.default_rng(42)
    W1 = (rng.standard_normal((h, r)) / np.sqrt(r)).astype(np.float32) * 4.0
    b1 = (rng.standard_normal(h) * 0.2).astype(np.float32)
    W2 = (rng.standard_normal((r, h)) / np.sqrt(h)).astype(np.float32) * 2.0
    b2 = (rng.standard_normal(r) * 1.0 - 0.5).astype(np.float32)
    base = prepared(S, L, 0)
    layer = S.with_rank_gate(base, torch.from_numpy(W1), torch.from_numpy(b1), torch.from_numpy(W2),
                             torch.from_numpy(b2), 0.8)
    rows = sample_rows(M, seed=43)
    q, s = O.quantize_rtn(L.W, 0)
    y_ref, _, gmean = O.linear_rank_gated(L.x[rows], q, s, 0, L.A, L.B, W1, b1, W2, b2, 0.8)
    for path in (S.PATH_FUSED, S.PATH_UNFUSED, S.PATH_SEMIFUSED):
        y, g = run_rows(S, layer, L.x, path, rows)
        assert_close(y, y_ref)
        assert np.max(np.abs(g - gmean)) <= GATE_TOL, path
