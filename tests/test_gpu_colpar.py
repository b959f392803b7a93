"""GPU parity of the column-parallel split, with the ranks emulated on one GPU:
each rank's shard is prepared from the full weights and run in turn (no kernel
waits on another), and the shards' outputs are assembled with the same
function the all-gather uses.  Checked against the CPU oracle of the whole
layer on the decode and tensor-core paths, with the scalar and the per-rank
gate, and bitwise against the whole layer's own call on the decode path
(every 16-channel strip is reduced the same way whichever CTA owns it)."""
import numpy as np
import pytest
import torch

from oracle import spear_oracle as O
from tests.test_gpu_parity import GATE_TOL, assert_close, dev_bf16, host_bits
from w4_gemm_gated_b200 import colpar, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4_gemm_gated_b200 import build
    build.build()
    from w4_gemm_gated_b200 import spear
    return spear


def _shards(S, L, group, world):
    W = torch.from_numpy(L.W).cuda()
    A, B, wg = dev_bf16(L.A), dev_bf16(L.B), dev_bf16(L.w_g)
    return [colpar.prepare_shard(W, group, A, B, wg, L.b_g, p, world) for p in range(world)]


@pytest.mark.parametrize("M,path", [(4, "decode"), (16, "decode"), (256, "fused"), (40, "fused")])
@pytest.mark.parametrize("world", [2, 3])
def test_column_shards_match_oracle(S, M, path, world):
    K, N, r, group = 4096, 3072, 64, 0
    L = synth.make_layer(M, K, N, r, b_g=-0.5, x_kind="t3", seed=1500 + M + world)
    p = S.PATH_DECODE if path == "decode" else S.PATH_FUSED
    x = dev_bf16(L.x)
    parts, ranges, gates = [], [], []
    for layer, rng in _shards(S, L, group, world):
        ws = S.make_workspace(layer, M)
        g = torch.zeros(M, dtype=torch.float32, device="cuda")
        parts.append(S.forward(layer, x, ws, gate_out=g, path=p))
        torch.cuda.synchronize()
        assert S.read_status(ws) == S.OK
        ranges.append(rng)
        gates.append(g.cpu().numpy())
    y = colpar.assemble(parts, ranges, N)
    q, s = O.quantize_rtn(L.W, group)
    y_ref, g_ref = O.linear(L.x, q, s, group, L.A, L.B, L.w_g, L.b_g)
    assert_close(y, y_ref)
    for g in gates:   # every rank computes the same gate from the replicated x
        assert np.max(np.abs(g - g_ref)) <= GATE_TOL
    if path == "decode":
        # the whole layer's own call gives the same bits
        W = torch.from_numpy(L.W).cuda()
        full = S.prepare_layer(W, group, dev_bf16(L.A), dev_bf16(L.B), dev_bf16(L.w_g), L.b_g)
        ws = S.make_workspace(full, M)
        y_full = S.forward(full, x, ws, path=p)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(y), host_bits(y_full))


def test_column_shards_rank_gate_group128(S):
    M, K, N, r, h, world = 64, 4096, 2048, 64, 16, 2
    L = synth.make_layer(M, K, N, r, b_g=0.0, x_kind="t3", seed=1600)
    rng = np.random.default_rng(1601)
    W1 = (rng.standard_normal((h, r)) / np.sqrt(r)).astype(np.float32) * 4.0
    b1 = (rng.standard_normal(h) * 0.2).astype(np.float32)
    W2 = (rng.standard_normal((r, h)) / np.sqrt(h)).astype(np.float32) * 2.0
    b2 = (rng.standard_normal(r) - 0.5).astype(np.float32)
    x = dev_bf16(L.x)
    parts, ranges = [], []
    for layer, rg in _shards(S, L, 128, world):
        layer = S.with_rank_gate(layer, torch.from_numpy(W1), torch.from_numpy(b1), torch.from_numpy(W2),
                                 torch.from_numpy(b2), 0.8)
        ws = S.make_workspace(layer, M)
        parts.append(S.forward(layer, x, ws, path=S.PATH_FUSED))
        torch.cuda.synchronize()
        assert S.read_status(ws) == S.OK
        ranges.append(rg)
    y = colpar.assemble(parts, ranges, N)
    q, s = O.quantize_rtn(L.W, 128)
    y_ref, _, _ = O.linear_rank_gated(L.x, q, s, 128, L.A, L.B, W1, b1, W2, b2, 0.8)
    assert_close(y, y_ref)
