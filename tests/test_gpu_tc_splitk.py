"""GPU parity of the tensor-core kernel's K parts at mid M, against the CPU
oracle.

While the 128-token tiles of a launch fill less than half the SMs (256-token
tiles are taken only where they fill at least half), the kernel splits every
tile's K into S = 2, 4 or 8 parts (at least 8 k-steps each), one CTA per
part.  Every part puts its fp32 accumulator in the workspace; each then sums,
in part order, its 256 / S output channels (the projection tile whole on part
0), and the gated projection's EC steps run in the last part.  Where no split
is taken but the tiles leave SMs idle, stream-K runs: every SM takes an equal
run of the tiles' concatenated k-steps, and the CTA that holds a tile's first
steps adds the other parts in k order and finishes it (with its EC steps).
The shapes below select each S and stream-K (the schedule computed here with
the launch's rule on this device's SM count and asserted), with the scalar
gate, the pages' per-rank gate, no EC, group-128 scales, and token counts that
leave the last 128-token block ragged or fill only its first 32-row quarter."""
import numpy as np
import pytest
import torch

from oracle import spear_oracle as O
from tests.test_gpu_parity import GATE_TOL, assert_close, dev_bf16, oracle_ref, prepared, run
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


def schedule(M, K, N, r, sms):
    """The launch's rule: 256-token tiles only from M = 512 up and when they fill
    at least half the SMs (persistent then); else 128-token tiles, projection
    tiles when r > 0, K parts S = 2, 4, 8 while the tiles fill at most half
    the SMs, and stream-K where no split was taken but tiles leave SMs idle.
    Returns ("persistent", 1), ("split", S) or ("streamk", most parts of a tile)."""
    if M >= 512:
        mb256 = (M + 255) // 256
        if 2 * ((mb256 if r else 0) + mb256 * (N // 256)) >= sms:
            return ("persistent", 1)
    mb = (M + 127) // 128
    ntiles = (mb if r else 0) + mb * (N // 256)
    kt = K // 64
    s = 1
    while s < 8 and ntiles * s * 2 <= sms and kt % (2 * s) == 0 and kt // (2 * s) >= 8:
        s *= 2
    if s > 1:
        return ("split", s)
    T = ntiles * kt
    if ntiles < sms and T // sms >= 8:
        lo = [c * T // sms for c in range(sms + 1)]
        most = max(sum(1 for c in range(sms) if lo[c] < (t + 1) * kt and lo[c + 1] > t * kt) for t in range(ntiles))
        return ("streamk", most)
    return ("persistent", 1)


CASES = [
    # M, K, N, r, group, expected schedule
    (32, 4096, 4096, 64, 0, ("split", 8)),      # 17 tiles: one 32-row quarter of one token block
    (100, 4096, 4096, 64, 128, ("split", 8)),   # ragged token block, grouped scales
    (256, 4096, 4096, 64, 0, ("split", 4)),     # 34 tiles
    (200, 4096, 4096, 32, 0, ("split", 4)),     # two blocks, the second ragged
    (128, 4096, 11008, 64, 0, ("split", 2)),    # 44 tiles
    (64, 1024, 4096, 16, 0, ("split", 2)),      # K = 1024: 16 k-steps, at most 2 parts
    (48, 4096, 4096, 0, 0, ("split", 8)),       # no EC: 16 output tiles only
    (512, 4096, 4096, 64, 0, ("split", 2)),     # 34 tall tiles would fill too few SMs: 68 short x 2
    (256, 4096, 11008, 64, 0, ("streamk", 3)),  # 88 tiles: one run of ~38 k-steps per SM, a tile on up to 3
    (384, 2048, 6144, 32, 0, ("streamk", 3)),   # 75 tiles of 32 k-steps, ~16 a CTA
    (300, 4096, 8192, 64, 128, ("streamk", 3)), # ragged last block, grouped scales
]


@pytest.mark.parametrize("M,K,N,r,group,want", CASES)
def test_k_parts_match_oracle(S, M, K, N, r, group, want):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert schedule(M, K, N, r, sms) == want
    L = synth.make_layer(M, K, N, r, b_g=-0.5, x_kind="t3", seed=1200 + M + r)
    layer = prepared(S, L, group)
    y, g, cnt, _ = run(S, layer, L.x, S.PATH_FUSED, gate=True)
    y_ref, g_ref, _, _ = oracle_ref(L, group)
    assert_close(y, y_ref)
    if r:
        gg = g.cpu().numpy()
        assert np.max(np.abs(gg - g_ref)) <= GATE_TOL
        assert int(cnt.item()) == int(np.sum(g_ref < 0.1))


@pytest.mark.parametrize("M,N", [(32, 4096), (256, 4096), (256, 11008)])
def test_k_parts_rank_gate(S, M, N):
    # the per-rank gate (h = 16) on the projection tile's part 0, after the sum
    K, r, h = 4096, 64, 16
    L = synth.make_layer(M, K, N, r, b_g=0.0, x_kind="t3", seed=1300 + M)
    rng = np.random.default_rng(1301 + M)
    W1 = (rng.standard_normal((h, r)) / np.sqrt(r)).astype(np.float32) * 4.0
    b1 = (rng.standard_normal(h) * 0.2).astype(np.float32)
    W2 = (rng.standard_normal((r, h)) / np.sqrt(h)).astype(np.float32) * 2.0
    b2 = (rng.standard_normal(r) - 0.5).astype(np.float32)
    base = prepared(S, L, 0, b_g=0.0)
    layer = S.with_rank_gate(base, torch.from_numpy(W1), torch.from_numpy(b1), torch.from_numpy(W2),
                             torch.from_numpy(b2), 0.8)
    y, _, _, _ = run(S, layer, L.x, S.PATH_FUSED)
    q, s = O.quantize_rtn(L.W, 0)
    y_ref, _, _ = O.linear_rank_gated(L.x, q, s, 0, L.A, L.B, W1, b1, W2, b2, 0.8)
    assert_close(y, y_ref)


def test_k_parts_repeat_and_reuse(S):
    # the same workspace across launches of different S: the partial flags are
    # epoch-tagged, so nothing stale is taken for a new launch's partial
    L = synth.make_layer(256, 4096, 4096, 64, b_g=-0.5, x_kind="t3", seed=1400)
    layer = prepared(S, L, 0)
    y_ref, _, _, _ = oracle_ref(L, 0)
    ws = S.make_workspace(layer, 256)
    for M in (256, 32, 256, 100, 32):
        x = dev_bf16(L.x[:M])
        y = S.forward(layer, x, ws, path=S.PATH_FUSED)
        torch.cuda.synchronize()
        assert S.read_status(ws) == S.OK
        assert_close(y, y_ref[:M])
