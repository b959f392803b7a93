"""Measured-time dispatcher on the GPU: after ``spear_dispatch_tune`` the table's
choice for every M bucket is a path whose independently re-measured time is
within 5 % of the fastest eligible path (or within timing noise of it)."""
import numpy as np
import pytest
import torch

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


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _median_us(S, layer, x, y, ws, path, flush, reps=15):
    stream = torch.cuda.current_stream()
    ts = []
    for i in range(reps + 3):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        S.forward(layer, x, ws, y=y, path=path, stream=stream)
        b.record(stream)
        b.synchronize()
        if i >= 3:
            ts.append(a.elapsed_time(b) * 1e3)
    return float(np.median(ts))


@pytest.mark.parametrize("shape,r,group", [((4096, 4096), 32, 0), ((4096, 14336), 128, 128)])
def test_dispatch_tune_picks_faster_path(S, shape, r, group):
    K, N = shape
    Ms = [1, 8, 32, 128, 512]
    L = synth.sweep_point(max(Ms), K, N, r)
    layer = S.prepare_layer(torch.from_numpy(L.W).cuda(), group, _bf16(L.A), _bf16(L.B), _bf16(L.w_g), L.b_g)
    x_all = _bf16(L.x)
    ws = S.make_workspace(layer, max(Ms))
    y_all = torch.empty((max(Ms), N), dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    S.dispatch_clear()
    S.dispatch_tune(layer, Ms, x_all, y_all, ws, flush=flush, reps=15)
    assert S.read_status(ws) == S.OK
    for M in Ms:
        choice = S.dispatch_choice(layer, M)
        paths = [S.PATH_FUSED, S.PATH_UNFUSED, S.PATH_SEMIFUSED] + ([S.PATH_DECODE] if M <= 16 else [])
        assert choice in paths
        assert S.dispatch_time_us(layer, M) > 0.0     # tuning records the chosen path's time
        x = x_all[:M].contiguous()
        y = y_all[:M]
        t = {p: _median_us(S, layer, x, y, ws, p, flush) for p in paths}
        best = min(t.values())
        # within 5 % of the fastest, or within 2 us of it (timing noise at small M)
        assert t[choice] <= max(1.05 * best, best + 2.0), (M, choice, t)
    # the SLO picker reads those times: with no overhead and an SLO equal to a
    # bucket's time, that bucket's chunk is the largest that fits
    t512 = S.dispatch_time_us(layer, 512)
    chunk, pred = S.slo_chunk([layer], 0, t512, Ms)
    assert pred <= t512 and chunk >= max(m for m in Ms if S.dispatch_time_us(layer, m) <= t512)
    S.dispatch_clear()
