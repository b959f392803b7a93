"""The allocation-free decode call, through the C ABI.

Some callers cannot allocate device memory where they run the layer (a
serving engine that owns the CUDA allocator, token loops in which an
allocation would synchronise the device); for them the library offers a
decode call whose scratch lives in a fixed array inside the library.  This
test checks that call against the regular workspace-based decode call on two
calls in a row (the second reuses the array the first one left behind).
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import spear_oracle as O
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


def _f64(t):
    return O.bf16_to_f64(t.cpu().view(torch.int16).numpy().view(np.uint16))


@pytest.mark.parametrize("M", [1, 16])
def test_noalloc_matches_workspace_call_twice(S, M):
    L = synth.decode(M, force_outlier=True)
    layer = S.prepare_layer(torch.from_numpy(L.W).cuda(), 0, _bf16(L.A), _bf16(L.B), _bf16(L.w_g), L.b_g)
    st = layer.struct()
    x = _bf16(L.x)
    stream = torch.cuda.current_stream().cuda_stream

    # the existing entry point with a caller workspace
    ws = S.make_workspace(layer, M)
    y_ref = torch.empty((M, layer.N), dtype=torch.bfloat16, device="cuda")
    g_ref = torch.zeros(M, dtype=torch.float32, device="cuda")
    rc = S.F["spear_linear_forward_path"](ctypes.byref(st), x.data_ptr(), M, y_ref.data_ptr(), ws.data_ptr(),
                                          ws.numel(), g_ref.data_ptr(), None, S.PATH_DECODE, stream)
    assert rc == S.OK, S.F["spear_last_error"]().decode()

    outs = []
    for _ in range(2):
        y = torch.full((M, layer.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        g = torch.zeros(M, dtype=torch.float32, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        rc = S.F["spear_linear_forward_decode_noalloc"](ctypes.byref(st), x.data_ptr(), M, y.data_ptr(),
                                                        g.data_ptr(), cnt.data_ptr(), stream)
        assert rc == S.OK, S.F["spear_last_error"]().decode()
        outs.append((y, g, cnt))
    torch.cuda.synchronize()

    yr = _f64(y_ref)
    bound = 1e-2 * np.max(np.abs(yr))
    for y, g, cnt in outs:
        yn = _f64(y)
        assert np.all(np.isfinite(yn))
        assert np.max(np.abs(yn - yr)) <= bound
        assert torch.allclose(g, g_ref, atol=1e-6)
        assert int(cnt.item()) == int((g_ref < 0.1).sum().item())
    # and both agree with the CPU oracle
    q, s = O.quantize_rtn(L.W, 0)
    y_o, _ = O.linear(L.x, q, s, 0, L.A, L.B, L.w_g, L.b_g)
    assert np.max(np.abs(_f64(outs[1][0]) - y_o)) <= 1e-2 * np.max(np.abs(y_o))


def test_noalloc_rejects_large_m(S):
    L = synth.make_layer(17, 1024, 1024, 16, seed=3)
    layer = S.prepare_layer(torch.from_numpy(L.W).cuda(), 0, _bf16(L.A), _bf16(L.B), _bf16(L.w_g), L.b_g)
    st = layer.struct()
    x = _bf16(L.x)
    y = torch.empty((17, 1024), dtype=torch.bfloat16, device="cuda")
    rc = S.F["spear_linear_forward_decode_noalloc"](ctypes.byref(st), x.data_ptr(), 17, y.data_ptr(), None, None,
                                                    None)
    assert rc == S.ERR_UNSUPPORTED_SHAPE
    assert "M <= 16" in S.F["spear_last_error"]().decode()
