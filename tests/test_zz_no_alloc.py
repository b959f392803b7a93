"""The allocation-free decode call, through the C ABI.

Some callers cannot allocate device memory where they run the layer (a
serving engine that owns the CUDA allocator, token loops in which an
allocation would synchronise the device); for them the library offers a
decode call whose scratch lives in a fixed array inside the library.  These
tests check that call against the regular workspace-based decode call on two
calls in a row (the second reuses the array the first one left behind), on
every decode kernel it can use, and that it leaves the device's free memory
unchanged.
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


def _run_pair(S, L, layer, M):
    """The workspace call and two allocation-free calls on the same input."""
    st = layer.struct()
    x = _bf16(L.x)
    stream = torch.cuda.current_stream().cuda_stream
    ws = S.make_workspace(layer, M)
    y_ref = torch.empty((M, layer.N), dtype=torch.bfloat16, device="cuda")
    rc = S.F["spear_linear_forward_path"](ctypes.byref(st), x.data_ptr(), M, y_ref.data_ptr(), ws.data_ptr(),
                                          ws.numel(), None, None, S.PATH_DECODE, stream)
    assert rc == S.OK, S.F["spear_last_error"]().decode()
    ys = []
    for _ in range(2):
        y = torch.full((M, layer.N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = S.F["spear_linear_forward_decode_noalloc"](ctypes.byref(st), x.data_ptr(), M, y.data_ptr(), None, None,
                                                        stream)
        assert rc == S.OK, S.F["spear_last_error"]().decode()
        ys.append(y)
    torch.cuda.synchronize()
    assert S.read_status_noalloc() == S.OK
    return y_ref, ys


@pytest.mark.parametrize("K,N,r", [(640, 1024, 128), (384, 512, 16)])
def test_noalloc_fallback_kernel_shapes(S, K, N, r):
    # K not a multiple of 512: neither the main decode kernel nor the earlier
    # one runs it, so the call uses the cluster split-K kernel and the other
    # half of the array's layout (projection rows and gated projection)
    M = 16
    L = synth.make_layer(M, K, N, r, b_g=-0.5, seed=40 + K)
    layer = S.prepare_layer(torch.from_numpy(L.W).cuda(), 0, _bf16(L.A), _bf16(L.B), _bf16(L.w_g), L.b_g)
    y_ref, ys = _run_pair(S, L, layer, M)
    q, s = O.quantize_rtn(L.W, 0)
    y_o, _ = O.linear(L.x, q, s, 0, L.A, L.B, L.w_g, L.b_g)
    bound = 1e-2 * np.max(np.abs(y_o))
    for y in ys:
        assert np.max(np.abs(_f64(y) - _f64(y_ref))) <= 1e-2 * np.max(np.abs(_f64(y_ref)))
        assert np.max(np.abs(_f64(y) - y_o)) <= bound


def _rank_layer(S, L, h, seed):
    rng = np.random.default_rng(seed)
    r = L.r
    W1 = torch.from_numpy((rng.standard_normal((h, r)) / np.sqrt(r)).astype(np.float32) * 4.0)
    b1 = torch.from_numpy((rng.standard_normal(h) * 0.2).astype(np.float32))
    W2 = torch.from_numpy((rng.standard_normal((r, h)) / np.sqrt(h)).astype(np.float32) * 2.0)
    b2 = torch.from_numpy((rng.standard_normal(r) - 0.5).astype(np.float32))
    base = S.prepare_layer(torch.from_numpy(L.W).cuda(), 0, _bf16(L.A), _bf16(L.B), _bf16(L.w_g), 0.0)
    return S.with_rank_gate(base, W1, b1, W2, b2, 0.8), (W1.numpy(), b1.numpy(), W2.numpy(), b2.numpy())


def test_noalloc_rank_gate_on_the_earlier_kernel(S):
    # K = 8192 is beyond the main decode kernel: the earlier one runs it, with the rank gate
    M = 4
    L = synth.make_layer(M, 8192, 1024, 64, b_g=0.0, seed=61)
    layer, (W1, b1, W2, b2) = _rank_layer(S, L, 16, 62)
    y_ref, ys = _run_pair(S, L, layer, M)
    q, s = O.quantize_rtn(L.W, 0)
    y_o, _, _ = O.linear_rank_gated(L.x, q, s, 0, L.A, L.B, W1, b1, W2, b2, 0.8)
    for y in ys:
        assert np.max(np.abs(_f64(y) - y_o)) <= 1e-2 * np.max(np.abs(y_o))


def test_noalloc_rank_gate_refused_on_the_fallback_kernel(S):
    L = synth.make_layer(4, 640, 1024, 64, b_g=0.0, seed=63)
    layer, _ = _rank_layer(S, L, 16, 64)
    st = layer.struct()
    x = _bf16(L.x)
    y = torch.empty((4, 1024), dtype=torch.bfloat16, device="cuda")
    rc = S.F["spear_linear_forward_decode_noalloc"](ctypes.byref(st), x.data_ptr(), 4, y.data_ptr(), None, None, None)
    assert rc == S.ERR_UNSUPPORTED_SHAPE
    assert "rank gate" in S.F["spear_last_error"]().decode()


def test_noalloc_allocates_no_device_memory(S):
    # after a first call (which may load the library's device code), two more
    # calls leave the device's free memory exactly as it was
    M = 16
    L = synth.decode(M, force_outlier=True)
    layer = S.prepare_layer(torch.from_numpy(L.W).cuda(), 0, _bf16(L.A), _bf16(L.B), _bf16(L.w_g), L.b_g)
    st = layer.struct()
    x = _bf16(L.x)
    y = torch.empty((M, layer.N), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    call = S.F["spear_linear_forward_decode_noalloc"]
    assert call(ctypes.byref(st), x.data_ptr(), M, y.data_ptr(), None, None, stream) == S.OK
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        assert call(ctypes.byref(st), x.data_ptr(), M, y.data_ptr(), None, None, stream) == S.OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert S.read_status_noalloc() == S.OK
