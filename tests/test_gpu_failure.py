"""Device-side failure handling, on the GPU, without a fault: a bounded wait is
made to run out and the kernel must report SPEAR_ERR_TIMEOUT, leave without
hanging (every role stops at its next check and waits for its copies in
flight), and leave the context usable, so that the next call after
spear_workspace_init matches the oracle again.

The expired wait is the decode kernel's wait for the published EC rows and
the tensor-core kernel's wait for the gated projection: the test hook makes
them expect a tag that no launch publishes, with a short cycle bound."""
import numpy as np
import pytest
import torch

from oracle import spear_oracle as O
from tests.test_gpu_parity import assert_close, dev_bf16, prepared
from w4_gemm_gated_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4_gemm_gated_b200 import build
    build.build()
    from w4_gemm_gated_b200 import spear
    yield spear
    spear.test_inject_timeout(0)


@pytest.mark.parametrize("kernel,M,path", [(1, 4, "decode"), (2, 256, "fused")])
def test_expired_wait_reports_timeout_then_recovers(S, kernel, M, path):
    L = synth.make_layer(M, 4096, 2048, 64, b_g=-0.5, x_kind="t3", seed=900 + M)
    layer = prepared(S, L, 0)
    x = dev_bf16(L.x)
    ws = S.make_workspace(layer, M)
    p = S.PATH_DECODE if path == "decode" else S.PATH_FUSED
    try:
        S.test_inject_timeout(kernel, 20000)
        S.forward(layer, x, ws, path=p)
        torch.cuda.synchronize()
    finally:
        S.test_inject_timeout(0)
    assert S.read_status(ws) == S.ERR_TIMEOUT
    # the context is still usable: re-initialise the workspace and run again
    S.F["spear_workspace_init"](ws.data_ptr(), ws.numel(), None)
    y = S.forward(layer, x, ws, path=p)
    torch.cuda.synchronize()
    assert S.read_status(ws) == S.OK
    q, s = O.quantize_rtn(L.W, 0)
    assert_close(y, O.linear(L.x, q, s, 0, L.A, L.B, L.w_g, L.b_g)[0])


def test_noalloc_status_is_sticky_until_read(S):
    """The allocation-free call's status word keeps a timeout across later
    calls (which clear the rest of the array's header) until it is read."""
    L = synth.make_layer(2, 4096, 2048, 32, b_g=-0.5, seed=950)
    layer = prepared(S, L, 0)
    x = dev_bf16(L.x)
    assert S.read_status_noalloc() == S.OK          # start from a clean word
    try:
        S.test_inject_timeout(1, 20000)
        S.forward_decode_noalloc(layer, x)
        torch.cuda.synchronize()
    finally:
        S.test_inject_timeout(0)
    y = S.forward_decode_noalloc(layer, x)           # a good call after the failed one
    torch.cuda.synchronize()
    assert S.read_status_noalloc() == S.ERR_TIMEOUT  # not erased by the good call
    assert S.read_status_noalloc() == S.OK           # read and cleared
    y = S.forward_decode_noalloc(layer, x)
    torch.cuda.synchronize()
    assert S.read_status_noalloc() == S.OK
    q, s = O.quantize_rtn(L.W, 0)
    assert_close(y, O.linear(L.x, q, s, 0, L.A, L.B, L.w_g, L.b_g)[0])
