"""The device-check build and buffer canaries (the sanitizer substitute: no
compute-sanitizer on these GPUs).

Odd shapes on every path and kernel (M tails, minimum K and N, the decode
fallbacks, both tensor-core tile heights, group-128 scales) run with guard rows
around y and guard bytes around the workspace; after each call the guards
must be intact, the status word clean and y equal to the CPU oracle's.  They
run once on the normal library and once, in a child process that sets
SPEAR_DEVICE_CHECKS=1, on the device-check build (libspear_checked.so), whose
bounds checks on the output stores and the workspace's partial slots, flags
and published rows report SPEAR_ERR_DEVICE_CHECK instead of touching memory
out of range.  The child also forces each kernel's output-store check to fail
(the guarded stores are skipped, so nothing out of range is touched) and
checks that the launch reports it and that the next call is clean again."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

G_ROWS = 8          # guard rows of y on each side
G_BYTES = 4096      # guard bytes of the workspace on each side
Y_GUARD = 0x7FAB    # a bf16 NaN pattern no kernel writes
WS_GUARD = 0xA5

# M, K, N, r, group, path
CASES = [
    (1, 1024, 512, 16, 0, "decode"),
    (5, 3072, 1024, 32, 128, "decode"),
    (16, 4096, 768, 64, 0, "decode"),
    (13, 640, 1024, 16, 0, "decode"),       # K not a multiple of 512: the cluster split-K kernel
    (4, 8192, 1024, 64, 0, "decode"),       # K beyond the main decode kernel: the earlier one
    (17, 1024, 512, 16, 0, "fused"),
    (129, 2048, 768, 32, 128, "fused"),
    (300, 1024, 1024, 64, 0, "fused"),
    (600, 1024, 1024, 64, 0, "fused"),      # M >= 512 on short tiles with K parts
    (2048, 1024, 4096, 32, 0, "fused"),     # tall tiles
    (40, 1024, 512, 16, 0, "unfused"),
    (40, 1024, 512, 16, 128, "semifused"),
]


def run_cases(S):
    """Every case with canaries; a list of result dicts."""
    from oracle import spear_oracle as O
    from w4_gemm_gated_b200 import synth

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

    paths = {"decode": S.PATH_DECODE, "fused": S.PATH_FUSED, "unfused": S.PATH_UNFUSED,
             "semifused": S.PATH_SEMIFUSED}
    out = []
    for (M, K, N, r, group, path) in CASES:
        L = synth.make_layer(M, K, N, r, b_g=-0.5, x_kind="t3", seed=2000 + M + K // 64 + N // 16)
        layer = S.prepare_layer(torch.from_numpy(L.W).cuda(), group, bf16(L.A), bf16(L.B), bf16(L.w_g), L.b_g)
        nbytes = S.workspace_bytes(layer, M)
        wsbuf = torch.full((nbytes + 2 * G_BYTES,), WS_GUARD, dtype=torch.uint8, device="cuda")
        ws = wsbuf[G_BYTES:G_BYTES + nbytes]
        assert S.F["spear_workspace_init"](ws.data_ptr(), nbytes, None) == S.OK
        ybuf = torch.full((M + 2 * G_ROWS, N), Y_GUARD, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        y = ybuf[G_ROWS:G_ROWS + M]
        S.forward(layer, bf16(L.x), ws, y=y, path=paths[path])
        torch.cuda.synchronize()
        status = S.read_status(ws)
        yb = ybuf.view(torch.int16).cpu().numpy()
        wb = wsbuf.cpu().numpy()
        q, s = O.quantize_rtn(L.W, group)
        y_ref, _ = O.linear(L.x, q, s, group, L.A, L.B, L.w_g, L.b_g)
        yg = O.bf16_to_f64(y.cpu().view(torch.int16).numpy().view(np.uint16))
        out.append({
            "case": [M, K, N, r, group, path], "status": int(status),
            "y_guards": bool(np.all(yb[:G_ROWS] == Y_GUARD) and np.all(yb[G_ROWS + M:] == Y_GUARD)),
            "ws_guards": bool(np.all(wb[:G_BYTES] == WS_GUARD) and np.all(wb[G_BYTES + nbytes:] == WS_GUARD)),
            "finite": bool(np.all(np.isfinite(yg))),
            "rel_err": float(np.max(np.abs(yg - y_ref)) / np.max(np.abs(y_ref))),
        })
    return out


def forced_checks(S):
    """Each kernel's forced output-store check: reported, then a clean call."""
    from w4_gemm_gated_b200 import synth

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

    res = {}
    for kernel, (M, path) in ((1, (4, S.PATH_DECODE)), (2, (64, S.PATH_FUSED))):
        L = synth.make_layer(M, 1024, 512, 16, b_g=-0.5, seed=2100 + kernel)
        layer = S.prepare_layer(torch.from_numpy(L.W).cuda(), 0, bf16(L.A), bf16(L.B), bf16(L.w_g), L.b_g)
        ws = S.make_workspace(layer, M)
        x = bf16(L.x)
        try:
            assert S.F["spear_test_force_device_check"](kernel) == S.OK
            S.forward(layer, x, ws, path=path)
            torch.cuda.synchronize()
        finally:
            S.F["spear_test_force_device_check"](0)
        forced = int(S.read_status(ws))
        S.F["spear_workspace_init"](ws.data_ptr(), ws.numel(), None)
        S.forward(layer, x, ws, path=path)
        torch.cuda.synchronize()
        res[kernel] = [forced, int(S.read_status(ws))]
    return res


def child_main():
    from w4_gemm_gated_b200 import spear as S
    print(json.dumps({"checks_enabled": int(S.F["spear_device_checks_enabled"]()), "lib": S.LIB_PATH,
                      "cases": run_cases(S), "forced": forced_checks(S)}), flush=True)


@pytest.fixture(scope="module")
def S():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from w4_gemm_gated_b200 import build
    build.build()
    build.build(checked=True)
    from w4_gemm_gated_b200 import spear
    return spear


def _check(results):
    for r in results:
        assert r["status"] == 0, r
        assert r["y_guards"] and r["ws_guards"], r
        assert r["finite"] and r["rel_err"] <= 1e-2, r


def test_canaries_normal_build(S):
    assert S.F["spear_device_checks_enabled"]() == 0
    _check(run_cases(S))


def test_device_check_build(S):
    env = dict(os.environ, SPEAR_DEVICE_CHECKS="1", PYTHONPATH=ROOT)
    proc = subprocess.run([sys.executable, "-c", "import tests.test_gpu_devchecks as t; t.child_main()"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert proc.returncode == 0, proc.stderr[-3000:]
    res = json.loads(proc.stdout.strip().splitlines()[-1])
    assert res["checks_enabled"] == 1 and res["lib"].endswith("libspear_checked.so")
    _check(res["cases"])
    ERR_DEVICE_CHECK, OK = 7, 0
    assert res["forced"] == {"1": [ERR_DEVICE_CHECK, OK], "2": [ERR_DEVICE_CHECK, OK]}
