"""C-ABI checks that need no GPU: the library loads, exports every function
that include/spear.h declares, and its host-side logic (size queries,
argument validation, dispatch table) behaves as documented."""
import ctypes
import os
import re

import numpy as np
import pytest

from tests.conftest import ROOT


def _header_functions():
    src = open(os.path.join(ROOT, "include", "spear.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_0-9]+\**\s+\**(spear_[A-Za-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def S():
    from w4_gemm_gated_b200 import build
    build.build()
    from w4_gemm_gated_b200 import spear
    return spear


def test_header_declares_expected_api():
    names = _header_functions()
    for must in ["spear_w4_quantize", "spear_w4_pack", "spear_w4_unpack", "spear_ec_prescale_B", "spear_ec_pack",
                 "spear_workspace_bytes", "spear_linear_forward", "spear_linear_forward_path",
                 "spear_dispatch_tune", "spear_dispatch_choice", "spear_dispatch_save", "spear_dispatch_load"]:
        assert must in names


def test_library_exports_every_header_symbol(S):
    lib = ctypes.CDLL(S.LIB_PATH)
    for name in _header_functions():
        assert hasattr(lib, name), name
    # and the binding declares a prototype for each of them
    assert set(_header_functions()) <= set(S.EXPORTS)


def test_size_queries(S):
    assert S.F["spear_w4_packed_bytes"](11008, 4096) == 11008 * 4096 // 2
    assert S.F["spear_w4_packed_bytes"](10, 64) == 0
    assert S.F["spear_scale_count"](512, 512, 0) == 512
    assert S.F["spear_scale_count"](4096, 14336, 128) == 112 * 4096
    assert S.F["spear_scale_count"](4096, 100, 128) == 0
    assert S.F["spear_ec_agt_count"](4096, 64) == 65 * 4096
    assert S.F["spear_ec_bpt_count"](11008, 64) == 11008 * 64
    assert S.version() >= 100
    assert S.F["spear_status_string"](S.ERR_WORKSPACE) == b"SPEAR_ERR_WORKSPACE"


def _layer(S, **kw):
    d = dict(K=512, N=512, group=0, r=16, w_packed=0x10000, scales=0x20000, AgT=0x30000, BpT=0x40000,
             b_g=0.0, gate_tau=0.1)
    d.update(kw)
    return S.LayerStruct(d["K"], d["N"], d["group"], d["r"], d["w_packed"], d["scales"], d["AgT"], d["BpT"],
                         d["b_g"], d["gate_tau"])


@pytest.mark.parametrize("kw,code", [
    (dict(K=500), 2), (dict(N=130), 2), (dict(r=8), 2), (dict(group=64), 2),
    (dict(w_packed=None), 1), (dict(AgT=None), 1), (dict(scales=0x20008), 3),
])
def test_forward_validation_before_launch(S, kw, code):
    st = _layer(S, **kw)
    rc = S.F["spear_linear_forward"](ctypes.byref(st), 0x50000, 4, 0x60000, 0x70000, 1 << 30, None, None, None)
    assert rc == code
    assert S.F["spear_last_error"]().decode()


def test_forward_rejects_bad_m_and_pointers(S):
    st = _layer(S)
    F = S.F["spear_linear_forward_path"]
    assert F(ctypes.byref(st), 0x50000, 0, 0x60000, 0x70000, 1 << 30, None, None, 0, None) == S.ERR_UNSUPPORTED_SHAPE
    assert F(ctypes.byref(st), None, 4, 0x60000, 0x70000, 1 << 30, None, None, 0, None) == S.ERR_INVALID_ARG
    assert F(ctypes.byref(st), 0x50004, 4, 0x60000, 0x70000, 1 << 30, None, None, 0, None) == S.ERR_ALIGNMENT
    assert F(ctypes.byref(st), 0x50000, 4, 0x60000, 0x70000, 1 << 30, None, None, 9, None) == S.ERR_INVALID_ARG
    assert F(ctypes.byref(st), 0x50000, 32, 0x60000, 0x70000, 1 << 30, None, None, S.PATH_DECODE, None) \
        == S.ERR_UNSUPPORTED_SHAPE
    assert F(ctypes.byref(st), 0x50000, 4, 0x60000, 0x70000, 16, None, None, 0, None) == S.ERR_WORKSPACE


def test_prep_calls_validate(S):
    assert S.F["spear_w4_pack"](None, 16, 64, 0x1000, None) == S.ERR_INVALID_ARG
    assert S.F["spear_w4_pack"](0x1000, 15, 64, 0x2000, None) == S.ERR_UNSUPPORTED_SHAPE
    assert S.F["spear_w4_unpack"](0x1000, 16, 60, 0x2000, None) == S.ERR_UNSUPPORTED_SHAPE
    assert S.F["spear_w4_quantize"](0x1000, 512, 512, 64, 0x2000, 0x3000, None) == S.ERR_UNSUPPORTED_SHAPE
    assert S.F["spear_ec_pack"](0x1000, 0x2000, 0x3000, 0x4000, 512, 512, 24, 0, 0x5000, 0x6000, None) \
        == S.ERR_UNSUPPORTED_SHAPE


def test_workspace_bytes_grows_with_m(S):
    st = _layer(S, K=4096, N=11008, r=64)
    a = S.F["spear_workspace_bytes"](ctypes.byref(st), 16)
    b = S.F["spear_workspace_bytes"](ctypes.byref(st), 2048)
    assert 0 < a < b
    assert S.F["spear_workspace_bytes"](ctypes.byref(st), 0) == 0


def test_dispatch_table_default_set_save_load(S, tmp_path):
    S.dispatch_clear()
    st = _layer(S, K=4096, N=4096, r=64)
    choice = S.F["spear_dispatch_choice"]
    assert choice(ctypes.byref(st), 1) == S.PATH_DECODE
    assert choice(ctypes.byref(st), 16) == S.PATH_DECODE
    assert choice(ctypes.byref(st), 17) == S.PATH_FUSED
    S.dispatch_set(4096, 4096, 64, 0, 100, S.PATH_UNFUSED)     # bucket 128
    assert choice(ctypes.byref(st), 65) == S.PATH_UNFUSED
    assert choice(ctypes.byref(st), 128) == S.PATH_UNFUSED
    assert choice(ctypes.byref(st), 129) == S.PATH_FUSED
    with pytest.raises(S.SpearError):
        S.dispatch_set(4096, 4096, 64, 0, 64, S.PATH_DECODE)   # decode only up to M = 16
    p = str(tmp_path / "lut.txt")
    S.dispatch_save(p)
    S.dispatch_clear()
    assert choice(ctypes.byref(st), 100) == S.PATH_FUSED
    S.dispatch_load(p)
    assert choice(ctypes.byref(st), 100) == S.PATH_UNFUSED
    bad = tmp_path / "bad.txt"
    bad.write_text("1 2 3\n")
    with pytest.raises(S.SpearError):
        S.dispatch_load(str(bad))
    S.dispatch_clear()


def test_dispatch_times_save_load_and_v1_lines(S, tmp_path):
    S.dispatch_clear()
    st = _layer(S, K=4096, N=4096, r=64)
    with pytest.raises(S.SpearError):
        S.dispatch_time_us(st, 8)                              # nothing measured yet
    S.dispatch_set_time(4096, 4096, 64, 0, 8, S.PATH_DECODE, 12.5)
    assert S.dispatch_time_us(st, 5) == pytest.approx(12.5)    # bucket 8
    with pytest.raises(S.SpearError):
        S.dispatch_set_time(4096, 4096, 64, 0, 8, S.PATH_DECODE, -1.0)
    S.dispatch_set(4096, 4096, 64, 0, 64, S.PATH_FUSED)        # path only: no time
    with pytest.raises(S.SpearError):
        S.dispatch_time_us(st, 64)
    p = tmp_path / "lut.txt"
    S.dispatch_save(str(p))
    S.dispatch_clear()
    S.dispatch_load(str(p))
    assert S.dispatch_time_us(st, 8) == pytest.approx(12.5)
    assert S.F["spear_dispatch_choice"](ctypes.byref(st), 64) == S.PATH_FUSED
    # a line without the time column loads as "not measured"
    p.write_text(f"4096 4096 64 0 32 {S.PATH_UNFUSED}\n")
    S.dispatch_clear()
    S.dispatch_load(str(p))
    assert S.F["spear_dispatch_choice"](ctypes.byref(st), 32) == S.PATH_UNFUSED
    with pytest.raises(S.SpearError):
        S.dispatch_time_us(st, 32)
    S.dispatch_clear()


def _rank_layer(S, h=16, **kw):
    st = _layer(S, **kw)
    st.gate_kind = S.GATE_RANK_MLP
    st.gate_hidden = h
    st.gate_w1, st.gate_b1, st.gate_w2, st.gate_b2 = 0x80000, 0x90000, 0xA0000, 0xB0000
    st.gate_alpha = 1.0
    return st


def test_dispatch_key_separates_gate_forms(S, tmp_path):
    # a scalar-gate and a rank-gate layer of the same (K, N, r, group) have
    # entries of their own, per bottleneck width, and the SLO picker reads the
    # entry of each layer's own gate form
    S.dispatch_clear()
    sc = _layer(S, K=4096, N=4096, r=64)
    rk = _rank_layer(S, K=4096, N=4096, r=64, h=16)
    rk32 = _rank_layer(S, K=4096, N=4096, r=64, h=32)
    S.dispatch_set_layer(sc, 256, S.PATH_FUSED, 40.0)
    S.dispatch_set_layer(rk, 256, S.PATH_SEMIFUSED, 90.0)
    choice = S.F["spear_dispatch_choice"]
    assert choice(ctypes.byref(sc), 256) == S.PATH_FUSED
    assert choice(ctypes.byref(rk), 256) == S.PATH_SEMIFUSED
    assert choice(ctypes.byref(rk32), 256) == S.PATH_FUSED          # no entry: the default
    assert S.dispatch_time_us(sc, 200) == pytest.approx(40.0)
    assert S.dispatch_time_us(rk, 200) == pytest.approx(90.0)
    with pytest.raises(S.SpearError):
        S.dispatch_time_us(rk32, 200)
    # the scalar-gate setter writes the scalar-gate entry only
    S.dispatch_set_time(4096, 4096, 64, 0, 256, S.PATH_UNFUSED, 55.0)
    assert S.dispatch_time_us(sc, 256) == pytest.approx(55.0)
    assert S.dispatch_time_us(rk, 256) == pytest.approx(90.0)
    arr = (ctypes.POINTER(S.LayerStruct) * 1)
    out, pred = ctypes.c_int(-1), ctypes.c_float(-1.0)
    chunks = (ctypes.c_int * 1)(256)
    rc = S.F["spear_slo_chunk"](arr(ctypes.pointer(sc)), 1, 0, 60.0, 0.0, chunks, 1, ctypes.byref(out),
                                ctypes.byref(pred))
    assert rc == S.OK and out.value == 256 and pred.value == pytest.approx(55.0)
    rc = S.F["spear_slo_chunk"](arr(ctypes.pointer(rk)), 1, 0, 60.0, 0.0, chunks, 1, ctypes.byref(out),
                                ctypes.byref(pred))
    assert rc == S.OK and out.value == 0                          # 90 us does not fit 60 us
    # the gate fields survive a save and load
    p = str(tmp_path / "lut.txt")
    S.dispatch_save(p)
    S.dispatch_clear()
    S.dispatch_load(p)
    assert S.dispatch_time_us(rk, 256) == pytest.approx(90.0)
    assert S.dispatch_time_us(sc, 256) == pytest.approx(55.0)
    S.dispatch_clear()


def test_timeout_injection_validates_its_arguments(S):
    assert S.F["spear_test_inject_timeout"](3, 1000) == S.ERR_INVALID_ARG
    assert S.F["spear_test_inject_timeout"](1, 0) == S.ERR_INVALID_ARG
    assert S.F["spear_test_inject_timeout"](-1, 1000) == S.ERR_INVALID_ARG
    assert S.F["spear_test_inject_timeout"](0, 0) == S.OK


def test_dispatch_table_from_another_device_is_refused(S, tmp_path):
    S.dispatch_clear()
    sc = _layer(S, K=4096, N=4096, r=64)
    S.dispatch_set_layer(sc, 64, S.PATH_FUSED, 30.0)
    p = tmp_path / "lut.txt"
    S.dispatch_save(str(p))
    lines = p.read_text().splitlines()
    assert lines[0].startswith("# spear dispatch table v3 sms=")
    S.dispatch_clear()
    S.dispatch_load(str(p))                                       # same device: accepted
    assert S.dispatch_time_us(sc, 64) == pytest.approx(30.0)
    S.dispatch_clear()
    other = tmp_path / "other.txt"
    other.write_text("# spear dispatch table v3 sms=7 device=Some Other GPU\n" + "\n".join(lines[1:]) + "\n")
    with pytest.raises(S.SpearError):
        S.dispatch_load(str(other))
    assert "Some Other GPU" in S.F["spear_last_error"]().decode()
    with pytest.raises(S.SpearError):                              # nothing was loaded
        S.dispatch_time_us(sc, 64)
    S.dispatch_clear()


def _brute_slo(times, decode, slo, overhead, chunks):
    """Enumerate every candidate: predicted = overhead + sum of the layers'
    tabled times at the power-of-two bucket of decode + chunk."""
    fits = []
    for c in chunks:
        M = decode + c
        if M < 1:
            continue
        b = 1
        while b < M:
            b *= 2
        t = overhead + sum(tl[b] for tl in times)
        if t <= slo:
            fits.append((c, t))
    if not fits:
        return 0, -1.0
    c = max(f[0] for f in fits)
    return c, [f[1] for f in fits if f[0] == c][0]


def test_slo_chunk_matches_enumeration(S):
    S.dispatch_clear()
    shapes = [(4096, 4096, 64, 0), (4096, 11008, 64, 0), (11008, 4096, 32, 128)]
    buckets = [1 << i for i in range(13)]
    rng = np.random.default_rng(7)
    times = []
    for (K, N, r, g) in shapes:
        # monotone in M, like a measured latency table
        t = np.cumsum(rng.uniform(0.5, 6.0, len(buckets))) + 5.0
        times.append(dict(zip(buckets, t.tolist())))
        for b, us in zip(buckets, t):
            path = S.PATH_DECODE if b <= 16 else S.PATH_FUSED
            S.dispatch_set_time(K, N, r, g, b, path, float(us))
    layers = [_layer(S, K=K, N=N, r=r, group=g) for (K, N, r, g) in shapes]
    chunks = [0, 16, 48, 64, 128, 256, 500, 1024, 2048]
    for decode in (0, 1, 7, 16, 100):
        for slo in (10.0, 40.0, 80.0, 150.0, 1e6):
            got = S.slo_chunk(layers, decode, slo, chunks, step_overhead_us=3.0)
            want = _brute_slo(times, decode, slo, 3.0, chunks)
            assert got[0] == want[0], (decode, slo, got, want)
            assert got[1] == pytest.approx(want[1], rel=1e-5)
    # the loosest SLO takes the largest candidate, an impossible one takes none
    assert S.slo_chunk(layers, 1, 1e6, chunks)[0] == 2048
    assert S.slo_chunk(layers, 1, 1.0, chunks) == (0, -1.0)
    # a bucket with no measured time is an error, not a guess
    with pytest.raises(S.SpearError):
        S.slo_chunk(layers, 1, 1e6, [8192])
    with pytest.raises(S.SpearError):
        S.slo_chunk(layers, 1, 100.0, [-4])
    S.dispatch_clear()


@pytest.mark.parametrize("kw,code", [
    (dict(gate_kind=2), 1),
    (dict(gate_kind=1, r=0), 1),
    (dict(gate_kind=1, gate_hidden=12), 2),
    (dict(gate_kind=1, gate_hidden=16, gate_w2=None), 1),
    (dict(gate_kind=1, gate_hidden=16, gate_b1=0x8004), 3),
])
def test_rank_gate_validation_before_launch(S, kw, code):
    d = dict(gate_kind=0, gate_hidden=0, gate_w1=0x80000, gate_b1=0x81000, gate_w2=0x82000, gate_b2=0x83000,
             gate_alpha=1.0)
    d.update(kw)
    st = _layer(S, **{k: v for k, v in kw.items() if k == "r"})
    for k in ("gate_kind", "gate_hidden", "gate_w1", "gate_b1", "gate_w2", "gate_b2", "gate_alpha"):
        setattr(st, k, d[k])
    rc = S.F["spear_linear_forward"](ctypes.byref(st), 0x50000, 4, 0x60000, 0x70000, 1 << 30, None, None, None)
    assert rc == code, S.F["spear_last_error"]().decode()
    assert S.F["spear_last_error"]().decode()


def test_binding_struct_and_constants_match_the_header(S, tmp_path):
    """The ctypes mirror of spear_layer has the C layout (every field offset and
    the size, as gcc lays out include/spear.h), and the binding's status, path
    and gate constants equal the header's enumerators."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    fields = [name for name, _ in S.LayerStruct._fields_]
    consts = {"OK": "SPEAR_OK"}
    consts.update({n: "SPEAR_" + n for n in dir(S)
                   if re.fullmatch(r"(ERR|PATH|GATE)_[A-Z_]+", n) and isinstance(getattr(S, n), int)})
    lines = ['#include <stdio.h>', '#include "spear.h"', "int main(void) {",
             '  printf("size %zu\\n", sizeof(spear_layer));']
    lines += [f'  printf("field {f} %zu\\n", offsetof(spear_layer, {f}));' for f in fields]
    lines += [f'  printf("const {py} %d\\n", (int){c});' for py, c in sorted(consts.items())]
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([gcc, "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    # tokens: "size" v, then ("field" | "const") name v triples
    size = int(out[1])
    got = {(out[i], out[i + 1]): int(out[i + 2]) for i in range(2, len(out), 3)}
    assert size == ctypes.sizeof(S.LayerStruct)
    for f in fields:
        assert got[("field", f)] == getattr(S.LayerStruct, f).offset, f
    assert len(consts) >= 14
    for py in consts:
        assert got[("const", py)] == getattr(S, py), py


def _c_kind(decl: str) -> str:
    """Kind of a C parameter or return type as the binding must pass it."""
    d = decl.strip()
    if "*" in d:
        return "ptr"
    t = re.sub(r"\b(const|unsigned|signed)\b", "", d).split()
    base = t[0] if t else ""
    if base == "long" and len(t) > 1 and t[1] == "long":
        return "long long"
    return {"int": "int", "size_t": "size_t", "float": "float", "void": "void"}.get(base, base)


def _ctypes_kind(t) -> str:
    if t is None:
        return "void"
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    return {ctypes.c_int: "int", ctypes.c_size_t: "size_t", ctypes.c_float: "float",
            ctypes.c_longlong: "long long"}.get(t, repr(t))


def test_binding_prototypes_match_the_header(S):
    """Every header function's parameters (count and kind: pointer, int, size_t,
    float) and return kind equal the binding's ctypes prototype."""
    src = open(os.path.join(ROOT, "include", "spear.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    decls = re.findall(r"^\s*((?:const\s+)?[A-Za-z_0-9]+\s*\**)\s*\**\s*(spear_[A-Za-z_0-9]+)\s*\(([^)]*)\)\s*;",
                       src, flags=re.M)
    assert len(decls) == len(_header_functions())
    for ret, name, params in decls:
        # the pointer star may sit with the name ("const char* spear_x(") or the type
        ret_kind = "ptr" if re.search(r"\*\s*" + name, src) or "*" in ret else _c_kind(ret)
        args = [p for p in (x.strip() for x in params.split(",")) if p and p != "void"]
        want = [_c_kind(p) for p in args]
        sig = S.EXPORTS[name]
        got = [_ctypes_kind(t) for t in sig[1:]]
        assert got == want, (name, got, want)
        assert _ctypes_kind(sig[0]) == ret_kind, (name, sig[0], ret)


def test_device_check_build_hooks(S):
    # the normal build reports its checks off; the forced-check hook validates
    # its argument (it has no effect here: no launch runs)
    assert S.F["spear_device_checks_enabled"]() == 0
    assert S.F["spear_test_force_device_check"](3) == S.ERR_INVALID_ARG
    assert S.F["spear_test_force_device_check"](-1) == S.ERR_INVALID_ARG
    assert S.F["spear_test_force_device_check"](0) == S.OK


def test_device_check_build_loads_with_its_variable(S):
    # SPEAR_DEVICE_CHECKS=1 makes the binding load the device-check build,
    # which exports the same symbols and reports its checks on
    import subprocess
    import sys
    from w4_gemm_gated_b200 import build
    build.build(checked=True)
    code = ("from w4_gemm_gated_b200 import spear as S; "
            "print(S.LIB_PATH.endswith('libspear_checked.so'), S.F['spear_device_checks_enabled']())")
    env = dict(os.environ, SPEAR_DEVICE_CHECKS="1", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                         timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.split() == ["True", "1"]


def test_tracing_switch(S):
    # NVTX ranges around the calls: off unless asked; a call traced with no
    # tool attached (and no GPU needed: it fails validation) still behaves
    assert S.F["spear_tracing_enabled"]() == (1 if os.environ.get("SPEAR_NVTX") == "1" else 0)
    try:
        assert S.F["spear_set_tracing"](1) == S.OK
        assert S.F["spear_tracing_enabled"]() == 1
        assert S.F["spear_w4_pack"](None, 16, 64, None, None) == S.ERR_INVALID_ARG
        assert S.F["spear_workspace_init"](None, 0, None) == S.ERR_INVALID_ARG
    finally:
        S.F["spear_set_tracing"](0)
    assert S.F["spear_tracing_enabled"]() == 0
