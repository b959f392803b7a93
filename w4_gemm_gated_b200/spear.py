"""ctypes binding of ``libspear.so`` (C ABI in ``include/spear.h``).

Argument marshalling only: every step of the layer runs in the CUDA library.
PyTorch tensors supply device memory and the current CUDA stream.  Importing
this module loads the library and raises ``ImportError`` if it is missing;
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import dataclasses
from dataclasses import dataclass

import torch

# SPEAR_DEVICE_CHECKS=1 loads the device-check build of the same library
# (bounds checks that report SPEAR_ERR_DEVICE_CHECK; built beside it)
_LIB_NAME = "libspear_checked.so" if os.environ.get("SPEAR_DEVICE_CHECKS") == "1" else "libspear.so"
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), _LIB_NAME)
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m w4_gemm_gated_b200.build`")
_lib = ctypes.CDLL(_LIB_PATH)

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_ALIGNMENT = 3
ERR_WORKSPACE = 4
ERR_CUDA = 5
ERR_TIMEOUT = 6
ERR_DEVICE_CHECK = 7

PATH_AUTO = 0
PATH_DECODE = 1
PATH_FUSED = 2
PATH_UNFUSED = 3
PATH_SEMIFUSED = 4
GATE_SCALAR = 0
GATE_RANK_MLP = 1
PATH_NAMES = {PATH_DECODE: "decode", PATH_FUSED: "fused", PATH_UNFUSED: "unfused", PATH_SEMIFUSED: "semifused"}

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
_f = ctypes.c_float


class LayerStruct(ctypes.Structure):
    """Mirror of ``spear_layer``."""

    _fields_ = [
        ("K", _i), ("N", _i), ("group", _i), ("r", _i),
        ("w_packed", _vp), ("scales", _vp), ("AgT", _vp), ("BpT", _vp),
        ("b_g", _f), ("gate_tau", _f),
        ("gate_kind", _i), ("gate_hidden", _i),
        ("gate_w1", _vp), ("gate_b1", _vp), ("gate_w2", _vp), ("gate_b2", _vp),
        ("gate_alpha", _f),
        ("prefetch_next", _vp),
    ]


def _proto(name, restype, *argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = list(argtypes)
    return fn


EXPORTS = {
    "spear_last_error": (ctypes.c_char_p,),
    "spear_status_string": (ctypes.c_char_p, _i),
    "spear_version": (_i,),
    "spear_w4_packed_bytes": (_sz, _i, _i),
    "spear_scale_count": (_sz, _i, _i, _i),
    "spear_w4_quantize": (_i, _vp, _i, _i, _i, _vp, _vp, _vp),
    "spear_w4_pack": (_i, _vp, _i, _i, _vp, _vp),
    "spear_w4_unpack": (_i, _vp, _i, _i, _vp, _vp),
    "spear_ec_prescale_B": (_i, _vp, _vp, _i, _i, _vp, _vp),
    "spear_ec_agt_count": (_sz, _i, _i),
    "spear_ec_bpt_count": (_sz, _i, _i),
    "spear_ec_pack": (_i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp),
    "spear_workspace_bytes": (_sz, ctypes.POINTER(LayerStruct), _i),
    "spear_workspace_init": (_i, _vp, _sz, _vp),
    "spear_linear_forward": (_i, ctypes.POINTER(LayerStruct), _vp, _i, _vp, _vp, _sz, _vp, _vp, _vp),
    "spear_linear_forward_path": (_i, ctypes.POINTER(LayerStruct), _vp, _i, _vp, _vp, _sz, _vp, _vp, _i, _vp),
    "spear_read_status": (_i, _vp, ctypes.POINTER(_i), _vp),
    "spear_linear_forward_decode_noalloc": (_i, ctypes.POINTER(LayerStruct), _vp, _i, _vp, _vp, _vp, _vp),
    "spear_read_status_noalloc": (_i, ctypes.POINTER(_i), _vp),
    "spear_test_inject_timeout": (_i, _i, ctypes.c_longlong),
    "spear_device_checks_enabled": (_i,),
    "spear_set_tracing": (_i, _i),
    "spear_tracing_enabled": (_i,),
    "spear_test_force_device_check": (_i, _i),
    "spear_dispatch_choice": (_i, ctypes.POINTER(LayerStruct), _i),
    "spear_dispatch_tune": (_i, ctypes.POINTER(LayerStruct), ctypes.POINTER(_i), _i, _vp, _vp, _vp, _sz, _vp, _sz,
                            _i, ctypes.POINTER(_f), _vp),
    "spear_dispatch_set": (_i, _i, _i, _i, _i, _i, _i),
    "spear_dispatch_set_time": (_i, _i, _i, _i, _i, _i, _i, _f),
    "spear_dispatch_set_layer": (_i, ctypes.POINTER(LayerStruct), _i, _i, _f),
    "spear_dispatch_time_us": (_i, ctypes.POINTER(LayerStruct), _i, ctypes.POINTER(_f)),
    "spear_dispatch_clear": (None,),
    "spear_dispatch_save": (_i, ctypes.c_char_p),
    "spear_dispatch_load": (_i, ctypes.c_char_p),
    "spear_slo_chunk": (_i, ctypes.POINTER(ctypes.POINTER(LayerStruct)), _i, _i, _f, _f, ctypes.POINTER(_i), _i,
                        ctypes.POINTER(_i), ctypes.POINTER(_f)),
}

F = {name: _proto(name, sig[0], *sig[1:]) for name, sig in EXPORTS.items()}
LIB_PATH = _LIB_PATH


class SpearError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{F['spear_status_string'](status).decode()}: {msg}")
        self.status = status


def _check(rc: int) -> None:
    if rc != OK:
        raise SpearError(rc, F["spear_last_error"]().decode())


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream: torch.cuda.Stream | None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def version() -> int:
    return F["spear_version"]()


# --------------------------------------------------------------------------
# one-off layer preparation
# --------------------------------------------------------------------------

def quantize(W: torch.Tensor, group: int = 0, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """W (K x N fp32, device) -> codes q (N x K int8) and fp16 scales."""
    K, N = W.shape
    q = torch.empty((N, K), dtype=torch.int8, device=W.device)
    ns = F["spear_scale_count"](N, K, group)
    if ns == 0:
        raise SpearError(ERR_UNSUPPORTED_SHAPE, f"bad shape K={K} N={N} group={group}")
    s = torch.empty(ns if group == 0 else (K // 128, N), dtype=torch.float16, device=W.device)
    _check(F["spear_w4_quantize"](_ptr(W), K, N, group, _ptr(q), _ptr(s), _stream(stream)))
    return q, s


def pack(q: torch.Tensor, stream=None) -> torch.Tensor:
    N, K = q.shape
    out = torch.empty(N * K // 2, dtype=torch.uint8, device=q.device)
    _check(F["spear_w4_pack"](_ptr(q), N, K, _ptr(out), _stream(stream)))
    return out


def unpack(packed: torch.Tensor, N: int, K: int, stream=None) -> torch.Tensor:
    q = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    _check(F["spear_w4_unpack"](_ptr(packed), N, K, _ptr(q), _stream(stream)))
    return q


def prescale_B(B: torch.Tensor, s: torch.Tensor, stream=None) -> torch.Tensor:
    r, N = B.shape
    out = torch.empty_like(B)
    _check(F["spear_ec_prescale_B"](_ptr(B), _ptr(s), r, N, _ptr(out), _stream(stream)))
    return out


def ec_pack(A: torch.Tensor, B: torch.Tensor, w_g: torch.Tensor, s: torch.Tensor, group: int,
            stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    K, r = A.shape
    N = B.shape[1]
    AgT = torch.empty((r + 1, K), dtype=torch.bfloat16, device=A.device)
    BpT = torch.empty((N, r), dtype=torch.bfloat16, device=A.device)
    _check(F["spear_ec_pack"](_ptr(A), _ptr(B), _ptr(w_g), _ptr(s), K, N, r, group, _ptr(AgT), _ptr(BpT),
                              _stream(stream)))
    return AgT, BpT


@dataclass
class Layer:
    """Device-resident prepared layer (keeps its tensors alive)."""

    K: int
    N: int
    group: int
    r: int
    w_packed: torch.Tensor
    scales: torch.Tensor
    AgT: torch.Tensor | None
    BpT: torch.Tensor | None
    b_g: float
    gate_tau: float = 0.1
    # the pages' per-rank gate gamma(t) = sigmoid(W2 relu(W1 t + b1) + b2) (fp32 device tensors)
    gate_kind: int = GATE_SCALAR
    gate_w1: torch.Tensor | None = None   # h x r
    gate_b1: torch.Tensor | None = None   # h
    gate_w2: torch.Tensor | None = None   # r x h
    gate_b2: torch.Tensor | None = None   # r
    gate_alpha: float = 1.0

    def struct(self) -> LayerStruct:
        rank = self.gate_kind == GATE_RANK_MLP
        return LayerStruct(self.K, self.N, self.group, self.r, _ptr(self.w_packed), _ptr(self.scales),
                           _ptr(self.AgT) if self.AgT is not None else None,
                           _ptr(self.BpT) if self.BpT is not None else None,
                           float(self.b_g), float(self.gate_tau),
                           int(self.gate_kind), int(self.gate_w1.shape[0]) if rank else 0,
                           _ptr(self.gate_w1) if rank else None, _ptr(self.gate_b1) if rank else None,
                           _ptr(self.gate_w2) if rank else None, _ptr(self.gate_b2) if rank else None,
                           float(self.gate_alpha))


def with_rank_gate(layer: Layer, W1: torch.Tensor, b1: torch.Tensor, W2: torch.Tensor, b2: torch.Tensor,
                   alpha: float) -> Layer:
    """The same prepared layer with the pages' per-rank gate instead of the scalar one
    (parameters copied to contiguous fp32 device tensors)."""
    dev = layer.w_packed.device

    def f32(t):
        return t.detach().to(device=dev, dtype=torch.float32).contiguous()

    return dataclasses.replace(layer, gate_kind=GATE_RANK_MLP, gate_w1=f32(W1), gate_b1=f32(b1),
                               gate_w2=f32(W2), gate_b2=f32(b2), gate_alpha=float(alpha))


def prepare_layer(W: torch.Tensor, group: int, A: torch.Tensor | None, B: torch.Tensor | None,
                  w_g: torch.Tensor | None, b_g: float, gate_tau: float = 0.1, stream=None) -> Layer:
    """Quantise, pack and lay out one layer on the device (all steps in CUDA)."""
    K, N = W.shape
    q, s = quantize(W, group, stream)
    w_packed = pack(q, stream)
    del q
    if A is not None:
        AgT, BpT = ec_pack(A, B, w_g, s, group, stream)
        r = A.shape[1]
    else:
        AgT = BpT = None
        r = 0
    return Layer(K, N, group, r, w_packed, s, AgT, BpT, b_g, gate_tau)


def layer_from_parts(K: int, N: int, group: int, w_packed: torch.Tensor, scales: torch.Tensor,
                     AgT: torch.Tensor | None, BpT: torch.Tensor | None, b_g: float,
                     gate_tau: float = 0.1) -> Layer:
    r = 0 if AgT is None else AgT.shape[0] - 1
    return Layer(K, N, group, r, w_packed, scales, AgT, BpT, b_g, gate_tau)


# --------------------------------------------------------------------------
# forward
# --------------------------------------------------------------------------

def workspace_bytes(layer: Layer, M_max: int) -> int:
    st = layer.struct()
    n = F["spear_workspace_bytes"](ctypes.byref(st), M_max)
    if n == 0:
        raise SpearError(ERR_INVALID_ARG, "spear_workspace_bytes rejected the layer / M_max")
    return n


def make_workspace(layer: Layer, M_max: int, device=None, stream=None) -> torch.Tensor:
    n = workspace_bytes(layer, M_max)
    ws = torch.empty(n, dtype=torch.uint8, device=device or layer.w_packed.device)
    _check(F["spear_workspace_init"](_ptr(ws), n, _stream(stream)))
    return ws


def forward(layer: Layer, x: torch.Tensor, ws: torch.Tensor, y: torch.Tensor | None = None,
            gate_out: torch.Tensor | None = None, mask_count: torch.Tensor | None = None,
            path: int = PATH_AUTO, stream=None, prefetch_next: Layer | None = None) -> torch.Tensor:
    """y = x . dequant(W4) + g * ((x . A) . B) for x (M x K bf16) on the device.
    prefetch_next: the layer the next call on this stream runs (an L2 warm-up hint)."""
    M, K = x.shape
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bf16")
    if y is None:
        y = torch.empty((M, layer.N), dtype=torch.bfloat16, device=x.device)
    st = layer.struct()
    nxt = None
    if prefetch_next is not None:
        nxt = prefetch_next.struct()   # kept alive until the call returns
        st.prefetch_next = ctypes.addressof(nxt)
    _check(F["spear_linear_forward_path"](ctypes.byref(st), _ptr(x), M, _ptr(y), _ptr(ws), ws.numel(),
                                          _ptr(gate_out), _ptr(mask_count), path, _stream(stream)))
    return y


def forward_decode_noalloc(layer: Layer, x: torch.Tensor, y: torch.Tensor | None = None,
                           gate_out: torch.Tensor | None = None, mask_count: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """Decode-path layer call for M <= 16 that allocates no device memory: its
    scratch is a fixed array inside the library (shared by all calls on a
    device, so calls must not overlap on the GPU)."""
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, layer.N), dtype=torch.bfloat16, device=x.device)
    st = layer.struct()
    _check(F["spear_linear_forward_decode_noalloc"](ctypes.byref(st), _ptr(x), M, _ptr(y), _ptr(gate_out),
                                                    _ptr(mask_count), _stream(stream)))
    return y


def read_status(ws: torch.Tensor, stream=None) -> int:
    v = _i(0)
    _check(F["spear_read_status"](_ptr(ws), ctypes.byref(v), _stream(stream)))
    return v.value


def test_inject_timeout(kernel: int, wait_cycles: int = 0) -> None:
    """Failure injection for tests: make one bounded device wait of the decode
    (kernel=1) or tensor-core (kernel=2) kernel expire after wait_cycles SM
    cycles in the launches that follow; kernel=0 turns it off."""
    _check(F["spear_test_inject_timeout"](kernel, wait_cycles))


def read_status_noalloc(stream=None) -> int:
    """Read and clear the status word of the allocation-free call's array."""
    v = _i(0)
    _check(F["spear_read_status_noalloc"](ctypes.byref(v), _stream(stream)))
    return v.value


# --------------------------------------------------------------------------
# dispatcher
# --------------------------------------------------------------------------

def dispatch_choice(layer: Layer, M: int) -> int:
    st = layer.struct()
    return F["spear_dispatch_choice"](ctypes.byref(st), M)


def dispatch_tune(layer: Layer, Ms: list[int], x: torch.Tensor, y: torch.Tensor, ws: torch.Tensor,
                  flush: torch.Tensor | None = None, reps: int = 20, stream=None) -> list[tuple[float, ...]]:
    """Median microseconds per M of (DECODE, FUSED, UNFUSED, SEMIFUSED), -1 where not run."""
    st = layer.struct()
    arr = (_i * len(Ms))(*Ms)
    times = (_f * (4 * len(Ms)))()
    _check(F["spear_dispatch_tune"](ctypes.byref(st), arr, len(Ms), _ptr(x), _ptr(y), _ptr(ws), ws.numel(),
                                    _ptr(flush), 0 if flush is None else flush.numel() * flush.element_size(),
                                    reps, times, _stream(stream)))
    return [tuple(times[4 * i + j] for j in range(4)) for i in range(len(Ms))]


def dispatch_set(K: int, N: int, r: int, group: int, M: int, path: int) -> None:
    _check(F["spear_dispatch_set"](K, N, r, group, M, path))


def dispatch_set_time(K: int, N: int, r: int, group: int, M: int, path: int, us: float) -> None:
    _check(F["spear_dispatch_set_time"](K, N, r, group, M, path, us))


def dispatch_set_layer(layer, M: int, path: int, us: float = -1.0) -> None:
    """Set the table entry of this layer's full key (shape, scale kind, gate form)."""
    st = layer if isinstance(layer, LayerStruct) else layer.struct()
    _check(F["spear_dispatch_set_layer"](ctypes.byref(st), M, path, us))


def dispatch_time_us(layer, M: int) -> float:
    st = layer.struct() if hasattr(layer, "struct") else layer
    out = _f()
    _check(F["spear_dispatch_time_us"](ctypes.byref(st), M, ctypes.byref(out)))
    return float(out.value)


def slo_chunk(layers: list, decode_tokens: int, slo_us: float, chunks: list[int],
              step_overhead_us: float = 0.0) -> tuple[int, float]:
    """Largest candidate prefill chunk whose predicted step time (overhead plus
    every layer's tabled time at M = decode_tokens + chunk) meets ``slo_us``;
    returns (chunk, predicted_us), (0, -1) if none fits."""
    structs = [l.struct() if hasattr(l, "struct") else l for l in layers]
    ptrs = (ctypes.POINTER(LayerStruct) * len(structs))(*[ctypes.pointer(s) for s in structs])
    arr = (_i * len(chunks))(*chunks)
    out, pred = _i(), _f()
    _check(F["spear_slo_chunk"](ptrs, len(structs), decode_tokens, slo_us, step_overhead_us, arr, len(chunks),
                                ctypes.byref(out), ctypes.byref(pred)))
    return int(out.value), float(pred.value)


def dispatch_clear() -> None:
    F["spear_dispatch_clear"]()


def dispatch_save(path: str) -> None:
    _check(F["spear_dispatch_save"](path.encode()))


def dispatch_load(path: str) -> None:
    _check(F["spear_dispatch_load"](path.encode()))
