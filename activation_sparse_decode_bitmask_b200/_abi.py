"""ctypes binding of libpi.so: argument marshalling only.

Every step of the hot path runs in the library's CUDA kernels; this module turns torch
tensors into device pointers and the current torch stream into a cudaStream_t.  If the
library is missing, importing this module raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, byref, c_int, c_int32, c_longlong, c_uint32, c_ulonglong, c_void_p
from typing import Dict, Optional, Sequence

import torch

from . import _build

PI_F32, PI_F16, PI_Q4_0 = 0, 1, 2
PI_RELU, PI_REGLU, PI_RELU2 = 0, 1, 2
PI_MAX_BATCH = 32
PI_NOALLOC_SCRATCH_BYTES = 256 * 1024
DIAG_SLOTS = 64   # diagnostic stamps per block and layer

STATUS = {0: "PI_OK", 1: "PI_ERR_ARG", 2: "PI_ERR_UNSUPPORTED", 3: "PI_ERR_OOM", 4: "PI_ERR_CUDA",
          5: "PI_ERR_TIMEOUT", 6: "PI_ERR_DEVICE"}

# every entry point the header declares, in declaration order
EXPORTS = ["pi_load_layer", "pi_reorder_hot_prefix", "pi_get_perm", "pi_layer_get_desc", "pi_free_layer",
           "pi_workspace_create", "pi_workspace_free", "pi_stream_status", "pi_workspace_active_total",
           "pi_workspace_layer_counts", "pi_diag_phase_clocks_enable", "pi_diag_phase_clocks_read",
           "pi_device_grid", "pi_diag_barrier_timeout", "pi_predict", "pi_predict_noalloc", "pi_compact_active",
           "pi_sparse_ffn", "pi_decode_stack", "pi_decode_stack_host", "pi_status_str", "pi_abi_version",
           "pi_kernel_launches"]


class PiError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_lib.pi_status_str(status).decode()})")


class LayerDesc(ctypes.Structure):
    _fields_ = [("d_model", c_int), ("d_ff", c_int), ("rank", c_int), ("act", c_int),
                ("w_dtype", c_int), ("x_dtype", c_int), ("p_dtype", c_int)]


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("w_up", "w_gate", "w_down", "s_up", "s_gate", "s_down",
                                        "bias", "p1", "p2", "thresh")]


class Trace(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ("x", "logits", "mask", "idx", "count", "y")]


def _load() -> ctypes.CDLL:
    if not os.path.exists(_build.LIB):
        raise ImportError(f"{_build.LIB} is not built; run __graft_entry__.build() (nvcc, sm_100a)")
    lib = ctypes.CDLL(_build.LIB)
    vp, i = c_void_p, c_int
    sig = {
        "pi_load_layer": (i, [POINTER(LayerDesc), POINTER(LayerWeights), vp, POINTER(vp)]),
        "pi_reorder_hot_prefix": (i, [vp, vp, i, vp]),
        "pi_get_perm": (i, [vp, vp, vp]),
        "pi_layer_get_desc": (i, [vp, POINTER(LayerDesc)]),
        "pi_free_layer": (None, [vp]),
        "pi_workspace_create": (i, [i, i, i, i, i, POINTER(vp)]),
        "pi_workspace_free": (None, [vp]),
        "pi_stream_status": (i, [vp, vp]),
        "pi_workspace_active_total": (i, [vp, POINTER(c_ulonglong)]),
        "pi_workspace_layer_counts": (i, [vp, vp, i]),
        "pi_diag_barrier_timeout": (i, [vp, c_longlong, vp]),
        "pi_diag_phase_clocks_enable": (i, [vp, i]),
        "pi_diag_phase_clocks_read": (i, [vp, vp, ctypes.c_size_t]),
        "pi_device_grid": (i, [vp]),
        "pi_predict": (i, [vp, vp, i, vp, vp, vp, vp]),
        "pi_predict_noalloc": (i, [vp, vp, i, vp, vp, vp, vp]),
        "pi_compact_active": (i, [vp, i, i, vp, vp, vp]),
        "pi_sparse_ffn": (i, [vp, vp, i, vp, vp, vp, vp, vp, vp]),
        "pi_decode_stack": (i, [vp, i, vp, i, POINTER(Trace), vp, vp]),
        "pi_decode_stack_host": (i, [vp, i, vp, vp, i, vp, vp]),
        "pi_status_str": (ctypes.c_char_p, [i]),
        "pi_abi_version": (i, []),
        "pi_kernel_launches": (ctypes.c_ulonglong, []),
    }
    for name, (res, args) in sig.items():
        try:
            fn = getattr(lib, name)
        except AttributeError as e:
            raise ImportError(f"{_build.LIB} lacks {name}; rebuild it with __graft_entry__.build()") from e
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib() -> ctypes.CDLL:
    return _lib


def _check(st: int, what: str) -> None:
    if st != 0:
        raise PiError(st, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


_DT = {"f32": PI_F32, "f16": PI_F16, "q4_0": PI_Q4_0}
_ACT = {"relu": PI_RELU, "reglu": PI_REGLU, "relu2": PI_RELU2}


def make_desc(d_model: int, d_ff: int, rank: int, act: str, w_dtype: str, x_dtype: str,
              p_dtype: str) -> LayerDesc:
    return LayerDesc(d_model, d_ff, rank, _ACT[act], _DT[w_dtype], _DT[x_dtype], _DT[p_dtype])


class Layer:
    """A library-owned layer (pi_layer*)."""

    def __init__(self, handle: int, desc: LayerDesc):
        self.handle = c_void_p(handle)
        self.desc = desc

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            _lib.pi_free_layer(h)
            self.handle = c_void_p(None)

    free = __del__


class Workspace:
    """Library-owned scratch (pi_workspace*)."""

    def __init__(self, d_max: int, f_max: int, r_max: int, B_max: int = 1, L_max: int = 1):
        h = c_void_p()
        _check(_lib.pi_workspace_create(d_max, f_max, r_max, B_max, L_max, byref(h)), "pi_workspace_create")
        self.handle = h

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value:
            _lib.pi_workspace_free(h)
            self.handle = c_void_p(None)

    free = __del__

    def status(self, stream=None) -> int:
        return _lib.pi_stream_status(self.handle, c_void_p(_stream(stream)))

    def active_total(self) -> int:
        v = c_ulonglong()
        _check(_lib.pi_workspace_active_total(self.handle, byref(v)), "pi_workspace_active_total")
        return int(v.value)

    def grid(self) -> int:
        return _lib.pi_device_grid(self.handle)

    def phase_clocks(self, on=True) -> None:
        """on: False/0 off, True/1 SM cycle stamps, 2 global-timer nanosecond stamps."""
        _check(_lib.pi_diag_phase_clocks_enable(self.handle, int(on)), "pi_diag_phase_clocks_enable")

    def read_phase_clocks(self, L_max: int):
        """[grid, L_max, 20] int64 SM cycle stamps of the last stack call."""
        import numpy as np
        g = self.grid()
        out = np.zeros((g, L_max, DIAG_SLOTS), dtype=np.int64)
        _check(_lib.pi_diag_phase_clocks_read(self.handle, out.ctypes.data, out.size), "pi_diag_phase_clocks_read")
        return out

    def layer_counts(self, L: int):
        out = (c_int32 * L)()
        _check(_lib.pi_workspace_layer_counts(self.handle, out, L), "pi_workspace_layer_counts")
        return list(out)


def load_layer(desc: LayerDesc, t: Dict[str, torch.Tensor], stream=None) -> Layer:
    """pi_load_layer from device tensors named like pi_synth's layers: w_up, w_gate, w_down
    (fp32/fp16) or q_up/s_up, q_gate/s_gate, q_down/s_down (Q4_0), bias, p1, p2, thresh."""
    w = LayerWeights()
    if "q_up" in t:
        w.w_up, w.s_up = _ptr(t["q_up"]), _ptr(t["s_up"])
        w.w_gate, w.s_gate = _ptr(t.get("q_gate")), _ptr(t.get("s_gate"))
        w.w_down, w.s_down = _ptr(t["q_down"]), _ptr(t["s_down"])
    else:
        w.w_up, w.w_gate, w.w_down = _ptr(t["w_up"]), _ptr(t.get("w_gate")), _ptr(t["w_down"])
    w.bias, w.p1, w.p2, w.thresh = _ptr(t["bias"]), _ptr(t["p1"]), _ptr(t["p2"]), _ptr(t["thresh"])
    h = c_void_p()
    _check(_lib.pi_load_layer(byref(desc), byref(w), c_void_p(_stream(stream)), byref(h)), "pi_load_layer")
    return Layer(h.value, desc)


def reorder_hot_prefix(layer: Layer, freq: torch.Tensor, hot_count: int = -1, stream=None) -> None:
    _check(_lib.pi_reorder_hot_prefix(layer.handle, _ptr(freq), hot_count, c_void_p(_stream(stream))),
           "pi_reorder_hot_prefix")


def get_perm(layer: Layer, out: torch.Tensor, stream=None) -> torch.Tensor:
    _check(_lib.pi_get_perm(layer.handle, _ptr(out), c_void_p(_stream(stream))), "pi_get_perm")
    return out


def predict(layer: Layer, x: torch.Tensor, B: int, mask: torch.Tensor, logits: Optional[torch.Tensor],
            ws: Workspace, stream=None) -> None:
    _check(_lib.pi_predict(layer.handle, _ptr(x), B, _ptr(mask), _ptr(logits), ws.handle,
                           c_void_p(_stream(stream))), "pi_predict")


def predict_noalloc(layer: Layer, x: torch.Tensor, B: int, mask: torch.Tensor, logits: Optional[torch.Tensor],
                    status: torch.Tensor, stream=None) -> None:
    """pi_predict without a workspace; `status` is a device int32 tensor of one element."""
    _check(_lib.pi_predict_noalloc(layer.handle, _ptr(x), B, _ptr(mask), _ptr(logits), _ptr(status),
                                   c_void_p(_stream(stream))), "pi_predict_noalloc")


def compact_active(mask: torch.Tensor, B: int, d_ff: int, idx: torch.Tensor, count: torch.Tensor,
                   stream=None) -> None:
    _check(_lib.pi_compact_active(_ptr(mask), B, d_ff, _ptr(idx), _ptr(count), c_void_p(_stream(stream))),
           "pi_compact_active")


def sparse_ffn(layer: Layer, x: torch.Tensor, B: int, mask: torch.Tensor, idx: torch.Tensor,
               count: torch.Tensor, y: torch.Tensor, ws: Workspace, stream=None) -> None:
    _check(_lib.pi_sparse_ffn(layer.handle, _ptr(x), B, _ptr(mask), _ptr(idx), _ptr(count), _ptr(y),
                              ws.handle, c_void_p(_stream(stream))), "pi_sparse_ffn")


def _layer_array(layers: Sequence[Layer]):
    arr = (c_void_p * len(layers))()
    for k, L in enumerate(layers):
        arr[k] = L.handle.value
    return arr


def decode_stack(layers: Sequence[Layer], x_inout: torch.Tensor, B: int, ws: Workspace,
                 trace: Optional[Dict[str, torch.Tensor]] = None, stream=None) -> None:
    tr = None
    if trace:
        tr = Trace(*(_ptr(trace.get(n)) for n in ("x", "logits", "mask", "idx", "count", "y")))
    _check(_lib.pi_decode_stack(_layer_array(layers), len(layers), _ptr(x_inout), B,
                                byref(tr) if tr is not None else None, ws.handle, c_void_p(_stream(stream))),
           "pi_decode_stack")


def decode_stack_host(layers: Sequence[Layer], x_host: torch.Tensor, x_out_host: torch.Tensor, B: int,
                      ws: Workspace, stream=None) -> None:
    if x_host.is_cuda or x_out_host.is_cuda:
        raise ValueError("decode_stack_host takes host tensors")
    _check(_lib.pi_decode_stack_host(_layer_array(layers), len(layers), c_void_p(x_host.data_ptr()),
                                     c_void_p(x_out_host.data_ptr()), B, ws.handle, c_void_p(_stream(stream))),
           "pi_decode_stack_host")


def diag_barrier_timeout(ws: Workspace, timeout_ns: int, stream=None) -> None:
    _check(_lib.pi_diag_barrier_timeout(ws.handle, int(timeout_ns), c_void_p(_stream(stream))),
           "pi_diag_barrier_timeout")


def status_str(st: int) -> str:
    return _lib.pi_status_str(st).decode()


def abi_version() -> int:
    return _lib.pi_abi_version()


def kernel_launches() -> int:
    """Kernels this library has launched in this process so far (host-side count)."""
    return int(_lib.pi_kernel_launches())
