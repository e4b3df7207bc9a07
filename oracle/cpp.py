"""Binding of the C++ oracle (oracle/pi_oracle.cpp): TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the benchmark's CPU-baseline leg may use
it.  The arithmetic is all in the C++ file (plain loops, double accumulation); this
module only passes the generator's stored tensors (fp32, fp16 bit patterns, Q4_0
nibble and scale planes) to it as host buffers and shapes the results.  It never
loads the CUDA library.

`build()` compiles the oracle with g++ into oracle/libpi_oracle.so (OpenMP over
independent outputs only, so results do not depend on the thread count; no FMA
contraction, so every product and sum is rounded as written).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Dict, List, Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pi_oracle.cpp")
LIB = os.path.join(HERE, "libpi_oracle.so")
FLAGS = ["-O2", "-std=c++17", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

ACT = {"relu": 0, "reglu": 1, "relu2": 2}
DT = {"f32": 0, "f16": 1, "q4_0": 2}


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp"
        subprocess.run(["g++", *FLAGS, "-o", tmp, SRC], check=True)
        os.replace(tmp, LIB)
    return LIB


class _Layer(C.Structure):
    _fields_ = [("d", C.c_int), ("f", C.c_int), ("r", C.c_int), ("act", C.c_int), ("w_dtype", C.c_int),
                ("p_dtype", C.c_int),
                ("w_up", C.c_void_p), ("w_gate", C.c_void_p), ("w_down", C.c_void_p),
                ("s_up", C.c_void_p), ("s_gate", C.c_void_p), ("s_down", C.c_void_p),
                ("bias", C.c_void_p), ("p1", C.c_void_p), ("p2", C.c_void_p), ("thresh", C.c_void_p)]


_lib = None
_lib_path = None   # another build of the oracle source (the tests' planted mistakes), or None


def use_library(path: Optional[str]) -> None:
    """Bind the following calls to the oracle library at `path` (None: the default)."""
    global _lib, _lib_path
    _lib, _lib_path = None, path


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(_lib_path or build())
        P, I, D = C.c_void_p, C.c_int, C.c_double
        L.pio_half_to_double.argtypes, L.pio_half_to_double.restype = [C.c_uint16], D
        L.pio_float_to_half.argtypes, L.pio_float_to_half.restype = [C.c_float], C.c_uint16
        L.pio_set_threads.argtypes, L.pio_set_threads.restype = [I], None
        L.pio_max_threads.argtypes, L.pio_max_threads.restype = [], I
        L.pio_predict.argtypes, L.pio_predict.restype = [P, I, P, P], I
        L.pio_pack_mask.argtypes, L.pio_pack_mask.restype = [P, I, I, P], None
        L.pio_compact.argtypes, L.pio_compact.restype = [P, I, I, P], I
        L.pio_sparse_ffn.argtypes, L.pio_sparse_ffn.restype = [P, I, P, P, P, I, P], I
        L.pio_dense_ffn.argtypes, L.pio_dense_ffn.restype = [P, I, P, P], I
        L.pio_glue.argtypes, L.pio_glue.restype = [I, I, P, P, I, P], None
        L.pio_true_mask.argtypes, L.pio_true_mask.restype = [P, I, P, P], I
        L.pio_layer_step.argtypes, L.pio_layer_step.restype = [P, I, P, I, P, P, P, P, P, P], I
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _x(x) -> np.ndarray:
    return np.ascontiguousarray(np.atleast_2d(np.asarray(x, np.float64)))


class Layer:
    """One layer in its stored formats (the generator's `to_numpy()` dict).  A dict with
    only p1, p2, thresh (and bias) gives a predictor-only layer: predictor_logits works,
    the FFN calls do not."""

    def __init__(self, t: Dict[str, np.ndarray], act: str):
        self.keep = {}
        q4 = "q_up" in t
        pred_only = not q4 and "w_up" not in t

        def buf(name, dtype=None):
            if name not in t or t[name] is None:
                return None
            a = np.ascontiguousarray(t[name])
            if dtype is not None:
                a = np.ascontiguousarray(a.view(dtype) if a.dtype.itemsize == np.dtype(dtype).itemsize else a.astype(dtype))
            self.keep[name] = a
            return a

        def fp(name):
            a = buf(name)
            if a is None:
                return None
            if a.dtype == np.float16:
                a = a.view(np.uint16)
                self.keep[name] = a
            return a

        if q4:
            up, gate, down = buf("q_up", np.uint8), buf("q_gate", np.uint8), buf("q_down", np.uint8)
            s_up, s_gate, s_down = (buf(k) for k in ("s_up", "s_gate", "s_down"))
            s_up, s_gate, s_down = (None if s is None else s.view(np.uint16) for s in (s_up, s_gate, s_down))
            for k, s in (("s_up", s_up), ("s_gate", s_gate), ("s_down", s_down)):
                self.keep[k] = s
            w_dtype = "q4_0"
            f = up.shape[0]
            d = up.shape[1] * 32
        elif pred_only:
            up = gate = down = s_up = s_gate = s_down = None
            w_dtype = "f16" if t["p1"].dtype == np.float16 else "f32"
            d, f = t["p1"].shape[0], t["p2"].shape[1]
        else:
            up, gate, down = fp("w_up"), fp("w_gate"), fp("w_down")
            s_up = s_gate = s_down = None
            w_dtype = "f16" if t["w_up"].dtype == np.float16 else "f32"
            f, d = up.shape
        p1, p2 = fp("p1"), fp("p2")
        p_dtype = "f16" if t["p1"].dtype == np.float16 else "f32"
        bias = buf("bias", np.float32) if "bias" in t else np.zeros(f, np.float32)
        self.keep["bias"] = bias
        thresh = buf("thresh", np.float32)
        self.pred_only = pred_only
        if not pred_only and (act == "reglu") != (gate is not None):
            raise ValueError("ReGLU needs a gate matrix; ReLU and squared ReLU have none")
        self.d, self.f, self.r, self.act = d, f, p1.shape[1], act
        self.s = _Layer(d, f, self.r, ACT[act], DT[w_dtype], DT[p_dtype], _p(up), _p(gate), _p(down),
                        _p(s_up), _p(s_gate), _p(s_down), _p(bias), _p(p1), _p(p2), _p(thresh))

    # ------------------------------------------------------------------ operations
    def predictor_logits(self, x) -> np.ndarray:
        x = _x(x)
        B = x.shape[0]
        out = np.empty((B, self.f), np.float64)
        lib().pio_predict(C.byref(self.s), B, _p(x), _p(out))
        return out

    def _ffn_check(self):
        if self.pred_only:
            raise ValueError("a predictor-only layer has no FFN weights")

    def true_mask(self, x) -> np.ndarray:
        """[B, f] bools: the firing pre-activation is > 0."""
        self._ffn_check()
        x = _x(x)
        out = np.empty((x.shape[0], self.f), np.uint8)
        lib().pio_true_mask(C.byref(self.s), x.shape[0], _p(x), _p(out))
        return out.astype(bool)

    def sparse_ffn(self, x, masks, idx) -> np.ndarray:
        self._ffn_check()
        x = _x(x)
        B = x.shape[0]
        m = np.ascontiguousarray(np.atleast_2d(np.asarray(masks, bool)).astype(np.uint8))
        ix = np.ascontiguousarray(np.asarray(idx, np.int32))
        y = np.empty((B, self.d), np.float64)
        lib().pio_sparse_ffn(C.byref(self.s), B, _p(x), _p(m), _p(ix), int(ix.size), _p(y))
        return y

    def dense_ffn(self, x) -> np.ndarray:
        self._ffn_check()
        x = _x(x)
        y = np.empty((x.shape[0], self.d), np.float64)
        lib().pio_dense_ffn(C.byref(self.s), x.shape[0], _p(x), _p(y))
        return y

    def layer_step(self, x, x_dtype: str) -> dict:
        self._ffn_check()
        x = _x(x)
        B, f, d = x.shape[0], self.f, self.d
        logits = np.empty((B, f), np.float64)
        words = np.empty((B, f // 32), np.uint32)
        idx = np.empty(f, np.int32)
        count = C.c_int(0)
        y = np.empty((B, d), np.float64)
        xn = np.empty((B, d), np.float64)
        lib().pio_layer_step(C.byref(self.s), B, _p(x), {"f32": 0, "f16": 1}[x_dtype], _p(logits), _p(words),
                             _p(idx), C.byref(count), _p(y), _p(xn))
        n = count.value
        bits = ((words[:, np.arange(f) // 32] >> (np.arange(f) % 32).astype(np.uint32)) & 1).astype(bool)
        return {"logits": logits, "bits": bits, "words": words, "idx": idx[:n].copy(), "count": n,
                "y": y, "x_next": xn.astype(np.float32 if x_dtype == "f32" else np.float16)}


def compact(words, f: int):
    w = np.ascontiguousarray(np.atleast_2d(np.asarray(words, np.uint32)))
    idx = np.empty(f, np.int32)
    n = lib().pio_compact(_p(w), w.shape[0], f, _p(idx))
    return idx[:n].copy(), int(n)


def stack_glue(x, y, x_dtype: Optional[str]) -> np.ndarray:
    """x_dtype "f32" / "f16" rounds the result; None leaves it in double."""
    x, y = _x(x), _x(y)
    out = np.empty_like(x)
    lib().pio_glue(x.shape[0], x.shape[1], _p(x), _p(y), {"f32": 0, "f16": 1, None: -1}[x_dtype], _p(out))
    if x_dtype == "f32":
        return out.astype(np.float32)
    if x_dtype == "f16":
        return out.astype(np.float16)
    return out


def decode_stack(x0, layers: List[Layer], x_dtype: str) -> List[dict]:
    """Run x0 [B, d] through every layer; one trace record per layer."""
    x = _x(x0)
    trace = []
    for L in layers:
        rec = L.layer_step(x, x_dtype)
        rec["x_in"] = x
        trace.append(rec)
        x = rec["x_next"].astype(np.float64)
    return trace


def half_to_double(h: int) -> float:
    return lib().pio_half_to_double(h)


def float_to_half_bits(v: float) -> int:
    return lib().pio_float_to_half(v)


def set_threads(n: int) -> None:
    lib().pio_set_threads(n)


def max_threads() -> int:
    return lib().pio_max_threads()
