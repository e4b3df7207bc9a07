"""Helpers shared by the GPU parity tests: build layers on the device, bring the exact
stored values to the host for the oracle, and compare results by the parity rules.

Parity rules (the pages' tolerances for this path):
  * mask bits are compared on the oracle's fp64 logits: bit-exact where |logit| >= 1e-3;
    flips inside that band are counted and reported, not failed;
  * compaction and index lists are bit-exact;
  * FFN outputs: max|y - y_ref| <= 1e-5 max|y_ref| for fp32, <= 1e-2 max|y_ref| for fp16
    and Q4_0 (fp32 accumulation on the device, fp64 in the oracle).
Every oracle input comes from the seeded generator or from the oracle itself; GPU
results are only ever compared, never fed to the oracle.

The oracle used here is the C++ one (oracle/pi_oracle.cpp through oracle/cpp.py): it
reads the generator's stored tensors directly and accumulates in double.
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import numpy as np
import torch

import pi_synth as S
from oracle import cpp as OC
from oracle import ffn as O

BAND = 1e-3


def y_tol(w_dtype: str) -> float:
    return 1e-5 if w_dtype == "f32" else 1e-2


def desc_of(pi, wl: S.Workload):
    return pi.make_desc(wl.d_model, wl.d_ff, wl.rank, wl.act, wl.w_dtype, wl.x_dtype, wl.p_dtype)


def build_layers(pi, wl: S.Workload, n_layers: int | None = None, keep_host: bool = True):
    """Generate layers on cuda, load them into the library; return (gpu layers, synth layers)."""
    n = wl.n_layers if n_layers is None else n_layers
    gl, sl = [], []
    for l in range(n):
        L = S.make_layer(wl, l, "cuda")
        gl.append(pi.load_layer(desc_of(pi, wl.at_layer(l)), L.tensors()))
        sl.append(L if keep_host else None)
    torch.cuda.synchronize()
    return gl, sl


def cpp_layer(L: S.SynthLayer) -> OC.Layer:
    """The whole layer, stored values, for the C++ oracle."""
    return OC.Layer(L.to_numpy(), L.workload.act)


def oracle_logits(L: S.SynthLayer, x: np.ndarray) -> np.ndarray:
    """The C++ oracle's fp64 logits, from the layer's stored predictor only."""
    t = {"p1": L.p1.cpu().numpy(), "p2": L.p2.cpu().numpy(), "thresh": L.thresh.cpu().numpy()}
    return OC.Layer(t, L.workload.act).predictor_logits(x)


def stored_rows(L: S.SynthLayer, rows: np.ndarray) -> Dict[str, np.ndarray]:
    """Stored tensors of the given neuron rows only (subset k = neuron rows[k])."""
    act = L.workload.act
    ri = torch.as_tensor(np.asarray(rows, np.int64), device=L.bias.device)
    t = {"bias": L.bias[ri], "p1": L.p1, "p2": L.p2[:, ri], "thresh": L.thresh[ri]}
    if L.q_up is not None:
        t.update(q_up=L.q_up[ri], s_up=L.s_up[ri], q_down=L.q_down[ri], s_down=L.s_down[ri])
        if act == "reglu":
            t.update(q_gate=L.q_gate[ri], s_gate=L.s_gate[ri])
    else:
        t.update(w_up=L.w_up[ri], w_down=L.w_down[:, ri].contiguous())
        if act == "reglu":
            t["w_gate"] = L.w_gate[ri]
    return {k: v.cpu().numpy() for k, v in t.items()}


def oracle_ffn_rows(x: np.ndarray, L: S.SynthLayer, bits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """The C++ oracle's sparse FFN over `idx` (ascending), computed from those rows only."""
    if len(idx) == 0:
        return np.zeros((np.atleast_2d(x).shape[0], L.workload.d_model))
    sub = OC.Layer(stored_rows(L, idx), L.workload.act)
    return sub.sparse_ffn(x, np.atleast_2d(bits)[:, idx], np.arange(len(idx)))


def mask_parity(logits_ref: np.ndarray, bits_gpu: np.ndarray):
    """(mismatches outside the band, flips inside the band, size of the band)."""
    ref = logits_ref > 0
    out = np.abs(logits_ref) >= BAND
    bad = int(np.count_nonzero((ref != bits_gpu) & out))
    flips = int(np.count_nonzero((ref != bits_gpu) & ~out))
    return bad, flips, int(np.count_nonzero(~out))


def rel_err(y: np.ndarray, y_ref: np.ndarray) -> float:
    scale = float(np.max(np.abs(y_ref))) if y_ref.size else 0.0
    if scale == 0.0:
        return float(np.max(np.abs(y))) if y.size else 0.0
    return float(np.max(np.abs(y - y_ref)) / scale)


def unpack_words(words: torch.Tensor, f: int) -> np.ndarray:
    return O.unpack_mask(words.cpu().numpy().astype(np.uint32), f)


def x_to_np(x: torch.Tensor) -> np.ndarray:
    return x.detach().cpu().double().numpy()


def cpp_layer_as(L: S.SynthLayer, act: str) -> OC.Layer:
    """The layer's stored tensors under another activation family (same weights)."""
    return OC.Layer(L.to_numpy(), act)
