"""Seeded synthetic layers and inputs, shared by the oracle tests and the CUDA path.

Everything here builds *inputs*: weights, biases, the fitted low-rank predictor and
its thresholds, firing frequencies and token vectors.  None of the sparse FFN's own
arithmetic (predictor evaluation, masking, compaction, activation, projections) lives
here.  Every random draw comes from a torch generator seeded from
(workload seed, layer, tensor id), so any single layer can be rebuilt on its own.

Readings of what the pages leave open (they give no weights, no predictor
architecture and no training code; unite.ai "PowerInfer: Mesin Inferensi LLM Cepat
dengan GPU Konsumen" §"Prediktor Kepadatan Adaptif" only says a predictor per layer
is trained offline):
  * firing probability of the neuron of rank k: p = min(cap, c * (k+1)^-alpha),
    ranks assigned over a seeded random neuron permutation;
  * bias b_i = ||w_i|| * Phi^-1(p_i) with ||w_i|| of the stored (rounded or
    dequantised) firing row, so P(w_i.x + b_i > 0) = p_i exactly for x ~ N(0, I);
    the bias sits on up for ReLU and on gate for ReGLU, none on down;
  * predictor = linear low-rank map  logit = P2^T (P1^T x) - t:
      - "rrls": reduced-rank least squares (Izenman 1975) of the true
        pre-activation signs on n_calib seeded samples, computed in fp64;
      - "sketch": P1 = a seeded Gaussian sketch Omega (d x r, N(0, 1/d)),
        P2[:, i] = Omega^T w_i scaled to unit logit variance on the calibration
        set, t_i = the empirical (1 - p_i) quantile of the calibration logits;
  * firing frequencies for the hot-neuron sort = the predicted firing rate of each
    neuron over the calibration samples;
  * Q4_0: q ~ U{0..15}, scale = fp16(|N(0, 0.02)|), value = (q - 8) * scale, blocks
    of 32 along d_model; packed with byte j of a block holding element j in its low
    nibble and element j + 16 in its high nibble; nibbles and scales kept in separate
    planes.  Down weights in Q4_0 are given neuron-major ([d_ff][d_model/32] blocks),
    the axis the blocks run along.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

from .workloads import Workload

_TORCH_DT = {"f32": torch.float32, "f16": torch.float16}

# tensor ids for the seed key
_T_PERM, _T_UP, _T_GATE, _T_DOWN = 0, 1, 2, 3
_T_UP_S, _T_GATE_S, _T_DOWN_S = 4, 5, 6
_T_OMEGA, _T_CALIB = 10, 11
_T_INPUT = 20
_CALIB_LAYER = 1_000_000


def seed_of(*key: int) -> int:
    """A 63-bit torch seed from an integer key, via numpy's SeedSequence hash."""
    st = np.random.SeedSequence([int(k) & 0xFFFFFFFF for k in key]).generate_state(2)
    return int((int(st[0]) << 31) ^ int(st[1])) & 0x7FFF_FFFF_FFFF_FFFF


def torch_gen(device, *key: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed_of(*key))
    return g


# ----------------------------------------------------------------------------- law
def powerlaw_by_rank(n: int, alpha: float, c: float, cap: float = 0.9) -> np.ndarray:
    """p of the neuron of rank k (0-based): min(cap, c * (k+1)^-alpha), fp64."""
    k = np.arange(1, n + 1, dtype=np.float64)
    return np.minimum(cap, c * k ** (-alpha))


def calibrate_c(n: int, alpha: float, mean_p: float, cap: float = 0.9) -> float:
    """The constant c for which the mean of powerlaw_by_rank equals mean_p (bisection)."""
    if not (0.0 < mean_p < cap):
        raise ValueError("mean_p must lie in (0, cap)")
    lo, hi = 0.0, 1.0
    while powerlaw_by_rank(n, alpha, hi, cap).mean() < mean_p:
        hi *= 2.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if powerlaw_by_rank(n, alpha, mid, cap).mean() < mean_p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def law_constant(w: Workload) -> float:
    return w.c if w.c is not None else calibrate_c(w.d_ff, w.alpha, w.mean_p, w.p_cap)


def firing_probs(w: Workload, layer: int) -> np.ndarray:
    """p_i per neuron (fp64): the power law over a seeded random neuron permutation."""
    by_rank = powerlaw_by_rank(w.d_ff, w.alpha, law_constant(w), w.p_cap)
    perm = torch.randperm(w.d_ff, generator=torch_gen("cpu", w.seed, layer, _T_PERM))
    p = np.empty(w.d_ff, dtype=np.float64)
    p[perm.numpy()] = by_rank
    return p


# ----------------------------------------------------------------------------- layer
@dataclass
class SynthLayer:
    """One generated layer.  Tensors live on `device`; fp32/fp16 weights in their
    stored dtype, Q4_0 weights as (nibble plane, scale plane)."""
    workload: Workload
    layer: int
    w_up: Optional[torch.Tensor]        # [f, d]            (f32/f16)
    w_gate: Optional[torch.Tensor]      # [f, d] or None    (f32/f16, ReGLU only)
    w_down: Optional[torch.Tensor]      # [d, f]            (f32/f16)
    q_up: Optional[torch.Tensor]        # [f, d/32, 16] u8  (Q4_0)
    s_up: Optional[torch.Tensor]        # [f, d/32] f16     (Q4_0)
    q_gate: Optional[torch.Tensor]
    s_gate: Optional[torch.Tensor]
    q_down: Optional[torch.Tensor]      # [f, d/32, 16] u8, neuron-major (Q4_0)
    s_down: Optional[torch.Tensor]      # [f, d/32] f16
    bias: torch.Tensor                  # [f] f32
    p1: torch.Tensor                    # [d, r] p_dtype
    p2: torch.Tensor                    # [r, f] p_dtype
    thresh: torch.Tensor                # [f] f32
    freq: torch.Tensor                  # [f] f32, predicted firing rate on calibration
    probs: np.ndarray                   # [f] f64, the law's p_i

    def tensors(self) -> Dict[str, torch.Tensor]:
        out = {}
        for k in ("w_up", "w_gate", "w_down", "q_up", "s_up", "q_gate", "s_gate",
                  "q_down", "s_down", "bias", "p1", "p2", "thresh", "freq"):
            v = getattr(self, k)
            if v is not None:
                out[k] = v
        return out

    def to_numpy(self) -> Dict[str, np.ndarray]:
        """Host copies (exact: same stored values) for the oracle."""
        return {k: v.detach().cpu().numpy() for k, v in self.tensors().items()}


def _q4_pack(q: torch.Tensor) -> torch.Tensor:
    """[rows, d] codes in 0..15 -> [rows, d/32, 16] bytes (low nibble element j,
    high nibble element j+16 of each 32-block)."""
    rows, d = q.shape
    qb = q.view(rows, d // 32, 32).to(torch.uint8)
    return (qb[:, :, :16] | (qb[:, :, 16:] << 4)).contiguous()


def _q4_matrix(w: Workload, layer: int, tid: int, sid: int, rows: int, device):
    """Random Q4_0 weights: packed nibbles, scales, and the fp32 values they encode."""
    d = w.d_model
    q = torch.randint(0, 16, (rows, d), generator=torch_gen(device, w.seed, layer, tid),
                      device=device, dtype=torch.int16)
    s = (torch.randn(rows, d // 32, generator=torch_gen(device, w.seed, layer, sid),
                     device=device) * w.w_std_q4).abs().to(torch.float16)
    vals = (q.to(torch.float32) - 8.0).view(rows, d // 32, 32) * s.float().unsqueeze(-1)
    return _q4_pack(q), s, vals.view(rows, d)


def _gauss_matrix(w: Workload, layer: int, tid: int, shape, std: float, device):
    g = torch_gen(device, w.seed, layer, tid)
    m = torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * std
    return m.to(_TORCH_DT[w.w_dtype])


def calibration_inputs(w: Workload, device, dtype=torch.float32) -> torch.Tensor:
    """n_calib x ~ N(0, I), shared by every layer of a workload."""
    g = torch_gen(device, w.seed, _CALIB_LAYER, _T_CALIB)
    return torch.randn(w.n_calib, w.d_model, generator=g, device=device, dtype=dtype)


def _fit_rrls(w: Workload, fire_rows: torch.Tensor, bias: torch.Tensor):
    """Reduced-rank least squares of sign(pre-activation) on n_calib samples (fp64)."""
    X = calibration_inputs(w, "cpu", torch.float64)
    W = fire_rows.detach().cpu().double()
    b = bias.detach().cpu().double()
    T = torch.where(X @ W.T + b > 0, 1.0, -1.0).double()
    xm, tm = X.mean(0), T.mean(0)
    Xc, Tc = X - xm, T - tm
    B = torch.linalg.solve(Xc.T @ Xc, Xc.T @ Tc)                 # d x f (OLS)
    M = Xc @ B
    evals, evecs = torch.linalg.eigh(M.T @ M)                     # ascending
    V = evecs[:, -w.rank:].flip(1)                                 # f x r, top first
    P1 = B @ V                                                     # d x r
    P2 = V.T                                                       # r x f
    t = -(tm - (xm @ P1) @ P2)
    dt = _TORCH_DT[w.p_dtype]
    return P1.to(dt), P2.to(dt), t.float(), B


def _fit_sketch(w: Workload, layer: int, fire_rows32: torch.Tensor,
                probs: np.ndarray, device):
    d, f, r = w.d_model, w.d_ff, w.rank
    dt = _TORCH_DT[w.p_dtype]
    g = torch_gen(device, w.seed, layer, _T_OMEGA)
    P1 = (torch.randn(d, r, generator=g, device=device) / math.sqrt(d)).to(dt)
    P1f = P1.float()
    P2raw = (fire_rows32 @ P1f).T.contiguous()                    # r x f
    X = calibration_inputs(w, device)
    z = X @ P1f                                                   # N x r
    std = (z @ P2raw).std(dim=0).clamp_min(1e-30)
    P2 = (P2raw / std).to(dt)
    logits = z @ P2.float()                                       # N x f
    n = w.n_calib
    k = np.clip(np.rint(n * (1.0 - probs)).astype(np.int64), 1, n) - 1
    kk = torch.from_numpy(k).to(device)
    t = torch.empty(f, device=device, dtype=torch.float32)
    chunk = 4096
    for c0 in range(0, f, chunk):
        c1 = min(f, c0 + chunk)
        srt = torch.sort(logits[:, c0:c1], dim=0).values
        t[c0:c1] = srt.gather(0, kk[c0:c1].unsqueeze(0)).squeeze(0)
    freq = (logits > t).float().mean(0)
    return P1, P2, t, freq


def make_layer(w: Workload, layer: int, device="cpu") -> SynthLayer:
    w = w.at_layer(layer)
    d, f = w.d_model, w.d_ff
    if f % 32 or d % 32:
        raise ValueError("d_model and d_ff must be multiples of 32")
    probs = firing_probs(w, layer)
    kw = dict(w_up=None, w_gate=None, w_down=None, q_up=None, s_up=None,
              q_gate=None, s_gate=None, q_down=None, s_down=None)
    std = 1.0 / math.sqrt(d)
    if w.w_dtype == "q4_0":
        kw["q_up"], kw["s_up"], up32 = _q4_matrix(w, layer, _T_UP, _T_UP_S, f, device)
        if w.act == "reglu":
            kw["q_gate"], kw["s_gate"], gate32 = _q4_matrix(w, layer, _T_GATE, _T_GATE_S, f, device)
        kw["q_down"], kw["s_down"], _ = _q4_matrix(w, layer, _T_DOWN, _T_DOWN_S, f, device)
        fire32 = gate32 if w.act == "reglu" else up32
    else:
        kw["w_up"] = _gauss_matrix(w, layer, _T_UP, (f, d), std, device)
        if w.act == "reglu":
            kw["w_gate"] = _gauss_matrix(w, layer, _T_GATE, (f, d), std, device)
        kw["w_down"] = _gauss_matrix(w, layer, _T_DOWN, (d, f), std, device)
        fire32 = (kw["w_gate"] if w.act == "reglu" else kw["w_up"]).float()
    norms = fire32.double().norm(dim=1)
    phi_inv = torch.special.ndtri(torch.from_numpy(probs).to(device))
    bias = (norms * phi_inv).float()
    if w.fit == "rrls":
        P1, P2, t, _ = _fit_rrls(w, fire32, bias)
        X = calibration_inputs(w, "cpu", torch.float32)
        logits = (X.double() @ P1.double()) @ P2.double() - t.double()
        freq = (logits > 0).float().mean(0)
        P1, P2, t, freq = (v.to(device) for v in (P1, P2, t, freq))
    elif w.fit == "sketch":
        P1, P2, t, freq = _fit_sketch(w, layer, fire32, probs, device)
    else:
        raise ValueError(w.fit)
    del fire32
    return SynthLayer(workload=w, layer=layer, bias=bias, p1=P1.contiguous(),
                      p2=P2.contiguous(), thresh=t.contiguous(), freq=freq.contiguous(),
                      probs=probs, **kw)


def make_inputs(w: Workload, n: int, device="cpu", stream_id: int = 0) -> torch.Tensor:
    """n token vectors x ~ N(0, I) in the activation dtype, [n, d_model]."""
    g = torch_gen(device, w.seed, _CALIB_LAYER + 1 + stream_id, _T_INPUT)
    x = torch.randn(n, w.d_model, generator=g, device=device, dtype=torch.float32)
    return x.to(_TORCH_DT[w.x_dtype])
