"""Workload descriptions for the seeded synthetic layers.

Each workload is a stack of ReLU or ReGLU FFN layers shaped like a real model, with
power-law neuron firing probabilities (the locality both PowerInfer pages describe:
GeekNews "Tüketici sınıfı GPU takılı PC'lerde yüksek hızlı büyük dil modeli serving" §"PowerInfer'in çözmeye çalıştığı sorun", and unite.ai
"PowerInfer: Mesin Inferensi LLM Cepat dengan GPU Konsumen", introduction).  The
datasets and trained checkpoints the pages profile are not available; these
synthetic layers stand in for them.

This module holds shapes and constants only: no arithmetic of the sparse FFN.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    d_model: int
    d_ff: int
    rank: int
    act: str                 # "relu" or "relu2" (bias on up), or "reglu" (bias on gate)
    w_dtype: str             # "f32" | "f16" | "q4_0"
    x_dtype: str             # "f32" | "f16"
    p_dtype: str             # "f32" | "f16"
    alpha: float             # power-law exponent of the firing probabilities
    c: Optional[float]       # power-law constant; None -> calibrated to mean_p
    mean_p: Optional[float]  # target mean firing probability (1 - sparsity)
    seed: int
    fit: str                 # "rrls" (reduced-rank least squares) | "sketch"
    p_cap: float = 0.9
    n_calib: int = 4096
    n_inputs: int = 64       # input vectors (single-layer workloads)
    prompt_len: int = 0      # untimed prompt vectors pushed before decode
    steps: int = 1           # decode steps
    batches: Tuple[int, ...] = (1,)
    w_std_q4: float = 0.02   # std of the |N(0, s)| Q4_0 block scales
    layer_mean_p: Optional[Tuple[float, ...]] = None   # per-layer mean firing probability (cycled)
    layer_rank: Optional[Tuple[int, ...]] = None       # per-layer predictor rank (cycled)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def at_layer(self, layer: int) -> "Workload":
        """The workload as layer `layer` sees it: its own density and predictor rank when
        the workload gives them per layer."""
        kw = {}
        if self.layer_mean_p:
            kw.update(mean_p=self.layer_mean_p[layer % len(self.layer_mean_p)], c=None)
        if self.layer_rank:
            kw.update(rank=self.layer_rank[layer % len(self.layer_rank)])
        return replace(self, **kw) if kw else self


# Single ReLU layer, fp32, d_model 512, d_ff 2048, rank-64 least-squares predictor.
# The literal constant 0.6 gives a mean firing probability of about 0.35 %.
FFN512_LIT = Workload(
    name="ffn512_relu_f32_lit", n_layers=1, d_model=512, d_ff=2048, rank=64,
    act="relu", w_dtype="f32", x_dtype="f32", p_dtype="f32", alpha=0.9, c=0.6,
    mean_p=None, seed=0, fit="rrls", n_inputs=64)

# The same layer with the constant calibrated so that about 90 % of neurons are
# inactive on average (mean firing probability 0.10).
FFN512_CAL = FFN512_LIT.with_(name="ffn512_relu_f32_cal", c=None, mean_p=0.10)

# Llama-2-7B-shaped ReGLU stack: 32 layers, 4096 x 11008, fp16, rank 512.
LLAMA2_7B = Workload(
    name="llama2_7b_reglu_f16", n_layers=32, d_model=4096, d_ff=11008, rank=512,
    act="reglu", w_dtype="f16", x_dtype="f16", p_dtype="f16", alpha=1.0, c=None,
    mean_p=0.10, seed=1, fit="sketch", steps=256)

# Falcon-40B-shaped ReLU stack: 60 layers, 8192 x 32768, fp16, rank 1024, 93 % sparse.
FALCON_40B = Workload(
    name="falcon40b_relu_f16", n_layers=60, d_model=8192, d_ff=32768, rank=1024,
    act="relu", w_dtype="f16", x_dtype="f16", p_dtype="f16", alpha=0.8, c=None,
    mean_p=0.07, seed=2, fit="sketch", prompt_len=64, steps=128)

# Llama-2-70B-shaped ReGLU stack in Q4_0: 80 layers, 8192 x 28672, rank 1024, 85 % sparse.
LLAMA2_70B_Q4 = Workload(
    name="llama2_70b_reglu_q4_0", n_layers=80, d_model=8192, d_ff=28672, rank=1024,
    act="reglu", w_dtype="q4_0", x_dtype="f16", p_dtype="f16", alpha=0.7, c=None,
    mean_p=0.15, seed=3, fit="sketch", prompt_len=8, steps=128)

# OPT-175B-shaped ReLU layers: 24 resident, 12288 x 49152, fp16, rank 1536, batch sweep.
OPT_175B = Workload(
    name="opt175b_relu_f16", n_layers=24, d_model=12288, d_ff=49152, rank=1536,
    act="relu", w_dtype="f16", x_dtype="f16", p_dtype="f16", alpha=0.9, c=None,
    mean_p=0.10, seed=4, fit="sketch", steps=16, batches=(1, 2, 4, 8, 16, 32))

ALL = {w.name: w for w in (FFN512_LIT, FFN512_CAL, LLAMA2_7B, FALCON_40B,
                           LLAMA2_70B_Q4, OPT_175B)}


def scaled(base: Workload, name: str, n_layers: int, d_model: int, d_ff: int,
           rank: int, **kw) -> Workload:
    """A smaller workload with the same law, dtypes and predictor fit as `base`."""
    return base.with_(name=name, n_layers=n_layers, d_model=d_model, d_ff=d_ff,
                      rank=rank, **kw)


def adaptive_ranks(base_rank: int, layer_mean_p: Tuple[float, ...], d_model: int,
                   floor: int = 64) -> Tuple[int, ...]:
    """Per-layer predictor ranks from per-layer densities.  The pages size each layer's
    predictor by the layer's own sparsity (a sparser layer gets a smaller predictor;
    unite.ai "PowerInfer: Mesin Inferensi LLM Cepat dengan GPU Konsumen", §"Prediktor
    Kepadatan Adaptif") but give no formula.  The reading here is the plainest one: the
    densest layer keeps the base rank, and every other layer gets the base rank in
    proportion to its mean firing probability, rounded to a multiple of 8 and kept within
    [floor, d_model]."""
    top = max(layer_mean_p)
    out = []
    for p in layer_mean_p:
        r = int(round(base_rank * p / top / 8.0)) * 8
        out.append(max(floor, min(d_model, r)))
    return tuple(out)


def _linear_profile(n: int, lo: float, hi: float) -> Tuple[float, ...]:
    return tuple(hi + (lo - hi) * l / (n - 1) for l in range(n))


# Llama-2-7B-shaped stack whose layers differ in density (a synthetic profile from 14 %
# active in the first layer down to 6 % in the last, 10 % on average, the base workload's
# mean), each with the adaptive predictor rank of its density.
_ADAPTIVE_P = _linear_profile(32, 0.06, 0.14)
LLAMA2_7B_ADAPTIVE = LLAMA2_7B.with_(name="llama2_7b_reglu_f16_adaptive_rank", layer_mean_p=_ADAPTIVE_P,
                                     layer_rank=adaptive_ranks(512, _ADAPTIVE_P, 4096))
