"""Oracle: a plain, slow, fp64 CPU statement of the activation-sparse FFN at decode.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this module; the library never does, and this module never
imports the library.  It shares no code with the CUDA path.

Sources (three web pages about PowerInfer; cited by page title and section):
  [GN]  GeekNews "Tüketici sınıfı GPU takılı PC'lerde yüksek hızlı büyük dil modeli serving"
        (tr.news.hada.io), sections "CPU/GPU hibrit çıkarım yöntemi", "Kuantizasyon ve
        uyumluluk", "Kısıtlar ve SSS".
  [KPD] Telegram channel КПД, "PowerInfer: Fast Large Language Model Serving with a
        Consumer-grade GPU", sections "Введение", "Метод".
  [UAI] unite.ai "PowerInfer: Mesin Inferensi LLM Cepat dengan GPU Konsumen", sections
        "Fase Online: Mesin Inferensi LLM yang Sadar Neuron", "Prediktor Kepadatan
        Adaptif", "Penempatan dan Pengelolaan Neuron", "Operator yang Sadar Neuron".

What it computes, for one layer and tokens x[b, :]:
  predictor  u = P1^T x ; logit_i = sum_k P2[k, i] u_k - t_i ; fires iff logit_i > 0
  compaction idx = ascending neuron ids whose bit is set in any token's mask
  activation ReLU : a_i = max(0, w_up_i . x + b_i)
             ReGLU: a_i = max(0, w_gate_i . x + b_i) * (w_up_i . x)
             a[b, i] = 0 where token b's own mask bit is 0
  down       y_j = sum over idx ascending of W_down[j, i] * a_i
  glue       v = x + y ; x' = (v - mean(v)) / sqrt(var(v) + 1e-6), rounded to the activation dtype
All arithmetic is fp64; stored values (fp16, Q4_0) are widened exactly.
"""
from __future__ import annotations

from typing import Dict, List, Optional, Sequence

import numpy as np

RMS_EPS = 1e-6


# ------------------------------------------------------------------ Q4_0 weights
def q4_0_unpack(nibbles: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Q4_0 rows -> fp64 values.

    [GN] §"Kuantizasyon ve uyumluluk" names INT4 Q4_0 as the optimised format: blocks
    of 32 four-bit codes q in 0..15 sharing one fp16 scale, value = (q - 8) * scale.
    Layout read here: byte j of a block carries element j in its low four bits and
    element j + 16 in its high four bits.

    nibbles: uint8 [rows, nblocks, 16]; scales: fp16 [rows, nblocks] -> [rows, 32*nblocks].
    """
    nib = np.asarray(nibbles, dtype=np.uint8)
    rows, nblk, sixteen = nib.shape
    assert sixteen == 16
    codes = np.empty((rows, nblk, 32), dtype=np.int64)
    codes[:, :, :16] = nib & 0x0F
    codes[:, :, 16:] = nib >> 4
    vals = (codes - 8).astype(np.float64) * np.asarray(scales, np.float16).astype(np.float64)[:, :, None]
    return vals.reshape(rows, nblk * 32)


# ------------------------------------------------------------------ weights as fp64
def layer_weights_f64(t: Dict[str, np.ndarray], act: str) -> Dict[str, np.ndarray]:
    """Widen one layer's stored tensors to fp64 in the oracle's own orientation:
    w_up/w_gate [f, d], w_down [d, f], bias/thresh [f], p1 [d, r], p2 [r, f]."""
    out: Dict[str, np.ndarray] = {}
    if "q_up" in t:
        out["w_up"] = q4_0_unpack(t["q_up"], t["s_up"])
        if act == "reglu":
            out["w_gate"] = q4_0_unpack(t["q_gate"], t["s_gate"])
        out["w_down"] = q4_0_unpack(t["q_down"], t["s_down"]).T   # neuron-major given
    else:
        out["w_up"] = np.asarray(t["w_up"]).astype(np.float64)
        if act == "reglu":
            out["w_gate"] = np.asarray(t["w_gate"]).astype(np.float64)
        out["w_down"] = np.asarray(t["w_down"]).astype(np.float64)
    out["bias"] = np.asarray(t["bias"]).astype(np.float64)
    out["p1"] = np.asarray(t["p1"]).astype(np.float64)
    out["p2"] = np.asarray(t["p2"]).astype(np.float64)
    out["thresh"] = np.asarray(t["thresh"]).astype(np.float64)
    return out


# ------------------------------------------------------------------ predictor
def predictor_logits(x: np.ndarray, p1: np.ndarray, p2: np.ndarray,
                     thresh: np.ndarray) -> np.ndarray:
    """logit[b, i] = sum_k P2[k, i] * (sum_j P1[j, k] * x[b, j]) - t_i.

    [UAI] §"Prediktor Kepadatan Adaptif": each layer has a small predictor, kept on
    the GPU, that says which neurons will be active; only those are processed.  The
    pages give no architecture; the linear low-rank form with a per-neuron threshold
    is the reading taken here.
    """
    x = np.atleast_2d(np.asarray(x, np.float64))
    u = x @ p1
    return u @ p2 - thresh


def fire_bits(logits: np.ndarray) -> np.ndarray:
    """Neuron fires iff its logit is strictly positive (logit 0 is inactive, the same
    convention as ReLU(0) = 0)."""
    return np.asarray(logits) > 0.0


def pack_mask(bits: np.ndarray) -> np.ndarray:
    """[B, f] bools -> [B, f/32] uint32 words; bit j of word w is neuron 32*w + j."""
    bits = np.atleast_2d(np.asarray(bits, bool))
    B, f = bits.shape
    assert f % 32 == 0
    words = np.zeros((B, f // 32), dtype=np.uint64)
    for j in range(32):
        words |= bits[:, j::32].astype(np.uint64) << np.uint64(j)
    return words.astype(np.uint32)


def unpack_mask(words: np.ndarray, f: int) -> np.ndarray:
    words = np.atleast_2d(np.asarray(words, np.uint32))
    B = words.shape[0]
    bits = np.zeros((B, f), dtype=bool)
    for j in range(32):
        bits[:, j::32] = (words >> np.uint32(j)) & np.uint32(1)
    return bits


# ------------------------------------------------------------------ compaction
def compact(words: np.ndarray, f: int):
    """Active-index list of the union over tokens of the per-token masks.

    [UAI] §"Operator yang Sadar Neuron": the operators touch individual rows and
    columns of the active neurons directly, with no conversion to a dense format.
    Returns (idx int32 ascending, count).
    """
    union = unpack_mask(words, f).any(axis=0)
    idx = np.flatnonzero(union).astype(np.int32)
    return idx, int(idx.size)


# ------------------------------------------------------------------ FFN
def _preacts(x: np.ndarray, w: Dict[str, np.ndarray], act: str, rows):
    """Per-token pre-activations of the given neuron rows (fp64)."""
    up = x @ w["w_up"][rows].T
    if act in ("relu", "relu2"):
        return up + w["bias"][rows], None
    gate = x @ w["w_gate"][rows].T
    return gate + w["bias"][rows], up


def activations(x: np.ndarray, w: Dict[str, np.ndarray], act: str,
                rows: np.ndarray) -> np.ndarray:
    """a[b, k] for neuron rows[k].  ReLU: max(0, up + b).  ReGLU: max(0, gate + b) * up.
    Squared ReLU ("relu2"): max(0, up + b)^2.

    [GN] §"Kısıtlar ve SSS": only ReLU / ReGLU / squared-ReLU models are supported,
    because those activations give exact zeros that can be skipped.
    """
    fire, up = _preacts(np.atleast_2d(x), w, act, rows)
    a = np.maximum(fire, 0.0)
    if act == "reglu":
        a = a * up
    elif act == "relu2":
        a = a * a
    return a


def down_accumulate(a: np.ndarray, w_down: np.ndarray, rows: Sequence[int]) -> np.ndarray:
    """y[b, :] = sum over k in list order of a[b, k] * W_down[:, rows[k]], fp64,
    accumulated one neuron at a time so the order of the sum is the list order."""
    a = np.atleast_2d(a)
    y = np.zeros((a.shape[0], w_down.shape[0]), dtype=np.float64)
    for k, i in enumerate(rows):
        y += a[:, k:k + 1] * w_down[:, i][None, :]
    return y


def sparse_ffn(x: np.ndarray, w: Dict[str, np.ndarray], act: str,
               masks: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Neuron-aware sparse FFN over the active list.

    [UAI] §"Fase Online: Mesin Inferensi LLM yang Sadar Neuron" and §"Operator yang Sadar Neuron": predicted-inactive neurons
    are skipped; the active ones are computed row by row (up/gate) and column by column
    (down).  masks: [B, f] bools (per token); idx: ascending union list.
    """
    x = np.atleast_2d(np.asarray(x, np.float64))
    idx = np.asarray(idx, np.int64)
    a = activations(x, w, act, idx)
    a = np.where(np.atleast_2d(masks)[:, idx], a, 0.0)
    return down_accumulate(a, w["w_down"], idx)


def dense_ffn(x: np.ndarray, w: Dict[str, np.ndarray], act: str) -> np.ndarray:
    """The dense FFN (ReLU, ReGLU or squared ReLU): every neuron, no predictor."""
    f = w["bias"].shape[0]
    rows = np.arange(f)
    return down_accumulate(activations(np.atleast_2d(x), w, act, rows), w["w_down"], rows)


def true_mask(x: np.ndarray, w: Dict[str, np.ndarray], act: str) -> np.ndarray:
    """m*_i = (firing pre-activation > 0): where ReLU passes a nonzero value."""
    f = w["bias"].shape[0]
    fire, _ = _preacts(np.atleast_2d(np.asarray(x, np.float64)), w, act, np.arange(f))
    return fire > 0.0


# ------------------------------------------------------------------ stack glue
def _round_act(v: np.ndarray, x_dtype: str) -> np.ndarray:
    v32 = v.astype(np.float32)
    if x_dtype == "f16":
        return v32.astype(np.float16)
    return v32


def stack_glue(x: np.ndarray, y: np.ndarray, x_dtype: str) -> np.ndarray:
    """x' = (v - mean(v)) / sqrt(var(v) + 1e-6) with v = x + y, per token, rounded to the
    activation dtype (through fp32, the glue's precision).  The pages have no layer stack;
    this residual + mean-centred normalisation keeps every layer input centred with unit
    variance, so the firing law of the next layer holds even when the weights have a
    nonzero mean (Q4_0 codes q - 8 have mean -1/2)."""
    v = np.atleast_2d(np.asarray(x, np.float64)) + y
    mu = np.mean(v, axis=1, keepdims=True)
    var = np.mean((v - mu) * (v - mu), axis=1, keepdims=True)
    return _round_act((v - mu) / np.sqrt(var + RMS_EPS), x_dtype)


def layer_step(x: np.ndarray, w: Dict[str, np.ndarray], act: str, x_dtype: str):
    """One layer: predict, compact, sparse FFN, glue.  Returns a trace record."""
    f = w["bias"].shape[0]
    logits = predictor_logits(x, w["p1"], w["p2"], w["thresh"])
    bits = fire_bits(logits)
    words = pack_mask(bits)
    idx, count = compact(words, f)
    y = sparse_ffn(x, w, act, bits, idx)
    x_next = stack_glue(x, y, x_dtype)
    return {"logits": logits, "bits": bits, "words": words, "idx": idx,
            "count": count, "y": y, "x_next": x_next}


def decode_stack(x0: np.ndarray, layers: List[Dict[str, np.ndarray]], act: str,
                 x_dtype: str) -> List[dict]:
    """Run x0 [B, d] through every layer; one trace record per layer."""
    x = np.atleast_2d(x0)
    trace = []
    for w in layers:
        rec = layer_step(x, w, act, x_dtype)
        rec["x_in"] = x
        trace.append(rec)
        x = rec["x_next"]
    return trace


# ------------------------------------------------------------------ hot prefix
def hot_order(freq: np.ndarray) -> np.ndarray:
    """perm[new] = original neuron id: neurons sorted by descending measured firing
    frequency, ties by ascending original id.

    [UAI] §"Penempatan dan Pengelolaan Neuron": neurons are placed by how often they
    fire, and a neuron table maps each placed neuron back to its original position in
    the weight matrices.  [KPD] §"Метод": activation statistics are collected offline.
    """
    freq = np.asarray(freq, np.float64)
    return np.array(sorted(range(freq.size), key=lambda i: (-freq[i], i)), dtype=np.int32)


def permute_layer(w: Dict[str, np.ndarray], perm: np.ndarray) -> Dict[str, np.ndarray]:
    """The same layer with its neurons stored in `perm` order."""
    out = dict(w)
    out["w_up"] = w["w_up"][perm]
    if "w_gate" in w:
        out["w_gate"] = w["w_gate"][perm]
    out["w_down"] = w["w_down"][:, perm]
    out["bias"] = w["bias"][perm]
    out["p2"] = w["p2"][:, perm]
    out["thresh"] = w["thresh"][perm]
    return out


def hot_prefix_len(freq_sorted: np.ndarray, batch: int) -> int:
    """Neurons (in hot order) that fire for at least one of `batch` independent tokens
    with probability >= 1/2: 1 - (1 - f_i)^batch >= 1/2."""
    f = np.asarray(freq_sorted, np.float64)
    return int(np.count_nonzero(1.0 - (1.0 - f) ** batch >= 0.5))


# ------------------------------------------------------------------ activation mass
def hot_fraction_for_mass(mass: np.ndarray, share: float = 0.8) -> float:
    """Smallest fraction of neurons (most massive first) whose mass reaches `share`
    of the total.  [KPD] §"Метод": 26 % of OPT-30B's neurons (43 % for Llama-2-70B)
    carry 80 % of the total activation magnitude."""
    m = np.sort(np.asarray(mass, np.float64))[::-1]
    c = np.cumsum(m)
    k = int(np.searchsorted(c, share * c[-1], side="left")) + 1
    return k / m.size
