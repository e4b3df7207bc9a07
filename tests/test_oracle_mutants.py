"""The pins have teeth: plant plausible mistakes in the oracle (on the CPU, through
monkeypatching) and check that at least one pin fails for each of them."""
import numpy as np
import pytest

from oracle import ffn as O
import test_oracle_pins as P
import test_oracle_stack_pins as SP

_orig = {name: getattr(O, name) for name in
         ("predictor_logits", "fire_bits", "activations", "sparse_ffn", "pack_mask",
          "compact", "q4_0_unpack", "stack_glue", "hot_order", "down_accumulate",
          "layer_weights_f64", "layer_step", "decode_stack")}


def _pins():
    yield lambda: P.test_brute_force_exact("relu", 0)
    yield lambda: P.test_brute_force_exact("reglu", 1)
    yield P.test_relu_single_neuron_by_hand
    yield P.test_reglu_single_neuron_by_hand
    yield P.test_relu2_single_neuron_by_hand
    yield lambda: P.test_brute_force_exact("relu2", 2)
    yield P.test_one_hot_input_selects_predictor_row
    yield P.test_logit_zero_is_inactive
    yield P.test_batch_masks_apply_per_token
    yield lambda: P.test_sparse_equals_dense_with_true_mask("relu")
    yield P.test_mask_words_lsb_first
    yield P.test_compaction_invariants
    yield P.test_q4_0_block_by_definition
    yield P.test_q4_0_scale_is_fp16
    yield P.test_stack_glue_closed_form
    yield P.test_hot_order_and_prefix
    yield P.test_permuted_layer_same_output
    yield SP.test_q4_down_plane_is_transposed
    yield SP.test_q4_layer_output_by_hand
    yield lambda: SP.test_two_layer_two_token_stack("relu")
    yield lambda: SP.test_two_layer_two_token_stack("reglu")
    yield SP.test_layer_step_record


def _mut_logits_plus_t(x, p1, p2, t):
    return _orig["predictor_logits"](x, p1, p2, -t)


def _mut_fire_ge(l):
    return np.asarray(l) >= 0.0


def _mut_act_no_bias(x, w, act, rows):
    w2 = dict(w)
    w2["bias"] = np.zeros_like(w["bias"])
    return _orig["activations"](x, w2, act, rows)


def _mut_act_relu_on_up(x, w, act, rows):
    if act != "reglu":
        return _orig["activations"](x, w, act, rows)
    x = np.atleast_2d(x)
    gate = x @ w["w_gate"][rows].T + w["bias"][rows]
    up = x @ w["w_up"][rows].T
    return gate * np.maximum(up, 0.0)


def _mut_act_bias_on_up(x, w, act, rows):
    if act != "reglu":
        return _orig["activations"](x, w, act, rows)
    x = np.atleast_2d(x)
    gate = x @ w["w_gate"][rows].T
    up = x @ w["w_up"][rows].T + w["bias"][rows]
    return np.maximum(gate, 0.0) * up


def _mut_relu2_unsquared(x, w, act, rows):
    return _orig["activations"](x, w, "relu" if act == "relu2" else act, rows)


def _mut_relu2_square_before_clamp(x, w, act, rows):
    if act != "relu2":
        return _orig["activations"](x, w, act, rows)
    x = np.atleast_2d(x)
    pre = x @ w["w_up"][rows].T + w["bias"][rows]
    return pre * pre


def _mut_sparse_ignores_token_mask(x, w, act, masks, idx):
    return _orig["sparse_ffn"](x, w, act, np.ones_like(np.atleast_2d(masks)), idx)


def _mut_pack_msb(bits):
    bits = np.atleast_2d(np.asarray(bits, bool))
    return _orig["pack_mask"](bits.reshape(bits.shape[0], -1, 32)[:, :, ::-1].reshape(bits.shape))


def _mut_compact_intersection(words, f):
    inter = O.unpack_mask(words, f).all(axis=0)
    idx = np.flatnonzero(inter).astype(np.int32)
    return idx, int(idx.size)


def _mut_q4_swap_halves(nib, sc):
    nib = np.asarray(nib, np.uint8)
    return _orig["q4_0_unpack"](((nib & 0x0F) << 4) | (nib >> 4), sc)


def _mut_q4_no_offset(nib, sc):
    return _orig["q4_0_unpack"](nib, sc) + 8.0 * np.repeat(
        np.asarray(sc, np.float16).astype(np.float64), 32, axis=1)


def _mut_q4_interleaved(nib, sc):
    v = _orig["q4_0_unpack"](nib, sc)
    rows, n = v.shape
    b = v.reshape(rows, n // 32, 2, 16).transpose(0, 1, 3, 2)
    return b.reshape(rows, n)


def _mut_glue_no_residual(x, y, x_dtype):
    return _orig["stack_glue"](np.zeros_like(np.atleast_2d(x), dtype=np.float64), y + 0 * np.atleast_2d(x), x_dtype) \
        if np.any(y) else _orig["stack_glue"](x, y, x_dtype)


def _mut_hot_order_ties_desc(freq):
    freq = np.asarray(freq, np.float64)
    return np.array(sorted(range(freq.size), key=lambda i: (-freq[i], -i)), dtype=np.int32)


def _mut_down_reverse(a, w_down, rows):
    a = np.atleast_2d(a)
    return _orig["down_accumulate"](a[:, ::-1], w_down, list(rows))


def _mut_q4_down_not_transposed(t, act):
    out = _orig["layer_weights_f64"](t, act)
    if "q_down" in t:
        out["w_down"] = O.q4_0_unpack(t["q_down"], t["s_down"])
    return out


def _mut_step_union_bits(x, w, act, x_dtype):
    f = w["bias"].shape[0]
    logits = O.predictor_logits(x, w["p1"], w["p2"], w["thresh"])
    bits = O.fire_bits(logits)
    words = O.pack_mask(bits)
    idx, count = O.compact(words, f)
    union = np.broadcast_to(np.atleast_2d(bits).any(axis=0), np.atleast_2d(bits).shape)
    y = O.sparse_ffn(x, w, act, union, idx)
    return {"logits": logits, "bits": bits, "words": words, "idx": idx, "count": count, "y": y,
            "x_next": O.stack_glue(x, y, x_dtype)}


def _mut_stack_keeps_x_in(x0, layers, act, x_dtype):
    x = np.atleast_2d(x0)
    trace = []
    for w in layers:
        rec = O.layer_step(x, w, act, x_dtype)
        rec["x_in"] = x
        trace.append(rec)
    return trace


MUTANTS = {
    "q4 down plane not transposed": ("layer_weights_f64", _mut_q4_down_not_transposed),
    "union mask as per-token bits": ("layer_step", _mut_step_union_bits),
    "next layer gets x_in": ("decode_stack", _mut_stack_keeps_x_in),
    "logit +t": ("predictor_logits", _mut_logits_plus_t),
    "fire >=": ("fire_bits", _mut_fire_ge),
    "act without bias": ("activations", _mut_act_no_bias),
    "reglu relu on up": ("activations", _mut_act_relu_on_up),
    "reglu bias on up": ("activations", _mut_act_bias_on_up),
    "relu2 not squared": ("activations", _mut_relu2_unsquared),
    "relu2 squared before the clamp": ("activations", _mut_relu2_square_before_clamp),
    "token mask ignored": ("sparse_ffn", _mut_sparse_ignores_token_mask),
    "mask words msb-first": ("pack_mask", _mut_pack_msb),
    "compact intersection": ("compact", _mut_compact_intersection),
    "q4 nibble halves swapped": ("q4_0_unpack", _mut_q4_swap_halves),
    "q4 missing -8": ("q4_0_unpack", _mut_q4_no_offset),
    "q4 interleaved nibbles": ("q4_0_unpack", _mut_q4_interleaved),
    "glue without residual": ("stack_glue", _mut_glue_no_residual),
    "hot order ties reversed": ("hot_order", _mut_hot_order_ties_desc),
    "down weights misaligned": ("down_accumulate", _mut_down_reverse),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    failures = 0
    for pin in _pins():
        try:
            pin()
        except Exception:
            failures += 1
    assert failures > 0, f"no pin caught mutant {name!r}"


def test_unmutated_oracle_passes_every_pin():
    for pin in _pins():
        pin()
