"""Pins of the oracle against things other than itself: exact rational brute force on
tiny layers, hand-built cases with known answers, the sparse = dense invariant, the
Q4_0 and mask-word definitions, and closed forms of the synthetic workload."""
from fractions import Fraction as Fr

import numpy as np
import pytest

from oracle import ffn as O


# ----------------------------------------------------------------- tiny exact layers
def _dyadic(rng, shape, num_lo, num_hi, den):
    return rng.integers(num_lo, num_hi + 1, size=shape).astype(np.float64) / den


def tiny_layer(act, seed=0, d=8, f=64, r=4):
    """A tiny layer whose values are small dyadic rationals, so every fp64 sum the
    oracle forms is exact and must equal the rational brute force bit for bit."""
    rng = np.random.default_rng(seed)
    w = {"w_up": _dyadic(rng, (f, d), -4, 4, 8),
         "w_down": _dyadic(rng, (d, f), -4, 4, 8),
         "bias": _dyadic(rng, (f,), -8, 8, 16),
         "p1": _dyadic(rng, (d, r), -4, 4, 4),
         "p2": _dyadic(rng, (r, f), -4, 4, 4),
         "thresh": _dyadic(rng, (f,), -16, 16, 8)}
    if act == "reglu":
        w["w_gate"] = _dyadic(rng, (f, d), -4, 4, 8)
    x = _dyadic(rng, (3, d), -8, 8, 4)
    return w, x


def brute_logits(x_row, w):
    d, r = w["p1"].shape
    f = w["p2"].shape[1]
    u = [sum((Fr(w["p1"][j, k]) * Fr(x_row[j]) for j in range(d)), Fr(0)) for k in range(r)]
    return [sum((Fr(w["p2"][k, i]) * u[k] for k in range(r)), Fr(0)) - Fr(w["thresh"][i])
            for i in range(f)]


def brute_act(x_row, w, act, i):
    d = len(x_row)
    up = sum((Fr(w["w_up"][i, j]) * Fr(x_row[j]) for j in range(d)), Fr(0))
    if act == "relu":
        return max(Fr(0), up + Fr(w["bias"][i]))
    if act == "relu2":
        return max(Fr(0), up + Fr(w["bias"][i])) ** 2
    gate = sum((Fr(w["w_gate"][i, j]) * Fr(x_row[j]) for j in range(d)), Fr(0))
    return max(Fr(0), gate + Fr(w["bias"][i])) * up


def brute_y(x_row, w, act, active):
    d = w["w_down"].shape[0]
    out = []
    for j in range(d):
        s = Fr(0)
        for i in active:
            s += Fr(w["w_down"][j, i]) * brute_act(x_row, w, act, i)
        out.append(s)
    return out


@pytest.mark.parametrize("act", ["relu", "reglu", "relu2"])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_exact(act, seed):
    w, x = tiny_layer(act, seed)
    f = w["bias"].size
    logits = O.predictor_logits(x, w["p1"], w["p2"], w["thresh"])
    bits = O.fire_bits(logits)
    words = O.pack_mask(bits)
    idx, count = O.compact(words, f)
    y = O.sparse_ffn(x, w, act, bits, idx)
    for b in range(x.shape[0]):
        bl = brute_logits(x[b], w)
        assert [float(v) for v in bl] == list(logits[b])
        assert [v > 0 for v in bl] == list(bits[b])
        by = brute_y(x[b], w, act, [i for i in range(f) if bl[i] > 0])
        assert [float(v) for v in by] == list(y[b])
    union = sorted({i for b in range(x.shape[0]) for i in range(f) if bits[b, i]})
    assert list(idx) == union and count == len(union)
    # dense FFN against the brute force over every neuron
    yd = O.dense_ffn(x, w, act)
    for b in range(x.shape[0]):
        assert [float(v) for v in brute_y(x[b], w, act, range(f))] == list(yd[b])


# ----------------------------------------------------------------- hand-built cases
def _one_neuron_layer(act, d=4, f=32, i=5):
    w = {"w_up": np.zeros((f, d)), "w_down": np.zeros((d, f)), "bias": np.zeros(f),
         "p1": np.zeros((d, 2)), "p2": np.zeros((2, f)), "thresh": np.ones(f)}
    w["w_up"][i] = [1.0, -2.0, 0.5, 3.0]
    w["w_down"][:, i] = [2.0, 0.0, -1.0, 4.0]
    w["bias"][i] = -0.25
    if act == "reglu":
        w["w_gate"] = np.zeros((f, d))
        w["w_gate"][i] = [0.5, 1.0, -1.0, 0.0]
    return w


def test_relu_single_neuron_by_hand():
    w = _one_neuron_layer("relu")
    x = np.array([[1.0, 1.0, 2.0, 0.5]])
    # up = 1 - 2 + 1 + 1.5 = 1.5 ; + bias -0.25 = 1.25 ; ReLU -> 1.25
    y = O.sparse_ffn(x, w, "relu", np.ones((1, 32), bool), np.array([5]))
    assert np.array_equal(y, [[2.5, 0.0, -1.25, 5.0]])
    # negative pre-activation: x = -x gives up = -1.5, -1.75 -> 0
    y = O.sparse_ffn(-x, w, "relu", np.ones((1, 32), bool), np.array([5]))
    assert np.array_equal(y, np.zeros((1, 4)))


def test_relu2_single_neuron_by_hand():
    w = _one_neuron_layer("relu")
    x = np.array([[1.0, 1.0, 2.0, 0.5]])
    # up + bias = 1.25 as in the ReLU case; squared -> 1.5625
    y = O.sparse_ffn(x, w, "relu2", np.ones((1, 32), bool), np.array([5]))
    assert np.array_equal(y, [[3.125, 0.0, -1.5625, 6.25]])
    # below the kink the square of the ReLU is still exactly zero
    y = O.sparse_ffn(-x, w, "relu2", np.ones((1, 32), bool), np.array([5]))
    assert np.array_equal(y, np.zeros((1, 4)))
    # a pre-activation under 1 shrinks: (0.5)^2 = 0.25
    x3 = np.array([[0.0, 0.0, 0.0, 0.25]])   # up = 0.75, + bias -> 0.5
    assert O.activations(x3, w, "relu2", np.array([5]))[0, 0] == 0.25


def test_reglu_single_neuron_by_hand():
    w = _one_neuron_layer("reglu")
    x = np.array([[2.0, 1.0, 0.0, -1.0]])
    # gate = 1 + 1 + 0 + 0 = 2 ; + bias -0.25 = 1.75 ; up = 2 - 2 + 0 - 3 = -3
    # a = ReLU(1.75) * (-3) = -5.25 (negative: ReLU is on the gate only)
    a = O.activations(x, w, "reglu", np.array([5]))
    assert a[0, 0] == -5.25
    y = O.sparse_ffn(x, w, "reglu", np.ones((1, 32), bool), np.array([5]))
    assert np.array_equal(y, [[-10.5, 0.0, 5.25, -21.0]])
    # gate negative -> 0 whatever up is
    x2 = np.array([[-2.0, -1.0, 0.0, -1.0]])
    assert O.activations(x2, w, "reglu", np.array([5]))[0, 0] == 0.0


def test_one_hot_input_selects_predictor_row():
    rng = np.random.default_rng(3)
    d, r, f = 6, 3, 64
    p1, p2, t = rng.normal(size=(d, r)), rng.normal(size=(r, f)), rng.normal(size=f)
    for j in range(d):
        e = np.zeros((1, d))
        e[0, j] = 1.0
        got = O.predictor_logits(e, p1, p2, t)[0]
        want = np.array([sum(p1[j, k] * p2[k, i] for k in range(r)) - t[i] for i in range(f)])
        assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_logit_zero_is_inactive():
    assert list(O.fire_bits(np.array([-1e-300, 0.0, -0.0, 1e-300]))) == [False, False, False, True]


def test_batch_masks_apply_per_token():
    w = _one_neuron_layer("relu")
    x = np.array([[1.0, 1.0, 2.0, 0.5], [1.0, 1.0, 2.0, 0.5]])
    masks = np.zeros((2, 32), bool)
    masks[1, 5] = True                      # neuron 5 active for token 1 only
    y = O.sparse_ffn(x, w, "relu", masks, np.array([5]))
    assert np.array_equal(y[0], np.zeros(4))
    assert np.array_equal(y[1], [2.5, 0.0, -1.25, 5.0])


# ----------------------------------------------------------------- invariants
@pytest.mark.parametrize("act", ["relu", "reglu", "relu2"])
def test_sparse_equals_dense_with_true_mask(act):
    """Skipped neurons contribute exact zeros, so with the true mask the sparse FFN
    is bit-identical to the dense one (unite.ai "PowerInfer: Mesin Inferensi LLM Cepat dengan GPU Konsumen",
    §"Fase Online: Mesin Inferensi LLM yang Sadar Neuron":
    inactive neurons are skipped)."""
    rng = np.random.default_rng(7)
    d, f = 48, 256
    w = {"w_up": rng.normal(size=(f, d)) / 7, "w_down": rng.normal(size=(d, f)) / 7,
         "bias": rng.normal(size=f) - 1.0}
    if act == "reglu":
        w["w_gate"] = rng.normal(size=(f, d)) / 7
    x = rng.normal(size=(4, d))
    m = O.true_mask(x, w, act)
    assert 0 < m.sum() < m.size
    idx, _ = O.compact(O.pack_mask(m), f)
    ys = O.sparse_ffn(x, w, act, m, idx)
    yd = O.dense_ffn(x, w, act)
    assert np.array_equal(ys, yd)
    # all-ones mask: the dense result as well; all-zero mask: exactly zero
    ones = np.ones((4, f), bool)
    assert np.array_equal(O.sparse_ffn(x, w, act, ones, np.arange(f)), yd)
    zero = np.zeros((4, f), bool)
    idx0, c0 = O.compact(O.pack_mask(zero), f)
    assert c0 == 0 and np.array_equal(O.sparse_ffn(x, w, act, zero, idx0), np.zeros((4, d)))
    # a true-mask subset that misses an active neuron changes the result
    if act == "relu":
        drop = m.copy()
        b, i = np.argwhere(m)[0]
        drop[b, i] = False
        assert not np.array_equal(O.sparse_ffn(x, w, act, drop, idx), yd)


def test_mask_words_lsb_first():
    bits = np.zeros((2, 64), bool)
    bits[0, 0] = True           # word 0 bit 0
    bits[0, 33] = True          # word 1 bit 1
    bits[1, 31] = True          # word 0 bit 31
    bits[1, 63] = True          # word 1 bit 31
    words = O.pack_mask(bits)
    assert words.dtype == np.uint32
    assert words.tolist() == [[1, 2], [0x80000000, 0x80000000]]
    assert np.array_equal(O.unpack_mask(words, 64), bits)


def test_compaction_invariants():
    rng = np.random.default_rng(11)
    for B, f, dens in [(1, 96, 0.1), (3, 2048, 0.05), (8, 1024, 0.3), (1, 64, 0.0), (2, 64, 1.0)]:
        bits = rng.random((B, f)) < dens
        words = O.pack_mask(bits)
        idx, count = O.compact(words, f)
        pop = sum(bin(int(v)).count("1") for v in np.bitwise_or.reduce(words, axis=0))
        assert count == pop == idx.size
        assert np.all(np.diff(idx) > 0) and (idx.size == 0 or (idx[0] >= 0 and idx[-1] < f))
        rebuilt = np.zeros(f, bool)
        rebuilt[idx] = True
        assert np.array_equal(rebuilt, bits.any(axis=0))


# ----------------------------------------------------------------- Q4_0
def test_q4_0_block_by_definition():
    """value = (q - 8) * scale; byte j holds element j (low nibble) and j+16 (high)."""
    nib = np.zeros((1, 2, 16), np.uint8)
    for j in range(16):
        nib[0, 0, j] = (j & 0xF) | (((15 - j) & 0xF) << 4)
    nib[0, 1, :] = 0x8F                      # low 15 -> +7 ; high 8 -> 0
    sc = np.array([[0.5, 0.25]], np.float16)
    v = O.q4_0_unpack(nib, sc)
    want0 = [(j - 8) * 0.5 for j in range(16)] + [((15 - j) - 8) * 0.5 for j in range(16)]
    want1 = [7 * 0.25] * 16 + [0.0] * 16
    assert v.shape == (1, 64)
    assert v[0].tolist() == want0 + want1


def test_q4_0_scale_is_fp16():
    nib = np.full((1, 1, 16), 0x99, np.uint8)          # every code 9 -> +1 * scale
    sc = np.array([[0.1]], np.float16)
    v = O.q4_0_unpack(nib, sc)
    assert np.all(v == float(np.float16(0.1)))
    assert float(np.float16(0.1)) != 0.1


# ----------------------------------------------------------------- glue, hot order
def test_stack_glue_closed_form():
    x = np.array([[3.0, -4.0, 0.0, 1.0]], np.float32)
    y = np.zeros((1, 4))
    out = O.stack_glue(x, y, "f32")
    # mean 0, var = (9 + 16 + 0 + 1) / 4 = 6.5
    sd = np.sqrt(6.5 + 1e-6)
    assert np.array_equal(out, np.array([[3 / sd, -4 / sd, 0, 1 / sd]], np.float32))
    # residual: x + y enters, and a constant offset is removed
    y2 = np.array([[1.0, 0.0, 0.0, 2.0]]) + 10.0
    v = np.array([4.0, -4.0, 0.0, 3.0]) + 10.0
    w = v - v.mean()
    assert np.allclose(O.stack_glue(x, y2, "f32")[0], w / np.sqrt(np.mean(w * w) + 1e-6), rtol=1e-6)
    assert O.stack_glue(x, y2, "f16").dtype == np.float16
    # the output is centred with unit variance (up to eps and rounding)
    rng = np.random.default_rng(2)
    o = O.stack_glue(rng.normal(size=(3, 256)), rng.normal(size=(3, 256)) + 5.0, "f32").astype(np.float64)
    assert np.allclose(o.mean(axis=1), 0, atol=1e-6) and np.allclose(o.var(axis=1), 1, atol=1e-5)


def test_hot_order_and_prefix():
    freq = np.array([0.1, 0.5, 0.5, 0.0, 0.9, 0.1])
    perm = O.hot_order(freq)
    assert perm.tolist() == [4, 1, 2, 0, 5, 3]
    assert sorted(perm.tolist()) == list(range(6))
    fs = freq[perm]
    assert O.hot_prefix_len(fs, 1) == 3                  # 0.9, 0.5, 0.5
    assert O.hot_prefix_len(fs, 8) == 5                  # 1 - 0.9^8 = 0.57 >= 0.5
    assert O.hot_prefix_len(fs, 6) == 3                  # 1 - 0.9^6 = 0.469 < 0.5
    assert O.hot_prefix_len(fs, 7) == 5                  # 1 - 0.9^7 = 0.522


def test_permuted_layer_same_output():
    w, x = tiny_layer("reglu", seed=5)
    f = w["bias"].size
    rng = np.random.default_rng(1)
    perm = O.hot_order(rng.random(f))
    wp = O.permute_layer(w, perm)
    lg, lgp = (O.predictor_logits(x, v["p1"], v["p2"], v["thresh"]) for v in (w, wp))
    assert np.array_equal(lgp, lg[:, perm])
    b, bp = O.fire_bits(lg), O.fire_bits(lgp)
    idx, _ = O.compact(O.pack_mask(b), f)
    idxp, _ = O.compact(O.pack_mask(bp), f)
    assert sorted(perm[idxp].tolist()) == idx.tolist()
    assert np.allclose(O.sparse_ffn(x, wp, "reglu", bp, idxp), O.sparse_ffn(x, w, "reglu", b, idx),
                       rtol=0, atol=1e-12)


def test_hot_fraction_for_mass():
    assert O.hot_fraction_for_mass(np.array([8.0, 1.0, 1.0])) == pytest.approx(1 / 3)
    assert O.hot_fraction_for_mass(np.array([1.0, 1.0, 1.0, 1.0, 1.0])) == pytest.approx(0.8)
    assert O.hot_fraction_for_mass(np.array([4.0, 3.0, 2.0, 1.0])) == pytest.approx(0.75)
