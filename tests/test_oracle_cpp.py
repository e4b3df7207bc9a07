"""The C++ oracle (oracle/pi_oracle.cpp) pinned on its own: exact rational brute force on
tiny layers, hand-built ReLU / ReGLU / Q4_0 cases, the binary16 values IEEE 754 fixes,
the glue's closed form and a two-layer, two-token stack; then checked against the
independent numpy statement (bit for bit on dyadic layers, within 1e-12 on the
synthetic ones); and its pins shown to have teeth by compiling copies of the source
with one planted mistake each."""
import os
import subprocess

import numpy as np
import pytest

import pi_synth as S
from oracle import cpp as OC
from oracle import ffn as O
import test_oracle_pins as P
import test_oracle_stack_pins as SP


def _f32_layer(w):
    """A tiny dyadic fp64 layer stored as fp32 (exact: small numerators over 2^k)."""
    t = {k: np.asarray(v, np.float32) for k, v in w.items()}
    assert all(np.array_equal(t[k].astype(np.float64), w[k]) for k in w)
    return t


# ----------------------------------------------------------------- pins
@pytest.mark.parametrize("act", ["relu", "reglu", "relu2"])
@pytest.mark.parametrize("seed", [0, 3])
def test_cpp_brute_force_exact(act, seed):
    w, x = P.tiny_layer(act, seed)
    L = OC.Layer(_f32_layer(w), act)
    f = w["bias"].size
    lg = L.predictor_logits(x)
    rec = L.layer_step(x, "f32")
    union = set()
    for b in range(x.shape[0]):
        bl = P.brute_logits(x[b], w)
        assert lg[b].tolist() == [float(v) for v in bl]
        bits = [v > 0 for v in bl]
        assert rec["bits"][b].tolist() == bits
        union |= {i for i in range(f) if bits[i]}
        assert rec["y"][b].tolist() == [float(v) for v in P.brute_y(x[b], w, act, [i for i in range(f) if bits[i]])]
        assert L.dense_ffn(x[b:b + 1])[0].tolist() == [float(v) for v in P.brute_y(x[b], w, act, range(f))]
    assert rec["idx"].tolist() == sorted(union) and rec["count"] == len(union)


def _hand_layer(act):
    w = P._one_neuron_layer(act)
    if act != "reglu":
        w.pop("w_gate", None)
    return OC.Layer(_f32_layer(w), act)


def test_cpp_relu_and_reglu_by_hand():
    x = np.array([[1.0, 1.0, 2.0, 0.5]])
    m = np.ones((1, 32), bool)
    assert _hand_layer("relu").sparse_ffn(x, m, [5]).tolist() == [[2.5, 0.0, -1.25, 5.0]]
    assert _hand_layer("relu").sparse_ffn(-x, m, [5]).tolist() == [[0.0, 0.0, 0.0, 0.0]]
    assert _hand_layer("relu2").sparse_ffn(x, m, [5]).tolist() == [[3.125, 0.0, -1.5625, 6.25]]
    x2 = np.array([[2.0, 1.0, 0.0, -1.0]])
    assert _hand_layer("reglu").sparse_ffn(x2, m, [5]).tolist() == [[-10.5, 0.0, 5.25, -21.0]]
    # token 0's bit is off: its y is exactly zero
    xx = np.vstack([x, x])
    mm = np.zeros((2, 32), bool)
    mm[1, 5] = True
    y = _hand_layer("relu").sparse_ffn(xx, mm, [5])
    assert y[0].tolist() == [0.0] * 4 and y[1].tolist() == [2.5, 0.0, -1.25, 5.0]


def test_cpp_q4_layer_by_hand():
    f, d = 2, 32
    q, nib, sc = SP._q4_layer_by_hand(f, d)
    t = {"q_up": nib, "s_up": sc, "q_down": nib, "s_down": sc,
         "bias": np.array([100.0, 0.0], np.float32), "p1": np.zeros((d, 1), np.float32),
         "p2": np.zeros((1, f), np.float32), "thresh": np.zeros(f, np.float32)}
    L = OC.Layer(t, "relu")
    x = np.zeros((1, d))
    x[0, 3] = 1.0
    a0 = (q[0, 3] - 8) * 0.5 + 100.0
    y = L.sparse_ffn(x, [[True, False]], [0])
    assert y[0].tolist() == [a0 * (q[0, j] - 8) * 0.5 for j in range(d)]
    # neuron 1 alone: its own row, scale 1.0
    x1 = np.zeros((1, d))
    x1[0, 0] = 1.0
    a1 = max(0.0, (q[1, 0] - 8) * 1.0)
    assert L.sparse_ffn(x1, [[False, True]], [1])[0].tolist() == [a1 * (q[1, j] - 8) * 1.0 for j in range(d)]


def test_cpp_binary16_values():
    """Values IEEE 754 binary16 fixes, decoded and encoded (round to nearest, ties even)."""
    cases = {0x3C00: 1.0, 0xC000: -2.0, 0x7BFF: 65504.0, 0x0001: 2.0 ** -24, 0x0400: 2.0 ** -14,
             0x03FF: 1023 * 2.0 ** -24, 0x3555: 0.333251953125, 0x8000: -0.0, 0x7C00: np.inf}
    for h, v in cases.items():
        assert OC.half_to_double(h) == v
        assert OC.float_to_half_bits(np.float32(v)) == h
    assert np.isnan(OC.half_to_double(0x7E00))
    # ties: 1 + 2^-11 lies halfway between 1 and 1 + 2^-10 -> even (1.0)
    assert OC.float_to_half_bits(np.float32(1 + 2.0 ** -11)) == 0x3C00
    assert OC.float_to_half_bits(np.float32(1 + 3 * 2.0 ** -11)) == 0x3C02
    assert OC.float_to_half_bits(np.float32(65519.0)) == 0x7BFF
    assert OC.float_to_half_bits(np.float32(65520.0)) == 0x7C00
    assert OC.float_to_half_bits(np.float32(2.0 ** -25)) == 0x0000          # tie -> even (0)
    assert OC.float_to_half_bits(np.float32(3 * 2.0 ** -25)) == 0x0002      # tie -> even (2)


def test_cpp_binary16_against_numpy():
    """Every binary16 pattern decodes as numpy's IEEE conversion does; fp32 values encode
    as numpy's cast does."""
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float64)
    got = np.array([OC.half_to_double(int(v)) for v in h])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got)) and np.array_equal(ref[~nan], got[~nan])
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.normal(size=20000) * 10, rng.random(20000) * 1e-4,
                           rng.random(2000) * 7e4]).astype(np.float32)
    with np.errstate(over="ignore"):
        ref16 = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ref16, np.array([OC.float_to_half_bits(float(v)) for v in vals], np.uint16))


def test_cpp_glue_closed_form():
    x = np.array([[3.0, -4.0, 0.0, 1.0]])
    out = OC.stack_glue(x, np.zeros((1, 4)), None)
    sd = np.sqrt(6.5 + 1e-6)
    assert np.allclose(out[0], [3 / sd, -4 / sd, 0.0, 1 / sd], rtol=1e-15, atol=0)
    y2 = np.array([[1.0, 0.0, 0.0, 2.0]]) + 10.0
    v = np.array([4.0, -4.0, 0.0, 3.0]) + 10.0
    w = v - v.mean()
    assert np.allclose(OC.stack_glue(x, y2, None)[0], w / np.sqrt(np.mean(w * w) + 1e-6), rtol=1e-15)
    assert OC.stack_glue(x, y2, "f16").dtype == np.float16


@pytest.mark.parametrize("act", ["relu", "reglu"])
def test_cpp_two_layer_stack(act):
    w1, x = P.tiny_layer(act, seed=21)
    w2, _ = P.tiny_layer(act, seed=22)
    x = x[:2]
    tr = OC.decode_stack(x, [OC.Layer(_f32_layer(w1), act), OC.Layer(_f32_layer(w2), act)], "f32")
    b1, union1 = SP._brute_layer(x, w1, act)
    assert tr[0]["idx"].tolist() == union1
    for b in range(2):
        lg, bits, y = b1[b]
        assert tr[0]["y"][b].tolist() == [float(v) for v in y]
        g = np.float32(SP._glue_closed_form(x[b], y))
        assert np.all(np.abs(tr[0]["x_next"][b] - g) <= 2 * np.spacing(np.abs(g)))
    assert np.array_equal(tr[1]["x_in"], tr[0]["x_next"].astype(np.float64))
    b2, union2 = SP._brute_layer(tr[0]["x_next"].astype(np.float64), w2, act)
    assert tr[1]["idx"].tolist() == union2
    for b in range(2):
        ref_y = np.array([float(v) for v in b2[b][2]])
        assert np.max(np.abs(tr[1]["y"][b] - ref_y)) <= 1e-12 * max(1.0, np.max(np.abs(ref_y)))


def test_cpp_compaction():
    rng = np.random.default_rng(11)
    for B, f, dens in [(1, 96, 0.1), (3, 2048, 0.05), (2, 64, 1.0), (1, 64, 0.0)]:
        bits = rng.random((B, f)) < dens
        words = O.pack_mask(bits)
        idx, n = OC.compact(words, f)
        assert idx.tolist() == np.flatnonzero(bits.any(axis=0)).tolist() and n == idx.size


# ----------------------------------------------------------------- against numpy
def test_cpp_matches_numpy_on_dyadic_layers():
    for act in ("relu", "reglu", "relu2"):
        w, x = P.tiny_layer(act, seed=9)
        L = OC.Layer(_f32_layer(w), act)
        r_np = O.layer_step(x, w, act, "f32")
        r_c = L.layer_step(x, "f32")
        for k in ("logits", "bits", "words", "idx", "y"):
            assert np.array_equal(r_np[k], r_c[k]), k
        assert np.array_equal(O.dense_ffn(x, w, act), L.dense_ffn(x))


@pytest.mark.parametrize("wl", [S.FFN512_CAL, S.scaled(S.LLAMA2_7B, "x16", 1, 512, 2048, 64),
                                S.scaled(S.FALCON_40B, "x16r", 1, 256, 1024, 32),
                                S.scaled(S.LLAMA2_70B_Q4, "xq4", 1, 512, 2048, 64)], ids=lambda w: w.name)
def test_cpp_matches_numpy_on_synthetic_layers(wl):
    t = S.make_layer(wl, 0, "cpu").to_numpy()
    hw = O.layer_weights_f64(t, wl.act)
    L = OC.Layer(t, wl.act)
    x = S.make_inputs(wl, 3, "cpu", stream_id=7).double().numpy()
    r_np = O.layer_step(x, hw, wl.act, wl.x_dtype)
    r_c = L.layer_step(x, wl.x_dtype)
    scale = max(1.0, np.max(np.abs(r_np["logits"])))
    assert np.max(np.abs(r_np["logits"] - r_c["logits"])) <= 1e-12 * scale
    clear = np.abs(r_np["logits"]) > 1e-9 * scale
    assert np.array_equal(r_np["bits"][clear], r_c["bits"][clear])
    if np.array_equal(r_np["bits"], r_c["bits"]):
        assert np.array_equal(r_np["idx"], r_c["idx"])
        assert np.max(np.abs(r_np["y"] - r_c["y"])) <= 1e-12 * np.max(np.abs(r_np["y"]))
    yd = O.dense_ffn(x, hw, wl.act)
    assert np.max(np.abs(yd - L.dense_ffn(x))) <= 1e-12 * np.max(np.abs(yd))


def test_cpp_results_do_not_depend_on_threads():
    wl = S.scaled(S.LLAMA2_7B, "thr", 1, 512, 2048, 64)
    L = OC.Layer(S.make_layer(wl, 0, "cpu").to_numpy(), wl.act)
    x = S.make_inputs(wl, 2, "cpu").double().numpy()
    n0 = OC.max_threads()
    try:
        OC.set_threads(1)
        a = L.layer_step(x, "f16")
        OC.set_threads(max(2, n0))
        b = L.layer_step(x, "f16")
    finally:
        OC.set_threads(n0)
    for k in ("logits", "y", "x_next"):
        assert np.array_equal(a[k], b[k])


# ----------------------------------------------------------------- planted mistakes
_MUTANTS = {
    "logit +t": [("logits[(size_t)b * f + i] = s - (double)L->thresh[i];",
                  "logits[(size_t)b * f + i] = s + (double)L->thresh[i];")],
    "fire >=": [("if (logits[(size_t)b * f + 32 * w + j] > 0.0) v |= 1u << j;",
                 "if (logits[(size_t)b * f + 32 * w + j] >= 0.0) v |= 1u << j;")],
    "no bias": [("const double a = up + (double)L->bias[i];", "const double a = up;")],
    "reglu clamps up": [("return (g > 0.0 ? g : 0.0) * up;", "return g * (up > 0.0 ? up : 0.0);")],
    "relu2 unsquared": [("return L->act == ACT_RELU2 ? rl * rl : rl;", "return rl;")],
    "q4 halves swapped": [("const int q = k < 16 ? (byte & 0x0F) : (byte >> 4);",
                           "const int q = k < 16 ? (byte >> 4) : (byte & 0x0F);")],
    "q4 without -8": [("return (double)(q - 8) * half_to_double", "return (double)q * half_to_double")],
    "down not transposed": [("return pvalue(L->w_dtype, L->w_down, (size_t)j * L->f + i);",
                             "return pvalue(L->w_dtype, L->w_down, (size_t)i * L->d + j);")],
    "token mask ignored": [("a[(size_t)b * count + k] = masks[(size_t)b * f + i] ? activation(L, x + (size_t)b * d, i) : 0.0;",
                            "a[(size_t)b * count + k] = activation(L, x + (size_t)b * d, i);")],
    "glue without residual": [("v[j] = x[(size_t)b * d + j] + y[(size_t)b * d + j];", "v[j] = y[(size_t)b * d + j];")],
    "compact intersection": [("uint32_t any = 0;", "uint32_t any = 1;"), ("any |= (words", "any &= (words")],
    "half exponent off by one": [("std::ldexp((double)(1024 + m), e - 25)", "std::ldexp((double)(1024 + m), e - 24)")],
    "half ties away": [("(rem == 0.5 && std::fmod(n, 2.0) == 1.0)", "(rem == 0.5)")],
}


def _cpp_pins():
    yield lambda: test_cpp_brute_force_exact("relu", 0)
    yield lambda: test_cpp_brute_force_exact("reglu", 3)
    yield lambda: test_cpp_brute_force_exact("relu2", 0)
    yield test_cpp_relu_and_reglu_by_hand
    yield test_cpp_q4_layer_by_hand
    yield test_cpp_binary16_values
    yield test_cpp_glue_closed_form
    yield lambda: test_cpp_two_layer_stack("relu")
    yield test_cpp_compaction


@pytest.fixture(scope="module")
def mutant_libs(tmp_path_factory):
    src = open(OC.SRC).read()
    out = {}
    d = tmp_path_factory.mktemp("oracle_mutants")
    for name, patches in _MUTANTS.items():
        s = src
        for old, new in patches:
            assert s.count(old) == 1, f"{name}: the text to patch is not in the oracle source once"
            s = s.replace(old, new)
        tag = "".join(ch if ch.isalnum() else "_" for ch in name)
        cpp, so = d / f"{tag}.cpp", d / f"{tag}.so"
        cpp.write_text(s)
        subprocess.run(["g++", *OC.FLAGS, "-o", str(so), str(cpp)], check=True)
        out[name] = str(so)
    return out


@pytest.mark.parametrize("name", sorted(_MUTANTS))
def test_cpp_mutant_is_caught(name, mutant_libs):
    OC.use_library(mutant_libs[name])
    try:
        failures = 0
        for pin in _cpp_pins():
            try:
                pin()
            except Exception:
                failures += 1
    finally:
        OC.use_library(None)
    assert failures > 0, f"no pin caught the planted mistake {name!r}"


def test_cpp_unmutated_passes_every_pin():
    for pin in _cpp_pins():
        pin()
