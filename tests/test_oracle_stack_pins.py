"""Pins of the oracle's composition steps against hand-built values and an exact
rational brute force: the widening of a Q4_0 layer (its neuron-major down plane must be
transposed into W_down[j][i]), one layer step, and a two-layer, two-token stack (the
second layer must see the first layer's glued output, and each token's y must use only
that token's own mask bits)."""
import math
from fractions import Fraction as Fr

import numpy as np
import pytest

from oracle import ffn as O
import test_oracle_pins as P


# ----------------------------------------------------------------- Q4_0 widening
def _q4_layer_by_hand(f=2, d=32):
    """Codes chosen so that neuron 0's and neuron 1's rows differ element by element,
    and so do the two nibble halves of every block."""
    q = np.zeros((f, d), np.int64)
    for i in range(f):
        for j in range(d):
            q[i, j] = (3 * j + 5 * i + 1 + 7 * ((j // 16) % 2)) % 16
    nib = np.zeros((f, d // 32, 16), np.uint8)
    for i in range(f):
        for blk in range(d // 32):
            for jj in range(16):
                nib[i, blk, jj] = q[i, 32 * blk + jj] | (q[i, 32 * blk + 16 + jj] << 4)
    sc = np.array([[0.5 * (i + 1)] * (d // 32) for i in range(f)], np.float16)
    return q, nib, sc


def test_q4_down_plane_is_transposed():
    """The Q4_0 down weights arrive neuron-major ([f][d/32] blocks); W_down[j][i] must be
    element j of neuron i's row, the value (q - 8) * scale."""
    for f, d in ((2, 32), (32, 32)):                     # the square case has no shape check
        q, nib, sc = _q4_layer_by_hand(f, d)
        t = {"q_up": nib, "s_up": sc, "q_down": nib, "s_down": sc,
             "bias": np.zeros(f, np.float32), "p1": np.zeros((d, 1), np.float32),
             "p2": np.zeros((1, f), np.float32), "thresh": np.zeros(f, np.float32)}
        w = O.layer_weights_f64(t, "relu")
        assert w["w_down"].shape == (d, f)
        for i in range(f):
            for j in range(d):
                want = (q[i, j] - 8) * float(sc[i, j // 32])
                assert w["w_down"][j, i] == want
                assert w["w_up"][i, j] == want


def test_q4_layer_output_by_hand():
    """One Q4_0 ReLU layer with one active neuron: y = a * (neuron's down row)."""
    f, d = 2, 32
    q, nib, sc = _q4_layer_by_hand(f, d)
    t = {"q_up": nib, "s_up": sc, "q_down": nib, "s_down": sc,
         "bias": np.array([100.0, 0.0], np.float32), "p1": np.zeros((d, 1), np.float32),
         "p2": np.zeros((1, f), np.float32), "thresh": np.zeros(f, np.float32)}
    w = O.layer_weights_f64(t, "relu")
    x = np.zeros((1, d))
    x[0, 3] = 1.0
    up0 = (q[0, 3] - 8) * 0.5
    a0 = max(0.0, up0 + 100.0)
    y = O.sparse_ffn(x, w, "relu", np.array([[True, False]]), np.array([0]))
    want = [a0 * (q[0, j] - 8) * 0.5 for j in range(d)]
    assert y[0].tolist() == want


# ----------------------------------------------------------------- stack
def _brute_layer(x_rows, w, act):
    """Exact logits, per-token bits, union list and per-token y (rationals)."""
    f = w["bias"].size
    out = []
    for xr in x_rows:
        lg = P.brute_logits(xr, w)
        bits = [v > 0 for v in lg]
        y = P.brute_y(xr, w, act, [i for i in range(f) if bits[i]])
        out.append((lg, bits, y))
    union = sorted({i for (_, bits, _) in out for i in range(f) if bits[i]})
    return out, union


def _glue_closed_form(x_row, y_row):
    v = [float(a) + float(b) for a, b in zip(x_row, y_row)]
    d = len(v)
    mean = math.fsum(v) / d
    var = math.fsum((a - mean) ** 2 for a in v) / d
    return [(a - mean) / math.sqrt(var + 1e-6) for a in v]


@pytest.mark.parametrize("act", ["relu", "reglu"])
def test_two_layer_two_token_stack(act):
    """decode_stack against a hand-composed brute force.  Layer 1 is exact in rationals
    up to the glue; the glue is its closed form with exactly rounded sums (fp32 output,
    within 2 ulp); layer 2 is the exact rational step of the oracle's own layer-1 output,
    compared within 1e-12 (its inputs carry full fp32 mantissas)."""
    w1, x = P.tiny_layer(act, seed=21)
    w2, _ = P.tiny_layer(act, seed=22)
    x = x[:2]
    tr = O.decode_stack(x, [w1, w2], act, "f32")
    assert len(tr) == 2
    b1, union1 = _brute_layer(x, w1, act)
    assert any(a != b for a, b in zip(b1[0][1], b1[1][1])), "the two tokens must fire differently"
    assert tr[0]["idx"].tolist() == union1 and tr[0]["count"] == len(union1)
    for b in range(2):
        lg, bits, y = b1[b]
        assert tr[0]["logits"][b].tolist() == [float(v) for v in lg]
        assert tr[0]["bits"][b].tolist() == bits
        assert tr[0]["y"][b].tolist() == [float(v) for v in y]
        g = np.float32(_glue_closed_form(x[b], y))
        got = tr[0]["x_next"][b]
        assert got.dtype == np.float32
        assert np.all(np.abs(got - g) <= 2 * np.spacing(np.abs(g))), (got, g)
    # the second layer runs on the first layer's glued output
    assert np.array_equal(tr[1]["x_in"], tr[0]["x_next"])
    x2 = tr[0]["x_next"].astype(np.float64)
    b2, union2 = _brute_layer(x2, w2, act)
    assert tr[1]["idx"].tolist() == union2
    for b in range(2):
        lg, bits, y = b2[b]
        assert tr[1]["bits"][b].tolist() == bits
        ref_l = np.array([float(v) for v in lg])
        assert np.max(np.abs(tr[1]["logits"][b] - ref_l)) <= 1e-12 * max(1.0, np.max(np.abs(ref_l)))
        ref_y = np.array([float(v) for v in y])
        assert np.max(np.abs(tr[1]["y"][b] - ref_y)) <= 1e-12 * max(1.0, np.max(np.abs(ref_y)))


def test_layer_step_record():
    """layer_step's record: words are the packed bits, idx/count their compaction, and
    x_next the glue of (x, y) rounded to the activation dtype."""
    w, x = P.tiny_layer("relu", seed=4)
    rec = O.layer_step(x, w, "relu", "f16")
    assert np.array_equal(rec["words"], O.pack_mask(rec["logits"] > 0))
    assert np.array_equal(rec["bits"], rec["logits"] > 0)
    idx, cnt = O.compact(rec["words"], w["bias"].size)
    assert np.array_equal(rec["idx"], idx) and rec["count"] == cnt
    assert rec["x_next"].dtype == np.float16
    for b in range(x.shape[0]):
        g = np.float32(_glue_closed_form(x[b], rec["y"][b])).astype(np.float16)
        assert np.all(np.abs(rec["x_next"][b].astype(np.float64) - g.astype(np.float64))
                      <= np.spacing(np.abs(g)).astype(np.float64))
