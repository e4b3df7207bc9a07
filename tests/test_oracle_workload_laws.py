"""Closed forms of the synthetic workloads, checked through the oracle.

The firing law, bias and activation mass have closed forms for Gaussian inputs, so
measuring them through the oracle's pre-activations and activations pins both the
generator and the oracle's activation arithmetic (a dropped or sign-flipped bias, or
ReLU applied to the wrong operand, moves the measured rates far outside the bands)."""
import math
import os

import numpy as np
import pytest
import torch
from scipy.stats import norm

import pi_synth as S
from oracle import ffn as O
from conftest import GOLDEN

N_SAMPLES = 4096


def _layer_np(w, layer=0):
    L = S.make_layer(w, layer, "cpu")
    return L, O.layer_weights_f64(L.to_numpy(), w.act)


def _samples(w, n=N_SAMPLES, stream=7):
    return S.make_inputs(w.with_(x_dtype="f32"), n, "cpu", stream_id=stream).double().numpy()


@pytest.mark.parametrize("wl", [S.FFN512_CAL,
                                S.scaled(S.LLAMA2_7B, "llama7b_law_d128", 1, 128, 11008, 64),
                                S.scaled(S.LLAMA2_70B_Q4, "llama70b_law_d256", 1, 256, 4096, 64)])
def test_firing_rate_matches_law(wl):
    L, w = _layer_np(wl)
    x = _samples(wl)
    rate = O.true_mask(x, w, wl.act).mean(axis=0)
    p = L.probs
    band = 4.0 * np.sqrt(p * (1 - p) / x.shape[0])
    ok = np.abs(rate - p) <= band
    assert ok.mean() >= 0.999, (ok.size - ok.sum(), ok.size)
    # mean density within 0.5 percentage points of the configured mean
    assert abs(rate.mean() - p.mean()) < 0.005
    if wl.mean_p is not None:
        assert abs(p.mean() - wl.mean_p) < 1e-9


def test_power_law_slope_recovered():
    wl = S.FFN512_CAL
    L, w = _layer_np(wl)
    x = _samples(wl)
    rate = np.sort(O.true_mask(x, w, wl.act).mean(axis=0))[::-1]
    c = S.law_constant(wl)
    n_cap = int(np.sum(S.powerlaw_by_rank(wl.d_ff, wl.alpha, c) >= wl.p_cap))
    ranks = np.arange(n_cap + 1, wl.d_ff // 10)
    slope = np.polyfit(np.log(ranks + 1.0), np.log(rate[ranks]), 1)[0]
    assert abs(-slope - wl.alpha) < 0.05, slope


def test_literal_constant_gives_sparse_law():
    """The single-layer workload's literal constant 0.6 gives a mean firing
    probability near 0.35 %, far sparser than the ~90 % sparsity it is said to give;
    the calibrated constant restores a mean of 0.10."""
    p_lit = S.powerlaw_by_rank(2048, 0.9, 0.6)
    assert 0.003 < p_lit.mean() < 0.004
    c = S.calibrate_c(2048, 0.9, 0.10)
    assert abs(c - 24.27) < 0.01


def _expected_relu_mass(norms, p):
    a = norm.ppf(p)
    return norms * (norm.pdf(a) + a * p)


def test_activation_mass_closed_form():
    """E[max(0, w.x + b)] = ||w|| (phi(a) + a p) with a = Phi^-1(p), for x ~ N(0, I)."""
    wl = S.FFN512_CAL
    L, w = _layer_np(wl)
    x = _samples(wl, n=8192, stream=9)
    emp = O.activations(x, w, "relu", np.arange(wl.d_ff)).mean(axis=0)
    exp = _expected_relu_mass(np.linalg.norm(w["w_up"], axis=1), L.probs)
    sd = np.sqrt(np.maximum(O.activations(x, w, "relu", np.arange(wl.d_ff)).var(axis=0), 1e-30) / x.shape[0])
    z = (emp - exp) / np.maximum(sd, 1e-12)
    assert np.mean(np.abs(z) < 4.5) > 0.998
    assert abs(emp.sum() / exp.sum() - 1) < 0.01


def _golden_hot():
    rows = {}
    with open(os.path.join(GOLDEN, "hot_set_statistic.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                name, frac, share = line.split()
                rows[name] = (float(frac), float(share))
    return rows


def test_hot_set_statistic_against_pages():
    """The Llama-2-70B-shaped law (exponent 0.7, 85 % sparse) is meant to reproduce the
    pages' 43 % of neurons carrying 80 % of the activation mass.  Computed from the
    closed-form per-neuron mass (equal row norms, so mass ~ phi(a) + a p), the law
    gives 0.40; accept 0.35 .. 0.50 around the printed 0.43."""
    g = _golden_hot()
    frac_pg, share = g["Llama-2-70B"]
    wl = S.LLAMA2_70B_Q4
    p = S.powerlaw_by_rank(wl.d_ff, wl.alpha, S.law_constant(wl))
    mass = _expected_relu_mass(np.ones_like(p), p)
    got = O.hot_fraction_for_mass(mass, share)
    assert abs(got - frac_pg) < 0.08 and 0.35 <= got <= 0.50, got
    # the OPT-30B figure (26 %) is below the 7B/40B/175B-shaped laws' hot fractions
    # (~0.2-0.3), the same regime
    frac_opt, _ = g["OPT-30B"]
    for w2 in (S.LLAMA2_7B, S.FALCON_40B, S.OPT_175B):
        p2 = S.powerlaw_by_rank(w2.d_ff, w2.alpha, S.law_constant(w2))
        h = O.hot_fraction_for_mass(_expected_relu_mass(np.ones_like(p2), p2), share)
        assert 0.1 < h < 0.4 and abs(h - frac_opt) < 0.12, (w2.name, h)


def test_rrls_fit_follows_stein():
    """Least squares of T = sign(w.x + b) on Gaussian x points along w (Stein's
    lemma): the population coefficient is s * w/||w|| with s = 2 phi(Phi^-1(p)), and
    with n samples in d dimensions the OLS noise has norm sqrt(sigma^2 d / n),
    sigma^2 = 4p(1-p) - s^2.  So cos(OLS column, w_i) ~ s / sqrt(s^2 + sigma^2 d/n)."""
    wl = S.FFN512_CAL
    L = S.make_layer(wl, 0, "cpu")
    from pi_synth.generate import _fit_rrls
    _, _, _, B = _fit_rrls(wl, L.w_up.float(), L.bias)
    W = L.w_up.double()
    cos = ((B.T * W).sum(1) / (B.norm(dim=0) * W.norm(dim=1))).numpy()
    p = L.probs
    s = 2 * norm.pdf(norm.ppf(p))
    sig2 = 4 * p * (1 - p) - s * s
    want = s / np.sqrt(s * s + sig2 * wl.d_model / wl.n_calib)
    sel = p >= 0.05
    assert sel.sum() > 50
    assert np.all(cos[sel] > want[sel] - 0.06), np.min(cos[sel] - want[sel])
    assert abs(np.mean(cos[sel] - want[sel])) < 0.02, np.mean(cos[sel] - want[sel])


def test_sketch_predictor_rates_follow_law():
    """The sketch predictor's thresholds are calibration quantiles, so on fresh inputs
    each neuron's predicted firing rate follows p_i (measured through the oracle's
    predictor), and the predicted density matches the configured mean."""
    wl = S.scaled(S.LLAMA2_7B, "llama7b_pred_d256", 1, 256, 2048, 32)
    L, w = _layer_np(wl)
    x = _samples(wl, n=8192, stream=3)
    rate = O.fire_bits(O.predictor_logits(x, w["p1"], w["p2"], w["thresh"])).mean(axis=0)
    p = L.probs
    band = 5.0 * np.sqrt(p * (1 - p) * (1.0 / x.shape[0] + 1.0 / wl.n_calib)) + 1.0 / wl.n_calib
    assert np.mean(np.abs(rate - p) <= band) > 0.998
    assert abs(rate.mean() - wl.mean_p) < 0.005
    # measured frequencies handed to the hot-neuron sort are these same rates
    assert np.allclose(L.freq.numpy(), p, atol=6 * math.sqrt(0.25 / wl.n_calib) + 1e-3)
