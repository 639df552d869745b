"""Pins of the big-fuse oracle (pre-map from an external projection), "FlashInfer mHC module deep
dive" §3.1-3.3 (dot_mix and sqrsum partials summed over the split axis, rstd = 1/sqrt(sqrsum/k +
rms_eps)), §4 (with_prenorm: the sum of squares from the residual, k = 4H), §5.2 (reference math).

The pins: the whole pre-map oracle (C, pinned in test_oracle_pins.py) is reproduced when dot_mix
and sqrsum are the true projection and sum of squares; a hand-computed one-hot logit; splitting
the partials any way changes nothing; scaling sqrsum and k together changes nothing; zero dot_mix
gives the base logits; with_prenorm equals big_fuse on the residual's own sum of squares.
"""

import math

import numpy as np
import pytest

import oracle
from mhc_hyper_connection_02_b200 import inputs

RNG = np.random.default_rng(777)


def _split(a, S):
    """S random parts (fp64) that add up to a in fp64 order (the last part takes the remainder)."""
    parts = [RNG.standard_normal(a.shape) * (np.abs(a).mean() + 1.0) for _ in range(S - 1)]
    parts.append(a - sum(parts))
    return np.stack(parts)


def test_true_projection_reproduces_pre_map():
    """With dot_mix = R_flat . hc_fn and sqrsum = sum R^2, k = 4H: the pre-map itself."""
    w = inputs.custom(9, 24, seed=3)
    ss, rstd, raw = oracle.norm_project(w.R, w.hc_fn, rms_eps=1e-6)
    got = oracle.big_fuse(raw, ss, w.R, w.hc_scale, w.hc_base, 4 * w.H, rms_eps=1e-6)
    ref = oracle.pre(w.R, w.hc_fn, w.hc_scale, w.hc_base, rms_eps=1e-6)
    np.testing.assert_allclose(got["rstd"], ref["rstd"], rtol=1e-15)
    for key in ("logits", "pre", "post", "comb", "y"):
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(oracle.sum_of_squares(w.R), ss, rtol=1e-14)


def test_one_hot_logit_by_hand():
    """T=1: dot_mix = c e_j, sqrsum = s: l_j = c / sqrt(s/k + eps) * scale[g(j)] + base[j]."""
    k, s, c, eps = 64, 48.0, 0.75, 1e-6
    scale = np.array([0.5, 1.5, 2.0], np.float32)
    base = np.linspace(-0.3, 0.4, 24).astype(np.float32)
    R = np.zeros((1, 4, 16), np.uint16)
    for j, g in ((2, 0), (6, 1), (13, 2)):
        d = np.zeros((1, 24), np.float32)
        d[0, j] = c
        out = oracle.big_fuse(d, np.array([s], np.float32), R, scale, base, k, rms_eps=eps)
        expect = c / math.sqrt(s / k + eps) * float(scale[g]) + float(base[j])
        assert out["logits"][0, j] == pytest.approx(expect, rel=1e-14)
        others = [i for i in range(24) if i != j]
        np.testing.assert_allclose(out["logits"][0, others], base[others].astype(np.float64),
                                   rtol=0, atol=0)
    d = np.zeros((1, 24), np.float32)
    d[0, 1] = c
    out = oracle.big_fuse(d, np.array([s], np.float32), R, scale, base, k, rms_eps=eps,
                          pre_eps=1e-6)
    l1 = c / math.sqrt(s / k + eps) * 0.5 + float(base[1])
    assert out["pre"][0, 1] == pytest.approx(1.0 / (1.0 + math.exp(-l1)) + 1e-6, rel=1e-14)


@pytest.mark.parametrize("S", [2, 4, 8, 16])
def test_split_invariance(S):
    w = inputs.custom(7, 16, seed=S)
    ss, _, raw = oracle.norm_project(w.R, w.hc_fn)
    one = oracle.big_fuse(raw, ss, w.R, w.hc_scale, w.hc_base, 4 * w.H)
    many = oracle.big_fuse(_split(raw, S), _split(ss, S), w.R, w.hc_scale, w.hc_base, 4 * w.H)
    for key in ("logits", "pre", "post", "comb", "y"):
        np.testing.assert_allclose(many[key], one[key], rtol=1e-9, atol=1e-11)


def test_k_and_sqrsum_scale_together():
    w = inputs.custom(5, 8, seed=11)
    ss, _, raw = oracle.norm_project(w.R, w.hc_fn)
    a = oracle.big_fuse(raw, ss, w.R, w.hc_scale, w.hc_base, 32, rms_eps=1e-6)
    b = oracle.big_fuse(raw, ss * 4.0, w.R, w.hc_scale, w.hc_base, 128, rms_eps=1e-6)
    for key in ("rstd", "pre", "post", "comb", "y"):
        np.testing.assert_allclose(b[key], a[key], rtol=1e-14, atol=1e-16)
    # A different k alone does change rstd: sqrt(ss/32 + eps) / sqrt(ss/64 + eps) -> sqrt(2).
    c = oracle.big_fuse(raw, ss, w.R, w.hc_scale, w.hc_base, 64, rms_eps=1e-6)
    np.testing.assert_allclose(c["rstd"] / a["rstd"], math.sqrt(2.0), rtol=1e-5)


def test_zero_dot_mix_gives_base_logits():
    w = inputs.custom(3, 8, seed=5)
    out = oracle.big_fuse(np.zeros((2, 3, 24), np.float32), np.full((2, 3), 5.0, np.float32), w.R,
                          w.hc_scale, w.hc_base, 32)
    np.testing.assert_array_equal(out["logits"], np.broadcast_to(w.hc_base.astype(np.float64),
                                                                 (3, 24)))


def test_with_prenorm_is_big_fuse_on_own_sum_of_squares():
    w = inputs.custom(6, 40, seed=2)
    _, _, raw = oracle.norm_project(w.R, w.hc_fn)
    d = raw.astype(np.float32)
    a = oracle.big_fuse_with_prenorm(d, w.R, w.hc_scale, w.hc_base)
    x = oracle.bf16_bits_to_f64(w.R).reshape(6, -1)
    b = oracle.big_fuse(d, (x * x).sum(axis=1), w.R, w.hc_scale, w.hc_base, 4 * 40)
    for key in ("rstd", "pre", "post", "comb", "y"):
        np.testing.assert_allclose(a[key], b[key], rtol=1e-13, atol=1e-15)
