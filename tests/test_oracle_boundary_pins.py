"""Pins of the model-boundary oracle: expand (glm5next_mhc.rs glm_hc_expand), the unweighted head
(hc_head_mean) and the weighted head (hyper_connection_dispatch.rs hc_head_site; the reading: the
pre-map's first gate group with its own [4H,4] weights)."""

import math

import numpy as np
import pytest
import torch

import oracle
from oracle import boundary

RNG = np.random.default_rng(99)


def rand_bits(shape, scale=1.0):
    t = torch.from_numpy((RNG.standard_normal(shape) * scale).astype(np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bits(values):
    t = torch.tensor(np.asarray(values, dtype=np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t)
    return b.view(torch.int16).numpy().view(np.uint16).copy()


def test_expand_copies_every_stream():
    h = rand_bits((3, 10))
    s = boundary.expand(h)
    assert s.shape == (3, 4, 10)
    for i in range(4):
        np.testing.assert_array_equal(s[:, i], h)


def test_head_mean_hand_values():
    R = bits([[[1.0, -2.0], [3.0, 0.5], [-4.0, 0.25], [8.0, 1.25]]]).reshape(1, 4, 2)
    np.testing.assert_array_equal(boundary.head_mean(R), [[2.0, 0.0]])


def test_head_mean_of_expanded_row_is_the_row():
    h = rand_bits((4, 33))
    np.testing.assert_array_equal(boundary.head_mean(boundary.expand(h)),
                                  oracle.bf16_bits_to_f64(h))


def test_head_zero_weights_closed_form():
    """hc_fn = 0: w_i = sigmoid(base_i) + hc_eps for every token."""
    R = rand_bits((5, 4, 8))
    base = np.array([0.0, math.log(3.0), -1.0, 2.0], np.float32)
    out = boundary.head(R, np.zeros((32, 4), np.float32), np.ones(1, np.float32), base,
                        hc_eps=1e-6)
    want = 1.0 / (1.0 + np.exp(-base.astype(np.float64))) + 1e-6
    np.testing.assert_allclose(out["weights"], np.broadcast_to(want, (5, 4)), rtol=1e-15)
    assert out["weights"][0, 0] == pytest.approx(0.5 + 1e-6, rel=1e-15)
    assert out["weights"][0, 1] == pytest.approx(0.75 + 1e-6, rel=1e-7)


@pytest.mark.parametrize("stream", range(4))
def test_head_one_hot_selects_stream(stream):
    R = rand_bits((3, 4, 24))
    base = np.full(4, -40.0, np.float32)
    base[stream] = 40.0
    out = boundary.head(R, np.zeros((96, 4), np.float32), np.ones(1, np.float32), base, hc_eps=0.0)
    np.testing.assert_array_equal(oracle.round_bf16(out["y"]),
                                  oracle.bf16_bits_to_f64(R[:, stream]))


def test_head_basis_logit_by_hand():
    """T=1, H=2: R = 2 e_k, hc_fn row k = v: l = 2 v / sqrt(4/8 + eps) * scale + base."""
    H, k = 2, 5
    R = np.zeros((1, 4, H), np.uint16)
    R.reshape(-1)[k] = bits([2.0])[0]
    fn = np.zeros((4 * H, 4), np.float32)
    v = np.array([0.5, -0.25, 1.0, 0.125], np.float32)
    fn[k] = v
    out = boundary.head(R, fn, np.array([1.5], np.float32), np.zeros(4, np.float32),
                        norm_eps=1e-6)
    rstd = 1.0 / math.sqrt(4.0 / 8 + 1e-6)
    np.testing.assert_allclose(out["logits"][0], 2.0 * v.astype(np.float64) * rstd * 1.5, rtol=1e-14)


def test_head_matches_pre_map_first_gate_group():
    """The reading: the head equals the pre-map (pinned oracle) on hc_fn padded to 24 columns,
    scale (s, 1, 1), base (b, 0...), pre_eps = hc_eps."""
    T, H = 6, 16
    R = rand_bits((T, 4, H))
    fn = (RNG.standard_normal((4 * H, 4)) * 0.05).astype(np.float32)
    fn24 = np.zeros((4 * H, 24), np.float32)
    fn24[:, :4] = fn
    base = (RNG.standard_normal(4) * 0.3).astype(np.float32)
    b24 = np.zeros(24, np.float32)
    b24[:4] = base
    out = boundary.head(R, fn, np.array([0.8], np.float32), base, norm_eps=1e-6, hc_eps=1e-6)
    ref = oracle.pre(R, fn24, np.array([0.8, 1, 1], np.float32), b24, rms_eps=1e-6, pre_eps=1e-6)
    np.testing.assert_allclose(out["weights"], ref["pre"], rtol=1e-12)
    np.testing.assert_allclose(out["y"], ref["y"], rtol=1e-12, atol=1e-14)
