"""Pins of the backward oracle (oracle/backward.py) against torch autograd on an independent float64
restatement of the forward maps ("FlashInfer mHC module deep dive" §2.1 post-map, §3.4 / §5.2
pre-map: RMS over 4H, projection, scale groups, sigmoid gates, softmax + eps then Sinkhorn rounds,
aggregate). Autograd derives the derivatives itself, so a dropped term, wrong sign or transposed
operand in the oracle's hand-written reverse pass fails here. Also pins the Sinkhorn forward states
the VJP replays against the C oracle's Sinkhorn."""

import numpy as np
import pytest
import torch

import oracle
from oracle import backward
from mhc_hyper_connection_02_b200 import inputs

RNG = np.random.default_rng(2024)


def bits_of(t):
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def rand_bits(shape, scale=1.0):
    return bits_of(torch.from_numpy((RNG.standard_normal(shape) * scale).astype(np.float32)))


def f64(bits):
    return torch.from_numpy(oracle.bf16_bits_to_f64(bits))


def torch_pre(R, W, sc, bs, rms_eps, pre_eps, post_mult, iters, eps):
    T, _, H = R.shape
    X = R.reshape(T, 4 * H)
    rstd = torch.rsqrt((X * X).sum(1) / (4 * H) + rms_eps)
    g = torch.tensor([0] * 4 + [1] * 4 + [2] * 16)
    lg = (X @ W) * rstd[:, None] * sc[g][None, :] + bs[None, :]
    pre = torch.sigmoid(lg[:, :4]) + pre_eps
    post = post_mult * torch.sigmoid(lg[:, 4:8])
    c = lg[:, 8:].reshape(T, 4, 4)
    A = torch.softmax(c, dim=2) + eps
    for _ in range(iters):
        A = A / A.sum(dim=2, keepdim=True)
        A = A / A.sum(dim=1, keepdim=True)
    y = (pre[:, :, None] * R).sum(1)
    return y, pre, post, A


@pytest.mark.parametrize("T,H,iters", [(3, 8, 20), (2, 5, 3), (4, 16, 50)])
def test_pre_backward_matches_autograd(T, H, iters):
    w = inputs.custom(T, H, seed=T * 10 + H)
    R = f64(w.R).requires_grad_(True)
    W = torch.from_numpy(w.hc_fn.astype(np.float64)).requires_grad_(True)
    sc = torch.from_numpy(w.hc_scale.astype(np.float64)).requires_grad_(True)
    bs = torch.from_numpy(w.hc_base.astype(np.float64)).requires_grad_(True)
    kw = dict(rms_eps=1e-6, pre_eps=1e-6, post_mult=2.0, iters=iters, eps=1e-6)
    y, pre, post, comb = torch_pre(R, W, sc, bs, **kw)
    d_y = rand_bits((T, H))
    d_pre = RNG.standard_normal((T, 4)).astype(np.float32)
    d_post = RNG.standard_normal((T, 4)).astype(np.float32)
    d_comb = RNG.standard_normal((T, 4, 4)).astype(np.float32)
    loss = ((y * f64(d_y)).sum() + (pre * torch.from_numpy(d_pre.astype(np.float64))).sum()
            + (post * torch.from_numpy(d_post.astype(np.float64))).sum()
            + (comb * torch.from_numpy(d_comb.astype(np.float64))).sum())
    loss.backward()
    dR, dW, dsc, dbs = backward.pre_backward(d_y, d_pre, d_post, d_comb, w.R, w.hc_fn, w.hc_scale,
                                             w.hc_base, **kw)
    np.testing.assert_allclose(dR, R.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dW, W.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dsc, sc.grad.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dbs, bs.grad.numpy(), rtol=1e-9, atol=1e-12)


def test_post_backward_matches_autograd():
    T, H = 3, 7
    x = rand_bits((T, H))
    Rb = rand_bits((T, 4, H))
    post = RNG.standard_normal((T, 4)).astype(np.float32)
    comb = RNG.standard_normal((T, 4, 4)).astype(np.float32)
    X = f64(x).requires_grad_(True)
    R = f64(Rb).requires_grad_(True)
    P = torch.from_numpy(post.astype(np.float64)).requires_grad_(True)
    C = torch.from_numpy(comb.astype(np.float64)).requires_grad_(True)
    out = X[:, None, :] * P[:, :, None] + torch.einsum("toh,ton->tnh", R, C)
    d_out = rand_bits((T, 4, H))
    (out * f64(d_out)).sum().backward()
    dx, dR, dp, dc = backward.post_backward(d_out, x, Rb, post, comb)
    for got, want in ((dx, X.grad), (dR, R.grad), (dp, P.grad), (dc, C.grad)):
        np.testing.assert_allclose(got, want.numpy(), rtol=1e-12, atol=1e-14)


def test_sinkhorn_states_match_c_oracle():
    lg = RNG.standard_normal((5, 4, 4)) * 2
    for t in range(5):
        _, states = backward._sinkhorn_forward_states(lg[t], 20, 1e-6)
        np.testing.assert_allclose(states[-1][2], oracle.sinkhorn(lg[t][None], 20, 1e-6)[0],
                                   rtol=1e-13, atol=1e-15)


def test_sinkhorn_vjp_finite_differences():
    """Central differences of the C oracle's Sinkhorn against the VJP."""
    lg = RNG.standard_normal((4, 4))
    dc = RNG.standard_normal((4, 4))
    dl = backward.sinkhorn_vjp(lg, dc, 20, 1e-6)
    h = 1e-6
    for o in range(4):
        for n in range(4):
            e = np.zeros((4, 4))
            e[o, n] = h
            fp = (oracle.sinkhorn((lg + e)[None], 20, 1e-6)[0] * dc).sum()
            fm = (oracle.sinkhorn((lg - e)[None], 20, 1e-6)[0] * dc).sum()
            assert abs((fp - fm) / (2 * h) - dl[o, n]) < 1e-6
