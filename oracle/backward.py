"""Oracle of the backward passes (fp64). TEST INFRASTRUCTURE ONLY.

The pages name backward kernels (rwkv-ops mhu_jax.py: _mhc_post_op_ffi_bwd returns the gradients of
layer_out, x_expanded, H_post and H_res; mhc_pre_op has a custom VJP over x_expanded and the raw
mix logits) but print no formulas. These are the exact derivatives of the forward definitions the
rest of the oracle follows ("FlashInfer mHC module deep dive" §2.1 post-map, §3.4 / §5.2 pre-map),
written out step by step in reverse order:

post-map  out[n][h] = x[h] post[n] + sum_o R[o][h] comb[o][n]
    d_x[h] = sum_n post[n] d_out[n][h];   d_R[o][h] = sum_n comb[o][n] d_out[n][h]
    d_post[n] = sum_h x[h] d_out[n][h];   d_comb[o][n] = sum_h R[o][h] d_out[n][h]

pre-map   X = R_flat; ss = sum X^2; rstd = (ss/K + rms_eps)^(-1/2); raw = X . hc_fn; m = raw rstd;
          l = m scale[g] + base; pre = sigmoid(l[0:4]) + pre_eps; post = post_mult sigmoid(l[4:8]);
          comb = Sinkhorn(l[8:24]); y = sum_i pre_i R_i
    with upstream gradients d_y [T,H], d_pre, d_post [T,4], d_comb [T,4,4]:
    d_pre_i += sum_h d_y[h] R_i[h];  d_l = d_pre sig'(l) | d_post post_mult sig'(l) | Sinkhorn VJP;
    d_scale[g] += sum_{j in g} d_l_j m_j;  d_base += d_l;  d_m = d_l scale[g];
    d_raw = d_m rstd;  d_rstd = sum_j d_m_j raw_j;  d_ss = -rstd^3 / (2K) d_rstd;
    d_X = d_y-part (pre_i d_y[h]) + d_raw . hc_fn^T + 2 X d_ss;  d_hc_fn = X^T d_raw.

Sinkhorn VJP: the forward is P = softmax(l) over each row, A0 = P + eps, then per round
B = A / rowsum(A), C = B / colsum(B). A normalisation Y = Z / s, s the sum of the row (or column)
of Z, has dZ = (dY - sum(dY * Y) over that row or column) / s. The softmax has
dl = P * (dA0 - sum_n dA0 * P) per row (the row-max shift cancels out of it).
"""

from __future__ import annotations

import numpy as np

from .c_oracle import bf16_bits_to_f64


def post_backward(d_out, x, R, post, comb):
    """d_out, R: uint16 bf16 bits [T,4,H]; x: bits [T,H]; post [T,4], comb [T,4,4] fp32.
    Returns fp64 d_x [T,H], d_R [T,4,H], d_post [T,4], d_comb [T,4,4]."""
    dO = bf16_bits_to_f64(d_out)
    X = bf16_bits_to_f64(x)
    Rf = bf16_bits_to_f64(R)
    P = np.asarray(post, dtype=np.float64).reshape(-1, 4)
    Cm = np.asarray(comb, dtype=np.float64).reshape(-1, 4, 4)
    d_x = np.einsum("tn,tnh->th", P, dO)
    d_R = np.einsum("ton,tnh->toh", Cm, dO)
    d_post = np.einsum("th,tnh->tn", X, dO)
    d_comb = np.einsum("toh,tnh->ton", Rf, dO)
    return d_x, d_R, d_post, d_comb


def _sinkhorn_forward_states(lg, iters, eps):
    """lg [4,4] fp64 logits. Returns the row softmax P and per round (B, rowsum, C, colsum)."""
    ex = np.exp(lg - lg.max(axis=1, keepdims=True))
    P = ex / ex.sum(axis=1, keepdims=True)
    A = P + eps
    states = []
    for _ in range(iters):
        rs = A.sum(axis=1, keepdims=True)
        B = A / rs
        cs = B.sum(axis=0, keepdims=True)
        C = B / cs
        states.append((B, rs, C, cs))
        A = C
    return P, states


def sinkhorn_vjp(lg, d_comb, iters, eps):
    """Gradient of Sinkhorn(lg) (fixed rounds) with respect to the logits lg [4,4]."""
    P, states = _sinkhorn_forward_states(lg, iters, eps)
    dA = np.array(d_comb, dtype=np.float64)
    for B, rs, C, cs in reversed(states):
        # C = B / cs (column normalisation)
        dB = (dA - (dA * C).sum(axis=0, keepdims=True)) / cs
        # B = A / rs (row normalisation)
        dA = (dB - (dB * B).sum(axis=1, keepdims=True)) / rs
    # A0 = P + eps, P = softmax(lg) per row
    return P * (dA - (dA * P).sum(axis=1, keepdims=True))


def pre_backward(d_y, d_pre, d_post, d_comb, R, hc_fn, scale, base, rms_eps=1e-6, pre_eps=0.0,
                 post_mult=2.0, iters=20, eps=1e-6, parts=False):
    """d_y: bits [T,H] (or None); d_pre, d_post [T,4], d_comb [T,4,4] fp32 (or None); R bits
    [T,4,H]; hc_fn [4H,24], scale [3], base [24] fp32. Returns fp64 d_R [T,4,H], d_hc_fn [4H,24],
    d_scale [3], d_base [24] (and, with parts=True, a dict of per-token intermediates)."""
    T, _, H = R.shape
    K = 4 * H
    X = bf16_bits_to_f64(R).reshape(T, K)
    W = np.asarray(hc_fn, dtype=np.float64)
    sc = np.asarray(scale, dtype=np.float64)
    bs = np.asarray(base, dtype=np.float64)
    g = np.array([0] * 4 + [1] * 4 + [2] * 16)
    ss = (X * X).sum(axis=1)
    rstd = 1.0 / np.sqrt(ss / K + rms_eps)
    raw = X @ W
    m = raw * rstd[:, None]
    lg = m * sc[g][None, :] + bs[None, :]
    sig = 1.0 / (1.0 + np.exp(-lg[:, :8]))
    pre = sig[:, :4] + pre_eps
    dY = np.zeros((T, H)) if d_y is None else bf16_bits_to_f64(d_y)
    dP = np.zeros((T, 4)) if d_pre is None else np.asarray(d_pre, np.float64).reshape(T, 4)
    dQ = np.zeros((T, 4)) if d_post is None else np.asarray(d_post, np.float64).reshape(T, 4)
    dC = np.zeros((T, 4, 4)) if d_comb is None else np.asarray(d_comb, np.float64).reshape(T, 4, 4)
    Rf = X.reshape(T, 4, H)
    d_pre_tot = dP + np.einsum("th,tih->ti", dY, Rf)
    dl = np.zeros((T, 24))
    dl[:, :4] = d_pre_tot * sig[:, :4] * (1.0 - sig[:, :4])
    dl[:, 4:8] = dQ * post_mult * sig[:, 4:8] * (1.0 - sig[:, 4:8])
    for t in range(T):
        dl[t, 8:] = sinkhorn_vjp(lg[t, 8:].reshape(4, 4), dC[t], iters, eps).reshape(16)
    d_base = dl.sum(axis=0)
    d_scale = np.array([(dl[:, g == k] * m[:, g == k]).sum() for k in range(3)])
    dm = dl * sc[g][None, :]
    d_raw = dm * rstd[:, None]
    d_rstd = (dm * raw).sum(axis=1)
    d_ss = -0.5 * rstd ** 3 / K * d_rstd
    dX = d_raw @ W.T + 2.0 * X * d_ss[:, None]
    dX = dX.reshape(T, 4, H) + pre[:, :, None] * dY[:, None, :]
    d_W = X.T @ d_raw
    if parts:  # intermediate per-token quantities (used by tests to size error bounds)
        return dX, d_W, d_scale, d_base, {"dl": dl, "m": m, "d_raw": d_raw, "d_ss": d_ss,
                                          "pre": pre, "X": X}
    return dX, d_W, d_scale, d_base
