"""Second, independent restatement of the mHC maps in NumPy fp64. TEST INFRASTRUCTURE ONLY.

Written separately from ``mhc_oracle.c`` (vectorised over tokens instead of loops) so that the two
can be checked against each other on tiny inputs. Sources as in ``mhc_oracle.h``:
"FlashInfer mHC module deep dive" §2.1, §3.4, §5.2; the rwkv-ops ``mhu_jax.py`` docstrings of
``mhc_pre_op`` and ``sinkhorn_knopp``; ``glm5next_mhc.rs`` ``glm_hc_post``.
"""

from __future__ import annotations

import numpy as np


def widen_bf16(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def sinkhorn(logits, iters, eps):
    """logits [T,4,4] -> doubly-stochastic estimate: row softmax plus eps on every entry, then
    `iters` rounds of (rows / row sums, columns / column sums)."""
    lg = np.asarray(logits, dtype=np.float64).reshape(-1, 4, 4)
    ex = np.exp(lg - lg.max(axis=2, keepdims=True))
    A = ex / ex.sum(axis=2, keepdims=True) + eps
    for _ in range(iters):
        A = A / A.sum(axis=2, keepdims=True)
        A = A / A.sum(axis=1, keepdims=True)
    return A


def pre(R_bits, hc_fn, scale, base, rms_eps=1e-6, pre_eps=0.0, post_mult=2.0, iters=20, eps=1e-6):
    R = widen_bf16(R_bits)                       # [T,4,H]
    T, hc, H = R.shape
    X = R.reshape(T, hc * H)                     # k = i*H + h
    W = np.asarray(hc_fn, dtype=np.float64)      # [4H,24]
    rstd = 1.0 / np.sqrt((X * X).sum(axis=1) / (hc * H) + rms_eps)
    mixes = (X @ W) * rstd[:, None]
    s = np.asarray(scale, dtype=np.float64)
    b = np.asarray(base, dtype=np.float64)
    group_scale = np.concatenate([np.full(4, s[0]), np.full(4, s[1]), np.full(16, s[2])])
    logits = mixes * group_scale[None, :] + b[None, :]
    sig = lambda v: 1.0 / (1.0 + np.exp(-v))  # noqa: E731
    pre_c = sig(logits[:, 0:4]) + pre_eps
    post_c = post_mult * sig(logits[:, 4:8])
    comb = sinkhorn(logits[:, 8:24].reshape(T, 4, 4), iters, eps)
    y = np.einsum("ti,tih->th", pre_c, R)
    return {"rstd": rstd, "logits": logits, "pre": pre_c, "post": post_c, "comb": comb, "y": y}


def post(x_bits, R_bits, post_coef, comb):
    x = widen_bf16(x_bits)                       # [T,H]
    R = widen_bf16(R_bits)                       # [T,4,H]
    p = np.asarray(post_coef, dtype=np.float32).astype(np.float64).reshape(-1, 4)
    c = np.asarray(comb, dtype=np.float32).astype(np.float64).reshape(-1, 4, 4)
    return x[:, None, :] * p[:, :, None] + np.einsum("toh,ton->tnh", R, c)
