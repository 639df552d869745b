"""Oracle of the pre-map from an external projection (fp64). TEST INFRASTRUCTURE ONLY.

"FlashInfer mHC module deep dive" §3.1-3.3 (mhc_pre_big_fuse): dot_mix [num_splits, T, 24] and
sqrsum [num_splits, T] are partial sums that the entry adds over the split axis; the RMS factor is
rstd = 1 / sqrt(sqrsum / k + rms_eps) with k passed in; the logits, gates, Sinkhorn comb and the
collapsed row follow §3.4 and the reference math of §5.2. §4 (mhc_pre_big_fuse_with_prenorm): the
same with one split, the sum of squares taken from the residual and k = 4H.

The split sum and rstd are written out here; the logits / gates / Sinkhorn and the aggregate are the
C oracle's ``coefficients`` and ``aggregate`` (mhc_oracle.c), pinned in test_oracle_pins.py.
"""

from __future__ import annotations

import numpy as np

from .c_oracle import aggregate, bf16_bits_to_f64, coefficients


def big_fuse(dot_mix, sqrsum, R, scale, base, k, rms_eps=1e-6, pre_eps=0.0, post_mult=2.0,
             iters=20, eps=1e-6, want_y=True):
    """dot_mix [S,T,24] (or [T,24]), sqrsum [S,T] (or [T]) fp32; R uint16 bf16 bits [T,4,H].
    Returns dict of fp64 arrays: ss, rstd, logits, pre, post, comb, y."""
    T = R.shape[0]
    d = np.asarray(dot_mix, dtype=np.float64).reshape(-1, T, 24)
    q = np.asarray(sqrsum, dtype=np.float64).reshape(-1, T)
    assert d.shape[0] == q.shape[0]
    raw = np.zeros((T, 24))
    ss = np.zeros(T)
    for s in range(d.shape[0]):  # the split axis, summed in order
        raw += d[s]
        ss += q[s]
    rstd = 1.0 / np.sqrt(ss / float(k) + rms_eps)
    logits, pre, post, comb = coefficients(raw, rstd, scale, base, pre_eps=pre_eps,
                                           post_mult=post_mult, iters=iters, eps=eps)
    out = {"ss": ss, "rstd": rstd, "logits": logits, "pre": pre, "post": post, "comb": comb}
    out["y"] = aggregate(R, pre) if want_y else None
    return out


def sum_of_squares(R):
    """sum_k R_flat[t, k]^2 over the flattened [4H] row, in fp64 (exact bf16 widening)."""
    x = bf16_bits_to_f64(R).reshape(R.shape[0], -1)
    return np.einsum("tk,tk->t", x, x)


def big_fuse_with_prenorm(dot_mix, R, scale, base, **kw):
    """§4: one split, the sum of squares from R, k = 4H."""
    T, _, H = R.shape
    return big_fuse(np.asarray(dot_mix).reshape(1, T, 24), sum_of_squares(R)[None, :], R, scale,
                    base, 4 * H, **kw)
