"""Oracle of the model-boundary operations (fp64). TEST INFRASTRUCTURE ONLY.

glm5next_mhc.rs: glm_hc_expand broadcasts each hidden row into the hc_mult streams; hc_head_mean
collapses the streams to their unweighted mean. hyper_connection_dispatch.rs hc_head_site: the
weighted head takes hc_fn / hc_scale / hc_base, a norm eps and hc_eps; the page does not show its
kernel. Read here as the pre-map's first gate group with its own weights: rstd over the flattened
row (K = 4H, as the pre-map's RMS step), w_i = sigmoid((R_flat . hc_fn[:, i]) * rstd * scale[0] +
base[i]) + hc_eps, y = sum_i w_i R_i.
"""

from __future__ import annotations

import numpy as np

from .c_oracle import bf16_bits_to_f64


def expand(hidden):
    """hidden uint16 [T,H] -> streams uint16 [T,4,H] (bit copies)."""
    h = np.asarray(hidden, dtype=np.uint16)
    return np.repeat(h[:, None, :], 4, axis=1)


def head_mean(R):
    """R uint16 [T,4,H] -> fp64 mean over the streams [T,H]."""
    x = bf16_bits_to_f64(R)
    return (x[:, 0] + x[:, 1] + x[:, 2] + x[:, 3]) / 4.0


def head(R, hc_fn, hc_scale, hc_base, norm_eps=1e-6, hc_eps=1e-6):
    """Weighted head. Returns dict: rstd [T], logits [T,4], weights [T,4], y [T,H] (fp64)."""
    T, _, H = R.shape
    x = bf16_bits_to_f64(R).reshape(T, 4 * H)
    ss = np.einsum("tk,tk->t", x, x)
    rstd = 1.0 / np.sqrt(ss / (4 * H) + norm_eps)
    raw = x @ np.asarray(hc_fn, dtype=np.float64)  # [T,4]
    logits = raw * rstd[:, None] * float(hc_scale[0]) + np.asarray(hc_base, np.float64)[None, :]
    w = 1.0 / (1.0 + np.exp(-logits)) + hc_eps
    xs = x.reshape(T, 4, H)
    y = np.einsum("ti,tih->th", w, xs)
    return {"rstd": rstd, "logits": logits, "weights": w, "y": y}
