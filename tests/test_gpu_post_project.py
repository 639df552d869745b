"""GPU parity of the post-map fused with the next site's projection partials (mhc_post_project),
through the C ABI.

out must match the fp64 post-map oracle (the post-map's rule) and be bitwise the GPU mhc_post's
result (same arithmetic, "FlashInfer mHC module deep dive" §2.1); the partials, summed over
splits, are the next site's projection and sum of squares of out (§3.1-3.3 dot_mix / sqrsum), so
mhc_pre_big_fuse on them must match the oracle chain -- the fp64 pre-map of the oracle's own
bf16-rounded post-map output (coefficients within 1e-5, y under tests/tolerance.py's rule).
"""

import numpy as np
import pytest
import torch

import oracle
import mhc_hyper_connection_02_b200 as mhc
from mhc_hyper_connection_02_b200 import inputs
from gpu_util import dev_bf16, dev_f32, host_bits, post_coefficients
from tolerance import COEF_TOL, U32, bf16_bits_to_f64, check_bf16, check_coef

pytestmark = pytest.mark.gpu


def _chain(w, wn, in_place=False, rows=None, label=""):
    """w: this site's inputs (x, R, post/comb from its own draws); wn: the next site's weights.

    out is checked against the oracle post-map directly, and is bitwise the GPU mhc_post's output.
    The next site is checked against the oracle chain: oracle pre-map of the oracle's own
    bf16-rounded post-map output. Where the GPU's out differs from that rounding (a value next to
    a bf16 rounding tie, at most one ulp), the token's bound carries the logit change those
    one-ulp differences cause, computed from the two bit patterns and hc_fn."""
    post, comb = post_coefficients(w)
    x, R = dev_bf16(w.x), dev_bf16(w.R)
    P, C = dev_f32(post), dev_f32(comb)
    ref_out = mhc.post(x, R, P, C)
    target = R if in_place else None
    out, dot, sq = mhc.post_project(x, R, P, C, dev_f32(wn.hc_fn), out=target)
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), f"{label}: out != post"
    S = mhc.post_project_splits(w.T, w.H)
    prm = mhc.make_params(iters=wn.iters, eps=wn.eps, rms_eps=wn.rms_eps, pre_eps=wn.pre_eps,
                          post_mult=wn.post_mult)
    y, pre, pst, cmb = mhc.pre_big_fuse(dot, sq, out, dev_f32(wn.hc_scale), dev_f32(wn.hc_base),
                                        4 * w.H, num_splits=S, params=prm)
    torch.cuda.synchronize()
    sel = (lambda a: a) if rows is None else (lambda a: a[rows])
    ob = sel(host_bits(out))
    xs, Rs, ps, cs = sel(w.x), sel(w.R), sel(post), sel(comb)
    # 1. out against the oracle post-map (the post-map's rule and derived bound).
    post_ref = oracle.post(xs, Rs, ps, cs)
    xa = np.abs(bf16_bits_to_f64(xs))[:, None, :]
    terms = xa * np.abs(ps.astype(np.float64))[:, :, None] + np.einsum(
        "toh,ton->tnh", np.abs(bf16_bits_to_f64(Rs)), np.abs(cs.astype(np.float64)))
    out_ref = oracle.round_bf16(post_ref)
    fail, need, worst = check_bf16(ob, post_ref, out_ref, 6 * U32 * terms)
    assert fail == 0, f"{label}: out vs oracle post"
    # 2. The next site against the oracle chain (oracle pre-map of the oracle's rounded out).
    ref_bits = torch.from_numpy(out_ref.astype(np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)
    ref = oracle.pre(ref_bits, wn.hc_fn, wn.hc_scale, wn.hc_base, rms_eps=wn.rms_eps,
                     pre_eps=wn.pre_eps, post_mult=wn.post_mult, iters=wn.iters, eps=wn.eps)
    ss, rstd, raw = oracle.norm_project(ref_bits, wn.hc_fn, rms_eps=wn.rms_eps)
    d_out = (bf16_bits_to_f64(ob) - bf16_bits_to_f64(ref_bits)).reshape(len(ob), -1)
    n_tie = int(np.count_nonzero(d_out))
    W = wn.hc_fn.astype(np.float64)
    d_raw = np.abs(d_out) @ np.abs(W)                       # |raw(gpu out) - raw(oracle out)|
    of = np.abs(bf16_bits_to_f64(ref_bits)).reshape(len(ob), -1)
    d_ss = (2 * of * np.abs(d_out) + d_out * d_out).sum(axis=1)
    K = 4 * w.H
    d_rstd = 0.5 * rstd ** 3 / K * d_ss * 1.01
    g = np.array([0] * 4 + [1] * 4 + [2] * 16)
    d_l = np.abs(wn.hc_scale.astype(np.float64))[g][None, :] * (
        d_raw * rstd[:, None] + np.abs(raw) * d_rstd[:, None])
    carry = 4.0 * d_l.max(axis=1)                           # per token, on every coefficient
    dsum = sel(dot.sum(0).cpu().numpy().astype(np.float64))
    qsum = sel(sq.sum(0).cpu().numpy().astype(np.float64))
    scale = of @ np.abs(W)
    assert np.all(np.abs(dsum - raw) <= 1e-5 * scale + 1e-6 + d_raw), f"{label}: dot_mix sums"
    assert np.all(np.abs(qsum - ss) <= 1e-5 * ss + 1e-6 + d_ss), f"{label}: sqrsum sums"
    t = (lambda a: a.cpu().numpy()) if rows is None else (lambda a: a.cpu().numpy()[rows])
    dmax = 0.0
    for got, name in ((pre, "pre"), (pst, "post"), (cmb, "comb")):
        d = np.abs(t(got).astype(np.float64) - ref[name]).reshape(len(ob), -1).max(axis=1)
        assert np.all(d <= COEF_TOL + carry), f"{label} {name}: {d.max():.3e}"
        dmax = max(dmax, float(d.max()))
    Rabs = np.abs(bf16_bits_to_f64(ref_bits))
    bound = (COEF_TOL + carry[:, None]) * Rabs.sum(axis=1) + 6 * U32 * np.einsum(
        "ti,tih->th", np.abs(ref["pre"]), Rabs) + np.abs(d_out.reshape(Rabs.shape)).sum(axis=1)
    fail, need, worst = check_bf16(sel(host_bits(y)), ref["y"], oracle.round_bf16(ref["y"]), bound)
    print(f"[post_project {label}] S={S} out-vs-oracle ok, next site |d|max={dmax:.2e} "
          f"tie-elements={n_tie} y: fail={fail} derived-bound={need} worst/tol={worst:.3f}")
    assert fail == 0


@pytest.mark.parametrize("T,H", [(1, 8), (7, 64), (64, 512), (130, 1000), (300, 4096),
                                 (5, 16392), (257, 7168), (3000, 1000)])
def test_post_project_chain(T, H):
    w = inputs.custom(T, H, seed=T + 3 * H)
    wn = inputs.custom(1, H, seed=T + 3 * H + 1)  # the next site's weights (hc_fn, scale, base)
    _chain(w, wn, label=f"T={T} H={H}")


def test_post_project_in_place():
    w = inputs.custom(96, 2048, seed=21)
    wn = inputs.custom(1, 2048, seed=22)
    _chain(w, wn, in_place=True, label="in place")


def test_post_project_large_sampled():
    w = inputs.large()
    wn = inputs.custom(1, w.H, seed=77)
    rows = np.concatenate([np.arange(0, 6), np.arange(4090, 4096), np.arange(8186, 8192)])
    _chain(w, wn, rows=rows, label="large")


def test_post_project_unsupported_and_errors():
    w = inputs.custom(4, 1001, seed=1)
    post, comb = post_coefficients(w)
    with pytest.raises(mhc.MhcError) as e:
        mhc.post_project(dev_bf16(w.x), dev_bf16(w.R), dev_f32(post), dev_f32(comb),
                         dev_f32(w.hc_fn))
    assert e.value.status == mhc.MHC_ERR_UNSUPPORTED
    w = inputs.custom(4, 64, seed=2)
    post, comb = post_coefficients(w)
    R = dev_bf16(w.R)
    with pytest.raises(mhc.MhcError) as e:  # out overlapping x
        xx = torch.empty(4 * 4 * 64 + 4 * 64, dtype=torch.bfloat16, device="cuda")
        xv = xx[: 4 * 64].view(4, 64)
        xv.copy_(dev_bf16(w.x))
        mhc.post_project(xv, R, dev_f32(post), dev_f32(comb), dev_f32(w.hc_fn),
                         out=xx[64: 64 + 4 * 4 * 64].view(4, 4, 64))
    assert e.value.status == mhc.MHC_ERR_ALIAS
