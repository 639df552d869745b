"""GPU parity of the post-map fused with the next site's projection partials (mhc_post_project),
through the C ABI.

out must be bitwise the post-map's own result (same arithmetic as mhc_post, "FlashInfer mHC
module deep dive" §2.1); the partials, summed over splits, are the next site's projection and sum
of squares of out (§3.1-3.3 dot_mix / sqrsum), so mhc_pre_big_fuse on them must match the fp64
pre-map oracle evaluated on out (coefficients within 1e-5, y under tests/tolerance.py's rule).
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
    """w: this site's inputs (x, R, post/comb from its own draws); wn: the next site's weights."""
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
    out_bits = host_bits(out)
    sel = (lambda a: a) if rows is None else (lambda a: a[rows])
    ob = sel(out_bits)
    ref = oracle.pre(ob, wn.hc_fn, wn.hc_scale, wn.hc_base, rms_eps=wn.rms_eps,
                     pre_eps=wn.pre_eps, post_mult=wn.post_mult, iters=wn.iters, eps=wn.eps)
    ss, _, raw = oracle.norm_project(ob, wn.hc_fn, rms_eps=wn.rms_eps)
    dsum = sel(dot.sum(0).cpu().numpy().astype(np.float64))
    qsum = sel(sq.sum(0).cpu().numpy().astype(np.float64))
    scale = np.abs(bf16_bits_to_f64(ob)).reshape(len(ob), -1) @ np.abs(wn.hc_fn.astype(np.float64))
    assert np.all(np.abs(dsum - raw) <= 1e-5 * scale + 1e-6), f"{label}: dot_mix sums"
    assert np.all(np.abs(qsum - ss) <= 1e-5 * ss + 1e-6), f"{label}: sqrsum sums"
    t = (lambda a: a.cpu().numpy()) if rows is None else (lambda a: a.cpu().numpy()[rows])
    dp = check_coef(t(pre), ref["pre"], f"{label} pre")
    dq = check_coef(t(pst), ref["post"], f"{label} post")
    dc = check_coef(t(cmb), ref["comb"], f"{label} comb")
    Rabs = np.abs(bf16_bits_to_f64(ob))
    bound = COEF_TOL * Rabs.sum(axis=1) + 6 * U32 * np.einsum("ti,tih->th", np.abs(ref["pre"]),
                                                               Rabs)
    fail, need, worst = check_bf16(sel(host_bits(y)), ref["y"], oracle.round_bf16(ref["y"]), bound)
    print(f"[post_project {label}] S={S} |d|pre={dp:.2e} post={dq:.2e} comb={dc:.2e} y: "
          f"fail={fail} derived-bound={need} worst/tol={worst:.3f}")
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
