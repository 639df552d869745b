"""GPU parity of the pre-map from an external projection (mhc_pre_big_fuse and
mhc_pre_big_fuse_with_prenorm) against the fp64 oracle, through the C ABI.

"FlashInfer mHC module deep dive" §3.1-3.3: dot_mix [num_splits,T,24] and sqrsum [num_splits,T]
summed over splits, rstd = 1/sqrt(sqrsum/k + rms_eps); §4: with_prenorm forms the sum of squares
from R with k = 4H; §3.4/§5.2: gates, Sinkhorn, y. Same bars as the pre-map: coefficients within
1e-5, y under tests/tolerance.py's rule.
"""

import numpy as np
import pytest
import torch

import oracle
import mhc_hyper_connection_02_b200 as mhc
from mhc_hyper_connection_02_b200 import inputs
from gpu_util import dev_bf16, dev_f32, host_bits
from tolerance import COEF_TOL, U32, bf16_bits_to_f64, check_bf16, check_coef

pytestmark = pytest.mark.gpu


def _compare(ref, R, outs, label, rows=None):
    y, pre, post, comb = outs
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.as_tensor(rows, device="cuda")])
    dp = check_coef(sel(pre).cpu().numpy(), ref["pre"], f"{label} pre")
    dq = check_coef(sel(post).cpu().numpy(), ref["post"], f"{label} post")
    dc = check_coef(sel(comb).cpu().numpy(), ref["comb"], f"{label} comb")
    Rabs = np.abs(bf16_bits_to_f64(R))
    bound = COEF_TOL * Rabs.sum(axis=1) + 6 * U32 * np.einsum("ti,tih->th", np.abs(ref["pre"]),
                                                               Rabs)
    fail, need, worst = check_bf16(host_bits(sel(y)), ref["y"], oracle.round_bf16(ref["y"]), bound)
    print(f"[{label}] |d|pre={dp:.2e} post={dq:.2e} comb={dc:.2e} y: fail={fail} "
          f"derived-bound={need} worst/tol={worst:.3f}")
    assert fail == 0


def _params():
    return mhc.make_params(iters=20, eps=1e-6, rms_eps=1e-6, pre_eps=1e-6, post_mult=1.0)


def _run(p, S, R_dev=None, prenorm=False):
    R = dev_bf16(p.R) if R_dev is None else R_dev
    if prenorm:
        outs = mhc.pre_big_fuse_with_prenorm(dev_f32(p.dot_mix[0]), R, dev_f32(p.hc_scale),
                                             dev_f32(p.hc_base), params=_params())
    else:
        outs = mhc.pre_big_fuse(dev_f32(p.dot_mix), dev_f32(p.sqrsum), R, dev_f32(p.hc_scale),
                                dev_f32(p.hc_base), 4 * p.H, num_splits=S, params=_params())
    torch.cuda.synchronize()
    return outs


def _oracle(p, prenorm=False, rows=None):
    kw = dict(rms_eps=1e-6, pre_eps=1e-6, post_mult=1.0, iters=20, eps=1e-6)
    R = p.R if rows is None else p.R[rows]
    if prenorm:
        d = p.dot_mix[0] if rows is None else p.dot_mix[0][rows]
        return oracle.big_fuse_with_prenorm(d, R, p.hc_scale, p.hc_base, **kw)
    d = p.dot_mix if rows is None else p.dot_mix[:, rows]
    q = p.sqrsum if rows is None else p.sqrsum[:, rows]
    return oracle.big_fuse(d, q, R, p.hc_scale, p.hc_base, 4 * p.H, **kw)


@pytest.mark.parametrize("S", [1, 2, 4, 8, 16])
def test_big_fuse_splits(S):
    p = inputs.partials(64, 512, S, seed=100 + S)
    _compare(_oracle(p), p.R, _run(p, S), f"big_fuse S={S}")


@pytest.mark.parametrize("T,H", [(1, 8), (19, 127), (33, 1000), (12, 1001), (40, 2048),
                                 (9, 4096), (21, 7168), (3, 16392)])
@pytest.mark.parametrize("prenorm", [False, True])
def test_big_fuse_shapes(T, H, prenorm):
    S = 1 if prenorm else 4
    p = inputs.partials(T, H, S, seed=T * 7 + H)
    _compare(_oracle(p, prenorm), p.R, _run(p, S, prenorm=prenorm),
             f"{'prenorm' if prenorm else 'big_fuse'} T={T} H={H}")


@pytest.mark.parametrize("prenorm", [False, True])
def test_big_fuse_unaligned_residual(prenorm):
    """R one element off a 16-byte boundary: the scalar loop path."""
    p = inputs.partials(11, 512, 1, seed=5)
    flat = torch.empty(p.R.size + 1, dtype=torch.bfloat16, device="cuda")
    R = flat[1:].view(11, 4, 512)
    R.copy_(dev_bf16(p.R))
    _compare(_oracle(p, prenorm), p.R, _run(p, 1, R_dev=R, prenorm=prenorm),
             f"unaligned prenorm={prenorm}")


def test_big_fuse_true_projection_matches_pre_map():
    """Partials that are the true split-K projection of a seeded workload (numpy fp64, rounded to
    fp32): big_fuse agrees with the oracle's pre-map and with the library's own mhc_pre."""
    w = inputs.custom(96, 1000, seed=9)
    x = bf16_bits_to_f64(w.R).reshape(w.T, -1)
    W = w.hc_fn.astype(np.float64)
    S, K = 4, 4 * w.H
    edges = np.linspace(0, K, S + 1).astype(int)
    dot = np.stack([x[:, a:b] @ W[a:b] for a, b in zip(edges, edges[1:])]).astype(np.float32)
    sq = np.stack([(x[:, a:b] ** 2).sum(1) for a, b in zip(edges, edges[1:])]).astype(np.float32)
    p = inputs.Partials(T=w.T, H=w.H, R=w.R, dot_mix=dot, sqrsum=sq, hc_scale=w.hc_scale,
                        hc_base=w.hc_base)
    prm = mhc.make_params(iters=w.iters, eps=w.eps, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                          post_mult=w.post_mult)
    R = dev_bf16(w.R)
    outs = mhc.pre_big_fuse(dev_f32(dot), dev_f32(sq), R, dev_f32(w.hc_scale), dev_f32(w.hc_base),
                            K, num_splits=S, params=prm)
    torch.cuda.synchronize()
    ref = oracle.pre(w.R, w.hc_fn, w.hc_scale, w.hc_base, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                     post_mult=w.post_mult, iters=w.iters, eps=w.eps)
    _compare(ref, w.R, outs, "true projection vs pre oracle")


def test_big_fuse_large_sampled():
    """T=8192, H=7168 (the headline size), one split and with_prenorm, on sampled tokens."""
    p = inputs.partials(8192, 7168, 1, seed=42)
    rows = np.concatenate([np.arange(0, 8), np.arange(4093, 4101), np.arange(8184, 8192)])
    R = dev_bf16(p.R)
    for prenorm in (False, True):
        outs = _run(p, 1, R_dev=R, prenorm=prenorm)
        _compare(_oracle(p, prenorm, rows), p.R[rows], outs, f"large prenorm={prenorm}", rows)


def test_big_fuse_empty_and_errors():
    p = inputs.partials(4, 64, 1, seed=1)
    R = dev_bf16(p.R)
    d, q = dev_f32(p.dot_mix), dev_f32(p.sqrsum)
    s, b = dev_f32(p.hc_scale), dev_f32(p.hc_base)
    with pytest.raises(mhc.MhcError) as e:
        mhc.pre_big_fuse(dev_f32(np.zeros((3, 4, 24), np.float32)),
                         dev_f32(np.zeros((3, 4), np.float32)), R, s, b, 256, num_splits=3)
    assert e.value.status == mhc.MHC_ERR_INVALID_ARG
    with pytest.raises(mhc.MhcError) as e:
        mhc.pre_big_fuse(d, q, R, s, b, 0)
    assert e.value.status == mhc.MHC_ERR_INVALID_ARG
    y, pre, post, comb = mhc.pre_big_fuse(d, q, R, s, b, 256)
    with pytest.raises(mhc.MhcError) as e:  # y overlapping R
        mhc.pre_big_fuse(d, q, R, s, b, 256, y=R.view(-1)[: 4 * 64].view(4, 64))
    assert e.value.status == mhc.MHC_ERR_ALIAS
    # T = 0: no launch, no error.
    R0 = torch.empty((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    n0 = mhc.launch_count()
    mhc.pre_big_fuse(torch.empty((1, 0, 24), device="cuda"), torch.empty((1, 0), device="cuda"),
                     R0, s, b, 256)
    assert mhc.launch_count() == n0
