"""GPU parity of the backward passes (mhc_post_backward, mhc_pre_backward) against the fp64
backward oracle (oracle/backward.py, pinned by autograd), through the C ABI.

Bars. bf16 gradients (d_x, d_R): tests/tolerance.py's rule, with the derived term sized from the
terms each output sums. fp32 sums (d_post, d_comb, d_hc_fn, d_scale, d_base) are sums of products
over H or T evaluated in fp32: |gpu - oracle| <= 1e-5 * sum|terms| + 1e-6 absolute (the summation's
worst-case rounding, n u with n <= 2^16 terms and u = 2^-24, is below 4e-3 sum|terms|; the fixed
tree order the kernels use stays far inside it, and a wrong term or sign moves the result by the
size of the terms). The pre-map backward recomputes the forward in fp32 (coefficients within
~1e-6 of fp64), so its per-token gradients carry a relative error of that order: its bars add
1e-4 * sum|terms|.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import backward
import mhc_hyper_connection_02_b200 as mhc
from mhc_hyper_connection_02_b200 import inputs
from gpu_util import dev_bf16, dev_f32, host_bits, post_coefficients
from tolerance import U32, bf16_bits_to_f64, check_bf16

pytestmark = pytest.mark.gpu


def _bits(arr):
    return torch.from_numpy(np.asarray(arr, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16).copy()


def _check_sum(gpu, ref, terms_abs, rel, name):
    err = np.abs(np.asarray(gpu, np.float64) - ref)
    tol = rel * terms_abs + 1e-6
    worst = float(np.max(err / tol)) if err.size else 0.0
    print(f"  {name}: max|err|={float(err.max()) if err.size else 0:.3e} worst/tol={worst:.3f}")
    assert np.all(err <= tol), name


@pytest.mark.parametrize("T,H", [(1, 8), (5, 127), (64, 512), (33, 1000), (16, 7168),
                                 (3, 16392), (1000, 1032), (500, 3000)])
def test_post_backward(T, H):
    w = inputs.custom(T, H, seed=11 * T + H)
    post, comb = post_coefficients(w)
    g = np.random.default_rng(T + H)
    d_out = _bits(g.standard_normal((T, 4, H)))
    dx, dR, dp, dc = mhc.post_backward(dev_bf16(d_out), dev_bf16(w.x), dev_bf16(w.R),
                                       dev_f32(post), dev_f32(comb))
    torch.cuda.synchronize()
    rx, rR, rp, rc = backward.post_backward(d_out, w.x, w.R, post, comb)
    G = np.abs(bf16_bits_to_f64(d_out))
    P = np.abs(post.astype(np.float64))
    C = np.abs(comb.astype(np.float64))
    bx = 5 * U32 * np.einsum("tn,tnh->th", P, G)
    bR = 5 * U32 * np.einsum("ton,tnh->toh", C, G)
    f1 = check_bf16(host_bits(dx), rx, oracle.round_bf16(rx), bx)
    f2 = check_bf16(host_bits(dR), rR, oracle.round_bf16(rR), bR)
    print(f"[post_backward T={T} H={H}] d_x fail={f1[0]} d_R fail={f2[0]}")
    assert f1[0] == 0 and f2[0] == 0
    X = np.abs(bf16_bits_to_f64(w.x))
    Rb = np.abs(bf16_bits_to_f64(w.R))
    _check_sum(dp.cpu().numpy(), rp, np.einsum("th,tnh->tn", X, G), 1e-5, "d_post")
    _check_sum(dc.cpu().numpy(), rc, np.einsum("toh,tnh->ton", Rb, G), 1e-5, "d_comb")


def _pre_case(T, H, seed, with_dy=True, with_comb=True):
    w = inputs.custom(T, H, seed=seed)
    g = np.random.default_rng(seed)
    d_y = _bits(g.standard_normal((T, H))) if with_dy else None
    d_pre = g.standard_normal((T, 4)).astype(np.float32)
    d_post = g.standard_normal((T, 4)).astype(np.float32)
    d_comb = g.standard_normal((T, 4, 4)).astype(np.float32) if with_comb else None
    return w, d_y, d_pre, d_post, d_comb


@pytest.mark.parametrize("T,H", [(1, 8), (5, 127), (64, 512), (130, 1000), (300, 2048),
                                 (20, 7168), (3, 1001), (1000, 1024), (513, 4096), (777, 256),
                                 (200, 1056), (3000, 64), (9000, 128)])
def test_pre_backward(T, H):
    w, d_y, d_pre, d_post, d_comb = _pre_case(T, H, seed=7 * T + H)
    prm = mhc.make_params(iters=w.iters, eps=w.eps, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                          post_mult=w.post_mult)
    dR, dW, ds, db = mhc.pre_backward(
        dev_bf16(w.R), dev_f32(w.hc_fn), dev_f32(w.hc_scale), dev_f32(w.hc_base),
        d_y=dev_bf16(d_y), d_pre=dev_f32(d_pre), d_post=dev_f32(d_post), d_comb=dev_f32(d_comb),
        params=prm)
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    rR, rW, rs, rb, pt = backward.pre_backward(d_y, d_pre, d_post, d_comb, w.R, w.hc_fn,
                                               w.hc_scale, w.hc_base, rms_eps=w.rms_eps,
                                               pre_eps=w.pre_eps, post_mult=w.post_mult,
                                               iters=w.iters, eps=w.eps, parts=True)
    Wa = np.abs(w.hc_fn.astype(np.float64))
    X = np.abs(pt["X"])
    terms = (np.abs(pt["d_raw"]) @ Wa.T + 2 * X * np.abs(pt["d_ss"])[:, None]).reshape(T, 4, H)
    terms = terms + np.abs(pt["pre"])[:, :, None] * np.abs(bf16_bits_to_f64(d_y))[:, None, :]
    f = check_bf16(host_bits(dR), rR, oracle.round_bf16(rR), (1e-4 + 30 * U32) * terms)
    print(f"[pre_backward T={T} H={H}] d_R fail={f[0]} derived-bound={f[1]} worst/tol={f[2]:.3f}")
    assert f[0] == 0
    _check_sum(dW.cpu().numpy(), rW, X.T @ np.abs(pt["d_raw"]), 1e-4, "d_hc_fn")
    g = np.array([0] * 4 + [1] * 4 + [2] * 16)
    ts = np.array([(np.abs(pt["dl"][:, g == k] * pt["m"][:, g == k])).sum() for k in range(3)])
    _check_sum(ds.cpu().numpy(), rs, ts, 1e-4, "d_scale")
    _check_sum(db.cpu().numpy(), rb, np.abs(pt["dl"]).sum(0), 1e-4, "d_base")


@pytest.mark.parametrize("T,H,dr_tensor,dw_tensor,dy_fold", [(300, 2048, True, True, True),
                                                            (130, 1000, False, False, False),
                                                            (200, 1056, False, True, False)])
def test_pre_backward_d_R_form(T, H, dr_tensor, dw_tensor, dy_fold):
    """H % 128 == 0 with d_y given takes the tcgen05 kernel that forms d_R and d_hc_fn in one
    pass over R (split operands, the tensor kernel, the d_hc_fn partials' sum: three launches);
    otherwise d_R runs on CUDA cores (one) and d_hc_fn on its own: where 4H % 128 == 0 the tcgen05
    d_hc_fn (transposed d_raw split, the tensor kernel, the partials' sum: three launches), else
    CUDA-core partials and their sum (two). The projections here are the tensor form (split +
    projection); with H % 64 == 0 it also forms d_pre's d_y term, otherwise a d_pre kernel runs;
    then coefficients and parameters."""
    w, d_y, d_pre, d_post, d_comb = _pre_case(T, H, seed=11)
    n0 = mhc.launch_count()
    mhc.pre_backward(dev_bf16(w.R), dev_f32(w.hc_fn), dev_f32(w.hc_scale), dev_f32(w.hc_base),
                     d_y=dev_bf16(d_y), d_pre=dev_f32(d_pre), d_post=dev_f32(d_post),
                     d_comb=dev_f32(d_comb), params=mhc.make_params(iters=w.iters))
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    grads = 3 if dr_tensor else 1 + (3 if dw_tensor else 2)
    assert mhc.launch_count() - n0 == 2 + (2 if dy_fold else 3) + grads


def test_pre_backward_optional_gradients_and_tensor_path():
    """T = 256 takes the tensor-core projection; d_y and d_comb absent (zero). Without d_y the
    projection does not form d_pre's term (a d_pre kernel runs), and d_R with d_hc_fn still takes
    the tensor kernel (no d_y tiles): 2 + 3 + 3 launches."""
    w, _, d_pre, d_post, _ = _pre_case(256, 512, seed=3, with_dy=False, with_comb=False)
    n0 = mhc.launch_count()
    dR, dW, ds, db = mhc.pre_backward(dev_bf16(w.R), dev_f32(w.hc_fn), dev_f32(w.hc_scale),
                                      dev_f32(w.hc_base), d_pre=dev_f32(d_pre),
                                      d_post=dev_f32(d_post),
                                      params=mhc.make_params(iters=w.iters))
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    assert mhc.launch_count() - n0 == 8
    rR, rW, rs, rb, pt = backward.pre_backward(None, d_pre, d_post, None, w.R, w.hc_fn, w.hc_scale,
                                               w.hc_base, iters=w.iters, parts=True)
    Wa = np.abs(w.hc_fn.astype(np.float64))
    X = np.abs(pt["X"])
    terms = (np.abs(pt["d_raw"]) @ Wa.T + 2 * X * np.abs(pt["d_ss"])[:, None]).reshape(256, 4, 512)
    f = check_bf16(host_bits(dR), rR, oracle.round_bf16(rR), (1e-4 + 30 * U32) * terms)
    assert f[0] == 0
    _check_sum(dW.cpu().numpy(), rW, X.T @ np.abs(pt["d_raw"]), 1e-4, "d_hc_fn")
    _check_sum(db.cpu().numpy(), rb, np.abs(pt["dl"]).sum(0), 1e-4, "d_base")


def test_backward_errors():
    w = inputs.custom(4, 64, seed=9)
    R = dev_bf16(w.R)
    post, comb = post_coefficients(w)
    with pytest.raises(mhc.MhcError) as e:  # d_x inside R is rejected before any launch
        L = mhc.lib()
        st = L.mhc_post_backward(R.data_ptr(), dev_bf16(w.x).data_ptr(), R.data_ptr(),
                                 dev_f32(post).data_ptr(), dev_f32(comb).data_ptr(), R.data_ptr(),
                                 torch.empty_like(R).data_ptr(),
                                 torch.empty(16, device="cuda").data_ptr(),
                                 torch.empty(64, device="cuda").data_ptr(), 4, 64, None)
        mhc._check(st, "mhc_post_backward")
    assert e.value.status == mhc.MHC_ERR_ALIAS
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(mhc.MhcError) as e:
        mhc.pre_backward(R, dev_f32(w.hc_fn), dev_f32(w.hc_scale), dev_f32(w.hc_base),
                         workspace=small)
    assert e.value.status == mhc.MHC_ERR_WORKSPACE_TOO_SMALL


def _sample_rows(T, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(T, 24, replace=False), [0, 127, 128, T - 1]]))


@pytest.mark.slow
def test_post_backward_large_sampled():
    """Full size (T=8192, H=7168), the launch bench.py times; every output is per token, so
    sampled tokens are checked against the oracle run on those tokens alone."""
    w = inputs.large()
    post, comb = post_coefficients(w)
    g = np.random.default_rng(101)
    d_out = _bits(g.standard_normal((w.T, 4, w.H), dtype=np.float32))
    dx, dR, dp, dc = mhc.post_backward(dev_bf16(d_out), dev_bf16(w.x), dev_bf16(w.R),
                                       dev_f32(post), dev_f32(comb))
    torch.cuda.synchronize()
    rows = _sample_rows(w.T, 5)
    rx, rR, rp, rc = backward.post_backward(d_out[rows], w.x[rows], w.R[rows], post[rows],
                                            comb[rows])
    G = np.abs(bf16_bits_to_f64(d_out[rows]))
    bx = 5 * U32 * np.einsum("tn,tnh->th", np.abs(post[rows].astype(np.float64)), G)
    bR = 5 * U32 * np.einsum("ton,tnh->toh", np.abs(comb[rows].astype(np.float64)), G)
    sel = torch.as_tensor(rows, device="cuda")
    f1 = check_bf16(host_bits(dx[sel]), rx, oracle.round_bf16(rx), bx)
    f2 = check_bf16(host_bits(dR[sel]), rR, oracle.round_bf16(rR), bR)
    print(f"[post_backward large sampled] d_x fail={f1[0]} d_R fail={f2[0]}")
    assert f1[0] == 0 and f2[0] == 0
    X = np.abs(bf16_bits_to_f64(w.x[rows]))
    Rb = np.abs(bf16_bits_to_f64(w.R[rows]))
    _check_sum(dp[sel].cpu().numpy(), rp, np.einsum("th,tnh->tn", X, G), 1e-5, "d_post")
    _check_sum(dc[sel].cpu().numpy(), rc, np.einsum("toh,tnh->ton", Rb, G), 1e-5, "d_comb")


@pytest.mark.slow
def test_pre_backward_large_sampled():
    """Full size (T=8192, H=7168), the launch bench.py times. d_R is per token: sampled tokens
    against the oracle on those tokens. d_hc_fn, d_scale and d_base are sums over all tokens: the
    oracle runs on chunks of 1024 tokens and its fp64 chunk sums are added."""
    w = inputs.large()
    g = np.random.default_rng(202)
    d_y = _bits(g.standard_normal((w.T, w.H), dtype=np.float32))
    d_pre = g.standard_normal((w.T, 4)).astype(np.float32)
    d_post = g.standard_normal((w.T, 4)).astype(np.float32)
    d_comb = g.standard_normal((w.T, 4, 4)).astype(np.float32)
    prm = mhc.make_params(iters=w.iters, eps=w.eps, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                          post_mult=w.post_mult)
    dR, dW, ds, db = mhc.pre_backward(
        dev_bf16(w.R), dev_f32(w.hc_fn), dev_f32(w.hc_scale), dev_f32(w.hc_base),
        d_y=dev_bf16(d_y), d_pre=dev_f32(d_pre), d_post=dev_f32(d_post), d_comb=dev_f32(d_comb),
        params=prm)
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    kw = dict(rms_eps=w.rms_eps, pre_eps=w.pre_eps, post_mult=w.post_mult, iters=w.iters,
              eps=w.eps, parts=True)
    Wa = np.abs(w.hc_fn.astype(np.float64))
    grp = np.array([0] * 4 + [1] * 4 + [2] * 16)
    rW = np.zeros((4 * w.H, 24))
    tW = np.zeros((4 * w.H, 24))
    rs = np.zeros(3)
    ts = np.zeros(3)
    rb = np.zeros(24)
    tb = np.zeros(24)
    for c0 in range(0, w.T, 1024):
        sl = slice(c0, min(w.T, c0 + 1024))
        _, cW, cs, cb, pt = backward.pre_backward(d_y[sl], d_pre[sl], d_post[sl], d_comb[sl],
                                                  w.R[sl], w.hc_fn, w.hc_scale, w.hc_base, **kw)
        rW += cW
        rs += cs
        rb += cb
        tW += np.abs(pt["X"]).T @ np.abs(pt["d_raw"])
        ts += np.array([(np.abs(pt["dl"][:, grp == k] * pt["m"][:, grp == k])).sum()
                        for k in range(3)])
        tb += np.abs(pt["dl"]).sum(0)
    _check_sum(dW.cpu().numpy(), rW, tW, 1e-4, "d_hc_fn")
    _check_sum(ds.cpu().numpy(), rs, ts, 1e-4, "d_scale")
    _check_sum(db.cpu().numpy(), rb, tb, 1e-4, "d_base")
    rows = _sample_rows(w.T, 6)
    rR, _, _, _, pt = backward.pre_backward(d_y[rows], d_pre[rows], d_post[rows], d_comb[rows],
                                            w.R[rows], w.hc_fn, w.hc_scale, w.hc_base, **kw)
    n = len(rows)
    X = np.abs(pt["X"])
    terms = (np.abs(pt["d_raw"]) @ Wa.T + 2 * X * np.abs(pt["d_ss"])[:, None]).reshape(n, 4, w.H)
    terms = terms + np.abs(pt["pre"])[:, :, None] * np.abs(bf16_bits_to_f64(d_y[rows]))[:, None, :]
    sel = torch.as_tensor(rows, device="cuda")
    f = check_bf16(host_bits(dR[sel]), rR, oracle.round_bf16(rR), (1e-4 + 30 * U32) * terms)
    print(f"[pre_backward large sampled] d_R fail={f[0]} derived-bound={f[1]} worst/tol={f[2]:.3f}")
    assert f[0] == 0
