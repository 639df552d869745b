"""mhc_pre_noalloc: the pre-map for callers that cannot allocate device memory (plugins whose host
framework owns all device allocations and gives them no workspace, and serving loops that must not
allocate per call). It keeps its scratch in a fixed array inside the library.

Checked through the C ABI against the existing entry point (mhc_pre, which takes a caller workspace)
on two calls in a row with different sizes, within the tolerances the other tests use. This file is
collected last so that a run stopping at the first failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import mhc_hyper_connection_02_b200 as mhc
from mhc_hyper_connection_02_b200 import inputs
from tolerance import COEF_TOL, REL, U32, ulp_bf16, bf16_bits_to_f64, check_bf16, check_coef

pytestmark = pytest.mark.gpu


def to_dev(w):
    return (torch.from_numpy(w.R.view(np.int16)).view(torch.bfloat16).cuda(),
            torch.from_numpy(w.hc_fn).cuda(), torch.from_numpy(w.hc_scale).cuda(),
            torch.from_numpy(w.hc_base).cuda())


def call_noalloc(R, W, S, B, T, H, params):
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    pre = torch.empty((T, 4), device="cuda")
    post = torch.empty((T, 4), device="cuda")
    comb = torch.empty((T, 4, 4), device="cuda")
    st = mhc.lib().mhc_pre_noalloc(R.data_ptr(), W.data_ptr(), S.data_ptr(), B.data_ptr(),
                                   y.data_ptr(), pre.data_ptr(), post.data_ptr(), comb.data_ptr(),
                                   T, H, ctypes.byref(params),
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == mhc.MHC_OK, mhc.status_string(st)
    return y, pre, post, comb


def assert_close(new, ref, R_bits):
    """The entry against mhc_pre: coefficients within the tolerance (1e-5); y under the bf16 rule,
    or, where y cancels, within one ulp plus what the two calls' admitted coefficient differences
    (each within 1e-5 of the oracle, so 2e-5 apart) and fp32 evaluation carry into y."""
    for a, b, name in zip(new[1:], ref[1:], ("pre", "post", "comb")):
        d = (a.double() - b.double()).abs().max().item()
        assert d <= COEF_TOL, f"{name}: {d}"
    yn = bf16_bits_to_f64(new[0].view(torch.int16).cpu().numpy().view(np.uint16))
    yr = bf16_bits_to_f64(ref[0].view(torch.int16).cpu().numpy().view(np.uint16))
    rsum = np.abs(bf16_bits_to_f64(R_bits)).sum(axis=1)
    u = ulp_bf16(yr)
    tol = np.maximum(np.maximum(u, REL * np.abs(yr)), 2 * u + (2 * COEF_TOL + 12 * U32) * rsum)
    assert np.all(np.abs(yn - yr) <= tol)


def assert_matches_oracle(new, w, rows):
    """The entry's own output against the fp64 oracle on the given tokens (same rules as the
    pre-map parity tests: coefficients within 1e-5, y under tests/tolerance.py)."""
    ref = oracle.pre(w.R[rows], w.hc_fn, w.hc_scale, w.hc_base, rms_eps=w.rms_eps,
                     pre_eps=w.pre_eps, post_mult=w.post_mult, iters=w.iters, eps=w.eps)
    idx = torch.as_tensor(rows, device="cuda")
    for got, name in zip(new[1:], ("pre", "post", "comb")):
        check_coef(got[idx].cpu().numpy(), ref[name], f"noalloc {name}")
    Rabs = np.abs(bf16_bits_to_f64(w.R[rows]))
    bound = COEF_TOL * Rabs.sum(axis=1) + 6 * U32 * np.einsum("ti,tih->th", np.abs(ref["pre"]), Rabs)
    yb = new[0][idx].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    fail, _, _ = check_bf16(yb, ref["y"], oracle.round_bf16(ref["y"]), bound)
    assert fail == 0


def test_noalloc_matches_mhc_pre_on_two_calls_in_a_row():
    for w in (inputs.decode(32), inputs.custom(7, 1000, seed=61)):
        params = mhc.make_params(iters=w.iters, eps=w.eps, rms_eps=w.rms_eps)
        R, W, S, B = to_dev(w)
        new = call_noalloc(R, W, S, B, w.T, w.H, params)
        ref = mhc.pre(R, W, S, B, params=params)
        torch.cuda.synchronize()
        assert mhc.device_status() == 0
        assert_close(new, ref, w.R)
        assert_matches_oracle(new, w, np.arange(w.T))


def test_noalloc_at_its_exact_scratch_limit():
    """T = 32768, H = 512: one split, 32768 records of 128 bytes fill the 4 MiB array exactly. An
    off-by-one in the size check or the record indexing would write past it (into other device
    globals, such as the status word) or be refused."""
    w = inputs.custom(32768, 512, seed=63)
    params = mhc.make_params(iters=w.iters, eps=w.eps, rms_eps=w.rms_eps)
    R, W, S, B = to_dev(w)
    new = call_noalloc(R, W, S, B, w.T, w.H, params)
    ref = mhc.pre(R, W, S, B, params=params)
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    assert_close(new, ref, w.R)
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(w.T - 64, w.T),
                                     np.random.default_rng(5).choice(w.T, 256, replace=False)]))
    assert_matches_oracle(new, w, rows)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    A = 1 << 40
    p = mhc.default_params()
    st = mhc.lib().mhc_pre_noalloc(A, A + (1 << 36), A + (2 << 36), A + (3 << 36), A + (4 << 36),
                                   A + (5 << 36), A + (6 << 36), A + (7 << 36), 32769, 512,
                                   ctypes.byref(p), None)
    assert st == mhc.MHC_ERR_SCRATCH_LIMIT
    assert mhc.status_string(st) == "MHC_ERR_SCRATCH_LIMIT"
