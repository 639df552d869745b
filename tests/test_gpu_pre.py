"""GPU parity of the fused pre-map against the fp64 oracle, through the C ABI.

Per token: rstd = 1/sqrt(sum(R^2)/(4H) + rms_eps); logits l = (R_flat . hc_fn)*rstd*scale[g] +
base; pre = sigmoid(l[0:4]) + pre_eps; post = post_mult*sigmoid(l[4:8]); comb = Sinkhorn of
l[8:24]; y = bf16(sum_i pre_i R_i) ("FlashInfer mHC module deep dive" §3.4, §4, §5.2; rwkv-ops
mhc_pre_op). Coefficients within 1e-5; y under the rule in tests/tolerance.py, where the derived
term admits the 1e-5 gate difference times sum_i |R_i| plus the fp32 evaluation of four terms.
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

PRE_PATHS = {"cuda_core": mhc.PRE_PATH_CUDA_CORE, "tensor": mhc.PRE_PATH_TENSOR,
             "tensor_split": mhc.PRE_PATH_TENSOR_SPLIT, "tensor_fused": mhc.PRE_PATH_TENSOR_FUSED,
             "tensor_wave": mhc.PRE_PATH_TENSOR_WAVE}


def run_pre(w, path=mhc.PATH_AUTO, params=None, R_dev=None):
    R = dev_bf16(w.R) if R_dev is None else R_dev
    p = params or mhc.make_params(iters=w.iters, eps=w.eps, rms_eps=w.rms_eps, pre_eps=w.pre_eps,
                                  post_mult=w.post_mult)
    y, pre, post, comb = mhc.pre(R, dev_f32(w.hc_fn), dev_f32(w.hc_scale), dev_f32(w.hc_base),
                                 params=p, path=path)
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    return y, pre, post, comb


def run_fused(w, R_dev=None):
    """The single-pass kernel, forced. Returns None where the library reports it cannot run this
    shape (MHC_ERR_UNSUPPORTED, before any launch); otherwise asserts that exactly its two launches
    (counter zeroing + the fused kernel) were enqueued, so a pass is the fused kernel's."""
    n0 = mhc.launch_count()
    try:
        outs = run_pre(w, mhc.PRE_PATH_TENSOR_FUSED, R_dev=R_dev)
    except mhc.MhcError as e:
        assert e.status == mhc.MHC_ERR_UNSUPPORTED
        assert mhc.launch_count() == n0
        return None
    assert mhc.launch_count() - n0 == 2, "the fused path must be exactly its two launches"
    return outs


def run_wave(w, R_dev=None):
    """The wavefront single pass, forced. None where the library reports it cannot run this shape
    (MHC_ERR_UNSUPPORTED, nothing launched); otherwise asserts its three launches (hc_fn split and
    counter reset, the wave kernel, the Sinkhorn pass), so a pass is the wave kernel's."""
    n0 = mhc.launch_count()
    try:
        outs = run_pre(w, mhc.PRE_PATH_TENSOR_WAVE, R_dev=R_dev)
    except mhc.MhcError as e:
        assert e.status == mhc.MHC_ERR_UNSUPPORTED
        assert mhc.launch_count() == n0
        return None
    assert mhc.launch_count() - n0 == 3, "the wave path must be exactly its three launches"
    return outs


def compare_pre(w, outs, rows=None, label="", pre_eps=None, post_mult=None, iters=None, eps=None):
    y, pre, post, comb = outs
    R = w.R if rows is None else w.R[rows]
    ref = oracle.pre(R, w.hc_fn, w.hc_scale, w.hc_base, rms_eps=w.rms_eps,
                     pre_eps=w.pre_eps if pre_eps is None else pre_eps,
                     post_mult=w.post_mult if post_mult is None else post_mult,
                     iters=w.iters if iters is None else iters, eps=w.eps if eps is None else eps)
    sel = (lambda t: t) if rows is None else (lambda t: t[torch.as_tensor(rows, device="cuda")])
    dp = check_coef(sel(pre).cpu().numpy(), ref["pre"], f"{label} pre")
    dq = check_coef(sel(post).cpu().numpy(), ref["post"], f"{label} post")
    dc = check_coef(sel(comb).cpu().numpy(), ref["comb"], f"{label} comb")
    Rabs = np.abs(bf16_bits_to_f64(R))
    bound = COEF_TOL * Rabs.sum(axis=1) + 6 * U32 * np.einsum("ti,tih->th", np.abs(ref["pre"]), Rabs)
    fail, need, worst = check_bf16(host_bits(sel(y)), ref["y"], oracle.round_bf16(ref["y"]), bound)
    print(f"[pre {label}] |d|pre={dp:.2e} post={dq:.2e} comb={dc:.2e} y: fail={fail} "
          f"derived-bound={need} worst/tol={worst:.3f} n={ref['y'].size}")
    assert fail == 0
    return max(dp, dq, dc)


@pytest.mark.parametrize("path", ["cuda_core", "tensor", "tensor_split", "tensor_fused",
                                  "tensor_wave"])
def test_pre_small_workload(path):
    w = inputs.small()
    if path == "tensor_fused":
        outs = run_fused(w)
        assert outs is not None, "the single-pass kernel supports T=64, H=512"
    elif path == "tensor_wave":
        outs = run_wave(w)
        assert outs is not None, "the wave kernel supports T=64, H=512"
    else:
        outs = run_pre(w, PRE_PATHS[path])
    compare_pre(w, outs, label=f"small {path}")


@pytest.mark.parametrize("T,H", [(1, 8), (33, 8), (5, 127), (130, 1000), (17, 1001), (64, 4096),
                                 (3, 16392)])
def test_pre_shapes(T, H):
    w = inputs.custom(T, H, seed=T + H)
    compare_pre(w, run_pre(w), label=f"T={T} H={H}")
    compare_pre(w, run_pre(w, mhc.PRE_PATH_CUDA_CORE), label=f"T={T} H={H} cuda_core")
    if H % 2 == 0:
        compare_pre(w, run_pre(w, mhc.PRE_PATH_TENSOR), label=f"T={T} H={H} tensor")
        compare_pre(w, run_pre(w, mhc.PRE_PATH_TENSOR_SPLIT), label=f"T={T} H={H} tensor-split")
    fused = run_fused(w)
    if fused is not None:
        compare_pre(w, fused, label=f"T={T} H={H} tensor-fused")
    else:
        assert H % 8 != 0 or H < 64, f"single-pass kernel refused T={T} H={H}"
    wave = run_wave(w)
    if wave is not None:
        compare_pre(w, wave, label=f"T={T} H={H} tensor-wave")
    else:
        assert H % 8 != 0 or H < 64, f"wave kernel refused T={T} H={H}"


@pytest.mark.parametrize("T,H", [(300, 7168), (129, 1000), (1, 4096), (520, 512)])
def test_pre_tensor_path_agrees_with_cuda_core_path(T, H):
    """Two GPU implementations of the projection (tcgen05 bf16x3 vs fp32 CUDA cores) agree within
    the coefficient tolerance, and each matches the oracle."""
    w = inputs.custom(T, H, seed=3 * T + H)
    a = run_pre(w, mhc.PRE_PATH_TENSOR)
    b = run_pre(w, mhc.PRE_PATH_CUDA_CORE)
    c = run_pre(w, mhc.PRE_PATH_TENSOR_SPLIT)
    others = [(b, "cuda_core"), (c, "tensor-split")]
    fused = run_fused(w)
    if fused is not None:
        others.append((fused, "tensor-fused"))
    wave = run_wave(w)
    if wave is not None:
        others.append((wave, "tensor-wave"))
    for other, oname in others:
        for x, y, name in zip(a[1:], other[1:], ("pre", "post", "comb")):
            d = (x.double() - y.double()).abs().max().item()
            print(f"[tensor vs {oname} T={T} H={H}] {name} max|d| = {d:.2e}")
            assert d <= COEF_TOL
    compare_pre(w, a, label=f"tensor T={T} H={H}")


@pytest.mark.parametrize("T", [1, 4, 16, 32])
def test_pre_decode(T):
    w = inputs.decode(T)
    compare_pre(w, run_pre(w), label=f"decode T={T}")


def test_pre_tail_workload():
    w = inputs.tail()
    compare_pre(w, run_pre(w), label="tail T=3000 H=1000")


def compare_pre_all(w, outs, label="", chunk=1024):
    """Every token, checked in chunks of `chunk` tokens (bounded host memory at the full size)."""
    for c0 in range(0, w.T, chunk):
        compare_pre(w, outs, rows=np.arange(c0, min(w.T, c0 + chunk)),
                    label=f"{label} [{c0}:{min(w.T, c0 + chunk)}]")


@pytest.mark.slow
def test_pre_large_full_batch():
    """T=8192, H=7168: every token of the default call (the launch bench.py times)."""
    w = inputs.large()
    compare_pre_all(w, run_pre(w), label="large")


@pytest.mark.slow
@pytest.mark.parametrize("path", ["tensor_fused", "tensor_wave", "tensor_split", "cuda_core"])
def test_pre_large_full_batch_each_path(path):
    """T=8192, H=7168, every token, on each forced path (the single-pass kernels run here with
    their record rings wrapping many times)."""
    w = inputs.large()
    if path == "tensor_fused":
        outs = run_fused(w)
    elif path == "tensor_wave":
        outs = run_wave(w)
    else:
        outs = run_pre(w, PRE_PATHS[path])
    assert outs is not None
    compare_pre_all(w, outs, label=f"large {path}")


@pytest.mark.parametrize("T,H", [(3000, 1000), (1000, 7168), (2000, 4096), (129, 64)])
def test_pre_fused_multi_tile(T, H):
    """The single-pass kernel over many tiles per group, ragged last tiles and K ranges that are not
    a multiple of 64 columns (H = 1000)."""
    w = inputs.custom(T, H, seed=T + 7 * H)
    outs = run_fused(w)
    assert outs is not None
    compare_pre(w, outs, label=f"fused T={T} H={H}")


@pytest.mark.parametrize("T,H", [(3000, 1000), (1000, 7168), (2000, 4096), (129, 64), (3072, 7168),
                                 (700, 16392), (1, 7168)])
def test_pre_wave_multi_tile(T, H):
    """The wavefront kernel: ranges that cross tile boundaries, ragged last tiles, K not a multiple
    of 64 columns (H = 1000), more than 64 pieces of a tile in flight over the record ring (T=3072)
    and y units narrower than a row (H = 16392: seventeen per token)."""
    w = inputs.custom(T, H, seed=T + 11 * H)
    outs = run_wave(w)
    assert outs is not None
    compare_pre(w, outs, label=f"wave T={T} H={H}")


def test_pre_wave_refuses_what_it_cannot_run():
    """H % 8 != 0 or H < 64: MHC_ERR_UNSUPPORTED with nothing launched."""
    for T, H in ((10, 1001), (10, 56)):
        w = inputs.custom(T, H, seed=5)
        assert run_wave(w) is None


def test_pre_params_other_than_default():
    w = inputs.custom(50, 256, seed=77)
    p = mhc.make_params(iters=50, eps=1e-3, rms_eps=1e-4, pre_eps=1e-6, post_mult=1.0)
    w.rms_eps = 1e-4
    outs = run_pre(w, params=p)
    compare_pre(w, outs, label="params", pre_eps=1e-6, post_mult=1.0, iters=50, eps=1e-3)
    outs = run_pre(w, mhc.PRE_PATH_TENSOR_WAVE, params=p)
    compare_pre(w, outs, label="params wave", pre_eps=1e-6, post_mult=1.0, iters=50, eps=1e-3)


@pytest.mark.parametrize("stream", range(4))
def test_pre_one_hot_gate_selects_its_stream(stream):
    """hc_fn = 0 and base[0:4] = +-40: pre is one-hot to fp32 precision, y == R[stream] bitwise."""
    w = inputs.custom(19, 520, seed=stream)
    w.hc_fn = np.zeros_like(w.hc_fn)
    base = np.zeros(24, np.float32)
    base[0:4] = -40.0
    base[stream] = 40.0
    w.hc_base = base
    y, pre, post, comb = run_pre(w)
    np.testing.assert_array_equal(host_bits(y), w.R[:, stream, :])
    assert torch.all(pre[:, stream] == 1.0)


def test_pre_zero_rows_give_base_logits():
    w = inputs.custom(8, 64, seed=3)
    w.R = np.zeros_like(w.R)
    compare_pre(w, run_pre(w), label="zero rows")


def test_pre_misaligned_inputs():
    T, H = 9, 300
    w = inputs.custom(T, H, seed=12)
    big = torch.zeros(T * 4 * H + 1, dtype=torch.bfloat16, device="cuda")
    big[1:] = dev_bf16(w.R).view(-1)
    R = big[1:].view(T, 4, H)
    compare_pre(w, run_pre(w, R_dev=R), label="misaligned R")


def test_pre_guard_bands_untouched():
    T, H = 21, 1000
    w = inputs.custom(T, H, seed=44)
    pad = 1024
    yb = torch.full((pad + T * H + pad,), 3.0, dtype=torch.bfloat16, device="cuda")
    cb = torch.full((pad + T * 16 + pad,), 3.0, device="cuda")
    y = yb[pad:pad + T * H].view(T, H)
    comb = cb[pad:pad + T * 16].view(T, 4, 4)
    p = mhc.make_params(iters=w.iters)
    outs = mhc.pre(dev_bf16(w.R), dev_f32(w.hc_fn), dev_f32(w.hc_scale), dev_f32(w.hc_base),
                   y=y, comb=comb, params=p)
    torch.cuda.synchronize()
    assert torch.all(yb[:pad] == 3.0) and torch.all(yb[pad + T * H:] == 3.0)
    assert torch.all(cb[:pad] == 3.0) and torch.all(cb[pad + T * 16:] == 3.0)
    compare_pre(w, outs, label="guard")


def test_pre_then_post_chain_matches_oracle_chain():
    """GPU pre -> GPU post against oracle pre -> (fp32) -> oracle post. The post-map inputs differ
    by at most the admitted coefficient error, which the bound carries through."""
    w = inputs.custom(40, 1024, seed=8)
    y, pre, post, comb = run_pre(w)
    out = mhc.post(dev_bf16(w.x), dev_bf16(w.R), post, comb)
    torch.cuda.synchronize()
    ref = oracle.pre(w.R, w.hc_fn, w.hc_scale, w.hc_base, iters=w.iters, eps=w.eps)
    ref_out = oracle.post(w.x, w.R, ref["post"].astype(np.float32), ref["comb"].astype(np.float32))
    xa = np.abs(bf16_bits_to_f64(w.x))[:, None, :]
    Ra = np.abs(bf16_bits_to_f64(w.R))
    bound = COEF_TOL * (xa + Ra.sum(axis=1)[:, None, :]) * 1.01 + 6 * U32 * (
        xa * 2 + Ra.sum(axis=1)[:, None, :])
    fail, need, worst = check_bf16(host_bits(out), ref_out, oracle.round_bf16(ref_out), bound)
    print(f"[chain] fail={fail} derived-bound={need} worst/tol={worst:.3f}")
    assert fail == 0
