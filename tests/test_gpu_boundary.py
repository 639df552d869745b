"""GPU parity of the model-boundary operations (mhc_expand, mhc_head_mean, mhc_head) against the
fp64 oracle through the C ABI: expand bitwise; the heads under tests/tolerance.py's bf16 rule,
the weighted head's weights within 1e-5."""

import numpy as np
import pytest
import torch

import oracle
from oracle import boundary
import mhc_hyper_connection_02_b200 as mhc
from mhc_hyper_connection_02_b200 import inputs
from gpu_util import dev_bf16, dev_f32, host_bits
from tolerance import COEF_TOL, U32, bf16_bits_to_f64, check_bf16, check_coef

pytestmark = pytest.mark.gpu

SHAPES = [(1, 8), (37, 127), (64, 512), (10, 1001), (130, 4096), (5, 16392)]


def _head_weights(H, seed):
    g = np.random.default_rng(seed)
    return ((g.standard_normal((4 * H, 4)) * 0.02).astype(np.float32),
            np.array([g.uniform(0.5, 1.5)], np.float32),
            (g.standard_normal(4) * 0.1).astype(np.float32))


@pytest.mark.parametrize("T,H", SHAPES)
def test_expand_bitwise(T, H):
    w = inputs.custom(T, H, seed=T + H)
    s = mhc.expand(dev_bf16(w.x))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bits(s), boundary.expand(w.x))


@pytest.mark.parametrize("T,H", SHAPES)
def test_head_mean(T, H):
    w = inputs.custom(T, H, seed=2 * T + H)
    y = mhc.head_mean(dev_bf16(w.R))
    torch.cuda.synchronize()
    v = boundary.head_mean(w.R)
    bound = 4 * U32 * np.abs(bf16_bits_to_f64(w.R)).sum(axis=1) * 0.25
    fail, need, worst = check_bf16(host_bits(y), v, oracle.round_bf16(v), bound)
    print(f"[head_mean T={T} H={H}] fail={fail} derived-bound={need} worst/tol={worst:.3f}")
    assert fail == 0


@pytest.mark.parametrize("T,H", SHAPES + [(200, 7168)])
def test_head_weighted(T, H):
    w = inputs.custom(T, H, seed=3 * T + H)
    fn, sc, bs = _head_weights(H, T + H)
    y, wts = mhc.head(dev_bf16(w.R), dev_f32(fn), dev_f32(sc), dev_f32(bs), norm_eps=1e-6,
                      hc_eps=1e-6)
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    ref = boundary.head(w.R, fn, sc, bs, norm_eps=1e-6, hc_eps=1e-6)
    d = check_coef(wts.cpu().numpy(), ref["weights"], f"head T={T} H={H} weights")
    Rabs = np.abs(bf16_bits_to_f64(w.R))
    bound = COEF_TOL * Rabs.sum(axis=1) + 6 * U32 * np.einsum("ti,tih->th",
                                                               np.abs(ref["weights"]), Rabs)
    fail, need, worst = check_bf16(host_bits(y), ref["y"], oracle.round_bf16(ref["y"]), bound)
    print(f"[head T={T} H={H}] |d|w={d:.2e} y: fail={fail} derived-bound={need} "
          f"worst/tol={worst:.3f}")
    assert fail == 0


def test_boundary_unaligned_and_errors():
    w = inputs.custom(9, 64, seed=4)
    flat = torch.empty(w.x.size + 1, dtype=torch.bfloat16, device="cuda")
    hid = flat[1:].view(9, 64)
    hid.copy_(dev_bf16(w.x))
    s = mhc.expand(hid)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bits(s), boundary.expand(w.x))
    R = dev_bf16(w.R)
    with pytest.raises(mhc.MhcError) as e:  # y inside R
        mhc.head_mean(R, y=R.view(-1)[: 9 * 64].view(9, 64))
    assert e.value.status == mhc.MHC_ERR_ALIAS
    fn, sc, bs = _head_weights(64, 1)
    with pytest.raises(mhc.MhcError) as e:
        mhc.head(R, dev_f32(fn), dev_f32(sc), dev_f32(bs), norm_eps=0.0)
    assert e.value.status == mhc.MHC_ERR_INVALID_ARG
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(mhc.MhcError) as e:
        mhc.head(R, dev_f32(fn), dev_f32(sc), dev_f32(bs), workspace=small)
    assert e.value.status == mhc.MHC_ERR_WORKSPACE_TOO_SMALL
