"""The bounded device waits give up with MHC_ERR_TIMEOUT and leave the GPU usable.

Every wait inside the library's kernels (mbarrier phases of the copy and MMA pipelines, cross-CTA
counters) is bounded by the GPU's global timer; on expiry the kernel records MHC_ERR_TIMEOUT in a
device status word and winds down instead of waiting forever or trapping. This test makes one such
wait run out on purpose -- the library's health-check kernel waits, through the same routine, on an
mbarrier nothing arrives at, with a 1 ms limit and no copy in flight -- and checks that the status
comes back, that reading it clears it, and that a normal pre-map call right after still matches the
fp64 oracle on the same device.
"""

import numpy as np
import pytest
import torch

import oracle
import mhc_hyper_connection_02_b200 as mhc
from mhc_hyper_connection_02_b200 import inputs
from gpu_util import dev_bf16, dev_f32
from tolerance import check_coef

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_gpu_stays_usable():
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    mhc.selftest_wait_timeout(1_000_000)
    assert mhc.device_status() == mhc.MHC_ERR_TIMEOUT
    assert mhc.device_status() == 0  # reading cleared the word
    w = inputs.custom(256, 512, seed=90)
    y, pre, post, comb = mhc.pre(dev_bf16(w.R), dev_f32(w.hc_fn), dev_f32(w.hc_scale),
                                 dev_f32(w.hc_base), params=mhc.make_params(iters=w.iters))
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    ref = oracle.pre(w.R, w.hc_fn, w.hc_scale, w.hc_base, iters=w.iters, want_y=False)
    for got, name in ((pre, "pre"), (post, "post"), (comb, "comb")):
        check_coef(got.cpu().numpy(), ref[name], name)


def test_selftest_rejects_limits_out_of_range():
    for bad in (0, 999, 2_000_000_000):
        with pytest.raises(mhc.MhcError) as e:
            mhc.selftest_wait_timeout(bad)
        assert e.value.status == mhc.MHC_ERR_INVALID_ARG
