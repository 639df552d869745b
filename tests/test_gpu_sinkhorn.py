"""GPU parity of the standalone Sinkhorn entry (mhc_sinkhorn) against the fp64 oracle:
A = softmax(l, each row) + eps, then `iters` rounds of (rows /= rowsum, columns /= colsum)
("FlashInfer mHC module deep dive" §3.4, §5.2). Coefficient bar: 1e-5."""

import numpy as np
import pytest
import torch

import oracle
import mhc_hyper_connection_02_b200 as mhc
from tolerance import check_coef

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 3, 1000, 4097])
@pytest.mark.parametrize("std,iters", [(1.0, 1), (1.0, 20), (3.0, 50)])
def test_sinkhorn_matches_oracle(T, std, iters):
    rng = np.random.default_rng(T * 7 + iters)
    logits = (rng.standard_normal((T, 4, 4)) * std).astype(np.float32)
    got = mhc.sinkhorn(torch.from_numpy(logits).cuda(), iters=iters, eps=1e-6)
    torch.cuda.synchronize()
    ref = oracle.sinkhorn(logits.astype(np.float64), iters=iters, eps=1e-6)
    d = check_coef(got.cpu().numpy(), ref, f"sinkhorn T={T} iters={iters}")
    print(f"[sinkhorn T={T} std={std} iters={iters}] max|d|={d:.2e}")


def test_sinkhorn_in_place_and_unaligned():
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((257, 4, 4)).astype(np.float32)
    ref = oracle.sinkhorn(logits.astype(np.float64), iters=20, eps=1e-6)
    a = torch.from_numpy(logits).cuda()
    mhc.sinkhorn(a, comb=a, iters=20, eps=1e-6)            # in place
    big = torch.zeros(257 * 16 + 1, device="cuda")
    big[1:] = torch.from_numpy(logits).cuda().view(-1)
    u = big[1:].view(257, 4, 4)                            # 4-byte offset: scalar loads
    got_u = mhc.sinkhorn(u, iters=20, eps=1e-6)
    torch.cuda.synchronize()
    check_coef(a.cpu().numpy(), ref, "in place")
    check_coef(got_u.cpu().numpy(), ref, "unaligned")


def test_sinkhorn_rank_one_is_uniform_and_doubly_stochastic():
    rng = np.random.default_rng(4)
    a, b = rng.standard_normal((64, 4, 1)), rng.standard_normal((64, 1, 4))
    got = mhc.sinkhorn(torch.from_numpy((a + b).astype(np.float32)).cuda(), iters=20, eps=1e-6)
    torch.cuda.synchronize()
    np.testing.assert_allclose(got.cpu().numpy(), 0.25, atol=1e-5)


def test_sinkhorn_large_eps_and_many_rounds():
    rng = np.random.default_rng(5)
    logits = (rng.standard_normal((999, 4, 4)) * 2).astype(np.float32)
    for iters, eps in ((200, 1e-6), (7, 0.5)):
        got = mhc.sinkhorn(torch.from_numpy(logits).cuda(), iters=iters, eps=eps)
        torch.cuda.synchronize()
        check_coef(got.cpu().numpy(), oracle.sinkhorn(logits.astype(np.float64), iters, eps),
                   f"iters={iters} eps={eps}")


@pytest.mark.parametrize("std,iters", [(1.0, 20), (3.0, 50)])
def test_sinkhorn_one_thread_per_token_form(std, iters):
    """From 65536 tokens the call runs one thread per token (16 registers, no shuffles). Every
    token against the oracle, aligned, unaligned and in place; and bit for bit the lane-quad
    form's result on the same logits (the sums are associated the same way)."""
    T = 70001
    rng = np.random.default_rng(int(std * 100) + iters)
    logits = (rng.standard_normal((T, 4, 4)) * std).astype(np.float32)
    ref = oracle.sinkhorn(logits.astype(np.float64), iters=iters, eps=1e-6)
    dev = torch.from_numpy(logits).cuda()
    got = mhc.sinkhorn(dev, iters=iters, eps=1e-6)
    big = torch.zeros(T * 16 + 1, device="cuda")
    big[1:] = dev.view(-1)
    got_u = mhc.sinkhorn(big[1:].view(T, 4, 4), iters=iters, eps=1e-6)
    inplace = dev.clone()
    mhc.sinkhorn(inplace, comb=inplace, iters=iters, eps=1e-6)
    quad = mhc.sinkhorn(dev[:4000].contiguous(), iters=iters, eps=1e-6)  # the lane-quad form
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    for g, name in ((got, "aligned"), (got_u, "unaligned"), (inplace, "in place")):
        d = check_coef(g.cpu().numpy(), ref, f"thread form {name}")
        print(f"[sinkhorn thread form {name} std={std} iters={iters}] max|d|={d:.2e}")
    assert torch.equal(got[:4000], quad)
