"""Pins of the fp64 CPU oracle against things other than itself (closed forms, invariants, special
cases that reduce to a library routine, brute force on tiny inputs, and an independent NumPy
restatement). Each test names the step and the passage it pins:

* [FI]  "FlashInfer mHC module deep dive": §2.1 post formula, §3.2 parameters, §3.4 kernel phases
        (sigmoid gates, softmax with row-max shift, Sinkhorn row->column rounds), §4 (RMS over 4*H),
        §5.2 test reference math (softmax, eps added to the entries, `iters` row -> column rounds).
* [RW]  rwkv-ops ``mhu_jax.py``: ``mhc_pre_op`` docstring (H_pre = sigmoid, H_post = 2*sigmoid,
        x_layer_in = sum(H_pre * x_expanded)).
* [GLM] ``glm5next_mhc.rs``: ``glm_hc_post`` (out[j] = post[j]*block_out + sum_i comb[i][j]*residual[i]).

A plausible mistake (dropped term, wrong sign, swapped index, transposed operand, eps in the wrong
place, wrong scale group) fails at least one of them.
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import numpy_ref

RNG = np.random.default_rng(12345)


def bits(values) -> np.ndarray:
    """bf16 bit patterns of values that are exactly representable in bf16 (checked)."""
    t = torch.tensor(np.asarray(values, dtype=np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.float(), t), "test value not exact in bf16"
    return b.view(torch.int16).numpy().view(np.uint16).copy()


def rand_bits(shape, scale=1.0) -> np.ndarray:
    t = torch.from_numpy((RNG.standard_normal(shape) * scale).astype(np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


# ----------------------------------------------------------------------------- Sinkhorn (a4, a7)

def test_sinkhorn_converges_to_doubly_stochastic():
    """[FI] §3.4: the comb matrix is made doubly stochastic. 1000 random 4x4 logit matrices."""
    logits = RNG.standard_normal((1000, 4, 4)) * 2.0
    comb, _ = oracle.sinkhorn_converge(logits, eps=1e-6, tol=1e-13, max_iters=10000)
    assert np.all(comb > 0)
    assert np.max(np.abs(comb.sum(axis=2) - 1.0)) < 1e-4
    assert np.max(np.abs(comb.sum(axis=1) - 1.0)) < 1e-4


def test_sinkhorn_scaling_invariance_at_convergence():
    """Sinkhorn's limit is unique: adding a constant per row and per column of the logits
    (D1 A D2 after exp) leaves the converged matrix unchanged. eps = 0 here: the eps added to the
    entries is not a row or column scaling, so the invariant holds for the eps-free iteration."""
    logits = RNG.standard_normal((200, 4, 4))
    a = RNG.standard_normal((200, 4, 1)) * 3.0
    b = RNG.standard_normal((200, 1, 4)) * 3.0
    c1, _ = oracle.sinkhorn_converge(logits, eps=0.0, tol=1e-15, max_iters=20000)
    c2, _ = oracle.sinkhorn_converge(logits + a + b, eps=0.0, tol=1e-15, max_iters=20000)
    assert np.max(np.abs(c1 - c2)) < 1e-9


@pytest.mark.parametrize("eps", [1e-6, 0.25])
def test_sinkhorn_rank_one_closed_form(eps):
    """Logits l[o][n] = a_o + b_n: every row's softmax is the same vector p_n = exp(b_n)/sum exp(b)
    (the row constant a_o cancels), so before any round every entry is p_n + eps ([FI] §5.2: eps is
    added to the softmax output). A row step keeps the four rows equal, and a column step then
    divides four equal entries by their sum: after one round or more, every entry is exactly 1/4.
    Pins eps on the entries (zero rounds) and plain, eps-free row and column sums (an eps added
    to the sums would leave v / (4 v + eps) instead of 1/4)."""
    a = RNG.standard_normal(4) * 2.0
    b = RNG.standard_normal(4)
    logits = a[:, None] + b[None, :]
    p = np.exp(b) / np.exp(b).sum()
    got0 = oracle.sinkhorn(logits[None], iters=0, eps=eps)[0]
    np.testing.assert_allclose(got0, np.tile(p + eps, (4, 1)), rtol=1e-14, atol=0)
    for iters in (1, 2, 3, 20):
        got = oracle.sinkhorn(logits[None], iters=iters, eps=eps)[0]
        np.testing.assert_allclose(got, 0.25, rtol=1e-14, atol=0)


def test_sinkhorn_permutation_equivariance_brute_force():
    """All 24 x 24 (row permutation, column permutation) pairs: SK(P l Q) = P SK(l) Q for the fixed
    20-round output (row max, row sums and column sums are all permutation-equivariant)."""
    logits = RNG.standard_normal((4, 4)) * 1.5
    base = oracle.sinkhorn(logits[None], iters=20, eps=1e-6)[0]
    perms = list(itertools.permutations(range(4)))
    batch = np.empty((len(perms) ** 2, 4, 4))
    expect = np.empty_like(batch)
    for i, (p, q) in enumerate(itertools.product(perms, perms)):
        batch[i] = logits[np.ix_(p, q)]
        expect[i] = base[np.ix_(p, q)]
    got = oracle.sinkhorn(batch, iters=20, eps=1e-6)
    assert np.max(np.abs(got - expect)) < 1e-14


def test_sinkhorn_permutation_dominant_stays_near_permutation():
    for p in itertools.permutations(range(4)):
        P = np.zeros((4, 4))
        P[np.arange(4), p] = 1.0
        logits = 12.0 * P + 0.1 * RNG.standard_normal((4, 4))
        comb, _ = oracle.sinkhorn_converge(logits[None], eps=1e-6)
        assert np.max(np.abs(comb[0] - P)) < 1e-4


M_HAND = np.array([[1, 2, 3, 4], [4, 3, 2, 1], [1, 1, 1, 1], [1, 2, 2, 5]], dtype=np.float64)


def test_sinkhorn_single_round_hand_example():
    """Worked by hand, eps = 0.05, one round, logits log(M) with M = [[1,2,3,4],[4,3,2,1],[1,1,1,1],
    [1,2,2,5]]. The row softmax gives M / rowsum: (.1,.2,.3,.4), (.4,.3,.2,.1), (.25,.25,.25,.25),
    (.1,.2,.2,.5); eps makes them (.15,.25,.35,.45), (.45,.35,.25,.15), (.3,.3,.3,.3),
    (.15,.25,.25,.55). Every row now sums to 1.2, so the row step divides everything by 1.2, and the
    column step divides by the column sums (1.05, 1.15, 1.15, 1.45) / 1.2. Result: entry / column
    sum of the eps-shifted matrix. Without eps on the entries the columns would be divided by
    (.85, .95, .95, 1.25) instead."""
    shifted = np.array([[.15, .25, .35, .45], [.45, .35, .25, .15], [.3, .3, .3, .3],
                        [.15, .25, .25, .55]])
    cols = np.array([1.05, 1.15, 1.15, 1.45])
    got = oracle.sinkhorn(np.log(M_HAND)[None], iters=1, eps=0.05)[0]
    np.testing.assert_allclose(got, shifted / cols[None, :], rtol=1e-14)


def test_sinkhorn_two_round_hand_example():
    """Pins the round count (`iters` counts full row -> column rounds). eps = 0, M as above, in
    exact rational arithmetic. Round 1: rows of M / rowsum already sum to 1; the column sums are
    (17/20, 19/20, 19/20, 5/4), giving C1 = [[2/17, 4/19, 6/19, 8/25], [8/17, 6/19, 4/19, 2/25],
    [5/17, 5/19, 5/19, 1/5], [2/17, 4/19, 4/19, 2/5]]. Round 2: C1's row sums are
    (7784/8075, 8696/8075, 1648/1615, 1516/1615); dividing the rows by them and then the columns by
    their new sums gives the fractions below. One round fewer or more (e.g. an extra column step
    straight after the softmax) misses them."""
    num = [[848664380, 1697328760, 2545993140, 678931504],
           [3038640080, 2278980060, 1519320040, 151932004],
           [2004248645, 2004248645, 2004248645, 400849729],
           [871504424, 1743008848, 1743008848, 871504424]]
    den = [6763057529, 7723566313, 7812570673, 2103217661]
    expect = np.array([[num[o][n] / den[n] for n in range(4)] for o in range(4)])
    got = oracle.sinkhorn(np.log(M_HAND)[None], iters=2, eps=0.0)[0]
    np.testing.assert_allclose(got, expect, rtol=1e-14)
    np.testing.assert_allclose(got.sum(axis=0), 1.0, rtol=1e-14)  # the last step is a column step


def test_sinkhorn_columns_sum_to_one_after_every_round():
    """The last operation of each round is a column normalisation, so every column sums to 1 (to
    rounding) after any number of rounds, while the rows only approach 1."""
    logits = RNG.standard_normal((500, 4, 4)) * 2.0
    for iters in (1, 3, 20):
        comb = oracle.sinkhorn(logits, iters=iters, eps=1e-6)
        assert np.max(np.abs(comb.sum(axis=1) - 1.0)) < 1e-14
    assert np.max(np.abs(oracle.sinkhorn(logits, iters=1, eps=1e-6).sum(axis=2) - 1.0)) > 1e-3


def test_sinkhorn_reading_gap_report(capsys):
    """Not a pin: a report of how far the other readings of the pages' Sinkhorn sit from the one the
    oracle follows ([FI] §5.2: softmax, eps added to every entry, then `iters` plain row -> column
    rounds). Variant 1 is rwkv-ops' (eps in the row and column sums, none on the entries); variant
    2 reads [FI] §3.4 as an extra column step straight after the softmax. On N(0,1) logits with 20
    rounds they agree to ~1e-5; on the near-permutation 3*N(0,1) logits with 50 rounds the fixed-
    round output has not converged and eps-sized entries still move it, so they differ by up to
    ~3e-2. The readings are not interchangeable at the 1e-5 coefficient tolerance."""
    gaps = {}
    for std, iters in ((1.0, 20), (3.0, 50)):
        logits = RNG.standard_normal((4000, 4, 4)) * std
        a = oracle.sinkhorn(logits, iters=iters, eps=1e-6)
        for v in (1, 2):
            b = oracle.sinkhorn_variant(logits, iters=iters, eps=1e-6, variant=v)
            gaps[(std, iters, v)] = float(np.max(np.abs(a - b)))
    with capsys.disabled():
        print(f"\n[sinkhorn reading gap] max|oracle - variant| by (std, iters, variant) = {gaps}")
    assert gaps[(1.0, 20, 1)] < 1e-4
    assert gaps[(3.0, 50, 1)] < 1e-1


# ----------------------------------------------------------------------------- norm + projection

def test_constant_row_rstd():
    """[FI] §4: RMS over the 4*H flattened row, eps inside the square root."""
    for c in (0.75, -3.0, 1.0):
        R = np.full((2, 4, 16), bits([c])[0], dtype=np.uint16)
        _, rstd, _ = oracle.norm_project(R, np.zeros((64, 24), np.float32), rms_eps=1e-6)
        np.testing.assert_allclose(rstd, 1.0 / math.sqrt(c * c + 1e-6), rtol=1e-15)


def test_zero_row_gives_base_logits():
    """A zero row: rstd = 1/sqrt(rms_eps), raw = 0, logits = base (assumption P9, no special case)."""
    R = np.zeros((1, 4, 8), np.uint16)
    base = RNG.standard_normal(24).astype(np.float32)
    out = oracle.pre(R, RNG.standard_normal((32, 24)).astype(np.float32),
                     np.ones(3, np.float32), base)
    np.testing.assert_allclose(out["rstd"], 1e3, rtol=1e-12)
    np.testing.assert_array_equal(out["logits"][0], base.astype(np.float64))
    assert np.all(out["y"] == 0.0)


def test_projection_brute_force_basis_T1_H8():
    """T=1, H=8 (K=32): for every basis row R = e_k (stream k//8, column k%8, value 1) the raw
    projection is hc_fn[k,:] exactly, ss = 1 and rstd = 1/sqrt(1/32 + eps). This pins the
    flattening order k = i*H + h and the orientation of hc_fn [4H,24]."""
    W = RNG.standard_normal((32, 24)).astype(np.float32)
    one = bits([1.0])[0]
    for k in range(32):
        R = np.zeros((1, 4, 8), np.uint16)
        R[0, k // 8, k % 8] = one
        ss, rstd, raw = oracle.norm_project(R, W, rms_eps=1e-6)
        assert ss[0] == 1.0
        np.testing.assert_allclose(rstd[0], 1.0 / math.sqrt(1.0 / 32 + 1e-6), rtol=1e-15)
        np.testing.assert_array_equal(raw[0], W[k].astype(np.float64))


def test_projection_linearity():
    W = RNG.standard_normal((64, 24)).astype(np.float32)
    for _ in range(20):
        k, m = RNG.choice(64, size=2, replace=False)
        a, b = float(RNG.integers(-8, 9)) / 4, float(RNG.integers(-8, 9)) / 4
        R = np.zeros((1, 4, 16), np.uint16)
        R[0, k // 16, k % 16] = bits([a])[0]
        R[0, m // 16, m % 16] = bits([b])[0]
        _, _, raw = oracle.norm_project(R, W)
        np.testing.assert_allclose(raw[0], a * W[k].astype(np.float64) + b * W[m].astype(np.float64), rtol=1e-15,
                                   atol=1e-15)


def test_logit_affine_scale_groups():
    """[FI] §5.2: logits[0:4] use scale[0], [4:8] scale[1], [8:24] scale[2], plus base."""
    H = 8
    W = np.zeros((4 * H, 24), np.float32)
    v = RNG.standard_normal(24).astype(np.float32)
    W[5] = v
    R = np.zeros((1, 4, H), np.uint16)
    R[0, 0, 5] = bits([2.0])[0]
    scale = np.array([0.5, 1.25, 2.0], np.float32)
    base = RNG.standard_normal(24).astype(np.float32)
    out = oracle.pre(R, W, scale, base, rms_eps=1e-6)
    rstd = 1.0 / math.sqrt(4.0 / 32 + 1e-6)
    group = [0] * 4 + [1] * 4 + [2] * 16
    expect = [2.0 * float(v[j]) * rstd * float(scale[group[j]]) + float(base[j]) for j in range(24)]
    np.testing.assert_allclose(out["logits"][0], expect, rtol=1e-14, atol=1e-15)


def test_gate_special_values():
    """[RW] mhc_pre_op: H_pre = sigmoid(l), H_post = 2*sigmoid(l). Logit 0 gives 1/2 exactly;
    logit ln 3 gives 3/4 (1/(1 + 1/3)); so pre = 3/4, post = 3/2 at l = ln 3, and a wrong sign
    (sigmoid(-l)) would give 1/4."""
    base = np.zeros(24, np.float32)
    base[1] = np.float32(math.log(3.0))
    base[5] = np.float32(math.log(3.0))
    R = np.zeros((1, 4, 8), np.uint16)
    out = oracle.pre(R, np.zeros((32, 24), np.float32), np.ones(3, np.float32), base,
                     pre_eps=1e-6, post_mult=2.0)
    ln3 = float(np.float32(math.log(3.0)))
    s = 1.0 / (1.0 + math.exp(-ln3))
    np.testing.assert_allclose(out["pre"][0], [0.5 + 1e-6, s + 1e-6, 0.5 + 1e-6, 0.5 + 1e-6],
                               rtol=1e-15)
    np.testing.assert_allclose(out["post"][0], [1.0, 2 * s, 1.0, 1.0], rtol=1e-15)
    assert abs(s - 0.75) < 1e-7


# ----------------------------------------------------------------------------- aggregate (a5)

@pytest.mark.parametrize("stream", range(4))
def test_one_hot_pre_selects_its_stream(stream):
    """hc_fn = 0 and base[0:4] = +40 on one stream, -40 elsewhere: pre is one-hot up to 4e-18, and
    y equals that stream of R (bitwise after bf16 rounding)."""
    T, H = 3, 40
    R = rand_bits((T, 4, H))
    base = np.zeros(24, np.float32)
    base[0:4] = -40.0
    base[stream] = 40.0
    out = oracle.pre(R, np.zeros((4 * H, 24), np.float32), np.ones(3, np.float32), base)
    assert np.max(np.abs(out["pre"] - np.eye(4)[stream])) < 1e-17
    yb = oracle.round_bf16(out["y"])
    np.testing.assert_array_equal(yb, oracle.bf16_bits_to_f64(R[:, stream, :]))


def test_equal_streams_aggregate():
    """All four streams equal to r: y = r * sum_i pre_i."""
    T, H = 4, 24
    r = rand_bits((T, 1, H))
    R = np.repeat(r, 4, axis=1)
    W = (RNG.standard_normal((4 * H, 24)) * 0.05).astype(np.float32)
    out = oracle.pre(R, W, np.ones(3, np.float32), np.zeros(24, np.float32))
    expect = oracle.bf16_bits_to_f64(r[:, 0, :]) * out["pre"].sum(axis=1)[:, None]
    np.testing.assert_allclose(out["y"], expect, rtol=1e-14, atol=1e-15)


# ----------------------------------------------------------------------------- post-map (a6)

def test_post_identity_comb_returns_residual():
    T, H = 5, 33
    R, x = rand_bits((T, 4, H)), rand_bits((T, H))
    comb = np.tile(np.eye(4, dtype=np.float32), (T, 1, 1))
    out = oracle.post(x, R, np.zeros((T, 4), np.float32), comb)
    np.testing.assert_array_equal(out, oracle.bf16_bits_to_f64(R))


def test_post_permutation_comb_permutes_streams():
    """comb[o][n] = 1 where n = p(o): new stream n is old stream p^-1(n) ([old][new] orientation)."""
    T, H = 2, 16
    R, x = rand_bits((T, 4, H)), rand_bits((T, H))
    for p in itertools.permutations(range(4)):
        P = np.zeros((4, 4), np.float32)
        P[np.arange(4), p] = 1.0
        out = oracle.post(x, R, np.zeros((T, 4), np.float32), np.tile(P, (T, 1, 1)))
        inv = np.argsort(p)
        np.testing.assert_array_equal(out, oracle.bf16_bits_to_f64(R[:, inv, :]))


def test_post_zero_comb_broadcasts_x():
    T, H = 3, 20
    R, x = rand_bits((T, 4, H)), rand_bits((T, H))
    out = oracle.post(x, R, np.ones((T, 4), np.float32), np.zeros((T, 4, 4), np.float32))
    for n in range(4):
        np.testing.assert_array_equal(out[:, n, :], oracle.bf16_bits_to_f64(x))


def test_post_brute_force_basis_T1_H8():
    """[GLM] glm_hc_post / [FI] §2.1: with R = e_(o,h) and x = 0, out[n,h'] = comb[o][n] at h'=h and
    0 elsewhere; with x = e_h and R = 0, out[n,h'] = post[n] at h'=h. Every basis input checked."""
    H = 8
    post = RNG.standard_normal((1, 4)).astype(np.float32)
    comb = RNG.standard_normal((1, 4, 4)).astype(np.float32)
    one = bits([1.0])[0]
    for o in range(4):
        for h in range(H):
            R = np.zeros((1, 4, H), np.uint16)
            R[0, o, h] = one
            out = oracle.post(np.zeros((1, H), np.uint16), R, post, comb)
            expect = np.zeros((1, 4, H))
            expect[0, :, h] = comb[0, o, :]
            np.testing.assert_array_equal(out, expect)
    for h in range(H):
        x = np.zeros((1, H), np.uint16)
        x[0, h] = one
        out = oracle.post(x, np.zeros((1, 4, H), np.uint16), post, comb)
        expect = np.zeros((1, 4, H))
        expect[0, :, h] = post[0]
        np.testing.assert_array_equal(out, expect)


# ----------------------------------------------------------------------------- bf16 rounding

def test_round_bf16_special_values():
    cases = {
        1.0 + 2.0 ** -8: 1.0,                          # tie -> even (mantissa 0)
        1.0 + 3 * 2.0 ** -8: 1.0 + 2.0 ** -6,          # tie -> even (mantissa 2)
        -(1.0 + 2.0 ** -8): -1.0,
        1.0 + 2.0 ** -8 + 2.0 ** -40: 1.0 + 2.0 ** -7,  # just above the tie
        2.0 ** -130: 2.0 ** -130,                      # subnormal, exact
        3 * 2.0 ** -134: 2.0 ** -132,                  # subnormal tie -> even
        2.0 ** -140: 0.0,                              # below half the smallest subnormal
        (2 - 2.0 ** -7) * 2.0 ** 127: (2 - 2.0 ** -7) * 2.0 ** 127,
        2.0 ** 128 * (1 - 2.0 ** -9): math.inf,        # rounds past the largest finite value
        0.0: 0.0,
    }
    got = oracle.round_bf16(np.array(list(cases)))
    np.testing.assert_array_equal(got, np.array(list(cases.values())))
    assert np.isnan(oracle.round_bf16(np.array([math.nan]))[0])


def test_round_bf16_matches_torch_on_fp32_values():
    """For values exactly representable in fp32, the rounding must equal torch's fp32 -> bf16
    conversion (a library round-to-nearest-even), including every tie."""
    v = np.concatenate([
        RNG.standard_normal(20000).astype(np.float32),
        (RNG.standard_normal(2000) * 1e-38).astype(np.float32),
        # ties: low 16 bits exactly 0x8000
        ((RNG.integers(0x3f000000, 0x41000000, 2000, dtype=np.uint32) & 0xffff0000) | 0x8000)
        .view(np.float32),
    ])
    expect = torch.from_numpy(v).to(torch.bfloat16).float().numpy().astype(np.float64)
    np.testing.assert_array_equal(oracle.round_bf16(v.astype(np.float64)), expect)


# ----------------------------------------------------------------------------- cross-restatement

@pytest.mark.parametrize("T,H", [(1, 8), (3, 16), (4, 127)])
def test_c_oracle_matches_numpy_restatement(T, H):
    R = rand_bits((T, 4, H))
    x = rand_bits((T, H))
    W = (RNG.standard_normal((4 * H, 24)) * 0.02).astype(np.float32)
    scale = (RNG.random(3) + 0.5).astype(np.float32)
    base = (RNG.standard_normal(24) * 0.1).astype(np.float32)
    a = oracle.pre(R, W, scale, base, pre_eps=1e-6, post_mult=2.0, iters=20, eps=1e-6)
    b = numpy_ref.pre(R, W, scale, base, pre_eps=1e-6, post_mult=2.0, iters=20, eps=1e-6)
    for key in ("rstd", "logits", "pre", "post", "comb", "y"):
        np.testing.assert_allclose(a[key], b[key], rtol=1e-12, atol=1e-13, err_msg=key)
    p32 = a["post"].astype(np.float32)
    c32 = a["comb"].astype(np.float32)
    np.testing.assert_allclose(oracle.post(x, R, p32, c32), numpy_ref.post(x, R, p32, c32),
                               rtol=1e-12, atol=1e-13)
