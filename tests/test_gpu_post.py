"""GPU parity of the post-map (all three kernels) against the fp64 oracle, through the C ABI.

out[t][n][h] = x[h]*post[n] + sum_o R[o][h]*comb[o][n] ("FlashInfer mHC module deep dive" §2.1,
glm5next_mhc.rs glm_hc_post). The oracle gets the very fp32 post/comb the kernel gets; those come
from the seeded draws (post = 2*sigmoid(z), comb = oracle Sinkhorn of z), never from the GPU.
"""

import numpy as np
import pytest
import torch

import oracle
import mhc_hyper_connection_02_b200 as mhc
from mhc_hyper_connection_02_b200 import inputs
from gpu_util import dev_bf16, dev_f32, host_bits, post_coefficients
from tolerance import U32, bf16_bits_to_f64, check_bf16

pytestmark = pytest.mark.gpu

PATHS = {"vec8": mhc.POST_PATH_VEC8, "persistent": mhc.POST_PATH_PERSISTENT,
         "scalar": mhc.POST_PATH_SCALAR}


def post_terms_bound(x_bits, R_bits, post, comb):
    """E = 6 * 2^-24 * (|x*post[n]| + sum_o |R[o]*comb[o][n]|): one product and four FMAs."""
    x = np.abs(bf16_bits_to_f64(x_bits))[:, None, :]
    R = np.abs(bf16_bits_to_f64(R_bits))
    s = x * np.abs(post.astype(np.float64))[:, :, None]
    s = s + np.einsum("toh,ton->tnh", R, np.abs(comb.astype(np.float64)))
    return 6 * U32 * s


def compare(out_dev, w, post, comb, rows=None, label=""):
    R, x = w.R, w.x
    if rows is not None:
        R, x, post, comb = R[rows], x[rows], post[rows], comb[rows]
    ref = oracle.post(x, R, post, comb)
    got = host_bits(out_dev if rows is None else out_dev[torch.as_tensor(rows, device="cuda")])
    fail, need, worst = check_bf16(got, ref, oracle.round_bf16(ref), post_terms_bound(x, R, post, comb))
    print(f"[post {label}] fail={fail} derived-bound={need} worst/tol={worst:.3f} n={ref.size}")
    assert fail == 0


def compare_all(out_dev, w, post, comb, label="", chunk=1024):
    """Every token, checked in chunks of `chunk` tokens (bounded host memory at the full size)."""
    for c0 in range(0, w.T, chunk):
        compare(out_dev, w, post, comb, rows=np.arange(c0, min(w.T, c0 + chunk)),
                label=f"{label} [{c0}:{min(w.T, c0 + chunk)}]")


def run(w, path, post, comb, out=None):
    x, R = dev_bf16(w.x), dev_bf16(w.R)
    o = mhc.post(x, R, dev_f32(post), dev_f32(comb), out=out, path=path)
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    return o


@pytest.mark.parametrize("H", [8, 64, 127, 512, 1000, 1001, 1536, 2048, 4096, 7168, 8192, 16392])
@pytest.mark.parametrize("path", ["vec8", "persistent", "scalar"])
def test_post_matches_oracle(H, path):
    if H % 8 and path != "scalar":
        pytest.skip("vector paths need H % 8 == 0")
    T = 37 if H <= 8192 else 9
    w = inputs.custom(T, H, seed=100 + H)
    post, comb = post_coefficients(w)
    out = run(w, PATHS[path], post, comb)
    compare(out, w, post, comb, label=f"H={H} {path}")


@pytest.mark.parametrize("path", ["vec8", "persistent", "scalar"])
def test_post_in_place_equals_out_of_place(path):
    w = inputs.custom(29, 4096, seed=5)
    post, comb = post_coefficients(w)
    ref = run(w, PATHS[path], post, comb)
    R = dev_bf16(w.R)
    o = mhc.post(dev_bf16(w.x), R, dev_f32(post), dev_f32(comb), out=R, path=PATHS[path])
    torch.cuda.synchronize()
    assert o.data_ptr() == R.data_ptr()
    assert torch.equal(R.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("path", ["vec8", "persistent", "scalar"])
def test_post_identity_permutation_and_broadcast(path):
    T, H = 11, 264
    w = inputs.custom(T, H, seed=9)
    zero = np.zeros((T, 4), np.float32)
    o = run(w, PATHS[path], zero, np.tile(np.eye(4, dtype=np.float32), (T, 1, 1)))
    np.testing.assert_array_equal(host_bits(o), w.R)                   # comb = I, post = 0
    p = (2, 0, 3, 1)
    P = np.zeros((4, 4), np.float32)
    P[np.arange(4), p] = 1.0
    o = run(w, PATHS[path], zero, np.tile(P, (T, 1, 1)))
    np.testing.assert_array_equal(host_bits(o), w.R[:, np.argsort(p), :])
    o = run(w, PATHS[path], np.ones((T, 4), np.float32), np.zeros((T, 4, 4), np.float32))
    for n in range(4):
        np.testing.assert_array_equal(host_bits(o)[:, n, :], w.x)      # comb = 0, post = 1


def test_post_misaligned_views_take_the_scalar_path():
    T, H = 13, 512
    w = inputs.custom(T, H, seed=21)
    post, comb = post_coefficients(w)
    x_big = torch.zeros(T * H + 1, dtype=torch.bfloat16, device="cuda")
    x_big[1:] = dev_bf16(w.x).view(-1)
    x = x_big[1:].view(T, H)                       # 2-byte offset: not 16-byte aligned
    R = dev_bf16(w.R)
    with pytest.raises(mhc.MhcError) as e:
        mhc.post(x, R, dev_f32(post), dev_f32(comb), path=mhc.POST_PATH_VEC8)
    assert e.value.status == mhc.MHC_ERR_UNSUPPORTED
    out = mhc.post(x, R, dev_f32(post), dev_f32(comb))   # auto -> scalar
    torch.cuda.synchronize()
    compare(out, w, post, comb, label="misaligned")


def test_post_guard_bands_untouched():
    T, H = 17, 1000
    w = inputs.custom(T, H, seed=33)
    post, comb = post_coefficients(w)
    pad = 4096
    for path in PATHS.values():
        buf = torch.full((pad + T * 4 * H + pad,), -7.0, dtype=torch.bfloat16, device="cuda")
        out = buf[pad:pad + T * 4 * H].view(T, 4, H)
        run(w, path, post, comb, out=out)
        assert torch.all(buf[:pad] == -7.0) and torch.all(buf[pad + T * 4 * H:] == -7.0)
        compare(out, w, post, comb, label=f"guard {path}")


def test_post_empty_and_single_token():
    w = inputs.custom(1, 8, seed=1)
    post, comb = post_coefficients(w)
    for path in PATHS.values():
        compare(run(w, path, post, comb), w, post, comb, label="T=1")
    e = torch.empty((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    o = mhc.post(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"), e,
                 torch.empty((0, 4), device="cuda"), torch.empty((0, 4, 4), device="cuda"))
    assert o.shape == (0, 4, 64)


def test_post_rejects_host_memory():
    """A host pointer in the residual slot is refused before any launch."""
    w = inputs.custom(4, 64, seed=2)
    post, comb = post_coefficients(w)
    R_host = torch.from_numpy(w.R.view(np.int16)).view(torch.bfloat16)
    out = torch.empty((4, 4, 64), dtype=torch.bfloat16, device="cuda")
    st = mhc.lib().mhc_post(dev_bf16(w.x).data_ptr(), R_host.data_ptr(), dev_f32(post).data_ptr(),
                            dev_f32(comb).data_ptr(), out.data_ptr(), 4, 64, None)
    assert st == mhc.MHC_ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["post4k", "tail"])
def test_post_workloads(name):
    """Every token of the post-only (T=4096, H=4096) and tail (T=3000, H=1000) workloads."""
    w = inputs.WORKLOADS[name]()
    post, comb = post_coefficients(w)
    for path in (["vec8", "persistent"] if w.H % 8 == 0 else []) + ["scalar"]:
        out = run(w, PATHS[path], post, comb)
        compare_all(out, w, post, comb, label=f"{name} {path}")


@pytest.mark.slow
def test_post_large_full_batch():
    """T=8192, H=7168, every token, for the default call (the persistent kernel bench.py times)
    and the vec8 kernel."""
    w = inputs.large()
    post, comb = post_coefficients(w)
    for path in (mhc.PATH_AUTO, mhc.POST_PATH_VEC8):
        out = run(w, path, post, comb)
        compare_all(out, w, post, comb, label=f"large path={path}")
        del out
        torch.cuda.empty_cache()


@pytest.mark.slow
@pytest.mark.parametrize("name", ["post4k", "large"])
def test_post_persistent_in_place_at_size(name):
    """In place (out == R) on the persistent kernel at sizes where every CTA runs many tiles, so
    its prefetch ring runs ahead of the in-place writes: equal, bit for bit, to out of place."""
    w = inputs.WORKLOADS[name]()
    post, comb = post_coefficients(w)
    x, p, c = dev_bf16(w.x), dev_f32(post), dev_f32(comb)
    ref = mhc.post(x, dev_bf16(w.R), p, c, path=mhc.POST_PATH_PERSISTENT)
    R = dev_bf16(w.R)
    o = mhc.post(x, R, p, c, out=R, path=mhc.POST_PATH_PERSISTENT)
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    assert o.data_ptr() == R.data_ptr()
    assert torch.equal(R.view(torch.int16), ref.view(torch.int16))
    if name == "post4k":
        compare_all(R, w, post, comb, label="post4k in place")
