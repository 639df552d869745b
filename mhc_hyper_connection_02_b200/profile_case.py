"""Runs one library entry point on seeded synthetic device inputs, `reps` times, so that a profiler
(Nsight Compute) can capture one launch of the kernel behind it.

    python -m mhc_hyper_connection_02_b200.profile_case <case> [--reps N]

Every case draws its inputs on the device from one seeded generator (R, x ~ N(0,1) rounded to
bf16; hc_fn ~ N(0, 0.02); scale ~ U(0.5, 1.5); base ~ N(0, 0.1)) and calls the library through the
binding; nothing else runs between the calls. `python -m mhc_hyper_connection_02_b200.profile_case
list` prints the cases with the kernels they exercise.
"""

from __future__ import annotations

import argparse
import sys

CASES = {
    # name: (what runs, kernels it launches)
    "pre_decode_T1": ("mhc_pre T=1 H=7168", "pre_cc_partial_klane_kernel, pre_cc_finish_kernel"),
    "pre_decode_T32": ("mhc_pre T=32 H=7168", "pre_cc_partial_staged_kernel, pre_cc_finish_kernel"),
    "pre_small": ("mhc_pre T=64 H=512", "pre_cc_partial_kernel, pre_cc_finish_kernel"),
    "pre_split_T3072": ("mhc_pre T=3072 H=7168, split tensor path",
                        "pre_tc_split_kernel, pre_tc_proj_kernel, pre_tc_coef_agg_kernel"),
    "pre_fused_T3072": ("mhc_pre T=3072 H=7168, single-pass path",
                        "pre_fused_zero_kernel, pre_fused_kernel"),
    "pre_large": ("mhc_pre T=8192 H=7168 (default path: the split chain)",
                  "pre_tc_split_kernel, pre_tc_proj_kernel, pre_tc_coef_agg_kernel"),
    "pre_fused_large": ("mhc_pre T=8192 H=7168, single-pass path",
                        "pre_fused_zero_kernel, pre_fused_kernel"),
    "pre_fused_T1024": ("mhc_pre T=1024 H=7168 (default path: the single pass)",
                        "pre_fused_zero_kernel, pre_fused_kernel"),
    "pre_wave_T3072": ("mhc_pre T=3072 H=7168, wavefront single pass",
                       "pre_wave_prep_kernel, pre_wave_kernel, sinkhorn_kernel"),
    "pre_wave_large": ("mhc_pre T=8192 H=7168, wavefront single pass",
                       "pre_wave_prep_kernel, pre_wave_kernel, sinkhorn_kernel"),
    "post_large": ("mhc_post T=8192 H=7168", "post_persistent_kernel"),
    "post_scalar_H1001": ("mhc_post T=8192 H=1001", "post_scalar_kernel"),
    "sinkhorn_T1M": ("mhc_sinkhorn T=1048576", "sinkhorn_kernel"),
    "big_fuse_loop_H1001": ("mhc_pre_big_fuse T=8192 H=1001, 4 splits",
                            "pre_bigfuse_coef_kernel, pre_bigfuse_loop_kernel"),
    "expand_scalar_H1001": ("mhc_expand T=8192 H=1001", "expand_scalar_kernel"),
    "head_mean_scalar_H1001": ("mhc_head_mean T=8192 H=1001", "head_mean_scalar_kernel"),
    "post_backward_large": ("mhc_post_backward T=8192 H=7168", "post_bwd_persistent_kernel"),
    "pre_backward_H1001": ("mhc_pre_backward T=4096 H=1001", "pre_bwd_* (dx scalar form)"),
    "pre_backward_large": ("mhc_pre_backward T=8192 H=7168",
                           "pre_bwd_* (d_R with d_hc_fn on tensor cores: pre_bwd_split_kernel, pre_bwd_drw_kernel)"),
}


def _inputs(T, H, seed=0):
    import torch
    g = torch.Generator(device="cuda").manual_seed(seed)
    R = torch.randn((T, 4, H), device="cuda", generator=g).to(torch.bfloat16)
    x = torch.randn((T, H), device="cuda", generator=g).to(torch.bfloat16)
    W = torch.randn((4 * H, 24), device="cuda", generator=g) * 0.02
    S = torch.rand(3, device="cuda", generator=g) + 0.5
    B = torch.randn(24, device="cuda", generator=g) * 0.1
    return g, R, x, W, S, B


def _coefficients(g, T):
    """post = 2 sigmoid(z) and a doubly stochastic comb (the library's own Sinkhorn of z)."""
    import torch
    from . import sinkhorn
    post = 2.0 * torch.sigmoid(torch.randn((T, 4), device="cuda", generator=g))
    comb = sinkhorn(torch.randn((T, 4, 4), device="cuda", generator=g))
    return post, comb


def make_call(case):
    import torch
    from . import (PRE_PATH_TENSOR_FUSED, PRE_PATH_TENSOR_SPLIT, PRE_PATH_TENSOR_WAVE,
                   POST_PATH_SCALAR, expand,
                   head_mean, post, post_backward, pre, pre_backward, pre_big_fuse, sinkhorn,
                   workspace_bytes)

    def pre_call(T, H, path=0):
        _, R, _, W, S, B = _inputs(T, H)
        ws = torch.empty(workspace_bytes(T, H), dtype=torch.uint8, device="cuda")
        y, p, q, c = pre(R, W, S, B, workspace=ws, path=path)
        return lambda: pre(R, W, S, B, y=y, pre=p, post=q, comb=c, workspace=ws, path=path)

    if case == "pre_decode_T1":
        return pre_call(1, 7168)
    if case == "pre_decode_T32":
        return pre_call(32, 7168)
    if case == "pre_small":
        return pre_call(64, 512)
    if case == "pre_split_T3072":
        return pre_call(3072, 7168, PRE_PATH_TENSOR_SPLIT)
    if case == "pre_fused_T3072":
        return pre_call(3072, 7168, PRE_PATH_TENSOR_FUSED)
    if case == "pre_large":
        return pre_call(8192, 7168)
    if case == "pre_fused_large":
        return pre_call(8192, 7168, PRE_PATH_TENSOR_FUSED)
    if case == "pre_wave_T3072":
        return pre_call(3072, 7168, PRE_PATH_TENSOR_WAVE)
    if case == "pre_wave_large":
        return pre_call(8192, 7168, PRE_PATH_TENSOR_WAVE)
    if case == "pre_fused_T1024":
        return pre_call(1024, 7168)
    if case in ("post_large", "post_scalar_H1001"):
        T, H = (8192, 7168) if case == "post_large" else (8192, 1001)
        g, R, x, _, _, _ = _inputs(T, H)
        pc, cc = _coefficients(g, T)
        out = torch.empty_like(R)
        path = POST_PATH_SCALAR if case == "post_scalar_H1001" else 0
        return lambda: post(x, R, pc, cc, out=out, path=path)
    if case == "sinkhorn_T1M":
        g = torch.Generator(device="cuda").manual_seed(0)
        lg = torch.randn((1 << 20, 4, 4), device="cuda", generator=g)
        out = torch.empty_like(lg)
        return lambda: sinkhorn(lg, comb=out)
    if case == "big_fuse_loop_H1001":
        T, H, S_ = 8192, 1001, 4
        g, R, _, _, S, B = _inputs(T, H)
        dot = torch.randn((S_, T, 24), device="cuda", generator=g) * 0.01
        sq = torch.rand((S_, T), device="cuda", generator=g) * (4 * H / S_)
        y, p, q, c = pre_big_fuse(dot, sq, R, S, B, 4 * H, num_splits=S_)
        return lambda: pre_big_fuse(dot, sq, R, S, B, 4 * H, num_splits=S_, y=y, pre=p, post=q,
                                    comb=c)
    if case == "expand_scalar_H1001":
        _, _, x, _, _, _ = _inputs(8192, 1001)
        st = torch.empty((8192, 4, 1001), dtype=torch.bfloat16, device="cuda")
        return lambda: expand(x, streams=st)
    if case == "head_mean_scalar_H1001":
        _, R, _, _, _, _ = _inputs(8192, 1001)
        y = torch.empty((8192, 1001), dtype=torch.bfloat16, device="cuda")
        return lambda: head_mean(R, y=y)
    if case == "post_backward_large":
        T, H = 8192, 7168
        g, R, x, _, _, _ = _inputs(T, H)
        pc, cc = _coefficients(g, T)
        dout = torch.randn((T, 4, H), device="cuda", generator=g).to(torch.bfloat16)
        return lambda: post_backward(dout, x, R, pc, cc)
    if case in ("pre_backward_H1001", "pre_backward_large"):
        T, H = (4096, 1001) if case == "pre_backward_H1001" else (8192, 7168)
        g, R, x, W, S, B = _inputs(T, H)
        dy = torch.randn((T, H), device="cuda", generator=g).to(torch.bfloat16)
        return lambda: pre_backward(R, W, S, B, d_y=dy)
    raise KeyError(case)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("case", choices=sorted(CASES) + ["list"])
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args(argv)
    if args.case == "list":
        for k, (what, kernels) in CASES.items():
            print(f"{k:24s} {what:45s} {kernels}")
        return 0
    import torch
    from . import device_status
    call = make_call(args.case)
    for _ in range(args.reps):
        call()
    torch.cuda.synchronize()
    st = device_status()
    print(f"{args.case}: {args.reps} calls, device status {st}")
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
