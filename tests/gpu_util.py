"""Helpers for the GPU tests: move seeded numpy inputs to the device and results back."""

import numpy as np
import torch

import oracle


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def post_coefficients(w):
    """The post-map's own coefficients for workload w: post = 2*sigmoid(z_post) (fp32, numpy) and
    comb = the oracle's Sinkhorn of z_comb with the workload's rounds, rounded to fp32."""
    z = w.z_post.astype(np.float64)
    post = (2.0 / (1.0 + np.exp(-z))).astype(np.float32)
    comb = oracle.sinkhorn(w.z_comb.astype(np.float64), iters=w.iters, eps=w.eps).astype(np.float32)
    return post, comb
