"""The library's calls under CUDA graph capture (the launch-bound serving loop): one pre-map +
post-map step captured once and replayed gives bitwise the eager results, for the tensor-core
split chain (chained with programmatic dependent launch), the single-pass cooperative kernel
(T=512, H=7168) and the CUDA-core decode path."""

import numpy as np
import pytest
import torch

import mhc_hyper_connection_02_b200 as mhc
from mhc_hyper_connection_02_b200 import inputs
from gpu_util import dev_bf16, dev_f32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,H", [(4, 7168), (256, 1024), (512, 7168)])
def test_graph_replay_matches_eager(T, H):
    w = inputs.custom(T, H, seed=T + H)
    R, x = dev_bf16(w.R), dev_bf16(w.x)
    W, sc, bs = dev_f32(w.hc_fn), dev_f32(w.hc_scale), dev_f32(w.hc_base)
    ws = torch.empty(mhc.workspace_bytes(T, H), dtype=torch.uint8, device="cuda")
    y, pre, post, comb = (torch.empty((T, H), dtype=torch.bfloat16, device="cuda"),
                          torch.empty((T, 4), device="cuda"), torch.empty((T, 4), device="cuda"),
                          torch.empty((T, 4, 4), device="cuda"))
    out = torch.empty_like(R)
    s = torch.cuda.Stream()

    def step():
        mhc.pre(R, W, sc, bs, y=y, pre=pre, post=post, comb=comb, workspace=ws, stream=s)
        mhc.post(x, R, post, comb, out=out, stream=s)

    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # eager, also does first-call setup outside the capture
    torch.cuda.synchronize()
    ref = [t.clone() for t in (y, pre, post, comb, out)]
    for t in (y, pre, post, comb, out):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert mhc.device_status() == 0
    for a, b in zip((y, pre, post, comb, out), ref):
        assert torch.equal(a.view(torch.uint8) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.uint8) if b.dtype == torch.bfloat16 else b)
    del g
