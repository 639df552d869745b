"""Seeded synthetic inputs for the mHC pre-map / post-map workloads.

This module draws random numbers and nothing else: it holds none of the method's arithmetic (no
norm, projection, gate or Sinkhorn), so both the CUDA path's tests/bench and the CPU oracle can use
it. Coefficients that a workload defines *through* the method (the post-map's ``post = 2*sigmoid(z)``
and ``comb = Sinkhorn(exp(z))``) are returned as the raw normal draws ``z_post`` / ``z_comb``; the
caller turns them into coefficients.

Recipe (one ``torch.Generator('cpu')`` per workload, seeded; draw order R, x, hc_fn, hc_scale,
hc_base, then the extras; fp32 draws rounded to bf16 with round-to-nearest-even):

=========  ======================================================================================
workload   distributions
=========  ======================================================================================
small      T=64, H=512; R, x ~ N(0,1); hc_fn [2048,24] ~ N(0, 0.02); scale = 1; base = 0; seed 0
post4k     T=4096, H=4096, post-map only; R, x ~ N(0,1); z_post [T,4], z_comb [T,4,4] ~ N(0,1);
           seed 1
large      T=8192, H=7168; R, x ~ N(0,1); hc_fn [28672,24] ~ N(0, 0.02); scale ~ U(0.5, 1.5);
           base ~ N(0, 0.1); seed 2
decode     T in {1,4,16,32}, H=7168; the large recipe with seed 3, drawn once at T=32, smaller T
           take the first T tokens
tail       T=3000, H=1000; the large weight recipe; R ~ N(0,1) times 100 where a Bernoulli(0.01)
           mask is set; z_comb ~ 3 * N(0,1) (near-permutation comb); 50 Sinkhorn rounds; seed 4
=========  ======================================================================================

Every pre+post workload also draws ``z_post`` [T,4] and ``z_comb`` [T,4,4] after the weights, so the
post-map can be checked on its own with coefficients that do not come from the pre-map.
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

HC = 4
MIX = 24


@dataclasses.dataclass
class Workload:
    name: str
    T: int
    H: int
    R: np.ndarray          # uint16 bf16 bits [T,4,H]
    x: np.ndarray          # uint16 bf16 bits [T,H]
    hc_fn: np.ndarray      # float32 [4H,24]
    hc_scale: np.ndarray   # float32 [3]
    hc_base: np.ndarray    # float32 [24]
    z_post: np.ndarray     # float32 [T,4]   raw normal draws for the post-map's post coefficients
    z_comb: np.ndarray     # float32 [T,4,4] raw draws (already scaled) for the comb logits
    iters: int = 20
    eps: float = 1e-6
    rms_eps: float = 1e-6
    pre_eps: float = 0.0
    post_mult: float = 2.0

    def take(self, T: int) -> "Workload":
        """The first T tokens (decode workloads share one draw)."""
        return dataclasses.replace(
            self, name=f"{self.name}_T{T}", T=T, R=self.R[:T], x=self.x[:T],
            z_post=self.z_post[:T], z_comb=self.z_comb[:T])


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def _draw(name, T, H, seed, *, unit_weights=False, outliers=False, comb_std=1.0, iters=20):
    g = torch.Generator("cpu").manual_seed(seed)
    R = torch.randn((T, HC, H), generator=g, dtype=torch.float32)
    x = torch.randn((T, H), generator=g, dtype=torch.float32)
    hc_fn = torch.randn((HC * H, MIX), generator=g, dtype=torch.float32) * 0.02
    if unit_weights:
        scale = torch.ones(3, dtype=torch.float32)
        base = torch.zeros(MIX, dtype=torch.float32)
    else:
        scale = torch.rand(3, generator=g, dtype=torch.float32) + 0.5
        base = torch.randn(MIX, generator=g, dtype=torch.float32) * 0.1
    if outliers:
        mask = torch.rand((T, HC, H), generator=g, dtype=torch.float32) < 0.01
        R = torch.where(mask, R * 100.0, R)
    z_post = torch.randn((T, HC), generator=g, dtype=torch.float32)
    z_comb = torch.randn((T, HC, HC), generator=g, dtype=torch.float32) * comb_std
    return Workload(name=name, T=T, H=H, R=_bf16_bits(R), x=_bf16_bits(x),
                    hc_fn=hc_fn.numpy().copy(), hc_scale=scale.numpy().copy(),
                    hc_base=base.numpy().copy(), z_post=z_post.numpy().copy(),
                    z_comb=z_comb.numpy().copy(), iters=iters)


def small(T: int = 64, H: int = 512, seed: int = 0) -> Workload:
    return _draw("small", T, H, seed, unit_weights=True)


def post4k(T: int = 4096, H: int = 4096, seed: int = 1) -> Workload:
    return _draw("post4k", T, H, seed)


def large(T: int = 8192, H: int = 7168, seed: int = 2) -> Workload:
    return _draw("large", T, H, seed)


def decode(T: int = 32, H: int = 7168, seed: int = 3) -> Workload:
    return _draw("decode", 32, H, seed).take(T) if T <= 32 else _draw("decode", T, H, seed)


def tail(T: int = 3000, H: int = 1000, seed: int = 4) -> Workload:
    return _draw("tail", T, H, seed, outliers=True, comb_std=3.0, iters=50)


def custom(T: int, H: int, seed: int, *, outliers=False, comb_std=1.0, iters=20) -> Workload:
    """The large recipe at any size (extra parity shapes such as H=127 or H=1001)."""
    return _draw(f"T{T}_H{H}_s{seed}", T, H, seed, outliers=outliers, comb_std=comb_std,
                 iters=iters)


@dataclasses.dataclass
class Partials:
    """Inputs of the pre-map from an external projection: split partials of the projection and of
    the sum of squares, with the residual they belong to."""
    T: int
    H: int
    R: np.ndarray        # uint16 bf16 bits [T,4,H]
    dot_mix: np.ndarray  # float32 [S,T,24]
    sqrsum: np.ndarray   # float32 [S,T]
    hc_scale: np.ndarray  # float32 [3]
    hc_base: np.ndarray   # float32 [24]


def partials(T: int, H: int, num_splits: int, seed: int) -> Partials:
    """The recipe of the FlashInfer article's minimal call (§5.1): R ~ N(0,1) bf16; per split
    dot_mix ~ 0.01 N(0,1) and sqrsum ~ U(0,1) * k / num_splits (k = 4H); scale ~ 0.1 N(0,1),
    base ~ 0.1 N(0,1). Draw order R, dot_mix, sqrsum, scale, base."""
    g = torch.Generator("cpu").manual_seed(seed)
    R = torch.randn((T, HC, H), generator=g, dtype=torch.float32)
    dot = torch.randn((num_splits, T, MIX), generator=g, dtype=torch.float32) * 0.01
    sq = torch.rand((num_splits, T), generator=g, dtype=torch.float32) * float(4 * H / num_splits)
    scale = torch.randn(3, generator=g, dtype=torch.float32) * 0.1
    base = torch.randn(MIX, generator=g, dtype=torch.float32) * 0.1
    return Partials(T=T, H=H, R=_bf16_bits(R), dot_mix=dot.numpy().copy(), sqrsum=sq.numpy().copy(),
                    hc_scale=scale.numpy().copy(), hc_base=base.numpy().copy())


WORKLOADS = {"small": small, "post4k": post4k, "large": large, "decode": decode, "tail": tail}
