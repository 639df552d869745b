"""Token sharding across ranks (one process per GPU).

Every token of the pre-map and the post-map is independent of every other ("FlashInfer mHC module
deep dive" §3.4: one CTA per token; glm5next_mhc.rs: grids over tokens), so a batch is split into
contiguous token ranges, one per rank, and no data-path collective is needed. The only exchange is
the benchmark's timing reduction (the slowest rank's time).
"""

from __future__ import annotations


def token_shards(T: int, world: int) -> list[tuple[int, int]]:
    """Contiguous [start, end) token ranges, one per rank, sizes differing by at most one."""
    if T < 0 or world < 1:
        raise ValueError("T >= 0 and world >= 1 required")
    base, extra = divmod(T, world)
    out, start = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((start, start + n))
        start += n
    return out


def global_max(value: float, device=None) -> float:
    """Max of `value` over the ranks of the default process group (the value itself when none)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(tokens_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)
