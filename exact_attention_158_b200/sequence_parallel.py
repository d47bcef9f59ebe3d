"""Sequence-sharded attention forward across GPUs, one process per GPU.

Sequence-length parallelism ("FlashAttention-2 GPU work partitioning", section 3: a long sequence
is divided among several workers) carried from thread blocks to devices: every rank holds one
contiguous range of each (b, h) sequence's keys and values and all of its queries.

    1. fa_fwd_keyrange: the partial (O normalised over the local keys each query sees, in fp32,
       and LSE) of every query over the local key range -- the CUDA kernel;
    2. an all-gather of the partials over the process group (NCCL between GPUs): d + 1 floats per
       query row per rank;
    3. fa_merge_partials: the rescaling merge ("Flash Attention" (myungum), section 2, steps
       11-12) of the gathered partials, locally on every rank -- a CUDA kernel.

Every rank ends with the full O and LSE.  The exchange is a plain collective here; the partial
and merge steps are this library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import fa_fwd_keyrange, fa_merge_partials


def key_ranges(N: int, world: int) -> list[tuple[int, int]]:
    """Contiguous [start, end) key ranges of a length-N sequence over `world` ranks, sizes
    differing by at most one (the first N % world ranges one longer)."""
    if N < world:
        raise ValueError("each rank needs at least one key")
    base, extra = divmod(N, world)
    out, start = [], 0
    for r in range(world):
        end = start + base + (1 if r < extra else 0)
        out.append((start, end))
        start = end
    return out


def _device_partial(q, k_local, v_local, k_pos0, causal, scale):
    return fa_fwd_keyrange(q, k_local, v_local, q_row0=0, k_pos0=k_pos0, causal=causal,
                           scale=scale, out_dtype=torch.float32)


def _device_merge(o_parts, lse_parts, out_dtype):
    return fa_merge_partials(o_parts, lse_parts, out_dtype=out_dtype)


def sequence_parallel_attention(q, k_local, v_local, k_pos0: int, causal: bool = False,
                                scale: float | None = None, out_dtype=torch.bfloat16, group=None,
                                *, partial=None, merge=None):
    """q [B, H, N, d] (the same on every rank); k_local, v_local [B, H, Nk, d]: this rank's keys
    and values at positions k_pos0 .. k_pos0 + Nk - 1 (the ranks' ranges tile 0 .. N - 1).
    Returns (o [B, H, N, d], lse [B, H, N]) on every rank.

    `partial(q, k, v, k_pos0, causal, scale) -> (o fp32, lse)` and
    `merge(o_parts, lse_parts, out_dtype) -> (o, lse)` default to the CUDA kernels; they are
    parameters so that the exchange logic can be exercised with other implementations."""
    partial = partial or _device_partial
    merge = merge or _device_merge
    o_part, lse_part = partial(q, k_local, v_local, k_pos0, causal, scale)
    world = dist.get_world_size(group)
    o_all = torch.empty((world, *o_part.shape), dtype=o_part.dtype, device=o_part.device)
    l_all = torch.empty((world, *lse_part.shape), dtype=lse_part.dtype, device=lse_part.device)
    dist.all_gather(list(o_all.unbind(0)), o_part.contiguous(), group=group)
    dist.all_gather(list(l_all.unbind(0)), lse_part.contiguous(), group=group)
    return merge(o_all, l_all, out_dtype)
