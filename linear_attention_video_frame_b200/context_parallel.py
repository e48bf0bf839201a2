"""Context-parallel frame-wise GDN scan over ranks (one process per GPU).

SANA-WM paper summary (paperlayer), appendix C.1, "Context-parallel
training": the latent sequence is sharded along time over P GPUs; every
rank owns one frame interval, summarises it by a compact transition
composite and input composite, all-gathers the summaries, composes them as
an exclusive prefix to recover its exact initial state, and scans its own
frames from there.  (SANA-WM digest, method details, "Context-Parallel +
Fused Triton" paragraph, says the same.)

Per rank, with the rank's q, k, v of shape [B, H, F_r, S, D]:
  1. la_gdn_interval_composite  -> (T_r, U_r)        one [2, B, H, D, D] buffer
  2. all-gather of that buffer   -> [P, 2, B, H, D, D] (one collective,
                                    2 B H D^2 floats per rank)
  3. la_gdn_compose_prefix       -> start state of every interval, and the
                                    state after the whole clip
  4. la_scan_gdn from start_r    -> this rank's outputs

Steps 1, 3 and 4 are this library's kernels; step 2 is torch.distributed
(NCCL between GPUs).  Every rank takes the same collective in the same
order.  The compute steps are reached through an `ops` object so that the
same orchestration runs on CPU ranks in tests.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

__all__ = ["frame_interval", "DeviceOps", "cp_scan_gdn"]


def frame_interval(F: int, world: int, rank: int) -> Tuple[int, int]:
    """Frames [f0, f1) of a clip of F frames that rank `rank` of `world`
    owns: contiguous intervals in rank order, sizes differing by at most one
    (the first F % world ranks hold one more frame)."""
    if world < 1 or not 0 <= rank < world or F < 0:
        raise ValueError(f"bad split: F={F} world={world} rank={rank}")
    base, extra = divmod(F, world)
    f0 = rank * base + min(rank, extra)
    return f0, f0 + base + (1 if rank < extra else 0)


class DeviceOps:
    """The three compute steps on this library's CUDA kernels."""

    dtype = torch.float32          # composites and states

    def composite(self, k, v, alpha, beta, k_scale: float, out: torch.Tensor) -> torch.Tensor:
        from . import la_gdn_interval_composite
        return la_gdn_interval_composite(k, v, alpha, beta, k_scale, out=out)

    def compose(self, gathered: torch.Tensor, state_in, state_out) -> torch.Tensor:
        from . import la_gdn_compose_prefix
        return la_gdn_compose_prefix(gathered, state_in=state_in, state_out=state_out)

    def scan(self, q, k, v, alpha, beta, k_scale: float, state_in) -> torch.Tensor:
        from . import la_scan_gdn
        return la_scan_gdn(q, k, v, alpha, beta, k_scale, state_in=state_in)


def cp_scan_gdn(q, k, v, alpha, beta, k_scale: float, state_in: Optional[torch.Tensor] = None,
                state_out: Optional[torch.Tensor] = None, group=None, ops=None) -> torch.Tensor:
    """The GDN scan of a clip whose frames are split over the ranks of
    `group` in rank order (see frame_interval).

    q, k, v [B, H, F_r, S, D], alpha, beta [B, H, F_r]: this rank's frames.
    state_in [B, H, D, D]: the state before the clip (the same on every
    rank), or None for zeros.  state_out [B, H, D, D]: if given, receives
    the state after the whole clip (the same on every rank).
    Returns this rank's outputs o [B, H, F_r, S, D].
    """
    ops = ops or DeviceOps()
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    B, H, _, _, D = k.shape
    mine = torch.empty((2, B, H, D, D), dtype=ops.dtype, device=k.device)
    ops.composite(k, v, alpha, beta, k_scale, mine)
    if world > 1:
        flat = torch.empty((world * 2, B, H, D, D), dtype=ops.dtype, device=k.device)
        dist.all_gather_into_tensor(flat, mine, group=group)     # rank order along dim 0
        gathered = flat.view(world, 2, B, H, D, D)
    else:
        gathered = mine[None]
    starts = ops.compose(gathered, state_in, state_out)
    return ops.scan(q, k, v, alpha, beta, k_scale, starts[rank])
