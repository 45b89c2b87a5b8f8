"""FP8 quantization of a tensor whose rows are split over several GPUs (one process per GPU).

Block modes (1x128, 128x128) shard with no communication: every block lies in
one shard as long as shard boundaries fall on multiples of the block height,
and each block's scale depends only on its own elements (mixed-precision
handbook, "FP8 training", per_block).

Per-tensor current scaling has one real exchange: the scale of the whole
tensor needs the amax of all shards (PyTorch-FP8 page s4.1), so each rank
reduces its shard's amax on its GPU, the ranks all-reduce (MAX) that one
fp32 value, and each rank then forms the scale and casts its shard.  Delayed
scaling (s4.2) needs no exchange before the cast; ShardedDelayedScaler
all-reduces the amax after it, for the history update, off the critical path.

The compute steps are the library's kernels.  ``ShardOps`` bundles them so
that a test can substitute a CPU implementation and check the collective
logic on gloo ranks without a GPU.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist


def row_shard(rows: int, world: int, rank: int, multiple: int = 128) -> tuple[int, int]:
    """Rows [start, stop) of `rank`: contiguous, balanced in units of `multiple` rows (the last shard takes
    the remainder), so that no 128-row block straddles two ranks."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    units = -(-rows // multiple)
    per, extra = divmod(units, world)
    u0 = rank * per + min(rank, extra)
    u1 = u0 + per + (1 if rank < extra else 0)
    return min(rows, u0 * multiple), min(rows, u1 * multiple)


@dataclass
class ShardOps:
    """The per-shard compute steps (default: the CUDA library)."""
    amax: Callable[[torch.Tensor], torch.Tensor]                          # x -> [1] fp32
    scale_from_amax: Callable[[torch.Tensor, int], torch.Tensor]          # amax, fmt -> [1] fp32
    cast: Callable[[torch.Tensor, int, torch.Tensor], torch.Tensor]       # x, fmt, scale -> codes
    blockwise: Callable[[torch.Tensor, tuple, int], tuple]                # x, block, fmt -> (codes, scales)


def library_ops() -> ShardOps:
    from . import binding as B

    def cast(x, fmt, scale):
        q, _, _ = B.fp8_quantize_per_tensor(x, fmt, scale_in=scale, want_amax=False)
        return q

    return ShardOps(amax=B.fp8_amax, scale_from_amax=B.fp8_scale_from_amax, cast=cast,
                    blockwise=lambda x, block, fmt: B.fp8_quantize_blockwise(x, block, fmt))


def _world(group) -> int:
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def quantize_per_tensor_sharded(x_local: torch.Tensor, fmt: int, group=None, ops: ShardOps | None = None):
    """Current per-tensor scaling of a row-sharded tensor.

    Returns (codes of this shard, the global scale [1], the global amax [1]); every rank gets the same
    scale, equal to the one the whole tensor would get on one GPU."""
    ops = ops or library_ops()
    amax = ops.amax(x_local)
    if _world(group) > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    scale = ops.scale_from_amax(amax, fmt)
    return ops.cast(x_local, fmt, scale), scale, amax


def quantize_blockwise_sharded(x_local: torch.Tensor, block=(1, 128), fmt: int = 0, ops: ShardOps | None = None):
    """Blockwise quantization of this rank's rows (shard boundaries on multiples of the block height):
    no communication; the result equals the unsharded one restricted to these rows."""
    ops = ops or library_ops()
    return ops.blockwise(x_local, tuple(block), fmt)


@dataclass
class DelayedOps:
    """The per-shard steps of delayed scaling (default: the CUDA library).

    new_state(window, fmt, algo, alpha, margin, device) -> state with .scale ([1] fp32, the scale the next
    cast uses); cast_amax(x, state) -> (codes, this shard's amax [1]) with the state's scale;
    update(state, amax) pushes the (global) amax into the history and refreshes state.scale."""
    new_state: Callable
    cast_amax: Callable
    update: Callable


def library_delayed_ops() -> DelayedOps:
    from . import binding as B

    def new_state(window, fmt, algo, alpha, margin, device):
        return B.DelayedScaler(window=window, fmt=fmt, device=device, algo=algo, alpha=alpha, margin=margin,
                               fused=False)

    def cast_amax(x, st):
        q, _, amax = B.fp8_quantize_per_tensor(x, st.fmt, scale_in=st.scale, scale_out=st.scale_used,
                                                amax_out=st.amax)
        return q, amax

    def update(st, amax):
        if st.algo == B.AMAX_WINDOW_MAX and st.margin == 1.0:
            B.fp8_amax_history_update(st.history, st.state, amax, st.scale, st.fmt)
        else:
            B.fp8_amax_history_update_ex(st.history, st.state, amax, st.scale, st.fmt, st.algo, st.alpha,
                                         st.margin)

    return DelayedOps(new_state=new_state, cast_amax=cast_amax, update=update)


class ShardedDelayedScaler:
    """Delayed scaling of a row-sharded tensor (PyTorch-FP8 page s4.2, over several GPUs).

    Each step casts this rank's rows with the scale every rank holds, reduces the shard's amax in the same
    pass, then all-reduces (MAX) that one fp32 and pushes the global amax into the history.  The exchange
    comes after the cast, so it is off the cast's critical path; every rank's history and next scale stay
    identical, equal to those of the whole tensor on one GPU."""

    def __init__(self, window: int = 16, fmt: int = 1, group=None, ops: DelayedOps | None = None,
                 device="cuda", algo: int = 0, alpha: float = 1.0, margin: float = 1.0):
        self.ops = ops or library_delayed_ops()
        self.group = group
        self.state = self.ops.new_state(window, fmt, algo, alpha, margin, device)

    @property
    def scale(self) -> torch.Tensor:
        return self.state.scale

    def step(self, x_local: torch.Tensor) -> torch.Tensor:
        q, amax = self.ops.cast_amax(x_local, self.state)
        if _world(self.group) > 1:
            dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=self.group)
        self.ops.update(self.state, amax)
        return q
