"""One DeltaQuant layer sharded by cubes across ranks (one per GPU).

X is cut along T into slabs of whole cubes: every quantity of the layer is
local to a cube (its mean, its kernel token and scale, its deltas, its rows of
Y) except the per-tensor delta scale, which needs the largest |delta| over all
cubes.  So each rank runs the statistics pass on its slab, the ranks take the
maximum of that one fp32 (a single all-reduce of four bytes), and each rank
then encodes its slab and runs both products.  The result on every row equals
the unsharded layer's bit for bit.  Host logic only: the work runs in the
library's kernels through its C ABI.
"""
from __future__ import annotations

import video_diffusion_w4a4_b200 as dq


def slab_frames(T: int, t: int, world: int, rank: int) -> tuple[int, int]:
    """Frames [t0, t1) of `rank`'s slab: whole cube layers along T (t0 a multiple of t), the
    ceil(T / t) layers spread as evenly as possible, earlier ranks taking the remainder."""
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside 0..{world - 1}")
    layers = -(-T // t)
    if world > layers:
        raise ValueError(f"{world} ranks for {layers} cube layers along T")
    q, r = divmod(layers, world)
    lo = rank * q + min(rank, r)
    hi = lo + q + (1 if rank < r else 0)
    return lo * t, min(hi * t, T)


def slab_cube(cube, T_slab: int) -> tuple[int, int, int]:
    """The cube to pass for a slab: only the last slab can hold fewer frames than the cube's
    depth, and its cubes are then the unsharded layer's ragged last layer, T_slab frames deep."""
    t, h, w = cube
    return (min(t, T_slab), h, w)


def forward_sharded(X_slab, T_slab: int, H: int, W: int, cube, Ci: int, Co: int, lowrank: int, packed_W, L1_mma,
                    L2_slab, Y_slab, workspace, allreduce_max, stream=None, stage_events=None,
                    start_event=None) -> None:
    """This process's slab of the layer.  X_slab / Y_slab: the slab's rows (device, BF16 bits),
    lowrank: the rank r of the low-rank factors L1, L2 (not the process's distributed rank),
    workspace: a uint8 device tensor of at least dq_workspace_bytes for the slab.  allreduce_max
    takes the slab's max |delta| as a one-element float32 tensor viewing the workspace and must
    leave the maximum over all ranks in it (e.g. torch.distributed.all_reduce(..., ReduceOp.MAX)
    on the stream's device).  stage_events (optional, 4 created CUDA events) time the encode
    stage and the two products as dq_linear_forward_ex does; start_event (optional) is recorded
    on the stream before the statistics pass."""
    import torch
    t, h, w = slab_cube(cube, T_slab)
    lay = dq.dq_workspace_layout_get(T_slab, H, W, t, h, w, Ci, Co, lowrank)
    nbytes = lay.total_bytes
    if workspace.numel() < nbytes:
        raise ValueError(f"workspace of {workspace.numel()} bytes, the slab needs {nbytes}")
    args = (X_slab, T_slab, H, W, t, h, w, Ci, Co, lowrank, packed_W, L1_mma, L2_slab, Y_slab, workspace, nbytes)
    if start_event is not None:
        start_event.record(stream)
    dq.dq_linear_forward_ex(*args, dq.DQ_STAGE_STATS, None, stream)
    amax = workspace[lay.off_scalars:lay.off_scalars + 4].view(torch.float32)
    allreduce_max(amax)
    dq.dq_linear_forward_ex(*args, dq.DQ_STAGE_ENCODE | dq.DQ_STAGE_KERNEL_GEMM | dq.DQ_STAGE_MAIN_GEMM,
                            stage_events, stream)
