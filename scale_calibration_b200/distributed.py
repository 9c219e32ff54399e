"""Token-sharded Local-Hessian calibration over several GPUs (one process per GPU).

The local Hessian is a sum over the calibration tokens ("NVIDIA Model Optimizer
Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块权重缩放算法实战指南", section
"入口 API 与校准流程", Phase 2: H = sum X^T X), so each rank accumulates the
tokens it holds and one all-reduce (sum) gives every rank the layer's H. The
pages note that the Hessian is not synchronised across data-parallel ranks
there; this module is that synchronisation. The sweep then needs no exchange:
each rank sweeps its share of the blocks with the summed H (whole matrices of
an expert bank, else a range of block columns; see sweep_shard).

Plumbing only: the arithmetic runs in liblh.so (lh_accumulate_hessian,
lh_sweep_scales, lh_fake_quant); torch.distributed (NCCL between GPUs) carries
the all-reduce of H, J KB per matrix (about 1 MB per dense layer).
"""
from __future__ import annotations

import numpy as np


def token_shard(n_tok: int, rank: int, world: int, offsets=None):
    """This rank's contiguous share [t0, t1) of the n_tok tokens and, for grouped
    tokens (offsets [G+1], non-decreasing), the group offsets of that share
    relative to t0 (groups cut at the share's ends; groups outside it are empty)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} out of range for world size {world}")
    t0 = n_tok * rank // world
    t1 = n_tok * (rank + 1) // world
    if offsets is None:
        return t0, t1, None
    off = np.asarray(offsets, np.int64)
    local = np.clip(off, t0, t1) - t0
    return t0, t1, local


def row_shard(c_out: int, rank: int, world: int):
    """This rank's contiguous share [r0, r1) of the c_out rows for the sweep."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} out of range for world size {world}")
    return c_out * rank // world, c_out * (rank + 1) // world


def sweep_shard(n_mats: int, c_out: int, J: int, rank: int, world: int):
    """This rank's share of the sweep and fake-quant, as (kind, lo, hi):
    ("mats", m0, m1): whole matrices [m0, m1) when there are at least as many
    matrices as ranks (an expert bank: W, H and the global amax of a share are
    contiguous, and each matrix's amax needs no exchange); ("cols", j0, j1): the
    block columns [j0, j1) of every row of a single matrix (H + j0 blocks is
    contiguous, and each rank keeps whole row tiles); ("rows", r0, r1) otherwise.
    Every rank gets a share of about the same number of blocks; a share may be
    empty when there are fewer units than ranks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} out of range for world size {world}")
    if n_mats >= world:
        return "mats", n_mats * rank // world, n_mats * (rank + 1) // world
    if n_mats == 1:
        return "cols", J * rank // world, J * (rank + 1) // world
    return ("rows",) + row_shard(c_out, rank, world)


def allreduce_hessian(H, group=None):
    """Sum the ranks' partial Hessians in place (every rank gets the total)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)
    return H


def sharded_sum(H, add_local, group=None):
    """H += the contributions of every rank: ranks other than the group's first
    start from zero, each adds its own part with add_local(H), then the
    all-reduce. H must hold the same values on every rank on entry (zeros, or the
    result of an earlier call), so the entry value is counted once."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_rank(group) != 0:
        H.zero_()
    add_local(H)
    return allreduce_hessian(H, group)


def accumulate_hessian_sharded(X_local, n_tok_local: int, c_in: int, offsets_local, n_groups: int, H, workspace,
                               workspace_bytes: int, stream=None, group=None, check_status: bool = True):
    """H += the tokens of every rank (see sharded_sum): this rank adds its own
    tokens with lh_accumulate_hessian. X_local: bf16 [n_tok_local, ld] on this
    rank's GPU; offsets_local: device int64 [n_groups + 1] (this rank's share, see
    token_shard) or None; H: f32 [n_groups, c_in/16, 16, 16]. The all-reduce is
    ordered after the kernels on torch's current stream, which `stream` (None: the
    default stream) must be; check_status=False skips the status read (and its
    synchronisation), to be done later with lh_workspace_status."""
    from ._binding import LH_BF16, LHError, lh_accumulate_hessian, lh_last_error_message, lh_workspace_status

    def add_local(Hl):
        lh_accumulate_hessian(X_local, LH_BF16, n_tok_local, c_in, X_local.stride(0), offsets_local, n_groups, Hl,
                              workspace, workspace_bytes, stream)
        if check_status:
            status = lh_workspace_status(workspace, stream)
            if status != 0:
                raise LHError(status, "lh_accumulate_hessian", lh_last_error_message())

    return sharded_sum(H, add_local, group)
