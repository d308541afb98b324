"""Sequence-parallel DiT self-attention step (context parallelism over N ranks).

The Neuron page ("Context parallelism") shards the token sequence S over the
ranks: each rank owns S/N tokens of Q, K and V, and its queries must still
attend every key; S must be divisible by the degree. The step here, per rank:

1. norm+RoPE of the local shard (per token, so purely local; RoPE positions
   from the global grid index of each token);
2. an all-gather of the normalised shards into the full packed buffer, one
   collective per batch element (a batch element's tokens are contiguous);
3. attention of the local query rows against every key.

The exchange is an all-gather through the collective library (NCCL over
NVLink on B200s), the plain form the page describes for where its ring kernel
does not run; the output of every rank equals the unsharded step's rows.
Compute is only ever the CUDA kernels of this package (`cuda_ops`); the ops
are passed in so that the same orchestration can be driven by other
implementations of the three steps (the tests drive it with the oracle over a
CPU process group to check the sharding itself).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Sequence


@dataclass
class SpOps:
    """The three steps of a rank's share of the path.

    norm_shard(qkv_local, s0) -> None        norm+RoPE in place; tokens start at s0
    gather(qkv_local) -> full               [B, S, 3D], ranks' shards in rank order
    attend_rows(full, q_row0, q_rows) -> out [B, q_rows, D]
    """
    norm_shard: Callable
    gather: Callable
    attend_rows: Callable


def shard_bounds(seq_len: int, world: int, rank: int):
    """(s0, s_local) of `rank`; S must divide evenly (as the page requires)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if seq_len % world != 0:
        raise ValueError(f"Sequence length {seq_len} is not divisible by the sequence-parallel degree {world}")
    s_local = seq_len // world
    return rank * s_local, s_local


def sequence_parallel_step(qkv_local, grid: Sequence[int], world: int, rank: int, ops: SpOps):
    """One rank's share: norm its shard in place, gather, attend its rows."""
    F, H, W = grid
    s0, s_local = shard_bounds(F * H * W, world, rank)
    if qkv_local.shape[1] != s_local:
        raise ValueError(f"rank {rank} holds {qkv_local.shape[1]} tokens, expected {s_local}")
    ops.norm_shard(qkv_local, s0)
    full = ops.gather(qkv_local)
    return ops.attend_rows(full, s0, s_local)


def cuda_ops(grid: Sequence[int], heads: int, gamma_q, gamma_k, group=None, stream=None) -> SpOps:
    """The package's kernels, with an NCCL all-gather per batch element
    (torch.distributed over `group`; a single-rank world gathers by copy)."""
    import torch
    import torch.distributed as dist

    import video_diffusion_transformer_packed_b200 as wan

    def norm_shard(qkv_local, s0):
        wan.qk_norm_rope_shard(qkv_local, grid, heads, s0, gamma_q, gamma_k, stream=stream)

    def gather(qkv_local):
        B, s_local, d3 = qkv_local.shape
        world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
        full = torch.empty((B, s_local * world, d3), dtype=qkv_local.dtype, device=qkv_local.device)
        for b in range(B):
            if world == 1:
                full[b].copy_(qkv_local[b])
            else:
                dist.all_gather_into_tensor(full[b], qkv_local[b].contiguous(), group=group)
        return full

    def attend_rows(full, q_row0, q_rows):
        return wan.self_attention_rows(full, heads, q_row0, q_rows, stream=stream)

    return SpOps(norm_shard, gather, attend_rows)
