"""Sequence-parallel DiT self-attention step (context parallelism over N ranks).

The Neuron page ("Context parallelism") shards the token sequence S over the
ranks: each rank owns S/N tokens of Q, K and V, and its queries must still
attend every key; S must be divisible by the degree. Two forms of a rank's
share are here.

All-gather form (`sequence_parallel_step`), the page's fallback:
1. norm+RoPE of the local shard (per token, so purely local; RoPE positions
   from the global grid index of each token);
2. an all-gather of the normalised shards into the full packed buffer, one
   collective per batch element (a batch element's tokens are contiguous);
3. attention of the local query rows against every key.

Ring form (`ring_attention_step`), the page's ring attention: after step 1,
the K|V columns of the shard travel around the ring, one neighbour exchange
per round, and each round's attention of the local queries against the chunk
in hand runs while the next chunk is in flight. A round folds the softmax
state of its key range into the rank's running state (the first round
writes it, wan_self_attention_partial; later rounds merge in the attention's
epilogue, wan_self_attention_accumulate), and the final state is normalised
(wan_attention_merge). No rank ever holds the full K/V. A chunk is 2/3 of
the bytes the all-gather moves per token (no Q).

Compute is only ever the CUDA kernels of this package (`cuda_ops`,
`cuda_ring_ops`); the exchanges are torch.distributed collectives or
point-to-point messages (NCCL over NVLink on B200s), ordered on the caller's
stream. The ops are passed in so that the same orchestration can be driven by
other implementations of the steps (the tests drive both forms with the oracle
over a CPU process group to check the sharding and the ring schedule).
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


def _on_stream(stream):
    """Context in which torch's current stream is `stream` (when given), so
    that the package's kernels (launched on the current stream) and
    torch.distributed's collectives (ordered against the current stream) share
    one order."""
    import contextlib

    import torch
    return torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()


def cuda_ops(grid: Sequence[int], heads: int, gamma_q, gamma_k, group=None, stream=None) -> SpOps:
    """The package's kernels, with an NCCL all-gather per batch element
    (torch.distributed over `group`; a single-rank world gathers by copy).
    Every step runs on `stream` (default: the current stream)."""
    import torch
    import torch.distributed as dist

    import video_diffusion_transformer_packed_b200 as wan

    def norm_shard(qkv_local, s0):
        with _on_stream(stream):
            wan.qk_norm_rope_shard(qkv_local, grid, heads, s0, gamma_q, gamma_k)

    def gather(qkv_local):
        with _on_stream(stream):
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
        with _on_stream(stream):
            return wan.self_attention_rows(full, heads, q_row0, q_rows)

    return SpOps(norm_shard, gather, attend_rows)


@dataclass
class RingOps:
    """The steps of a rank's share in ring form.

    norm_shard(qkv_local, s0) -> None   norm+RoPE in place; tokens start at s0
    kv_chunk(qkv_local) -> kv          the shard's K|V, the part that travels
    exchange(kv) -> handle             start sending kv to rank + 1 and
                                       receiving the next chunk from rank - 1
    received(handle) -> kv             the received chunk, once it is in
    attend(qkv_local, kv, state) -> state
                                       the softmax state of the local queries
                                       against the keys of kv, folded into
                                       `state` (None in the first round)
    finalize(state) -> out             [B, s_local, heads*128]
    """
    norm_shard: Callable
    kv_chunk: Callable
    exchange: Callable
    received: Callable
    attend: Callable
    finalize: Callable


def ring_order(world: int, rank: int):
    """Owners of the chunks `rank` holds in rounds 0 .. world-1: its own, then
    each left neighbour's in turn (every exchange passes chunks to the right)."""
    return [(rank - i) % world for i in range(world)]


def ring_attention_step(qkv_local, grid: Sequence[int], world: int, rank: int, ops: RingOps):
    """One rank's share in ring form: norm its shard in place, then `world`
    rounds of (start the next exchange, fold the chunk in hand into the state)."""
    F, H, W = grid
    s0, s_local = shard_bounds(F * H * W, world, rank)
    if qkv_local.shape[1] != s_local:
        raise ValueError(f"rank {rank} holds {qkv_local.shape[1]} tokens, expected {s_local}")
    ops.norm_shard(qkv_local, s0)
    kv = ops.kv_chunk(qkv_local)
    state = None
    for i in range(world):
        handle = ops.exchange(kv) if i + 1 < world else None  # in flight during this round's attention
        state = ops.attend(qkv_local, kv, state)
        if handle is not None:
            kv = ops.received(handle)
    return ops.finalize(state)


def cuda_ring_ops(grid: Sequence[int], heads: int, gamma_q, gamma_k, group=None, stream=None) -> RingOps:
    """The package's kernels in ring form: the round's attention merged into
    the running state in its epilogue, on `stream` (default: the current
    stream), K|V chunks exchanged with
    the ring neighbours by NCCL point-to-point messages. The messages are
    enqueued before the round's attention and are ordered after the work
    already on the stream (the chunk being sent is complete); the next round's
    attention waits for the received chunk. Plain device buffers only: no
    peer-memory loads."""
    import torch
    import torch.distributed as dist

    import video_diffusion_transformer_packed_b200 as wan

    D = heads * 128

    def world_rank():
        if dist.is_available() and dist.is_initialized():
            return dist.get_world_size(group), dist.get_rank(group)
        return 1, 0

    def norm_shard(qkv_local, s0):
        with _on_stream(stream):
            wan.qk_norm_rope_shard(qkv_local, grid, heads, s0, gamma_q, gamma_k)

    def kv_chunk(qkv_local):
        with _on_stream(stream):
            return qkv_local[..., D:].contiguous()

    def exchange(kv):
        world, rank = world_rank()
        with _on_stream(stream):
            buf = torch.empty_like(kv)
            peers = [dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world,
                     dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world]
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, kv, peers[0], group),
                                           dist.P2POp(dist.irecv, buf, peers[1], group)])
            return reqs, buf

    def received(handle):
        reqs, buf = handle
        with _on_stream(stream):
            for r in reqs:
                r.wait()
        return buf

    def attend(qkv_local, kv, state):
        with _on_stream(stream):
            if state is None:
                return wan.self_attention_partial(qkv_local, heads, kv)
            return wan.self_attention_partial(qkv_local, heads, kv, o=state[0], ml=state[1], accumulate=True)

    def finalize(state):
        with _on_stream(stream):
            return wan.attention_merge(state[0], state[1], finalize=True)

    return RingOps(norm_shard, kv_chunk, exchange, received, attend, finalize)
