"""The sequence-parallel orchestration (video_diffusion_transformer_packed_b200.sp)
over a CPU process group (gloo), driven by the oracle's steps.

All-gather form (world 2): each rank norms its shard with global RoPE
positions, the shards are gathered in rank order, each rank attends its query
rows, and the union of the ranks' outputs equals the unsharded oracle's
exactly. Ring form (worlds 2 and 3): the K|V chunks travel to the right
neighbour by point-to-point messages, each rank meets them in ring order, the
rounds' softmax states merge, and the union of the outputs equals the
unsharded oracle up to fp64 rounding. The CUDA kernels behind the same
orchestration are checked on one GPU by tests/test_gpu_sp.py."""
import datetime
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import sp

GRID, HEADS, BATCH = (2, 4, 6), 2, 2  # S = 48


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    w = wi.Workload("sp", BATCH, GRID, HEADS)
    return w, *wi.inputs_for(w, seed=5)


def _oracle_ops(full_in, gq, gk):
    D = HEADS * 128
    scale = 1 / math.sqrt(128)

    def norm_shard(qkv_local, s0):
        B, s_local, _ = qkv_local.shape
        tokens = [(b, s0 + i) for b in range(B) for i in range(s_local)]
        rows = oracle.qk_norm_rope_tokens(full_in, GRID, HEADS, gq, gk, wi.EPS, wi.THETA, tokens)
        qkv_local[..., :2 * D] = rows.view(B, s_local, 2 * D)

    def gather(qkv_local):
        world = dist.get_world_size()
        parts = [torch.empty_like(qkv_local) for _ in range(world)]
        dist.all_gather(parts, qkv_local.contiguous())
        return torch.cat(parts, dim=1)

    def attend_rows(full, q_row0, q_rows):
        rows = [(b, h, q_row0 + i) for b in range(BATCH) for i in range(q_rows) for h in range(HEADS)]
        out = oracle.attention_rows(full, HEADS, rows, scale)
        return torch.from_numpy(out).view(BATCH, q_rows, HEADS * 128)

    return sp.SpOps(norm_shard, gather, attend_rows)


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        w, qkv, gq, gk = _inputs()
        s0, s_local = sp.shard_bounds(w.seq_len, world, rank)
        local = qkv[:, s0:s0 + s_local].clone()
        out = sp.sequence_parallel_step(local, GRID, world, rank, _oracle_ops(qkv, gq, gk))
        dist.barrier()
        results[rank] = (s0, out.numpy())
    finally:
        dist.destroy_process_group()


def test_sequence_parallel_orchestration_gloo_world2():
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    w, qkv, gq, gk = _inputs()
    normed = oracle.qk_norm_rope(qkv, GRID, HEADS, gq, gk, wi.EPS, wi.THETA)
    ref = oracle.attention_full(normed, HEADS, 1 / math.sqrt(128)).reshape(BATCH, w.seq_len, HEADS * 128)
    got = np.concatenate([results[r][1] for r in range(2)], axis=1)
    assert [results[r][0] for r in range(2)] == [0, w.seq_len // 2]
    assert np.array_equal(got, ref)


def _oracle_ring_ops(full_in, gq, gk, seen):
    D = HEADS * 128
    scale = 1 / math.sqrt(128)
    norm_shard = _oracle_ops(full_in, gq, gk).norm_shard

    def kv_chunk(qkv_local):
        return qkv_local[..., D:].clone()

    def exchange(kv):
        world, rank = dist.get_world_size(), dist.get_rank()
        buf = torch.empty_like(kv)
        reqs = [dist.isend(kv.contiguous(), (rank + 1) % world), dist.irecv(buf, (rank - 1) % world)]
        return reqs, buf

    def received(handle):
        reqs, buf = handle
        for r in reqs:
            r.wait()
        return buf

    def attend(qkv_local, kv, state):
        B, s_local, _ = qkv_local.shape
        seen.append(kv[0, 0, 0].item())  # which chunk this round met (its first K value)
        rows = [(b, h, i) for b in range(B) for i in range(s_local) for h in range(HEADS)]
        part = oracle.attention_partial_rows(qkv_local, HEADS, kv, 0, kv.shape[1], rows, scale)
        return part if state is None else oracle.merge_partial(state, part)

    def finalize(state):
        return torch.from_numpy(oracle.finalize_partial(state)).view(BATCH, -1, HEADS * 128)

    return sp.RingOps(norm_shard, kv_chunk, exchange, received, attend, finalize)


def _ring_worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        w, qkv, gq, gk = _inputs()
        s0, s_local = sp.shard_bounds(w.seq_len, world, rank)
        local = qkv[:, s0:s0 + s_local].clone()
        seen = []
        out = sp.ring_attention_step(local, GRID, world, rank, _oracle_ring_ops(qkv, gq, gk, seen))
        dist.barrier()
        results[rank] = (s0, out.numpy(), seen)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_attention_schedule_gloo(world):
    ctx = mp.get_context("spawn")
    results = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_ring_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    w, qkv, gq, gk = _inputs()
    normed = oracle.qk_norm_rope(qkv, GRID, HEADS, gq, gk, wi.EPS, wi.THETA)
    ref = oracle.attention_full(normed, HEADS, 1 / math.sqrt(128)).reshape(BATCH, w.seq_len, HEADS * 128)
    s_local = w.seq_len // world
    got = np.concatenate([results[r][1] for r in range(world)], axis=1)
    assert [results[r][0] for r in range(world)] == [r * s_local for r in range(world)]
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)
    # every rank met every chunk once, in ring order (its own first, then its left neighbours')
    D = HEADS * 128
    first_k = [float(normed[0, r * s_local, D].float()) for r in range(world)]
    for r in range(world):
        assert results[r][2] == [first_k[c] for c in sp.ring_order(world, r)]


def test_ring_order():
    assert sp.ring_order(4, 1) == [1, 0, 3, 2]
    assert sp.ring_order(1, 0) == [0]
    assert all(sorted(sp.ring_order(8, r)) == list(range(8)) for r in range(8))


def test_shard_bounds():
    assert sp.shard_bounds(32760, 8, 3) == (3 * 4095, 4095)
    with pytest.raises(ValueError, match="not divisible"):
        sp.shard_bounds(32760, 16, 0)
    with pytest.raises(ValueError):
        sp.shard_bounds(48, 2, 2)
