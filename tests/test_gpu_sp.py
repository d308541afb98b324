"""The CUDA side of sequence parallelism on one GPU.

All-gather form: N ranks simulated in one process, one after another
(norm+RoPE of every shard, the gather as a concatenation in rank order,
attention of every rank's rows -- no kernel waits on another), and the
single-rank path through sp.cuda_ops; the outputs equal the unsharded
wan_dit_attn bit for bit, and a shard's rows match the oracle.

Ring form: every rank's rounds run one after another on one GPU, each
"remote" K|V chunk a local buffer of its own; the partial states and their
merge match the oracle at the attention bound."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import assert_attention_close

import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import build as wan_build
from video_diffusion_transformer_packed_b200 import sp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


@pytest.mark.parametrize("idx,world", [(0, 2), (0, 4), (1, 2), (1, 8), (4, 2)])
def test_simulated_ranks_equal_the_unsharded_step(idx, world):
    w = wi.WORKLOADS[idx]
    if w.seq_len % world:
        pytest.skip("sequence not divisible")
    qkv, gq, gk = wi.inputs_for(w, seed=idx + world)
    gq, gk = gq.cuda(), gk.cuda()
    ref_buf = qkv.cuda()
    ref = wan.dit_attn(ref_buf, w.grid, w.heads, gq, gk)
    s_local = w.seq_len // world
    shards = [qkv[:, r * s_local:(r + 1) * s_local].contiguous().cuda() for r in range(world)]
    for r, sh in enumerate(shards):
        wan.qk_norm_rope_shard(sh, w.grid, w.heads, r * s_local, gq, gk)
    full = torch.cat(shards, dim=1)
    assert torch.equal(full.view(torch.int16), ref_buf.view(torch.int16))
    outs = [wan.self_attention_rows(full, w.heads, r * s_local, s_local) for r in range(world)]
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    assert torch.equal(torch.cat(outs, dim=1).view(torch.int16), ref.view(torch.int16))


def test_single_rank_through_cuda_ops():
    w = wi.WORKLOADS[0]
    qkv, gq, gk = wi.inputs_for(w, seed=3)
    gq, gk = gq.cuda(), gk.cuda()
    ref = wan.dit_attn(qkv.cuda(), w.grid, w.heads, gq, gk)
    out = sp.sequence_parallel_step(qkv.cuda(), w.grid, 1, 0, sp.cuda_ops(w.grid, w.heads, gq, gk))
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_query_row_ranges_at_ragged_offsets():
    """Row ranges that start and end inside 128-row tiles."""
    w = wi.WORKLOADS[1]
    qkv, gq, gk = wi.inputs_for(w, seed=8)
    d = qkv.cuda()
    wan.qk_norm_rope(d, w.grid, w.heads, gq.cuda(), gk.cuda())
    ref = wan.self_attention(d, w.heads)
    for r0, n in [(0, 1), (77, 300), (7799, 1), (1000, 6800)]:
        got = wan.self_attention_rows(d, w.heads, r0, n)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), ref[:, r0:r0 + n].view(torch.int16))


def test_shards_starting_mid_row_with_many_batch_boundaries():
    """Shards of 525 tokens (3.5 rows of 150) over a batch of 40: every CTA's
    token range crosses batch boundaries, where the shard's grid positions
    restart at s0, and long column runs step the rotations one by one; the
    shards must reproduce the full-buffer norm+RoPE bit for bit."""
    grid, heads, batch, world = (2, 7, 150), 1, 40, 4
    S = grid[0] * grid[1] * grid[2]
    qkv = wi.packed_qkv(batch, S, heads, seed=31)
    gq, gk = wi.gammas(heads, 32, 33)
    gq, gk = gq.cuda(), gk.cuda()
    ref = qkv.cuda()
    wan.qk_norm_rope(ref, grid, heads, gq, gk)
    s_local = S // world
    shards = [qkv[:, r * s_local:(r + 1) * s_local].contiguous().cuda() for r in range(world)]
    for r, sh in enumerate(shards):
        wan.qk_norm_rope_shard(sh, grid, heads, r * s_local, gq, gk)
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    assert torch.equal(torch.cat(shards, dim=1).view(torch.int16), ref.view(torch.int16))


SCALE = 1 / math.sqrt(128)
LOG2E = 1.4426950408889634


def _normed(idx, seed):
    w = wi.WORKLOADS[idx]
    qkv, gq, gk = wi.inputs_for(w, seed=seed)
    d = qkv.cuda()
    wan.qk_norm_rope(d, w.grid, w.heads, gq.cuda(), gk.cuda())
    torch.cuda.synchronize()
    return w, d


def _sampled(w, out_rows, rows):
    """out_rows [B, n, D] (GPU) at (b, h, i) -> [len(rows), 128] on the CPU."""
    oc = out_rows.view(out_rows.shape[0], out_rows.shape[1], w.heads, 128)
    r = torch.from_numpy(rows).cuda()
    return oc[r[:, 0], r[:, 2], r[:, 1]].cpu()


def test_shard_rows_match_the_oracle():
    """wan_self_attention_rows for a rank's shard (rows [3900, 7800) of the
    5-frame 480p grid) against the oracle's attention of the same rows."""
    w, d = _normed(1, seed=21)
    r0, n = 3900, 3900
    out = wan.self_attention_rows(d, w.heads, r0, n)
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    local = wi.sample_rows(n, 24, seed=22).numpy()
    rows = np.array([(0, h, i) for h in (0, 17, 39) for i in local], dtype=np.int64)
    ref = oracle.attention_rows(d.cpu(), w.heads, rows + np.array([0, 0, r0]), SCALE)
    assert_attention_close(_sampled(w, out, rows), ref, "shard rows")


@pytest.mark.parametrize("k0,kn", [(0, 7800), (1000, 1), (129, 3000), (7799, 1), (3900, 3900)])
def test_partial_state_matches_the_oracle_state(k0, kn):
    """A key range of the packed buffer: the state's O / l is the attention of
    that range (flat bound against the oracle's), and its reference max lies
    within 8 below the range's largest scaled logit (base 2)."""
    w, d = _normed(1, seed=23)
    o, ml = wan.self_attention_partial(d, w.heads, d, k_row0=k0, k_rows=kn)
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    local = wi.sample_rows(w.seq_len, 16, seed=24).numpy()
    rows = np.array([(0, h, i) for h in (0, 39) for i in local], dtype=np.int64)
    ro, rml = oracle.attention_partial_rows(d.cpu(), w.heads, d.cpu(), k0, kn, rows, SCALE)
    r = torch.from_numpy(rows).cuda()
    go = o[r[:, 0], r[:, 2], r[:, 1]].double().cpu().numpy()
    gml = ml[r[:, 0], r[:, 2], r[:, 1]].double().cpu().numpy()
    got = torch.from_numpy(go / gml[:, 1:2])
    assert_attention_close(got, ro / rml[:, 1:2], f"partial [{k0}, {k0 + kn})")
    m_true = rml[:, 0] * LOG2E
    assert np.all(gml[:, 0] <= m_true + 1e-3) and np.all(gml[:, 0] >= m_true - 8.0 - 1e-3)


@pytest.mark.parametrize("idx,world", [(1, 2), (1, 4), (1, 8), (4, 2), (0, 4)])
def test_ring_rounds_simulated_on_one_gpu(idx, world):
    """Every rank's ring rounds, one after another: its own K|V chunk, then
    its left neighbours' in ring order, each chunk a separate [B, S/N, 2D]
    buffer; partial states merged round by round and finalised. The union of
    the ranks' outputs against the oracle on sampled rows of every rank, and
    against the unsharded kernel."""
    w, d = _normed(idx, seed=25 + world)
    S, D = w.seq_len, w.dim
    if S % world:
        pytest.skip("sequence not divisible")
    s_local = S // world
    shards = [d[:, r * s_local:(r + 1) * s_local].contiguous() for r in range(world)]
    chunks = [sh[..., D:].contiguous() for sh in shards]
    outs = []
    for r in range(world):
        state = None
        for c in sp.ring_order(world, r):
            part = wan.self_attention_partial(shards[r], w.heads, chunks[c])
            if state is None:
                state = part
            else:
                wan.attention_merge(state[0], state[1], part[0], part[1])
        outs.append(wan.attention_merge(state[0], state[1], finalize=True))
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    out = torch.cat(outs, dim=1)
    dense = wan.self_attention(d, w.heads)
    torch.cuda.synchronize()
    assert float((out.float() - dense.float()).abs().max()) <= 2e-2
    local = wi.sample_rows(s_local, 6, seed=26).numpy()
    idx_rows = np.concatenate([r * s_local + local for r in range(world)])
    rows = np.array([(b, h, i) for b in range(w.batch) for h in (0, w.heads - 1) for i in idx_rows],
                    dtype=np.int64)
    ref = oracle.attention_rows(d.cpu(), w.heads, rows, SCALE)
    assert_attention_close(_sampled(w, out, rows), ref, f"ring world {world}")


def test_ring_and_gather_forms_on_a_side_stream():
    """Both orchestrations at world size 1 with an explicit non-default
    stream: every kernel, copy and merge is ordered on that stream, so the
    results equal the unsharded step's."""
    w = wi.WORKLOADS[1]
    qkv, gq, gk = wi.inputs_for(w, seed=27)
    gq, gk = gq.cuda(), gk.cuda()
    ref = wan.dit_attn(qkv.cuda(), w.grid, w.heads, gq, gk)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    a = qkv.cuda()
    b = qkv.cuda()
    torch.cuda.synchronize()
    out_g = sp.sequence_parallel_step(a, w.grid, 1, 0, sp.cuda_ops(w.grid, w.heads, gq, gk, stream=side))
    out_r = sp.ring_attention_step(b, w.grid, 1, 0, sp.cuda_ring_ops(w.grid, w.heads, gq, gk, stream=side))
    side.synchronize()
    assert torch.equal(out_g.view(torch.int16), ref.view(torch.int16))
    assert float((out_r.float() - ref.float()).abs().max()) <= 2e-2
    rows = np.array([(0, h, i) for h in (0, 39) for i in wi.sample_rows(w.seq_len, 16, seed=28).tolist()],
                    dtype=np.int64)
    normed = oracle.qk_norm_rope(qkv, w.grid, w.heads, gq.cpu(), gk.cpu(), wi.EPS, wi.THETA)
    assert_attention_close(_sampled(w, out_r, rows), oracle.attention_rows(normed, w.heads, rows, SCALE), "ring")


def test_ring_rounds_at_the_bench_shape_sampled_rows():
    """The bench's ring side measurement, in its launch configuration: 8
    simulated ranks over the 832x480, 81-frame CFG batch (2 x 32760 tokens,
    40 heads), each rank's rounds over the 8 K|V chunks, partial states merged
    round by round. Sampled rows of every rank (its first and last rows and
    random ones) on the first and last heads of both batch elements, against
    the oracle at the attention bound."""
    w, d = _normed(2, seed=29)
    world, D = 8, w.dim
    s_local = w.seq_len // world
    shards = [d[:, r * s_local:(r + 1) * s_local].contiguous() for r in range(world)]
    chunks = [sh[..., D:].contiguous() for sh in shards]
    acc = (torch.empty((w.batch, s_local, w.heads, 128), dtype=torch.float32, device="cuda"),
           torch.empty((w.batch, s_local, w.heads, 2), dtype=torch.float32, device="cuda"))
    part = (torch.empty_like(acc[0]), torch.empty_like(acc[1]))
    outs = []
    for r in range(world):
        for i, c in enumerate(sp.ring_order(world, r)):
            dst = acc if i == 0 else part
            wan.self_attention_partial(shards[r], w.heads, chunks[c], o=dst[0], ml=dst[1])
            if i > 0:
                wan.attention_merge(acc[0], acc[1], part[0], part[1])
        outs.append(wan.attention_merge(acc[0], acc[1], finalize=True))
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    out = torch.cat(outs, dim=1)
    local = wi.sample_rows(s_local, 3, seed=30).numpy()
    idx_rows = np.concatenate([r * s_local + local for r in range(world)])
    rows = np.array([(b, h, i) for b in range(w.batch) for h in (0, w.heads - 1) for i in idx_rows], dtype=np.int64)
    ref = oracle.attention_rows(d.cpu(), w.heads, rows, SCALE)
    assert_attention_close(_sampled(w, out, rows), ref, "ring at the bench shape")


@pytest.mark.parametrize("idx,world", [(1, 4), (4, 2)])
def test_ring_rounds_accumulated_in_the_epilogue(idx, world):
    """The ring rounds with every round after the first merged into the
    running state by the attention's epilogue (wan_self_attention_accumulate),
    against the oracle on sampled rows of every rank, and against the same
    rounds merged by the separate merge kernel (same arithmetic, so the two
    agree to fp32 rounding)."""
    w, d = _normed(idx, seed=31 + world)
    S, D = w.seq_len, w.dim
    s_local = S // world
    shards = [d[:, r * s_local:(r + 1) * s_local].contiguous() for r in range(world)]
    chunks = [sh[..., D:].contiguous() for sh in shards]
    outs_acc, outs_merge = [], []
    for r in range(world):
        order = sp.ring_order(world, r)
        o, ml = wan.self_attention_partial(shards[r], w.heads, chunks[order[0]])
        o2, ml2 = o.clone(), ml.clone()
        for c in order[1:]:
            wan.self_attention_partial(shards[r], w.heads, chunks[c], o=o, ml=ml, accumulate=True)
            part = wan.self_attention_partial(shards[r], w.heads, chunks[c])
            wan.attention_merge(o2, ml2, part[0], part[1])
        outs_acc.append(wan.attention_merge(o, ml, finalize=True))
        outs_merge.append(wan.attention_merge(o2, ml2, finalize=True))
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    out = torch.cat(outs_acc, dim=1)
    assert float((out.float() - torch.cat(outs_merge, dim=1).float()).abs().max()) <= 1e-2
    local = wi.sample_rows(s_local, 6, seed=32).numpy()
    idx_rows = np.concatenate([r * s_local + local for r in range(world)])
    rows = np.array([(b, h, i) for b in range(w.batch) for h in (0, w.heads - 1) for i in idx_rows],
                    dtype=np.int64)
    ref = oracle.attention_rows(d.cpu(), w.heads, rows, SCALE)
    assert_attention_close(_sampled(w, out, rows), ref, f"accumulated ring world {world}")
