"""The CUDA side of sequence parallelism on one GPU: N ranks simulated in one
process, one after another (norm+RoPE of every shard, the gather as a
concatenation in rank order, attention of every rank's rows -- no kernel waits
on another), and the single-rank path through sp.cuda_ops; the outputs equal
the unsharded wan_dit_attn bit for bit."""
import pytest
import torch

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
