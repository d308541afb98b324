"""GPU parity of wan_qk_norm_rope against the fp64 oracle: every Q/K element
within 1 bf16 ulp, V untouched bit for bit."""
import pytest
import torch

import oracle
import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import build as wan_build
from helpers import bf16_ulp_distance

pytestmark = pytest.mark.gpu
EPS, THETA = wi.EPS, wi.THETA


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


def run_gpu(qkv, grid, heads, gq, gk):
    d = qkv.cuda()
    wan.qk_norm_rope(d, grid, heads, gq.cuda(), gk.cuda(), EPS, THETA)
    torch.cuda.synchronize()
    return d.cpu()


def check_full(qkv, grid, heads, gq, gk):
    got = run_gpu(qkv, grid, heads, gq, gk)
    ref = oracle.qk_norm_rope(qkv, grid, heads, gq, gk, EPS, THETA)
    D = heads * wi.HEAD_DIM
    dist = bf16_ulp_distance(got[..., :2 * D], ref[..., :2 * D])
    assert int(dist.max()) <= 1, f"max ulp distance {int(dist.max())}"
    assert torch.equal(got[..., 2 * D:].view(torch.int16), qkv[..., 2 * D:].view(torch.int16))
    return float((dist > 0).float().mean())


@pytest.mark.parametrize("batch,grid,heads", [
    (1, (5, 8, 8), 12),     # the tiny Wan grid
    (2, (1, 1, 1), 1),      # one token, one head
    (1, (3, 5, 7), 3),      # odd head count: a partial last vector group
    (2, (2, 3, 4), 40),     # A14B width
    (1, (4, 4, 4), 64),     # widest accepted hidden size
    (3, (1, 2, 3), 24),     # TI2V-5B width
    (1, (21, 2, 3), 5),     # many frames: large frame angles
])
def test_norm_rope_matches_oracle(batch, grid, heads):
    w = wi.Workload("t", batch, grid, heads)
    qkv, gq, gk = wi.inputs_for(w, seed=100 + heads)
    frac = check_full(qkv, grid, heads, gq, gk)
    assert frac < 0.02  # 1-ulp ties are rare


def test_full_width_reduction_with_head_magnitudes():
    """Heads carry magnitudes 2^(h%7-3): a per-head norm would be off by far more than 1 ulp."""
    grid, heads = (2, 3, 4), 12
    qkv = wi.head_magnitude_qkv(1, 24, heads, seed=7)
    gq, gk = wi.gammas(heads, 8, 9)
    check_full(qkv, grid, heads, gq, gk)


def test_gamma_indexed_per_channel_across_heads():
    """Distinct gammas per head: reusing head 0's weights would fail."""
    grid, heads = (2, 2, 2), 6
    w = wi.Workload("t", 1, grid, heads)
    qkv, _, _ = wi.inputs_for(w, seed=10)
    gq = torch.cat([torch.full((128,), 0.5 + 0.2 * h) for h in range(heads)]).to(torch.bfloat16)
    gk = torch.cat([torch.full((128,), 1.5 - 0.15 * h) for h in range(heads)]).to(torch.bfloat16)
    check_full(qkv, grid, heads, gq, gk)


def test_large_positions_on_720p_axes():
    """Positions up to (20, 44, 79): the largest angles of the 720p grid."""
    grid, heads = (21, 45, 80), 1
    S = 21 * 45 * 80
    qkv = wi.packed_qkv(1, S, heads, seed=12)
    gq, gk = wi.gammas(heads, 13, 14)
    check_full(qkv, grid, heads, gq, gk)


@pytest.mark.parametrize("batch,grid", [
    (1, (4, 60, 150)),   # columns past 64 and 128, rows past the token range of a CTA
    (2, (130, 2, 70)),   # frames past 128, a batch boundary inside CTAs' ranges
    (3, (5, 97, 31)),    # rows past 64, odd sizes
])
def test_rotation_carried_across_long_axes(batch, grid):
    """Tens of thousands of tokens at one head: every CTA walks many
    consecutive tokens, so the kernel's step-by-step rotation update, its
    fresh evaluation at wraps, jumps and every 64th position, and the batch
    boundary all run; every element is checked."""
    heads = 1
    w = wi.Workload("t", batch, grid, heads)
    qkv = wi.packed_qkv(batch, w.seq_len, heads, seed=sum(grid))
    gq, gk = wi.gammas(heads, 15, 16)
    check_full(qkv, grid, heads, gq, gk)


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_full_size_workloads_sampled_tokens(idx):
    w = wi.WORKLOADS[idx]
    qkv, gq, gk = wi.inputs_for(w, seed=0)
    d = qkv.cuda()
    wan.qk_norm_rope(d, w.grid, w.heads, gq.cuda(), gk.cuda(), EPS, THETA)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(idx)
    S = w.seq_len
    toks = [(0, 0), (w.batch - 1, S - 1)] + [
        (int(torch.randint(w.batch, (1,), generator=g)), int(torch.randint(S, (1,), generator=g)))
        for _ in range(254)]
    ref = oracle.qk_norm_rope_tokens(qkv, w.grid, w.heads, gq, gk, EPS, THETA, toks)
    D = w.dim
    b_idx = torch.tensor([t[0] for t in toks])
    s_idx = torch.tensor([t[1] for t in toks])
    got = d[b_idx.cuda(), s_idx.cuda()].cpu()
    assert int(bf16_ulp_distance(got[:, :2 * D], ref).max()) <= 1
    assert torch.equal(got[:, 2 * D:].view(torch.int16), qkv[b_idx, s_idx, 2 * D:].view(torch.int16))
