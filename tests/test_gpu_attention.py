"""GPU parity of wan_self_attention against the fp64 oracle:
max-abs error <= 2e-2 and relative Frobenius error <= 1e-2."""
import math

import numpy as np
import pytest
import torch

import oracle
import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import build as wan_build
from helpers import assert_attention_close

pytestmark = pytest.mark.gpu
HD = wi.HEAD_DIM
SCALE = 1.0 / math.sqrt(HD)


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


def gpu_attention(qkv, heads, scale=0.0):
    d = qkv.cuda()
    out = wan.self_attention(d, heads, scale=scale)
    assert wan.device_error() == 0
    torch.cuda.synchronize()
    assert torch.equal(d.cpu().view(torch.int16), qkv.view(torch.int16))  # input untouched
    return out.cpu()


@pytest.mark.parametrize("S", [1, 7, 64, 127, 128, 129, 255, 256, 257, 320, 383, 700])
def test_tails_and_small_sequences(S):
    heads = 2
    qkv = wi.packed_qkv(1, S, heads, seed=S)
    got = gpu_attention(qkv, heads)
    ref = oracle.attention_full(qkv, heads, SCALE)
    assert_attention_close(got.view(1, S, heads, HD), ref, f"S={S}")


def test_tiny_wan_grid_after_oracle_norm_rope():
    w = wi.WORKLOADS[0]
    qkv, gq, gk = wi.inputs_for(w, seed=0)
    normed = oracle.qk_norm_rope(qkv, w.grid, w.heads, gq, gk, wi.EPS, wi.THETA)
    got = gpu_attention(normed, w.heads)
    ref = oracle.attention_full(normed, w.heads, SCALE)
    assert_attention_close(got.view(1, w.seq_len, w.heads, HD), ref, "tiny")


def test_batches_do_not_leak():
    """Two batches with different content and magnitudes (batch 1: queries
    doubled, so its softmax is sharper, and values halved); rows past S in the
    last tile must read as zeros of the same batch, not the next batch's tokens."""
    S, heads = 200, 3
    D = heads * HD
    second = wi.packed_qkv(1, S, heads, seed=33).float()
    second[..., :D] *= 2.0
    second[..., 2 * D:] *= 0.5
    qkv = torch.cat([wi.packed_qkv(1, S, heads, seed=3), second.to(torch.bfloat16)])
    got = gpu_attention(qkv, heads)
    ref = oracle.attention_full(qkv, heads, SCALE)
    assert_attention_close(got.view(2, S, heads, HD), ref, "batch")


def test_peaked_logits_force_rescaling():
    """Query rows aligned with one late key: the running max jumps late,
    so O must be rescaled inside the tile loop."""
    S, heads = 600, 1
    qkv = wi.packed_qkv(1, S, heads, seed=4).float()
    qkv[0, :, :HD] = 4.0 * qkv[0, 550, HD:2 * HD]
    qkv = qkv.to(torch.bfloat16)
    got = gpu_attention(qkv, heads)
    ref = oracle.attention_full(qkv, heads, SCALE)
    assert_attention_close(got.view(1, S, heads, HD), ref, "peaked")


def test_large_scale_spread_logits():
    S, heads = 515, 2
    qkv = wi.packed_qkv(1, S, heads, seed=5)
    got = gpu_attention(qkv, heads, scale=0.5)
    ref = oracle.attention_full(qkv, heads, 0.5)
    assert_attention_close(got.view(1, S, heads, HD), ref, "scale 0.5")


def test_constant_v_gives_v():
    S, heads = 300, 2
    qkv = wi.packed_qkv(1, S, heads, seed=6).float()
    cst = torch.linspace(-2, 2, heads * HD)
    qkv[0, :, 2 * heads * HD:] = cst
    qkv = qkv.to(torch.bfloat16)
    got = gpu_attention(qkv, heads)
    exp = cst.to(torch.bfloat16).float().expand(S, -1)
    assert float((got[0].float() - exp).abs().max()) <= 2e-2


def test_head_count_extremes():
    for heads, S in ((1, 130), (64, 140)):
        qkv = wi.packed_qkv(1, S, heads, seed=heads)
        got = gpu_attention(qkv, heads)
        ref = oracle.attention_full(qkv, heads, SCALE)
        assert_attention_close(got.view(1, S, heads, HD), ref, f"heads={heads}")


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_full_size_workloads_sampled_rows(idx):
    """Full-size Wan workloads in the bench's launch configuration, checked on
    sampled query rows of sampled (batch, head) pairs, including the first
    row, the last row and the whole last (ragged) tile."""
    w = wi.WORKLOADS[idx]
    qkv, gq, gk = wi.inputs_for(w, seed=0)
    d = qkv.cuda()
    wan.qk_norm_rope(d, w.grid, w.heads, gq.cuda(), gk.cuda(), wi.EPS, wi.THETA)
    out = wan.self_attention(d, w.heads)
    assert wan.device_error() == 0
    normed = d.cpu()  # attention's input, as the GPU produced it (checked separately to 1 ulp)
    g = torch.Generator().manual_seed(idx)
    pairs = [(0, 0), (w.batch - 1, w.heads - 1)] + [
        (int(torch.randint(w.batch, (1,), generator=g)), int(torch.randint(w.heads, (1,), generator=g)))
        for _ in range(2)]
    rows = []
    for (b, h) in pairs:
        for i in wi.sample_rows(w.seq_len, 24, seed=b * 100 + h).tolist():
            rows.append((b, h, i))
    rows = np.array(rows, dtype=np.int64)
    ref = oracle.attention_rows(normed, w.heads, rows, SCALE)
    oc = out.view(w.batch, w.seq_len, w.heads, HD)
    got = oc[torch.from_numpy(rows[:, 0]).cuda(), torch.from_numpy(rows[:, 2]).cuda(),
             torch.from_numpy(rows[:, 1]).cuda()].cpu()
    assert_attention_close(got, ref, w.name)


# The 832x480, 81-frame token grid (21, 30, 52): S = 32760, 256 key tiles, the
# last one ragged (120 keys).
LONG_S = 32760


def _rows_of_head(S, idx):
    idx = np.asarray(idx, dtype=np.int64)
    return np.stack([np.zeros_like(idx), np.zeros_like(idx), idx], axis=1)


def test_full_length_late_peak_every_row():
    """Every query equals the key of a token in the last key tile, so each
    row's running max is set by N(0,1) logits for 255 tiles and jumps by about
    16 (log2 units) in the last one: the lazy rescale fires there, after the
    row sum has accumulated 32700 keys, and the peak and the bulk weigh about
    the same. All 32760 rows of the head against the oracle at the flat bound."""
    S, heads = LONG_S, 1
    qkv = wi.packed_qkv(1, S, heads, seed=41)
    t = torch.randint(S - 60, S, (S,), generator=torch.Generator().manual_seed(42))
    qkv[0, :, :HD] = qkv[0, t, HD:2 * HD]
    got = gpu_attention(qkv, heads)
    ref = oracle.attention_rows(qkv, heads, _rows_of_head(S, np.arange(S)), SCALE)
    assert_attention_close(got.view(S, HD), ref, "late peak, every row")


def test_full_length_rising_max_sampled_rows():
    """Keys scaled by 2^(4 j / S): each row's tile maxima grow from about 2.5
    to about 40 (natural-log units) along the 256 tiles, so the running max is
    raised, and O and the row sum rescaled, every few tiles through the whole
    loop, and the result is dominated by a few late keys whose weights reach
    the bf16 rounding of P at its largest. Sampled rows (always the first, the
    last and the ragged last tile) against the oracle at the flat bound."""
    S, heads = LONG_S, 1
    qkv = wi.packed_qkv(1, S, heads, seed=43)
    g = torch.exp2(4.0 * torch.arange(S, dtype=torch.float32) / S)
    qkv[0, :, HD:2 * HD] = (qkv[0, :, HD:2 * HD].float() * g[:, None]).to(torch.bfloat16)
    got = gpu_attention(qkv, heads)
    idx = wi.sample_rows(S, 4096, seed=44).numpy()
    ref = oracle.attention_rows(qkv, heads, _rows_of_head(S, idx), SCALE)
    assert_attention_close(got.view(S, HD)[torch.from_numpy(idx)], ref, "rising max, sampled rows")


def test_full_length_equal_scores_give_the_mean_of_v():
    """Q = 0: every score is 0 and every probability exactly 1, so each row's
    output is the mean of V over all 32760 keys, the ragged last tile
    included: the row sum counts 32760 ones and O sums 32760 rows of V in
    fp32. Sampled rows against the oracle at the flat bound, and every element
    against the closed form within the output's bf16 rounding."""
    S, heads = LONG_S, 1
    qkv = wi.packed_qkv(1, S, heads, seed=45)
    qkv[0, :, :HD] = 0
    got = gpu_attention(qkv, heads).view(S, HD).double()
    idx = wi.sample_rows(S, 256, seed=46).numpy()
    ref = oracle.attention_rows(qkv, heads, _rows_of_head(S, idx), SCALE)
    assert_attention_close(got[torch.from_numpy(idx)].float(), ref, "equal scores, sampled rows")
    mean = qkv[0, :, 2 * HD:3 * HD].double().mean(0)
    err = (got - mean).abs()
    assert bool((err <= 2.0 ** -8 * mean.abs() + 1e-7).all()), float(err.max())
