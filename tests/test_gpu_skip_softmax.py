"""Skip-Softmax (threshold mode) through the C ABI against the oracle's
skip-aware reference: threshold 0 gives the dense kernel's bits; on inputs with
local, peaked attention the kernel output matches the oracle restricted to the
kept tiles, group by group, wherever the oracle's decisions are clear of the
threshold by a margin that rounding of fp32 scores cannot cross; the skip
counters equal what the oracle's decisions imply."""
import math

import numpy as np
import pytest
import torch

import oracle
import wan_inputs as wi
import video_diffusion_transformer_packed_b200 as wan
from video_diffusion_transformer_packed_b200 import build as wan_build
from helpers import assert_attention_close

pytestmark = pytest.mark.gpu
HD = 128
SCALE = 1.0 / math.sqrt(HD)
MARGIN = 1e-3  # log2 units; fp32 score rounding is far below this


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


def local_qkv(batch, S, heads, seed, alpha=0.6, reach=8):
    return wi.local_peaked_qkv(batch, S, heads, seed, alpha, reach)


def oracle_groups(qkv, heads, threshold):
    B, S, _ = qkv.shape
    groups = [(b, h, g) for b in range(B) for h in range(heads) for g in range((S + 31) // 32)]
    out, sk, margin = oracle.attention_skip_groups(qkv, heads, groups, SCALE, threshold)
    return groups, out, sk, margin


def expected_counts(groups, sk, S):
    """(group-tiles skipped, products skipped) implied by the oracle's decisions;
    a product is skipped when the four groups of a 128-row query tile all skip
    (groups wholly past S exist in the kernel and never skip)."""
    n_groups_per_bh = (S + 31) // 32
    group_tiles = int(sk.sum())
    products = 0
    per_bh = {}
    for (b, h, g), row in zip(groups, sk):
        per_bh.setdefault((b, h), {})[g] = row
    for rows in per_bh.values():
        for qt in range((S + 127) // 128):
            gs = [4 * qt + w for w in range(4)]
            if any(g >= n_groups_per_bh for g in gs):
                continue
            products += int(np.logical_and.reduce([rows[g] for g in gs]).sum())
    return group_tiles, products


def test_threshold_zero_is_the_dense_kernel():
    qkv = local_qkv(1, 700, 3, seed=1).cuda()
    dense = wan.self_attention(qkv, 3)
    sparse = wan.self_attention_sparse(qkv, 3, 0.0)
    torch.cuda.synchronize()
    assert torch.equal(dense.view(torch.int16), sparse.view(torch.int16))
    assert wan.skip_stats() == (0, 0)


@pytest.mark.parametrize("S,heads,batch,threshold", [
    (700, 2, 1, 0.02),
    (700, 2, 1, 0.2),
    (1000, 1, 2, 0.05),
    (640, 2, 1, 0.6),
    (321, 1, 1, 0.05),
    (512, 1, 1, 1.0),  # the largest threshold: every tile that does not raise the running max is skipped
])
def test_skip_softmax_matches_oracle(S, heads, batch, threshold):
    qkv = local_qkv(batch, S, heads, seed=S + heads)
    groups, ref, sk, margin = oracle_groups(qkv, heads, threshold)
    wan.skip_stats()  # clear
    out = wan.self_attention_sparse(qkv.cuda(), heads, threshold)
    got_tiles, got_products = wan.skip_stats()
    out = out.cpu().float().view(batch, S, heads, HD)
    clear = margin > MARGIN
    assert clear.mean() > 0.8, "too few decisions clear of the threshold to test"
    gots, refs = [], []
    for (b, h, g), o, ok in zip(groups, ref, clear):
        if not ok:
            continue
        n = min(32, S - 32 * g)
        gots.append(out[b, 32 * g:32 * g + n, h].numpy())
        refs.append(o[:n])
    assert_attention_close(torch.from_numpy(np.concatenate(gots)), np.concatenate(refs),
                           f"skip S={S} thr={threshold}")
    exp_tiles, exp_products = expected_counts(groups, sk, S)
    if clear.all():
        assert (got_tiles, got_products) == (exp_tiles, exp_products)
    else:
        n_unclear = int((~clear).sum()) * ((S + 127) // 128)
        assert abs(got_tiles - exp_tiles) <= n_unclear
    if threshold >= 0.05:
        assert exp_tiles > 0  # the case exercises skipping


def test_skipping_really_skips_products():
    """A long local sequence: key tiles past a query tile's diagonal neighbour
    are skipped by all four groups once the running max holds the peak (tiles
    before the peak cannot be: their running max is still low), so nearly all
    of those P V products are dropped; the counts equal the oracle's."""
    S, heads = 4096, 2
    qkv_h = local_qkv(1, S, heads, seed=3)
    qkv = qkv_h.cuda()
    wan.skip_stats()
    wan.self_attention_sparse(qkv, heads, 0.05)
    tiles, products = wan.skip_stats()
    n_t = S // 128
    after_diagonal = heads * sum(max(0, n_t - 1 - (qt + 1)) for qt in range(n_t))
    assert products > 0.9 * after_diagonal
    groups, _, sk, margin = oracle_groups(qkv_h, heads, 0.05)
    assert (margin > MARGIN).all()
    assert (tiles, products) == expected_counts(groups, sk, S)


def test_skip_softmax_full_size_sampled_groups():
    """The bench shape (2 x 32760 tokens, 40 heads) with local peaked inputs at
    threshold 0.05, in the bench's launch configuration: sampled 32-row groups
    (the first, the last -- ragged, so never skipping -- and random ones)
    against the oracle's skip-aware reference, where its decisions are clear."""
    import wan_inputs as wi_
    w = wi_.BY_NAME["a14b_480p_81f_cfg_b2"]
    qkv = local_qkv(w.batch, w.seq_len, w.heads, seed=5)
    wan.skip_stats()
    out = wan.self_attention_sparse(qkv.cuda(), w.heads, 0.05)
    tiles, products = wan.skip_stats()
    assert products > 0
    n_groups = (w.seq_len + 31) // 32
    g = torch.Generator().manual_seed(11)
    groups = [(0, 0, 0), (w.batch - 1, w.heads - 1, n_groups - 1)] + [
        (int(torch.randint(w.batch, (1,), generator=g)), int(torch.randint(w.heads, (1,), generator=g)),
         int(torch.randint(n_groups, (1,), generator=g))) for _ in range(4)]
    ref, sk, margin = oracle.attention_skip_groups(qkv, w.heads, groups, SCALE, 0.05)
    assert not sk[1].any()  # the ragged last group never skips
    assert sk[2:].any()      # random groups do skip
    oc = out.cpu().float().view(w.batch, w.seq_len, w.heads, HD)
    gots, refs = [], []
    for (b, h, gg), o, m in zip(groups, ref, margin):
        if m <= MARGIN:
            continue
        n = min(32, w.seq_len - 32 * gg)
        gots.append(oc[b, 32 * gg:32 * gg + n, h].numpy())
        refs.append(o[:n])
    assert len(gots) >= 4
    assert_attention_close(torch.from_numpy(np.concatenate(gots)), np.concatenate(refs), "skip full size")
