"""Pins of the oracle's Skip-Softmax (threshold mode) reference against things
other than itself: a closed-form case whose decision flips exactly at
threshold = exp(-q.k) and whose outputs are known in closed form on both sides,
the dense definition at threshold 0, monotonicity of the skipped set in the
threshold, invariance under permuting keys inside a tile, and the rule that a
group holding rows past S never skips."""
import math

import numpy as np
import pytest
import torch

import oracle

HD = 128


def _closed_form_qkv(S=384):
    """Group 0 queries q = (2, 0, ...), key 0 = (2, 0, ...), every other key 0:
    row scores (scale 1) are 4 at key 0 and 0 elsewhere. V: key 0 -> e0, the
    other keys of tile 0 -> e1, keys of later tiles -> e2. Group 1 queries are 0."""
    qkv = torch.zeros(1, S, 3 * HD, dtype=torch.bfloat16)
    qkv[0, :32, 0] = 2.0
    qkv[0, 0, HD + 0] = 2.0
    qkv[0, 0, 2 * HD + 0] = 1.0
    qkv[0, 1:128, 2 * HD + 1] = 1.0
    qkv[0, 128:, 2 * HD + 2] = 1.0
    return qkv


def test_closed_form_decision_and_outputs():
    S = 384
    qkv = _closed_form_qkv(S)
    e4 = math.exp(4.0)
    # threshold just above exp(-4): tiles 1 and 2 are skipped for group 0
    out, sk, margin = oracle.attention_skip_groups(qkv, 1, [(0, 0, 0)], 1.0, 0.0190)
    assert sk[0].tolist() == [False, True, True]
    exp_skip = np.zeros(HD)
    exp_skip[0], exp_skip[1] = e4 / (e4 + 127), 127 / (e4 + 127)
    np.testing.assert_allclose(out[0], np.broadcast_to(exp_skip, (32, HD)), rtol=0, atol=1e-14)
    assert abs(margin[0] - abs(-4 * math.log2(math.e) - math.log2(0.0190))) < 1e-12
    # threshold just below: dense
    out, sk, _ = oracle.attention_skip_groups(qkv, 1, [(0, 0, 0)], 1.0, 0.0180)
    assert not sk.any()
    exp_dense = np.zeros(HD)
    exp_dense[0], exp_dense[1], exp_dense[2] = e4 / (e4 + 383), 127 / (e4 + 383), 256 / (e4 + 383)
    np.testing.assert_allclose(out[0], np.broadcast_to(exp_dense, (32, HD)), rtol=0, atol=1e-14)
    # group 1 has zero queries: all scores 0, tile maxima equal the running max,
    # so it skips only once the threshold exceeds 1
    _, sk, _ = oracle.attention_skip_groups(qkv, 1, [(0, 0, 1)], 1.0, 0.99)
    assert not sk.any()
    out, sk, _ = oracle.attention_skip_groups(qkv, 1, [(0, 0, 1)], 1.0, 1.01)
    assert sk[0].tolist() == [False, True, True]
    np.testing.assert_allclose(out[0][:, 1], 127 / 128, atol=1e-14)  # tile 0 only: uniform over 128 keys
    np.testing.assert_allclose(out[0][:, 0], 1 / 128, atol=1e-14)


def _random_qkv(S, heads, seed, peak=0.0):
    g = torch.Generator().manual_seed(seed)
    qkv = torch.randn(1, S, 3 * heads * HD, generator=g)
    if peak:
        # give each query a copy of one key so that some rows are peaked
        for h in range(heads):
            src = torch.randint(0, S, (S,), generator=g)
            qkv[0, :, h * HD:(h + 1) * HD] = peak * qkv[0, src, heads * HD + h * HD:heads * HD + (h + 1) * HD]
    return qkv.to(torch.bfloat16)


def test_threshold_zero_is_dense():
    S, heads = 700, 2
    qkv = _random_qkv(S, heads, seed=5)
    groups = [(0, h, g) for h in range(heads) for g in range((S + 31) // 32)]
    out, sk, margin = oracle.attention_skip_groups(qkv, heads, groups, 1 / math.sqrt(HD), 0.0)
    assert not sk.any() and np.isinf(margin).all()
    rows = [(0, h, 32 * g + i) for (_, h, g) in groups for i in range(32) if 32 * g + i < S]
    dense = oracle.attention_rows(qkv, heads, rows, 1 / math.sqrt(HD))
    got = out.reshape(-1, HD)[~np.isnan(out.reshape(-1, HD)[:, 0])]
    np.testing.assert_allclose(got, dense, rtol=0, atol=1e-13)


def test_skipped_set_grows_with_threshold():
    S, heads = 900, 1
    qkv = _random_qkv(S, heads, seed=6, peak=0.35)
    groups = [(0, 0, g) for g in range((S + 31) // 32)]
    prev = None
    counts = []
    for thr in (0.0, 0.01, 0.05, 0.2, 0.5, 0.9):
        _, sk, _ = oracle.attention_skip_groups(qkv, heads, groups, 1 / math.sqrt(HD), thr)
        if prev is not None:
            assert (sk >= prev).all()  # a tile skipped at a lower threshold stays skipped
        prev = sk
        counts.append(int(sk.sum()))
    assert counts[0] == 0 and counts[-1] > counts[1]


def test_permuting_keys_inside_a_tile_changes_nothing():
    S, heads = 512, 1
    qkv = _random_qkv(S, heads, seed=7, peak=0.3)
    perm = torch.arange(S)
    g = torch.Generator().manual_seed(8)
    for t in range(S // 128):
        perm[128 * t:128 * (t + 1)] = 128 * t + torch.randperm(128, generator=g)
    shuffled = qkv.clone()
    shuffled[0, :, HD:] = qkv[0, perm, HD:]  # K and V rows move together; Q stays
    groups = [(0, 0, gg) for gg in range(S // 32)]
    a = oracle.attention_skip_groups(qkv, heads, groups, 1 / math.sqrt(HD), 0.1)
    b = oracle.attention_skip_groups(shuffled, heads, groups, 1 / math.sqrt(HD), 0.1)
    assert (a[1] == b[1]).all()
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-13)


@pytest.mark.parametrize("S", [300, 321])
def test_group_with_padding_rows_never_skips(S):
    qkv = _random_qkv(S, 1, seed=9, peak=0.5)
    last = (S - 1) // 32
    _, sk, _ = oracle.attention_skip_groups(qkv, 1, [(0, 0, last)], 1 / math.sqrt(HD), 0.9)
    assert (not sk.any()) == (S % 32 != 0)
