"""Pins of the oracle's ring-round attention (one key range's softmax state)
and of its merge, against what the mathematics fixes: the states of any split
of the keys merge, in any order, into the plain attention (itself pinned
against scaled_dot_product_attention); one key gives l = 1 and o = v; a pure
Python evaluation on a tiny case; a K|V chunk buffer reads like the packed
buffer; a state that carries no weight leaves the merge unchanged."""
import math

import numpy as np
import pytest
import torch

import oracle
import wan_inputs as wi

HD = 128
SCALE = 1 / math.sqrt(HD)


def _rows(B, heads, idx):
    return np.array([(b, h, i) for b in range(B) for i in idx for h in range(heads)], dtype=np.int64)


def _kv_chunk(qkv, heads):
    """The K|V columns of a packed buffer as their own [B, S, 2D] buffer."""
    D = heads * HD
    return qkv[..., D:].contiguous()


@pytest.mark.parametrize("split,order", [
    ((300,), None), ((128, 172), None), ((1, 299), (1, 0)), ((100, 100, 100), (2, 0, 1)),
    ((7, 93, 200), (1, 2, 0)), ((150, 150), (1, 0)),
])
def test_partials_of_any_split_merge_to_the_attention(split, order):
    B, S, heads = 2, 300, 2
    qkv = wi.packed_qkv(B, S, heads, seed=61)
    rows = _rows(B, heads, [0, 1, 127, 128, 200, 299])
    ref = oracle.attention_rows(qkv, heads, rows, SCALE)
    starts = np.cumsum((0,) + split[:-1])
    parts = [oracle.attention_partial_rows(qkv, heads, qkv, int(k0), int(n), rows, SCALE)
             for k0, n in zip(starts, split)]
    order = order or tuple(range(len(parts)))
    state = parts[order[0]]
    for i in order[1:]:
        state = oracle.merge_partial(state, parts[i])
    got = oracle.finalize_partial(state)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)
    # the merged maximum is the largest logit over all keys
    full_m = oracle.attention_partial_rows(qkv, heads, qkv, 0, S, rows, SCALE)[1][:, 0]
    assert np.array_equal(state[1][:, 0], full_m)


def test_one_key_gives_unit_weight_and_its_value():
    B, S, heads = 1, 40, 3
    qkv = wi.packed_qkv(B, S, heads, seed=62)
    D = heads * HD
    rows = _rows(B, heads, [0, 5, 39])
    o, ml = oracle.attention_partial_rows(qkv, heads, qkv, 17, 1, rows, SCALE)
    assert np.all(ml[:, 1] == 1.0)
    for r, (b, h, i) in enumerate(rows):
        v = qkv[b, 17, 2 * D + h * HD:2 * D + (h + 1) * HD].double().numpy()
        k = qkv[b, 17, D + h * HD:D + (h + 1) * HD].double().numpy()
        q = qkv[b, i, h * HD:(h + 1) * HD].double().numpy()
        assert np.array_equal(o[r], v)
        assert math.isclose(ml[r, 0], float(q @ k) * SCALE, rel_tol=1e-13)


def test_pure_python_brute_force_on_a_tiny_range():
    B, S, heads = 1, 9, 1
    qkv = wi.packed_qkv(B, S, heads, seed=63)
    t = qkv[0].double().tolist()
    i, k0, n, scale = 4, 2, 5, 0.3
    logits = [scale * sum(t[i][d] * t[j][HD + d] for d in range(HD)) for j in range(k0, k0 + n)]
    m = max(logits)
    w = [math.exp(a - m) for a in logits]
    o_ref = [sum(w[jj] * t[k0 + jj][2 * HD + d] for jj in range(n)) for d in range(HD)]
    o, ml = oracle.attention_partial_rows(qkv, heads, qkv, k0, n, [(0, 0, i)], scale)
    assert math.isclose(ml[0, 0], m, rel_tol=1e-13)
    assert math.isclose(ml[0, 1], sum(w), rel_tol=1e-13)
    assert np.allclose(o[0], o_ref, rtol=1e-12, atol=1e-13)


def test_a_kv_chunk_buffer_reads_like_the_packed_buffer():
    B, S, heads = 2, 260, 2
    qkv = wi.packed_qkv(B, S, heads, seed=64)
    rows = _rows(B, heads, [3, 259])
    a = oracle.attention_partial_rows(qkv, heads, qkv, 130, 120, rows, SCALE)
    b = oracle.attention_partial_rows(qkv, heads, _kv_chunk(qkv, heads), 130, 120, rows, SCALE)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    # and another buffer's keys really are read: a different chunk changes the state
    other = _kv_chunk(wi.packed_qkv(B, S, heads, seed=65), heads)
    c = oracle.attention_partial_rows(qkv, heads, other, 130, 120, rows, SCALE)
    assert not np.allclose(a[0], c[0])


def test_merge_with_a_weightless_state_is_the_identity_and_merge_commutes():
    B, S, heads = 1, 200, 2
    qkv = wi.packed_qkv(B, S, heads, seed=66)
    rows = _rows(B, heads, [0, 100, 199])
    a = oracle.attention_partial_rows(qkv, heads, qkv, 0, 90, rows, SCALE)
    b = oracle.attention_partial_rows(qkv, heads, qkv, 90, 110, rows, SCALE)
    far = (b[0], np.stack([b[1][:, 0] - 2000.0, b[1][:, 1]], axis=1))  # exp(-2000) = 0 in fp64
    same = oracle.merge_partial(a, far)
    assert np.array_equal(same[0], a[0]) and np.array_equal(same[1], a[1])
    ab, ba = oracle.merge_partial(a, b), oracle.merge_partial(b, a)
    assert np.allclose(ab[0], ba[0], rtol=1e-15, atol=0) and np.array_equal(ab[1][:, 0], ba[1][:, 0])
