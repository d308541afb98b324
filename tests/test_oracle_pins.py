"""Pins for the fp64 oracle: each test ties a step of the oracle to something
other than the oracle itself -- a library routine computing a special case,
a closed form, an invariant of the mathematics, or brute force.

Steps pinned (see oracle/wan_oracle.c):
  bf16 rounding          -> torch's float32->bf16 conversion (RNE) on float32 inputs
  RMSNorm over full D    -> torch.nn.functional.rms_norm in fp64; constant-row closed form;
                            unit-gamma mean square; scale invariance up to eps;
                            per-head-magnitude input separates full-width from per-head
  gamma indexing         -> per-head distinct gammas scale exactly their head
  rounding point         -> token 0 (zero angle) equals round(norm) bit for bit
  3D RoPE                -> numpy complex rotation; unit first frequency per axis;
                            axis isolation of the 44/42/42 split; norm preservation;
                            relative-position property; geometric frequency ladder
  attention              -> torch SDPA in fp64; rows sum to 1; constant V; S = 1;
                            key permutation; peaked logits; pure-Python brute force
"""
import cmath
import math

import numpy as np
import pytest
import torch

import oracle
import wan_inputs as wi

HD = 128
EPS = 1e-6
THETA = 1e4


def bf16(x):
    """fp64 -> bf16 with a single rounding (pinned by the first test below)."""
    return oracle.to_bf16(np.asarray(x, dtype=np.float64))


# ---------------------------------------------------------------- bf16 rounding
def test_round_bf16_matches_torch_on_float32_values():
    """On float32 inputs torch's RNE conversion rounds once, so the two must agree."""
    g = torch.Generator().manual_seed(0)
    x = torch.randn(20000, generator=g, dtype=torch.float32) * 3
    # exact ties: a bf16 value plus half an ulp, for both parities of the last bit
    base = torch.randn(2000, generator=g).to(torch.bfloat16).float()
    bits = base.view(torch.int32)
    ties = (bits + 0x8000).view(torch.float32)
    x = torch.cat([x, ties, -ties])
    ref = x.to(torch.bfloat16).double().numpy()
    got = np.array([oracle.round_bf16(float(v)) for v in x.double().numpy()])
    assert np.array_equal(ref, got)
    assert np.array_equal(oracle.to_bf16(x.double().numpy()).double().numpy(), ref)


# ---------------------------------------------------------------------- RMSNorm
def test_rmsnorm_matches_library_rms_norm_fp64():
    heads = 3
    x = wi.packed_qkv(1, 17, heads, seed=11)[0, :, : heads * HD]
    gq, _ = wi.gammas(heads, 4, 5)
    ref = torch.nn.functional.rms_norm(x.double(), (heads * HD,), weight=gq.double(), eps=EPS)
    got = oracle.rmsnorm(x, gq, EPS)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-13, atol=0)


def test_rmsnorm_constant_row_closed_form():
    # x_c = 0.5 everywhere: mean square 0.25, y = gamma * 0.5 / sqrt(0.25 + eps)
    heads = 2
    x = torch.full((1, heads * HD), 0.5).to(torch.bfloat16)
    g = torch.ones(heads * HD).to(torch.bfloat16)
    got = oracle.rmsnorm(x, g, EPS)
    assert np.allclose(got, 0.5 / math.sqrt(0.25 + 1e-6), rtol=1e-15, atol=0)
    # and eps matters at this precision (guards a dropped eps)
    assert abs(got[0, 0] - 1.0) > 1e-7


def test_rmsnorm_unit_gamma_gives_unit_mean_square():
    """With gamma = 1, mean(y^2) = ms / (ms + eps) exactly in real arithmetic:
    1 up to eps / ms (a dropped mean, a sum instead of the mean, or a missing
    square root all break it)."""
    heads = 4
    x = wi.packed_qkv(1, 9, heads, seed=21)[0, :, : heads * HD]
    g = torch.ones(heads * HD).to(torch.bfloat16)
    y = oracle.rmsnorm(x, g, EPS)
    ms = (x.double().numpy() ** 2).mean(axis=1)
    np.testing.assert_allclose((y ** 2).mean(axis=1), ms / (ms + EPS), rtol=1e-13, atol=0)
    assert np.all(np.abs((y ** 2).mean(axis=1) - 1.0) < 2e-6)


def test_rmsnorm_scale_invariance_up_to_eps():
    """y(c x) = x / sqrt(ms + eps / c^2): scaling the row by c = 4 (exact in
    bf16) leaves y unchanged up to the eps term, and the change has the sign
    and size eps predicts."""
    heads = 2
    x = wi.packed_qkv(1, 5, heads, seed=22)[0, :, : heads * HD]
    gq, _ = wi.gammas(heads, 6, 7)
    y1 = oracle.rmsnorm(x, gq, EPS)
    y4 = oracle.rmsnorm((x.double() * 4).to(torch.bfloat16), gq, EPS)
    ms = (x.double().numpy() ** 2).mean(axis=1, keepdims=True)
    # |y4| / |y1| = sqrt((ms + eps) / (ms + eps / 16)) > 1
    ratio = np.sqrt((ms + EPS) / (ms + EPS / 16))
    np.testing.assert_allclose(y4, y1 * ratio, rtol=1e-13, atol=0)
    assert np.all(ratio > 1.0) and np.all(ratio - 1.0 < 1e-6)


def test_rmsnorm_is_full_width_not_per_head():
    heads = 6
    x = wi.head_magnitude_qkv(1, 9, heads, seed=3)[0, :, : heads * HD]
    g = torch.ones(heads * HD).to(torch.bfloat16)
    got = oracle.rmsnorm(x, g, EPS)
    full = torch.nn.functional.rms_norm(x.double(), (heads * HD,), eps=EPS).numpy()
    per_head = torch.nn.functional.rms_norm(x.double().view(9, heads, HD), (HD,), eps=EPS)
    per_head = per_head.reshape(9, heads * HD).numpy()
    np.testing.assert_allclose(got, full, rtol=1e-13)
    assert np.max(np.abs(got - per_head)) > 0.5  # the two readings are far apart here


def test_gamma_is_indexed_by_full_channel():
    heads = 4
    x = wi.packed_qkv(1, 5, heads, seed=8)[0, :, : heads * HD]
    g1 = torch.ones(heads * HD)
    g2 = g1.clone()
    g2[2 * HD:3 * HD] = 2.0  # only head 2's weights differ
    y1 = oracle.rmsnorm(x, g1.to(torch.bfloat16), EPS)
    y2 = oracle.rmsnorm(x, g2.to(torch.bfloat16), EPS)
    np.testing.assert_array_equal(y2[:, 2 * HD:3 * HD], 2.0 * y1[:, 2 * HD:3 * HD])
    np.testing.assert_array_equal(np.delete(y2, np.s_[2 * HD:3 * HD], axis=1),
                                  np.delete(y1, np.s_[2 * HD:3 * HD], axis=1))


def test_rounding_point_token0_is_rounded_norm():
    """At token 0 all angles are zero, so the fused step must equal round_bf16(norm)."""
    heads = 2
    w = wi.Workload("t", 1, (2, 2, 3), heads)
    qkv, gq, gk = wi.inputs_for(w, seed=21)
    out = oracle.qk_norm_rope(qkv, w.grid, heads, gq, gk, EPS, THETA)
    D = heads * HD
    for which, g in ((0, gq), (1, gk)):
        y = oracle.rmsnorm(qkv[0, :1, which * D:(which + 1) * D], g, EPS)
        ref = bf16(y).view(torch.int16)
        assert torch.equal(out[0, :1, which * D:(which + 1) * D].view(torch.int16), ref)
    # V passes through untouched
    assert torch.equal(out[..., 2 * D:].view(torch.int16), qkv[..., 2 * D:].view(torch.int16))


def test_rounding_point_is_before_rope():
    """Rotating the unrounded norm (no bf16 point) gives a different result on
    some elements; the oracle matches the rounded-then-rotated chain exactly."""
    heads = 2
    w = wi.Workload("t", 1, (3, 4, 5), heads)
    qkv, gq, gk = wi.inputs_for(w, seed=22)
    out = oracle.qk_norm_rope(qkv, w.grid, heads, gq, gk, EPS, THETA)
    D = heads * HD
    y = oracle.rmsnorm(qkv[0, :, :D], gq, EPS)
    yr = bf16(y).double().numpy()
    with_point = bf16(oracle.rope(yr, 0, heads, w.grid, THETA)).view(torch.int16)
    without_point = bf16(oracle.rope(y, 0, heads, w.grid, THETA)).view(torch.int16)
    assert torch.equal(out[0, :, :D].view(torch.int16), with_point)
    assert not torch.equal(with_point, without_point)


# ------------------------------------------------------------------------- RoPE
def _grid_index(grid, f, h, w):
    F, H, W = grid
    return (f * H + h) * W + w


def _complex_rotate(y, pairs_angle):
    """Rotate adjacent pairs of a 128-vector by given angles with numpy complex numbers."""
    z = y[0::2] + 1j * y[1::2]
    z = z * np.exp(1j * pairs_angle)
    out = np.empty_like(y)
    out[0::2], out[1::2] = z.real, z.imag
    return out


@pytest.mark.parametrize("pos,pair,angle", [((2, 0, 0), 0, 2.0), ((0, 3, 0), 22, 3.0),
                                            ((0, 0, 5), 43, 5.0), ((1, 1, 1), 0, 1.0)])
def test_rope_first_pair_of_each_axis_turns_by_position(pos, pair, angle):
    """The first pair of each axis has frequency theta^0 = 1: angle = position."""
    grid = (4, 5, 6)
    rng = np.random.default_rng(0)
    y = rng.standard_normal((1, HD))
    s = _grid_index(grid, *pos)
    got = oracle.rope(y, s, 1, grid, THETA)[0]
    u, v = y[0, 2 * pair], y[0, 2 * pair + 1]
    assert got[2 * pair] == pytest.approx(u * math.cos(angle) - v * math.sin(angle), abs=1e-14)
    assert got[2 * pair + 1] == pytest.approx(u * math.sin(angle) + v * math.cos(angle), abs=1e-14)


def test_rope_axis_isolation_44_42_42():
    grid = (3, 3, 3)
    rng = np.random.default_rng(1)
    y = rng.standard_normal((1, HD))
    spans = {(1, 0, 0): (0, 44), (0, 1, 0): (44, 86), (0, 0, 1): (86, 128)}
    for pos, (a, b) in spans.items():
        got = oracle.rope(y, _grid_index(grid, *pos), 1, grid, THETA)[0]
        changed = np.nonzero(np.abs(got - y[0]) > 0)[0]
        assert changed.min() == a and changed.max() == b - 1


def test_rope_matches_complex_rotation_and_frequency_ladder():
    """Against numpy complex rotation; frequencies within an axis form the
    geometric ladder 1, r, r^2, ... with r = theta^(-2/d_a)."""
    grid = (21, 30, 52)
    rng = np.random.default_rng(2)
    heads = 2
    y = rng.standard_normal((3, heads * HD))
    toks = [(20, 29, 51), (7, 0, 13), (0, 15, 0)]
    for t, pos in enumerate(toks):
        s = _grid_index(grid, *pos)
        got = oracle.rope(y[t:t + 1], s, heads, grid, THETA)[0]
        ang = []
        for axis, d_a in enumerate((44, 42, 42)):
            r = THETA ** (-2.0 / d_a)
            ang += [pos[axis] * r ** j for j in range(d_a // 2)]
        ang = np.array(ang)
        for h in range(heads):
            ref = _complex_rotate(y[t, h * HD:(h + 1) * HD], ang)
            np.testing.assert_allclose(got[h * HD:(h + 1) * HD], ref, rtol=0, atol=1e-12)


def test_rope_preserves_pair_norms():
    grid = (5, 8, 8)
    rng = np.random.default_rng(3)
    y = rng.standard_normal((320, 3 * HD))
    got = oracle.rope(y, 0, 3, grid, THETA)
    n0 = y[:, 0::2] ** 2 + y[:, 1::2] ** 2
    n1 = got[:, 0::2] ** 2 + got[:, 1::2] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-13)


def test_rope_dot_depends_only_on_offset():
    """<R(p) q, R(p') k> is unchanged when p and p' shift together along any axis."""
    grid = (6, 7, 8)
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, HD))
    k = rng.standard_normal((1, HD))

    def dot(pq, pk):
        a = oracle.rope(q, _grid_index(grid, *pq), 1, grid, THETA)[0]
        b = oracle.rope(k, _grid_index(grid, *pk), 1, grid, THETA)[0]
        return float(a @ b)

    base = dot((1, 2, 3), (0, 5, 1))
    for d in [(1, 0, 0), (0, 1, 0), (0, 0, 1), (4, 1, 4)]:
        sh = dot(tuple(a + b for a, b in zip((1, 2, 3), d)), tuple(a + b for a, b in zip((0, 5, 1), d)))
        assert sh == pytest.approx(base, abs=1e-11)
    assert abs(dot((1, 2, 3), (0, 5, 2)) - base) > 1e-3  # and it does depend on the offset


def test_rope_pair_layout_is_observable():
    """Adjacent pairs vs half-split pairs give different outputs: the layout is a real choice."""
    grid = (2, 2, 2)
    y = np.random.default_rng(5).standard_normal((1, HD))
    a = oracle.rope(y, 7, 1, grid, THETA)
    b = oracle.rope(y, 7, 1, grid, THETA, half_split=True)
    assert np.max(np.abs(a - b)) > 0.1


# -------------------------------------------------------------------- attention
def _qkv(B, S, heads, seed):
    return wi.packed_qkv(B, S, heads, seed)


def _split(qkv, heads):
    B, S, _ = qkv.shape
    x = qkv.double().view(B, S, 3, heads, HD)
    return x[:, :, 0].transpose(1, 2), x[:, :, 1].transpose(1, 2), x[:, :, 2].transpose(1, 2)


def test_attention_matches_library_sdpa_fp64():
    B, S, heads = 2, 75, 3
    qkv = _qkv(B, S, heads, 30)
    q, k, v = _split(qkv, heads)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=1 / math.sqrt(HD))
    got = oracle.attention_full(qkv, heads, 1 / math.sqrt(HD))
    np.testing.assert_allclose(got, ref.transpose(1, 2).numpy(), rtol=1e-12, atol=1e-14)


def test_attention_rows_are_convex_weights():
    """With V rows set to one-hot vectors e_j the output row is the softmax row:
    non-negative and summing to 1."""
    S, heads = 100, 1
    qkv = _qkv(1, S, heads, 31).float() * 3
    qkv[0, :, 2 * HD:] = 0
    qkv[0, torch.arange(S), 2 * HD + torch.arange(S)] = 1.0
    qkv = qkv.to(torch.bfloat16)
    got = oracle.attention_full(qkv, heads, 1 / math.sqrt(HD))[0, :, 0]
    w = got[:, :S]
    assert (w >= 0).all()
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-13)


def test_attention_constant_v_and_single_key():
    S, heads = 40, 2
    qkv = _qkv(1, S, heads, 32).float()
    cst = torch.randn(heads * HD, generator=torch.Generator().manual_seed(1))
    qkv[0, :, 2 * heads * HD:] = cst
    qkv = qkv.to(torch.bfloat16)
    got = oracle.attention_full(qkv, heads, 0.1)
    np.testing.assert_allclose(got.reshape(1, S, heads * HD),
                               cst.to(torch.bfloat16).double().expand(1, S, -1).numpy(), rtol=1e-13)
    one = _qkv(1, 1, heads, 33)
    got1 = oracle.attention_full(one, heads, 0.3)
    np.testing.assert_array_equal(got1.reshape(-1), one[0, 0, 2 * heads * HD:].double().numpy())


def test_attention_key_permutation_invariance():
    S, heads = 50, 2
    qkv = _qkv(1, S, heads, 34)
    perm = torch.randperm(S, generator=torch.Generator().manual_seed(2))
    D = heads * HD
    p = qkv.clone()
    p[0, :, D:] = qkv[0, perm, D:]  # permute K and V rows together, keep Q in place
    a = oracle.attention_full(qkv, heads, 0.2)
    b = oracle.attention_full(p, heads, 0.2)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-15)


def test_attention_peaked_logits_pick_one_value():
    S, heads = 64, 1
    qkv = _qkv(1, S, heads, 35).float()
    t = 17
    qkv[0, :, :HD] = 6.0 * qkv[0, t, HD:2 * HD]  # every query aligned with key t
    qkv = qkv.to(torch.bfloat16)
    got = oracle.attention_full(qkv, heads, 1 / math.sqrt(HD))[0, :, 0]
    np.testing.assert_allclose(got, qkv[0, t, 2 * HD:].double().numpy()[None, :].repeat(S, 0),
                               atol=1e-6)


def test_attention_brute_force_pure_python():
    """Tiny case, written as plain loops without max subtraction and with fsum."""
    S, heads = 6, 2
    qkv = _qkv(1, S, heads, 36)
    x = qkv.double()[0].tolist()
    D = heads * HD
    scale = 1 / math.sqrt(HD)
    got = oracle.attention_full(qkv, heads, scale)[0]
    for h in range(heads):
        for i in range(S):
            q = x[i][h * HD:(h + 1) * HD]
            e = [math.exp(scale * math.fsum(a * b for a, b in zip(q, x[j][D + h * HD:D + (h + 1) * HD])))
                 for j in range(S)]
            z = math.fsum(e)
            for d in range(HD):
                o = math.fsum(e[j] * x[j][2 * D + h * HD + d] for j in range(S)) / z
                assert got[i, h, d] == pytest.approx(o, rel=1e-12, abs=1e-15)


def test_attention_rows_subset_equals_full():
    B, S, heads = 2, 30, 2
    qkv = _qkv(B, S, heads, 37)
    full = oracle.attention_full(qkv, heads, 0.09)
    rows = [(1, 1, 29), (0, 0, 0), (1, 0, 7)]
    sub = oracle.attention_rows(qkv, heads, rows, 0.09)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(sub[r], full[b, i, h])


def test_full_chain_brute_force_tiny_grid():
    """norm -> bf16 -> RoPE -> bf16 on a (1,2,3) grid, written with Python's
    cmath, against the oracle's fused step."""
    grid, heads = (1, 2, 3), 1
    w = wi.Workload("t", 1, grid, heads)
    qkv, gq, gk = wi.inputs_for(w, seed=40)
    out = oracle.qk_norm_rope(qkv, grid, heads, gq, gk, EPS, THETA)
    x = qkv.double()[0].tolist()
    D = heads * HD
    for s in range(6):
        pos = (0, s // 3, s % 3)
        for which, g in ((0, gq.double().tolist()), (1, gk.double().tolist())):
            row = x[s][which * D:(which + 1) * D]
            r = 1 / math.sqrt(math.fsum(v * v for v in row) / D + EPS)
            y = [float(bf16(row[c] * r * g[c])) for c in range(D)]
            ref = []
            for p in range(HD // 2):
                axis, j, d_a = (0, p, 44) if p < 22 else ((1, p - 22, 42) if p < 43 else (2, p - 43, 42))
                z = complex(y[2 * p], y[2 * p + 1]) * cmath.exp(1j * pos[axis] * THETA ** (-2 * j / d_a))
                ref += [z.real, z.imag]
            got = out[0, s, which * D:(which + 1) * D].double()
            exp = bf16(ref).double()
            # one-ulp slack: the reference rotates in a different order of operations
            ulp = torch.ldexp(torch.ones_like(exp), torch.frexp(exp.abs().clamp_min(1e-30)).exponent - 8)
            assert bool(((got - exp).abs() <= ulp).all())


def test_token_subset_equals_full_buffer():
    w = wi.Workload("t", 2, (3, 4, 5), 2)
    qkv, gq, gk = wi.inputs_for(w, seed=41)
    full = oracle.qk_norm_rope(qkv, w.grid, 2, gq, gk, EPS, THETA)
    toks = [(0, 0), (1, 59), (1, 17), (0, 33)]
    sub = oracle.qk_norm_rope_tokens(qkv, w.grid, 2, gq, gk, EPS, THETA, toks)
    D = 2 * HD
    for r, (b, s) in enumerate(toks):
        assert torch.equal(sub[r].view(torch.int16), full[b, s, :2 * D].view(torch.int16))
