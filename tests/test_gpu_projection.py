"""The projection GEMM (wan_linear) and the norm+RoPE that takes its row
statistics, through the C ABI, against the oracle.

GEMM bound, per element: the exact product c = sum_k x_k w_k (fp64) against
the kernel's bf16 output y: |y - c| <= 2^-8 |c| (the bf16 rounding, with
margin) + 2^-16 sum_k |x_k w_k| (fp32 accumulation over K terms in any
order). The statistics must equal the fp64 sums of squares of the kernel's own
bf16 outputs (exact squares; only the order of the additions may differ:
relative 1e-12; a zero output counts as 2^-127, hence an absolute
256 * 2^-126). The norm+RoPE fed by the statistics must stay within 1 bf16
ulp of the oracle, like the reducing kernel."""
import numpy as np
import pytest
import torch

import oracle
import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import build as wan_build
from helpers import assert_attention_close, bf16_ulp_distance

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


def _operands(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    return x, w


def _check_rows(y, x, w, rows):
    ref = oracle.linear_rows(x, w, rows)
    got = y.reshape(-1, y.shape[-1])[torch.as_tensor(rows)].double().cpu().numpy()
    xa = x.reshape(-1, x.shape[-1])[torch.as_tensor(rows)].double().abs().numpy()
    mag = xa @ w.double().abs().numpy().T
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -16 * mag
    assert (err <= bound).all(), f"worst {float((err / bound).max()):.2f} of the bound"


@pytest.mark.parametrize("M,N,K", [(1000, 512, 256), (300, 768, 5120), (257, 256, 64), (1, 256, 128)])
def test_linear_matches_oracle(M, N, K):
    x, w = _operands(M, N, K, seed=M + N + K)
    y, _ = wan.linear(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    _check_rows(y, x, w, list(range(M)))


def test_statistics_are_the_sums_of_squares_of_the_outputs():
    M, N, K = 700, 1536, 512
    x, w = _operands(M, N, K, seed=4)
    y, stats = wan.linear(x.cuda(), w.cuda(), stat_cols=1024)
    torch.cuda.synchronize()
    yv = y.double().cpu().numpy()
    ref = (yv[:, :1024] ** 2).reshape(M, 4, 256).sum(axis=2)
    np.testing.assert_allclose(stats.cpu().numpy(), ref, rtol=1e-12, atol=256 * 2.0 ** -126)


@pytest.mark.parametrize("grid,heads,batch", [((5, 8, 8), 12, 1), ((2, 10, 13), 4, 2)])
def test_norm_with_projection_statistics(grid, heads, batch):
    """x -> QKV projection (with the statistic) -> norm+RoPE from the statistic:
    within 1 ulp of the oracle's norm+RoPE of the projection's output, and V
    untouched."""
    w_ = wi.Workload("case", batch, grid, heads)
    D = w_.dim
    x, wqkv = _operands(batch * w_.seq_len, 3 * D, D, seed=heads)
    gq, gk = wi.gammas(heads)
    qkv, stats = wan.linear(x.cuda(), wqkv.cuda(), stat_cols=2 * D)
    qkv = qkv.view(batch, w_.seq_len, 3 * D)
    before = qkv.cpu().clone()
    wan.qk_norm_rope_stats(qkv, grid, heads, gq.cuda(), gk.cuda(), stats)
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    ref = oracle.qk_norm_rope(before, grid, heads, gq, gk, wi.EPS, wi.THETA)
    got = qkv.cpu()
    assert int(bf16_ulp_distance(got[..., :2 * D], ref[..., :2 * D]).max()) <= 1
    assert torch.equal(got[..., 2 * D:].view(torch.int16), before[..., 2 * D:].view(torch.int16))


def test_qkv_projection_full_size_sampled_rows():
    """The bench workload's QKV projection (2 x 32760 tokens, 5120 -> 15360)
    with the statistic, in full: sampled rows against the oracle, statistics
    of sampled rows against the outputs."""
    w_ = wi.BY_NAME["a14b_480p_81f_cfg_b2"]
    M, D = w_.batch * w_.seq_len, w_.dim
    x, w = _operands(M, 3 * D, D, seed=7)
    y, stats = wan.linear(x.cuda(), w.cuda(), stat_cols=2 * D)
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    rows = sorted({0, M - 1, M - 2} | set(torch.randint(0, M, (24,), generator=torch.Generator().manual_seed(3)).tolist()))
    _check_rows(y, x, w, rows)
    yv = y[torch.as_tensor(rows).cuda()].double().cpu().numpy()
    ref = (yv[:, :2 * D] ** 2).reshape(len(rows), 2 * D // 256, 256).sum(axis=2)
    np.testing.assert_allclose(stats[torch.as_tensor(rows).cuda()].cpu().numpy(), ref, rtol=1e-12,
                               atol=256 * 2.0 ** -126)


@pytest.mark.parametrize("name", ["tiny_5x8x8_h12_b1", "a14b_480p_81f_cfg_b2"])
def test_block_chain_against_the_oracle_chain(name):
    """The DiT block's self-attention from activations to the output
    projection, all on the GPU through the C ABI:
        wan_linear (QKV projection, with the norm's statistic)
        -> wan_qk_norm_rope_stats -> wan_self_attention
        -> wan_linear (output projection, tokens x D -> D),
    against the oracle's chain from the same activations and weights:
        linear_bf16 -> qk_norm_rope -> attention_rows (rounded to bf16, the
        output's storage type) -> linear_rows,
    on sampled tokens (every token of the tiny grid; at the bench shape the
    first, the last, the ragged last tile and random ones), every output
    channel, at the attention bar. Each stage is also checked on the GPU's
    own input to it, so that a failure names its stage."""
    w_ = wi.BY_NAME[name]
    B, S, D, heads = w_.batch, w_.seq_len, w_.dim, w_.heads
    g = torch.Generator().manual_seed(71)
    x = torch.randn(B * S, D, generator=g).to(torch.bfloat16)
    wqkv = (torch.randn(3 * D, D, generator=g) / D ** 0.5).to(torch.bfloat16)
    wo = (torch.randn(D, D, generator=g) / D ** 0.5).to(torch.bfloat16)
    gq, gk = wi.gammas(heads)
    # GPU chain
    qkv, stats = wan.linear(x.cuda(), wqkv.cuda(), stat_cols=2 * D)
    qkv = qkv.view(B, S, 3 * D)
    proj = qkv.cpu()
    wan.qk_norm_rope_stats(qkv, w_.grid, heads, gq.cuda(), gk.cuda(), stats)
    normed = qkv.cpu()
    attn = wan.self_attention(qkv, heads)
    y, _ = wan.linear(attn.view(B * S, D), wo.cuda())
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    attn_h = attn.cpu().view(B * S, D)
    if S <= 4096:
        toks = np.arange(B * S)
    else:
        local = wi.sample_rows(S, 20, seed=72).numpy()
        toks = np.concatenate([b * S + local for b in range(B)])
    # stage by stage, each on the GPU's own input
    _check_rows(proj.view(B * S, 3 * D), x, wqkv, toks)
    tk = np.stack([toks // S, toks % S], axis=1)
    nr = oracle.qk_norm_rope_tokens(proj, w_.grid, heads, gq, gk, wi.EPS, wi.THETA, tk)
    assert int(bf16_ulp_distance(normed.view(B * S, 3 * D)[torch.from_numpy(toks), :2 * D], nr).max()) <= 1
    rows = np.array([(t // S, h, t % S) for t in toks for h in range(heads)], dtype=np.int64)
    a_ref = oracle.attention_rows(normed, heads, rows, 1 / 128 ** 0.5)
    assert_attention_close(attn_h[torch.from_numpy(toks)].view(-1, 128), a_ref, f"{name}: attention stage")
    _check_rows(y.cpu(), attn_h, wo, toks)
    # the oracle's own chain from the activations
    o_proj = oracle.linear_bf16(x, wqkv).view(B, S, 3 * D)
    o_normed = oracle.qk_norm_rope(o_proj, w_.grid, heads, gq, gk, wi.EPS, wi.THETA)
    o_attn = oracle.to_bf16(oracle.attention_rows(o_normed, heads, rows, 1 / 128 ** 0.5)).view(len(toks), D)
    o_y = oracle.linear_rows(o_attn, wo, np.arange(len(toks)))
    assert_attention_close(y.cpu()[torch.from_numpy(toks)], o_y, f"{name}: chain output")
