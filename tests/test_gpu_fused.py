"""The chained entry point: wan_dit_attn equals the two separate calls bit for
bit, keeps the packed storage (V untouched), and matches the oracle chain."""
import math

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


@pytest.mark.parametrize("idx", [0, 1])
def test_dit_attn_equals_separate_calls(idx):
    w = wi.WORKLOADS[idx]
    qkv, gq, gk = wi.inputs_for(w, seed=1)
    gq, gk = gq.cuda(), gk.cuda()
    a = qkv.cuda()
    out_a = wan.dit_attn(a, w.grid, w.heads, gq, gk)
    b = qkv.cuda()
    wan.qk_norm_rope(b, w.grid, w.heads, gq, gk)
    out_b = wan.self_attention(b, w.heads)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(out_a.view(torch.int16), out_b.view(torch.int16))
    D = w.dim
    assert torch.equal(a[..., 2 * D:].cpu().view(torch.int16), qkv[..., 2 * D:].view(torch.int16))


def test_in_place_equals_out_of_place_copy():
    """Running on a view inside a larger allocation gives the same bits as on a fresh buffer."""
    w = wi.WORKLOADS[0]
    qkv, gq, gk = wi.inputs_for(w, seed=2)
    big = torch.zeros(qkv.numel() + 4096, dtype=torch.bfloat16, device="cuda")
    view = big[2048:2048 + qkv.numel()].view(qkv.shape)
    view.copy_(qkv.cuda())
    fresh = qkv.cuda()
    wan.qk_norm_rope(view, w.grid, w.heads, gq.cuda(), gk.cuda())
    wan.qk_norm_rope(fresh, w.grid, w.heads, gq.cuda(), gk.cuda())
    torch.cuda.synchronize()
    assert torch.equal(view.view(torch.int16), fresh.view(torch.int16))
    assert int(big[:2048].abs().max()) == 0 and int(big[2048 + qkv.numel():].abs().max()) == 0


def test_chain_matches_oracle_chain_tiny():
    w = wi.WORKLOADS[0]
    qkv, gq, gk = wi.inputs_for(w, seed=3)
    d = qkv.cuda()
    out = wan.dit_attn(d, w.grid, w.heads, gq.cuda(), gk.cuda())
    torch.cuda.synchronize()
    normed = oracle.qk_norm_rope(qkv, w.grid, w.heads, gq, gk, wi.EPS, wi.THETA)
    D = w.dim
    assert int(bf16_ulp_distance(d.cpu()[..., :2 * D], normed[..., :2 * D]).max()) <= 1
    ref = oracle.attention_full(normed, w.heads, 1.0 / math.sqrt(wi.HEAD_DIM))
    assert_attention_close(out.cpu().view(1, w.seq_len, w.heads, wi.HEAD_DIM), ref, "chain")


def test_gpu_argument_errors():
    w = wi.WORKLOADS[0]
    qkv, gq, gk = wi.inputs_for(w, seed=4)
    d = qkv.cuda()
    lib = wan.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    # misaligned qkv (2 bytes into the allocation)
    st = lib.wan_self_attention(d.data_ptr() + 2, d.data_ptr() + 2 * d.numel() + 4096, 1, w.seq_len,
                                w.heads, 128, 0.0, stream)
    assert st == 2
    # out inside qkv
    st = lib.wan_self_attention(d.data_ptr(), d.data_ptr() + 1024, 1, w.seq_len, w.heads, 128, 0.0, stream)
    assert st == 9
    before = d.clone()
    with pytest.raises(ValueError):  # grid does not match the buffer: refused before any launch
        wan.qk_norm_rope(d, (5, 8, 9), w.heads, gq.cuda(), gk.cuda())
    with pytest.raises(wan.WanError):  # eps <= 0
        wan.qk_norm_rope(d, w.grid, w.heads, gq.cuda(), gk.cuda(), eps=0.0)
    torch.cuda.synchronize()
    assert torch.equal(before.view(torch.int16), d.view(torch.int16))
