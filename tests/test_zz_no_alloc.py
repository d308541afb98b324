"""wan_dit_attn_host_static: the host-buffer step for callers that cannot
allocate device memory (a host application with no device allocator of its
own, a process whose device memory another runtime's pool holds, a caller
that cannot afford cudaMalloc's device-wide synchronisation). It runs
through a device array inside the library, so the caller passes only its
page-locked host input and output and the norm weights.

Two calls in a row through the C ABI, with different shapes, each checked
against wan_dit_attn_host (the same step through device buffers the caller
allocates) at the attention tolerance. The second call runs on the array
that still holds the first call's data. This file is collected last, so a
run that stops at the first failure has run every other test before it."""
import ctypes

import pytest
import torch

import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from helpers import assert_attention_close
from video_diffusion_transformer_packed_b200 import build as wan_build

pytestmark = pytest.mark.gpu

CASES = [  # (grid, heads, batch, seed): the tiny Wan grid, then a smaller, batched one
    ((5, 8, 8), 12, 1, 0),
    ((2, 10, 13), 4, 2, 1),
]


@pytest.fixture(scope="module")
def lib():
    wan_build.build()
    return wan.load_library()


def _pinned(t):
    p = torch.empty_like(t).pin_memory()
    p.copy_(t)
    return p


def test_static_staging_matches_caller_buffers_on_two_calls_in_a_row(lib):
    stream = torch.cuda.current_stream()
    runs = []
    for grid, heads, batch, seed in CASES:
        w = wi.Workload("case", batch, grid, heads)
        qkv, gq, gk = wi.inputs_for(w, seed=seed)
        qkv_host = _pinned(qkv)
        out_host = torch.empty((batch, w.seq_len, w.dim), dtype=torch.bfloat16).pin_memory()
        gq_d, gk_d = gq.cuda(), gk.cuda()
        F, H, W = grid
        status = lib.wan_dit_attn_host_static(qkv_host.data_ptr(), out_host.data_ptr(), batch, F, H, W, heads,
                                              128, gq_d.data_ptr(), gk_d.data_ptr(), wi.EPS, wi.THETA, 0.0, 0, 0,
                                              ctypes.c_void_p(stream.cuda_stream))
        assert status == 0, wan.STATUS.get(status, status)
        runs.append((w, qkv_host, gq_d, gk_d, out_host))
    stream.synchronize()
    assert wan.device_error() == 0
    for w, qkv_host, gq_d, gk_d, out_host in runs:
        ref = wan.dit_attn_host(qkv_host, w.grid, w.heads, gq_d, gk_d)
        torch.cuda.synchronize()
        assert_attention_close(out_host, ref.double().numpy(), f"static staging {w.grid} x {w.heads} heads")


def test_static_staging_refuses_steps_beyond_its_buffer(lib):
    # batch * S * heads * 128 above WAN_HOST_STATIC_MAX_ELEMENTS (8 Mi): refused
    # before anything is launched or read (the pointers are never touched).
    fake = 0x10000
    grid, heads = (5, 30, 52), 40  # 7800 tokens x 5120 channels = 39.9 Mi elements
    status = lib.wan_dit_attn_host_static(fake, fake, 1, *grid, heads, 128, fake, fake, wi.EPS, wi.THETA, 0.0, 0, 0,
                                          None)
    assert status == 12  # WAN_ERR_TOO_LARGE
    assert b"WAN_HOST_STATIC_MAX_ELEMENTS" in lib.wan_status_string(12)
