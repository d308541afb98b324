"""The host-buffer entry point wan_dit_attn_host: the pipelined step (strided
host->device copies of Q|K and of V head chunks, per-batch norm+RoPE, attention
per head chunk, device->host copies of the output) gives the same bits as the
device-resident wan_dit_attn, for every chunking, ragged shapes included; it
leaves qkv_host untouched, leaves the normalised buffer in qkv_dev, orders
itself on the caller's stream, and refuses pageable host memory."""
import math

import pytest
import torch

import oracle
import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import build as wan_build
from helpers import assert_attention_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


def _device_reference(qkv, w, gq, gk):
    d = qkv.cuda()
    out = wan.dit_attn(d, w.grid, w.heads, gq, gk)
    torch.cuda.synchronize()
    return d, out


def _pinned(t):
    return t.contiguous().pin_memory()


# (grid, heads, batch): the tiny Wan grid, a ragged S with a head count that
# no chunk size divides, and the A14B head count at batch 2 (CFG)
CASES = [((5, 8, 8), 12, 1), ((2, 10, 13), 7, 2), ((1, 9, 29), 40, 2)]


@pytest.mark.parametrize("grid,heads,batch", CASES)
@pytest.mark.parametrize("hc", [0, 1, 3, 8, 64])
def test_host_pipeline_equals_device_path(grid, heads, batch, hc):
    if hc > heads:
        hc = heads
    w = wi.Workload("case", batch, grid, heads)
    qkv, gq, gk = wi.inputs_for(w, seed=11)
    gq, gk = gq.cuda(), gk.cuda()
    ref_qkv, ref_out = _device_reference(qkv, w, gq, gk)
    qkv_h = _pinned(qkv)
    keep = qkv_h.clone()
    qkv_d = torch.full_like(ref_qkv, float("nan"))
    out_d = torch.full_like(ref_out, float("nan"))
    out_h = wan.dit_attn_host(qkv_h, w.grid, w.heads, gq, gk, qkv_dev=qkv_d, out_dev=out_d,
                              heads_per_chunk=hc)
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    assert torch.equal(out_h.view(torch.int16), ref_out.cpu().view(torch.int16))
    assert torch.equal(qkv_d.view(torch.int16), ref_qkv.view(torch.int16))
    assert torch.equal(qkv_h.view(torch.int16), keep.view(torch.int16))  # input only read


def test_host_pipeline_matches_oracle_tiny():
    w = wi.WORKLOADS[0]
    qkv, gq, gk = wi.inputs_for(w, seed=12)
    out_h = wan.dit_attn_host(_pinned(qkv), w.grid, w.heads, gq.cuda(), gk.cuda())
    torch.cuda.synchronize()
    normed = oracle.qk_norm_rope(qkv, w.grid, w.heads, gq, gk, wi.EPS, wi.THETA)
    ref = oracle.attention_full(normed, w.heads, 1.0 / math.sqrt(wi.HEAD_DIM))
    assert_attention_close(out_h.view(1, w.seq_len, w.heads, wi.HEAD_DIM), ref, "host pipeline vs oracle")


def test_host_pipeline_is_ordered_on_a_side_stream():
    """Back-to-back calls on one non-default stream, reusing the device buffers:
    each call waits for the previous one's copies, and a later kernel on the
    stream sees the output written."""
    w = wi.Workload("case", 2, (2, 10, 13), 7)
    gq_h, gk_h = wi.gammas(w.heads)
    gq, gk = gq_h.cuda(), gk_h.cuda()
    s = torch.cuda.Stream()
    qkv_d = torch.empty((w.batch, w.seq_len, 3 * w.dim), dtype=torch.bfloat16, device="cuda")
    out_d = torch.empty((w.batch, w.seq_len, w.dim), dtype=torch.bfloat16, device="cuda")
    outs, refs = [], []
    for seed in (21, 22, 23):
        qkv = wi.packed_qkv(w.batch, w.seq_len, w.heads, seed=seed)
        _, ref = _device_reference(qkv, w, gq, gk)
        refs.append(ref.cpu())
        outs.append(wan.dit_attn_host(_pinned(qkv), w.grid, w.heads, gq, gk, qkv_dev=qkv_d,
                                      out_dev=out_d, heads_per_chunk=3, stream=s))
    s.synchronize()
    for o, r in zip(outs, refs):
        assert torch.equal(o.view(torch.int16), r.view(torch.int16))


def test_host_pipeline_refuses_pageable_or_foreign_memory():
    w = wi.WORKLOADS[0]
    qkv, gq, gk = wi.inputs_for(w, seed=13)
    gq, gk = gq.cuda(), gk.cuda()
    with pytest.raises(TypeError):
        wan.dit_attn_host(qkv, w.grid, w.heads, gq, gk)  # pageable: refused by the binding
    lib = wan.load_library()
    qkv_d = qkv.cuda()
    out_d = torch.empty((1, w.seq_len, w.dim), dtype=torch.bfloat16, device="cuda")
    out_pageable = torch.empty((1, w.seq_len, w.dim), dtype=torch.bfloat16)
    args = [qkv.data_ptr(), out_pageable.data_ptr(), qkv_d.data_ptr(), out_d.data_ptr(), 1, *w.grid,
            w.heads, 128, gq.data_ptr(), gk.data_ptr(), wi.EPS, wi.THETA, 0.0, 0, 0, None]
    assert lib.wan_dit_attn_host(*args) == 10  # pageable host memory
    qkv_h, out_h = _pinned(qkv), _pinned(out_pageable)
    args[0], args[1] = qkv_h.data_ptr(), out_h.data_ptr()
    args[2] = qkv_h.data_ptr()  # a host buffer where device memory is required
    assert lib.wan_dit_attn_host(*args) == 10
    args[2] = qkv_d.data_ptr()
    assert lib.wan_dit_attn_host(*args) == 0
    torch.cuda.synchronize()


def test_overlapped_calls_with_alternating_buffers():
    """WAN_HOST_OVERLAP_INPUT with two alternating device buffer sets on one
    stream: every call's output equals the device path's."""
    w = wi.Workload("case", 2, (2, 10, 13), 7)
    gq_h, gk_h = wi.gammas(w.heads)
    gq, gk = gq_h.cuda(), gk_h.cuda()
    s = torch.cuda.Stream()
    sets = [(torch.empty((w.batch, w.seq_len, 3 * w.dim), dtype=torch.bfloat16, device="cuda"),
             torch.empty((w.batch, w.seq_len, w.dim), dtype=torch.bfloat16, device="cuda")) for _ in range(2)]
    outs, refs = [], []
    for k, seed in enumerate((31, 32, 33, 34)):
        qkv = wi.packed_qkv(w.batch, w.seq_len, w.heads, seed=seed)
        _, ref = _device_reference(qkv, w, gq, gk)
        refs.append(ref.cpu())
        qd, od = sets[k % 2]
        outs.append(wan.dit_attn_host(_pinned(qkv), w.grid, w.heads, gq, gk, qkv_dev=qd, out_dev=od,
                                      heads_per_chunk=3, overlap_input=True, stream=s))
    s.synchronize()
    for o, r in zip(outs, refs):
        assert torch.equal(o.view(torch.int16), r.view(torch.int16))


@pytest.mark.parametrize("n_sets", [2, 1])
def test_overlapped_calls_when_kernels_outlast_the_transfer(n_sets):
    """One head at S = 75600: each call's attention takes about twice its input
    transfer, so the copy stream runs ahead of the kernels. Eight overlapped
    calls on two alternating buffer sets (or one set reused by every call):
    a call's copies into a set must wait for the kernels of the call that used
    it before, and every output must equal the device path's."""
    w = wi.Workload("case", 1, (21, 45, 80), 1)
    gq_h, gk_h = wi.gammas(w.heads)
    gq, gk = gq_h.cuda(), gk_h.cuda()
    s = torch.cuda.Stream()
    sets = [(torch.empty((w.batch, w.seq_len, 3 * w.dim), dtype=torch.bfloat16, device="cuda"),
             torch.empty((w.batch, w.seq_len, w.dim), dtype=torch.bfloat16, device="cuda"))
            for _ in range(n_sets)]
    inputs = [_pinned(wi.packed_qkv(w.batch, w.seq_len, w.heads, seed=40 + k)) for k in range(8)]
    refs = [_device_reference(x.clone(), w, gq, gk)[1].cpu() for x in inputs]
    outs = []
    for k, x in enumerate(inputs):
        qd, od = sets[k % n_sets]
        outs.append(wan.dit_attn_host(x, w.grid, w.heads, gq, gk, qkv_dev=qd, out_dev=od,
                                      overlap_input=True, stream=s))
    s.synchronize()
    assert wan.device_error() == 0
    for o, r in zip(outs, refs):
        assert torch.equal(o.view(torch.int16), r.view(torch.int16))


def test_temporary_pinned_input_survives_until_the_step_is_done():
    """The input's copies run on the library's streams after the call returns.
    A temporary pinned input must not go back to torch's pinned-memory cache
    (which would hand the same block to the next pin_memory() at once) before
    they are done: the returned output keeps it referenced. Same-size pinned
    buffers filled with other data right after the call would take its block
    otherwise; the result must still be the step of the original input."""
    w = wi.Workload("case", 2, (5, 20, 26), 8)
    qkv, gq, gk = wi.inputs_for(w, seed=71)
    gq_d, gk_d = gq.cuda(), gk.cuda()
    ref = wan.dit_attn(qkv.cuda(), w.grid, w.heads, gq_d, gk_d).cpu()
    s = torch.cuda.Stream()
    for trial in range(5):  # without the reference, 2 of 5 such trials read recycled data
        with torch.cuda.stream(s):
            out_h = wan.dit_attn_host(qkv.contiguous().pin_memory(), w.grid, w.heads, gq_d, gk_d, stream=s)
            others = [torch.full_like(qkv, float(k + 3)).pin_memory() for k in range(4)]
        s.synchronize()
        assert torch.equal(out_h.view(torch.int16), ref.view(torch.int16)), trial
        assert all(float(o[0, 0, 0]) == k + 3 for k, o in enumerate(others))


def test_device_temporaries_stay_reserved_while_a_side_stream_step_runs():
    """Called on a stream other than torch's current one and without device
    buffers, the step makes qkv_dev and out_dev itself and drops them when
    the call returns, while its copies and kernels still run. Tensors of the
    same sizes allocated on the current stream right after the call, and
    overwritten there while the step runs, must not get their memory: the
    result must still be the step of the input."""
    w = wi.Workload("case", 1, (21, 30, 52), 2)  # S = 32760: about a millisecond each of copy and attention
    qkv, gq, gk = wi.inputs_for(w, seed=73)
    gq_d, gk_d = gq.cuda(), gk.cuda()
    ref = wan.dit_attn(qkv.cuda(), w.grid, w.heads, gq_d, gk_d).cpu()
    qkv_p = _pinned(qkv)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    for trial in range(3):
        out_h = wan.dit_attn_host(qkv_p, w.grid, w.heads, gq_d, gk_d, stream=s)
        a = torch.empty(qkv.shape, dtype=torch.bfloat16, device="cuda")
        o = torch.empty((w.batch, w.seq_len, w.dim), dtype=torch.bfloat16, device="cuda")
        for k in range(6):  # overwrite both at intervals spanning the step
            torch.cuda._sleep(400_000)
            a.fill_(float(k + 1))
            o.fill_(float(-k - 1))
        s.synchronize()
        torch.cuda.synchronize()
        assert torch.equal(out_h.view(torch.int16), ref.view(torch.int16)), trial
