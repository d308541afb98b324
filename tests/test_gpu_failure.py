"""Failure detection on the GPU without a GPU fault: the attention kernel's
waits are bounded, so a pipeline that never receives its data reports a
timeout through the device error word, writes nothing, and leaves the CUDA
context usable for the next (correct) launch."""
import math

import pytest
import torch

import oracle
import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import build as wan_build
from helpers import assert_attention_close

pytestmark = pytest.mark.gpu

ERR_MMA, ERR_SOFTMAX = 2, 4


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


def test_stalled_pipeline_times_out_and_context_survives():
    S, heads = 256, 1
    qkv = wi.packed_qkv(1, S, heads, seed=9)
    d = qkv.cuda()
    assert wan.device_error() == 0
    out = torch.full((1, S, heads * 128), 7.0, dtype=torch.bfloat16, device="cuda")
    wan.selftest_wait_timeout(d, heads, out=out, wait_limit_ns=20_000_000)
    code = wan.device_error()
    assert code & ERR_MMA and code & ERR_SOFTMAX, code
    assert wan.device_error() == 0  # reading clears the word
    assert bool((out == 7.0).all())  # nothing was written
    # the context still works: a normal launch is correct and reports no error
    got = wan.self_attention(d, heads)
    assert wan.device_error() == 0
    ref = oracle.attention_full(qkv, heads, 1.0 / math.sqrt(128))
    assert_attention_close(got.cpu().view(1, S, heads, 128), ref, "after self-test")


def test_selftest_rejects_bad_limits():
    d = wi.packed_qkv(1, 128, 1, seed=1).cuda()
    with pytest.raises(wan.WanError):
        wan.selftest_wait_timeout(d, 1, wait_limit_ns=10)
