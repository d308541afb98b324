"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/*.h, and rejects invalid arguments before touching CUDA."""
import ctypes
import glob
import os
import re

import pytest

import video_diffusion_transformer_packed_b200 as wan
from video_diffusion_transformer_packed_b200 import build as wan_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    wan_build.build()
    return wan.load_library()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"WAN_API\s+[\w\s\*]+?\b(wan_\w+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_three_entry_points():
    names = declared_functions()
    for n in ("wan_qk_norm_rope", "wan_self_attention", "wan_dit_attn"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings(lib):
    assert lib.wan_abi_version() == 2
    for code in range(10):
        assert lib.wan_status_string(code)
    assert lib.wan_status_string(99) == b"unknown status"


FAKE = 0x10000  # a 16-byte-aligned address that is never dereferenced: validation fails first


@pytest.mark.parametrize("args,status", [
    # (qkv, batch, F, H, W, heads, head_dim, gq, gk, eps, theta)
    ((None, 1, 2, 2, 2, 1, 128, FAKE, FAKE, 1e-6, 1e4), 1),
    ((FAKE, 1, 2, 2, 2, 1, 128, None, FAKE, 1e-6, 1e4), 1),
    ((FAKE + 2, 1, 2, 2, 2, 1, 128, FAKE, FAKE, 1e-6, 1e4), 2),
    ((FAKE, 1, 2, 2, 2, 1, 64, FAKE, FAKE, 1e-6, 1e4), 4),
    ((FAKE, 0, 2, 2, 2, 1, 128, FAKE, FAKE, 1e-6, 1e4), 3),
    ((FAKE, 1, 0, 2, 2, 1, 128, FAKE, FAKE, 1e-6, 1e4), 3),
    ((FAKE, 1, 2, 2, 2, 0, 128, FAKE, FAKE, 1e-6, 1e4), 3),
    ((FAKE, 1, 2, 2, 2, 65, 128, FAKE, FAKE, 1e-6, 1e4), 3),
    ((FAKE, 1, 65536, 65536, 2, 1, 128, FAKE, FAKE, 1e-6, 1e4), 3),
    ((FAKE, 1, 2, 2, 2, 1, 128, FAKE, FAKE, 0.0, 1e4), 5),
    ((FAKE, 1, 2, 2, 2, 1, 128, FAKE, FAKE, float("nan"), 1e4), 5),
    ((FAKE, 1, 2, 2, 2, 1, 128, FAKE, FAKE, 1e-6, 1.0), 5),
])
def test_norm_rope_rejects_bad_arguments(lib, args, status):
    assert lib.wan_qk_norm_rope(*args, None) == status


@pytest.mark.parametrize("args,status", [
    # (qkv, out, batch, seq_len, heads, head_dim, scale)
    ((None, FAKE, 1, 8, 1, 128, 0.0), 1),
    ((FAKE, None, 1, 8, 1, 128, 0.0), 1),
    ((FAKE, FAKE * 16 + 8, 1, 8, 1, 128, 0.0), 2),
    ((FAKE, FAKE * 16, 1, 8, 1, 127, 0.0), 4),
    ((FAKE, FAKE * 16, 1, 0, 1, 128, 0.0), 3),
    ((FAKE, FAKE * 16, 1, 2**31, 1, 128, 0.0), 3),
    ((FAKE, FAKE * 16, 1, 8, 1, 128, float("inf")), 5),
    ((FAKE, FAKE + 256, 1, 8, 1, 128, 0.0), 9),  # out overlaps qkv
])
def test_attention_rejects_bad_arguments(lib, args, status):
    assert lib.wan_self_attention(*args, None) == status


def test_dit_attn_validates_both_steps(lib):
    assert lib.wan_dit_attn(FAKE, FAKE + 64, 1, 2, 2, 2, 1, 128, FAKE, FAKE, 1e-6, 1e4, 0.0, None) == 9
    assert lib.wan_dit_attn(FAKE, FAKE * 16, 1, 2, 2, 2, 1, 128, FAKE, FAKE, -1.0, 1e4, 0.0, None) == 5


def test_valid_arguments_without_a_b200_fail_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = lib.wan_qk_norm_rope(FAKE, 1, 2, 2, 2, 1, 128, FAKE, FAKE, 1e-6, 1e4, None)
    assert st == 6  # WAN_ERR_UNSUPPORTED_DEVICE: no silent fallback
    with pytest.raises(TypeError):
        wan.self_attention(torch.zeros(1, 8, 384, dtype=torch.bfloat16), 1)


def test_selftest_entry_point_validates_before_launch(lib):
    # (qkv, out, batch, seq_len, heads, head_dim, wait_limit_ns)
    assert lib.wan_selftest_wait_timeout(None, FAKE, 1, 8, 1, 128, 10**7, None) == 1
    assert lib.wan_selftest_wait_timeout(FAKE, FAKE * 16, 1, 8, 1, 128, 10, None) == 5
    assert lib.wan_selftest_wait_timeout(FAKE, FAKE * 16, 1, 8, 1, 64, 10**7, None) == 4
