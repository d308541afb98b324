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
    for n in ("wan_qk_norm_rope", "wan_self_attention", "wan_dit_attn", "wan_dit_attn_host"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_status_strings(lib):
    assert lib.wan_abi_version() == 12
    for code in range(14):
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


def test_host_pipeline_validates_before_touching_memory(lib):
    # (qkv_host, out_host, qkv_dev, out_dev, batch, F, H, W, heads, head_dim, gq, gk, eps, theta,
    #  scale, heads_per_chunk)
    ok = (FAKE * 64, FAKE * 128, FAKE, FAKE * 16, 1, 2, 2, 2, 4, 128, FAKE, FAKE, 1e-6, 1e4, 0.0, 0)

    def call(**kw):
        a = list(ok)
        names = ["qh", "oh", "qd", "od", "b", "F", "H", "W", "heads", "hd", "gq", "gk", "eps", "theta",
                 "scale", "hc"]
        for k, v in kw.items():
            if k != "flags":
                a[names.index(k)] = v
        return lib.wan_dit_attn_host(*a, kw.get("flags", 0), None) if "flags" in kw else lib.wan_dit_attn_host(*a, 0, None)

    assert call(qh=None) == 1
    assert call(oh=None) == 1
    assert call(qd=None) == 1
    assert call(qd=FAKE + 8) == 2
    assert call(hd=64) == 4
    assert call(heads=0) == 3
    assert call(eps=0.0) == 5
    assert call(od=FAKE + 64) == 9  # out_dev overlaps qkv_dev
    assert call(hc=-1) == 5
    assert call(hc=5) == 5  # more than heads
    assert call(flags=2) == 5  # unknown flag
    assert call(b=5000, hc=1, od=2**40) == 3  # more pieces than the pipeline takes
    import torch
    if not torch.cuda.is_available():
        assert call() == 6  # valid arguments, no B200: fails loudly


def test_sparse_attention_validates_threshold(lib):
    # (qkv, out, batch, seq_len, heads, head_dim, scale, threshold)
    assert lib.wan_self_attention_sparse(FAKE, FAKE * 16, 1, 8, 1, 128, 0.0, -0.1, None) == 5
    assert lib.wan_self_attention_sparse(FAKE, FAKE * 16, 1, 8, 1, 128, 0.0, float("nan"), None) == 5
    # a weight is compared with the row's largest one: a threshold above 1 would drop the maximum
    assert lib.wan_self_attention_sparse(FAKE, FAKE * 16, 1, 8, 1, 128, 0.0, 1.0001, None) == 5
    assert lib.wan_self_attention_sparse(FAKE, FAKE * 16, 1, 8, 1, 128, 0.0, 2.0, None) == 5
    assert lib.wan_self_attention_sparse(FAKE, FAKE * 16, 1, 8, 1, 127, 0.0, 0.1, None) == 4
    assert lib.wan_self_attention_sparse(FAKE, FAKE + 64, 1, 8, 1, 128, 0.0, 0.1, None) == 9


def test_fp8_entry_points_validate(lib):
    # wan_quantize_fp8(qkv, qk8, v8t, batch, S, heads, head_dim, s_pitch, iq, ik, iv)
    far1, far2 = 2**40, 2**41
    assert lib.wan_quantize_fp8(None, far1, far2, 1, 8, 1, 128, 16, 1.0, 1.0, 1.0, None) == 1
    assert lib.wan_quantize_fp8(FAKE, far1 + 8, far2, 1, 8, 1, 128, 16, 1.0, 1.0, 1.0, None) == 2
    assert lib.wan_quantize_fp8(FAKE, far1, far2, 1, 20, 1, 128, 16, 1.0, 1.0, 1.0, None) == 3  # pitch < S
    assert lib.wan_quantize_fp8(FAKE, far1, far2, 1, 8, 1, 128, 24, 1.0, 1.0, 1.0, None) == 3  # pitch % 16
    assert lib.wan_quantize_fp8(FAKE, far1, far2, 1, 8, 1, 128, 16, 0.0, 1.0, 1.0, None) == 5
    assert lib.wan_quantize_fp8(FAKE, FAKE + 1024, far2, 1, 8, 1, 128, 16, 1.0, 1.0, 1.0, None) == 9
    # wan_self_attention_fp8(qk8, v8t, out, batch, S, heads, head_dim, s_pitch, scale, sq, sk, sv)
    assert lib.wan_self_attention_fp8(far1, far2, FAKE, 1, 8, 1, 64, 16, 0.0, 1.0, 1.0, 1.0, None) == 4
    assert lib.wan_self_attention_fp8(far1, far2, FAKE, 1, 8, 1, 128, 16, 0.0, -1.0, 1.0, 1.0, None) == 5
    assert lib.wan_self_attention_fp8(far1, far1 + 64, FAKE, 1, 8, 1, 128, 16, 0.0, 1.0, 1.0, 1.0, None) == 9
    assert lib.wan_qkv_amax(FAKE, 1, 8, 1, 128, None, None) == 1
    assert lib.wan_qkv_amax(FAKE, 1, 8, 1, 128, FAKE + 2, None) == 2
    import torch
    if not torch.cuda.is_available():
        assert lib.wan_self_attention_fp8(far1, far2, FAKE, 1, 8, 1, 128, 16, 0.0, 1.0, 1.0, 1.0, None) == 6


def test_linear_validates(lib):
    far = 2**40
    # (x, w, y, M, N, K, stats, stat_cols)
    assert lib.wan_linear(None, FAKE, far, 4, 256, 64, None, 0, None) == 1
    assert lib.wan_linear(FAKE + 4, FAKE, far, 4, 256, 64, None, 0, None) == 2
    assert lib.wan_linear(FAKE, FAKE, far, 4, 200, 64, None, 0, None) == 3   # N % 256
    assert lib.wan_linear(FAKE, FAKE, far, 4, 256, 100, None, 0, None) == 3  # K % 64
    assert lib.wan_linear(FAKE, FAKE, far, 4, 256, 64, 2**41, 512, None) == 3  # stat_cols > N
    assert lib.wan_linear(FAKE, FAKE, far, 4, 256, 64, 2**41 + 4, 256, None) == 2
    assert lib.wan_linear(FAKE, FAKE, FAKE + 64, 4, 256, 64, None, 0, None) == 9  # y overlaps x
    assert lib.wan_qk_norm_rope_stats(FAKE, 1, 2, 2, 2, 2, 128, FAKE, FAKE, 1e-6, 1e4, None, None) == 1
    assert lib.wan_qk_norm_rope_stats(FAKE, 1, 2, 2, 2, 1, 128, FAKE, FAKE, 1e-6, 1e4, 2**41, None) == 3  # D=128
    import torch
    if not torch.cuda.is_available():
        assert lib.wan_linear(FAKE, FAKE, far, 4, 256, 64, None, 0, None) == 6


def test_ring_entry_points_validate(lib):
    far1, far2, far3 = 2**40, 2**41, 2**42
    # wan_self_attention_partial(q, Sq, q_row0, q_rows, kv, kv_rows, kv_pitch, k_row0, k_rows, o, ml, B, heads, hd, scale)
    ok = (FAKE, 8, 0, 8, far1, 8, 256, 0, 8, far2, far3, 1, 1, 128, 0.0, None)
    def call(**kw):
        a = list(ok)
        names = ["q", "Sq", "q0", "qn", "kv", "kvr", "pitch", "k0", "kn", "o", "ml", "B", "h", "hd", "sc", "st"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return lib.wan_self_attention_partial(*a)
    assert call(q=None) == 1 and call(o=None) == 1
    assert call(ml=far3 + 8) == 2
    assert call(hd=64) == 4
    assert call(q0=4, qn=5) == 3              # query rows past Sq
    assert call(k0=1, kn=8) == 3              # keys past kv_rows
    assert call(kn=0) == 3
    assert call(pitch=128) == 3               # narrower than K|V
    assert call(pitch=260) == 3               # rows not whole 16-byte units
    assert call(sc=float("inf")) == 5
    assert call(o=FAKE + 16) == 9             # o overlaps q
    assert call(ml=far2 + 64) == 9            # ml overlaps o
    # the accumulating form validates like the partial one
    acc_args = list(ok)
    assert lib.wan_self_attention_accumulate(*acc_args[:9], None, *acc_args[10:]) == 1
    acc_args[13] = 64
    assert lib.wan_self_attention_accumulate(*acc_args) == 4
    # wan_attention_merge(o_acc, ml_acc, o_part, ml_part, out, n_units, head_dim)
    assert lib.wan_attention_merge(far1, far2, None, None, None, 4, 128, None) == 1  # nothing to do
    assert lib.wan_attention_merge(far1, far2, far3, None, None, 4, 128, None) == 1  # o_part without ml_part
    assert lib.wan_attention_merge(far1, far2, None, None, far3, 4, 64, None) == 4
    assert lib.wan_attention_merge(far1, far2, None, None, far3, 0, 128, None) == 3
    assert lib.wan_attention_merge(far1 + 8, far2, None, None, far3, 4, 128, None) == 2
    assert lib.wan_attention_merge(far1, far1 + 256, None, None, far3, 4, 128, None) == 9  # ml in o
    assert lib.wan_attention_merge(far1, far2, None, None, far1 + 1024, 4, 128, None) == 9  # out in o
    import torch
    if not torch.cuda.is_available():
        assert call() == 6
        assert lib.wan_attention_merge(far1, far2, None, None, far3, 4, 128, None) == 6


def test_sequence_shard_entry_points_validate(lib):
    # wan_qk_norm_rope_shard(qkv, batch, F, H, W, s0, s_local, heads, head_dim, gq, gk, eps, theta)
    assert lib.wan_qk_norm_rope_shard(FAKE, 1, 2, 2, 2, 4, 5, 1, 128, FAKE, FAKE, 1e-6, 1e4, None) == 3
    assert lib.wan_qk_norm_rope_shard(FAKE, 1, 2, 2, 2, -1, 4, 1, 128, FAKE, FAKE, 1e-6, 1e4, None) == 3
    assert lib.wan_qk_norm_rope_shard(None, 1, 2, 2, 2, 0, 4, 1, 128, FAKE, FAKE, 1e-6, 1e4, None) == 1
    # wan_self_attention_rows(qkv, out, batch, S, heads, head_dim, q_row0, q_rows, scale)
    assert lib.wan_self_attention_rows(FAKE, 2**40, 1, 8, 1, 128, 6, 3, 0.0, None) == 3
    assert lib.wan_self_attention_rows(FAKE, 2**40, 1, 8, 1, 128, 0, 0, 0.0, None) == 3
    assert lib.wan_self_attention_rows(FAKE, FAKE + 64, 1, 8, 1, 128, 0, 4, 0.0, None) == 9


C_CALLER = r"""
#include <stdio.h>
#include "wan_attn.h"

int main(void) {
  int32_t s;
  printf("abi %d\n", (int)wan_abi_version());
  for (s = 0; s <= 13; ++s) printf("status %d %s\n", (int)s, wan_status_string(s));
  /* argument errors are reported before any CUDA call */
  printf("null %d\n", (int)wan_qk_norm_rope(NULL, 1, 1, 1, 1, 1, 128, NULL, NULL, 1e-6f, 1e4f, NULL));
  printf("head_dim %d\n", (int)wan_self_attention((const void*)16, (void*)4096, 1, 1, 1, 64, 0.f, NULL));
  return 0;
}
"""


def test_header_compiles_as_c_and_links(lib, tmp_path):
    """A plain C99 caller: the header compiles with warnings as errors, the
    program links against the library, and the calls that need no GPU answer
    (ABI version, status text, argument validation)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(wan.library_path())
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(wan.library_path()),
                    "-Wl,-rpath," + libdir], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    assert out[0] == f"abi {lib.wan_abi_version()}"
    texts = [line.split(" ", 2)[2] for line in out[1:15]]
    assert all(texts) and len(set(texts)) == 14
    assert out[15] == "null 1"          # WAN_ERR_NULL
    assert out[16] == "head_dim 4"      # WAN_ERR_HEAD_DIM


def test_build_refuses_a_split_register_kernel_with_another_register_count():
    """The per-warpgroup register split is only valid at the register count
    the source names: a ptxas report with another count fails the build."""
    name = "_ZN3wan44_GLOBAL__N__fa96f1d5_11_attn_fwd_cu_a33b3c8a15attn_fwd_kernelILb0ELb0EEEv14CUtensorMap_st"
    fp8 = "_ZN3wan45_GLOBAL__N__2abe_12_attn_fwd_fp8_cu_2abe942719attn_fwd_fp8_kernelE14CUtensorMap_st"
    import re as _re
    want = {src: int(_re.search(r"constexpr int kLaunchRegs = (\d+);", open(os.path.join(wan_build.CSRC, src)).read()).group(1))
            for src, _ in wan_build.SPLIT_REGISTER_KERNELS
            if _re.search(r"constexpr int kLaunchRegs", open(os.path.join(wan_build.CSRC, src)).read())}
    good = (f"ptxas info    : Compiling entry function '{name}' for 'sm_100a'\n"
            f"ptxas info    : Used {want.get('attn_fwd.cu', 168)} registers, used 1 barriers\n"
            f"ptxas info    : Compiling entry function '{fp8}' for 'sm_100a'\n"
            f"ptxas info    : Used {want.get('attn_fwd_fp8.cu', 168)} registers, used 1 barriers\n")
    wan_build.check_register_splits(good)
    bad = good.replace(f"Used {want.get('attn_fwd_fp8.cu', 168)} registers", "Used 170 registers")
    with pytest.raises(RuntimeError, match="kLaunchRegs"):
        wan_build.check_register_splits(bad)
