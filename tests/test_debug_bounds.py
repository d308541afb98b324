"""The debug-bounds build (device-side index checks, debug_bounds.cuh) on
the CPU: the check and its fault record, compiled as host code, against
hand-worked cases; and the libraries' wan_debug_bounds entry point (the
release build reports itself disabled without touching a device, the debug
build reports itself enabled)."""
import ctypes
import os
import subprocess

import pytest

from video_diffusion_transformer_packed_b200 import build as wan_build

CSRC = os.path.join(wan_build.PKG, "csrc")

PROGRAM = r'''
#include <cstdio>
#include "debug_bounds.cuh"
using namespace wan::bounds;
int main() {
  unsigned long long w[2] = {0ull, 0ull};
  // in range: [0, 8) and [56, 64) of 64; an empty range at the end
  const int a = check(w, kNormStore, 0, 8, 64), b = check(w, kNormStore, 56, 8, 64), c = check(w, kNormStore, 64, 0, 64);
  // out of range: one past the end, a negative offset, an offset past the end
  const int d = check(w, kAttnOut, 57, 8, 64);
  const unsigned long long first = w[0];
  const int e = check(w, kGemmY, -16, 8, 64), f = check(w, kMergeOut, 1ll << 40, 1, 64);
  printf("%d %d %d %d %d %d\n", a, b, c, d, e, f);
  printf("%llu %llu %llu\n", first, w[0], w[1]);
  printf("%u %lld %u %lld\n", site_of(encode(kGemmY, -16)), (long long)offset_of(encode(kGemmY, -16)),
         site_of(encode(kMergeOut, (1ll << 40) + 3)), (long long)offset_of(encode(kMergeOut, (1ll << 40) + 3)));
  return 0;
}
'''


def test_check_records_the_first_failure_and_counts_all(tmp_path):
    src = tmp_path / "bounds_check.cu"
    src.write_text(PROGRAM)
    exe = tmp_path / "bounds_check"
    subprocess.run([wan_build.nvcc(), "-std=c++17", "-DWAN_DEBUG_BOUNDS", "-I", CSRC, str(src), "-o", str(exe)],
                   check=True, capture_output=True)
    lines = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    assert lines[0].split() == ["1", "1", "1", "0", "0", "0"]
    first, kept, count = (int(x) for x in lines[1].split())
    # site kAttnOut = 7 in the high byte, offset 57 below; later failures keep it
    assert first == (7 << 56) | 57 and kept == first and count == 3
    # the 56-bit offset field round-trips negative and large offsets
    assert lines[2].split() == ["16", "-16", "20", str((1 << 40) + 3)]


def _call(lib_path):
    lib = ctypes.CDLL(lib_path)
    lib.wan_debug_bounds.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32),
                                     ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64)]
    lib.wan_debug_bounds.restype = ctypes.c_int32
    en, first, count = ctypes.c_int32(-1), ctypes.c_uint64(9), ctypes.c_uint64(9)
    st = lib.wan_debug_bounds(None, ctypes.byref(en), ctypes.byref(first), ctypes.byref(count))
    assert lib.wan_debug_bounds(None, None, ctypes.byref(first), ctypes.byref(count)) == 1  # WAN_ERR_NULL
    return st, en.value, first.value, count.value


def test_release_library_reports_disabled_without_a_device():
    st, en, first, count = _call(wan_build.build())
    assert (st, en, first, count) == (0, 0, 0, 0)


def test_debug_library_is_built_with_the_checks():
    st, en, first, count = _call(wan_build.build(debug_bounds=True))
    assert en == 1
    # no device here: the synchronisation fails (WAN_ERR_LAUNCH); with one, nothing was launched yet
    assert st in (0, 7) and first == 0 and count == 0
