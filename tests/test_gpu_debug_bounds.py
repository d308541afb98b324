"""The GPU parity tests rerun against the debug-bounds build
(libwanattn_debug.so): every instrumented global- and shared-memory access of
every kernel checks its range against its buffer's extent, and each rerun test
must also leave no failed check behind (the conftest fixture asserts that under
WAN_DEBUG_BOUNDS=1). The rerun covers ragged tails, single tokens, batch and
head boundaries, sequence shards, partial states, the FP8 path and the
projection GEMM; the full-length cases are left to the release run."""
import os
import subprocess
import sys

import pytest

from video_diffusion_transformer_packed_b200 import build as wan_build

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
FILES = ["test_gpu_norm_rope.py", "test_gpu_attention.py", "test_gpu_skip_softmax.py", "test_gpu_fp8.py",
         "test_gpu_projection.py", "test_gpu_sp.py", "test_gpu_fused.py", "test_gpu_guard_bands.py"]


def test_parity_suite_passes_under_the_debug_bounds_build():
    wan_build.build(debug_bounds=True)
    env = dict(os.environ, WAN_DEBUG_BOUNDS="1")
    cmd = [sys.executable, "-m", "pytest", *[os.path.join(HERE, f) for f in FILES], "-m", "gpu", "-q", "-x",
           "-p", "no:cacheprovider", "-k", "not full_length"]
    res = subprocess.run(cmd, env=env, cwd=os.path.dirname(HERE), capture_output=True, text=True, timeout=2400)
    assert res.returncode == 0, res.stdout[-4000:] + res.stderr[-2000:]
    assert " passed" in res.stdout and " failed" not in res.stdout, res.stdout[-2000:]
