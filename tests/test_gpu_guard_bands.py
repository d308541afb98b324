"""Guard bands: every buffer a kernel writes sits inside a larger allocation
whose 4 KB before and after it are filled with a byte pattern, and the pattern
must be intact after the call. This checks the writes themselves against the
caller's buffers (the debug-bounds build checks the kernels' index arithmetic
against the extents they derive); the shapes are ragged so that tails, partial
tiles and the last rows of a batch are written."""
import ctypes

import pytest
import torch

import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import build as wan_build

pytestmark = pytest.mark.gpu

GUARD = 4096  # bytes on each side
PATTERN = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


class Guarded:
    """A tensor of `shape` and `dtype` in the middle of a pattern-filled allocation."""

    def __init__(self, shape, dtype, fill=None):
        self.shape, self.dtype = tuple(shape), dtype
        esize = torch.tensor([], dtype=dtype).element_size()
        n = 1
        for s in shape:
            n *= s
        self.nbytes = n * esize
        self.raw = torch.full((GUARD + self.nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + self.nbytes].view(dtype).view(self.shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self):
        torch.cuda.synchronize()
        return bool((self.raw[:GUARD] == PATTERN).all()) and bool((self.raw[GUARD + self.nbytes:] == PATTERN).all())


def _case(grid, heads, batch, seed):
    w = wi.Workload("guard", batch, grid, heads)
    return w, wi.inputs_for(w, seed=seed)


@pytest.mark.parametrize("grid,heads,batch", [((3, 5, 7), 2, 2), ((1, 1, 1), 1, 1), ((2, 9, 15), 3, 1)])
def test_norm_rope_writes_only_its_buffer(grid, heads, batch):
    w, (qkv, gq, gk) = _case(grid, heads, batch, seed=1)
    buf = Guarded(qkv.shape, torch.bfloat16, qkv.cuda())
    wan.qk_norm_rope(buf.t, grid, heads, gq.cuda(), gk.cuda())
    assert buf.intact()
    assert wan.device_error() == 0


@pytest.mark.parametrize("S,heads,batch", [(1, 1, 1), (130, 2, 2), (300, 3, 1)])
def test_attention_writes_only_out(S, heads, batch):
    qkv = wi.packed_qkv(batch, S, heads, seed=S).cuda()
    out = Guarded((batch, S, heads * 128), torch.bfloat16)
    wan.self_attention(qkv, heads, out=out.t)
    assert out.intact()
    q_rows = min(37, S)
    rows = Guarded((batch, q_rows, heads * 128), torch.bfloat16)
    wan.self_attention_rows(qkv, heads, S - q_rows, q_rows, out=rows.t)
    assert rows.intact()
    sparse = Guarded((batch, S, heads * 128), torch.bfloat16)
    wan.self_attention_sparse(qkv, heads, 0.05, out=sparse.t)
    assert sparse.intact()
    assert wan.device_error() == 0


def test_partial_state_and_merge_write_only_their_buffers():
    B, S, heads = 2, 300, 2
    qkv = wi.packed_qkv(B, S, heads, seed=7).cuda()
    o = Guarded((B, S, heads, 128), torch.float32)
    ml = Guarded((B, S, heads, 2), torch.float32)
    wan.self_attention_partial(qkv, heads, qkv, k_row0=0, k_rows=170, o=o.t, ml=ml.t)
    o2 = Guarded((B, S, heads, 128), torch.float32)
    ml2 = Guarded((B, S, heads, 2), torch.float32)
    wan.self_attention_partial(qkv, heads, qkv, k_row0=170, k_rows=130, o=o2.t, ml=ml2.t)
    wan.attention_merge(o.t, ml.t, o2.t, ml2.t)
    out = Guarded((B, S, heads * 128), torch.bfloat16)
    wan.attention_merge(o.t, ml.t, finalize=True, out=out.t)
    o3 = Guarded((B, S, heads, 128), torch.float32)
    ml3 = Guarded((B, S, heads, 2), torch.float32)
    wan.self_attention_partial(qkv, heads, qkv, k_row0=0, k_rows=170, o=o3.t, ml=ml3.t)
    wan.self_attention_partial(qkv, heads, qkv, k_row0=170, k_rows=130, o=o3.t, ml=ml3.t, accumulate=True)
    assert all(g.intact() for g in (o, ml, o2, ml2, out, o3, ml3))
    assert wan.device_error() == 0


def test_fp8_path_writes_only_its_buffers():
    B, S, heads = 2, 200, 2
    qkv = wi.packed_qkv(B, S, heads, seed=3).cuda()
    pitch = wan.fp8_pitch(S)
    qk8 = Guarded((B, S, 2 * heads * 128), torch.uint8)
    v8t = Guarded((B, heads, 128, pitch), torch.uint8)
    wan.quantize_fp8(qkv, heads, (100.0, 100.0, 100.0), qk8=qk8.t, v8t=v8t.t)
    out = Guarded((B, S, heads * 128), torch.bfloat16)
    wan.self_attention_fp8(qk8.t, v8t.t, heads, (0.01, 0.01, 0.01), out=out.t)
    assert qk8.intact() and v8t.intact() and out.intact()
    assert wan.device_error() == 0


@pytest.mark.parametrize("M,N,K", [(257, 512, 128), (1, 256, 64)])
def test_linear_writes_only_y_and_its_statistics(M, N, K):
    g = torch.Generator().manual_seed(M)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16).cuda()
    y = Guarded((M, N), torch.bfloat16)
    st = Guarded((M, N // 256), torch.float64)
    lib = wan.load_library()
    status = lib.wan_linear(x.data_ptr(), w.data_ptr(), y.t.data_ptr(), M, N, K, st.t.data_ptr(), N,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == 0
    assert y.intact() and st.intact()
    assert wan.device_error() == 0
