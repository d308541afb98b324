"""Wan2.2 DiT self-attention hot path for B200 (sm_100a): Python binding.

A thin ctypes layer over the C ABI in ``include/wan_attn.h`` (library
``_lib/libwanattn.so``, built by ``python -m video_diffusion_transformer_packed_b200.build``).
It only marshals arguments -- tensor pointers, sizes and the current CUDA
stream -- and turns a nonzero status into ``WanError``. Every step of the
path runs in the library's kernels; there is no other implementation here,
and a missing library is an error, not a fallback.

    qk_norm_rope(qkv, grid, heads, gamma_q, gamma_k)   # in place on qkv
    out = self_attention(qkv, heads)
    out = dit_attn(qkv, grid, heads, gamma_q, gamma_k)   # both, chained
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

__all__ = ["WanError", "load_library", "library_path", "qk_norm_rope", "self_attention",
           "self_attention_sparse", "skip_stats", "qkv_amax", "quantize_fp8", "self_attention_fp8",
           "fp8_pitch", "linear", "qk_norm_rope_stats", "qk_norm_rope_shard", "self_attention_rows", "dit_attn", "dit_attn_host", "device_error", "selftest_wait_timeout", "HEAD_DIM", "EPS",
           "THETA", "STATUS"]

HEAD_DIM = 128
EPS = 1e-6
THETA = 10000.0
STATUS = {0: "WAN_OK", 1: "WAN_ERR_NULL", 2: "WAN_ERR_ALIGN", 3: "WAN_ERR_SHAPE",
          4: "WAN_ERR_HEAD_DIM", 5: "WAN_ERR_PARAM", 6: "WAN_ERR_UNSUPPORTED_DEVICE",
          7: "WAN_ERR_LAUNCH", 8: "WAN_ERR_DEVICE_TIMEOUT", 9: "WAN_ERR_ALIAS",
          10: "WAN_ERR_MEMORY_KIND", 11: "WAN_ERR_KERNEL_IMAGE", 12: "WAN_ERR_TOO_LARGE",
          13: "WAN_ERR_BOUNDS"}

_HERE = os.path.dirname(os.path.abspath(__file__))
# WAN_DEBUG_BOUNDS=1 in the environment selects the debug-bounds build
# (device-side index checks; see debug_bounds()), built by
# `python -m video_diffusion_transformer_packed_b200.build --debug-bounds`.
_LIB_PATH = os.path.join(_HERE, "_lib", "libwanattn_debug.so" if os.environ.get("WAN_DEBUG_BOUNDS") == "1"
                         else "libwanattn.so")
_lib = None
_lock = threading.Lock()


class WanError(RuntimeError):
    """A nonzero wan_status from the library."""

    def __init__(self, status: int, where: str):
        self.status = status
        msg = load_library().wan_status_string(status).decode()
        super().__init__(f"{where}: {STATUS.get(status, status)} ({msg})")


def library_path() -> str:
    return _LIB_PATH


def load_library() -> ctypes.CDLL:
    """Load libwanattn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                                   "`python -m video_diffusion_transformer_packed_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            P, I64, I32, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
            lib.wan_status_string.argtypes = [I32]
            lib.wan_status_string.restype = ctypes.c_char_p
            lib.wan_abi_version.argtypes = []
            lib.wan_abi_version.restype = I32
            lib.wan_qk_norm_rope.argtypes = [P, I64, I32, I32, I32, I32, I32, P, P, F, F, P]
            lib.wan_qk_norm_rope.restype = I32
            lib.wan_self_attention.argtypes = [P, P, I64, I64, I32, I32, F, P]
            lib.wan_self_attention.restype = I32
            lib.wan_dit_attn.argtypes = [P, P, I64, I32, I32, I32, I32, I32, P, P, F, F, F, P]
            lib.wan_dit_attn.restype = I32
            lib.wan_device_error.argtypes = [P, ctypes.POINTER(I32)]
            lib.wan_device_error.restype = I32
            lib.wan_selftest_wait_timeout.argtypes = [P, P, I64, I64, I32, I32, I64, P]
            lib.wan_selftest_wait_timeout.restype = I32
            lib.wan_dit_attn_host.argtypes = [P, P, P, P, I64, I32, I32, I32, I32, I32, P, P, F, F, F,
                                              I32, I32, P]
            lib.wan_dit_attn_host.restype = I32
            lib.wan_self_attention_sparse.argtypes = [P, P, I64, I64, I32, I32, F, F, P]
            lib.wan_self_attention_sparse.restype = I32
            lib.wan_skip_stats.argtypes = [P, ctypes.POINTER(I64), ctypes.POINTER(I64)]
            lib.wan_skip_stats.restype = I32
            lib.wan_qkv_amax.argtypes = [P, I64, I64, I32, I32, P, P]
            lib.wan_qkv_amax.restype = I32
            lib.wan_quantize_fp8.argtypes = [P, P, P, I64, I64, I32, I32, I64, F, F, F, P]
            lib.wan_quantize_fp8.restype = I32
            lib.wan_self_attention_fp8.argtypes = [P, P, P, I64, I64, I32, I32, I64, F, F, F, F, P]
            lib.wan_self_attention_fp8.restype = I32
            lib.wan_linear.argtypes = [P, P, P, I64, I64, I64, P, I64, P]
            lib.wan_linear.restype = I32
            lib.wan_qk_norm_rope_stats.argtypes = [P, I64, I32, I32, I32, I32, I32, P, P, F, F, P, P]
            lib.wan_qk_norm_rope_stats.restype = I32
            lib.wan_qk_norm_rope_shard.argtypes = [P, I64, I32, I32, I32, I64, I64, I32, I32, P, P, F, F, P]
            lib.wan_qk_norm_rope_shard.restype = I32
            lib.wan_self_attention_rows.argtypes = [P, P, I64, I64, I32, I32, I64, I64, F, P]
            lib.wan_self_attention_rows.restype = I32
            lib.wan_self_attention_partial.argtypes = [P, I64, I64, I64, P, I64, I64, I64, I64, P, P, I64, I32,
                                                       I32, F, P]
            lib.wan_self_attention_partial.restype = I32
            lib.wan_self_attention_accumulate.argtypes = lib.wan_self_attention_partial.argtypes
            lib.wan_self_attention_accumulate.restype = I32
            lib.wan_attention_merge.argtypes = [P, P, P, P, P, I64, I32, P]
            lib.wan_attention_merge.restype = I32
            lib.wan_dit_attn_host_static.argtypes = [P, P, I64, I32, I32, I32, I32, I32, P, P, F, F, F, I32, I32, P]
            lib.wan_dit_attn_host_static.restype = I32
            lib.wan_debug_bounds.argtypes = [P, ctypes.POINTER(I32), ctypes.POINTER(ctypes.c_uint64),
                                             ctypes.POINTER(ctypes.c_uint64)]
            lib.wan_debug_bounds.restype = I32
            _lib = lib
    return _lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise WanError(status, where)


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _on_stream(stream, device):
    """Context that makes `stream` (a torch stream, an object with a
    `cuda_stream` handle, a raw cudaStream_t, or None for the current stream)
    torch's current stream on `device`."""
    import contextlib
    import torch
    if stream is None:
        return contextlib.nullcontext()
    if not isinstance(stream, torch.cuda.Stream):
        stream = torch.cuda.ExternalStream(_stream(stream), device=device)
    return torch.cuda.stream(stream)


def _check_packed(qkv, heads: int, grid=None) -> None:
    """Shapes the C ABI cannot see (it takes raw pointers): refuse mismatches
    here, before anything is launched."""
    if qkv.dim() != 3 or qkv.shape[2] != 3 * heads * HEAD_DIM:
        raise ValueError(f"qkv must be [B, S, 3*heads*{HEAD_DIM}], got {tuple(qkv.shape)}")
    if grid is not None and grid[0] * grid[1] * grid[2] != qkv.shape[1]:
        raise ValueError(f"grid {tuple(grid)} has {grid[0] * grid[1] * grid[2]} tokens, "
                         f"qkv has {qkv.shape[1]}")


def _check_out(out, qkv, heads: int) -> None:
    if tuple(out.shape) != (qkv.shape[0], qkv.shape[1], heads * HEAD_DIM):
        raise ValueError(f"out must be [B, S, heads*{HEAD_DIM}], got {tuple(out.shape)}")


def _check_gamma(g, heads: int, name: str) -> None:
    if g.numel() != heads * HEAD_DIM:
        raise ValueError(f"{name} must have heads*{HEAD_DIM} elements, got {g.numel()}")


def _bf16_cuda(t, name: str) -> int:
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous bfloat16 CUDA tensor")
    return t.data_ptr()


def qk_norm_rope(qkv, grid: Sequence[int], heads: int, gamma_q, gamma_k, eps: float = EPS,
                 theta: float = THETA, stream=None):
    """Q/K RMSNorm + bf16 round + 3D RoPE in place on packed qkv [B, F*H*W, 3*heads*128].
    Within 1 bf16 ulp of the exact definition for finite inputs with |x| < 2^64
    and |x * gamma| < 2^128 (the kernel forms squares and gamma products exactly
    in fp32; larger magnitudes overflow there)."""
    F, H, W = grid
    B = qkv.shape[0]
    _check_packed(qkv, heads, grid)
    _check_gamma(gamma_q, heads, "gamma_q")
    _check_gamma(gamma_k, heads, "gamma_k")
    _check(load_library().wan_qk_norm_rope(_bf16_cuda(qkv, "qkv"), B, F, H, W, heads, HEAD_DIM,
                                           _bf16_cuda(gamma_q, "gamma_q"),
                                           _bf16_cuda(gamma_k, "gamma_k"), eps, theta,
                                           _stream(stream)), "wan_qk_norm_rope")
    return qkv


def self_attention(qkv, heads: int, out=None, scale: float = 0.0, stream=None):
    """Softmax attention over packed qkv [B, S, 3*heads*128] -> out [B, S, heads*128]."""
    import torch
    _check_packed(qkv, heads)
    B, S, _ = qkv.shape
    if out is None:
        out = torch.empty((B, S, heads * HEAD_DIM), dtype=torch.bfloat16, device=qkv.device)
    _check_out(out, qkv, heads)
    _check(load_library().wan_self_attention(_bf16_cuda(qkv, "qkv"), _bf16_cuda(out, "out"), B, S,
                                             heads, HEAD_DIM, scale, _stream(stream)),
           "wan_self_attention")
    return out


def self_attention_sparse(qkv, heads: int, threshold: float, out=None, scale: float = 0.0, stream=None):
    """Softmax attention with Skip-Softmax in threshold mode (0 = dense)."""
    import torch
    _check_packed(qkv, heads)
    B, S, _ = qkv.shape
    if out is None:
        out = torch.empty((B, S, heads * HEAD_DIM), dtype=torch.bfloat16, device=qkv.device)
    _check_out(out, qkv, heads)
    _check(load_library().wan_self_attention_sparse(_bf16_cuda(qkv, "qkv"), _bf16_cuda(out, "out"), B, S,
                                                    heads, HEAD_DIM, scale, float(threshold),
                                                    _stream(stream)), "wan_self_attention_sparse")
    return out


def skip_stats(stream=None):
    """Synchronise; return and clear (group-tiles skipped, P V products skipped)."""
    g, p = ctypes.c_int64(0), ctypes.c_int64(0)
    _check(load_library().wan_skip_stats(_stream(stream), ctypes.byref(g), ctypes.byref(p)), "wan_skip_stats")
    return g.value, p.value


E4M3_MAX = 448.0


def _u8_cuda(t, name: str) -> int:
    import torch
    if t.dtype != torch.uint8 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous uint8 CUDA tensor")
    return t.data_ptr()


def qkv_amax(qkv, heads: int, stream=None):
    """max |x| of Q, K and V of a packed bf16 buffer: float32 CUDA tensor [3],
    written asynchronously on `stream` (synchronise it before reading)."""
    import torch
    _check_packed(qkv, heads)
    B, S, _ = qkv.shape
    amax = torch.empty(3, dtype=torch.float32, device=qkv.device)
    _check(load_library().wan_qkv_amax(_bf16_cuda(qkv, "qkv"), B, S, heads, HEAD_DIM, amax.data_ptr(),
                                       _stream(stream)), "wan_qkv_amax")
    return amax


def fp8_pitch(seq_len: int) -> int:
    return (seq_len + 15) // 16 * 16


def quantize_fp8(qkv, heads: int, inv_scales, qk8=None, v8t=None, stream=None):
    """e4m3 codes of a packed bf16 buffer: (qk8 [B, S, 2*heads*128],
    v8t [B, heads, 128, s_pitch]) with codes e4m3(fl32(x * inv_scale))."""
    import torch
    _check_packed(qkv, heads)
    B, S, _ = qkv.shape
    pitch = fp8_pitch(S)
    if qk8 is None:
        qk8 = torch.empty((B, S, 2 * heads * HEAD_DIM), dtype=torch.uint8, device=qkv.device)
    if v8t is None:
        v8t = torch.empty((B, heads, HEAD_DIM, pitch), dtype=torch.uint8, device=qkv.device)
    if tuple(qk8.shape) != (B, S, 2 * heads * HEAD_DIM) or v8t.dim() != 4 or tuple(v8t.shape[:3]) != (B, heads, HEAD_DIM):
        raise ValueError("qk8 must be [B, S, 2*heads*128] and v8t [B, heads, 128, s_pitch]")
    iq, ik, iv = (float(x) for x in inv_scales)
    _check(load_library().wan_quantize_fp8(_bf16_cuda(qkv, "qkv"), _u8_cuda(qk8, "qk8"), _u8_cuda(v8t, "v8t"), B, S,
                                           heads, HEAD_DIM, v8t.shape[3], iq, ik, iv, _stream(stream)),
           "wan_quantize_fp8")
    return qk8, v8t


def self_attention_fp8(qk8, v8t, heads: int, scales, out=None, scale: float = 0.0, stream=None):
    """FP8 attention on e4m3 codes (quantize_fp8) dequantised with `scales`
    (scale_q, scale_k, scale_v): out bf16 [B, S, heads*128]."""
    import torch
    B, S, d2 = qk8.shape
    if d2 != 2 * heads * HEAD_DIM or v8t.dim() != 4 or tuple(v8t.shape[:3]) != (B, heads, HEAD_DIM):
        raise ValueError("qk8 must be [B, S, 2*heads*128] and v8t [B, heads, 128, s_pitch]")
    if out is None:
        out = torch.empty((B, S, heads * HEAD_DIM), dtype=torch.bfloat16, device=qk8.device)
    if tuple(out.shape) != (B, S, heads * HEAD_DIM):
        raise ValueError("out must be [B, S, heads*128]")
    sq, sk, sv = (float(x) for x in scales)
    _check(load_library().wan_self_attention_fp8(_u8_cuda(qk8, "qk8"), _u8_cuda(v8t, "v8t"), _bf16_cuda(out, "out"),
                                                 B, S, heads, HEAD_DIM, v8t.shape[3], scale, sq, sk, sv,
                                                 _stream(stream)), "wan_self_attention_fp8")
    return out


def linear(x, w, y=None, stat_cols: int = 0, stream=None):
    """Y = X W^T (bf16, fp32 accumulation) for X [..., K] and W [N, K]; with
    stat_cols > 0 also returns the fp64 sums of squares of the bf16 outputs per
    row and 256-column tile of the first stat_cols columns: (y, stats) with
    stats [M, stat_cols // 256], else (y, None)."""
    import torch
    K = x.shape[-1]
    M = x.numel() // K
    N = w.shape[0]
    if w.dim() != 2 or w.shape[1] != K:
        raise ValueError(f"w must be [N, {K}], got {tuple(w.shape)}")
    if y is None:
        y = torch.empty((*x.shape[:-1], N), dtype=torch.bfloat16, device=x.device)
    if y.numel() != M * N:
        raise ValueError("y must hold M x N elements")
    stats = None
    if stat_cols:
        stats = torch.empty((M, stat_cols // 256), dtype=torch.float64, device=x.device)
    _check(load_library().wan_linear(_bf16_cuda(x, "x"), _bf16_cuda(w, "w"), _bf16_cuda(y, "y"), M, N, K,
                                     stats.data_ptr() if stats is not None else None, int(stat_cols),
                                     _stream(stream)), "wan_linear")
    return y, stats


def qk_norm_rope_stats(qkv, grid: Sequence[int], heads: int, gamma_q, gamma_k, stats, eps: float = EPS,
                       theta: float = THETA, stream=None):
    """qk_norm_rope taking each token's sums of squares from the QKV
    projection's statistics (linear(..., stat_cols=2*heads*128))."""
    import torch
    F, H, W = grid
    B = qkv.shape[0]
    _check_packed(qkv, heads, grid)
    _check_gamma(gamma_q, heads, "gamma_q")
    _check_gamma(gamma_k, heads, "gamma_k")
    if stats.dtype != torch.float64 or not stats.is_cuda or tuple(stats.shape) != (B * qkv.shape[1], 2 * heads * HEAD_DIM // 256):
        raise ValueError("stats must be float64 CUDA [B*S, 2*heads*128/256]")
    _check(load_library().wan_qk_norm_rope_stats(_bf16_cuda(qkv, "qkv"), B, F, H, W, heads, HEAD_DIM,
                                                 _bf16_cuda(gamma_q, "gamma_q"), _bf16_cuda(gamma_k, "gamma_k"),
                                                 eps, theta, stats.data_ptr(), _stream(stream)),
           "wan_qk_norm_rope_stats")
    return qkv


def qk_norm_rope_shard(qkv_local, grid: Sequence[int], heads: int, s0: int, gamma_q, gamma_k, eps: float = EPS,
                       theta: float = THETA, stream=None):
    """qk_norm_rope on a sequence shard: qkv_local [B, s_local, 3*heads*128]
    holds tokens [s0, s0 + s_local) of every batch element's grid."""
    F, H, W = grid
    B, S_l, d3 = qkv_local.shape
    if d3 != 3 * heads * HEAD_DIM:
        raise ValueError("qkv_local must be [B, s_local, 3*heads*128]")
    _check_gamma(gamma_q, heads, "gamma_q")
    _check_gamma(gamma_k, heads, "gamma_k")
    _check(load_library().wan_qk_norm_rope_shard(_bf16_cuda(qkv_local, "qkv_local"), B, F, H, W, int(s0), S_l,
                                                 heads, HEAD_DIM, _bf16_cuda(gamma_q, "gamma_q"),
                                                 _bf16_cuda(gamma_k, "gamma_k"), eps, theta, _stream(stream)),
           "wan_qk_norm_rope_shard")
    return qkv_local


def self_attention_rows(qkv, heads: int, q_row0: int, q_rows: int, out=None, scale: float = 0.0, stream=None):
    """Attention of query rows [q_row0, q_row0 + q_rows) of the full packed
    buffer against every key: out [B, q_rows, heads*128]."""
    import torch
    _check_packed(qkv, heads)
    B, S, _ = qkv.shape
    if out is None:
        out = torch.empty((B, q_rows, heads * HEAD_DIM), dtype=torch.bfloat16, device=qkv.device)
    if tuple(out.shape) != (B, q_rows, heads * HEAD_DIM):
        raise ValueError("out must be [B, q_rows, heads*128]")
    _check(load_library().wan_self_attention_rows(_bf16_cuda(qkv, "qkv"), _bf16_cuda(out, "out"), B, S, heads,
                                                  HEAD_DIM, int(q_row0), int(q_rows), scale, _stream(stream)),
           "wan_self_attention_rows")
    return out


def _f32_cuda(t, name: str) -> int:
    import torch
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
        raise TypeError(f"{name} must be a contiguous float32 CUDA tensor")
    return t.data_ptr()


def self_attention_partial(q_qkv, heads: int, kv, q_row0: int = 0, q_rows=None, k_row0: int = 0, k_rows=None,
                           o=None, ml=None, scale: float = 0.0, stream=None, accumulate: bool = False):
    """Softmax state of query rows [q_row0, q_row0 + q_rows) of the packed
    q_qkv [B, Sq, 3*heads*128] against keys [k_row0, k_row0 + k_rows) of kv
    [B, Skv, pitch] (K then V in its last 2*heads*128 columns: a packed QKV
    buffer or a K|V chunk). Returns (o [B, q_rows, heads, 128] fp32,
    ml [B, q_rows, heads, 2] fp32): O and (m, l) in base 2. With accumulate,
    o and ml must hold a state over other keys already, and the range's state
    is merged into them (wan_self_attention_accumulate)."""
    import torch
    _check_packed(q_qkv, heads)
    B, Sq, _ = q_qkv.shape
    if kv.dim() != 3 or kv.shape[0] != B or kv.shape[2] < 2 * heads * HEAD_DIM:
        raise ValueError("kv must be [B, Skv, pitch] with K and V in its last 2*heads*128 columns")
    q_rows = Sq - q_row0 if q_rows is None else q_rows
    k_rows = kv.shape[1] - k_row0 if k_rows is None else k_rows
    if o is None:
        o = torch.empty((B, q_rows, heads, HEAD_DIM), dtype=torch.float32, device=q_qkv.device)
    if ml is None:
        ml = torch.empty((B, q_rows, heads, 2), dtype=torch.float32, device=q_qkv.device)
    if tuple(o.shape) != (B, q_rows, heads, HEAD_DIM) or tuple(ml.shape) != (B, q_rows, heads, 2):
        raise ValueError("o must be [B, q_rows, heads, 128] and ml [B, q_rows, heads, 2]")
    if accumulate and (o is None or ml is None):
        raise ValueError("accumulate needs the state (o, ml) to merge into")
    fn = load_library().wan_self_attention_accumulate if accumulate else load_library().wan_self_attention_partial
    _check(fn(_bf16_cuda(q_qkv, "q_qkv"), Sq, int(q_row0), int(q_rows), _bf16_cuda(kv, "kv"), kv.shape[1],
              kv.shape[2], int(k_row0), int(k_rows), _f32_cuda(o, "o"), _f32_cuda(ml, "ml"), B, heads, HEAD_DIM,
              scale, _stream(stream)), "wan_self_attention_accumulate" if accumulate else "wan_self_attention_partial")
    return o, ml


def attention_merge(o_acc, ml_acc, o_part=None, ml_part=None, out=None, finalize: bool = False, stream=None):
    """(o_acc, ml_acc) := merge with (o_part, ml_part) when given; with
    finalize, also returns out = bf16(O / l) shaped like o_acc without its last
    axis split ([B, rows, heads*128] for o_acc [B, rows, heads, 128])."""
    import torch
    if o_acc.shape[-1] != HEAD_DIM or tuple(ml_acc.shape) != tuple(o_acc.shape[:-1]) + (2,):
        raise ValueError("o_acc must be [..., 128] and ml_acc [..., 2] over the same units")
    if (o_part is None) != (ml_part is None):
        raise ValueError("o_part and ml_part go together")
    if o_part is not None and (o_part.shape != o_acc.shape or ml_part.shape != ml_acc.shape):
        raise ValueError("the partial state must have the accumulator's shape")
    n_units = o_acc.numel() // HEAD_DIM
    if finalize and out is None:
        out = torch.empty(tuple(o_acc.shape[:-2]) + (o_acc.shape[-2] * HEAD_DIM,), dtype=torch.bfloat16,
                          device=o_acc.device)
    if out is not None and out.numel() != n_units * HEAD_DIM:
        raise ValueError("out must hold 128 values per unit")
    _check(load_library().wan_attention_merge(
        _f32_cuda(o_acc, "o_acc"), _f32_cuda(ml_acc, "ml_acc"),
        _f32_cuda(o_part, "o_part") if o_part is not None else None,
        _f32_cuda(ml_part, "ml_part") if ml_part is not None else None,
        _bf16_cuda(out, "out") if out is not None else None, n_units, HEAD_DIM, _stream(stream)),
        "wan_attention_merge")
    return out


def dit_attn(qkv, grid: Sequence[int], heads: int, gamma_q, gamma_k, out=None, eps: float = EPS,
             theta: float = THETA, scale: float = 0.0, stream=None):
    """qk_norm_rope (in place on qkv) then self_attention, chained on one stream."""
    import torch
    F, H, W = grid
    _check_packed(qkv, heads, grid)
    _check_gamma(gamma_q, heads, "gamma_q")
    _check_gamma(gamma_k, heads, "gamma_k")
    B, S, _ = qkv.shape
    if out is None:
        out = torch.empty((B, S, heads * HEAD_DIM), dtype=torch.bfloat16, device=qkv.device)
    _check_out(out, qkv, heads)
    _check(load_library().wan_dit_attn(_bf16_cuda(qkv, "qkv"), _bf16_cuda(out, "out"), B, F, H, W,
                                       heads, HEAD_DIM, _bf16_cuda(gamma_q, "gamma_q"),
                                       _bf16_cuda(gamma_k, "gamma_k"), eps, theta, scale,
                                       _stream(stream)), "wan_dit_attn")
    return out


def _bf16_pinned(t, name: str) -> int:
    import torch
    if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous() or not t.is_pinned():
        raise TypeError(f"{name} must be a contiguous bfloat16 tensor in page-locked host memory")
    return t.data_ptr()


def dit_attn_host(qkv_host, grid: Sequence[int], heads: int, gamma_q, gamma_k, out_host=None,
                  qkv_dev=None, out_dev=None, heads_per_chunk: int = 0, eps: float = EPS,
                  theta: float = THETA, scale: float = 0.0, overlap_input: bool = False, stream=None):
    """The step for packed qkv in page-locked host memory: host->device copies,
    qk_norm_rope, self_attention and the device->host copy of the output,
    overlapped chunk by chunk inside the library. qkv_dev / out_dev are the
    device buffers it runs through (allocated on the current device when not
    given); qkv_host is only read, asynchronously (the returned out_host keeps a
    reference to it until it is freed). Asynchronous on `stream`: synchronise
    it before reading out_host. overlap_input: the call does not wait for earlier
    work on `stream`; it still waits for earlier calls of this function that
    use the same device buffers (the caller guarantees nothing else does), so
    alternating two buffer sets overlaps one call's input transfer with the
    previous call's kernels."""
    import torch
    F, H, W = grid
    _check_packed(qkv_host, heads, grid)
    _check_gamma(gamma_q, heads, "gamma_q")
    _check_gamma(gamma_k, heads, "gamma_k")
    B, S, _ = qkv_host.shape
    dev = gamma_q.device
    if out_host is None:
        out_host = torch.empty((B, S, heads * HEAD_DIM), dtype=torch.bfloat16).pin_memory()
    # Device buffers made here are dropped when the call returns, while the
    # library's streams still use them. Allocated on the call's stream, which
    # the library makes wait for its last copy, torch's caching allocator
    # hands their memory out again only in that stream's order.
    with _on_stream(stream, dev):
        if qkv_dev is None:
            qkv_dev = torch.empty(qkv_host.shape, dtype=torch.bfloat16, device=dev)
        if out_dev is None:
            out_dev = torch.empty((B, S, heads * HEAD_DIM), dtype=torch.bfloat16, device=dev)
    _check_out(out_host, qkv_host, heads)
    _check_packed(qkv_dev, heads, grid)
    if tuple(qkv_dev.shape) != tuple(qkv_host.shape):
        raise ValueError("qkv_dev must have the shape of qkv_host")
    _check_out(out_dev, qkv_host, heads)
    _check(load_library().wan_dit_attn_host(_bf16_pinned(qkv_host, "qkv_host"),
                                            _bf16_pinned(out_host, "out_host"),
                                            _bf16_cuda(qkv_dev, "qkv_dev"), _bf16_cuda(out_dev, "out_dev"),
                                            B, F, H, W, heads, HEAD_DIM, _bf16_cuda(gamma_q, "gamma_q"),
                                            _bf16_cuda(gamma_k, "gamma_k"), eps, theta, scale,
                                            int(heads_per_chunk), 1 if overlap_input else 0, _stream(stream)),
           "wan_dit_attn_host")
    # The copies out of qkv_host run on the library's own streams, which
    # torch's pinned-memory cache does not see: a temporary qkv_host freed
    # now could be handed to another pin_memory() and overwritten while it
    # is still being read. The output keeps it alive.
    out_host._wan_source = qkv_host
    return out_host


def dit_attn_host_static(qkv_host, grid: Sequence[int], heads: int, gamma_q, gamma_k, out_host=None,
                         heads_per_chunk: int = 0, eps: float = EPS, theta: float = THETA, scale: float = 0.0,
                         overlap_input: bool = False, stream=None):
    """dit_attn_host through the library's own device buffer instead of caller
    buffers (for callers that cannot allocate device memory): nothing is
    allocated on the device; batch * S * heads * 128 must not exceed
    WAN_HOST_STATIC_MAX_ELEMENTS (8 Mi). Asynchronous on `stream`."""
    import torch
    F, H, W = grid
    _check_packed(qkv_host, heads, grid)
    _check_gamma(gamma_q, heads, "gamma_q")
    _check_gamma(gamma_k, heads, "gamma_k")
    B, S, _ = qkv_host.shape
    if out_host is None:
        out_host = torch.empty((B, S, heads * HEAD_DIM), dtype=torch.bfloat16).pin_memory()
    _check_out(out_host, qkv_host, heads)
    _check(load_library().wan_dit_attn_host_static(_bf16_pinned(qkv_host, "qkv_host"),
                                                   _bf16_pinned(out_host, "out_host"), B, F, H, W, heads,
                                                   HEAD_DIM, _bf16_cuda(gamma_q, "gamma_q"),
                                                   _bf16_cuda(gamma_k, "gamma_k"), eps, theta, scale,
                                                   int(heads_per_chunk), 1 if overlap_input else 0,
                                                   _stream(stream)), "wan_dit_attn_host_static")
    out_host._wan_source = qkv_host  # read asynchronously: see dit_attn_host
    return out_host


def selftest_wait_timeout(qkv, heads: int, out=None, wait_limit_ns: int = 20_000_000, stream=None):
    """Launch the attention kernel with its loads suppressed so that its bounded
    waits run out; read the outcome with device_error() (nonzero expected)."""
    import torch
    _check_packed(qkv, heads)
    B, S, _ = qkv.shape
    if out is None:
        out = torch.empty((B, S, heads * HEAD_DIM), dtype=torch.bfloat16, device=qkv.device)
    _check_out(out, qkv, heads)
    _check(load_library().wan_selftest_wait_timeout(_bf16_cuda(qkv, "qkv"), _bf16_cuda(out, "out"), B, S,
                                                    heads, HEAD_DIM, int(wait_limit_ns), _stream(stream)),
           "wan_selftest_wait_timeout")
    return out


def debug_bounds(stream=None):
    """Reads and clears the debug-bounds records (wan_debug_bounds): returns
    (enabled, count, site, offset) -- enabled is False for the release build,
    which records nothing and touches no device; site and offset name the
    first failed check (0, 0 when none failed)."""
    lib = load_library()
    handle = 0
    if stream is not None:
        handle = _stream(stream)
    else:
        import torch
        if torch.cuda.is_available():
            handle = _stream(None)
    en, first, count = ctypes.c_int32(0), ctypes.c_uint64(0), ctypes.c_uint64(0)
    st = lib.wan_debug_bounds(ctypes.c_void_p(handle), ctypes.byref(en), ctypes.byref(first), ctypes.byref(count))
    if st not in (0, 13):
        raise WanError(st, "wan_debug_bounds")
    rec = first.value
    off = rec & ((1 << 56) - 1)
    if off >= 1 << 55:
        off -= 1 << 56
    return bool(en.value), count.value, rec >> 56, off if rec else 0


def device_error(stream=None) -> int:
    """Synchronise and return (and clear) the attention kernel's device error word."""
    code = ctypes.c_int32(0)
    st = load_library().wan_device_error(_stream(stream), ctypes.byref(code))
    if st not in (0, 8):
        raise WanError(st, "wan_device_error")
    return code.value
