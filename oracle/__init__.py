"""fp64 CPU oracle for the Wan2.2 DiT self-attention path.

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the bench's
CPU-baseline leg may import this; the product path never does. The arithmetic
lives in ``wan_oracle.c`` (plain C, fp64, OpenMP over independent rows); this
module builds it with gcc and marshals arrays through ctypes.

bf16 tensors are exchanged as torch.bfloat16 tensors (their bit patterns are
handed to C as uint16).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "wan_oracle.c")
LIB = os.path.join(HERE, "_build", "libwan_oracle.so")
HEAD_DIM = 128
SPLIT = (44, 42, 42)

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (gcc, fp64, strict IEEE: no fast-math, no contraction)."""
    os.makedirs(os.path.dirname(LIB), exist_ok=True)
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-ffp-contract=off", "-fno-fast-math", SRC, "-o", tmp, "-lm"])
        os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P, I64, I32, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
            lib.wan_oracle_round_bf16.argtypes = [D]
            lib.wan_oracle_round_bf16.restype = D
            lib.wan_oracle_f64_to_bf16.argtypes = [P, P, I64]
            lib.wan_oracle_rmsnorm.argtypes = [P, I64, I64, I64, P, D, P]
            lib.wan_oracle_rope.argtypes = [P, I64, I64, I32, I32, I32, D, P, I32]
            lib.wan_oracle_qk_norm_rope.argtypes = [P, P, I64, I32, I32, I32, I32, P, P, D, D]
            lib.wan_oracle_qk_norm_rope_tokens.argtypes = [P, I64, I32, I32, I32, I32, P, P, D, D,
                                                           P, I64, P]
            lib.wan_oracle_attention_rows.argtypes = [P, I64, I64, I32, D, P, I64, P]
            lib.wan_oracle_attention_partial_rows.argtypes = [P, I64, P, I64, I64, I64, I64, I32, D, P, I64, P, P]
            lib.wan_oracle_attention_skip_groups.argtypes = [P, I64, I64, I32, D, D, P, I64, P, P, P]
            lib.wan_oracle_e4m3_encode.argtypes = [D]
            lib.wan_oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.wan_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.wan_oracle_e4m3_decode.restype = D
            lib.wan_oracle_quantize_e4m3.argtypes = [P, I64, ctypes.c_float, P]
            lib.wan_oracle_attention_fp8_rows.argtypes = [P, P, I64, I64, I64, I32, D, D, D, D, P, I64, P]
            _lib = lib
    return _lib


def _bits(t: torch.Tensor) -> np.ndarray:
    assert t.dtype == torch.bfloat16
    return np.ascontiguousarray(t.contiguous().view(torch.int16).numpy().view(np.uint16))


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def round_bf16(x: float) -> float:
    """fp64 -> nearest bf16 value, ties to even (as a Python float)."""
    return _load().wan_oracle_round_bf16(float(x))


def to_bf16(y) -> torch.Tensor:
    """fp64 array -> bf16 tensor, each value rounded once, to nearest-even."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    _load().wan_oracle_f64_to_bf16(_ptr(y), _ptr(out), y.size)
    return torch.from_numpy(out.view(np.int16)).view(torch.bfloat16)


def rmsnorm(x: torch.Tensor, gamma: torch.Tensor, eps: float) -> np.ndarray:
    """Step 1: x [n, d] bf16 -> x * rsqrt(mean(x^2) + eps) * gamma, fp64, unrounded."""
    xb = _bits(x.reshape(-1, x.shape[-1]))
    n, d = xb.shape
    y = np.empty((n, d), dtype=np.float64)
    g = _bits(gamma)
    _load().wan_oracle_rmsnorm(_ptr(xb), n, d, d, _ptr(g), float(eps), _ptr(y))
    return y


def rope(y: np.ndarray, seq0: int, heads: int, grid, theta: float, split=SPLIT,
         half_split: bool = False) -> np.ndarray:
    """Step 3: rotate y [n, heads*128] fp64 for tokens seq0..seq0+n-1 of grid (F,H,W)."""
    y = np.ascontiguousarray(y, dtype=np.float64).copy()
    n = y.shape[0]
    sp = (ctypes.c_int32 * 3)(*split)
    _, H, W = grid
    _load().wan_oracle_rope(_ptr(y), n, seq0, heads, H, W, float(theta),
                            ctypes.cast(sp, ctypes.c_void_p), int(half_split))
    return y


def qk_norm_rope(qkv: torch.Tensor, grid, heads: int, gamma_q: torch.Tensor,
                 gamma_k: torch.Tensor, eps: float, theta: float) -> torch.Tensor:
    """Steps 1-3 on a packed [B, S, 3*heads*128] bf16 buffer; returns a new buffer."""
    B, S, D3 = qkv.shape
    F, H, W = grid
    assert S == F * H * W and D3 == 3 * heads * HEAD_DIM
    src = _bits(qkv)
    dst = np.empty_like(src)
    _load().wan_oracle_qk_norm_rope(_ptr(src), _ptr(dst), B, F, H, W, heads,
                                    _ptr(_bits(gamma_q)), _ptr(_bits(gamma_k)),
                                    float(eps), float(theta))
    return torch.from_numpy(dst.view(np.int16)).view(torch.bfloat16).reshape(B, S, D3)


def qk_norm_rope_tokens(qkv: torch.Tensor, grid, heads: int, gamma_q: torch.Tensor,
                        gamma_k: torch.Tensor, eps: float, theta: float, tokens) -> torch.Tensor:
    """Steps 1-3 for listed (b, s) tokens: bf16 [n, 2*heads*128] ([Q | K] per token)."""
    B, S, D3 = qkv.shape
    F, H, W = grid
    assert S == F * H * W and D3 == 3 * heads * HEAD_DIM
    tk = np.ascontiguousarray(np.asarray(tokens, dtype=np.int64).reshape(-1, 2))
    assert (tk >= 0).all() and (tk[:, 0] < B).all() and (tk[:, 1] < S).all()
    out = np.empty((tk.shape[0], 2 * heads * HEAD_DIM), dtype=np.uint16)
    src = _bits(qkv)
    _load().wan_oracle_qk_norm_rope_tokens(_ptr(src), B, F, H, W, heads, _ptr(_bits(gamma_q)),
                                           _ptr(_bits(gamma_k)), float(eps), float(theta), _ptr(tk),
                                           tk.shape[0], _ptr(out))
    return torch.from_numpy(out.view(np.int16)).view(torch.bfloat16)


def attention_rows(qkv: torch.Tensor, heads: int, rows, scale: float) -> np.ndarray:
    """Step 4 for listed (b, h, i) query rows of a packed buffer; fp64 [n, 128]."""
    B, S, D3 = qkv.shape
    assert D3 == 3 * heads * HEAD_DIM
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    assert (r[:, 0] < B).all() and (r[:, 1] < heads).all() and (r[:, 2] < S).all() and (r >= 0).all()
    out = np.empty((r.shape[0], HEAD_DIM), dtype=np.float64)
    src = _bits(qkv)
    _load().wan_oracle_attention_rows(_ptr(src), B, S, heads, float(scale), _ptr(r), r.shape[0],
                                      _ptr(out))
    return out


def attention_partial_rows(q_qkv: torch.Tensor, heads: int, kv: torch.Tensor, k_row0: int, k_rows: int, rows,
                           scale: float):
    """Step 4 over the keys [k_row0, k_row0 + k_rows) of kv [B, Skv, pitch]
    (K then V in its last 2*heads*128 columns) for listed (b, h, i) rows of the
    packed q_qkv: the softmax state (o fp64 [n, 128], ml fp64 [n, 2] = (m, l)),
    o = sum_j exp(a_j - m) v_j, l = sum_j exp(a_j - m), m = max_j a_j."""
    B, Sq, D3 = q_qkv.shape
    assert D3 == 3 * heads * HEAD_DIM and kv.shape[0] == B and kv.shape[2] >= 2 * heads * HEAD_DIM
    assert 0 <= k_row0 and k_rows >= 1 and k_row0 + k_rows <= kv.shape[1]
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    assert (r[:, 0] < B).all() and (r[:, 1] < heads).all() and (r[:, 2] < Sq).all() and (r >= 0).all()
    o = np.empty((r.shape[0], HEAD_DIM), dtype=np.float64)
    ml = np.empty((r.shape[0], 2), dtype=np.float64)
    qb, kb = _bits(q_qkv), _bits(kv)
    _load().wan_oracle_attention_partial_rows(_ptr(qb), Sq, _ptr(kb), kv.shape[1], kv.shape[2], int(k_row0),
                                              int(k_rows), heads, float(scale), _ptr(r), r.shape[0], _ptr(o),
                                              _ptr(ml))
    return o, ml


def merge_partial(a, b):
    """Two softmax states over disjoint key ranges -> the state over their
    union (fp64): m = max(m_a, m_b), each side scaled by exp(its m - m)."""
    (oa, mla), (ob, mlb) = a, b
    m = np.maximum(mla[..., 0], mlb[..., 0])
    wa, wb = np.exp(mla[..., 0] - m), np.exp(mlb[..., 0] - m)
    o = oa * wa[..., None] + ob * wb[..., None]
    ml = np.stack([m, mla[..., 1] * wa + mlb[..., 1] * wb], axis=-1)
    return o, ml


def finalize_partial(state) -> np.ndarray:
    """The attention output of a softmax state: o / l."""
    o, ml = state
    return o / ml[..., 1:2]


def attention_skip_groups(qkv: torch.Tensor, heads: int, groups, scale: float, threshold: float):
    """Step 4 with Skip-Softmax (threshold mode) for listed (b, h, g) groups of
    32 query rows: (out fp64 [n, 32, 128] (rows past S: NaN), skipped bool
    [n, ceil(S/128)], margin fp64 [n]) -- see wan_oracle_attention_skip_groups."""
    B, S, D3 = qkv.shape
    assert D3 == 3 * heads * HEAD_DIM
    g = np.ascontiguousarray(np.asarray(groups, dtype=np.int64).reshape(-1, 3))
    assert (g[:, 0] < B).all() and (g[:, 1] < heads).all() and (g[:, 2] * 32 < S).all() and (g >= 0).all()
    n_tiles = (S + 127) // 128
    out = np.empty((g.shape[0], 32, HEAD_DIM), dtype=np.float64)
    skipped = np.zeros((g.shape[0], n_tiles), dtype=np.uint8)
    margin = np.empty(g.shape[0], dtype=np.float64)
    src = _bits(qkv)
    _load().wan_oracle_attention_skip_groups(_ptr(src), B, S, heads, float(scale), float(threshold),
                                             _ptr(g), g.shape[0], _ptr(out), _ptr(skipped), _ptr(margin))
    return out, skipped.astype(bool), margin


def e4m3_encode(v: float) -> int:
    """e4m3 code of a finite value (round to nearest even, saturating at +-448)."""
    return int(_load().wan_oracle_e4m3_encode(float(v)))


def e4m3_decode(c: int) -> float:
    return float(_load().wan_oracle_e4m3_decode(int(c)))


def quantize_e4m3(x: torch.Tensor, inv_scale: float) -> np.ndarray:
    """Codes (uint8, same shape) of a bf16 tensor: e4m3(fl32(x * inv_scale))."""
    assert x.dtype == torch.bfloat16
    src = np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))
    out = np.empty(src.shape, dtype=np.uint8)
    _load().wan_oracle_quantize_e4m3(_ptr(src), src.size, float(np.float32(inv_scale)), _ptr(out))
    return out


def fp8_operands(qkv: torch.Tensor, heads: int, inv_sq: float, inv_sk: float, inv_sv: float, s_pitch: int):
    """The e4m3 operands of the FP8 variant from a packed bf16 buffer: qk8
    [B, S, 2D] (Q then K of each token) and v8t [B, heads, 128, s_pitch] (V
    transposed, zero codes past S)."""
    B, S, D3 = qkv.shape
    D = D3 // 3
    qk8 = np.concatenate([quantize_e4m3(qkv[..., :D], inv_sq), quantize_e4m3(qkv[..., D:2 * D], inv_sk)], axis=-1)
    v8 = quantize_e4m3(qkv[..., 2 * D:], inv_sv).reshape(B, S, heads, HEAD_DIM)
    v8t = np.zeros((B, heads, HEAD_DIM, s_pitch), dtype=np.uint8)
    v8t[..., :S] = v8.transpose(0, 2, 3, 1)
    return np.ascontiguousarray(qk8), v8t


def attention_fp8_rows(qk8: np.ndarray, v8t: np.ndarray, heads: int, rows, scale: float, sq: float,
                       sk: float, sv: float) -> np.ndarray:
    """Step 4 on e4m3 operands (dequantised, fp64) for listed (b, h, i) rows: [n, 128]."""
    B, S, D2 = qk8.shape
    assert D2 == 2 * heads * HEAD_DIM and v8t.shape[:3] == (B, heads, HEAD_DIM)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    out = np.empty((r.shape[0], HEAD_DIM), dtype=np.float64)
    qk8 = np.ascontiguousarray(qk8)
    v8t = np.ascontiguousarray(v8t)
    _load().wan_oracle_attention_fp8_rows(_ptr(qk8), _ptr(v8t), B, S, v8t.shape[3], heads, float(scale),
                                          float(sq), float(sk), float(sv), _ptr(r), r.shape[0], _ptr(out))
    return out


def linear_rows(x: torch.Tensor, w: torch.Tensor, rows) -> np.ndarray:
    """The QKV (or output) projection Y = X W^T for listed rows of X [M, K]
    (bf16 values, exact in fp64), in fp64 with numpy's matrix product: [n, N].
    The projection precedes the path (TensorRT-LLM PR "[visual_gen] Optimize
    Wan2.2 Dataflow": the fused QKV projection output is the packed buffer)."""
    xr = x.reshape(-1, x.shape[-1])[torch.as_tensor(np.asarray(rows, dtype=np.int64))].double().numpy()
    return xr @ w.double().numpy().T


def linear_bf16(x: torch.Tensor, w: torch.Tensor, chunk: int = 4096) -> torch.Tensor:
    """The projection Y = X W^T for every row of X [M, K], each output rounded
    once to bf16 (RNE): the packed buffer as the projection stores it.
    Evaluated `chunk` rows at a time with linear_rows."""
    M = x.reshape(-1, x.shape[-1]).shape[0]
    out = torch.empty((M, w.shape[0]), dtype=torch.bfloat16)
    for r0 in range(0, M, chunk):
        r1 = min(r0 + chunk, M)
        out[r0:r1] = to_bf16(linear_rows(x, w, np.arange(r0, r1)))
    return out


def attention_full(qkv: torch.Tensor, heads: int, scale: float) -> np.ndarray:
    """Step 4 for every row: fp64 [B, S, heads, 128]."""
    B, S, _ = qkv.shape
    b, h, i = np.meshgrid(np.arange(B), np.arange(heads), np.arange(S), indexing="ij")
    rows = np.stack([b.transpose(0, 2, 1).ravel(), h.transpose(0, 2, 1).ravel(),
                     i.transpose(0, 2, 1).ravel()], axis=1)
    return attention_rows(qkv, heads, rows, scale).reshape(B, S, heads, HEAD_DIM)
