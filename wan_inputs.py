"""Seeded synthetic inputs and workload shapes for the Wan2.2 DiT self-attention path.

This module is shared by the CUDA path's tests/bench and by the oracle's tests.
It holds only shapes and seeded random numbers -- none of the method's
arithmetic (no normalisation, rotation or softmax lives here).

Shapes follow the Wan2.2 pages:
  * token count: AWS Neuron "Optimizing High-Quality Offline Video Generation",
    section "Grounding in an output spec" -- sides rounded down to a multiple
    of 16, 8x spatial / 4x temporal VAE compression, DiT patch 2 per spatial
    dim; 832x480 at 81 frames gives S = 21*30*52 = 32760.
  * 40 heads x 128 (A14B, hidden 5120) and S = 75600 at 1280x720: TensorRT-LLM
    PR "[visual_gen] Optimize Wan2.2 Dataflow", "Isolated Operator Results".
Value distributions (packed QKV ~ N(0,1), RMSNorm gammas ~ U(0.5, 1.5)) are
the synthetic stand-ins for activations and trained weights, which are not
available.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import torch

HEAD_DIM = 128
EPS = 1e-6
THETA = 10000.0
ROPE_SPLIT = (44, 42, 42)  # head dims given to (frame, height, width)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    grid: Tuple[int, int, int]  # (F, H, W) token grid, w fastest
    heads: int

    @property
    def seq_len(self) -> int:
        f, h, w = self.grid
        return f * h * w

    @property
    def dim(self) -> int:
        return self.heads * HEAD_DIM

    @property
    def attn_flop(self) -> float:
        """Dense attention FLOP: two S x S x 128 contractions per (batch, head)."""
        s = self.seq_len
        return 4.0 * self.batch * self.heads * s * s * HEAD_DIM

    @property
    def norm_rope_bytes(self) -> float:
        """Algorithmic HBM bytes of the in-place Q/K norm+RoPE: read+write Q and K."""
        return 8.0 * self.dim * self.seq_len * self.batch

    def describe(self) -> Dict[str, object]:
        f, h, w = self.grid
        return {"workload": self.name, "batch": self.batch, "grid_fhw": [f, h, w],
                "seq_len": self.seq_len, "heads": self.heads, "head_dim": HEAD_DIM}


def dit_token_grid(width: int, height: int, frames: int) -> Tuple[int, int, int]:
    """(F, H, W) DiT token grid of a Wan2.2 clip (16-rounding, VAE 8x/4x, patch 2)."""
    w_lat = ((width // 16) * 16) // 8
    h_lat = ((height // 16) * 16) // 8
    t_lat = (frames - 1) // 4 + 1
    return (t_lat, h_lat // 2, w_lat // 2)


WORKLOADS: List[Workload] = [
    Workload("tiny_5x8x8_h12_b1", 1, (5, 8, 8), 12),
    Workload("a14b_480p_5f_b1", 1, (5, 30, 52), 40),
    Workload("a14b_480p_81f_cfg_b2", 2, dit_token_grid(832, 480, 81), 40),
    Workload("a14b_720p_81f_b1", 1, dit_token_grid(1280, 720, 81), 40),
    # TI2V-5B: latent 31x44x78 (16x VAE), patch 1x2x2 -> (31, 22, 39).
    Workload("ti2v5b_704p_121f_cfg_b2", 2, (31, 22, 39), 24),
]
BY_NAME = {w.name: w for w in WORKLOADS}
BENCH_WORKLOAD = WORKLOADS[2]


def packed_qkv(batch: int, seq_len: int, heads: int, seed: int = 0,
               chunk_rows: int = 4096) -> torch.Tensor:
    """Packed [B, S, 3*heads*128] bf16 ~ N(0,1) on the CPU, from a seeded generator.

    Generated in row chunks so that the fp32 temporaries stay small; the result
    depends only on (shape, seed) and the chunking is fixed.
    """
    d3 = 3 * heads * HEAD_DIM
    out = torch.empty((batch, seq_len, d3), dtype=torch.bfloat16)
    g = torch.Generator().manual_seed(seed)
    flat = out.view(batch * seq_len, d3)
    for r0 in range(0, batch * seq_len, chunk_rows):
        r1 = min(r0 + chunk_rows, batch * seq_len)
        flat[r0:r1] = torch.randn((r1 - r0, d3), generator=g, dtype=torch.float32).to(torch.bfloat16)
    return out


def local_peaked_qkv(batch: int, seq_len: int, heads: int, seed: int = 0, alpha: float = 0.6,
                     reach: int = 8) -> torch.Tensor:
    """Packed [B, S, 3*heads*128] bf16 whose attention is local and peaked: K and
    V ~ N(0,1) as in packed_qkv, and the query of token i is alpha times the key
    of a token drawn uniformly within `reach` positions of i (clamped to the
    sequence). A stand-in for the concentrated attention maps that make
    Skip-Softmax pay off on real activations, which are not available here.
    """
    out = packed_qkv(batch, seq_len, heads, seed)
    D = heads * HEAD_DIM
    g = torch.Generator().manual_seed(seed + 7919)
    for b in range(batch):
        src = (torch.arange(seq_len) + torch.randint(-reach, reach + 1, (seq_len,), generator=g)).clamp(0, seq_len - 1)
        for r0 in range(0, seq_len, 4096):
            r1 = min(r0 + 4096, seq_len)
            out[b, r0:r1, :D] = (alpha * out[b, src[r0:r1], D:2 * D].float()).to(torch.bfloat16)
    return out


def gammas(heads: int, seed_q: int = 1, seed_k: int = 2) -> Tuple[torch.Tensor, torch.Tensor]:
    """RMSNorm weights for Q and K over the full hidden dim, bf16 ~ U(0.5, 1.5)."""
    d = heads * HEAD_DIM
    gq = (torch.rand(d, generator=torch.Generator().manual_seed(seed_q)) + 0.5).to(torch.bfloat16)
    gk = (torch.rand(d, generator=torch.Generator().manual_seed(seed_k)) + 0.5).to(torch.bfloat16)
    return gq, gk


def inputs_for(w: Workload, seed: int = 0):
    qkv = packed_qkv(w.batch, w.seq_len, w.heads, seed)
    gq, gk = gammas(w.heads, seed + 1, seed + 2)
    return qkv, gq, gk


def head_magnitude_qkv(batch: int, seq_len: int, heads: int, seed: int = 3) -> torch.Tensor:
    """Packed QKV whose Q and K heads carry magnitudes 2**(h % 7 - 3).

    A per-head normalisation and a full-width one give different results on
    this input (the review comments on the TensorRT-LLM PR ask for exactly
    this parity case).
    """
    qkv = packed_qkv(batch, seq_len, heads, seed).float()
    d = heads * HEAD_DIM
    scale = torch.tensor([2.0 ** (h % 7 - 3) for h in range(heads)]).repeat_interleave(HEAD_DIM)
    qkv[..., :d] *= scale
    qkv[..., d:2 * d] *= scale
    return qkv.to(torch.bfloat16)


def sample_rows(seq_len: int, n: int, seed: int, tile: int = 128) -> torch.Tensor:
    """Seeded query-row sample: always the first and last rows and the rows of
    the last (possibly partial) tile, plus uniform random rows."""
    last_tile0 = ((seq_len - 1) // tile) * tile
    fixed = {0, seq_len - 1} | set(range(last_tile0, seq_len))
    g = torch.Generator().manual_seed(seed)
    rnd = torch.randint(0, seq_len, (n,), generator=g).tolist()
    rows = sorted(fixed | set(rnd))
    return torch.tensor(rows, dtype=torch.int64)
