"""Shared comparison helpers for the parity tests (no method arithmetic here)."""
import numpy as np
import torch

# Tolerances for the attention output against the fp64 oracle: max-abs error
# and relative Frobenius error (the bar set for this path).
ATTN_MAX_ABS = 2e-2
ATTN_REL_FRO = 1e-2


def bf16_ulp_distance(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """Distance in units of the last place between two bf16 tensors (0 = identical,
    1 = adjacent representable values), via the monotone integer order of bf16."""
    def mono(t):
        i = t.contiguous().view(torch.int16).to(torch.int32)
        return torch.where(i < 0, -(i & 0x7FFF), i)
    return (mono(a) - mono(b)).abs()


def attention_errors(got: torch.Tensor, ref: np.ndarray):
    """(max-abs, relative Frobenius) of a GPU bf16 output against fp64 reference values."""
    g = got.double().cpu().numpy().reshape(ref.shape)
    d = g - ref
    return float(np.max(np.abs(d))), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))


def assert_attention_close(got, ref, what=""):
    """The bar: max-abs <= 2e-2 and relative Frobenius <= 1e-2, flat, whatever
    the magnitude of the outputs."""
    mx, rf = attention_errors(got, ref)
    assert mx <= ATTN_MAX_ABS and rf <= ATTN_REL_FRO, f"{what}: max-abs {mx:.3e}, rel-Frobenius {rf:.3e}"
    return mx, rf
