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


def assert_attention_close(got, ref, what="", scaled=False):
    """The bar: max-abs <= 2e-2 and relative Frobenius <= 1e-2. The absolute
    bound is meant for Wan-shaped data, whose outputs stay well below 1; with
    scaled=True (structured inputs whose outputs reach a magnitude M > 1) it is
    2e-2 * max(1, M), since rounding the output to bf16 alone costs up to M * 2^-9."""
    mx, rf = attention_errors(got, ref)
    bound = ATTN_MAX_ABS * (max(1.0, float(np.max(np.abs(ref)))) if scaled else 1.0)
    assert mx <= bound and rf <= ATTN_REL_FRO, f"{what}: max-abs {mx:.3e} (bound {bound:.2e}), rel-Frobenius {rf:.3e}"
    return mx, rf
