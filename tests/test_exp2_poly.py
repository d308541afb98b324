"""The FP8 attention kernel evaluates 2^x for an eighth of its probabilities
with a polynomial on the FMA pipe. Checks, on the CPU: the embedded coefficients are
the ones exp2_poly.py fits; the fit is minimax (equioscillating) with max
relative error below 1e-4; and the kernel's float32 steps (magic-number
rounding, Horner with FMAs, exponent-field add, clamp at -126), emulated with
numpy, stay within that bound of np.exp2 over the whole range the softmax uses."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "video_diffusion_transformer_packed_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("exp2_poly", os.path.join(CSRC, "exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_constants():
    src = open(os.path.join(CSRC, "attn_fwd_fp8.cu")).read()
    vals = {}
    for name in ("C0", "C1", "C2", "C3"):
        vals[name] = int(re.search(r"kPoly%s = (0x[0-9A-F]{8})u" % name, src).group(1), 16)
    return [np.array(vals[f"C{i}"], dtype=np.uint32).view(np.float32).item() for i in range(4)]


def test_kernel_embeds_the_fitted_coefficients():
    fit = _fit_module().coefficients_f32()
    assert _kernel_constants() == fit


def test_fit_is_minimax_and_accurate():
    m = _fit_module()
    c = np.array(m.remez(), dtype=np.float64)
    grid = np.linspace(-0.5, 0.5, 200001)
    e = np.polyval(c[::-1], grid) * np.exp2(-grid) - 1.0
    # equioscillation: the error reaches +-E with alternating signs at 5 points
    emax = np.max(np.abs(e))
    assert emax < 1e-4
    assert abs(e[0]) > 0.99 * emax and abs(e[-1]) > 0.99 * emax
    assert m.max_rel_error_f32(m.coefficients_f32()) < 1e-4


def _fma32(a, b, c):
    # float32 FMA: the float64 product of two float32 is exact; one rounding to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _emulate(x):
    c0, c1, c2, c3 = (np.float32(v) for v in _kernel_constants())
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    j = (x + magic).astype(np.float32)
    f = (x - (j - magic).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    bits = p.view(np.uint32) + (j.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_emulated_kernel_steps_match_exp2():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), rng.uniform(-30, 8, 400000)]).astype(np.float32)
    got = _emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.2e-4
    # integers are reproduced to the polynomial's error
    ints = np.arange(-120, 9, dtype=np.float32)
    assert np.allclose(_emulate(ints), np.exp2(ints.astype(np.float64)), rtol=1e-4)


def test_emulated_clamp_and_masked_scores():
    out = _emulate(np.array([-np.inf, -1000.0, -126.5], dtype=np.float32)).astype(np.float64)
    assert np.all(out >= 0) and np.all(out < 2.0 ** -125)
