"""FP8 (e4m3) variant through the C ABI: amax and quantiser codes bit-exact
against torch and the oracle (integer work), and the FP8 attention against the
oracle's attention on the same dequantised codes.

Tolerance of the FP8 attention. The operands' own rounding is shared with the
oracle, which works on the dequantised codes; what differs is that the kernel
rounds each probability p_j (normalised so that the row's largest is at least
1) to e4m3 before the P V product: |p^_j - p_j| <= max(2^-4 p_j, 2^-10)
(relative in e4m3's normal range, absolute in its subnormal range), plus the
relative error of the exponential itself (below 1.2e-4 for the eighth the
kernel evaluates with its polynomial, far smaller for MUFU ex2). With the
row sum taken over the unrounded p_j, every output element then obeys
  |o^_i - o_i| <= sum_j max((2^-4 + 1.2e-4) p_j, 2^-10) |v_j| / sum_j p_j
plus the bf16 rounding of the output (2^-8 |o_i| here, with margin for the
fp32 accumulation). That per-element bound is checked for every element. On
rows whose weights spread over many keys the errors do not average out
relative to the output itself (RMS about 2^-4/sqrt(3) = 3.6 %), so the
relative Frobenius error is bounded by 6e-2."""
import math

import numpy as np
import pytest
import torch

import oracle
import video_diffusion_transformer_packed_b200 as wan
import wan_inputs as wi
from video_diffusion_transformer_packed_b200 import build as wan_build
from helpers import attention_errors

pytestmark = pytest.mark.gpu
HD = 128
FP8_REL_FRO = 6e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    wan_build.build()


def scales_from(amax):
    """(scales, inverse scales) as fp32: s = amax / 448, inv = 448 / amax."""
    a = np.asarray(amax, dtype=np.float32)
    return (a / np.float32(448.0)).tolist(), (np.float32(448.0) / a).tolist()


def test_amax_matches_torch():
    w = wi.WORKLOADS[1]
    qkv, _, _ = wi.inputs_for(w, seed=2)
    got = wan.qkv_amax(qkv.cuda(), w.heads).cpu().numpy()
    D = w.dim
    ref = [float(qkv[..., i * D:(i + 1) * D].float().abs().max()) for i in range(3)]
    assert got.tolist() == ref


@pytest.mark.parametrize("batch,S,heads,inv", [
    (1, 320, 12, (37.25, 41.5, 60.0)),
    (2, 261, 7, (1.0, 2.0, 0.5)),
    (1, 129, 3, (448.0 / 4.4, 448.0 / 5.1, 448.0 / 4.9)),
])
def test_quantiser_codes_are_bit_exact(batch, S, heads, inv):
    qkv = wi.packed_qkv(batch, S, heads, seed=S)
    qk8, v8t = wan.quantize_fp8(qkv.cuda(), heads, inv)
    pitch = wan.fp8_pitch(S)
    ref_qk, ref_vt = oracle.fp8_operands(qkv, heads, *[float(np.float32(x)) for x in inv], pitch)
    assert np.array_equal(qk8.cpu().numpy(), ref_qk)
    assert np.array_equal(v8t.cpu().numpy(), ref_vt)


def test_quantiser_saturates():
    qkv = (wi.packed_qkv(1, 64, 1, seed=1).float() * 100).to(torch.bfloat16)
    qk8, v8t = wan.quantize_fp8(qkv.cuda(), 1, (10.0, 10.0, 10.0))
    ref_qk, ref_vt = oracle.fp8_operands(qkv, 1, 10.0, 10.0, 10.0, 64)
    assert np.array_equal(qk8.cpu().numpy(), ref_qk) and np.array_equal(v8t.cpu().numpy(), ref_vt)
    assert (qk8.cpu().numpy() & 0x7F).max() == 0x7E  # saturated codes present


def elementwise_bound(qk8, v8t, heads, rows, scale, sq, sk, sv, ref):
    """The per-element bound of the module docstring for listed (b, h, i) rows."""
    lut = np.array([oracle.e4m3_decode(c) if (c & 0x7F) != 0x7F else 0.0 for c in range(256)])
    B, S, d2 = qk8.shape
    D = d2 // 2
    bound = np.empty((len(rows), HD))
    cache = {}
    for r, (b, h, i) in enumerate(rows):
        if (b, h) not in cache:
            cache = {(b, h): (lut[qk8[b, :, D + h * HD:D + (h + 1) * HD]] * sk, lut[v8t[b, h, :, :S]].T * sv)}
        k, v = cache[(b, h)]
        q = lut[qk8[b, i, h * HD:(h + 1) * HD]] * sq
        a = (k @ q) * scale
        p = np.exp(a - a.max())
        bound[r] = (np.maximum((2.0 ** -4 + 1.2e-4) * p, 2.0 ** -10) @ np.abs(v)) / p.sum()
    return bound + 2.0 ** -8 * np.abs(ref) + 1e-6


def _fp8_case(batch, S, heads, seed, peaked=False):
    qkv = (wi.local_peaked_qkv(batch, S, heads, seed) if peaked else wi.packed_qkv(batch, S, heads, seed))
    d = qkv.cuda()
    sc, inv = scales_from(wan.qkv_amax(d, heads).cpu().numpy())
    qk8, v8t = wan.quantize_fp8(d, heads, inv)
    out = wan.self_attention_fp8(qk8, v8t, heads, sc)
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    return qkv, qk8.cpu().numpy(), v8t.cpu().numpy(), sc, out.cpu()


@pytest.mark.parametrize("batch,S,heads,peaked", [
    (1, 320, 12, False),
    (2, 261, 7, False),
    (1, 700, 2, True),
    (1, 1, 3, False),
    (1, 127, 2, False),
    (2, 257, 1, True),
])
def test_fp8_attention_matches_oracle(batch, S, heads, peaked):
    qkv, qk8, v8t, sc, out = _fp8_case(batch, S, heads, seed=S + 1, peaked=peaked)
    rows = [(b, h, i) for b in range(batch) for h in range(heads) for i in range(S)]
    ref = oracle.attention_fp8_rows(qk8, v8t, heads, rows, 1 / math.sqrt(HD), *sc)
    got = out.view(batch, S, heads, HD).permute(0, 2, 1, 3).reshape(-1, HD)
    mx, rf = attention_errors(got, ref)
    assert rf <= FP8_REL_FRO, f"rel-Fro {rf:.3e}"
    err = np.abs(got.double().numpy() - ref)
    bound = elementwise_bound(qk8, v8t, heads, rows, 1 / math.sqrt(HD), *sc, ref)
    worst = float((err / bound).max())
    assert worst <= 1.0, f"element error reaches {worst:.2f} of its bound (max-abs {mx:.3e})"


def test_fp8_attention_fidelity_to_the_bf16_path():
    """Against the unquantised fp64 attention of the same bf16 buffer: the
    divergence of the whole FP8 path (operand and P rounding) stays within
    twice the FP8 bound."""
    w = wi.WORKLOADS[0]
    qkv, _, _, _, out = _fp8_case(w.batch, w.seq_len, w.heads, seed=9)
    ref = oracle.attention_full(qkv, w.heads, 1 / math.sqrt(HD))
    mx, rf = attention_errors(out.view(1, w.seq_len, w.heads, HD), ref)
    assert rf <= 2 * FP8_REL_FRO, f"rel-Fro {rf:.3e}"


@pytest.mark.parametrize("idx", [2, 4])
def test_fp8_full_size_sampled_rows(idx):
    """Full-size workloads in the bench's configuration (normalised buffer,
    per-tensor amax/448 scales): sampled rows of sampled (batch, head) pairs,
    first and last rows and the whole ragged last tile included, against the
    oracle on the kernel's own codes (which are checked bit-exact above)."""
    w = wi.WORKLOADS[idx]
    qkv, gq, gk = wi.inputs_for(w, seed=0)
    d = qkv.cuda()
    wan.qk_norm_rope(d, w.grid, w.heads, gq.cuda(), gk.cuda(), wi.EPS, wi.THETA)
    sc, inv = scales_from(wan.qkv_amax(d, w.heads).cpu().numpy())
    qk8, v8t = wan.quantize_fp8(d, w.heads, inv)
    out = wan.self_attention_fp8(qk8, v8t, w.heads, sc)
    torch.cuda.synchronize()
    assert wan.device_error() == 0
    qk8, v8t = qk8.cpu().numpy(), v8t.cpu().numpy()
    g = torch.Generator().manual_seed(idx)
    pairs = [(0, 0), (w.batch - 1, w.heads - 1),
             (int(torch.randint(w.batch, (1,), generator=g)), int(torch.randint(w.heads, (1,), generator=g)))]
    rows = [(b, h, i) for (b, h) in pairs for i in wi.sample_rows(w.seq_len, 16, seed=b * 100 + h).tolist()]
    ref = oracle.attention_fp8_rows(qk8, v8t, w.heads, rows, 1 / math.sqrt(HD), *sc)
    oc = out.view(w.batch, w.seq_len, w.heads, HD).cpu()
    got = torch.stack([oc[b, i, h] for (b, h, i) in rows])
    mx, rf = attention_errors(got, ref)
    assert rf <= FP8_REL_FRO, f"{w.name}: rel-Fro {rf:.3e}"
    err = np.abs(got.double().numpy() - ref)
    bound = elementwise_bound(qk8, v8t, w.heads, rows, 1 / math.sqrt(HD), *sc, ref)
    assert float((err / bound).max()) <= 1.0, f"{w.name}: max-abs {mx:.3e}"
