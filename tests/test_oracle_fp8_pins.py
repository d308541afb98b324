"""Pins of the oracle's FP8 (e4m3) pieces against things other than itself:
the encoder against torch's float8_e4m3fn conversion over every finite bf16
value in range (and over fp32 products at a non-trivial scale), saturation in
closed form, the code round trip, the transposed V layout, and FP8 attention
on values the e4m3 grid holds exactly against the dense oracle."""
import math

import numpy as np
import pytest
import torch

import oracle

HD = 128


def _all_bf16_in_range():
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    x = bits.view(torch.bfloat16)
    f = x.float()
    keep = torch.isfinite(f) & (f.abs() < 464.0)
    return x[keep]


def test_encoder_matches_torch_on_every_bf16_in_range():
    x = _all_bf16_in_range()
    ours = oracle.quantize_e4m3(x, 1.0)
    ref = x.float().to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (ours == ref).all()


@pytest.mark.parametrize("inv_scale", [1.0 / 0.0123, 37.25, 0.0078125])
def test_encoder_matches_torch_on_fp32_products(inv_scale):
    x = _all_bf16_in_range()
    inv32 = np.float32(inv_scale)
    prod = x.float() * float(inv32)  # fp32 products, as the reading prescribes
    keep = prod.abs() < 464.0
    ours = oracle.quantize_e4m3(x[keep], float(inv32))
    ref = prod[keep].to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert keep.sum() > 1000 and (ours == ref).all()


def test_saturation_and_signed_zero():
    for v in (464.0, 480.0, 1e4, 3.0e38):
        assert oracle.e4m3_encode(v) == 0x7E and oracle.e4m3_encode(-v) == 0xFE
    assert oracle.e4m3_encode(0.0) == 0x00 and oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(2.0 ** -11) == 0x00 and oracle.e4m3_encode(-(2.0 ** -11)) == 0x80
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert math.isnan(oracle.e4m3_decode(0x7F))


def test_code_round_trip():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c


def test_transposed_v_layout():
    B, S, heads = 2, 37, 3
    g = torch.Generator().manual_seed(3)
    qkv = torch.randn(B, S, 3 * heads * HD, generator=g).to(torch.bfloat16)
    qk8, v8t = oracle.fp8_operands(qkv, heads, 1.0, 1.0, 2.0, 48)
    D = heads * HD
    v8 = oracle.quantize_e4m3(qkv[..., 2 * D:], 2.0).reshape(B, S, heads, HD)
    for b, h, d, j in [(0, 0, 0, 0), (1, 2, 127, 36), (0, 1, 5, 17)]:
        assert v8t[b, h, d, j] == v8[b, j, h, d]
    assert (v8t[..., S:] == 0).all()
    assert (qk8[..., :D] == oracle.quantize_e4m3(qkv[..., :D], 1.0)).all()


def test_fp8_attention_on_exact_values_is_the_dense_attention():
    """Codes whose values the bf16 grid also holds: FP8 attention with unit
    scales must equal the dense oracle on the decoded buffer."""
    B, S, heads = 1, 200, 2
    g = torch.Generator().manual_seed(4)
    D = heads * HD
    codes = torch.randint(0, 256, (B, S, 3 * D), generator=g, dtype=torch.int32).to(torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38  # no NaN codes
    codes[(codes & 0x78) >= 0x50] &= 0x87  # keep |values| small so exponentials stay tame
    dec = torch.tensor(np.vectorize(oracle.e4m3_decode)(codes.numpy()), dtype=torch.float64)
    qkv = (dec * 0.25).to(torch.bfloat16)  # exact: a power-of-two scaling of e4m3 values
    assert torch.equal(qkv.double(), dec * 0.25)
    qk8, v8t = oracle.fp8_operands(qkv, heads, 4.0, 4.0, 4.0, 208)
    rows = [(0, h, i) for h in range(heads) for i in range(0, S, 7)]
    got = oracle.attention_fp8_rows(qk8, v8t, heads, rows, 1 / math.sqrt(HD), 0.25, 0.25, 0.25)
    ref = oracle.attention_rows(qkv, heads, rows, 1 / math.sqrt(HD))
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)
