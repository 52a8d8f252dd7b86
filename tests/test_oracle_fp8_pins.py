"""Pins of the oracle's FP8 (E4M3) input decoding and FP8 attention against facts outside
the oracle: hand-decoded codes from the format's definition, every one of the 256 codes
against PyTorch's float8_e4m3fn conversion (a library witness), and the reduction of FP8
attention to attention of the dequantised values."""

import math

import numpy as np
import pytest
import torch

import oracle


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x38, 1.0), (0xB8, -1.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9),
    (0x08, 2.0 ** -6), (0x3C, 1.5), (0x40, 2.0), (0x7E, 448.0), (0xFE, -448.0),
    (0x28, 0.25), (0x30, 0.5), (0x3F, 1.875),
])
def test_hand_decoded_codes(code, value):
    # value = (-1)^s · (1 + m/8) · 2^(e - 7), or m · 2^-9 when e = 0
    assert oracle.e4m3_to_float([code])[0] == value


def test_nan_code_and_negative_zero():
    v = oracle.e4m3_to_float([0x7F, 0xFF, 0x80])
    assert math.isnan(v[0]) and math.isnan(v[1])
    assert v[2] == 0.0 and math.copysign(1.0, v[2]) == -1.0


def test_all_codes_match_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_to_float(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])


def test_fp8_attention_is_attention_of_dequantised_inputs():
    rng = np.random.default_rng(3)
    L, d = 9, 16
    q8, k8, v8 = (rng.integers(0, 256, size=(L, d)).astype(np.uint8) for _ in range(3))
    for a in (q8, k8, v8):  # keep away from the NaN code
        a[(a & 0x7F) == 0x7F] = 0x3A
    sq, sk, sv = 0.01, 0.02, 0.5
    o, lse = oracle.attention_forward_fp8(q8, k8, v8, sq, sk, sv, 0.3, True)
    q = torch.from_numpy(q8).view(torch.float8_e4m3fn).double().numpy() * sq
    k = torch.from_numpy(k8).view(torch.float8_e4m3fn).double().numpy() * sk
    v = torch.from_numpy(v8).view(torch.float8_e4m3fn).double().numpy() * sv
    o2, l2 = oracle.attention_forward(q, k, v, 0.3, True)
    np.testing.assert_allclose(o, o2, atol=1e-15)
    np.testing.assert_allclose(lse, l2, atol=1e-15)


def test_planted_decoder_mistake_is_caught(monkeypatch):
    import oracle.attn_ref as ref
    real = ref.e4m3_to_float

    def bias8(codes):  # wrong exponent bias
        return real(codes) / 2.0

    monkeypatch.setattr(oracle, "e4m3_to_float", bias8)
    with pytest.raises(AssertionError):
        test_hand_decoded_codes(0x38, 1.0)
    monkeypatch.setattr(oracle, "e4m3_to_float", real)
