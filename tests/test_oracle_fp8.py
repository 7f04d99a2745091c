"""Pins for the e4m3 oracle (CPU only): the code table against torch's
float8_e4m3fn and closed-form values, round trips, rounding ties, saturation,
and fp8 attention equal to the 16-bit definition on dequantised values."""
import math

import numpy as np
import pytest
import torch

from oracle import fp8
from oracle import paged_attention as pa


def _torch_decode(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    mine, lib = fp8.e4m3_decode(codes), _torch_decode(codes)
    assert np.array_equal(np.isnan(mine), np.isnan(lib))
    ok = ~np.isnan(mine)
    assert np.array_equal(mine[ok], lib[ok])


@pytest.mark.parametrize("code,value", [(0x38, 1.0), (0xB8, -1.0), (0x7E, 448.0), (0xFE, -448.0), (0x01, 2.0 ** -9),
                                        (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x3C, 1.5), (0x40, 2.0),
                                        (0x00, 0.0)])
def test_closed_form_values(code, value):
    assert fp8.e4m3_decode([code])[0] == value


def test_nan_codes():
    assert np.isnan(fp8.e4m3_decode([0x7F, 0xFF])).all()
    assert fp8.e4m3_encode([float("nan")])[0] == 0x7F


def test_round_trip_every_finite_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(fp8.e4m3_encode(fp8.e4m3_decode(codes)), codes)


def test_encode_matches_torch_in_range_including_ties():
    rng = np.random.default_rng(8)
    x = np.concatenate([rng.standard_normal(5000) * 30, rng.uniform(-448, 448, 5000)])
    mags = fp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (mags[:-1] + mags[1:]) / 2  # exact ties between neighbours
    x = np.concatenate([x, mids, -mids]).astype(np.float32)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.e4m3_encode(x.astype(np.float64)), lib)


def test_ties_go_to_even_mantissa():
    # between 1.0 (0x38, mantissa 0) and 1.125 (0x39): tie -> 0x38; between 1.125 and 1.25: tie -> 0x3A
    assert fp8.e4m3_encode([1.0625])[0] == 0x38
    assert fp8.e4m3_encode([1.1875])[0] == 0x3A


def test_saturation():
    enc = fp8.e4m3_encode([448.0, 460.0, 1e6, -1e6, math.inf, -math.inf])
    assert enc.tolist() == [0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE]


def test_quantize_rows_uses_fp32_product():
    rows = np.array([[1.0, -3.0, 0.3]], dtype=np.float32)
    codes = fp8.quantize_rows(rows, 0.5)  # x * 2
    assert fp8.e4m3_decode(codes).tolist() == [[2.0, -6.0, 0.625]]


def test_fp8_attention_is_the_definition_on_dequantised_values():
    rng = np.random.default_rng(9)
    nb, hkv, bs, d = 6, 2, 16, 32
    kc = fp8.e4m3_encode(rng.standard_normal((nb, hkv, bs, d)) * 4).astype(np.uint8)
    vc = fp8.e4m3_encode(rng.standard_normal((nb, hkv, bs, d)) * 4).astype(np.uint8)
    q = rng.standard_normal((2, 4, d)).astype(np.float16)
    tables = np.array([[3, 1, 0], [5, 2, 4]], dtype=np.int32)
    lens = np.array([40, 33])
    got = fp8.paged_decode_attention_fp8(q, kc, vc, tables, lens, 0.2, 0.25, 0.5)
    want = pa.paged_decode_attention(q.astype(np.float32), (fp8.e4m3_decode(kc) * 0.25).astype(np.float32),
                                     (fp8.e4m3_decode(vc) * 0.5).astype(np.float32), tables, lens, 0.2, "f32")
    assert np.max(np.abs(got - want)) < 1e-12  # all dequantised values are exact in fp32
