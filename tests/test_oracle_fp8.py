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


# ---------------------------------------------------------------------------
# kv_append_fp8: the quantising append ("LLM inference optimisation:
# principles overview" §5.1, an FP8 KV cache), pinned against codes worked out
# by hand from the e4m3 definition (sign << 7 | exponent field << 3 | mantissa,
# bias 7; subnormals m/8 * 2^-6; 0x7E = 448 the largest finite).
# ---------------------------------------------------------------------------
_NB, _HKV, _BS, _D = 3, 2, 4, 4
_K_SCALE, _V_SCALE = 0.5, 0.125  # the append multiplies by 2 (K) and by 8 (V): exact in fp32
_SLOTS = np.array([6, -1, 9])    # token 0 -> block 1 offset 2; token 1 is padding; token 2 -> block 2 offset 1
_SENTINEL = 0x55

_K_ROWS = np.array([
    [[0.5, -0.75, 1.0, 224.0], [0.53125, -0.0, 2.0 ** -10, 1000.0]],
    [[9.0, 9.0, 9.0, 9.0], [9.0, 9.0, 9.0, 9.0]],  # padding row: never written
    [[1.75, 8.5, -0.375, 0.59375], [-224.0, 0.125, 0.1875, 4.0]],
], dtype=np.float32)
# 2x: 1, -1.5, 2, 448 | 1.0625 (tie -> even mantissa 0), -0, 2^-9 (smallest subnormal), 2000 (saturates)
#     3.5, 17 (tie -> even), -0.75, 1.1875 (tie -> even mantissa 2) | -448, 0.25, 0.375, 8
_K_CODES = {0: [[0x38, 0xBC, 0x40, 0x7E], [0x38, 0x80, 0x01, 0x7E]],
            2: [[0x46, 0x58, 0xB4, 0x3A], [0xFE, 0x28, 0x2C, 0x50]]}

_V_ROWS = np.array([
    [[0.25, 0.1875, -0.4375, 0.09375], [0.01171875, -56.0, 2.0 ** -12, 0.0]],
    [[-9.0, -9.0, -9.0, -9.0], [-9.0, -9.0, -9.0, -9.0]],
    [[1.0, -2.0, 0.5, 0.15625], [3.0, 0.0390625, -0.0078125, 60.0]],
], dtype=np.float32)
# 8x: 2, 1.5, -3.5, 0.75 | 0.09375 = 1.5 * 2^-4, -448, 2^-9, 0
#     8, -16, 4, 1.25 | 24, 0.3125, -0.0625, 480 (saturates)
_V_CODES = {0: [[0x40, 0x3C, 0xC6, 0x34], [0x1C, 0xFE, 0x01, 0x00]],
            2: [[0x50, 0xD8, 0x48, 0x3A], [0x5C, 0x2A, 0x98, 0x7E]]}


def _check_append_fp8(append):
    """Runs ``append`` (kv_append_fp8's signature) on the hand-worked case and
    asserts every byte of both pools."""
    kc = np.full((_NB, _HKV, _BS, _D), _SENTINEL, dtype=np.uint8)
    vc = np.full((_NB, _HKV, _BS, _D), _SENTINEL, dtype=np.uint8)
    k_out, v_out = append(kc, vc, _K_ROWS, _V_ROWS, _SLOTS, _K_SCALE, _V_SCALE)
    want_k = np.full_like(kc, _SENTINEL)
    want_v = np.full_like(vc, _SENTINEL)
    for tok, slot in ((0, 6), (2, 9)):
        blk, off = slot // _BS, slot % _BS
        want_k[blk, :, off, :] = np.array(_K_CODES[tok], dtype=np.uint8)
        want_v[blk, :, off, :] = np.array(_V_CODES[tok], dtype=np.uint8)
    assert np.array_equal(k_out, want_k), "K pool bytes differ from the hand-worked codes"
    assert np.array_equal(v_out, want_v), "V pool bytes differ from the hand-worked codes"
    assert np.array_equal(kc, np.full_like(kc, _SENTINEL)), "the input pool was modified in place"


def test_kv_append_fp8_matches_hand_worked_codes():
    _check_append_fp8(fp8.kv_append_fp8)


def test_kv_append_fp8_planted_mistakes_are_caught(monkeypatch):
    """Plausible slips in the quantising append, each planted into the oracle
    and each turning the hand-worked pin red."""
    orig_append = fp8.kv_append_fp8
    mutants = {
        "K and V scales swapped": lambda kc, vc, k, v, s, ks, vs: orig_append(kc, vc, k, v, s, vs, ks),
        "K rows into the V pool": lambda kc, vc, k, v, s, ks, vs: orig_append(kc, vc, v, k, s, vs, ks),
        "multiply by the scale instead of dividing": lambda kc, vc, k, v, s, ks, vs: orig_append(
            kc, vc, k, v, s, 1.0 / ks, 1.0 / vs),
    }

    def block_and_offset_swapped(kc, vc, k, v, slots, ks, vs):
        kq, vq = fp8.quantize_rows(k, ks), fp8.quantize_rows(v, vs)
        ko, vo = kc.copy(), vc.copy()
        for i, s in enumerate(slots.tolist()):
            if s >= 0:
                off, blk = divmod(int(s), _BS)
                ko[blk % _NB, :, off % _BS, :] = kq[i]
                vo[blk % _NB, :, off % _BS, :] = vq[i]
        return ko, vo

    def padding_written(kc, vc, k, v, slots, ks, vs):
        kq, vq = fp8.quantize_rows(k, ks), fp8.quantize_rows(v, vs)
        ko, vo = kc.copy(), vc.copy()
        for i, s in enumerate(slots.tolist()):
            blk, off = divmod(int(s), _BS)  # slot -1 lands in the last block, offset 3
            ko[blk, :, off, :] = kq[i]
            vo[blk, :, off, :] = vq[i]
        return ko, vo

    mutants["block and offset swapped"] = block_and_offset_swapped
    mutants["padding slot written"] = padding_written

    # rounding slips inside the encoder the append uses
    orig_encode = fp8.e4m3_encode
    mags = fp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))

    def truncating(x):
        x = np.asarray(x, dtype=np.float64)
        out = [int(np.searchsorted(mags, min(abs(v), 448.0), side="right")) - 1 | (0x80 if np.signbit(v) else 0)
               for v in x.reshape(-1).tolist()]
        return np.array(out, dtype=np.uint8).reshape(x.shape)

    encode_mutants = {
        "ties away from zero": lambda x: orig_encode(np.asarray(x, dtype=np.float64) * (1 + 2.0 ** -40)),
        "no saturation (overflow to NaN)": lambda x: np.where(np.abs(np.asarray(x, dtype=np.float64)) > 448,
                                                               np.uint8(0x7F), orig_encode(x)).astype(np.uint8),
        "truncation instead of rounding": truncating,
    }
    survivors = []
    for name, fn in mutants.items():
        try:
            _check_append_fp8(fn)
            survivors.append(name)
        except AssertionError:
            pass
    for name, fn in encode_mutants.items():
        monkeypatch.setattr(fp8, "e4m3_encode", fn)
        try:
            _check_append_fp8(fp8.kv_append_fp8)
            survivors.append(name)
        except AssertionError:
            pass
        monkeypatch.setattr(fp8, "e4m3_encode", orig_encode)
    assert not survivors, f"mutants that survived the pin: {survivors}"


def test_decode_over_full_range_codes_needs_p_beyond_f16():
    """How precise the softmax weights P must be when they meet e4m3 V in a
    tensor-core product: over pools whose codes span the whole e4m3 range (V
    up to 448 * v_scale), a single f16 P (11 significant bits) misses the
    2e-3 output tolerance, while P as two f16 halves (hi + lo, about 22 bits)
    stays far inside it.  (The e4m3 decode kernel carries P as four e4m3
    terms, about 16 bits: tests/test_fp8_terms.py.)  Both products are
    simulated here in float64 from the rounded weights, the sum of weights in
    fp32; the reference is the oracle's definition."""
    rng = np.random.default_rng(5)

    def codes(shape):
        c = rng.integers(0, 256, size=shape).astype(np.uint8)
        c[(c & 0x7F) == 0x7F] ^= 1  # no NaN codes
        return c

    worst_single, worst_pair = 0.0, 0.0
    for _ in range(60):
        L = int(rng.integers(1, 2000))
        kc, vc = codes((1, 1, L, 128)), codes((1, 1, L, 128))
        q = rng.standard_normal((1, 1, 128)).astype(np.float16)
        ref = fp8.paged_decode_attention_fp8(q, kc, vc, np.zeros((1, 1), np.int32), np.array([L]), 1 / np.sqrt(128),
                                             0.25, 0.5)[0, 0]
        K = fp8.e4m3_decode(kc[0, 0]) * 0.25
        V = fp8.e4m3_decode(vc[0, 0]) * 0.5
        s = K @ q[0, 0].astype(np.float64) / np.sqrt(128)
        p = np.exp(s - s.max()).astype(np.float32)
        hi = p.astype(np.float16).astype(np.float64)
        lo = (p.astype(np.float64) - hi).astype(np.float16).astype(np.float64)
        den = float(p.astype(np.float64).sum())
        tol = 2e-3 * np.maximum(1.0, np.abs(ref))
        worst_single = max(worst_single, float(np.max(np.abs(hi @ V / den - ref) / tol)))
        worst_pair = max(worst_pair, float(np.max(np.abs((hi + lo) @ V / den - ref) / tol)))
    assert worst_single > 1.0, "a single f16 P would meet the tolerance here"
    assert worst_pair < 0.05
