"""FP8 e4m3 KV-cache storage, oracle side — TEST INFRASTRUCTURE ONLY.

The optimisation-overview page (§5.1) stores the KV cache in FP8
(`--kv-cache-dtype fp8`) so that a layer's cache takes half the bytes.  The
reading taken here: each stored K (or V) element is an e4m3 code; its value
is ``k_scale * e4m3_value(code)`` (one fp32 scale per pool).  The decode
computes attention exactly as for 16-bit pools on those dequantised values.

e4m3 (the "fn" variant: no infinities): 1 sign bit, 4 exponent bits with bias
7, 3 mantissa bits.  Exponent field 0 holds the subnormals
``m/8 · 2^-6``; exponent field e ≥ 1 holds ``(1 + m/8) · 2^(e-7)``; the code
with all exponent and mantissa bits set (0x7F / 0xFF) is NaN, so the largest
finite magnitude is 1.75 · 2^8 = 448.

Quantising an input row for the append (done by the library on the device):
multiply by the fp32 reciprocal of the scale, then round to the nearest e4m3
value, ties to even mantissa, saturating to ±448 (NaN stays NaN).  The product
is taken in fp32 here too, so both sides round the same fp32 number.
"""
from __future__ import annotations

import numpy as np

from . import paged_attention as pa

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Values (float64) of e4m3 codes (uint8)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    sub = (m / 8.0) * 2.0 ** -6
    norm = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    val = sign * np.where(e == 0, sub, norm)
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


def _all_finite_magnitudes() -> np.ndarray:
    codes = np.arange(0x7F, dtype=np.uint8)  # 0x00 .. 0x7E, ascending magnitude
    return e4m3_decode(codes)


_MAGS = _all_finite_magnitudes()


def e4m3_encode(x) -> np.ndarray:
    """Nearest e4m3 code of each float value (ties to even mantissa),
    saturating finite values to ±448; NaN maps to 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint8)
    flat, res = x.reshape(-1), out.reshape(-1)
    for i, v in enumerate(flat.tolist()):
        if v != v:
            res[i] = 0x7F
            continue
        sign = 0x80 if (v < 0 or (v == 0 and np.signbit(v))) else 0
        a = min(abs(v), E4M3_MAX)
        k = int(np.searchsorted(_MAGS, a))  # first magnitude >= a
        if k < len(_MAGS) and _MAGS[k] == a:
            code = k
        else:
            lo, hi = k - 1, k
            dlo, dhi = a - _MAGS[lo], _MAGS[hi] - a
            if dlo < dhi:
                code = lo
            elif dhi < dlo:
                code = hi
            else:  # tie: the even mantissa
                code = lo if (lo & 1) == 0 else hi
        res[i] = sign | code
    return out


def quantize_rows(rows: np.ndarray, scale: float) -> np.ndarray:
    """e4m3 codes of ``rows / scale`` as the append computes it: the fp32
    product with the fp32 reciprocal of the scale, then e4m3_encode."""
    inv = np.float32(1.0 / float(scale))
    prod = (np.asarray(rows, dtype=np.float32) * inv).astype(np.float32)
    return e4m3_encode(prod.astype(np.float64))


def paged_decode_attention_fp8(q, k_codes, v_codes, block_tables, seq_lens, scale, k_scale, v_scale,
                               q_dtype: str = "f16") -> np.ndarray:
    """Decode attention over e4m3 pools ``[NB, Hkv, bs, D]`` (uint8 codes):
    the same definition as paged_attention.paged_decode_attention on the
    dequantised values ``k_scale * e4m3(k)``, ``v_scale * e4m3(v)``."""
    kf = e4m3_decode(k_codes) * float(k_scale)
    vf = e4m3_decode(v_codes) * float(v_scale)
    qf = pa.to_f64(q, q_dtype)
    return pa.paged_decode_attention(qf, kf, vf, block_tables, seq_lens, scale, "f64")


def kv_append_fp8(k_codes, v_codes, k_rows, v_rows, slot_mapping, k_scale, v_scale):
    """The append into e4m3 pools: each new row is quantised (quantize_rows)
    and written into its slot; ``slot < 0`` writes nothing."""
    kq = quantize_rows(k_rows, k_scale)
    vq = quantize_rows(v_rows, v_scale)
    return pa.kv_append(k_codes, v_codes, kq, vq, slot_mapping)
