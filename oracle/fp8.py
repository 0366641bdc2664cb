"""Oracle for FP8 (e4m3) K/V rows -- TEST INFRASTRUCTURE ONLY (imported by ``tests/`` alone).

The project page ("03 End-to-end KV transport", item 01 "Precision") sends the K/V in FP8 to halve
the transfer bytes (raw communication about 79 -> 40 ms in the 14B diagnostic), and converts them
back before attention.  The pages do not give the format variant or the scale granularity.  The
readings taken here:

* **Format: e4m3 "fn".** One sign bit, four exponent bits with bias 7, three mantissa bits.  There
  are no infinities, codes 0x7F and 0xFF are NaN, and the largest finite magnitude is
  1.75 * 2^8 = 448.
* **Encoding:** round to nearest, ties to the even code.  Magnitudes above 448 saturate to 448.
* **Scale:** one fp32 scale per (token, head) row of ``head_dim`` values.  Two chunks may share a
  page, so a per-page scale could not be fixed when the first of them is written.  For a row with
  largest magnitude ``amax > 0``: ``inv = 448 / amax`` and ``scale = amax / 448``, both fp32
  divisions, and ``code = e4m3(x * inv)`` with an fp32 product.  A row of zeros gets scale 0 and
  codes 0, and so does a row whose ``448 / amax`` overflows fp32 (``amax`` below about 1.3e-36):
  no scale could carry it back, and values that small mean nothing in bf16 K/V.  Every step is
  fp32, as on the device, because these values decide the integer codes.
* **Dequantization:** ``bf16_rne(fp32(decode(code)) * scale)``, which is what attention reads.

Every function is pinned by ``tests/test_oracle_fp8.py``: the value table against the format's
closed form, the encoder against PyTorch's own float8_e4m3fn cast and against brute force over all
codes, the saturation and tie cases, and the error bound of a quantize/dequantize round trip.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
NAN_CODE = 0x7F


def e4m3_values() -> np.ndarray:
    """Magnitude of every non-negative finite code 0x00..0x7E, in code order (ascending)."""
    vals = np.empty(127, np.float64)
    for code in range(127):
        e, m = code >> 3, code & 7
        vals[code] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_VALS = e4m3_values()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 codes -> float32 values (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8)
    mag = c & 0x7F
    out = np.where(mag == NAN_CODE, np.nan, _VALS[np.minimum(mag, 126)])
    return np.where(c & 0x80, -out, out).astype(np.float32)


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """float32 values -> uint8 codes: nearest representable magnitude, ties to the even code,
    saturating at 448; the sign is kept (also for results that round to zero)."""
    y = np.asarray(y, dtype=np.float32)
    a = np.abs(y).astype(np.float64)              # exact: every float32 is a float64
    hi = np.clip(np.searchsorted(_VALS, a, side="left"), 0, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _VALS[lo]
    d_hi = _VALS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(a >= E4M3_MAX, 126, code)     # saturate to the largest finite value
    sign = np.signbit(y).astype(np.int64) << 7
    return (code | sign).astype(np.uint8)


def quantize_rows(x) -> tuple:
    """x: [..., D] float32 (bf16 values widened) -> (codes uint8 [..., D], scale float32 [...])."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1).astype(np.float32)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1)).astype(np.float32)
    with np.errstate(over="ignore"):
        inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    # a row of zeros, or one so small that 448 / amax overflows fp32, is stored as zeros
    live = nz & np.isfinite(inv)
    inv = np.where(live, inv, np.float32(0)).astype(np.float32)
    scale = np.where(live, safe / np.float32(E4M3_MAX), np.float32(0)).astype(np.float32)
    y = (x * inv[..., None]).astype(np.float32)
    return e4m3_encode(y), scale


def dequantize_rows_f32(codes, scale) -> np.ndarray:
    """fp32 product decode(code) * scale (before the bf16 rounding)."""
    v = e4m3_decode(codes)
    return (v * np.asarray(scale, dtype=np.float32)[..., None]).astype(np.float32)


def dequantize_rows(codes, scale):
    """The bf16 rows attention reads: round-to-nearest-even of the fp32 product (a torch bf16
    tensor, so callers can compare its bits)."""
    import torch
    return torch.from_numpy(dequantize_rows_f32(codes, scale)).to(torch.bfloat16)
