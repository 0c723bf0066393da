"""Element codecs of the oracle: 16-bit floats and the OCP 8-bit E4M3 format.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Caches hold raw bits: uint16 words for fp16/bf16, uint8 codes for e4m3.
The pages say only that an FP8 cache stores keys and values at 8-bit
precision and roughly halves the memory of a 16-bit cache ("PagedAttention",
Ultralytics glossary, §İlgili Teknikler, FP8 bullet).  They name no format,
rounding or scale, so the reading taken here is:

* format: OCP 8-bit floating point, E4M3 ("fn" variant): 1 sign bit, 4
  exponent bits with bias 7, 3 mantissa bits, subnormals when the exponent
  field is 0, no infinities, S.1111.111 is NaN, largest finite value 448;
* quantise: q = RNE_e4m3(fp32(x) / fp32(scale)), saturating finite overflow
  and +-inf to +-448 ("satfinite"); NaN maps to a NaN code (0x7F);
* dequantise: x = decode(q) * scale, with one per-tensor scale for K and one
  for V.

The division is taken in fp32, the precision in which the GPU kernel takes
it, because the resulting code is an integer decided by floating point.

Pins: ``e4m3_decode`` is checked exhaustively against the format's closed
form values (powers of two, 448, the subnormal ladder); decode->encode is
the identity on every finite code; ``e4m3_encode_f32`` agrees with the
library cast ``torch.float8_e4m3fn`` on random and edge values inside the
finite range, and saturates by definition outside it.  The 16-bit decoders
are checked against ``np.float16`` / ``torch.bfloat16`` conversions.
"""

from __future__ import annotations

import numpy as np

E4M3_BIAS = 7
E4M3_MAX = 448.0
E4M3_NAN_CODE = 0x7F


def f16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit patterns (uint16) -> float64 values (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64 values (exact).

    A bfloat16 word is the upper half of an IEEE binary32 word, so the value
    is the binary32 number whose high 16 bits are the word and whose low 16
    bits are zero.
    """
    w = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):  # NaN payloads pass through unchanged
        return w.view(np.float32).astype(np.float64)


def _e4m3_value(code: int) -> float:
    """Value of one E4M3 code from the format's definition."""
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        # subnormal: 2^(1 - bias) * (m / 8)
        return sign * (2.0 ** (1 - E4M3_BIAS)) * (m / 8.0)
    return sign * (2.0 ** (e - E4M3_BIAS)) * (1.0 + m / 8.0)


_E4M3_TABLE = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 E4M3 codes -> float64 values (exact; NaN codes give NaN)."""
    return _E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_finite_values() -> np.ndarray:
    """The 127 non-negative finite E4M3 values, ascending (codes 0x00..0x7E)."""
    return _E4M3_TABLE[:0x7F].copy()


def e4m3_encode_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to E4M3 codes: nearest value, ties to even code.

    Non-negative finite codes 0x00..0x7E are monotone in value, so the two
    neighbours of |x| are adjacent codes and "even" means the code's low bit
    (the mantissa's last bit) is 0.  Values at or beyond 448 (and +-inf)
    saturate to +-448.  The sign of x (also of -0.0 and of values that round
    to zero) becomes the code's sign bit.  NaN becomes code 0x7F.
    """
    xf = np.asarray(x, dtype=np.float32)
    a = np.abs(xf.astype(np.float64))
    vals = _E4M3_TABLE[:0x7F]
    out = np.empty(xf.shape, dtype=np.uint8)
    flat_a = a.reshape(-1)
    flat_o = out.reshape(-1)
    nan = np.isnan(flat_a)
    sat = ~nan & (flat_a >= E4M3_MAX)
    mid = ~nan & ~sat
    am = flat_a[mid]
    hi = np.searchsorted(vals, am, side="left")  # vals[hi-1] < am <= vals[hi]
    hi = np.clip(hi, 1, 0x7E)
    lo = hi - 1
    dlo = am - vals[lo]
    dhi = vals[hi] - am
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(am == vals[hi], hi, code)  # exact hits
    flat_o[mid] = code.astype(np.uint8)
    flat_o[sat] = 0x7E
    flat_o[nan] = E4M3_NAN_CODE
    neg = np.signbit(xf.reshape(-1)) & ~nan
    flat_o[neg] |= np.uint8(0x80)
    return out


def decode_cache(raw: np.ndarray, cache_dtype: str, scale: float = 1.0) -> np.ndarray:
    """Raw cache words -> float64 values.

    ``cache_dtype`` is one of ``"f16"``, ``"bf16"``, ``"e4m3"``; for e4m3 the
    decoded value is multiplied by the per-tensor ``scale`` in float64.
    """
    if cache_dtype == "f16":
        return f16_bits_to_f64(raw)
    if cache_dtype == "bf16":
        return bf16_bits_to_f64(raw)
    if cache_dtype == "e4m3":
        return e4m3_decode(raw) * float(scale)
    raise ValueError(f"unknown cache dtype {cache_dtype!r}")
