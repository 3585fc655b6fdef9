"""Storage formats of the recurrent state, written from the format definitions.

Test infrastructure only (see ``oracle/__init__.py``).

* bf16: the upper half of an IEEE-754 binary32 word (1 sign, 8 exponent,
  7 fraction bits). Rounding from binary32 is round-to-nearest, ties to even.
* fp8 E4M3 (OCP 8-bit floating point, "E4M3" variant): 1 sign bit, 4 exponent
  bits with bias 7, 3 fraction bits. Exponent field 0 holds subnormals
  ``m * 2**-9``; fields 1..15 hold ``(1 + m/8) * 2**(e-7)``; the pattern with
  exponent 15 and fraction 7 is NaN; there is no infinity, so the largest finite
  magnitude is ``1.75 * 2**8 = 448``.
* Tile codec: one dynamic scale per ``[K, block_v]`` tile of each
  (sequence, head) state, as the ModelOpt linear-attention config page states
  for ``state.block_v`` (LinearAttentionConfig), with ``fp8_e4m3`` the decode
  default (``recurrent_decode``: ``state_format='fp8_e4m3', block_v=64``).
  The pages fix neither the scale formula nor the rounding, so the codec is
  the plainest reading, done in binary32 so that it is exactly reproducible:

      amax  = max |x| over the tile
      s     = amax / 448            (binary32 division, round to nearest even)
      r     = 1 / s                 (binary32 division)
      code  = E4M3(x * r)           (binary32 product, then round to nearest
                                     even onto the E4M3 grid, saturating to
                                     +-448)
      x'    = value(code) * s       (binary32 product)

  A tile whose ``amax`` is 0, or whose ``r`` overflows binary32 (amax below
  about 1.3e-36), is stored as scale 0 with all codes +0 and decodes to 0.

Every function here works on numpy arrays and uses numpy's IEEE binary32 and
binary64 arithmetic; nothing is shared with the CUDA path.
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_NAN_CODE = 0x7F


# ----------------------------------------------------------------------------
# bf16
# ----------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact binary32 values."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """binary32 -> bf16 bit patterns, round to nearest, ties to even.

    Dropping the low 16 bits of the binary32 word keeps 7 fraction bits. To
    round to nearest-even, add ``0x7FFF`` plus the lowest kept bit before
    truncating: a remainder above half carries into the kept part, one below
    half does not, and an exact half carries only when the kept part is odd.
    The carry propagates into the exponent where it must (including the
    overflow of the largest finite values to infinity). NaN stays NaN.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        rounded = np.where(nan, ((u >> np.uint64(16)) | np.uint64(0x40)).astype(np.uint16), rounded)
    return rounded


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round binary32 values to the nearest bf16 value (returned as binary32)."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# ----------------------------------------------------------------------------
# fp8 E4M3
# ----------------------------------------------------------------------------

def e4m3_value(code: np.ndarray) -> np.ndarray:
    """Decode E4M3 codes (uint8) to their exact values as binary64."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """binary32 -> E4M3 code, round to nearest with ties to even, saturating.

    For a finite magnitude ``a``, the grid step at ``a`` is ``2**(E-3)`` where
    ``E = max(floor(log2 a), -6)`` (the subnormal range shares the step of the
    smallest normal binade). ``a / step`` is exact (power-of-two scaling), so
    ``rint`` (round half to even) gives the nearest grid point exactly.
    Magnitudes past 448 (and infinities) saturate to 448; NaN maps to the NaN
    code 0x7F.
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    finite_pos = np.isfinite(a) & (a > 0)
    safe = np.where(finite_pos, a, 1.0)
    _, ex = np.frexp(safe)               # safe = f * 2**ex, f in [0.5, 1)
    E = np.maximum(ex - 1, -6)
    step = np.exp2((E - 3).astype(np.float64))
    q = np.rint(safe / step)             # grid index inside the binade
    # q == 16 means the value rounded up into the next binade: 16 * 2**(E-3)
    # is 8 * 2**(E-2), the first point of binade E+1.
    E = np.where(q == 16, E + 1, E)
    q = np.where(q == 16, 8, q)
    sub = q < 8                          # only possible when E == -6
    exp_field = np.where(sub, 0, E + 7)
    frac = np.where(sub, q, q - 8)
    code = (exp_field.astype(np.int64) << 3) | frac.astype(np.int64)
    # saturate: anything beyond the largest finite (field 15, fraction 6)
    code = np.where((exp_field > 15) | ((exp_field == 15) & (frac > 6)), 0x7E, code)
    code = np.where(np.isinf(a), 0x7E, code)
    code = np.where(a == 0, 0, code)
    code = np.where(np.isnan(x), E4M3_NAN_CODE, code)
    neg = np.signbit(x) & ~np.isnan(x)
    code = np.where(neg, code | 0x80, code)
    return code.astype(np.uint8)


# ----------------------------------------------------------------------------
# Tile codec: one scale per [K, block_v] tile
# ----------------------------------------------------------------------------

def tile_scale_and_reciprocal(amax: np.float32):
    """Return (s, r) in binary32, or (0, None) for a tile stored as zeros."""
    amax = np.float32(amax)
    if amax == 0:
        return np.float32(0.0), None
    s = np.float32(amax / np.float32(E4M3_MAX))
    with np.errstate(over="ignore", divide="ignore"):
        r = np.float32(np.float32(1.0) / s)
    if not np.isfinite(r):
        return np.float32(0.0), None
    return s, r


def quantize_tile(tile: np.ndarray):
    """Encode one tile (any shape, binary32) -> (codes uint8, scale binary32)."""
    t = np.asarray(tile, dtype=np.float32)
    amax = np.float32(np.max(np.abs(t))) if t.size else np.float32(0)
    s, r = tile_scale_and_reciprocal(amax)
    if r is None:
        return np.zeros(t.shape, dtype=np.uint8), np.float32(0.0)
    y = (t * r).astype(np.float32)       # binary32 product, round to nearest even
    return e4m3_encode(y), s


def dequantize_tile(codes: np.ndarray, scale) -> np.ndarray:
    """Decode one tile -> binary32 values ``value(code) * s``."""
    vals = e4m3_value(codes).astype(np.float32)   # every finite E4M3 value is exact in binary32
    return (vals * np.float32(scale)).astype(np.float32)


def quantize_state(S_kv: np.ndarray, block_v: int):
    """Encode a logical [K, V] state: returns codes [K, V] and scales [V/block_v]."""
    S = np.asarray(S_kv, dtype=np.float32)
    K, V = S.shape
    if V % block_v:
        raise ValueError("block_v must divide V")
    codes = np.zeros((K, V), dtype=np.uint8)
    scales = np.zeros(V // block_v, dtype=np.float32)
    for j in range(V // block_v):
        c, s = quantize_tile(S[:, j * block_v:(j + 1) * block_v])
        codes[:, j * block_v:(j + 1) * block_v] = c
        scales[j] = s
    return codes, scales


def dequantize_state(codes_kv: np.ndarray, scales: np.ndarray, block_v: int) -> np.ndarray:
    """Decode a logical [K, V] code array with its [V/block_v] scales -> binary32."""
    codes = np.asarray(codes_kv, dtype=np.uint8)
    K, V = codes.shape
    out = np.zeros((K, V), dtype=np.float32)
    for j in range(V // block_v):
        out[:, j * block_v:(j + 1) * block_v] = dequantize_tile(
            codes[:, j * block_v:(j + 1) * block_v], scales[j])
    return out
