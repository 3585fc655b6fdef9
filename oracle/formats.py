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

* int8_hadamard32 codec: the ModelOpt linear-attention config page
  (LinearAttentionConfig, and LinearAttentionDecodeConfig ``state_codec``)
  says only that this decode codec fixes its scales to one key channel and
  32 values, while ``block_v`` stays the execution tile width. The rest is
  the plainest reading of the name, stated here once:

      x     = S[k, 32 g : 32 g + 32]       (one key channel, 32 values)
      y     = R x,  R = H32 / sqrt(32)     (H32 the Sylvester Hadamard matrix,
                                            natural order; R is symmetric and
                                            orthonormal, so R R = I)
      amax  = max |y|;  s = amax / 127;  r = 1 / s      (binary32)
      code  = clamp(rint(y * r), -127, 127) as int8     (binary32 product,
                                                         ties to even)
      x'    = R (code * s)                 (binary32 product, then R)

  so the stored scale array is ``[V / 32, K]`` per state (group-major). R is
  applied in binary32 by the butterfly of the fast Walsh-Hadamard transform:
  stages of span 1, 2, 4, 8, 16, each turning the pair at (i, i + span),
  ``i & span == 0``, into (a + b, a - b), then one product with the binary32
  nearest to 1/sqrt(32) (bit pattern 0x3E3504F3, exactly a quarter of the
  nearest binary32 to 1/sqrt(2)). Every codec decision is thereby a binary32
  computation with one fixed rounding order. A group whose ``amax`` is 0, or
  whose ``r`` overflows binary32, stores scale 0 and codes 0. For finite
  inputs ``|y * r|`` stays below 127.5, so the clamp never changes a code.

Every function here works on numpy arrays and uses numpy's IEEE binary32 and
binary64 arithmetic; nothing is shared with the CUDA path.
"""

from __future__ import annotations

import math

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


# ----------------------------------------------------------------------------
# int8_hadamard32: one scale per key channel and 32 values, after a
# Walsh-Hadamard rotation of the 32 values
# ----------------------------------------------------------------------------

H32 = 32
INT8_CODE_MAX = 127
INV_SQRT32_F32 = np.array([0x3E3504F3], dtype=np.uint32).view(np.float32)[0]


def fwht32(x: np.ndarray) -> np.ndarray:
    """Unnormalised 32-point Walsh-Hadamard transform along the last axis.

    Natural (Sylvester) order, computed in the dtype of ``x`` by butterfly
    stages of span 1, 2, 4, 8, 16: the pair (a, b) at positions (i, i + span)
    with ``i & span == 0`` becomes (a + b, a - b).
    """
    y = np.array(x, copy=True)
    if y.shape[-1] != H32:
        raise ValueError("last axis must hold 32 values")
    lead = y.shape[:-1]
    span = 1
    while span < H32:
        y = y.reshape(lead + (H32 // (2 * span), 2, span))
        a = y[..., 0, :].copy()
        b = y[..., 1, :].copy()
        y[..., 0, :] = a + b
        y[..., 1, :] = a - b
        y = y.reshape(lead + (H32,))
        span *= 2
    return y


def hadamard32(x: np.ndarray) -> np.ndarray:
    """The orthonormal rotation R = H32 / sqrt(32) along the last axis.

    binary32 input: the binary32 butterflies, then one binary32 product with
    the nearest binary32 to 1/sqrt(32). Any other input: float64 throughout.
    """
    x = np.asarray(x)
    if x.dtype == np.float32:
        return (fwht32(x) * INV_SQRT32_F32).astype(np.float32)
    return fwht32(x.astype(np.float64)) * (1.0 / math.sqrt(32.0))


def h32_scales(amax: np.ndarray):
    """Per-group (s, r) in binary32 from the groups' amax; groups stored as
    zeros get s = 0 and r = 0."""
    amax = np.asarray(amax, dtype=np.float32)
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        s = (amax / np.float32(INT8_CODE_MAX)).astype(np.float32)
        r = (np.float32(1.0) / s).astype(np.float32)
    zero = ~(amax > 0) | ~np.isfinite(r)
    return np.where(zero, np.float32(0), s).astype(np.float32), np.where(zero, np.float32(0), r).astype(np.float32)


def int8_round(y: np.ndarray) -> np.ndarray:
    """binary32 values -> int8 codes: nearest integer, ties to even, clamped
    to [-127, 127]."""
    return np.clip(np.rint(np.asarray(y, np.float64)), -INT8_CODE_MAX, INT8_CODE_MAX).astype(np.int8)


def quantize_rotated_groups(y: np.ndarray):
    """Rotated groups ``y [..., 32]`` (binary32) -> (codes int8 [..., 32], scales [...])."""
    y = np.asarray(y, np.float32)
    amax = np.max(np.abs(y), axis=-1)
    s, r = h32_scales(amax)
    codes = int8_round((y * r[..., None]).astype(np.float32))
    return codes, s


def quantize_state_h32(S_kv: np.ndarray):
    """Encode a logical [K, V] state: codes int8 [K, V] (rotated groups in
    place of the values) and scales [V / 32, K] binary32."""
    S = np.asarray(S_kv, dtype=np.float32)
    K, V = S.shape
    if V % H32:
        raise ValueError("V must be a multiple of 32")
    y = hadamard32(S.reshape(K, V // H32, H32))
    codes, s = quantize_rotated_groups(y)
    return codes.reshape(K, V), np.ascontiguousarray(s.T)


def dequantize_state_h32(codes_kv: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Decode a logical [K, V] int8 code array with its [V / 32, K] scales -> binary32."""
    codes = np.asarray(codes_kv, dtype=np.int8)
    K, V = codes.shape
    sc = np.asarray(scales, np.float32).T               # [K, V / 32]
    yq = (codes.reshape(K, V // H32, H32).astype(np.float32) * sc[..., None]).astype(np.float32)
    return hadamard32(yq).reshape(K, V)
