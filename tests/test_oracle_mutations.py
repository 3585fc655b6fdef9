"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch every one of them: a pin set that a dropped term, a wrong sign, a
swapped index or a transposed operand slips through would not be a pin."""

import math

import numpy as np
import pytest

from oracle import formats
from oracle import gdn as O
from pins import ALL_PINS


def _step_readout_before_write(S, q_hat, k_hat, v, alpha, beta):
    S = O.decay(S, alpha)
    o = O.readout(S, q_hat)
    v_old = O.delta_read(S, k_hat)
    S = O.delta_write(S, k_hat, O.delta_residual(v, v_old, beta))
    return o, S


def _step_read_before_decay(S, q_hat, k_hat, v, alpha, beta):
    v_old = O.delta_read(S, k_hat)
    S = O.decay(S, alpha)
    S = O.delta_write(S, k_hat, O.delta_residual(v, v_old, beta))
    return O.readout(S, q_hat), S


def _resolve_ignoring_new_page(page_indices, page_indptr, last_page_len, bb):
    last = int(page_indptr[bb + 1]) - 1
    return int(page_indices[last]), int(page_indices[last])


def _resolve_writing_old_page(page_indices, page_indptr, last_page_len, bb):
    r, w = _ORIG_RESOLVE(page_indices, page_indptr, last_page_len, bb)
    return r, r


_ORIG_RESOLVE = O.resolve_pages
_ORIG_SUFFIX = O.suffix_pages


def _suffix_read_too_late(page_indices, page_indptr, last_page_len, page_size, T, bb):
    """Reads the page of position L-T (the suffix's first token) instead of L-T-1."""
    read, snaps, final = _ORIG_SUFFIX(page_indices, page_indptr, last_page_len, page_size, T, bb)
    p0, p1 = int(page_indptr[bb]), int(page_indptr[bb + 1])
    L = (p1 - p0 - 1) * page_size + int(last_page_len[bb])
    return int(page_indices[p0 + (L - T) // page_size]), snaps, final
_ORIG_QUANT_TILE = formats.quantize_tile


def _tile_wrong_max(tile):
    t = np.asarray(tile, np.float32)
    amax = np.float32(np.max(np.abs(t)))
    if amax == 0:
        return np.zeros(t.shape, np.uint8), np.float32(0)
    s = np.float32(amax / np.float32(256.0))
    return formats.e4m3_encode((t * (np.float32(1) / s)).astype(np.float32)), s


def _e4m3_half_away(x):
    """Round half away from zero: nudge each value one binary32 ulp outwards."""
    x = np.asarray(x, np.float32)
    return _ORIG_E4M3(np.nextafter(x, np.sign(x) * np.inf).astype(np.float32))


_ORIG_E4M3 = formats.e4m3_encode
_ORIG_FWHT = formats.fwht32
_ORIG_H32_QUANT = formats.quantize_state_h32
_ORIG_H32_DEQUANT = formats.dequantize_state_h32


def _fwht_wrong_sign(x):
    """Butterfly (a + b, b - a) instead of (a + b, a - b)."""
    y = np.array(x, copy=True)
    lead = y.shape[:-1]
    span = 1
    while span < 32:
        y = y.reshape(lead + (32 // (2 * span), 2, span))
        a, b = y[..., 0, :].copy(), y[..., 1, :].copy()
        y[..., 0, :] = a + b
        y[..., 1, :] = b - a
        y = y.reshape(lead + (32,))
        span *= 2
    return y


def _h32_scales_128(amax):
    amax = np.asarray(amax, np.float32)
    with np.errstate(all="ignore"):
        s = (amax / np.float32(128)).astype(np.float32)
        r = (np.float32(1) / s).astype(np.float32)
    zero = ~(amax > 0) | ~np.isfinite(r)
    return np.where(zero, 0, s).astype(np.float32), np.where(zero, 0, r).astype(np.float32)


def _int8_half_away(y):
    y = np.asarray(y, np.float64)
    return np.clip(np.sign(y) * np.floor(np.abs(y) + 0.5), -127, 127).astype(np.int8)


def _h32_group_along_keys(S_kv):
    """Groups of 32 key channels per value column instead of 32 values per key channel."""
    S = np.asarray(S_kv, np.float32)
    K, V = S.shape
    if K % 32:
        c, s = _ORIG_H32_QUANT(S)
        return c, s[::-1].copy()
    c, s = _ORIG_H32_QUANT(np.ascontiguousarray(S.T))
    return c.T.copy(), s


def _h32_dequant_unrotated(codes_kv, scales):
    codes = np.asarray(codes_kv, np.int8)
    K, V = codes.shape
    sc = np.asarray(scales, np.float32).T
    return (codes.reshape(K, V // 32, 32).astype(np.float32) * sc[..., None]).astype(np.float32).reshape(K, V)

_ORIG_STEP_UNIT = O.step_unit


def _step_unit_stored_ignored(S0, tokens, state_dtype, readout_mode="working", block_v=64):
    """readout='stored' silently treated as 'working'."""
    return _ORIG_STEP_UNIT(S0, tokens, state_dtype, "working", block_v)


def _step_unit_encode_at_end(S0, tokens, state_dtype, readout_mode="working", block_v=64):
    """The state is carried at full precision between tokens; only what is
    stored (and read by a stored readout) passes through the format."""
    S = S0
    for (q_hat, k_hat, v, alpha, beta) in tokens:
        o, S = O.gated_delta_step(S, q_hat, k_hat, v, alpha, beta)
        S_st, payload = O.write_event(S, state_dtype, block_v)
        if readout_mode == "stored" and state_dtype != "f32":
            o = O.readout(S_st, q_hat)
        yield o, payload


MUTATIONS = {
    "stored_readout_ignored": (O, "step_unit", _step_unit_stored_ignored),
    "encode_after_last_token_only": (O, "step_unit", _step_unit_encode_at_end),
    "read_transposed": (O, "delta_read", lambda S, k: S @ k),
    "residual_sign": (O, "delta_residual", lambda v, v_old, beta: beta * (v_old - np.asarray(v, float))),
    "residual_no_beta": (O, "delta_residual", lambda v, v_old, beta: np.asarray(v, float) - v_old),
    "decay_dropped": (O, "decay", lambda S, alpha: S),
    "decay_value_axis": (O, "decay", lambda S, alpha: S * float(alpha) if np.ndim(alpha) == 0
                         else S * np.asarray(alpha)[None, :]),
    "write_transposed": (O, "delta_write", lambda S, k, u: S + np.outer(u, k)),
    "write_dropped": (O, "delta_write", lambda S, k, u: S),
    "readout_before_write": (O, "gated_delta_step", _step_readout_before_write),
    "read_before_decay": (O, "gated_delta_step", _step_read_before_decay),
    "gqa_modulo": (O, "key_head_of", lambda hv, H, HV: hv % H),
    "gate_sign": (O, "gdn_alpha", lambda A, a, d: math.exp(min(
        math.exp(float(A)) * float(O.softplus(float(a) + float(d))), 700.0))),
    "gate_no_dt_bias": (O, "gdn_alpha", lambda A, a, d: math.exp(-math.exp(float(A)) * float(O.softplus(float(a))))),
    "kda_gate_no_dt_bias": (O, "kda_alpha", lambda A, g, d: np.exp(-math.exp(float(A)) * O.softplus(np.asarray(g, float)))),
    "softplus_plain_relu": (O, "softplus", lambda x: np.maximum(np.asarray(x, float), 0.0)),
    "sigmoid_missing": (O, "sigmoid", lambda x: np.asarray(x, float)),
    "l2_no_eps_norm_sq": (O, "l2_normalize", lambda x: np.asarray(x, float) / (float(np.sum(np.asarray(x, float) ** 2)) + 1e-6)),
    "qk_scale_dropped": (O, "prepare_qk", lambda q, k, scale, use=True: (O.l2_normalize(q), O.l2_normalize(k))
                         if use else (np.asarray(q, float), np.asarray(k, float))),
    "new_page_ignored": (O, "resolve_pages", _resolve_ignoring_new_page),
    "write_to_read_page": (O, "resolve_pages", _resolve_writing_old_page),
    "suffix_read_too_late": (O, "suffix_pages", _suffix_read_too_late),
    "bf16_truncates": (formats, "f32_to_bf16_bits",
                       lambda x: (np.ascontiguousarray(np.asarray(x, np.float32)).view(np.uint32) >> 16).astype(np.uint16)),
    "e4m3_half_away": (formats, "e4m3_encode", _e4m3_half_away),
    "tile_scale_256": (formats, "quantize_tile", _tile_wrong_max),
    "h32_butterfly_sign": (formats, "fwht32", _fwht_wrong_sign),
    "h32_unnormalised": (formats, "hadamard32", lambda x: _ORIG_FWHT(np.asarray(x))),
    "h32_scale_128": (formats, "h32_scales", _h32_scales_128),
    "int8_half_away": (formats, "int8_round", _int8_half_away),
    "h32_group_along_keys": (formats, "quantize_state_h32", _h32_group_along_keys),
    "h32_decode_unrotated": (formats, "dequantize_state_h32", _h32_dequant_unrotated),
}


def _pins_fail():
    failed = []
    for pin in ALL_PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except Exception as e:  # an exception from a broken oracle counts as a catch
            failed.append(pin.__name__)
    return failed


def test_unmutated_oracle_passes_all_pins():
    assert _pins_fail() == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    mod, attr, fn = MUTATIONS[name]
    monkeypatch.setattr(mod, attr, fn)
    failed = _pins_fail()
    assert failed, f"planted mistake '{name}' passed every pin"
