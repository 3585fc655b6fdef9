"""Plain float64 CPU oracle of gated delta-rule decode over a state pool.

Test infrastructure only (see ``oracle/__init__.py``). Slow by design: one
(sequence, value head) at a time, one token at a time, in the literal order
the pages give, so that a reader can check each line against them.

Sources, by page and section:

* Circuit.LLM.Mixer, "Delta rule" (``deltaAttnStep``): with S right-acting
  (``o = q S``; rows of S index the key dimension), one step is
  ``v_old = k S``, ``u = beta (v - v_old)``, ``S' = S + k^T u``, ``o = q S'``.
* Circuit.LLM.Mixer, "Gated memory" (``gatedDeltaStep``): decay first,
  ``S <- alpha S``, then the delta step; ``kdaLiteStep``: the decay is a
  vector over the key channels (each key row of S is scaled by its own alpha).
  ``scanMixer`` / ``gatedDeltaPrefill``: a sequence is the steps in order.
* flashinfer.gdn_paged.gated_delta_rule_decode_paged: q/k L2-normalised when
  ``use_qk_l2norm`` (default True); ``scale=None``; the copy-on-new-page rule
  of the description paragraph; ``state_pool [num_pages, HV, V, K]``;
  ``last_page_len`` includes the decoded token; Notes: a new-page sequence
  owns at least two pages.
* max.nn.state_space.kda_decode: q and k L2-normalised and q scaled by
  ``1/sqrt(key_head_dim)`` in the op; per-key-channel gate from ``raw_gate``
  "before dt_bias is added", ``a_log [HV]``, ``dt_bias [HV, K]``;
  ``beta_mode`` logits (sigmoid applied) or probability (used as is);
  ``cu_seqlens`` exclusive prefix offsets; ``state_layout`` K_FIRST/V_FIRST.
* modelopt.torch.quantization.linear_attention.decode
  (``recurrent_decode_reference``): a state write event per token; an empty
  call performs no write. ...linear_attention.config
  (LinearAttentionDecodeConfig ``readout``: ``working`` or ``stored``).

Readings where the pages are silent (each one is a convention, not a pin):

* L2 norm: ``x / sqrt(sum x^2 + 1e-6)``.
* softplus: ``max(x, 0) + log1p(exp(-|x|))`` with no threshold.
* GDN gate: ``alpha = exp(-exp(A_log[hv]) * softplus(a + dt_bias[hv]))``;
  KDA applies the same form per key channel with ``dt_bias[hv, i]``.
* ``beta = sigmoid(b) = 1 / (1 + exp(-b))``.
* default ``scale = 1/sqrt(K)`` (the KDA page's value; the GDN page's
  ``scale=None``).
* GQA: value head ``hv`` reads key head ``hv // (HV // H)``.
* padded entries: a negative slot index (or an index past the pool) skips the
  unit: output 0, nothing written.
* state storage per token: fp32 states keep full precision across a
  multi-token call (the oracle holds float64); bf16 states are rounded to
  bf16 after every token; fp8 and int8_hadamard32 states are re-encoded
  after every token.
  ``readout='working'`` reads ``o`` from the state before that rounding,
  ``'stored'`` after it.

Layouts: ``K_FIRST`` stores a state as ``[K][V]`` (V contiguous), ``V_FIRST``
as ``[V][K]`` (K contiguous, the paged pool's ``[num_pages, HV, V, K]``).
"""

from __future__ import annotations

import math
from typing import Callable, Dict, Iterable, Optional, Tuple

import numpy as np

from . import formats

L2NORM_EPS = 1e-6
LAYOUTS = ("K_FIRST", "V_FIRST")
STATE_DTYPES = ("f32", "bf16", "fp8_e4m3", "int8_hadamard32")


# ----------------------------------------------------------------------------
# token prologue: activations
# ----------------------------------------------------------------------------

def softplus(x):
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def l2_normalize(x):
    x = np.asarray(x, dtype=np.float64)
    return x / math.sqrt(float(np.sum(x * x)) + L2NORM_EPS)


def gdn_alpha(A_log_h, a_t, dt_bias_h):
    """Scalar decay of one (token, value head): exp(-exp(A_log) softplus(a + dt_bias))."""
    g = -math.exp(float(A_log_h)) * float(softplus(float(a_t) + float(dt_bias_h)))
    return math.exp(g)


def kda_alpha(a_log_h, raw_gate_t, dt_bias_h):
    """Per-key-channel decay vector [K] of one (token, value head)."""
    g = -math.exp(float(a_log_h)) * softplus(np.asarray(raw_gate_t, np.float64)
                                             + np.asarray(dt_bias_h, np.float64))
    return np.exp(g)


def beta_of(b_t, beta_mode="logits"):
    if beta_mode == "logits":
        return float(sigmoid(float(b_t)))
    if beta_mode == "probability":
        return float(b_t)
    raise ValueError(beta_mode)


def prepare_qk(q, k, scale, use_qk_l2norm=True):
    """Return (q_hat, k_hat): optionally L2-normalised, q multiplied by scale."""
    if use_qk_l2norm:
        return l2_normalize(q) * scale, l2_normalize(k)
    return np.asarray(q, np.float64) * scale, np.asarray(k, np.float64)


# ----------------------------------------------------------------------------
# the recurrence (Circuit.LLM.Mixer, "Delta rule" and "Gated memory")
# ----------------------------------------------------------------------------

def decay(S, alpha):
    """S <- alpha S. A scalar scales all of S; a [K] vector scales each key row."""
    alpha = np.asarray(alpha, dtype=np.float64)
    if alpha.ndim == 0:
        return float(alpha) * S
    return alpha[:, None] * S


def delta_read(S, k_hat):
    """v_old = k S: what the key already retrieves (k is a row vector, S is [K, V])."""
    return k_hat @ S


def delta_residual(v, v_old, beta):
    """u = beta (v - v_old)."""
    return beta * (np.asarray(v, np.float64) - v_old)


def delta_write(S, k_hat, u):
    """S' = S + k^T u (outer product of the key column and the update row)."""
    return S + np.outer(k_hat, u)


def readout(S, q_hat):
    """o = q S."""
    return q_hat @ S


def gated_delta_step(S, q_hat, k_hat, v, alpha, beta):
    """One gated delta step on a float64 [K, V] state: decay, read, write, read out."""
    S = decay(S, alpha)
    v_old = delta_read(S, k_hat)
    u = delta_residual(v, v_old, beta)
    S = delta_write(S, k_hat, u)
    o = readout(S, q_hat)
    return o, S


# ----------------------------------------------------------------------------
# stored state <-> float64 [K, V]
# ----------------------------------------------------------------------------

def _to_kv(stored2d, layout):
    if layout == "K_FIRST":
        return stored2d
    if layout == "V_FIRST":
        return stored2d.T
    raise ValueError(layout)


def _from_kv(kv2d, layout):
    return np.ascontiguousarray(_to_kv(kv2d, layout))   # the transpose is its own inverse


def load_state(stored2d, layout, state_dtype, scales=None, block_v=64):
    """Decode one stored (slot, head) state to a C-ordered float64 [K, V]
    array (the same memory order whatever the layout, so that the products
    that follow sum in the same order as on a state carried between tokens)."""
    return np.ascontiguousarray(_load_state_any_order(stored2d, layout, state_dtype, scales, block_v))


def _load_state_any_order(stored2d, layout, state_dtype, scales, block_v):
    if state_dtype == "f32":
        kv = np.asarray(stored2d, np.float32)
        return _to_kv(kv, layout).astype(np.float64)
    if state_dtype == "bf16":
        kv = formats.bf16_bits_to_f32(stored2d)
        return _to_kv(kv, layout).astype(np.float64)
    if state_dtype == "fp8_e4m3":
        codes_kv = _to_kv(np.asarray(stored2d, np.uint8), layout)
        return formats.dequantize_state(codes_kv, np.asarray(scales, np.float32),
                                        block_v).astype(np.float64)
    if state_dtype == "int8_hadamard32":
        codes_kv = _to_kv(np.asarray(stored2d, np.int8), layout)
        return formats.dequantize_state_h32(codes_kv, scales).astype(np.float64)
    raise ValueError(state_dtype)


def write_event(S, state_dtype, block_v=64):
    """Round a float64 state the way its storage does after one token.

    Returns (S_stored_as_float64, payload) where payload is what is written
    to the pool: fp32 array, bf16 bits, or (codes, scales) for fp8 and
    int8_hadamard32.
    """
    if state_dtype == "f32":
        s32 = S.astype(np.float32)
        return s32.astype(np.float64), s32
    if state_dtype == "bf16":
        bits = formats.f32_to_bf16_bits(S.astype(np.float32))
        return formats.bf16_bits_to_f32(bits).astype(np.float64), bits
    if state_dtype == "fp8_e4m3":
        codes, scales = formats.quantize_state(S.astype(np.float32), block_v)
        deq = formats.dequantize_state(codes, scales, block_v)
        return deq.astype(np.float64), (codes, scales)
    if state_dtype == "int8_hadamard32":
        codes, scales = formats.quantize_state_h32(S.astype(np.float32))
        deq = formats.dequantize_state_h32(codes, scales)
        return deq.astype(np.float64), (codes, scales)
    raise ValueError(state_dtype)


def store_state(payload, layout, state_dtype):
    """Payload from ``write_event`` -> (stored 2-D array in the layout, scales or None)."""
    if state_dtype in ("fp8_e4m3", "int8_hadamard32"):
        codes, scales = payload
        return _from_kv(codes, layout), scales
    return _from_kv(payload, layout), None


# ----------------------------------------------------------------------------
# one (sequence, value head) over its tokens
# ----------------------------------------------------------------------------

def step_unit(S0, tokens, state_dtype, readout_mode="working", block_v=64):
    """Run one state over its tokens, yielding (o, payload) after every token.

    ``S0``: float64 [K, V] (already decoded). ``tokens``: iterable of
    ``(q_hat, k_hat, v, alpha, beta)``. ``payload`` is what the pool would
    hold if the state were stored right then. fp32 states carry float64
    between tokens (a stored copy is rounded once); bf16 and coded states pass
    through their storage after every token (a write event).
    """
    S = S0
    for (q_hat, k_hat, v, alpha, beta) in tokens:
        o, S = gated_delta_step(S, q_hat, k_hat, v, alpha, beta)
        if state_dtype == "f32":
            _, payload = write_event(S, "f32")
        else:
            S, payload = write_event(S, state_dtype, block_v)
            if readout_mode == "stored":
                o = readout(S, q_hat)
        yield o, payload


def run_unit(S0, tokens, state_dtype, readout_mode="working", block_v=64):
    """All of a unit's tokens: (outputs [T, V], final payload or None when
    there are no tokens)."""
    outs, payload = [], None
    for o, payload in step_unit(S0, tokens, state_dtype, readout_mode, block_v):
        outs.append(o)
    if not outs:
        return np.zeros((0, S0.shape[1])), None
    return np.stack(outs), payload


def key_head_of(hv, H, HV):
    """Key head read by value head hv: each key head serves HV/H consecutive value heads."""
    return hv // (HV // H)


def _scale_of(scale, K):
    return 1.0 / math.sqrt(K) if (scale is None or scale <= 0) else float(scale)


# ----------------------------------------------------------------------------
# GDN on a slot pool: B sequences, T tokens each
# ----------------------------------------------------------------------------

def gdn_decode_slots(q, k, v, a, b, A_log, dt_bias, state_pool, state_indices, *,
                     layout="V_FIRST", state_dtype="f32", state_scales=None,
                     block_v=64, scale=None, use_qk_l2norm=True,
                     readout_mode="working", num_slots=None, units=None):
    """GDN decode of B sequences with T tokens each against a slot pool.

    q, k: [B, T, H, K]; v: [B, T, HV, V]; a, b: [B, T, HV]; A_log, dt_bias:
    [HV]; state_pool[slot, hv] -> stored 2-D state (f32 array, bf16 bits,
    fp8 or int8 codes); state_scales[slot, hv] -> [V/block_v] (fp8) or
    [V/32, K] (int8_hadamard32); state_indices [B].

    Returns (out [B, T, HV, V] float64, writes) where writes maps
    (slot, hv) -> (stored 2-D array, scales or None). ``units`` restricts the
    work to an iterable of (b, hv) pairs (other outputs are NaN).
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64); a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    sc = _scale_of(scale, K)
    out = np.full((B, T, HV, V), np.nan) if units is not None else np.zeros((B, T, HV, V))
    writes: Dict[Tuple[int, int], tuple] = {}
    todo = [(bb, hv) for bb in range(B) for hv in range(HV)] if units is None else list(units)
    for (bb, hv) in todo:
        slot = int(state_indices[bb])
        if slot < 0 or (num_slots is not None and slot >= num_slots):
            out[bb, :, hv, :] = 0.0
            continue
        h = key_head_of(hv, H, HV)
        S0 = load_state(state_pool[slot, hv], layout, state_dtype,
                        None if state_scales is None else state_scales[slot, hv], block_v)
        toks = []
        for t in range(T):
            qh, kh = prepare_qk(q[bb, t, h], k[bb, t, h], sc, use_qk_l2norm)
            toks.append((qh, kh, v[bb, t, hv], gdn_alpha(A_log[hv], a[bb, t, hv], dt_bias[hv]),
                         beta_of(b[bb, t, hv])))
        o, payload = run_unit(S0, toks, state_dtype, readout_mode, block_v)
        if payload is None:
            continue
        out[bb, :, hv, :] = o
        writes[(slot, hv)] = store_state(payload, layout, state_dtype)
    return out, writes


# ----------------------------------------------------------------------------
# GDN on a paged pool, one token (flashinfer.gdn_paged.gated_delta_rule_decode_paged)
# ----------------------------------------------------------------------------

def resolve_pages(page_indices, page_indptr, last_page_len, bb):
    """(read_page, write_page) of sequence bb by the copy-on-new-page rule.

    The decoded token sits in the sequence's last page. If it opens that page
    (last_page_len == 1) the state is read from the page before and written
    to the new page; otherwise the last page is read and written in place.
    """
    last = int(page_indptr[bb + 1]) - 1
    write = int(page_indices[last])
    if int(last_page_len[bb]) == 1:
        if last - 1 < int(page_indptr[bb]):
            raise ValueError("a sequence that opens a new page must own at least two pages")
        read = int(page_indices[last - 1])
    else:
        read = write
    return read, write


def suffix_pages(page_indices, page_indptr, last_page_len, page_size, T, bb):
    """Pages a T-token suffix of sequence bb touches.

    The sequence holds L = (pages - 1) * page_size + last_page_len tokens;
    the suffix is its last T tokens (positions L-T .. L-1) and at least one
    token precedes it. A page holds the state after its last token, so the
    state is read from the page of position L-T-1, every page whose last
    position falls inside the suffix (except the last page) receives the
    state after that position, and the final state goes to the last page.
    For T == 1 this is the copy-on-new-page rule.
    Returns (read_page, [(t, page)], last_page) with t the suffix index
    after which the snapshot is taken.
    """
    p0, p1 = int(page_indptr[bb]), int(page_indptr[bb + 1])
    npg = p1 - p0
    L = (npg - 1) * page_size + int(last_page_len[bb])
    if npg < 1 or L < T + 1:
        raise ValueError("a suffix needs at least one token before it")
    read = int(page_indices[p0 + (L - T - 1) // page_size])
    snaps = [(t, int(page_indices[p0 + (L - T + t) // page_size])) for t in range(T - 1)
             if (L - T + t) % page_size == page_size - 1]
    return read, snaps, int(page_indices[p1 - 1])


def gdn_decode_paged(q, k, v, a, b, A_log, dt_bias, state_pool, page_indices, page_indptr,
                     last_page_len, *, state_dtype="f32", state_scales=None, block_v=64,
                     scale=None, use_qk_l2norm=True, readout_mode="working", slots=None,
                     units=None, page_size=None, layout="V_FIRST"):
    """GDN decode of the last T tokens of each sequence on a paged pool
    (stored ``[num_pages, HV, V, K]`` for V_FIRST).

    q, k: [B, T, H, K]; v: [B, T, HV, V]; a, b: [B, T, HV]. T == 1 follows
    the copy-on-new-page rule and needs no page_size; ``slots``, when given
    for T == 1, is a [B, 2] array of (read_page, write_page) used as is (the
    page says precomputed rows are not checked against the page table).
    T > 1 needs page_size and writes a snapshot to every page that fills up
    inside the suffix (``suffix_pages``).
    Returns (out [B, T, HV, V], writes keyed by (page, hv)).
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64); a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    if T > 1 and not page_size:
        raise ValueError("a multi-token suffix needs page_size")
    sc = _scale_of(scale, K)
    out = np.full((B, T, HV, V), np.nan) if units is not None else np.zeros((B, T, HV, V))
    writes = {}
    todo = [(bb, hv) for bb in range(B) for hv in range(HV)] if units is None else list(units)
    for (bb, hv) in todo:
        if T == 1:
            if slots is not None:
                read, write = int(slots[bb][0]), int(slots[bb][1])
            else:
                read, write = resolve_pages(page_indices, page_indptr, last_page_len, bb)
            snaps = []
        else:
            read, snaps, write = suffix_pages(page_indices, page_indptr, last_page_len, page_size, T, bb)
        h = key_head_of(hv, H, HV)
        S0 = load_state(state_pool[read, hv], layout, state_dtype,
                        None if state_scales is None else state_scales[read, hv], block_v)
        toks = []
        for t in range(T):
            qh, kh = prepare_qk(q[bb, t, h], k[bb, t, h], sc, use_qk_l2norm)
            toks.append((qh, kh, v[bb, t, hv], gdn_alpha(A_log[hv], a[bb, t, hv], dt_bias[hv]),
                         beta_of(b[bb, t, hv])))
        snap_at = dict(snaps)
        for t, (o, payload) in enumerate(step_unit(S0, toks, state_dtype, readout_mode, block_v)):
            out[bb, t, hv, :] = o
            if t in snap_at:
                writes[(snap_at[t], hv)] = store_state(payload, layout, state_dtype)
        writes[(write, hv)] = store_state(payload, layout, state_dtype)
    return out, writes


def gdn_prefill_paged(q, k, v, a, b, A_log, dt_bias, cu_seqlens, state_pool, page_indices, page_indptr,
                      last_page_len, page_size, *, state_dtype="f32", state_scales=None, block_v=64,
                      scale=None, use_qk_l2norm=True, readout_mode="working", layout="V_FIRST",
                      units=None):
    """Append varlen token runs to paged sequences (prefill, or continued prefill).

    Sequence bb gets n = cu_seqlens[bb+1] - cu_seqlens[bb] new tokens, the
    last n of its L tokens (L from the page table). The sequence is the scan
    of single steps over them (Circuit.LLM.Mixer, scanMixer /
    gatedDeltaPrefill). The state starts from zero when the sequence has no
    earlier token (L == n), else from the page of position L-n-1; every page
    that fills inside the run keeps the state after its last token, the
    final state goes to the last page (``suffix_pages``). q, k: [total, H,
    K]; v: [total, HV, V]; a, b: [total, HV].
    Returns (out [total, HV, V], writes keyed by (page, hv)).
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64); a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    total, H, K = q.shape
    HV, V = v.shape[1], v.shape[2]
    sc = _scale_of(scale, K)
    B = len(cu_seqlens) - 1
    out = np.full((total, HV, V), np.nan) if units is not None else np.zeros((total, HV, V))
    writes = {}
    todo = [(bb, hv) for bb in range(B) for hv in range(HV)] if units is None else list(units)
    for (bb, hv) in todo:
        bos, eos = int(cu_seqlens[bb]), int(cu_seqlens[bb + 1])
        n = eos - bos
        if n == 0:
            continue
        p0, p1 = int(page_indptr[bb]), int(page_indptr[bb + 1])
        L = (p1 - p0 - 1) * page_size + int(last_page_len[bb])
        if L == n:       # a fresh sequence: the state starts at zero
            S0 = np.zeros((K, V))
            snaps = [(t, int(page_indices[p0 + t // page_size])) for t in range(n - 1)
                     if t % page_size == page_size - 1]
            final = int(page_indices[p1 - 1])
        else:
            read, snaps, final = suffix_pages(page_indices, page_indptr, last_page_len, page_size, n, bb)
            S0 = load_state(state_pool[read, hv], layout, state_dtype,
                            None if state_scales is None else state_scales[read, hv], block_v)
        h = key_head_of(hv, H, HV)
        toks = []
        for t in range(bos, eos):
            qh, kh = prepare_qk(q[t, h], k[t, h], sc, use_qk_l2norm)
            toks.append((qh, kh, v[t, hv], gdn_alpha(A_log[hv], a[t, hv], dt_bias[hv]), beta_of(b[t, hv])))
        snap_at = dict(snaps)
        for t, (o, payload) in enumerate(step_unit(S0, toks, state_dtype, readout_mode, block_v)):
            out[bos + t, hv, :] = o
            if t in snap_at:
                writes[(snap_at[t], hv)] = store_state(payload, layout, state_dtype)
        writes[(final, hv)] = store_state(payload, layout, state_dtype)
    return out, writes


def paged_decode_slots(page_indices, page_indptr, last_page_len):
    """[B, 2] int64 rows (read_page, write_page) for every sequence of the table."""
    B = len(page_indptr) - 1
    return np.array([resolve_pages(page_indices, page_indptr, last_page_len, bb)
                     for bb in range(B)], dtype=np.int64).reshape(B, 2)


# ----------------------------------------------------------------------------
# KDA, varlen, slot pool (max.nn.state_space.kda_decode)
# ----------------------------------------------------------------------------

def kda_decode_varlen(q, k, v, raw_gate, beta_logits, a_log, dt_bias, cu_seqlens, state_pool,
                      state_indices, *, layout="K_FIRST", state_dtype="f32",
                      state_scales=None, block_v=64, beta_mode="logits",
                      readout_mode="working", num_slots=None, units=None):
    """KDA recurrence over varlen sequences, mutating one slot per sequence.

    q, k: [total, Hk, K]; v: [total, HV, V]; raw_gate: [total, HV, K];
    beta_logits: [total, HV]; a_log: [HV]; dt_bias: [HV, K]; cu_seqlens:
    [B+1]; state_indices: [B]. q and k are always L2-normalised and q scaled
    by 1/sqrt(K). A zero-length sequence writes nothing.
    Returns (out [total, HV, V], writes keyed by (slot, hv)).
    """
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    g = np.asarray(raw_gate, np.float64); bl = np.asarray(beta_logits, np.float64)
    total, Hk, K = q.shape
    HV, V = v.shape[1], v.shape[2]
    sc = 1.0 / math.sqrt(K)
    B = len(cu_seqlens) - 1
    out = np.full((total, HV, V), np.nan) if units is not None else np.zeros((total, HV, V))
    writes = {}
    todo = [(bb, hv) for bb in range(B) for hv in range(HV)] if units is None else list(units)
    for (bb, hv) in todo:
        bos, eos = int(cu_seqlens[bb]), int(cu_seqlens[bb + 1])
        slot = int(state_indices[bb])
        if slot < 0 or (num_slots is not None and slot >= num_slots):
            out[bos:eos, hv, :] = 0.0
            continue
        if eos <= bos:
            continue
        h = key_head_of(hv, Hk, HV)
        S0 = load_state(state_pool[slot, hv], layout, state_dtype,
                        None if state_scales is None else state_scales[slot, hv], block_v)
        toks = []
        for t in range(bos, eos):
            qh, kh = prepare_qk(q[t, h], k[t, h], sc, True)
            toks.append((qh, kh, v[t, hv], kda_alpha(a_log[hv], g[t, hv], dt_bias[hv]),
                         beta_of(bl[t, hv], beta_mode)))
        o, payload = run_unit(S0, toks, state_dtype, readout_mode, block_v)
        out[bos:eos, hv, :] = o
        writes[(slot, hv)] = store_state(payload, layout, state_dtype)
    return out, writes


# ----------------------------------------------------------------------------
# codec over whole arrays (the exported quantise/dequantise calls)
# ----------------------------------------------------------------------------

def state_quantize_fp8(src, block_v, layout):
    """src [N, *2-D state in layout*] binary32 -> (codes same shape, scales [N, V/block_v])."""
    src = np.asarray(src, np.float32)
    N = src.shape[0]
    codes = np.zeros(src.shape, np.uint8)
    scales = None
    for n in range(N):
        kv = _to_kv(src[n], layout)
        c, s = formats.quantize_state(kv, block_v)
        codes[n] = _from_kv(c, layout)
        if scales is None:
            scales = np.zeros((N, s.shape[0]), np.float32)
        scales[n] = s
    return codes, scales


def state_dequantize_fp8(codes, scales, block_v, layout):
    codes = np.asarray(codes, np.uint8)
    out = np.zeros(codes.shape, np.float32)
    for n in range(codes.shape[0]):
        kv = formats.dequantize_state(_to_kv(codes[n], layout), scales[n], block_v)
        out[n] = _from_kv(kv, layout)
    return out


def state_quantize_h32(src, layout):
    """src [N, *2-D state in layout*] binary32 -> (codes int8 same shape, scales [N, V/32, K])."""
    src = np.asarray(src, np.float32)
    codes = np.zeros(src.shape, np.int8)
    scales = []
    for n in range(src.shape[0]):
        c, s = formats.quantize_state_h32(_to_kv(src[n], layout))
        codes[n] = _from_kv(c, layout)
        scales.append(s)
    K = _to_kv(src[0], layout).shape[0] if src.shape[0] else 0
    return codes, (np.stack(scales) if scales else np.zeros((0, 0, K), np.float32))


def state_dequantize_h32(codes, scales, layout):
    codes = np.asarray(codes, np.int8)
    out = np.zeros(codes.shape, np.float32)
    for n in range(codes.shape[0]):
        out[n] = _from_kv(formats.dequantize_state_h32(_to_kv(codes[n], layout), scales[n]), layout)
    return out
