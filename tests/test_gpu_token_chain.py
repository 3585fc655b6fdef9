"""Per-token checks of multi-token runs on bf16, fp8 and int8_hadamard32 states.

A bf16 or coded state passes through its storage format after every token
(modelopt ... linear_attention.decode, recurrent_decode_reference: token
write events). Where the GPU's and the oracle's binary32 working states
straddle a rounding boundary of the format, the two store neighbouring
values, and the difference is carried into the later tokens; so a T-token
call is held to the oracle only within one code step (1e-2 on outputs).

These tests make that check conditional. They run the same tokens as T
one-token GPU calls, threaded through the device pool. Each call is
compared with the oracle started from the pool the GPU left before it:
outputs at 1e-4 for a working readout (it reads the binary32 state); for a
stored readout, the output at 1e-4 against q^ times the state the kernel
stored (one neighbouring code at a large element already moves o by
|q^_i| times a code step, a few per cent of the slice at worst, so the
oracle's own stored readout is no tighter reference); states within one
code step and >= 99.9 % identical. Then the T-token call's
final pool (codes and scales, snapshots included) must match the chain's
within one code step and >= 99.9 % identical. The drivers covered are the
slot pool (both readouts), the paged suffix with page snapshots, KDA
varlen and the paged prefill scan.
"""

import numpy as np
import pytest
import torch

import gated_delta_rule_80_b200 as G
import workloads as W
from gdn_cases import (check_outputs, check_state, check_stored_readout, dev, dev_in, host,
                       pool_host, slice_rel_err)
from oracle import gdn as O

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

STORED = ("bf16", "fp8_e4m3", "int8_hadamard32")
COND_TOL = 1e-4


def _snap(pool, scales):
    return pool_host(pool), (scales.cpu().numpy() if scales is not None else None)


def _final_matches(init, pool_T, sc_T, pool_C, sc_C, state_dtype, layout):
    """Every (slot, hv) that either run changed: the T-token call's state
    within one code step of the chain's (check_state), >= 99.9 % identical."""
    n_slots, HV = init.shape[:2]
    keys = [(s, hv) for s in range(n_slots) for hv in range(HV)
            if not (np.array_equal(init[s, hv], pool_T[s, hv]) and np.array_equal(init[s, hv], pool_C[s, hv]))]
    assert keys, "neither run wrote anything"
    ref = {key: (pool_C[key], None if sc_C is None else sc_C[key]) for key in keys}
    check_state(pool_T, sc_T, ref, state_dtype, layout)
    return keys


# ----------------------------------------------------------------------------
# slot pool
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("readout", ["working", "stored"])
@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
@pytest.mark.parametrize("state_dtype", STORED)
def test_slots_run_token_by_token(state_dtype, layout, readout):
    seed, B, T, H, HV, K, V, num_slots = 401, 5, 4, 2, 4, 128, 128, 9
    t = W.gdn_tokens(seed, B, T, H, HV, K, V, "bf16")
    idx = W.slot_indices(seed, B, num_slots)
    pool, scales = W.device_pool(seed, num_slots, HV, K, V, layout, state_dtype)
    init, init_sc = _snap(pool, scales)
    pool_c = pool.clone()
    sc_c = scales.clone() if scales is not None else None
    di = dev(idx.astype(np.int32))

    def call(sl, p, sc):
        return host(G.gdn_decode_slots(*(dev_in(t[n][:, sl], "bf16") for n in ("q", "k", "v", "a", "b")),
                                       dev(t["A_log"]), dev(t["dt_bias"]), p, di, state_scales=sc,
                                       state_layout=layout, readout=readout, output_dtype=torch.float32))

    call(slice(None), pool, scales)
    units = [(b, hv) for b in range(B) for hv in range(HV)]
    for s in range(T):
        before, sc_b = _snap(pool_c, sc_c)
        o1 = call(slice(s, s + 1), pool_c, sc_c)
        after, sc_a = _snap(pool_c, sc_c)
        ts = {n: (x[:, s:s + 1] if n not in ("A_log", "dt_bias") else x) for n, x in t.items()}
        ref, writes = O.gdn_decode_slots(ts["q"], ts["k"], ts["v"], ts["a"], ts["b"], t["A_log"], t["dt_bias"],
                                         before, idx, layout=layout, state_dtype=state_dtype, state_scales=sc_b,
                                         readout_mode=readout)
        if readout == "working":
            check_outputs(o1, ref, units, lambda x, b, hv: x[b, :, hv, :], COND_TOL, "f32")
        else:
            # the state each side stores may differ by one code step (checked
            # below); the output must be q^ times the state the kernel stored
            check_stored_readout(o1, ts, idx, after, sc_a, units, layout, None, True, num_slots,
                                 state_dtype=state_dtype)
        check_state(after, sc_a, writes, state_dtype, layout)
    final_T, final_T_sc = _snap(pool, scales)
    final_C, final_C_sc = _snap(pool_c, sc_c)
    keys = _final_matches(init, final_T, final_T_sc, final_C, final_C_sc, state_dtype, layout)
    assert set(keys) <= {(int(sl), hv) for sl in idx for hv in range(HV)}


# ----------------------------------------------------------------------------
# paged suffix (page snapshots)
# ----------------------------------------------------------------------------

def _truncated_table(pt, lens, ps):
    """The CSR table of the same sequences cut to ``lens`` tokens each."""
    ind, ptr, last = [], [0], []
    for bb, L in enumerate(lens):
        p0 = int(pt.page_indptr[bb])
        npg = -(-int(L) // ps)
        ind.extend(int(x) for x in pt.page_indices[p0:p0 + npg])
        ptr.append(len(ind))
        last.append(int(L) - ps * (npg - 1))
    return np.array(ind, np.int32), np.array(ptr, np.int32), np.array(last, np.int32)


@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
@pytest.mark.parametrize("state_dtype", STORED)
def test_paged_suffix_token_by_token(state_dtype, layout):
    seed, B, H, HV, K, V, ps, T = 411, 4, 1, 2, 128, 128, 4, 6
    pt = W.paged_table(seed, B, ps, 40, 0, 0, min_len=T + ps + 1)
    t = W.gdn_tokens(seed, B, T, H, HV, K, V, "bf16")
    pool, scales = W.device_pool(seed, pt.num_pages, HV, K, V, layout, state_dtype)
    init, _ = _snap(pool, scales)
    pool_c = pool.clone()
    sc_c = scales.clone() if scales is not None else None
    tok = lambda sl: [dev_in(t[n][:, sl], "bf16") for n in ("q", "k", "v", "a", "b")]
    q, k, v, a, b = tok(slice(None))
    ind, ptr, last = _truncated_table(pt, pt.seq_lens, ps)
    G.gdn_decode_paged(q, k, v, dev(t["A_log"]), a, dev(t["dt_bias"]), b, state_pool=pool,
                       page_indices=dev(ind), page_indptr=dev(ptr), last_page_len=dev(last), page_size=ps,
                       state_scales=scales, state_layout=layout, output_dtype=torch.float32)
    units = [(bb, hv) for bb in range(B) for hv in range(HV)]
    for s in range(T):
        lens = [int(L) - T + s + 1 for L in pt.seq_lens]
        ind, ptr, last = _truncated_table(pt, lens, ps)
        before, sc_b = _snap(pool_c, sc_c)
        q, k, v, a, b = tok(slice(s, s + 1))
        o1 = host(G.gdn_decode_paged(q, k, v, dev(t["A_log"]), a, dev(t["dt_bias"]), b, state_pool=pool_c,
                                     page_indices=dev(ind), page_indptr=dev(ptr), last_page_len=dev(last),
                                     page_size=ps, state_scales=sc_c, state_layout=layout,
                                     output_dtype=torch.float32))
        after, sc_a = _snap(pool_c, sc_c)
        ts = {n: x[:, s:s + 1] for n, x in t.items() if n not in ("A_log", "dt_bias")}
        ref, writes = O.gdn_decode_paged(ts["q"], ts["k"], ts["v"], ts["a"], ts["b"], t["A_log"], t["dt_bias"],
                                         before, ind, ptr, last, state_dtype=state_dtype, state_scales=sc_b,
                                         layout=layout)
        check_outputs(o1, ref, units, lambda x, bb, hv: x[bb, :, hv, :], COND_TOL, "f32")
        check_state(after, sc_a, writes, state_dtype, layout)
    final_T, final_T_sc = _snap(pool, scales)
    final_C, final_C_sc = _snap(pool_c, sc_c)
    keys = _final_matches(init, final_T, final_T_sc, final_C, final_C_sc, state_dtype, layout)
    # the suffix crosses a page boundary in every sequence: snapshots were compared too
    assert len({pg for pg, _ in keys}) > B


# ----------------------------------------------------------------------------
# KDA varlen
# ----------------------------------------------------------------------------

def _kda_rows(t, sel):
    return {n: (t[n][sel] if n not in ("a_log", "dt_bias") else t[n]) for n in t}


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
@pytest.mark.parametrize("state_dtype", STORED)
def test_kda_run_token_by_token(state_dtype, layout):
    seed, B, Hk, HV, K, V, num_slots = 421, 4, 2, 4, 128, 128, 6
    cu = W.varlen_offsets(seed, B, 6, min_len=2)
    lens = np.diff(cu)
    t = W.kda_tokens(seed, int(cu[-1]), Hk, HV, K, V, "bf16")
    idx = W.slot_indices(seed, B, num_slots)
    pool, scales = W.device_pool(seed, num_slots, HV, K, V, layout, state_dtype)
    init, _ = _snap(pool, scales)
    pool_c = pool.clone()
    sc_c = scales.clone() if scales is not None else None
    di = dev(idx.astype(np.int32))

    def call(tt, cu_, p, sc):
        return host(G.kda_decode_varlen(*(dev_in(tt[n], "bf16") for n in ("q", "k", "v", "raw_gate", "beta_logits")),
                                        dev(t["a_log"]), dev(t["dt_bias"]), dev(np.asarray(cu_, np.int32)), p, di,
                                        state_scales=sc, state_layout=layout, output_dtype=torch.float32))

    call(t, cu, pool, scales)
    for s in range(int(lens.max())):
        live = [bb for bb in range(B) if lens[bb] > s]
        sel = np.array([int(cu[bb]) + s for bb in live])
        cu_s = np.concatenate([[0], np.cumsum([1 if lens[bb] > s else 0 for bb in range(B)])]).astype(np.int32)
        ts = _kda_rows(t, sel)
        before, sc_b = _snap(pool_c, sc_c)
        o1 = call(ts, cu_s, pool_c, sc_c)
        after, sc_a = _snap(pool_c, sc_c)
        ref, writes = O.kda_decode_varlen(ts["q"], ts["k"], ts["v"], ts["raw_gate"], ts["beta_logits"], t["a_log"],
                                          t["dt_bias"], cu_s, before, idx, layout=layout, state_dtype=state_dtype,
                                          state_scales=sc_b)
        units = [(bb, hv) for bb in range(B) for hv in range(HV)]
        check_outputs(o1, ref, units, lambda x, bb, hv: x[int(cu_s[bb]):int(cu_s[bb + 1]), hv, :], COND_TOL, "f32")
        check_state(after, sc_a, writes, state_dtype, layout)
        # a sequence with no token left keeps its slot bit for bit
        for bb in range(B):
            if lens[bb] <= s:
                assert np.array_equal(after[int(idx[bb])], before[int(idx[bb])])
    final_T, final_T_sc = _snap(pool, scales)
    final_C, final_C_sc = _snap(pool_c, sc_c)
    _final_matches(init, final_T, final_T_sc, final_C, final_C_sc, state_dtype, layout)


# ----------------------------------------------------------------------------
# paged prefill scan (fresh and continued runs)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
@pytest.mark.parametrize("state_dtype", STORED)
def test_prefill_scan_token_by_token(state_dtype, layout):
    seed, B, H, HV, K, V, ps = 431, 4, 1, 2, 128, 128, 4
    pt = W.paged_table(seed, B, ps, 14, 0, 0, min_len=3)
    cu = W.prefill_runs(seed, pt.seq_lens.tolist(), 2)
    n = np.diff(cu)
    t = W.varlen_gdn_tokens(seed, int(cu[-1]), H, HV, K, V, "bf16")
    pool, scales = W.device_pool(seed, pt.num_pages, HV, K, V, layout, state_dtype)
    init, _ = _snap(pool, scales)
    pool_c = pool.clone()
    sc_c = scales.clone() if scales is not None else None

    def call(tt, cu_, lens, p, sc):
        ind, ptr, last = _truncated_table(pt, lens, ps)
        return host(G.gdn_prefill_paged(*(dev_in(tt[nm], "bf16") for nm in ("q", "k", "v", "a", "b")),
                                        dev(t["A_log"]), dev(t["dt_bias"]), dev(np.asarray(cu_, np.int32)),
                                        state_pool=p, page_indices=dev(ind), page_indptr=dev(ptr),
                                        last_page_len=dev(last), page_size=ps, state_scales=sc,
                                        state_layout=layout, output_dtype=torch.float32)), (ind, ptr, last)

    call(t, cu, pt.seq_lens, pool, scales)
    assert n.max() >= 3 and (n == pt.seq_lens).any()      # at least one fresh sequence
    for s in range(int(n.max())):
        live = [bb for bb in range(B) if n[bb] > s]
        sel = np.array([int(cu[bb]) + s for bb in live])
        cu_s = np.concatenate([[0], np.cumsum([1 if n[bb] > s else 0 for bb in range(B)])]).astype(np.int32)
        lens = [int(pt.seq_lens[bb]) - int(n[bb]) + s + 1 if n[bb] > s else int(pt.seq_lens[bb])
                for bb in range(B)]
        ts = {nm: (x[sel] if nm not in ("A_log", "dt_bias") else x) for nm, x in t.items()}
        before, sc_b = _snap(pool_c, sc_c)
        o1, (ind, ptr, last) = call(ts, cu_s, lens, pool_c, sc_c)
        after, sc_a = _snap(pool_c, sc_c)
        ref, writes = O.gdn_prefill_paged(ts["q"], ts["k"], ts["v"], ts["a"], ts["b"], t["A_log"], t["dt_bias"],
                                          cu_s, before, ind, ptr, last, ps, state_dtype=state_dtype,
                                          state_scales=sc_b, layout=layout)
        units = [(bb, hv) for bb in range(B) for hv in range(HV)]
        check_outputs(o1, ref, units, lambda x, bb, hv: x[int(cu_s[bb]):int(cu_s[bb + 1]), hv, :], COND_TOL, "f32")
        check_state(after, sc_a, writes, state_dtype, layout)
    final_T, final_T_sc = _snap(pool, scales)
    final_C, final_C_sc = _snap(pool_c, sc_c)
    _final_matches(init, final_T, final_T_sc, final_C, final_C_sc, state_dtype, layout)
