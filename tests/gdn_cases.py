"""Shared drivers of the GPU parity tests: build one case from the seeded
generators, run it through the C ABI (via the Python binding) and through the
oracle on the same values, and compare.

Tolerances (max relative error per (sequence, value head) slice,
max|x - ref| / max|ref|): fp32 state 1e-4 on outputs and states; bf16 state
2e-2; fp8 state: outputs 1e-4 (working readout reads the fp32 state), stored
codes within one E4M3 step of the oracle's after dequantisation and >= 99.9%
identical; int8_hadamard32 state: outputs 1e-4, scales within 1e-5, codes
within one code step (compared as code * scale, the rotated values) and
>= 99.9% identical. bf16 outputs add the bf16 rounding of the output, 2^-8.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import gated_delta_rule_80_b200 as G
import workloads as W
from oracle import formats
from oracle import gdn as O

TOL = {"f32": 1e-4, "bf16": 2e-2, "fp8_e4m3": 1e-4, "int8_hadamard32": 1e-4}
CODED = ("fp8_e4m3", "int8_hadamard32")
BF16_OUT = 2.0 ** -8
# Outer bounds for outputs that a coded state's rounding feeds back into.
# Where the GPU's and the oracle's binary32 working states straddle a rounding
# boundary of the format, the two store neighbouring codes. A stored readout,
# and every later token of a multi-token run, then moves by |q^_i| times one
# code step (up to 2^-3 of the element for E4M3; amax / 127 of the group for
# int8_hadamard32). That is not bounded relative to the output slice, so
# 1e-2 is an end-to-end sanity bound only, met by the cases below. The parity
# claim for these outputs is the conditional one in test_gpu_token_chain:
# every token as its own call, checked at 1e-4 against the oracle started
# from the state the GPU stored (a stored readout against q^ times that
# stored state), codes within one step of the oracle's.
TOL_FP8_STORED = 1e-2
TOL_FP8_RUN = 1e-2


def out_tol(state_dtype, readout, multi_token):
    if state_dtype in CODED and (readout == "stored" or multi_token):
        return TOL_FP8_RUN
    return TOL[state_dtype]


def dev(x: np.ndarray, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def dev_in(x: np.ndarray, in_dtype: str):
    return dev(x.astype(np.float32), W.torch_dtype(in_dtype))


def slice_rel_err(x: np.ndarray, ref: np.ndarray) -> float:
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    den = max(float(np.max(np.abs(ref))), 1e-30)
    return float(np.max(np.abs(x - ref))) / den


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def pool_host(pool: torch.Tensor) -> np.ndarray:
    """Device pool -> numpy in the oracle's stored representation."""
    if pool.dtype == torch.bfloat16:
        return pool.view(torch.int16).cpu().numpy().view(np.uint16)
    return pool.cpu().numpy()


def check_outputs(out_gpu: np.ndarray, out_ref: np.ndarray, units, slicer, tol: float, out_dtype: str):
    """units: iterable of (b, hv); slicer(arr, b, hv) -> the slice."""
    worst = 0.0
    lim = tol + (BF16_OUT if out_dtype == "bf16" else 0.0)
    for (b, hv) in units:
        ref = slicer(out_ref, b, hv)
        if ref.size == 0:
            continue
        e = slice_rel_err(slicer(out_gpu, b, hv), ref)
        worst = max(worst, e)
        assert e <= lim, f"output slice (b={b}, hv={hv}): rel err {e:.3g} > {lim:.3g}"
    return worst


def check_state(pool_after: np.ndarray, scales_after, writes, state_dtype: str, layout: str, block_v=64):
    """Compare every written (slot, hv) state with the oracle's."""
    worst = 0.0
    n_codes = n_same = 0
    for (slot, hv), (st_ref, sc_ref) in writes.items():
        got = pool_after[slot, hv]
        if state_dtype == "f32":
            e = slice_rel_err(got, st_ref)
        elif state_dtype == "bf16":
            e = slice_rel_err(formats.bf16_bits_to_f32(got), formats.bf16_bits_to_f32(st_ref))
        elif state_dtype == "int8_hadamard32":
            sc_got = scales_after[slot, hv]
            assert np.allclose(sc_got, sc_ref, rtol=1e-5, atol=0), (slot, hv)
            kv_got = O._to_kv(got, layout)
            kv_ref = O._to_kv(st_ref, layout)
            s_got = np.repeat(sc_got.T.astype(np.float64), 32, axis=1)      # [K, V]
            s_ref = np.repeat(sc_ref.T.astype(np.float64), 32, axis=1)
            rot_got = kv_got.astype(np.float64) * s_got
            rot_ref = kv_ref.astype(np.float64) * s_ref
            lim = 1.002 * np.maximum(s_got, s_ref) + 1e-30                  # one code step
            assert np.all(np.abs(rot_got - rot_ref) <= lim), f"int8 state (slot={slot}, hv={hv}) off by > 1 step"
            n_codes += got.size
            n_same += int(np.sum(got == st_ref))
            e = slice_rel_err(formats.dequantize_state_h32(kv_got, sc_got),
                              formats.dequantize_state_h32(kv_ref, sc_ref))
            worst = max(worst, e)
            continue
        else:
            sc_got = scales_after[slot, hv]
            assert np.allclose(sc_got, sc_ref, rtol=1e-5, atol=0), (slot, hv, sc_got, sc_ref)
            kv_got = O._to_kv(got, layout)
            kv_ref = O._to_kv(st_ref, layout)
            deq_got = formats.dequantize_state(kv_got, sc_got, block_v).astype(np.float64)
            deq_ref = formats.dequantize_state(kv_ref, sc_ref, block_v).astype(np.float64)
            # one E4M3 step at the larger of the two magnitudes, in units of the tile scale
            a = np.maximum(np.abs(deq_got), np.abs(deq_ref)) / np.repeat(np.maximum(sc_ref, 1e-38), block_v)[None, :]
            step = np.exp2(np.maximum(np.floor(np.log2(np.maximum(a, 1e-30))), -6) - 3)
            lim = step * np.repeat(sc_ref, block_v)[None, :] * 1.0001 + 1e-30
            assert np.all(np.abs(deq_got - deq_ref) <= lim), f"fp8 state (slot={slot}, hv={hv}) off by > 1 step"
            n_codes += got.size
            n_same += int(np.sum(got == st_ref))
            e = slice_rel_err(deq_got, deq_ref)
            worst = max(worst, e)
            continue
        worst = max(worst, e)
        assert e <= TOL[state_dtype], f"state (slot={slot}, hv={hv}): rel err {e:.3g}"
    if n_codes:
        assert n_same / n_codes >= 0.999, f"only {n_same / n_codes:.5f} of {state_dtype} codes identical"
    return worst


def check_untouched(pool_before: np.ndarray, pool_after: np.ndarray, written_keys, scales_before=None,
                    scales_after=None):
    """Every (slot, hv) that is not written is bit-identical."""
    mask = np.ones(pool_before.shape[:2], dtype=bool)
    for (slot, hv) in written_keys:
        mask[slot, hv] = False
    a = pool_before[mask].view(np.uint8)
    b = pool_after[mask].view(np.uint8)
    assert np.array_equal(a, b), "a state that should be untouched changed"
    if scales_before is not None:
        assert np.array_equal(scales_before[mask].view(np.uint32), scales_after[mask].view(np.uint32))


def check_stored_readout(out_gpu, t, idx, pool_after, scales_after, units, layout, scale, use_qk_l2norm,
                         num_slots, block_v=64, state_dtype="fp8_e4m3"):
    """Validity of a stored readout: the last token's output is q^ times the
    state the kernel stored (decoded by the oracle's codec)."""
    K = t["q"].shape[-1]
    H, HV = t["q"].shape[2], t["v"].shape[2]
    sc = O._scale_of(scale, K)
    for (b, hv) in units:
        s = int(idx[b])
        if not 0 <= s < num_slots:
            continue
        qh, _ = O.prepare_qk(t["q"][b, -1, O.key_head_of(hv, H, HV)], t["k"][b, -1, 0], sc, use_qk_l2norm)
        S = O.load_state(pool_after[s, hv], layout, state_dtype,
                         None if scales_after is None else scales_after[s, hv], block_v)
        e = slice_rel_err(out_gpu[b, -1, hv], qh @ S)
        assert e <= 1e-4, f"stored readout (b={b}, hv={hv}) is not q^T of the stored state: {e:.3g}"


# ----------------------------------------------------------------------------
# GDN slot pool case
# ----------------------------------------------------------------------------

def gdn_slots_case(seed, B, T, H, HV, K, V, num_slots, layout="V_FIRST", state_dtype="f32",
                   in_dtype="bf16", out_dtype="f32", index_dtype="i32", readout="working",
                   indices=None, use_qk_l2norm=True, scale=None, tokens=None, block_v=64,
                   check=True, units=None, zero_slots=()):
    """Run one GDN slot decode on the GPU and the oracle; assert parity. Returns a dict.
    `zero_slots` start from an all-zero state (codes and scales)."""
    t = tokens or W.gdn_tokens(seed, B, T, H, HV, K, V, in_dtype)
    idx = np.asarray(indices if indices is not None else W.slot_indices(seed, B, num_slots), np.int64)
    live = [int(s) for s in idx if 0 <= s < num_slots]
    exact = set(live) if units is None else {int(idx[b]) for b, _ in units if 0 <= idx[b] < num_slots}
    pool, scales = W.device_pool(seed, num_slots, HV, K, V, layout, state_dtype, block_v,
                                 exact_slots=sorted(exact))
    for zs in zero_slots:
        pool[zs] = 0
        if scales is not None:
            scales[zs] = 0
    before = pool_host(pool)
    sc_before = scales.cpu().numpy() if scales is not None else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = G.gdn_decode_slots(
        dev_in(t["q"], in_dtype), dev_in(t["k"], in_dtype), dev_in(t["v"], in_dtype),
        dev_in(t["a"], in_dtype), dev_in(t["b"], in_dtype), dev(t["A_log"]), dev(t["dt_bias"]),
        pool, dev(idx.astype(np.int32 if index_dtype == "i32" else np.int64)), state_scales=scales,
        state_layout=layout, block_v=block_v, scale=scale, use_qk_l2norm=use_qk_l2norm,
        output_dtype=W.torch_dtype(out_dtype), readout=readout, err_flags=err)
    torch.cuda.synchronize()
    after = pool_host(pool)
    sc_after = scales.cpu().numpy() if scales is not None else None
    res = dict(out=host(out), pool_before=before, pool_after=after, scales_before=sc_before,
               scales_after=sc_after, err=int(err.item()), idx=idx, tokens=t)
    if not check:
        return res
    ref_out, writes = O.gdn_decode_slots(
        t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], before, idx,
        layout=layout, state_dtype=state_dtype, state_scales=sc_before, block_v=block_v,
        scale=scale, use_qk_l2norm=use_qk_l2norm, readout_mode=readout, num_slots=num_slots,
        units=units)
    todo = [(b, hv) for b in range(B) for hv in range(HV)] if units is None else units
    res["out_err"] = check_outputs(res["out"], ref_out, todo, lambda x, b, hv: x[b, :, hv, :],
                                   out_tol(state_dtype, readout, T > 1), out_dtype)
    if state_dtype in CODED and readout == "stored":
        check_stored_readout(res["out"], t, idx, after, sc_after, todo, layout, scale, use_qk_l2norm,
                             num_slots, block_v, state_dtype)
    res["state_err"] = check_state(after, sc_after, writes, state_dtype, layout, block_v)
    written = {(s, hv) for s in live for hv in range(HV)} if T > 0 else set()
    check_untouched(before, after, written, sc_before, sc_after)
    res["writes"] = writes
    res["ref_out"] = ref_out
    return res


# ----------------------------------------------------------------------------
# GDN paged case
# ----------------------------------------------------------------------------

def gdn_paged_case(seed, B, H, HV, K, V, page_size, max_len, n_share, share_pages, force_lens=None,
                   state_dtype="f32", in_dtype="bf16", out_dtype="f32", index_dtype="i32",
                   use_slots=False, units=None, spare_pages=0, readout="working", layout="V_FIRST", T=1,
                   min_len=2):
    pt = W.paged_table(seed, B, page_size, max_len, n_share, share_pages, force_lens,
                       spare_pages, min_len=max(min_len, T + 1)).cast(index_dtype)
    t = W.gdn_tokens(seed, B, T, H, HV, K, V, in_dtype)
    rows = O.paged_decode_slots(pt.page_indices, pt.page_indptr, pt.last_page_len) if T == 1 else None
    if T == 1:
        touched = sorted(set(rows.reshape(-1).tolist()))
    else:
        touched = sorted({pg for bb in range(B)
                          for pg in ([O.suffix_pages(pt.page_indices, pt.page_indptr, pt.last_page_len, page_size, T, bb)[0]])})
    pool, scales = W.device_pool(seed, pt.num_pages, HV, K, V, layout, state_dtype,
                                 exact_slots=touched)
    snap = pool.clone()
    sc_snap = scales.clone() if scales is not None else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pi, pp, pl = dev(pt.page_indices), dev(pt.page_indptr), dev(pt.last_page_len)
    slots = None
    if use_slots:
        slots = G.gdn_paged_decode_slots(pi, pp, pl, pt.num_pages, page_size, err_flags=err)
    out = G.gdn_decode_paged(
        dev_in(t["q"], in_dtype), dev_in(t["k"], in_dtype), dev_in(t["v"], in_dtype),
        dev(t["A_log"]), dev_in(t["a"], in_dtype), dev(t["dt_bias"]), dev_in(t["b"], in_dtype),
        state_pool=pool, page_indices=pi, page_indptr=pp, last_page_len=pl, slots=slots,
        state_scales=scales, state_layout=layout, page_size=page_size,
        output_dtype=W.torch_dtype(out_dtype), readout=readout, err_flags=err)
    torch.cuda.synchronize()
    res = dict(err=int(err.item()), table=pt, rows=rows)
    if slots is not None:
        res["slots"] = slots.cpu().numpy()
    # the oracle reads only the pages it needs, from the generator
    states, sc = W.host_pool(seed, touched, HV, K, V, layout, state_dtype)
    all_units = [(b, hv) for b in range(B) for hv in range(HV)]
    todo = all_units if units is None else units
    ref_out, writes = O.gdn_decode_paged(
        t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], states, pt.page_indices,
        pt.page_indptr, pt.last_page_len, state_dtype=state_dtype, state_scales=sc,
        readout_mode=readout, units=todo, page_size=page_size, layout=layout)
    out_h = host(out)
    res["out_err"] = check_outputs(out_h, ref_out, todo, lambda x, b, hv: x[b, :, hv, :],
                                   out_tol(state_dtype, readout, T > 1), out_dtype)
    # written pages: compare the sampled units; every other page must be bit-identical
    write_pages = sorted({pg for (pg, _) in writes}) if units is None else sorted(set(rows[:, 1].tolist()))
    wp = torch.tensor(write_pages, device="cuda")
    after_w = pool_host(pool[wp])
    sc_after_w = scales[wp].cpu().numpy() if scales is not None else None
    pos = {pg: i for i, pg in enumerate(write_pages)}
    sub_writes = {(pos[pg], hv): w for (pg, hv), w in writes.items()}
    res["state_err"] = check_state(after_w, sc_after_w, sub_writes, state_dtype, layout)
    if state_dtype in CODED and readout == "stored" and T == 1:
        # the conditional check: o is q^ times the state the kernel stored in
        # the sequence's write page
        dst = np.array([pos.get(int(rows[bb, 1]), -1) for bb in range(B)])
        check_stored_readout(out_h, t, dst, after_w, sc_after_w, todo, layout, None, True, len(write_pages),
                             64, state_dtype)
    keep = torch.ones(pt.num_pages, dtype=torch.bool, device="cuda")
    keep[wp] = False
    assert torch.equal(pool[keep], snap[keep]), "a page that is not a write page changed"
    if scales is not None:
        assert torch.equal(scales[keep], sc_snap[keep])
    res["write_pages"] = write_pages
    res["writes"] = writes
    return res


# ----------------------------------------------------------------------------
# paged prefill case
# ----------------------------------------------------------------------------

def gdn_prefill_case(seed, B, H, HV, K, V, page_size, max_len, state_dtype="f32", in_dtype="bf16",
                     out_dtype="f32", index_dtype="i32", layout="V_FIRST", fresh_every=2, scale=None,
                     use_qk_l2norm=True, units=None, cu=None, min_len=2):
    """One paged prefill on the GPU against the oracle. ``units`` restricts the
    oracle (and the comparison) to some (sequence, value head) pairs; the
    pages that must stay untouched are still checked for every sequence."""
    pt = W.paged_table(seed, B, page_size, max_len, 0, 0, min_len=min_len).cast(index_dtype)
    cu = np.asarray(cu if cu is not None else W.prefill_runs(seed, pt.seq_lens.tolist(), fresh_every), np.int32)
    total = int(cu[-1])
    t = W.varlen_gdn_tokens(seed, total, H, HV, K, V, in_dtype)
    reads, written = set(), set()
    for bb in range(B):
        n = int(cu[bb + 1] - cu[bb])
        if n == 0:
            continue
        L = int(pt.seq_lens[bb])
        if n < L:
            rd, snaps, last = O.suffix_pages(pt.page_indices, pt.page_indptr, pt.last_page_len, page_size, n, bb)
            reads.add(rd)
            written.update(pg for _, pg in snaps)
        else:  # a fresh sequence fills every page it owns
            p0 = int(pt.page_indptr[bb])
            written.update(int(pt.page_indices[p0 + i]) for i in range((L - 1) // page_size))
            last = int(pt.page_indices[int(pt.page_indptr[bb + 1]) - 1])
        written.add(last)
    pool, scales = W.device_pool(seed, pt.num_pages, HV, K, V, layout, state_dtype, exact_slots=sorted(reads))
    snap = pool.clone()
    sc_snap = scales.clone() if scales is not None else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = G.gdn_prefill_paged(
        dev_in(t["q"], in_dtype), dev_in(t["k"], in_dtype), dev_in(t["v"], in_dtype), dev_in(t["a"], in_dtype),
        dev_in(t["b"], in_dtype), dev(t["A_log"]), dev(t["dt_bias"]), dev(cu), state_pool=pool,
        page_indices=dev(pt.page_indices), page_indptr=dev(pt.page_indptr), last_page_len=dev(pt.last_page_len),
        page_size=page_size, state_scales=scales, state_layout=layout, output_dtype=W.torch_dtype(out_dtype),
        scale=scale, use_qk_l2norm=use_qk_l2norm, err_flags=err)
    torch.cuda.synchronize()
    states, sc = W.host_pool(seed, sorted(reads), HV, K, V, layout, state_dtype)
    ref_out, writes = O.gdn_prefill_paged(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], cu,
                                          states, pt.page_indices, pt.page_indptr, pt.last_page_len, page_size,
                                          state_dtype=state_dtype, state_scales=sc, layout=layout, scale=scale,
                                          use_qk_l2norm=use_qk_l2norm, units=units)
    todo = [(bb, hv) for bb in range(B) for hv in range(HV)] if units is None else list(units)
    res = dict(err=int(err.item()), cu=cu, table=pt)
    res["out_err"] = check_outputs(host(out), ref_out, todo, lambda x, bb, hv: x[int(cu[bb]):int(cu[bb + 1]), hv, :],
                                   out_tol(state_dtype, "working", True), out_dtype)
    write_pages = sorted(written)
    assert {pg for (pg, _) in writes} <= set(write_pages)
    wp = torch.tensor(write_pages, device="cuda", dtype=torch.long)
    pos = {pg: i for i, pg in enumerate(write_pages)}
    res["state_err"] = check_state(pool_host(pool[wp]), scales[wp].cpu().numpy() if scales is not None else None,
                                   {(pos[pg], hv): w for (pg, hv), w in writes.items()}, state_dtype, layout)
    keep = torch.ones(pt.num_pages, dtype=torch.bool, device="cuda")
    keep[wp] = False
    assert torch.equal(pool[keep], snap[keep]), "a page the runs do not fill changed"
    if scales is not None:
        assert torch.equal(scales[keep], sc_snap[keep])
    res["write_pages"] = write_pages
    return res


# ----------------------------------------------------------------------------
# KDA varlen case
# ----------------------------------------------------------------------------

def kda_case(seed, B, Hk, HV, K, V, num_slots, max_len, layout="K_FIRST", state_dtype="f32",
             in_dtype="bf16", out_dtype="f32", beta_mode="logits", cu=None, indices=None,
             readout="working", tokens=None):
    cu = np.asarray(cu if cu is not None else W.varlen_offsets(seed, B, max_len), np.int32)
    total = int(cu[-1])
    t = tokens or W.kda_tokens(seed, total, Hk, HV, K, V, in_dtype)
    if beta_mode == "probability":
        t = dict(t, beta_logits=W.as_dtype_values(1.0 / (1.0 + np.exp(-t["beta_logits"])), in_dtype))
    idx = np.asarray(indices if indices is not None else W.slot_indices(seed, B, num_slots), np.int64)
    live = sorted(set(int(s) for s in idx if 0 <= s < num_slots))
    pool, scales = W.device_pool(seed, num_slots, HV, K, V, layout, state_dtype, exact_slots=live)
    before = pool_host(pool)
    sc_before = scales.cpu().numpy() if scales is not None else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = G.kda_decode_varlen(
        dev_in(t["q"], in_dtype), dev_in(t["k"], in_dtype), dev_in(t["v"], in_dtype),
        dev_in(t["raw_gate"], in_dtype), dev_in(t["beta_logits"], in_dtype), dev(t["a_log"]),
        dev(t["dt_bias"]), dev(cu), pool, dev(idx.astype(np.int32)),
        output_dtype=W.torch_dtype(out_dtype), beta_mode=beta_mode, state_layout=layout,
        state_scales=scales, readout=readout, err_flags=err)
    torch.cuda.synchronize()
    after = pool_host(pool)
    sc_after = scales.cpu().numpy() if scales is not None else None
    ref_out, writes = O.kda_decode_varlen(
        t["q"], t["k"], t["v"], t["raw_gate"], t["beta_logits"], t["a_log"], t["dt_bias"], cu, before, idx,
        layout=layout, state_dtype=state_dtype, state_scales=sc_before, beta_mode=beta_mode,
        readout_mode=readout, num_slots=num_slots)
    out_h = host(out)
    units = [(b, hv) for b in range(B) for hv in range(HV)]
    res = dict(out=out_h, err=int(err.item()), writes=writes, pool_before=before, pool_after=after, cu=cu)
    res["out_err"] = check_outputs(out_h, ref_out, units,
                                   lambda x, b, hv: x[int(cu[b]):int(cu[b + 1]), hv, :],
                                   out_tol(state_dtype, readout, True), out_dtype)
    res["state_err"] = check_state(after, sc_after, writes, state_dtype, layout)
    check_untouched(before, after, writes.keys(), sc_before, sc_after)
    return res
