"""Parity of the CUDA decode kernels (through the C ABI) with the oracle."""

import math

import numpy as np
import pytest
import torch

import gated_delta_rule_80_b200 as G
import workloads as W
from gdn_cases import (check_outputs, dev, dev_in, gdn_paged_case, gdn_prefill_case, gdn_slots_case, host,
                       kda_case, pool_host, slice_rel_err)
from oracle import formats
from oracle import gdn as O

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


# ----------------------------------------------------------------------------
# tiny recurrence: B=1, H=HV=4, K=V=32, fp32, 16 tokens
# ----------------------------------------------------------------------------

def test_tiny_sixteen_single_steps_and_one_suffix():
    w = W.WORKLOADS["tiny"]
    t = W.gdn_tokens(w.seed, w.B, w.T, w.H, w.HV, w.K, w.V, "f32")
    idx = np.array([1], np.int64)   # slots 0 and 2 are canaries
    pool, _ = W.device_pool(w.seed, w.num_slots, w.HV, w.K, w.V, w.layout, "f32", exact_slots=[0, 1, 2])
    init = pool_host(pool)
    one = {n: t[n] for n in t}
    outs = []
    for s in range(w.T):
        step = {n: (x[:, s:s + 1] if x.ndim >= 3 else x) for n, x in one.items()}
        o = G.gdn_decode_slots(dev(step["q"]), dev(step["k"]), dev(step["v"]), dev(step["a"]),
                               dev(step["b"]), dev(t["A_log"]), dev(t["dt_bias"]), pool,
                               dev(idx.astype(np.int32)), output_dtype=torch.float32)
        outs.append(host(o)[:, 0])
    torch.cuda.synchronize()
    stepped = pool_host(pool)
    # oracle: the 16 single steps threading the state through an fp32 pool
    p = init.copy()
    ref = []
    for s in range(w.T):
        o1, w1 = O.gdn_decode_slots(t["q"][:, s:s + 1], t["k"][:, s:s + 1], t["v"][:, s:s + 1],
                                    t["a"][:, s:s + 1], t["b"][:, s:s + 1], t["A_log"], t["dt_bias"], p, idx)
        ref.append(o1[:, 0])
        for (slot, hv), (st, _) in w1.items():
            p[slot, hv] = st
    for s in range(w.T):
        for hv in range(w.HV):
            assert slice_rel_err(outs[s][0, hv], ref[s][0, hv]) <= 1e-4
    for hv in range(w.HV):
        assert slice_rel_err(stepped[1, hv], p[1, hv]) <= 1e-4
    assert np.array_equal(stepped[[0, 2]], init[[0, 2]])
    # one T=16 call from the same initial state equals the 16 steps
    pool.copy_(torch.from_numpy(init).cuda())
    out16 = host(G.gdn_decode_slots(dev(t["q"]), dev(t["k"]), dev(t["v"]), dev(t["a"]), dev(t["b"]),
                                    dev(t["A_log"]), dev(t["dt_bias"]), pool, dev(idx.astype(np.int32)),
                                    output_dtype=torch.float32))
    for s in range(w.T):
        for hv in range(w.HV):
            assert slice_rel_err(out16[0, s, hv], outs[s][0, hv]) <= 1e-4
    suffix = pool_host(pool)
    for hv in range(w.HV):
        assert slice_rel_err(suffix[1, hv], stepped[1, hv]) <= 1e-4
    assert np.array_equal(suffix[[0, 2]], init[[0, 2]])


def test_tiny_suffix_against_oracle():
    w = W.WORKLOADS["tiny"]
    gdn_slots_case(w.seed, w.B, w.T, w.H, w.HV, w.K, w.V, w.num_slots, in_dtype="f32", out_dtype="f32",
                   indices=[1])


# ----------------------------------------------------------------------------
# slot pool: layouts, state dtypes, suffix lengths, head dims
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
@pytest.mark.parametrize("state_dtype", ["f32", "bf16", "fp8_e4m3"])
@pytest.mark.parametrize("T", [1, 3])
def test_slots_small(layout, state_dtype, T):
    r = gdn_slots_case(11 + T, B=5, T=T, H=2, HV=4, K=128, V=128, num_slots=12, layout=layout,
                       state_dtype=state_dtype)
    assert r["err"] == 0


@pytest.mark.parametrize("K,V", [(32, 32), (64, 64), (32, 128), (128, 64), (64, 32)])
@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_slots_head_dims(K, V, layout):
    gdn_slots_case(21, B=3, T=2, H=1, HV=3, K=K, V=V, num_slots=5, layout=layout, state_dtype="f32",
                   in_dtype="f32")


@pytest.mark.parametrize("K,V", [(32, 64), (64, 128), (128, 128)])
def test_slots_fp8_head_dims(K, V):
    gdn_slots_case(22, B=3, T=2, H=1, HV=2, K=K, V=V, num_slots=4, state_dtype="fp8_e4m3")


def test_slots_gqa_int64_no_l2norm_custom_scale():
    gdn_slots_case(23, B=4, T=2, H=2, HV=8, K=64, V=128, num_slots=6, index_dtype="i64",
                   use_qk_l2norm=False, scale=0.3, in_dtype="f32")


@pytest.mark.parametrize("state_dtype", ["bf16", "fp8_e4m3"])
@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_slots_stored_readout(state_dtype, layout):
    gdn_slots_case(24, B=3, T=3, H=1, HV=2, K=128, V=128, num_slots=4, layout=layout,
                   state_dtype=state_dtype, readout="stored")


def test_slots_bf16_outputs():
    gdn_slots_case(25, B=4, T=1, H=2, HV=4, K=128, V=128, num_slots=6, out_dtype="bf16")


def test_slots_padded_and_out_of_range():
    """-1 is a padded entry (zero output, nothing touched, no flag); 99 is past
    the pool (zero output, nothing touched, slot-range flag)."""
    r = gdn_slots_case(26, B=4, T=2, H=1, HV=2, K=128, V=128, num_slots=6, indices=[3, -1, 99, 0])
    assert r["err"] == G.GDN_FLAG_SLOT_RANGE
    assert np.all(r["out"][1] == 0) and np.all(r["out"][2] == 0)
    assert set(s for (s, _) in r["writes"]) == {3, 0}


@pytest.mark.parametrize("state_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_alpha1_beta0_keeps_state_bit_exact(state_dtype, layout):
    B, T, H, HV, K, V = 3, 2, 1, 2, 128, 128
    t = W.gdn_tokens(27, B, T, H, HV, K, V, "f32")
    t["A_log"] = np.full(HV, -np.inf, np.float32)
    t["b"] = np.full((B, T, HV), -np.inf, np.float32)
    r = gdn_slots_case(27, B, T, H, HV, K, V, num_slots=5, layout=layout, state_dtype=state_dtype,
                       in_dtype="f32", tokens=t)
    assert np.array_equal(r["pool_after"], r["pool_before"])


def test_alpha0_beta1_writes_outer_product():
    B, T, H, HV, K, V = 2, 1, 1, 2, 128, 128
    t = W.gdn_tokens(28, B, T, H, HV, K, V, "f32")
    t["A_log"] = np.full(HV, 60.0, np.float32)
    t["b"] = np.full((B, T, HV), np.inf, np.float32)
    r = gdn_slots_case(28, B, T, H, HV, K, V, num_slots=3, in_dtype="f32", tokens=t, layout="K_FIRST")
    for b in range(B):
        s = int(r["idx"][b])
        kh = O.l2_normalize(t["k"][b, 0, 0])
        for hv in range(HV):
            assert slice_rel_err(r["pool_after"][s, hv], np.outer(kh, t["v"][b, 0, hv])) <= 1e-5


def test_unit_key_overwrite_on_gpu():
    """beta = 1: after the write the key reads back exactly v (to fp32 rounding)."""
    B, T, H, HV, K, V = 2, 1, 1, 2, 128, 128
    t = W.gdn_tokens(29, B, T, H, HV, K, V, "f32")
    t["b"] = np.full((B, T, HV), np.inf, np.float32)
    r = gdn_slots_case(29, B, T, H, HV, K, V, num_slots=3, in_dtype="f32", tokens=t)
    for b in range(B):
        s = int(r["idx"][b])
        kh = O.l2_normalize(t["k"][b, 0, 0])
        for hv in range(HV):
            S = r["pool_after"][s, hv].T.astype(np.float64)   # V_FIRST -> [K, V]
            assert slice_rel_err(kh @ S, t["v"][b, 0, hv]) <= 1e-5


def test_empty_batch_launches_nothing():
    pool = torch.zeros((2, 2, 128, 128), device="cuda")
    z = lambda *s: torch.zeros(s, device="cuda")
    out = G.gdn_decode_slots(z(0, 1, 1, 128), z(0, 1, 1, 128), z(0, 1, 2, 128), z(0, 1, 2), z(0, 1, 2),
                             z(2), z(2), pool, torch.zeros(0, dtype=torch.int32, device="cuda"))
    assert out.shape == (0, 1, 2, 128) and not pool.any()


# ----------------------------------------------------------------------------
# slot pool at the full size the bench times (64 of 256 slots, bf16 in/out)
# ----------------------------------------------------------------------------

def test_slots_full_size_bench_config():
    w = W.WORKLOADS["slots"]
    r = gdn_slots_case(w.seed, w.B, w.T, w.H, w.HV, w.K, w.V, w.num_slots, layout=w.layout,
                       state_dtype="f32", in_dtype="bf16", out_dtype="bf16")
    assert r["err"] == 0


# ----------------------------------------------------------------------------
# paged pool
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("index_dtype", ["i32", "i64"])
@pytest.mark.parametrize("use_slots", [False, True])
def test_paged_small(index_dtype, use_slots):
    r = gdn_paged_case(31, B=12, H=2, HV=4, K=128, V=128, page_size=16, max_len=200, n_share=4,
                       share_pages=3, force_lens={0: 49, 1: 49, 5: 17}, index_dtype=index_dtype,
                       use_slots=use_slots, spare_pages=3)
    assert r["err"] == 0
    # the two sharers that open a new page read the last shared page and leave it untouched
    pt = r["table"]
    assert r["rows"][0][0] == pt.shared_pages[-1] and r["rows"][1][0] == pt.shared_pages[-1]
    assert pt.shared_pages[-1] not in r["write_pages"]
    if use_slots:
        assert np.array_equal(r["slots"], r["rows"])


@pytest.mark.parametrize("state_dtype", ["bf16", "fp8_e4m3"])
def test_paged_state_dtypes(state_dtype):
    gdn_paged_case(32, B=6, H=1, HV=2, K=128, V=128, page_size=8, max_len=60, n_share=2, share_pages=2,
                   force_lens={0: 17}, state_dtype=state_dtype)


@pytest.mark.parametrize("T,page_size", [(2, 16), (5, 4), (19, 4), (9, 8)])
@pytest.mark.parametrize("state_dtype", ["f32", "bf16"])
def test_paged_suffix(T, page_size, state_dtype):
    """The last T tokens on a paged pool: read from the page of the token
    before the suffix, a snapshot in every page that fills inside it, the
    final state in the last page, every other page untouched."""
    # suffixes start past the 2 shared pages, so no two sequences write one page
    r = gdn_paged_case(34 + T, B=7, H=1, HV=2, K=128, V=128, page_size=page_size, max_len=60,
                       n_share=2, share_pages=2, state_dtype=state_dtype, T=T,
                       min_len=T + 2 * page_size + 1)
    assert r["err"] == 0
    n_snap = len(r["write_pages"]) - 7
    if T - 1 >= page_size:   # a page boundary falls inside every suffix
        assert n_snap >= 7


@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_paged_suffix_layouts_and_fp8(layout):
    gdn_paged_case(36, B=4, H=2, HV=4, K=128, V=128, page_size=8, max_len=40, n_share=0, share_pages=0,
                   state_dtype="fp8_e4m3", T=6, layout=layout)
    gdn_paged_case(37, B=4, H=2, HV=4, K=64, V=64, page_size=8, max_len=40, n_share=0, share_pages=0,
                   T=3, layout=layout)


def test_paged_full_size():
    w = W.WORKLOADS["paged"]
    r = gdn_paged_case(w.seed, w.B, w.H, w.HV, w.K, w.V, w.page_size, w.max_len, w.n_share, w.share_pages,
                       force_lens={0: 1025, 1: 1025}, in_dtype="bf16", out_dtype="bf16")
    assert r["err"] == 0


def test_paged_malformed_rows_flag_and_skip():
    """Sequences whose page-table entries are malformed get zero output and a
    flag; the pool is untouched for them and correct for the rest."""
    B, H, HV, K, V = 4, 1, 2, 128, 128
    num_pages = 8
    ind = np.array([0, 1, 2, 3, 4, 5, 6], np.int32)
    ptr = np.array([0, 2, 3, 5, 7], np.int32)   # seq1 owns one page
    last = np.array([5, 1, 9, 0], np.int32)     # seq1 opens a page with no page before; seq2 > page_size; seq3 == 0
    t = W.gdn_tokens(33, B, 1, H, HV, K, V, "f32")
    pool, _ = W.device_pool(33, num_pages, HV, K, V, "V_FIRST", "f32", exact_slots=[1])
    before = pool_host(pool)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = G.gdn_decode_paged(dev(t["q"]), dev(t["k"]), dev(t["v"]), dev(t["A_log"]), dev(t["a"]),
                             dev(t["dt_bias"]), dev(t["b"]), state_pool=pool, page_indices=dev(ind),
                             page_indptr=dev(ptr), last_page_len=dev(last), page_size=8, err_flags=err,
                             output_dtype=torch.float32)
    torch.cuda.synchronize()
    o = host(out)
    after = pool_host(pool)
    assert int(err.item()) == G.GDN_FLAG_PAGE_TABLE
    assert np.all(o[1:] == 0)
    assert np.array_equal(after[2:], before[2:]) and np.array_equal(after[0], before[0])
    ref, writes = O.gdn_decode_paged(t["q"][:1], t["k"][:1], t["v"][:1], t["a"][:1], t["b"][:1], t["A_log"],
                                     t["dt_bias"], before, ind, ptr[:2], last[:1])
    for hv in range(HV):
        assert slice_rel_err(o[0, 0, hv], ref[0, 0, hv]) <= 1e-4
        assert slice_rel_err(after[1, hv], writes[(1, hv)][0]) <= 1e-4


def test_paged_slots_helper_flags_out_of_range_page():
    ind = np.array([0, 1, 50], np.int64)
    ptr = np.array([0, 1, 3], np.int64)
    last = np.array([3, 1], np.int64)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rows = G.gdn_paged_decode_slots(dev(ind), dev(ptr), dev(last), num_pages=8, page_size=4, err_flags=err)
    torch.cuda.synchronize()
    assert rows.cpu().numpy().tolist() == [[0, 0], [-1, -1]]
    assert int(err.item()) == G.GDN_FLAG_PAGE_RANGE


# ----------------------------------------------------------------------------
# KDA varlen
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_kda_config_full(layout):
    w = W.WORKLOADS["kda"]
    r = kda_case(w.seed, w.B, w.H, w.HV, w.K, w.V, w.num_slots, w.max_len, layout=layout)
    assert r["err"] == 0


def test_kda_layouts_agree():
    w = W.WORKLOADS["kda"]
    a = kda_case(w.seed, 8, w.H, w.HV, w.K, w.V, w.num_slots, w.max_len, layout="K_FIRST")
    b = kda_case(w.seed, 8, w.H, w.HV, w.K, w.V, w.num_slots, w.max_len, layout="V_FIRST")
    for hv in range(w.HV):
        assert slice_rel_err(a["out"][:, hv], b["out"][:, hv]) <= 1e-4
    for (slot, hv) in a["writes"]:
        assert slice_rel_err(a["pool_after"][slot, hv], b["pool_after"][slot, hv].T) <= 1e-4


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_kda_empty_sequences_probability_beta_gqa(layout):
    r = kda_case(41, B=5, Hk=2, HV=4, K=64, V=128, num_slots=7, max_len=6, layout=layout,
                 cu=[0, 3, 3, 7, 7, 9], beta_mode="probability", indices=[2, 4, -1, 6, 0])
    assert set(s for (s, _) in r["writes"]) == {2, 0}   # empty and padded sequences write nothing
    assert np.all(r["out"][3:7] == 0)


@pytest.mark.parametrize("state_dtype", ["bf16", "fp8_e4m3"])
def test_kda_state_dtypes(state_dtype):
    kda_case(42, B=4, Hk=2, HV=2, K=128, V=128, num_slots=6, max_len=4, state_dtype=state_dtype)


def test_kda_bad_seqlens_flag():
    r_cu = np.array([0, 3, 2, 4], np.int32)   # sequence 1 has eos < bos
    Hk = HV = 1
    K = V = 32
    t = W.kda_tokens(43, 4, Hk, HV, K, V, "f32")
    pool, _ = W.device_pool(43, 3, HV, K, V, "K_FIRST", "f32")
    before = pool_host(pool)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.kda_decode_varlen(dev(t["q"]), dev(t["k"]), dev(t["v"]), dev(t["raw_gate"]), dev(t["beta_logits"]),
                        dev(t["a_log"]), dev(t["dt_bias"]), dev(r_cu), pool,
                        dev(np.array([0, 1, 2], np.int32)), err_flags=err)
    torch.cuda.synchronize()
    assert int(err.item()) == G.GDN_FLAG_SEQLENS
    assert np.array_equal(pool_host(pool)[1], before[1])


def test_kda_single_sequence_equals_single_steps():
    K = V = 128
    HV = Hk = 2
    T = 6
    t = W.kda_tokens(44, T, Hk, HV, K, V, "bf16")
    pool, _ = W.device_pool(44, 2, HV, K, V, "K_FIRST", "f32", exact_slots=[1])
    init = pool.clone()
    idx = dev(np.array([1], np.int32))
    ins = {n: dev_in(t[n], "bf16") for n in ("q", "k", "v", "raw_gate", "beta_logits")}
    outT = host(G.kda_decode_varlen(ins["q"], ins["k"], ins["v"], ins["raw_gate"], ins["beta_logits"],
                                    dev(t["a_log"]), dev(t["dt_bias"]), dev(np.array([0, T], np.int32)),
                                    pool, idx, output_dtype=torch.float32))
    fused = pool_host(pool)
    pool.copy_(init)
    for s in range(T):
        o1 = host(G.kda_decode_varlen(*(ins[n][s:s + 1] for n in ("q", "k", "v", "raw_gate", "beta_logits")),
                                      dev(t["a_log"]), dev(t["dt_bias"]), dev(np.array([0, 1], np.int32)),
                                      pool, idx, output_dtype=torch.float32))
        for hv in range(HV):
            assert slice_rel_err(o1[0, hv], outT[s, hv]) <= 1e-4
    stepped = pool_host(pool)
    for hv in range(HV):
        assert slice_rel_err(stepped[1, hv], fused[1, hv]) <= 1e-4


# ----------------------------------------------------------------------------
# fp8 E4M3 state: codec bit-exactness and the large-batch decode
# ----------------------------------------------------------------------------

def _adversarial_states(N, K, V, layout, seed=51):
    r = np.random.default_rng(seed)
    shape = (N, K, V) if layout == "K_FIRST" else (N, V, K)
    x = (r.standard_normal(shape) * 0.1).astype(np.float32)
    flat = x.reshape(N, -1)
    flat[0] = 0.0                                                # amax == 0
    flat[1] = -np.abs(flat[1])                                   # all negative
    flat[2, :] = np.float32(1e-30) * r.standard_normal(flat.shape[1]).astype(np.float32)  # subnormal codes
    if N > 3:
        flat[3] = np.float32(2.0 ** -3) * np.rint(flat[3] * 64)     # many exact ties after scaling
    if N > 4:
        flat[4, :] = 1e-37                                       # r overflows -> stored as zero
    return x


@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
@pytest.mark.parametrize("K,V", [(128, 128), (32, 64), (64, 128), (256, 256), (256, 64)])
def test_fp8_codec_bit_exact(layout, K, V):
    N = 9
    x = _adversarial_states(N, K, V, layout)
    codes, scales = G.gdn_state_quantize_fp8(dev(x), layout=layout)
    ref_codes, ref_scales = O.state_quantize_fp8(x, 64, layout)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_scales.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    deq = G.gdn_state_dequantize_fp8(codes, scales, layout=layout).cpu().numpy()
    ref_deq = O.state_dequantize_fp8(ref_codes, ref_scales, 64, layout)
    assert np.array_equal(deq.view(np.uint32), ref_deq.view(np.uint32))


def test_fp8_large_batch_reduced():
    w = W.WORKLOADS["fp8"]
    gdn_slots_case(w.seed, B=24, T=1, H=w.H, HV=w.HV, K=w.K, V=w.V, num_slots=64, state_dtype="fp8_e4m3")


@pytest.mark.parametrize("K,V", [(32, 64), (64, 128), (128, 64), (256, 128)])
@pytest.mark.parametrize("in_dtype", ["bf16", "f32"])
def test_slots_fp8_single_token_shapes(K, V, in_dtype):
    """Single-token fp8 decode (the streaming kernel) for every head dim and
    both input dtypes (bf16 and f32 token rows take different copy shapes)."""
    gdn_slots_case(28, B=5, T=1, H=1, HV=2, K=K, V=V, num_slots=7, state_dtype="fp8_e4m3", in_dtype=in_dtype)


def test_slots_fp8_single_token_padded_int64_no_l2norm():
    r = gdn_slots_case(29, B=6, T=1, H=2, HV=4, K=128, V=128, num_slots=7, state_dtype="fp8_e4m3",
                       index_dtype="i64", indices=[3, -1, 99, 0, 5, -1], use_qk_l2norm=False, scale=0.3)
    assert r["err"] == G.GDN_FLAG_SLOT_RANGE
    assert np.all(r["out"][[1, 2, 5]] == 0)
    assert set(s for (s, _) in r["writes"]) == {3, 0, 5}


def test_fp8_many_tiles_per_cta_with_padding():
    """Enough tiles that each persistent CTA streams a few dozen of them across
    sequence boundaries, with padded and out-of-range sequences among them;
    checked on a sample of (sequence, head) pairs."""
    B, H, HV, K, V, num_slots = 256, 16, 32, 128, 128, 260
    idx = np.random.default_rng(30).permutation(num_slots)[:B].astype(np.int64)
    idx[::7] = -1
    idx[5] = num_slots + 3
    r = np.random.default_rng(31)
    units = sorted({(int(b), int(h)) for b, h in zip(r.integers(0, B, 300), r.integers(0, HV, 300))})
    units += [(b, h) for b in (0, 5, 7) for h in (0, HV - 1)]
    res = gdn_slots_case(30, B, 1, H, HV, K, V, num_slots, state_dtype="fp8_e4m3", indices=idx,
                         units=sorted(set(units)))
    assert res["err"] == G.GDN_FLAG_SLOT_RANGE
    assert np.all(res["out"][idx < 0] == 0) and np.all(res["out"][5] == 0)


def test_fp8_large_batch_full_size_sampled():
    w = W.WORKLOADS["fp8"]
    r = np.random.default_rng(52)
    units = sorted({(int(b), int(h)) for b, h in zip(r.integers(0, w.B, 400), r.integers(0, w.HV, 400))})
    gdn_slots_case(w.seed, w.B, w.T, w.H, w.HV, w.K, w.V, w.num_slots, state_dtype="fp8_e4m3",
                   in_dtype="bf16", out_dtype="bf16", units=units)


# ----------------------------------------------------------------------------
# head dims of 256
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
@pytest.mark.parametrize("state_dtype", ["f32", "bf16", "fp8_e4m3"])
@pytest.mark.parametrize("T", [1, 3])
def test_head_dim_256(layout, state_dtype, T):
    gdn_slots_case(61 + T, B=3, T=T, H=1, HV=2, K=256, V=256, num_slots=5, layout=layout,
                   state_dtype=state_dtype)


@pytest.mark.parametrize("K,V", [(256, 64), (64, 256), (256, 32), (32, 256)])
@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_head_dim_256_mixed(K, V, layout):
    gdn_slots_case(63, B=2, T=2, H=1, HV=2, K=K, V=V, num_slots=3, layout=layout, in_dtype="f32")


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_kda_head_dim_256(layout):
    kda_case(64, B=3, Hk=2, HV=2, K=256, V=256, num_slots=4, max_len=4, layout=layout)


def test_paged_head_dim_256():
    gdn_paged_case(65, B=5, H=1, HV=2, K=256, V=256, page_size=8, max_len=40, n_share=2, share_pages=1,
                   force_lens={0: 9})


# ----------------------------------------------------------------------------
# paged prefill (fresh and continued runs)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("state_dtype", ["f32", "bf16", "fp8_e4m3"])
@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_prefill_paged(state_dtype, layout):
    r = gdn_prefill_case(71, B=6, H=1, HV=2, K=128, V=128, page_size=8, max_len=45, state_dtype=state_dtype,
                         layout=layout)
    assert r["err"] == 0
    assert int(r["cu"][-1] - r["cu"][-2]) == 0   # the last sequence appends nothing


def test_prefill_paged_long_runs_int64():
    r = gdn_prefill_case(72, B=3, H=2, HV=4, K=64, V=128, page_size=16, max_len=300, index_dtype="i64",
                         fresh_every=1)
    assert r["err"] == 0 and len(r["write_pages"]) >= 3


@pytest.mark.parametrize("state_dtype", ["fp8_e4m3", "int8_hadamard32"])
def test_paged_coded_many_tiles_per_cta(state_dtype):
    """Paged single-token decode of the coded states at a size where each
    persistent CTA streams several tiles across sequences (with shared prefix
    pages and new-page sequences), checked on a sample of (sequence, head)."""
    B, HV = 64, 32
    r = np.random.default_rng(33)
    units = sorted({(int(b), int(h)) for b, h in zip(r.integers(0, B, 160), r.integers(0, HV, 160))})
    res = gdn_paged_case(33, B=B, H=16, HV=HV, K=128, V=128, page_size=64, max_len=256, n_share=8,
                         share_pages=2, force_lens={0: 129, 1: 129}, state_dtype=state_dtype, units=units)
    assert res["err"] == 0


@pytest.mark.parametrize("in_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("readout", ["working", "stored"])
def test_fp8_single_token_k128_readouts_zero_tile(in_dtype, readout):
    """K = 128 single-token fp8 decode (the streaming kernel): both readouts
    and input dtypes, GQA, V = 256 (two units of two tiles per head), a padded
    and an out-of-range slot, and a sequence whose state and v are zero, so
    that its tiles stay zero (scale 0, +0 codes)."""
    B, H, HV, K, V = 6, 2, 4, 128, 256
    t = W.gdn_tokens(31, B, 1, H, HV, K, V, in_dtype)
    t["v"][4] = 0.0
    r = gdn_slots_case(31, B=B, T=1, H=H, HV=HV, K=K, V=V, num_slots=8, state_dtype="fp8_e4m3",
                       in_dtype=in_dtype, indices=[5, -1, 0, 11, 7, 2], readout=readout, tokens=t,
                       zero_slots=[7])
    assert r["err"] == G.GDN_FLAG_SLOT_RANGE
    assert np.all(r["out"][[1, 3]] == 0)
    assert not r["pool_after"][7].any() and not r["scales_after"][7].any()


@pytest.mark.parametrize("readout", ["working", "stored"])
def test_fp8_k128_paged_single_token(readout):
    """K = 128 single-token fp8 decode on a paged pool (copy-on-new-page for
    the sequences whose last page is new), both readouts; the stored readout
    is also held at 1e-4 to q^ times the state written to the page."""
    gdn_paged_case(32, B=6, H=1, HV=2, K=128, V=128, page_size=8, max_len=60, n_share=2, share_pages=2,
                   force_lens={0: 17, 1: 9}, state_dtype="fp8_e4m3", readout=readout)
