"""Paged prefill of fp32 states on the tensor cores (64-token chunks, K = V =
128, bf16 token inputs, page_size a multiple of 64) against the oracle's scan
of single steps: fresh and continued runs, runs that start and end inside a
page, page sizes of 64 and 128, GQA, int64 page tables, bf16 outputs."""

import numpy as np
import pytest
import torch

from gdn_cases import gdn_prefill_case

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


def test_prefill_tc_fresh_and_continued_page64():
    r = gdn_prefill_case(111, B=6, H=1, HV=2, K=128, V=128, page_size=64, max_len=300)
    assert r["err"] == 0
    lens = np.diff(r["cu"])
    assert lens.max() > 128 and (lens % 64 != 0).any()   # several chunks and ragged tails


def test_prefill_tc_short_runs_inside_one_chunk():
    r = gdn_prefill_case(112, B=5, H=1, HV=2, K=128, V=128, page_size=64, max_len=60, fresh_every=3)
    assert r["err"] == 0


def test_prefill_tc_page128_gqa_int64_bf16_out():
    r = gdn_prefill_case(113, B=4, H=2, HV=4, K=128, V=128, page_size=128, max_len=520, fresh_every=1,
                         index_dtype="i64", out_dtype="bf16")
    assert r["err"] == 0 and len(r["write_pages"]) >= 4


def test_prefill_tc_no_l2norm_custom_scale():
    r = gdn_prefill_case(114, B=3, H=1, HV=2, K=128, V=128, page_size=64, max_len=200, use_qk_l2norm=False,
                         scale=0.05)
    assert r["err"] == 0


def test_prefill_tc_bench_config_sampled():
    """8 fresh sequences of 1024 tokens, H=16, HV=32 (the prefill bench
    workload's shape), oracle on sampled (sequence, head) pairs."""
    B, L = 8, 1024
    cu = np.arange(B + 1, dtype=np.int32) * L
    units = [(0, 0), (3, 17), (7, 31), (5, 8)]
    r = gdn_prefill_case(115, B=B, H=16, HV=32, K=128, V=128, page_size=64, max_len=L, min_len=L, cu=cu,
                         units=units, out_dtype="bf16")
    assert r["err"] == 0


def _prefill_tc_call(t, cu, ind, ptr, last, pool, page_size, err):
    import gated_delta_rule_80_b200 as G
    from gdn_cases import dev, dev_in
    return G.gdn_prefill_paged(
        dev_in(t["q"], "bf16"), dev_in(t["k"], "bf16"), dev_in(t["v"], "bf16"), dev_in(t["a"], "bf16"),
        dev_in(t["b"], "bf16"), dev(t["A_log"]), dev(t["dt_bias"]), dev(cu), state_pool=pool,
        page_indices=dev(ind), page_indptr=dev(ptr), last_page_len=dev(last), page_size=page_size,
        output_dtype=torch.float32, err_flags=err)


def test_prefill_tc_malformed_tables_flag_and_skip():
    """A sequence with a malformed page table or an out-of-range page gets zero
    outputs and a flag and leaves the pool untouched; a zero-length run touches
    nothing; the well-formed sequence is right."""
    import gated_delta_rule_80_b200 as G
    import workloads as W
    from gdn_cases import host, pool_host, slice_rel_err
    from oracle import gdn as O
    H, HV, K, V, ps = 1, 2, 128, 128, 64
    n0, n1, n2 = 70, 10, 5
    cu = np.array([0, n0, n0 + n1, n0 + n1 + n2, n0 + n1 + n2], np.int32)
    ind = np.array([0, 1, 2, 999, 5], np.int32)
    ptr = np.array([0, 2, 3, 4, 5], np.int32)
    last = np.array([n0 - ps, 0, n2, 64], np.int32)  # seq1: last_page_len 0; seq2: page 999; seq3: nothing new
    num_pages = 8
    t = W.varlen_gdn_tokens(121, int(cu[-1]), H, HV, K, V, "bf16")
    pool, _ = W.device_pool(121, num_pages, HV, K, V, "V_FIRST", "f32")
    before = pool_host(pool)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _prefill_tc_call(t, cu, ind, ptr, last, pool, ps, err)
    torch.cuda.synchronize()
    o, after = host(out), pool_host(pool)
    assert int(err.item()) == G.GDN_FLAG_PAGE_TABLE | G.GDN_FLAG_PAGE_RANGE
    assert not o[n0:].any()
    assert np.array_equal(after[2:], before[2:])
    sl = slice(0, n0)
    ref, writes = O.gdn_prefill_paged(t["q"][sl], t["k"][sl], t["v"][sl], t["a"][sl], t["b"][sl], t["A_log"],
                                      t["dt_bias"], cu[:2], {}, ind[:2], ptr[:2], last[:1], ps)
    for hv in range(HV):
        assert slice_rel_err(o[:n0, hv], ref[:, hv]) <= 1e-4
        for pg in (0, 1):
            assert slice_rel_err(after[pg, hv], writes[(pg, hv)][0]) <= 1e-4


def test_prefill_tc_bad_seqlens_flag():
    """cu_seqlens past total_tokens or out of order: the flag is raised, those
    sequences touch nothing, and the sequence before them is right."""
    import gated_delta_rule_80_b200 as G
    import workloads as W
    from gdn_cases import host, pool_host, slice_rel_err
    from oracle import gdn as O
    H, HV, K, V, ps = 1, 2, 128, 128, 64
    cu = np.array([0, 40, 200, 110], np.int32)     # seq1 ends past the 110 tokens, seq2 runs backwards
    ind = np.array([0, 1, 2, 3], np.int32)
    ptr = np.array([0, 1, 2, 4], np.int32)
    last = np.array([40, 64, 6], np.int32)
    t = W.varlen_gdn_tokens(122, 110, H, HV, K, V, "bf16")
    pool, _ = W.device_pool(122, 4, HV, K, V, "V_FIRST", "f32")
    before = pool_host(pool)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _prefill_tc_call(t, cu, ind, ptr, last, pool, ps, err)
    torch.cuda.synchronize()
    o, after = host(out), pool_host(pool)
    assert int(err.item()) == G.GDN_FLAG_SEQLENS
    assert np.array_equal(after[1:], before[1:])
    ref, writes = O.gdn_prefill_paged(t["q"][:40], t["k"][:40], t["v"][:40], t["a"][:40], t["b"][:40], t["A_log"],
                                      t["dt_bias"], cu[:2], {}, ind[:1], ptr[:2], last[:1], ps)
    for hv in range(HV):
        assert slice_rel_err(o[:40, hv], ref[:, hv]) <= 1e-4
        assert slice_rel_err(after[0, hv], writes[(0, hv)][0]) <= 1e-4
