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
