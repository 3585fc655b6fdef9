"""KDA varlen with long runs: the chunked tensor-core kernel against the oracle.

kda_decode_varlen runs a call on the chunked kernel when the state is fp32,
K = V = 128, the inputs are bf16 and the runs average at least 32 tokens;
the chunked form is the scan of single steps written for blocks of tokens
(Circuit.LLM.Mixer, "Gated memory", kdaLiteStep; a prefill is the steps in
order), so its outputs and final states are held to the oracle's scan at the
fp32-state tolerance, 1e-4, for runs of 33 to 1024 tokens, partial chunks
included.
"""

import numpy as np
import pytest
import torch

import gated_delta_rule_80_b200 as G
import workloads as W
from gdn_cases import check_outputs, check_state, check_untouched, dev, dev_in, host, kda_case, pool_host
from oracle import gdn as O

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_kda_long_runs_against_oracle(layout):
    """Runs of 70, 129, 40 and 33 tokens (partial last chunks), one empty
    sequence, GQA (two value heads per key head), fp32 outputs."""
    cu = np.concatenate([[0], np.cumsum([70, 0, 129, 40, 33])]).astype(np.int32)
    r = kda_case(501, B=5, Hk=2, HV=4, K=128, V=128, num_slots=9, max_len=0, layout=layout, cu=cu)
    assert r["err"] == 0


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_kda_long_runs_bf16_out_probability_beta_padded_slot(layout):
    cu = np.concatenate([[0], np.cumsum([64, 96, 50])]).astype(np.int32)
    r = kda_case(502, B=3, Hk=4, HV=4, K=128, V=128, num_slots=5, max_len=0, layout=layout, cu=cu,
                 indices=[3, -1, 0], out_dtype="bf16", beta_mode="probability")
    assert r["err"] == 0


def test_kda_thousand_token_run_sampled():
    """One sequence of 1024 tokens and one of 512 on 32 value heads (the
    heads of the KDA configuration), checked on 6 heads."""
    B, Hk, HV, K, V = 2, 32, 32, 128, 128
    cu = np.array([0, 1024, 1536], np.int32)
    total = int(cu[-1])
    t = W.kda_tokens(503, total, Hk, HV, K, V, "bf16")
    idx = np.array([1, 0])
    pool, _ = W.device_pool(503, 2, HV, K, V, "K_FIRST", "f32", exact_slots=[0, 1])
    before = pool_host(pool)
    out = host(G.kda_decode_varlen(*(dev_in(t[n], "bf16") for n in ("q", "k", "v", "raw_gate", "beta_logits")),
                                   dev(t["a_log"]), dev(t["dt_bias"]), dev(cu), pool, dev(idx.astype(np.int32)),
                                   state_layout="K_FIRST", output_dtype=torch.float32))
    after = pool_host(pool)
    heads = [0, 5, 11, 17, 26, 31]
    sub = lambda x, hh: x[:, hh]
    ref_out, writes = O.kda_decode_varlen(sub(t["q"], heads), sub(t["k"], heads), sub(t["v"], heads),
                                          sub(t["raw_gate"], heads),
                                          sub(t["beta_logits"], heads), t["a_log"][heads], t["dt_bias"][heads], cu,
                                          before[:, heads], idx, layout="K_FIRST")
    # the oracle ran on the heads picked above with the key heads of a
    # one-to-one map (Hk == HV), so its head j is head heads[j] here
    units = [(b, j) for b in range(B) for j in range(len(heads))]
    check_outputs(out[:, heads], ref_out, units,
                  lambda x, b, j: x[int(cu[b]):int(cu[b + 1]), j, :], 1e-4, "f32")
    check_state(after[:, heads], None, writes, "f32", "K_FIRST")


def _kda_call(t, cu, pool, idx, layout):
    return host(G.kda_decode_varlen(*(dev_in(t[n], "bf16") for n in ("q", "k", "v", "raw_gate", "beta_logits")),
                                    dev(t["a_log"]), dev(t["dt_bias"]), dev(np.asarray(cu, np.int32)), pool,
                                    dev(np.asarray(idx, np.int32)), state_layout=layout,
                                    output_dtype=torch.float32))


def test_kda_chunked_equals_short_calls():
    """The chunked form equals the scan: a 96-token run in one call (chunked)
    and the same run in 24 calls of 4 tokens (runs too short for chunks, so
    the scan) agree within the fp32 tolerance."""
    K = V = 128
    HV = Hk = 2
    T = 96
    t = W.kda_tokens(504, T, Hk, HV, K, V, "bf16")
    pool, _ = W.device_pool(504, 2, HV, K, V, "V_FIRST", "f32", exact_slots=[1])
    init = pool.clone()
    out_long = _kda_call(t, [0, T], pool, [1], "V_FIRST")
    fused = pool_host(pool)
    pool.copy_(init)
    outs = []
    for s0 in range(0, T, 4):
        part = {n: (x[s0:s0 + 4] if n not in ("a_log", "dt_bias") else x) for n, x in t.items()}
        outs.append(_kda_call(part, [0, 4], pool, [1], "V_FIRST"))
    stepped = pool_host(pool)
    out_short = np.concatenate(outs)
    for hv in range(HV):
        e = np.max(np.abs(out_long[:, hv] - out_short[:, hv])) / np.max(np.abs(out_short[:, hv]))
        assert e <= 1e-4, e
        e = np.max(np.abs(fused[1, hv] - stepped[1, hv])) / np.max(np.abs(stepped[1, hv]))
        assert e <= 1e-4, e


def test_kda_long_runs_bad_seqlens_flag():
    """A malformed cu_seqlens on the chunked path: the sequence is skipped
    with GDN_FLAG_SEQLENS and the other sequences still match the oracle."""
    K = V = 128
    HV = Hk = 2
    cu = np.array([0, 80, 60, 150], np.int32)          # sequence 1 runs backwards
    total = 150
    t = W.kda_tokens(505, total, Hk, HV, K, V, "bf16")
    idx = np.array([0, 1, 2])
    pool, _ = W.device_pool(505, 3, HV, K, V, "K_FIRST", "f32", exact_slots=[0, 1, 2])
    before = pool_host(pool)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.kda_decode_varlen(*(dev_in(t[n], "bf16") for n in ("q", "k", "v", "raw_gate", "beta_logits")),
                        dev(t["a_log"]), dev(t["dt_bias"]), dev(cu), pool, dev(idx.astype(np.int32)),
                        state_layout="K_FIRST", output_dtype=torch.float32, err_flags=err)
    torch.cuda.synchronize()
    assert int(err.item()) == G.GDN_FLAG_SEQLENS
    after = pool_host(pool)
    assert np.array_equal(after[1], before[1])
    good = np.array([0, 80], np.int32)
    ref_out, writes = O.kda_decode_varlen(t["q"], t["k"], t["v"], t["raw_gate"], t["beta_logits"], t["a_log"],
                                          t["dt_bias"], good, before, idx[:1], layout="K_FIRST")
    check_state(after, None, writes, "f32", "K_FIRST")
    check_untouched(before[[1]], after[[1]], [])
