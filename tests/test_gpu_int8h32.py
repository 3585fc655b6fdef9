"""int8_hadamard32 state (one scale per key channel and 32 values, the
ModelOpt linear-attention decode codec): the codec calls bit for bit against
the oracle, and every decode path on an int8 pool against the oracle."""

import numpy as np
import pytest
import torch

import gated_delta_rule_80_b200 as G
import workloads as W
from gdn_cases import dev, gdn_paged_case, gdn_prefill_case, gdn_slots_case, kda_case
from oracle import gdn as O

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

I8 = "int8_hadamard32"


def _codec_states(N, K, V, layout, seed=91):
    """States with the codec's edge cases in the first few: a zero state, a
    state of one spike per group, an all-negative state, values near the
    bottom of binary32 (r overflows), groups whose rotated values take two
    magnitudes only, and a spread of magnitudes across key channels."""
    r = np.random.default_rng(seed)
    kv = (r.standard_normal((N, K, V)) * 0.1).astype(np.float32)
    kv[0] = 0.0
    kv[1] = 0.0
    kv[1, :, ::32] = r.standard_normal((K, V // 32)).astype(np.float32)
    kv[2] = -np.abs(kv[2])
    kv[3] = np.float32(1e-39)
    kv[4, :, :] = 0.0
    kv[4, :, 0::32] = 127.0 / np.sqrt(np.float32(32.0))
    kv[4, :, 1::32] = np.float32(0.5) / np.sqrt(np.float32(32.0))
    kv[5] *= np.exp(r.uniform(-20, 20, (K, 1))).astype(np.float32)
    x = kv if layout == "K_FIRST" else np.ascontiguousarray(kv.transpose(0, 2, 1))
    return x


@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
@pytest.mark.parametrize("K,V", [(128, 128), (32, 32), (64, 128), (256, 256), (256, 64), (32, 256)])
def test_int8h32_codec_bit_exact(layout, K, V):
    x = _codec_states(8, K, V, layout)
    codes, scales = G.gdn_state_quantize_int8h32(dev(x), layout=layout)
    ref_codes, ref_scales = O.state_quantize_h32(x, layout)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_scales.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert not codes[0].any() and not scales[0].any() and not scales[3].any()
    deq = G.gdn_state_dequantize_int8h32(codes, scales, layout=layout).cpu().numpy()
    ref_deq = O.state_dequantize_h32(ref_codes, ref_scales, layout)
    assert np.array_equal(deq.view(np.uint32), ref_deq.view(np.uint32))


@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
@pytest.mark.parametrize("T", [1, 3])
def test_int8h32_slots(layout, T):
    gdn_slots_case(92 + T, B=5, T=T, H=2, HV=4, K=128, V=128, num_slots=7, layout=layout, state_dtype=I8)


@pytest.mark.parametrize("K,V", [(32, 64), (64, 128), (128, 64), (256, 256), (256, 64), (32, 256)])
@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_int8h32_head_dims(K, V, layout):
    gdn_slots_case(94, B=3, T=2, H=1, HV=2, K=K, V=V, num_slots=4, layout=layout, state_dtype=I8, in_dtype="f32")


@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
@pytest.mark.parametrize("T", [1, 2])
def test_int8h32_stored_readout(layout, T):
    gdn_slots_case(95, B=4, T=T, H=1, HV=2, K=64, V=128, num_slots=6, layout=layout, state_dtype=I8,
                   readout="stored")


def test_int8h32_bf16_outputs_padded_int64():
    r = gdn_slots_case(96, B=4, T=1, H=1, HV=2, K=128, V=128, num_slots=5, state_dtype=I8, out_dtype="bf16",
                       index_dtype="i64", indices=[3, -1, 0, 7])
    assert r["err"] == 1            # slot 7 is out of range
    assert not r["out"][1].any() and not r["out"][3].any()


@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_int8h32_paged(layout):
    gdn_paged_case(97, B=6, H=1, HV=2, K=128, V=128, page_size=8, max_len=60, n_share=2, share_pages=2,
                   force_lens={0: 17, 1: 9}, state_dtype=I8, layout=layout)


@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_int8h32_paged_suffix(layout):
    gdn_paged_case(98, B=4, H=1, HV=2, K=64, V=128, page_size=4, max_len=40, n_share=0, share_pages=0,
                   state_dtype=I8, T=6, layout=layout, min_len=6 + 2 * 4 + 1)


@pytest.mark.parametrize("layout", ["V_FIRST", "K_FIRST"])
def test_int8h32_prefill(layout):
    r = gdn_prefill_case(99, B=5, H=1, HV=2, K=128, V=128, page_size=8, max_len=40, state_dtype=I8, layout=layout)
    assert r["err"] == 0


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_int8h32_kda(layout):
    kda_case(100, B=4, Hk=2, HV=2, K=128, V=128, num_slots=6, max_len=5, layout=layout, state_dtype=I8)


def test_int8h32_large_batch_reduced():
    w = W.WORKLOADS["int8"]
    gdn_slots_case(w.seed, B=24, T=1, H=w.H, HV=w.HV, K=w.K, V=w.V, num_slots=64, state_dtype=I8)


def test_int8h32_full_size_sampled():
    w = W.WORKLOADS["int8"]
    r = np.random.default_rng(101)
    units = sorted({(int(b), int(h)) for b, h in zip(r.integers(0, w.B, 300), r.integers(0, w.HV, 300))})
    gdn_slots_case(w.seed, w.B, w.T, w.H, w.HV, w.K, w.V, w.num_slots, state_dtype=I8,
                   in_dtype="bf16", out_dtype="bf16", units=units)


@pytest.mark.parametrize("K,V", [(32, 64), (64, 128), (128, 64), (256, 128), (256, 64)])
@pytest.mark.parametrize("in_dtype", ["bf16", "f32"])
def test_int8h32_single_token_shapes(K, V, in_dtype):
    """Single-token V_FIRST decode (the streaming kernel) for every head dim and
    both input dtypes (their token rows take different copy shapes)."""
    gdn_slots_case(101, B=5, T=1, H=1, HV=2, K=K, V=V, num_slots=7, state_dtype=I8, in_dtype=in_dtype)


def test_int8h32_single_token_padded_stored_readout_k256():
    r = gdn_slots_case(102, B=5, T=1, H=1, HV=2, K=256, V=128, num_slots=6, state_dtype=I8,
                       indices=[3, -1, 99, 0, 5], readout="stored", index_dtype="i64")
    assert r["err"] == G.GDN_FLAG_SLOT_RANGE
    assert np.all(r["out"][[1, 2]] == 0)


@pytest.mark.parametrize("in_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("readout", ["working", "stored"])
def test_int8h32_single_token_k128_group_kernel(in_dtype, readout):
    """K = 128 single-token V_FIRST decode (one warp per scale group): both
    readouts and input dtypes, a padded slot, an out-of-range slot, GQA,
    V = 256 (eight groups per head), and a sequence whose state and v are
    zero, so that its groups stay zero (scales 0, codes 0)."""
    t = W.gdn_tokens(103, 6, 1, 2, 4, 128, 256, in_dtype)
    t["v"][4] = 0.0
    r = gdn_slots_case(103, B=6, T=1, H=2, HV=4, K=128, V=256, num_slots=8, state_dtype=I8, in_dtype=in_dtype,
                       indices=[5, -1, 0, 11, 7, 2], readout=readout, index_dtype="i32", tokens=t,
                       zero_slots=[7])
    assert r["err"] == G.GDN_FLAG_SLOT_RANGE
    assert np.all(r["out"][[1, 3]] == 0)
    assert not r["pool_after"][7].any() and not r["scales_after"][7].any()


def test_int8h32_many_groups_per_warp_with_padding():
    """Enough groups that every warp of the K = 128 kernel streams dozens of
    them across sequence boundaries, with padded and out-of-range sequences
    among them and four value heads per key head; checked on a sample of
    (sequence, head) pairs and on the padded rows."""
    B, H, HV, K, V, num_slots = 256, 8, 32, 128, 128, 260
    idx = np.random.default_rng(104).permutation(num_slots)[:B].astype(np.int64)
    idx[::7] = -1
    idx[5] = num_slots + 3
    r = np.random.default_rng(105)
    units = sorted({(int(b), int(h)) for b, h in zip(r.integers(0, B, 300), r.integers(0, HV, 300))})
    units += [(b, h) for b in (0, 4, 6, 8) for h in (0, HV - 1)]
    res = gdn_slots_case(104, B, 1, H, HV, K, V, num_slots, state_dtype=I8, indices=idx, units=sorted(set(units)))
    assert res["err"] == G.GDN_FLAG_SLOT_RANGE
    assert np.all(res["out"][idx < 0] == 0) and np.all(res["out"][5] == 0)


def test_int8h32_k128_no_l2norm_custom_scale():
    """K = 128 single-token decode without the q/k L2 norm and with a custom
    q scale (the norms and the scale enter the group kernel only through the
    reduced dots)."""
    gdn_slots_case(106, B=5, T=1, H=2, HV=4, K=128, V=128, num_slots=7, state_dtype=I8, in_dtype="f32",
                   use_qk_l2norm=False, scale=0.3)


@pytest.mark.parametrize("readout", ["working", "stored"])
def test_int8h32_k128_paged_single_token(readout):
    """K = 128 single-token decode on a paged pool (copy-on-new-page for the
    sequences whose last page is new) through the group kernel, both readouts."""
    gdn_paged_case(107, B=6, H=1, HV=2, K=128, V=128, page_size=8, max_len=60, n_share=2, share_pages=2,
                   force_lens={0: 17, 1: 9}, state_dtype=I8, readout=readout)
