"""Host logic of the seeded input generators (CPU only)."""

import numpy as np

import workloads as W


def test_paged_table_invariants():
    w = W.WORKLOADS["paged"]
    pt = W.paged_table(w.seed, w.B, w.page_size, w.max_len, w.n_share, w.share_pages,
                       force_lens={0: 1025, 1: 1025})
    assert pt.page_indptr[0] == 0 and np.all(np.diff(pt.page_indptr) >= 1)
    assert len(pt.page_indices) == pt.page_indptr[-1]
    assert np.all((pt.last_page_len >= 1) & (pt.last_page_len <= w.page_size))
    assert np.all((pt.seq_lens >= 2) & (pt.seq_lens <= w.max_len))
    npages = np.diff(pt.page_indptr)
    assert np.array_equal(npages, -(-pt.seq_lens // w.page_size))
    # sharers start with the same prefix pages and go past it
    for b in range(w.n_share):
        row = pt.page_indices[pt.page_indptr[b]:pt.page_indptr[b + 1]]
        assert np.array_equal(row[:w.share_pages], pt.shared_pages)
        assert pt.seq_lens[b] > w.share_pages * w.page_size
    # forced sequences open a new page right after the shared prefix
    assert pt.last_page_len[0] == 1 and pt.last_page_len[1] == 1
    # write pages (last page of each sequence) are distinct and never shared
    last = pt.page_indices[pt.page_indptr[1:] - 1]
    assert len(set(last.tolist())) == w.B
    assert not set(last.tolist()) & set(pt.shared_pages.tolist())
    # every page id is used, only the shared ones more than once
    ids, counts = np.unique(pt.page_indices, return_counts=True)
    assert len(ids) == pt.num_pages and ids.max() == pt.num_pages - 1
    assert set(ids[counts > 1].tolist()) == set(pt.shared_pages.tolist())


def test_slot_rotations_disjoint_and_reproducible():
    sets = [W.slot_indices(1, 64, 256, r) for r in range(4)]
    allv = np.concatenate(sets)
    assert len(set(allv.tolist())) == 256
    assert np.array_equal(sets[0], W.slot_indices(1, 64, 256, 0))


def test_varlen_offsets():
    cu = W.varlen_offsets(3, 32, 8)
    lens = np.diff(cu)
    assert cu[0] == 0 and np.all((lens >= 1) & (lens <= 8)) and cu.dtype == np.int32


def test_layouts_hold_same_logical_state():
    a, _ = W.slot_state(3, 5, 2, 8, 4, "K_FIRST", "f32")
    b, _ = W.slot_state(3, 5, 2, 8, 4, "V_FIRST", "f32")
    assert np.array_equal(a, b.transpose(0, 2, 1))
    bits, _ = W.slot_state(3, 5, 2, 8, 4, "V_FIRST", "bf16")
    assert bits.dtype == np.uint16 and bits.shape == (2, 4, 8)
    codes, scales = W.slot_state(4, 0, 2, 8, 128, "V_FIRST", "fp8_e4m3", 64)
    assert codes.dtype == np.uint8 and scales.shape == (2, 2)
    assert not np.any((codes & 0x7F) == 0x7F)   # no NaN codes
    c8k, s8k = W.slot_state(5, 1, 2, 8, 64, "K_FIRST", "int8_hadamard32")
    c8v, s8v = W.slot_state(5, 1, 2, 8, 64, "V_FIRST", "int8_hadamard32")
    assert c8k.dtype == np.int8 and np.array_equal(c8k, c8v.transpose(0, 2, 1))
    assert s8k.shape == (2, 2, 8) and np.array_equal(s8k, s8v) and np.all(s8k > 0)
    assert int(np.abs(c8k.astype(int)).max()) <= 127


def test_bf16_inputs_are_representable():
    t = W.gdn_tokens(1, 2, 1, 2, 4, 8, 8, "bf16")
    for n in ("q", "k", "v", "a", "b"):
        x = t[n].view(np.uint32)
        assert np.all((x & 0xFFFF) == 0)


def test_profile_traffic_lookup_never_raises():
    """bench.py reads the committed ncu summaries: a summary whose listed
    kernel sources changed or are gone reports no traffic instead of failing."""
    import bench
    assert bench.source_digest(["no_such_kernel.cuh"]) is None
    for wl in W.WORKLOADS:
        t, src = bench.profiled_traffic(wl)
        assert t is None or t >= 0  # an L2-resident workload can read no DRAM at all
        assert (src is None) == (t is None)
        assert src is None or src.startswith(f"profiles/gdn_decode_{wl}_ncu.md")


def test_oracle_all_cores_workers():
    """The all-cores CPU baseline: separate oracle interpreters over one
    window, summed; a worker that cannot run its job reports failure."""
    import bench
    B, T, H, HV, K, V = 2, 1, 1, 2, 32, 32
    t = W.gdn_tokens(5, B, T, H, HV, K, V, "f32")
    idx = np.array([0, 1])
    states, _ = W.host_pool(5, idx.tolist(), HV, K, V, "V_FIRST", "f32")
    args = tuple(t[n] for n in ("q", "k", "v", "a", "b")) + (t["A_log"], t["dt_bias"], states, idx)
    job = {"fn": "gdn_decode_slots", "args": args, "kw": {"layout": "V_FIRST"}, "tokens_per_call": B * T}
    v = bench.oracle_all_cores([job, job], 0.3)
    assert v is not None and v > 0
    assert bench.oracle_all_cores([dict(job, fn="no_such_function")], 0.3) is None
    assert 1 <= bench.host_cores(4) <= 4


def test_reference_arm_json_line():
    """bench.py --impl reference times the oracle on the host and prints one
    JSON line; a rank other than 0 prints nothing and exits 0."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "2", "--warmup", "1"]
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=root, env=env)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["steps"] == 2 and d["value"] > 0
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    r1 = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=root,
                        env=dict(os.environ, RANK="1", WORLD_SIZE="2"))
    assert r1.returncode == 0 and not r1.stdout.strip()
