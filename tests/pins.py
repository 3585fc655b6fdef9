"""Pins of the oracle to facts fixed outside it.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
a closed form, an invariant the pages state, an independent formulation, or a
library routine. They take no arguments and run in well under a second each
so that ``test_oracle_mutations`` can re-run all of them against oracles with
a planted mistake.

Sources: Circuit.LLM.Mixer ("Delta rule": deltaAttnStep; "Gated memory":
gatedDeltaStep with alpha = 1 a pure delta rule and alpha = 0 forgetting
everything before the write, kdaLiteStep; the delta write overwrites what the
key already stores; prefill is the scan of steps);
flashinfer.gdn_paged.gated_delta_rule_decode_paged (copy-on-new-page rule);
modelopt ... linear_attention.decode (an empty call performs no write);
max.nn.state_space.kda_decode (q, k normalised, q scaled by 1/sqrt(K)).
"""

from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

from oracle import formats
from oracle import gdn as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand_case(seed, K=8, V=8):
    r = np.random.default_rng(seed)
    S = r.standard_normal((K, V))
    q = r.standard_normal(K)
    k = r.standard_normal(K)
    v = r.standard_normal(V)
    return S, q, k, v


def _loops_matvec(x, S):
    """x S by explicit loops (independent of numpy's matmul)."""
    K, V = S.shape
    return np.array([sum(float(x[i]) * float(S[i, j]) for i in range(K)) for j in range(V)])


# ----------------------------------------------------------------------------
# recurrence
# ----------------------------------------------------------------------------

def pin_alpha1_beta0_keeps_state():
    """alpha = 1, beta = 0: the state is unchanged and o = q S0."""
    S, q, k, v = _rand_case(1)
    o, S1 = O.gated_delta_step(S, q, k, v, 1.0, 0.0)
    assert np.array_equal(S1, S), "alpha=1, beta=0 must leave S bit-identical"
    assert np.allclose(o, _loops_matvec(q, S), rtol=0, atol=1e-12)


def pin_alpha0_beta1_writes_outer_product():
    """alpha = 0, beta = 1: S' = k v^T (forget all, then write); o = (q.k) v."""
    S, q, k, v = _rand_case(2)
    o, S1 = O.gated_delta_step(S, q, k, v, 0.0, 1.0)
    ref = np.array([[k[i] * v[j] for j in range(len(v))] for i in range(len(k))])
    assert np.allclose(S1, ref, rtol=0, atol=1e-12)
    assert np.allclose(o, sum(q[i] * k[i] for i in range(len(k))) * v, rtol=0, atol=1e-12)


def pin_unit_key_overwrites():
    """Unit-norm key and beta = 1: k S' = v, whatever alpha and S were."""
    for seed, alpha in ((3, 0.37), (4, 1.0), (5, np.linspace(0.1, 0.9, 8))):
        S, q, k, v = _rand_case(seed)
        kh = k / np.linalg.norm(k)
        _, S1 = O.gated_delta_step(S, q, kh, v, alpha, 1.0)
        assert np.allclose(_loops_matvec(kh, S1), v, rtol=0, atol=1e-12)


def pin_orthonormal_keys_recall():
    """alpha = 1, beta = 1, T <= K orthonormal keys: every key recalls its value."""
    r = np.random.default_rng(6)
    K, V, T = 8, 5, 6
    Qm, _ = np.linalg.qr(r.standard_normal((K, K)))
    keys = Qm[:, :T].T
    vals = r.standard_normal((T, V))
    S = r.standard_normal((K, V))
    for t in range(T):
        _, S = O.gated_delta_step(S, keys[0], keys[t], vals[t], 1.0, 1.0)
    for t in range(T):
        assert np.allclose(_loops_matvec(keys[t], S), vals[t], rtol=0, atol=1e-11)


def pin_beta0_decay_product():
    """beta = 0 for every token: S_T = (prod alpha_t) S_0, per key row for KDA."""
    S, q, k, v = _rand_case(7)
    alphas = [0.9, 0.5, 0.77, 0.31]
    X = S
    for a in alphas:
        _, X = O.gated_delta_step(X, q, k, v, a, 0.0)
    assert np.allclose(X, np.prod(alphas) * S, rtol=1e-14, atol=0)
    r = np.random.default_rng(8)
    vecs = r.uniform(0.1, 1.0, size=(4, S.shape[0]))
    X = S
    for a in vecs:
        _, X = O.gated_delta_step(X, q, k, v, a, 0.0)
    assert np.allclose(X, np.prod(vecs, axis=0)[:, None] * S, rtol=1e-14, atol=0)


def _transition_run(S, qs, ks, vs, alphas, betas):
    """Independent formulation: S_t = A_t S_{t-1} + beta_t k_t v_t^T with
    A_t = (I - beta_t k_t k_t^T) diag(alpha_t); o_t = q_t S_t."""
    K = S.shape[0]
    outs = []
    for q, k, v, a, b in zip(qs, ks, vs, alphas, betas):
        D = np.diag(np.broadcast_to(np.asarray(a, np.float64), (K,)))
        A = (np.eye(K) - b * np.outer(k, k)) @ D
        S = A @ S + b * np.outer(k, v)
        outs.append(q @ S)
    return np.array(outs), S


def pin_transition_matrix_formulation():
    """The literal steps equal the transition-matrix form on tiny random inputs."""
    for seed in range(4):
        r = np.random.default_rng(100 + seed)
        K, V, T = int(r.integers(2, 9)), int(r.integers(2, 9)), int(r.integers(1, 7))
        S0 = r.standard_normal((K, V))
        qs = [O.l2_normalize(r.standard_normal(K)) / math.sqrt(K) for _ in range(T)]
        ks = [O.l2_normalize(r.standard_normal(K)) for _ in range(T)]
        vs = [r.standard_normal(V) for _ in range(T)]
        if seed % 2:
            al = [r.uniform(0.05, 1.0, size=K) for _ in range(T)]
        else:
            al = [float(r.uniform(0.05, 1.0)) for _ in range(T)]
        be = [float(r.uniform(0.0, 1.0)) for _ in range(T)]
        S = S0
        outs = []
        for t in range(T):
            o, S = O.gated_delta_step(S, qs[t], ks[t], vs[t], al[t], be[t])
            outs.append(o)
        ref_o, ref_S = _transition_run(S0, qs, ks, vs, al, be)
        assert np.allclose(np.array(outs), ref_o, rtol=0, atol=1e-12)
        assert np.allclose(S, ref_S, rtol=0, atol=1e-12)


def pin_exact_rational_step():
    """One gated step on 2x2 rational inputs, evaluated exactly with Fractions
    straight from the definitions (decay, v_old = k S, u = beta (v - v_old),
    S' = S + k^T u, o = q S')."""
    F = Fraction
    S = [[F(1), F(2)], [F(3), F(4)]]
    k = [F(3, 5), F(4, 5)]
    q = [F(1, 2), F(-1, 3)]
    v = [F(1), F(-1)]
    alpha, beta = F(1, 2), F(3, 4)
    Sd = [[alpha * x for x in row] for row in S]
    v_old = [k[0] * Sd[0][j] + k[1] * Sd[1][j] for j in range(2)]
    u = [beta * (v[j] - v_old[j]) for j in range(2)]
    S1 = [[Sd[i][j] + k[i] * u[j] for j in range(2)] for i in range(2)]
    o = [q[0] * S1[0][j] + q[1] * S1[1][j] for j in range(2)]
    oo, SS = O.gated_delta_step(np.array([[1.0, 2.0], [3.0, 4.0]]), np.array([0.5, -1 / 3]),
                                np.array([0.6, 0.8]), np.array([1.0, -1.0]), 0.5, 0.75)
    assert np.allclose(SS, np.array([[float(x) for x in r] for r in S1]), rtol=0, atol=1e-15)
    assert np.allclose(oo, np.array([float(x) for x in o]), rtol=0, atol=1e-15)


# ----------------------------------------------------------------------------
# activations
# ----------------------------------------------------------------------------

def pin_activations():
    assert abs(float(O.softplus(0.0)) - math.log(2.0)) < 1e-15
    for x in np.linspace(-30, 30, 61):
        assert abs(float(O.softplus(x)) - math.log1p(math.exp(x))) <= 1e-14 * max(1.0, abs(x))
    assert abs(float(O.softplus(40.0)) - 40.0) < 1e-15
    assert float(O.sigmoid(0.0)) == 0.5
    assert float(O.sigmoid(-np.inf)) == 0.0 and float(O.sigmoid(np.inf)) == 1.0
    for x in (-3.0, -0.2, 0.7, 5.0):
        assert abs(float(O.sigmoid(x)) - 0.5 * (1 + math.tanh(x / 2))) < 1e-15
    # gate limits: alpha = 1 when A_log -> -inf or a + dt_bias -> -inf; alpha -> 0 for huge A_log
    assert O.gdn_alpha(-np.inf, 0.3, 0.1) == 1.0
    assert O.gdn_alpha(0.5, -np.inf, 0.0) == 1.0
    assert O.gdn_alpha(50.0, 0.0, 0.0) == 0.0
    # one value by hand: A_log = ln 2, a + dt_bias = 0 -> g = -2 ln 2, alpha = 1/4
    assert abs(O.gdn_alpha(math.log(2.0), 0.25, -0.25) - 0.25) < 1e-15
    # KDA with every channel alike is the GDN gate on each channel
    vec = O.kda_alpha(0.7, np.full(5, 0.2), np.full(5, -0.4))
    assert np.allclose(vec, O.gdn_alpha(0.7, 0.2, -0.4), rtol=1e-15, atol=0)
    assert O.beta_of(0.3, "probability") == 0.3


def pin_l2_and_scale():
    x = np.array([3.0, 4.0])
    y = O.l2_normalize(x)
    assert abs(y[0] - 3 / math.sqrt(25 + O.L2NORM_EPS)) < 1e-16
    assert np.array_equal(O.l2_normalize(np.zeros(4)), np.zeros(4))
    qh, kh = O.prepare_qk(np.array([0.0, 2.0]), np.array([5.0, 0.0]), 0.5, True)
    assert abs(qh[1] - 0.5 * 2 / math.sqrt(4 + 1e-6)) < 1e-16 and kh[1] == 0.0
    qh, kh = O.prepare_qk(np.array([0.0, 2.0]), np.array([5.0, 0.0]), 0.5, False)
    assert qh[1] == 1.0 and kh[0] == 5.0


# ----------------------------------------------------------------------------
# pool drivers
# ----------------------------------------------------------------------------

def _tiny_pool(seed, num_slots, HV, K, V, layout="V_FIRST"):
    r = np.random.default_rng(seed)
    shape = (num_slots, HV) + ((K, V) if layout == "K_FIRST" else (V, K))
    return (r.standard_normal(shape) * 0.1).astype(np.float32)


def _tiny_tokens(seed, B, T, H, HV, K, V):
    r = np.random.default_rng(seed)
    return dict(q=r.standard_normal((B, T, H, K)), k=r.standard_normal((B, T, H, K)),
                v=r.standard_normal((B, T, HV, V)), a=r.standard_normal((B, T, HV)),
                b=r.standard_normal((B, T, HV)), A_log=r.uniform(0, 2.8, HV),
                dt_bias=r.uniform(-1, 1, HV))


def pin_slots_driver_limits():
    """Through the slot driver: alpha=1/beta=0 keeps every written slot
    bit-identical; alpha=0/beta=1 writes k v^T; a negative slot writes nothing."""
    B, T, H, HV, K, V = 2, 1, 1, 2, 4, 3
    pool = _tiny_pool(11, 4, HV, K, V)
    t = _tiny_tokens(12, B, T, H, HV, K, V)
    keep = dict(t, A_log=np.full(HV, -np.inf), b=np.full((B, T, HV), -np.inf))
    out, writes = O.gdn_decode_slots(keep["q"], keep["k"], keep["v"], keep["a"], keep["b"],
                                     keep["A_log"], keep["dt_bias"], pool, [2, 0])
    for (slot, hv), (st, _) in writes.items():
        assert np.array_equal(st, pool[slot, hv])
    qh = O.l2_normalize(t["q"][0, 0, 0]) / math.sqrt(K)
    assert np.allclose(out[0, 0, 1], _loops_matvec(qh, pool[2, 1].T.astype(np.float64)), atol=1e-12)
    wipe = dict(t, A_log=np.full(HV, 60.0), b=np.full((B, T, HV), np.inf))
    out, writes = O.gdn_decode_slots(wipe["q"], wipe["k"], wipe["v"], wipe["a"], wipe["b"],
                                     wipe["A_log"], wipe["dt_bias"], pool, [1, -1])
    kh = O.l2_normalize(t["k"][0, 0, 0])
    st, _ = writes[(1, 0)]
    assert np.allclose(st.T, np.outer(kh, t["v"][0, 0, 0]).astype(np.float32), atol=1e-7)
    assert set(writes) == {(1, 0), (1, 1)}
    assert np.all(out[1] == 0.0)


def pin_sequential_equals_single_steps():
    """A T-token call equals T one-token calls that thread the state through
    the pool (the scan of gatedDeltaPrefill), for GDN slots and KDA varlen."""
    B, T, H, HV, K, V = 2, 5, 1, 2, 6, 4
    pool = _tiny_pool(21, 3, HV, K, V)
    t = _tiny_tokens(22, B, T, H, HV, K, V)
    idx = [2, 0]
    outT, wT = O.gdn_decode_slots(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"],
                                  t["dt_bias"], pool, idx)
    p = pool.astype(np.float64).copy()
    for s in range(T):
        o1, w1 = O.gdn_decode_slots(t["q"][:, s:s + 1], t["k"][:, s:s + 1], t["v"][:, s:s + 1],
                                    t["a"][:, s:s + 1], t["b"][:, s:s + 1], t["A_log"],
                                    t["dt_bias"], p, idx)
        assert np.allclose(o1[:, 0], outT[:, s], rtol=0, atol=1e-6)
        for (slot, hv), (st, _) in w1.items():
            p[slot, hv] = st
    for (slot, hv), (st, _) in wT.items():
        assert np.allclose(p[slot, hv], st, rtol=0, atol=1e-6)
    # KDA: one sequence of T tokens vs T sequences of one token on the same slot
    r = np.random.default_rng(23)
    Hk = 2
    q = r.standard_normal((T, Hk, K)); k = r.standard_normal((T, Hk, K))
    v = r.standard_normal((T, HV, V)); g = r.standard_normal((T, HV, K))
    bl = r.standard_normal((T, HV)); al = r.uniform(0, 2.8, HV); db = r.uniform(-1, 1, (HV, K))
    kpool = _tiny_pool(24, 2, HV, K, V, "K_FIRST")
    oT, wT = O.kda_decode_varlen(q, k, v, g, bl, al, db, [0, T], kpool, [1])
    p = kpool.astype(np.float64).copy()
    for s in range(T):
        o1, w1 = O.kda_decode_varlen(q[s:s + 1], k[s:s + 1], v[s:s + 1], g[s:s + 1], bl[s:s + 1],
                                     al, db, [0, 1], p, [1])
        assert np.allclose(o1[0], oT[s], rtol=0, atol=1e-6)
        for (slot, hv), (st, _) in w1.items():
            p[slot, hv] = st
    for (slot, hv), (st, _) in wT.items():
        assert np.allclose(p[slot, hv], st, rtol=0, atol=1e-6)


def pin_empty_sequence_writes_nothing():
    HV, K, V = 2, 4, 4
    pool = _tiny_pool(31, 3, HV, K, V, "K_FIRST")
    r = np.random.default_rng(32)
    total = 2
    out, writes = O.kda_decode_varlen(r.standard_normal((total, 2, K)), r.standard_normal((total, 2, K)),
                                      r.standard_normal((total, HV, V)), r.standard_normal((total, HV, K)),
                                      r.standard_normal((total, HV)), np.ones(HV), np.zeros((HV, K)),
                                      [0, 0, 2, 2], pool, [0, 1, 2])
    assert set(s for (s, _) in writes) == {1}


def read_paged_cases():
    cases = []
    with open(os.path.join(GOLDEN, "paged_rule_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            ind, ptr, last, exp = [p.split() for p in line.split(";")]
            cases.append(([int(x) for x in ind], [int(x) for x in ptr], [int(x) for x in last],
                          [tuple(int(y) for y in e.split(",")) for e in exp]))
    return cases


def pin_paged_rule():
    """The copy-on-new-page rule on hand-derived page tables (golden fixture),
    and through the paged driver: the read page is decoded, only write pages
    are written, a shared page read by a new-page sequence stays untouched."""
    for ind, ptr, last, exp in read_paged_cases():
        got = [tuple(r) for r in O.paged_decode_slots(ind, ptr, last).tolist()]
        assert got == exp, (ind, ptr, last, got, exp)
    HV, K, V, H = 2, 4, 4, 1
    pool = _tiny_pool(41, 14, HV, K, V)
    ind, ptr, last = [10, 11, 12, 10, 11, 13], [0, 3, 6], [7, 1]
    t = _tiny_tokens(42, 2, 1, H, HV, K, V)
    out, writes = O.gdn_decode_paged(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"],
                                     t["dt_bias"], pool, ind, ptr, last)
    assert set(p for (p, _) in writes) == {12, 13}
    # sequence 1 opens page 13 from page 11: same result as a slot call reading slot 11
    o_s, w_s = O.gdn_decode_slots(t["q"][1:], t["k"][1:], t["v"][1:], t["a"][1:], t["b"][1:],
                                  t["A_log"], t["dt_bias"], pool, [11])
    assert np.array_equal(out[1], o_s[0])
    for hv in range(HV):
        assert np.array_equal(writes[(13, hv)][0], w_s[(11, hv)][0])


def pin_gqa_map_is_used():
    """G = 2: value heads 0,1 read key head 0 and 2,3 read key head 1. The
    map itself is a convention (parity unpinned); this only pins that it is
    applied, by comparing against single-head calls with the key head picked."""
    B, T, H, HV, K, V = 1, 1, 2, 4, 4, 3
    pool = _tiny_pool(51, 1, HV, K, V)
    t = _tiny_tokens(52, B, T, H, HV, K, V)
    out, _ = O.gdn_decode_slots(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"],
                                t["dt_bias"], pool, [0])
    for hv in range(HV):
        kh = hv // 2
        o1, _ = O.gdn_decode_slots(t["q"][:, :, kh:kh + 1], t["k"][:, :, kh:kh + 1],
                                   t["v"][:, :, hv:hv + 1], t["a"][:, :, hv:hv + 1],
                                   t["b"][:, :, hv:hv + 1], t["A_log"][hv:hv + 1],
                                   t["dt_bias"][hv:hv + 1], pool[:, hv:hv + 1], [0])
        assert np.array_equal(o1[0, 0, 0], out[0, 0, hv])


def pin_layouts_agree():
    """K_FIRST and V_FIRST pools holding the same logical states give the same
    outputs and the same logical written states."""
    B, T, H, HV, K, V = 1, 3, 1, 2, 4, 6
    kf = _tiny_pool(61, 1, HV, K, V, "K_FIRST")
    vf = np.ascontiguousarray(kf.transpose(0, 1, 3, 2))
    t = _tiny_tokens(62, B, T, H, HV, K, V)
    o1, w1 = O.gdn_decode_slots(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"],
                                t["dt_bias"], kf, [0], layout="K_FIRST")
    o2, w2 = O.gdn_decode_slots(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"],
                                t["dt_bias"], vf, [0], layout="V_FIRST")
    assert np.array_equal(o1, o2)
    for key in w1:
        assert np.array_equal(w1[key][0], w2[key][0].T)


# ----------------------------------------------------------------------------
# formats
# ----------------------------------------------------------------------------

def read_e4m3_points():
    pts = []
    with open(os.path.join(GOLDEN, "e4m3_points.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                c, val = line.split()
                pts.append((int(c, 16), float(val)))
    return pts


def pin_e4m3_format():
    for code, val in read_e4m3_points():
        got = float(formats.e4m3_value(np.uint8(code)))
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), (hex(code), got, val)
    codes = np.arange(256, dtype=np.uint8)
    vals = formats.e4m3_value(codes)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254
    # encode(decode(c)) == c for every finite code
    rt = formats.e4m3_encode(vals[finite].astype(np.float32))
    assert np.array_equal(rt, codes[finite])
    # ties go to the even code: midpoints between neighbours of the positive grid
    pos = np.sort(vals[(vals > 0) & finite])
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    enc = formats.e4m3_encode(mids)
    lo = formats.e4m3_encode(pos[:-1].astype(np.float32))
    hi = formats.e4m3_encode(pos[1:].astype(np.float32))
    assert np.all(enc == np.where(lo % 2 == 0, lo, hi))
    # saturation
    assert formats.e4m3_encode(np.float32(1e6)) == 0x7E
    assert formats.e4m3_encode(np.float32(-np.inf)) == 0xFE
    assert formats.e4m3_encode(np.float32(463.9)) == 0x7E


def pin_e4m3_matches_torch():
    """Round-to-nearest-even onto the E4M3 grid agrees with torch's
    float8_e4m3fn conversion for every in-range binary32 value tried."""
    import torch
    r = np.random.default_rng(71)
    x = np.concatenate([r.standard_normal(20000) * 50, r.standard_normal(20000) * 0.01,
                        r.uniform(-448, 448, 20000), r.standard_normal(5000) * 1e-4]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(formats.e4m3_encode(x), ref)


def pin_bf16_matches_torch():
    import torch
    r = np.random.default_rng(72)
    x = np.concatenate([r.standard_normal(50000).astype(np.float32),
                        (r.standard_normal(5000) * 1e-39).astype(np.float32),
                        np.array([3.3895314e38, -3.3895314e38, 0.0, -0.0, 1.0, np.inf], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(formats.f32_to_bf16_bits(x), ref)
    # round trip of every bf16 bit pattern that is not NaN
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = formats.bf16_bits_to_f32(bits)
    keep = ~np.isnan(vals)
    assert np.array_equal(formats.f32_to_bf16_bits(vals[keep]), bits[keep])


def pin_tile_codec():
    r = np.random.default_rng(73)
    x = (r.standard_normal((8, 4)) * 0.3).astype(np.float32)
    codes, s = formats.quantize_tile(x)
    amax = np.max(np.abs(x))
    assert s == np.float32(amax / np.float32(448.0))
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert codes[i] & 0x7F == 0x7E   # the largest magnitude lands on +-448
    deq = formats.dequantize_tile(codes, s)
    # error at most half a grid step of the value's binade (step <= |x|/8, and 2^-9 * s below 2^-6 * s)
    a = np.abs(x / s).astype(np.float64)
    step = np.exp2(np.maximum(np.floor(np.log2(np.maximum(a, 1e-30))), -6) - 3)
    assert np.all(np.abs(deq - x) <= (0.5 * step + 1e-6 * a) * s + 1e-12)
    z, s0 = formats.quantize_tile(np.zeros((3, 3), np.float32))
    assert s0 == 0 and not z.any()
    assert not formats.dequantize_tile(z, s0).any()
    # a tile of one repeated value encodes to +-448 everywhere
    c, s1 = formats.quantize_tile(np.full((2, 2), -0.125, np.float32))
    assert np.all(c == 0xFE) and np.allclose(formats.dequantize_tile(c, s1), -0.125)


def pin_fp8_state_codec_per_tile():
    """quantize_state gives each [K, block_v] column block its own scale."""
    r = np.random.default_rng(74)
    S = r.standard_normal((4, 8)).astype(np.float32)
    S[:, 4:] *= 100
    codes, scales = formats.quantize_state(S, 4)
    assert scales[1] > 50 * scales[0]
    for j in range(2):
        c, s = formats.quantize_tile(S[:, 4 * j:4 * j + 4])
        assert s == scales[j] and np.array_equal(c, codes[:, 4 * j:4 * j + 4])




# ----------------------------------------------------------------------------
# multi-token suffix on a paged pool
# ----------------------------------------------------------------------------

def read_suffix_cases():
    cases = []
    with open(os.path.join(GOLDEN, "paged_suffix_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            ind, ptr, last, ps, T, read, snaps, final = [p.strip() for p in line.split(";")]
            snap = [] if snaps == "-" else [tuple(int(y) for y in z.split(":")) for z in snaps.split()]
            cases.append(([int(x) for x in ind.split()], [int(x) for x in ptr.split()], [int(last)],
                          int(ps), int(T), int(read), snap, int(final)))
    return cases


def pin_paged_suffix_rule():
    """The suffix page rule on hand-derived tables, and T == 1 agrees with
    the copy-on-new-page rule on every table of the single-token fixture."""
    for ind, ptr, last, ps, T, read, snaps, final in read_suffix_cases():
        got = O.suffix_pages(ind, ptr, last, ps, T, 0)
        assert got == (read, snaps, final), (ind, ptr, last, ps, T, got)
    for ind, ptr, last, exp in read_paged_cases():
        for bb in range(len(ptr) - 1):
            n = ptr[bb + 1] - ptr[bb]
            ps = 64
            if last[bb] > ps:
                continue
            r, snaps, w = O.suffix_pages(ind, ptr, last, ps, 1, bb)
            assert (r, w) == exp[bb] and snaps == []


def pin_paged_suffix_equals_single_steps():
    """A T-token suffix equals T single-token paged calls on the sequence
    growing by one token each time, threaded through the pool."""
    ps, HV, K, V, H = 3, 2, 4, 4, 1
    ind = [4, 0, 2, 5, 1]
    L, T = 14, 7                       # 5 pages: positions 0..14? L = 4*3 + 2
    last = [L - ps * (len(ind) - 1)]
    pool = _tiny_pool(81, 6, HV, K, V).astype(np.float64)
    t = _tiny_tokens(82, 1, T, H, HV, K, V)
    out, writes = O.gdn_decode_paged(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], pool,
                                     ind, [0, len(ind)], last, page_size=ps)
    p = pool.copy()
    for s in range(T):
        Ls = L - T + s + 1
        npg = -(-Ls // ps)
        o1, w1 = O.gdn_decode_paged(t["q"][:, s:s + 1], t["k"][:, s:s + 1], t["v"][:, s:s + 1], t["a"][:, s:s + 1],
                                    t["b"][:, s:s + 1], t["A_log"], t["dt_bias"], p, ind[:npg], [0, npg],
                                    [Ls - ps * (npg - 1)])
        assert np.allclose(o1[0, 0], out[0, s], rtol=0, atol=1e-6)
        for (page, hv), (st, _) in w1.items():
            p[page, hv] = st
    for (page, hv), (st, _) in writes.items():
        assert np.allclose(p[page, hv], st, rtol=0, atol=1e-6), (page, hv)
    # pages the suffix does not reach keep their content
    touched = {pg for (pg, _) in writes}
    for pg in range(6):
        if pg not in touched:
            assert np.array_equal(p[pg], pool[pg])


def pin_prefill_matches_decode_and_split():
    """A fresh prefill of L tokens from a zero state equals: (a) the slot
    decode of the same L tokens from a zero state, with the page snapshots
    equal to the states after each page's last token; (b) a prefill of the
    first n tokens followed by a continued prefill of the rest."""
    ps, H, HV, K, V = 4, 1, 2, 4, 4
    L = 11
    ind = [3, 0, 5]                    # pages of positions 0-3, 4-7, 8-10
    t = _tiny_tokens(91, 1, L, H, HV, K, V)
    tok = {n: t[n][0] for n in ("q", "k", "v", "a", "b")}
    pool = _tiny_pool(92, 6, HV, K, V).astype(np.float64)
    out, writes = O.gdn_prefill_paged(tok["q"], tok["k"], tok["v"], tok["a"], tok["b"], t["A_log"], t["dt_bias"],
                                      [0, L], pool, ind, [0, 3], [3], ps)
    zero = np.zeros((1, HV, V, K))
    ref_out, _ = O.gdn_decode_slots(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], zero, [0])
    assert np.allclose(out, ref_out[0], rtol=0, atol=1e-12)
    for n_pref, page in ((4, 3), (8, 0), (11, 5)):
        _, w = O.gdn_decode_slots(t["q"][:, :n_pref], t["k"][:, :n_pref], t["v"][:, :n_pref], t["a"][:, :n_pref],
                                  t["b"][:, :n_pref], t["A_log"], t["dt_bias"], zero, [0])
        for hv in range(HV):
            assert np.allclose(writes[(page, hv)][0], w[(0, hv)][0], rtol=0, atol=1e-6)
    assert {pg for (pg, _) in writes} == {3, 0, 5}
    # split: 6 tokens (pages 3 and half of 0), then the remaining 5
    o1, w1 = O.gdn_prefill_paged(*(tok[n][:6] for n in ("q", "k", "v", "a", "b")), t["A_log"], t["dt_bias"],
                                 [0, 6], pool, ind[:2], [0, 2], [2], ps)
    p = pool.copy()
    for (pg, hv), (st, _) in w1.items():
        p[pg, hv] = st
    o2, w2 = O.gdn_prefill_paged(*(tok[n][6:] for n in ("q", "k", "v", "a", "b")), t["A_log"], t["dt_bias"],
                                 [0, 5], p, ind, [0, 3], [3], ps)
    assert np.allclose(np.concatenate([o1, o2]), out, rtol=0, atol=1e-6)
    for key in writes:
        got = w2[key][0] if key in w2 else w1[key][0]
        assert np.allclose(got, writes[key][0], rtol=0, atol=1e-6), key


# ----------------------------------------------------------------------------
# int8_hadamard32 state codec (ModelOpt linear-attention config: one scale per
# key channel and 32 values)
# ----------------------------------------------------------------------------

def pin_hadamard32_matches_scipy():
    """R = H32 / sqrt(32) against scipy's Sylvester Hadamard matrix; R R = I."""
    import scipy.linalg
    Hs = scipy.linalg.hadamard(32).astype(np.float64) / math.sqrt(32.0)
    R = formats.hadamard32(np.eye(32))            # row i is R e_i (R is symmetric)
    assert np.allclose(R, Hs, rtol=0, atol=1e-15)
    x = np.random.default_rng(80).standard_normal((3, 5, 32))
    assert np.allclose(formats.hadamard32(x), x @ Hs.T, rtol=0, atol=1e-13)
    assert np.allclose(formats.hadamard32(formats.hadamard32(x)), x, rtol=0, atol=1e-13)
    x32 = x.astype(np.float32)
    y32 = formats.hadamard32(x32)
    assert y32.dtype == np.float32
    assert np.allclose(y32, x32.astype(np.float64) @ Hs.T, rtol=0, atol=4e-6)


def pin_hadamard32_closed_forms():
    """R 1 = sqrt(32) e_0; R e_j has entries (-1)^popcount(i & j) / sqrt(32)."""
    y = formats.hadamard32(np.ones(32))
    assert abs(y[0] - math.sqrt(32.0)) < 1e-13 and np.all(np.abs(y[1:]) < 1e-13)
    for j in (0, 1, 5, 17, 31):
        e = np.zeros(32)
        e[j] = 1.0
        ref = np.array([(-1.0) ** bin(i & j).count("1") for i in range(32)]) / math.sqrt(32.0)
        assert np.allclose(formats.hadamard32(e), ref, rtol=0, atol=1e-15), j
    # 0x3E3504F3 is the binary32 nearest to 1/sqrt(32): its neighbours are farther
    c = float(formats.INV_SQRT32_F32)
    lo = float(np.nextafter(np.float32(c), np.float32(0)))
    hi = float(np.nextafter(np.float32(c), np.float32(1)))
    err = lambda z: abs(Fraction(z) ** 2 * 32 - 1)
    assert err(c) < err(lo) and err(c) < err(hi)


def pin_int8_rounding_points():
    """With amax = 127 the scale is 1, and codes are the integers nearest to
    the rotated values, ties to even."""
    y = np.zeros(32, np.float32)
    pts = [127.0, 2.5, -2.5, 3.5, 0.5, -0.5, 1.5, 126.5, -126.5, 0.49999997, -1.5000001, 64.0]
    want = [127, 2, -2, 4, 0, 0, 2, 126, -126, 0, -2, 64]
    y[:len(pts)] = pts
    codes, s = formats.quantize_rotated_groups(y[None])
    assert s[0] == np.float32(1.0)
    assert codes[0, :len(want)].tolist() == want and not codes[0, len(want):].any()
    # a group at a scale that is a power of two rounds the same way
    codes2, s2 = formats.quantize_rotated_groups((y * np.float32(2.0 ** -9))[None])
    assert s2[0] == np.float32(2.0 ** -9) and np.array_equal(codes2, codes)


def pin_h32_codec_groups():
    """One scale per key channel and 32 values: scales [V/32, K]; a state that
    is nonzero in one key row, or in one 32-value group, sets only those scales."""
    r = np.random.default_rng(81)
    K, V = 6, 96
    S = np.zeros((K, V), np.float32)
    S[4] = r.standard_normal(V)
    codes, sc = formats.quantize_state_h32(S)
    assert sc.shape == (V // 32, K)
    assert np.all(sc[:, 4] > 0) and not np.delete(sc, 4, axis=1).any()
    assert not np.delete(codes, 4, axis=0).any()
    S = np.zeros((K, V), np.float32)
    S[:, 32:64] = r.standard_normal((K, 32))
    codes, sc = formats.quantize_state_h32(S)
    assert np.all(sc[1] > 0) and not sc[0].any() and not sc[2].any()
    assert not codes[:, :32].any() and not codes[:, 64:].any()
    # each group is the codec of its own 32 values
    S = r.standard_normal((K, V)).astype(np.float32)
    codes, sc = formats.quantize_state_h32(S)
    for k in range(K):
        for g in range(V // 32):
            c1, s1 = formats.quantize_rotated_groups(formats.hadamard32(S[k, 32 * g:32 * g + 32])[None])
            assert s1[0] == sc[g, k] and np.array_equal(c1[0], codes[k, 32 * g:32 * g + 32])


def pin_h32_codec_error_and_extremes():
    """Round trip error within the rotated-domain bound (half a code step per
    element, carried over unchanged by an orthonormal rotation); the largest
    rotated value codes to +-127; zero groups store 0; sign symmetry; a spike
    spreads over the whole group."""
    r = np.random.default_rng(82)
    K, V = 8, 64
    S = (r.standard_normal((K, V)) * np.exp(r.uniform(-6, 6, (K, 1)))).astype(np.float32)
    S[3, :32] = 0
    codes, sc = formats.quantize_state_h32(S)
    deq = formats.dequantize_state_h32(codes, sc)
    Hs = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(32)] for i in range(32)]) / math.sqrt(32)
    for k in range(K):
        for g in range(V // 32):
            x = S[k, 32 * g:32 * g + 32].astype(np.float64)
            y = Hs @ x
            amax = np.max(np.abs(y))
            if amax == 0:
                assert sc[g, k] == 0 and not codes[k, 32 * g:32 * g + 32].any()
                assert not deq[k, 32 * g:32 * g + 32].any()
                continue
            assert abs(sc[g, k] - amax / 127) <= 2e-6 * amax / 127
            assert np.max(np.abs(codes[k, 32 * g:32 * g + 32].astype(int))) == 127
            err = np.linalg.norm(deq[k, 32 * g:32 * g + 32] - x)
            assert err <= math.sqrt(32) * 0.5 * sc[g, k] * (1 + 1e-4) + 1e-5 * np.linalg.norm(x), (k, g)
    cn, sn = formats.quantize_state_h32(-S)
    assert np.array_equal(sn, sc) and np.array_equal(cn, -codes)
    spike = np.zeros((1, 32), np.float32)
    spike[0, 7] = 3.0
    c, s = formats.quantize_state_h32(spike)
    assert np.all(np.abs(c.astype(int)) == 127)
    assert np.allclose(formats.dequantize_state_h32(c, s), spike, rtol=0, atol=1e-6)


def pin_h32_state_decode_is_codec_around_f32_step():
    """A decode on an int8_hadamard32 pool is the fp32 decode of the decoded
    state, with the new state stored through the codec (both layouts)."""
    r = np.random.default_rng(83)
    B, T, H, HV, K, V = 2, 2, 1, 2, 8, 32
    q, k = r.standard_normal((B, T, H, K)), r.standard_normal((B, T, H, K))
    v = r.standard_normal((B, T, HV, V))
    a, b = r.standard_normal((B, T, HV)), r.standard_normal((B, T, HV))
    A_log, dt = r.uniform(0, 2, HV), r.uniform(-1, 1, HV)
    for layout in ("K_FIRST", "V_FIRST"):
        pool8, sc8, pool32 = {}, {}, {}
        for slot in range(2):
            for hv in range(HV):
                c = np.clip(np.rint(r.standard_normal((K, V)) * 40), -127, 127).astype(np.int8)
                s = r.uniform(1e-3, 2e-3, (V // 32, K)).astype(np.float32)
                pool8[slot, hv] = O._from_kv(c, layout)
                sc8[slot, hv] = s
                pool32[slot, hv] = O._from_kv(formats.dequantize_state_h32(c, s), layout)
        idx = np.array([1, 0])
        o8, w8 = O.gdn_decode_slots(q, k, v, a, b, A_log, dt, pool8, idx, layout=layout,
                                    state_dtype="int8_hadamard32", state_scales=sc8)
        o32, w32 = O.gdn_decode_slots(q[:, :1], k[:, :1], v[:, :1], a[:, :1], b[:, :1], A_log, dt, pool32, idx,
                                      layout=layout)
        assert np.array_equal(o8[:, :1], o32)
        first8 = O.gdn_decode_slots(q[:, :1], k[:, :1], v[:, :1], a[:, :1], b[:, :1], A_log, dt, pool8, idx,
                                    layout=layout, state_dtype="int8_hadamard32", state_scales=sc8)[1]
        for key, (st32, _) in w32.items():
            c, s = formats.quantize_state_h32(O._to_kv(st32, layout))
            assert np.array_equal(O._to_kv(first8[key][0], layout), c) and np.array_equal(first8[key][1], s)
        assert set(w8) == set(w32)


# ----------------------------------------------------------------------------
# per-token write events and the readout flag
# (modelopt ... linear_attention.decode, recurrent_decode_reference: one
# sequence runs with explicit token write events, and an empty call performs
# no write; ...linear_attention.config, LinearAttentionDecodeConfig.readout:
# 'working' or 'stored')
# ----------------------------------------------------------------------------

CODED = ("bf16", "fp8_e4m3", "int8_hadamard32")


def _encode_kv(S_kv, state_dtype, layout):
    """A float [K, V] state put into a pool entry of ``state_dtype`` through
    the pinned format routines: (stored 2-D array in the layout, scales)."""
    S32 = np.asarray(S_kv, np.float32)
    if state_dtype == "f32":
        return O._from_kv(S32, layout), None
    if state_dtype == "bf16":
        return O._from_kv(formats.f32_to_bf16_bits(S32), layout), None
    if state_dtype == "fp8_e4m3":
        c, s = formats.quantize_state(S32, 64)
        return O._from_kv(c, layout), s
    c, s = formats.quantize_state_h32(S32)
    return O._from_kv(c, layout), s


def _decode_entry(stored, scales, state_dtype, layout):
    """A pool entry back to a float64 [K, V] state through the pinned format
    routines (not through the oracle's load_state)."""
    kv = O._to_kv(np.asarray(stored), layout)
    if state_dtype == "f32":
        return kv.astype(np.float64)
    if state_dtype == "bf16":
        return formats.bf16_bits_to_f32(kv).astype(np.float64)
    if state_dtype == "fp8_e4m3":
        return formats.dequantize_state(kv, scales, 64).astype(np.float64)
    return formats.dequantize_state_h32(kv, scales).astype(np.float64)


def _coded_pool(seed, slots, HV, K, V, state_dtype, layout):
    """Pool and scales as dicts keyed by (slot, hv); states ~ N(0, 0.1)."""
    r = np.random.default_rng(seed)
    pool, scales = {}, {}
    for s in range(slots):
        for hv in range(HV):
            pool[s, hv], scales[s, hv] = _encode_kv(r.standard_normal((K, V)) * 0.1, state_dtype, layout)
    return pool, scales


def _slots_call(t, pool, scales, idx, state_dtype, layout, readout_mode, sl=slice(None)):
    return O.gdn_decode_slots(t["q"][:, sl], t["k"][:, sl], t["v"][:, sl], t["a"][:, sl], t["b"][:, sl],
                              t["A_log"], t["dt_bias"], pool, idx, layout=layout, state_dtype=state_dtype,
                              state_scales=scales, readout_mode=readout_mode)


def _apply(pool, scales, writes):
    pool, scales = dict(pool), dict(scales)
    for key, (st, sc) in writes.items():
        pool[key], scales[key] = st, sc
    return pool, scales


def _same_entry(x, y):
    (a, sa), (b, sb) = x, y
    return np.array_equal(a, b) and (sa is None and sb is None or np.array_equal(sa, sb))


def pin_token_write_events_thread_through_the_pool():
    """A T-token call on a bf16, fp8 or int8_hadamard32 pool equals T
    one-token calls that pass the state through the pool between tokens,
    bit for bit (outputs and every stored byte and scale), for either
    readout; and it differs from carrying the state at full precision
    across the call and encoding it once at the end, so the rounding of
    every token is what the equality checks."""
    B, T, H, HV, K, V = 2, 4, 1, 2, 8, 64
    idx = [2, 0]
    for n, sd in enumerate(CODED):
        layout = ("V_FIRST", "K_FIRST")[n % 2]
        t = _tiny_tokens(300 + n, B, T, H, HV, K, V)
        pool, scales = _coded_pool(310 + n, 3, HV, K, V, sd, layout)
        for ro in ("working", "stored"):
            outT, wT = _slots_call(t, pool, scales, idx, sd, layout, ro)
            p, sc = pool, scales
            for s in range(T):
                o1, w1 = _slots_call(t, p, sc, idx, sd, layout, ro, slice(s, s + 1))
                assert np.array_equal(o1[:, 0], outT[:, s]), (sd, ro, s)
                p, sc = _apply(p, sc, w1)
            assert set(wT) == {(sl, hv) for sl in idx for hv in range(HV)}
            for key in wT:
                assert _same_entry(wT[key], (p[key], sc[key])), (sd, ro, key)
        # full precision across the call, encoded once: a different pool
        f64 = {key: O._from_kv(_decode_entry(pool[key], scales[key], sd, layout), layout) for key in pool}
        _, w64 = O.gdn_decode_slots(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], f64, idx,
                                    layout=layout)
        differs = 0
        for key in wT:
            once = _encode_kv(O._to_kv(w64[key][0], layout), sd, layout)
            differs += not _same_entry(once, wT[key])
        assert differs > 0, sd


def pin_stored_readout_reads_the_stored_state():
    """readout='stored': every token's output is q^ times the state the pool
    holds after that token (decoded by the format routines, product by
    loops). readout='working': the output of a one-token call equals the
    fp32-state call on the decoded pool, and the stored payload is that
    call's new state encoded (the codec wraps the fp32 step). The two
    readouts differ on these coded pools."""
    B, T, H, HV, K, V = 1, 3, 1, 2, 8, 64
    idx = [1]
    for n, sd in enumerate(CODED):
        layout = ("K_FIRST", "V_FIRST")[n % 2]
        t = _tiny_tokens(320 + n, B, T, H, HV, K, V)
        pool, scales = _coded_pool(330 + n, 2, HV, K, V, sd, layout)
        outS, _ = _slots_call(t, pool, scales, idx, sd, layout, "stored")
        outW, _ = _slots_call(t, pool, scales, idx, sd, layout, "working")
        p, sc = pool, scales
        for s in range(T):
            o1, w1 = _slots_call(t, p, sc, idx, sd, layout, "stored", slice(s, s + 1))
            p, sc = _apply(p, sc, w1)
            for hv in range(HV):
                qh = O.l2_normalize(t["q"][0, s, 0]) / math.sqrt(K)
                S_after = _decode_entry(p[idx[0], hv], sc[idx[0], hv], sd, layout)
                ref = _loops_matvec(qh, S_after)
                scale = np.max(np.abs(ref))
                assert np.max(np.abs(o1[0, 0, hv] - ref)) <= 1e-12 * scale, (sd, s, hv)
                assert np.max(np.abs(outS[0, s, hv] - ref)) <= 1e-12 * scale, (sd, s, hv)
            assert np.max(np.abs(outW[0] - outS[0])) > 1e-6 * np.max(np.abs(outS[0])), sd
        # working readout: the codec around the fp32 step, one token from the initial pool
        dec = {key: O._from_kv(_decode_entry(pool[key], scales[key], sd, layout).astype(np.float32), layout)
               for key in pool}
        o32, w32 = _slots_call(t, dec, None, idx, "f32", layout, "working", slice(0, 1))
        oW, wW = _slots_call(t, pool, scales, idx, sd, layout, "working", slice(0, 1))
        assert np.array_equal(o32, oW), sd
        for key in w32:
            assert _same_entry(_encode_kv(O._to_kv(w32[key][0], layout), sd, layout), wW[key]), (sd, key)


def pin_token_write_events_paged_and_kda():
    """The same per-token write events on the other drivers: a paged suffix
    (every page snapshot and the final page) and a KDA varlen sequence equal
    one-token calls threaded through the pool, bit for bit, on bf16 and fp8
    pools."""
    ps, H, HV, K, V = 3, 1, 2, 8, 64
    ind = [4, 0, 2, 5, 1]
    L, T = 14, 7
    last = [L - ps * (len(ind) - 1)]
    for n, sd in enumerate(("bf16", "fp8_e4m3")):
        pool, scales = _coded_pool(340 + n, 6, HV, K, V, sd, "V_FIRST")
        t = _tiny_tokens(350 + n, 1, T, H, HV, K, V)
        out, writes = O.gdn_decode_paged(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"], pool,
                                         ind, [0, len(ind)], last, page_size=ps, state_dtype=sd,
                                         state_scales=scales)
        p, sc = pool, scales
        for s in range(T):
            Ls = L - T + s + 1
            npg = -(-Ls // ps)
            o1, w1 = O.gdn_decode_paged(t["q"][:, s:s + 1], t["k"][:, s:s + 1], t["v"][:, s:s + 1],
                                        t["a"][:, s:s + 1], t["b"][:, s:s + 1], t["A_log"], t["dt_bias"], p,
                                        ind[:npg], [0, npg], [Ls - ps * (npg - 1)], state_dtype=sd,
                                        state_scales=sc)
            assert np.array_equal(o1[0, 0], out[0, s]), (sd, s)
            p, sc = _apply(p, sc, w1)
        assert len({pg for (pg, _) in writes}) >= 2
        for key in writes:
            assert _same_entry(writes[key], (p[key], sc[key])), (sd, key)
        # KDA: one sequence of T tokens vs T one-token sequences on the same slot
        r = np.random.default_rng(360 + n)
        q = r.standard_normal((T, H, K)); k = r.standard_normal((T, H, K))
        v = r.standard_normal((T, HV, V)); g = r.standard_normal((T, HV, K))
        bl = r.standard_normal((T, HV)); al = r.uniform(0, 2.8, HV); db = r.uniform(-1, 1, (HV, K))
        kp, ks = _coded_pool(370 + n, 2, HV, K, V, sd, "K_FIRST")
        oT, wT = O.kda_decode_varlen(q, k, v, g, bl, al, db, [0, T], kp, [1], state_dtype=sd, state_scales=ks)
        p, sc = kp, ks
        for s in range(T):
            o1, w1 = O.kda_decode_varlen(q[s:s + 1], k[s:s + 1], v[s:s + 1], g[s:s + 1], bl[s:s + 1], al, db,
                                         [0, 1], p, [1], state_dtype=sd, state_scales=sc)
            assert np.array_equal(o1[0], oT[s]), (sd, s)
            p, sc = _apply(p, sc, w1)
        for key in wT:
            assert _same_entry(wT[key], (p[key], sc[key])), (sd, key)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
