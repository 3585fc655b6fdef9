"""Seeded synthetic inputs for gated delta-rule decode, shared by the tests,
the bench and the oracle.

This module holds none of the method's arithmetic: only random draws, casts
to the storage dtypes through torch's own conversions, and index
bookkeeping (slot permutations, CSR page tables, varlen offsets). Both the
CUDA path and the oracle consume exactly the values it returns; values for
bf16 inputs are returned as binary32 arrays that hold bf16-representable
numbers.

Workloads (sizes and distributions of the decode problems the pages pose):

* ``tiny``  GDN, B=1, H=HV=4, K=V=32, T=16, fp32 everything; seed 0.
* ``slots`` GDN slot pool, T=1, B=64, H=16, HV=32, K=V=128, bf16 q/k/v/a/b,
  fp32 pool [256, 32, 128, 128] V_FIRST, indices a random 64-of-256; seed 1.
* ``paged`` GDN paged pool, T=1, B=128, page_size=64, lengths U[2, 4096],
  16 sequences sharing a 1024-token prefix of full pages, fp32 pool
  [num_pages, 32, 128, 128]; seed 2.
* ``kda``   KDA varlen, 32 sequences of U[1, 8] tokens, Hk=HV=32,
  K=V=128, bf16 q/k/v/raw_gate/beta_logits, fp32 pool [64, 32, 128, 128];
  K_FIRST then V_FIRST; seed 3.
* ``kda_long`` KDA varlen with long runs (a prefill): 8 sequences of
  U[512, 1024] tokens, otherwise as ``kda``, fp32 pool [8, 32, 128, 128]
  K_FIRST; seed 6.
* ``fp8``   GDN slot pool, T=1, B=1024, H=16, HV=32, K=V=128, bf16 inputs,
  fp8_e4m3 pool [1024, 32, 128, 128] with one fp32 scale per [128, 64] tile,
  indices a random permutation of 1024; seed 4.
* ``int8``  as ``fp8`` with an int8_hadamard32 pool [1024, 32, 128, 128] and
  fp32 scales [1024, 32, 4, 128] (one per 32 values of a key channel); seed 5.

Distributions (all workloads): q, k, v ~ N(0, 1); A_log ~ U(0, 2.8);
a ~ N(0, 1); dt_bias ~ U(-1, 1); b ~ N(0, 1); initial state ~ N(0, 0.1)
(0.1 read as the standard deviation); KDA raw_gate ~ N(0, 1) and
beta_logits ~ N(0, 1).
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Sequence

import numpy as np
import torch

# stream ids for independent draws from one seed
_TOKENS, _PARAMS, _STATE, _INDEX, _LENGTHS, _PAGES = 1, 2, 3, 4, 5, 6


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # 'gdn_slots' | 'gdn_paged' | 'kda_varlen'
    seed: int
    B: int
    T: int
    H: int
    HV: int
    K: int
    V: int
    in_dtype: str             # 'f32' | 'bf16'
    state_dtype: str          # 'f32' | 'bf16' | 'fp8_e4m3' | 'int8_hadamard32'
    layout: str               # 'K_FIRST' | 'V_FIRST'
    num_slots: int = 0        # slot pools
    page_size: int = 0        # paged pools
    max_len: int = 0          # paged: lengths U[2, max_len]; kda: tokens U[min_len, max_len]
    min_len: int = 1          # kda: shortest run
    n_share: int = 0          # paged: sequences sharing the prefix
    share_pages: int = 0      # paged: full pages in the shared prefix
    block_v: int = 64


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", "gdn_slots", 0, B=1, T=16, H=4, HV=4, K=32, V=32,
                     in_dtype="f32", state_dtype="f32", layout="V_FIRST", num_slots=3),
    "slots": Workload("slots", "gdn_slots", 1, B=64, T=1, H=16, HV=32, K=128, V=128,
                      in_dtype="bf16", state_dtype="f32", layout="V_FIRST", num_slots=256),
    "paged": Workload("paged", "gdn_paged", 2, B=128, T=1, H=16, HV=32, K=128, V=128,
                      in_dtype="bf16", state_dtype="f32", layout="V_FIRST", page_size=64,
                      max_len=4096, n_share=16, share_pages=16),
    "kda": Workload("kda", "kda_varlen", 3, B=32, T=0, H=32, HV=32, K=128, V=128,
                    in_dtype="bf16", state_dtype="f32", layout="K_FIRST", num_slots=64,
                    max_len=8),
    "kda_long": Workload("kda_long", "kda_varlen", 6, B=8, T=0, H=32, HV=32, K=128, V=128,
                         in_dtype="bf16", state_dtype="f32", layout="K_FIRST", num_slots=8,
                         max_len=1024, min_len=512),
    "fp8": Workload("fp8", "gdn_slots", 4, B=1024, T=1, H=16, HV=32, K=128, V=128,
                    in_dtype="bf16", state_dtype="fp8_e4m3", layout="V_FIRST",
                    num_slots=1024, block_v=64),
    "int8": Workload("int8", "gdn_slots", 5, B=1024, T=1, H=16, HV=32, K=128, V=128,
                     in_dtype="bf16", state_dtype="int8_hadamard32", layout="V_FIRST",
                     num_slots=1024),
}


def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), *[int(s) for s in stream]])


def as_dtype_values(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round a binary32 array to the input dtype (via torch) and return binary32 values."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(dtype)


def torch_dtype(dtype: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]


# ----------------------------------------------------------------------------
# token inputs
# ----------------------------------------------------------------------------

def gdn_tokens(seed, B, T, H, HV, K, V, in_dtype="bf16", stream=0) -> Dict[str, np.ndarray]:
    """q, k [B,T,H,K]; v [B,T,HV,V]; a, b [B,T,HV]; A_log, dt_bias [HV] (fp32)."""
    r = _rng(seed, _TOKENS, stream)
    d = {
        "q": r.standard_normal((B, T, H, K), dtype=np.float32),
        "k": r.standard_normal((B, T, H, K), dtype=np.float32),
        "v": r.standard_normal((B, T, HV, V), dtype=np.float32),
        "a": r.standard_normal((B, T, HV), dtype=np.float32),
        "b": r.standard_normal((B, T, HV), dtype=np.float32),
    }
    d = {n: as_dtype_values(x, in_dtype) for n, x in d.items()}
    p = _rng(seed, _PARAMS)
    d["A_log"] = p.uniform(0.0, 2.8, size=HV).astype(np.float32)
    d["dt_bias"] = p.uniform(-1.0, 1.0, size=HV).astype(np.float32)
    return d


def varlen_gdn_tokens(seed, total, H, HV, K, V, in_dtype="bf16", stream=0) -> Dict[str, np.ndarray]:
    """GDN token inputs on a varlen token axis: q, k [total,H,K]; v [total,HV,V];
    a, b [total,HV]; A_log, dt_bias [HV] (fp32)."""
    d = gdn_tokens(seed, 1, total, H, HV, K, V, in_dtype, stream)
    return {n: (x[0] if n not in ("A_log", "dt_bias") else x) for n, x in d.items()}


def prefill_runs(seed, lens, fresh_every=2):
    """New-run lengths for prefill tests: every ``fresh_every``-th sequence is
    fresh (the whole sequence is new), the others append U[1, L-1] tokens,
    and the last one appends nothing. Returns cu_seqlens [B+1] int32."""
    r = _rng(seed, _LENGTHS, 7)
    n = []
    for bb, L in enumerate(lens):
        if bb == len(lens) - 1 and len(lens) > 2:
            n.append(0)
        elif bb % fresh_every == 0 or L < 2:
            n.append(int(L))
        else:
            n.append(int(r.integers(1, L)))
    return np.concatenate([[0], np.cumsum(n)]).astype(np.int32)


def kda_tokens(seed, total, Hk, HV, K, V, in_dtype="bf16", stream=0) -> Dict[str, np.ndarray]:
    """q, k [total,Hk,K]; v [total,HV,V]; raw_gate [total,HV,K]; beta_logits
    [total,HV]; a_log [HV]; dt_bias [HV,K] (fp32)."""
    r = _rng(seed, _TOKENS, stream)
    d = {
        "q": r.standard_normal((total, Hk, K), dtype=np.float32),
        "k": r.standard_normal((total, Hk, K), dtype=np.float32),
        "v": r.standard_normal((total, HV, V), dtype=np.float32),
        "raw_gate": r.standard_normal((total, HV, K), dtype=np.float32),
        "beta_logits": r.standard_normal((total, HV), dtype=np.float32),
    }
    d = {n: as_dtype_values(x, in_dtype) for n, x in d.items()}
    p = _rng(seed, _PARAMS)
    d["a_log"] = p.uniform(0.0, 2.8, size=HV).astype(np.float32)
    d["dt_bias"] = p.uniform(-1.0, 1.0, size=(HV, K)).astype(np.float32)
    return d


# ----------------------------------------------------------------------------
# indices
# ----------------------------------------------------------------------------

def slot_permutation(seed, num_slots) -> np.ndarray:
    return _rng(seed, _INDEX).permutation(num_slots).astype(np.int64)


def slot_indices(seed, B, num_slots, rotation=0) -> np.ndarray:
    """The ``rotation``-th disjoint block of B slots of one random permutation."""
    perm = slot_permutation(seed, num_slots)
    if (rotation + 1) * B > num_slots:
        raise ValueError("not enough slots for this rotation")
    return perm[rotation * B:(rotation + 1) * B].copy()


def varlen_offsets(seed, B, max_len, min_len=1) -> np.ndarray:
    """cu_seqlens [B+1] (int32) of lengths U[min_len, max_len]."""
    lens = _rng(seed, _LENGTHS).integers(min_len, max_len + 1, size=B)
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


@dataclasses.dataclass
class PageTable:
    page_indices: np.ndarray     # [nnz] int64
    page_indptr: np.ndarray      # [B+1] int64
    last_page_len: np.ndarray    # [B] int64
    seq_lens: np.ndarray         # [B] tokens including the decoded one
    num_pages: int
    shared_pages: np.ndarray     # physical ids of the shared prefix pages

    def cast(self, index_dtype: str) -> "PageTable":
        dt = {"i32": np.int32, "i64": np.int64}[index_dtype]
        return dataclasses.replace(self, page_indices=self.page_indices.astype(dt),
                                   page_indptr=self.page_indptr.astype(dt),
                                   last_page_len=self.last_page_len.astype(dt))


def paged_table(seed, B, page_size, max_len, n_share, share_pages, force_lens=None,
                spare_pages=0, min_len=2) -> PageTable:
    """CSR page table of B sequences with lengths U[min_len, max_len].

    Sequences 0..n_share-1 share their first ``share_pages`` full pages and
    have lengths above the shared prefix (resampled), so that their last
    page is their own. ``force_lens`` maps sequence -> length (e.g. exactly
    one past the shared prefix, so that the decoded token opens a new page
    and the state is read from the last shared page). Physical page ids are
    a random permutation over all distinct pages (plus ``spare_pages``).
    """
    r = _rng(seed, _LENGTHS)
    prefix = share_pages * page_size
    lens = r.integers(min_len, max_len + 1, size=B)
    for bb in range(min(n_share, B)):
        while lens[bb] <= prefix:
            lens[bb] = r.integers(min_len, max_len + 1)
    for bb, L in (force_lens or {}).items():
        lens[bb] = L
    npages = -(-lens // page_size)
    own = np.array([npages[bb] - (share_pages if bb < n_share else 0) for bb in range(B)])
    n_distinct = (share_pages if n_share else 0) + int(own.sum())
    num_pages = n_distinct + spare_pages
    perm = _rng(seed, _PAGES).permutation(num_pages)
    shared = perm[:share_pages] if n_share else perm[:0]
    cursor = len(shared)
    rows, indptr = [], [0]
    for bb in range(B):
        mine = perm[cursor:cursor + own[bb]]
        cursor += own[bb]
        row = np.concatenate([shared, mine]) if bb < n_share else mine
        rows.append(row)
        indptr.append(indptr[-1] + len(row))
    last = lens - page_size * (npages - 1)
    return PageTable(np.concatenate(rows).astype(np.int64), np.array(indptr, np.int64),
                     last.astype(np.int64), lens.astype(np.int64), int(num_pages),
                     shared.astype(np.int64))


# ----------------------------------------------------------------------------
# initial states
# ----------------------------------------------------------------------------

def state_shape(K, V, layout):
    return (K, V) if layout == "K_FIRST" else (V, K)


def slot_state(seed, slot, HV, K, V, layout, state_dtype, block_v=64):
    """Initial stored content of one slot (or page): ([HV, *layout 2-D*], scales or None).

    f32: N(0, 0.1) values. bf16: the same rounded by torch (bits as uint16).
    fp8_e4m3: codes from torch's float8_e4m3fn cast of N(0, 1) * 100 clipped
    to +-440, with one scale ~ 1e-3 * U(0.75, 1.25) per [K, block_v] tile, so
    that decoded values are near N(0, 0.1).
    int8_hadamard32: codes N(0, 1) * 42 rounded and clipped to +-127, with
    one scale ~ (0.1 / 42) * U(0.75, 1.25) per (32-value group, key channel),
    scales [HV, V / 32, K]; decoded values are again near N(0, 0.1).
    The logical [K, V] content is drawn first and then laid out, so a K_FIRST
    and a V_FIRST pool built from one seed hold the same logical states.
    """
    r = _rng(seed, _STATE, slot)
    if state_dtype in ("f32", "bf16"):
        logical = (r.standard_normal((HV, K, V), dtype=np.float32) * np.float32(0.1))
    elif state_dtype == "fp8_e4m3":
        logical = np.clip(r.standard_normal((HV, K, V), dtype=np.float32) * np.float32(100.0),
                          -440.0, 440.0)
    elif state_dtype == "int8_hadamard32":
        logical = np.clip(np.rint(r.standard_normal((HV, K, V), dtype=np.float32) * np.float32(42.0)),
                          -127, 127).astype(np.int8)
    else:
        raise ValueError(state_dtype)
    stored = logical if layout == "K_FIRST" else np.ascontiguousarray(logical.transpose(0, 2, 1))
    if state_dtype == "f32":
        return np.ascontiguousarray(stored), None
    if state_dtype == "bf16":
        bits = torch.from_numpy(np.ascontiguousarray(stored)).to(torch.bfloat16).view(torch.int16)
        return bits.numpy().view(np.uint16), None
    if state_dtype == "int8_hadamard32":
        scales = (np.float32(0.1 / 42.0) * r.uniform(0.75, 1.25, size=(HV, V // 32, K))).astype(np.float32)
        return np.ascontiguousarray(stored), scales
    codes = torch.from_numpy(np.ascontiguousarray(stored)).to(torch.float8_e4m3fn).view(torch.uint8)
    scales = (np.float32(1e-3) * r.uniform(0.75, 1.25, size=(HV, V // block_v))).astype(np.float32)
    return codes.numpy(), scales


def host_pool(seed, slots: Sequence[int], HV, K, V, layout, state_dtype, block_v=64):
    """Dict-backed pool of the listed slots: returns (states, scales) where
    states[slot, hv] and scales[slot, hv] index like the device pool."""
    states, scales = {}, {}
    for s in slots:
        st, sc = slot_state(seed, int(s), HV, K, V, layout, state_dtype, block_v)
        for hv in range(HV):
            states[int(s), hv] = st[hv]
            if sc is not None:
                scales[int(s), hv] = sc[hv]
    return states, (scales if scales else None)


def torch_state_dtype(state_dtype):
    return {"f32": torch.float32, "bf16": torch.bfloat16, "fp8_e4m3": torch.uint8,
            "int8_hadamard32": torch.int8}[state_dtype]


def device_pool(seed, num_slots, HV, K, V, layout, state_dtype, block_v=64,
                exact_slots: Optional[Sequence[int]] = None, device="cuda"):
    """Allocate and fill a device pool [num_slots, HV, *layout*] (+ fp8 or int8 scales).

    Slots in ``exact_slots`` get the per-slot seeded host content of
    ``slot_state`` (what the oracle regenerates); every other slot gets the
    same distribution from a seeded torch generator on the device.
    """
    shape = (num_slots, HV) + state_shape(K, V, layout)
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + 17)
    scales = None
    if state_dtype == "fp8_e4m3":
        pool = torch.empty(shape, dtype=torch.uint8, device=device)
        scales = torch.empty((num_slots, HV, V // block_v), dtype=torch.float32, device=device)
        chunk = max(1, (1 << 28) // (HV * K * V))
        for s0 in range(0, num_slots, chunk):
            s1 = min(num_slots, s0 + chunk)
            x = torch.randn((s1 - s0,) + shape[1:], generator=g, device=device) * 100.0
            pool[s0:s1] = x.clamp_(-440.0, 440.0).to(torch.float8_e4m3fn).view(torch.uint8)
        scales.uniform_(0.75e-3, 1.25e-3, generator=g)
    elif state_dtype == "int8_hadamard32":
        pool = torch.empty(shape, dtype=torch.int8, device=device)
        scales = torch.empty((num_slots, HV, V // 32, K), dtype=torch.float32, device=device)
        chunk = max(1, (1 << 28) // (HV * K * V))
        for s0 in range(0, num_slots, chunk):
            s1 = min(num_slots, s0 + chunk)
            x = torch.randn((s1 - s0,) + shape[1:], generator=g, device=device) * 42.0
            pool[s0:s1] = x.round_().clamp_(-127.0, 127.0).to(torch.int8)
        scales.uniform_(0.75 * 0.1 / 42.0, 1.25 * 0.1 / 42.0, generator=g)
    else:
        pool = torch.empty(shape, dtype=torch_state_dtype(state_dtype), device=device)
        chunk = max(1, (1 << 28) // (HV * K * V))
        for s0 in range(0, num_slots, chunk):
            s1 = min(num_slots, s0 + chunk)
            pool[s0:s1].normal_(0.0, 0.1, generator=g)
    for s in (exact_slots or []):
        st, sc = slot_state(seed, int(s), HV, K, V, layout, state_dtype, block_v)
        if state_dtype == "bf16":
            pool[int(s)].copy_(torch.from_numpy(st.view(np.int16)).view(torch.bfloat16))
        else:
            pool[int(s)].copy_(torch.from_numpy(st))
        if sc is not None:
            scales[int(s)].copy_(torch.from_numpy(sc))
    return pool, scales
