"""Benchmark of gated delta-rule decode on B200.

Default workload: slot-pool GDN decode, T=1, B=64 sequences, H=16 key heads,
HV=32 value heads, K=V=128, bf16 q/k/v/a/b, fp32 state pool
[256, 32, 128, 128] (V_FIRST), bf16 output. One step = one decode call over
the batch: every sequence's state is read, advanced one token and written
back in place. Steps rotate over 4 disjoint sets of 64 slots (512 MiB of
state per cycle, 4x the L2), so no step finds its state in L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload slots|paged|kda|kda_long|fp8|int8|tiny|prefill]

Prints one JSON line (rank 0). Under torchrun each rank runs its own batch
on its own GPU (weak scaling; the sequences are independent, no data-path
collective); timing is the max over ranks.
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "decode tokens/s and achieved HBM GB/s (% of ~8 TB/s) at 1×B200, by config"
L2_BYTES = 126 * 2 ** 20
MIN_REPS, MAX_REPS = 5, 20000
E2E_STEPS = 64
PROFILES = os.path.join(ROOT, "profiles")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", choices=["slots", "paged", "kda", "kda_long", "fp8", "int8", "tiny", "prefill"],
                    default="slots")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--seconds", type=float, default=1.0,
                    help="device time each timed configuration covers (repetitions of --steps steps)")
    ap.add_argument("--headline-only", action="store_true", help="skip the by_config entries")
    ap.add_argument("--batch", type=int, default=0,
                    help="sequences of the headline workload (default: the workload's own); a smaller batch keeps "
                         "a profiler capture of the paged pool to a few GB")
    ap.add_argument("--warm-seconds", type=float, default=0.3, help="clock warm-up before each timed configuration")
    return ap.parse_args()


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------

def dist_setup(gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time (NCCL ranks reduce on their GPU, gloo on the host)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(local_ms: float, tokens_per_step: int, steps: int, world: int):
    """Whole-job throughput of a weak-scaling run: every rank processed
    tokens_per_step * steps tokens; the job took the slowest rank's time."""
    total_ms = max_over_ranks(local_ms, world)
    return total_ms, world * tokens_per_step * steps / (total_ms / 1e3)


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML)
# ----------------------------------------------------------------------------

class ClockSampler:
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._on = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            try:   # match the CUDA device to its NVML handle by UUID
                uuid = "GPU-" + str(torch.cuda.get_device_properties(index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            if self._on.is_set():
                try:
                    self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                    r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    for name, bit in self.REASONS.items():
                        if r & bit:
                            self.reasons.add(name)
                except Exception:
                    pass
            time.sleep(0.005)

    def __enter__(self):
        if self.nv is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def timing(self, on: bool):
        (self._on.set if on else self._on.clear)()

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self.t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(self.reasons)}


# ----------------------------------------------------------------------------
# workloads on the device
# ----------------------------------------------------------------------------

def in_t(x, dt):
    return torch.from_numpy(np.ascontiguousarray(x)).to(W.torch_dtype(dt)).cuda()


def describe_slots(w: W.Workload) -> str:
    return (f"slot-pool GDN decode T={w.T}: B={w.B}, H={w.H}, HV={w.HV}, K=V={w.K}, {w.in_dtype} q/k/v/a/b, "
            f"{w.state_dtype} state_pool [{w.num_slots},{w.HV},{w.V},{w.K}] {w.layout}, bf16 output")


class SlotsRun:
    """GDN slot pool, T=1 (the 'slots', 'fp8', 'int8' and 'tiny' workloads)."""

    def __init__(self, w: W.Workload, rank: int):
        import gated_delta_rule_80_b200 as G
        self.G, self.w = G, w
        seed = w.seed + 1000 * rank
        self.seed = seed
        t = W.gdn_tokens(seed, w.B, w.T, w.H, w.HV, w.K, w.V, w.in_dtype)
        self.host_tokens = t
        self.q, self.k, self.v = in_t(t["q"], w.in_dtype), in_t(t["k"], w.in_dtype), in_t(t["v"], w.in_dtype)
        self.a, self.b = in_t(t["a"], w.in_dtype), in_t(t["b"], w.in_dtype)
        self.A_log, self.dt_bias = in_t(t["A_log"], "f32"), in_t(t["dt_bias"], "f32")
        self.pool, self.scales = W.device_pool(seed, w.num_slots, w.HV, w.K, w.V, w.layout, w.state_dtype,
                                               w.block_v)
        self.n_rot = w.num_slots // w.B
        self.idx = [torch.from_numpy(W.slot_indices(seed, w.B, w.num_slots, r).astype(np.int32)).cuda()
                    for r in range(self.n_rot)]
        self.out = torch.empty((w.B, w.T, w.HV, w.V), dtype=torch.bfloat16, device="cuda")
        sb = {"f32": 4, "bf16": 2, "fp8_e4m3": 1, "int8_hadamard32": 1}[w.state_dtype]
        # codes plus scales, each read and written once
        sc_per_head = {"fp8_e4m3": (w.V // w.block_v) * 4, "int8_hadamard32": (w.V // 32) * w.K * 4}
        state = 2 * w.HV * (w.K * w.V * sb + sc_per_head.get(w.state_dtype, 0))
        ib = 2 if w.in_dtype == "bf16" else 4
        io = (2 * w.H * w.K + w.HV * w.V + 2 * w.HV) * ib + w.HV * w.V * 2 + 4
        self.tokens_per_step = w.B * w.T
        # the state is read and written once per call, token inputs/outputs once per token
        self.bytes_per_step = state * w.B + io * w.B * w.T + w.HV * 8   # + A_log, dt_bias
        self.bytes_per_token = self.bytes_per_step / self.tokens_per_step
        self.l2_note = (f"rotating {self.n_rot} disjoint slot sets "
                        f"({self.n_rot * w.B * 2 * w.HV * w.K * w.V * sb // 2 // 2**20} MiB of state per cycle)"
                        if self.n_rot > 1 else "state touched per step > L2 (every slot every step)")

    def step(self, i):
        self.G.gdn_decode_slots(self.q, self.k, self.v, self.a, self.b, self.A_log, self.dt_bias, self.pool,
                                self.idx[i % self.n_rot], state_scales=self.scales, state_layout=self.w.layout,
                                block_v=self.w.block_v, output=self.out)

    def e2e_setup(self):
        """Buffers of the end-to-end loop. A step's inputs (q, k, v, a, b and
        the slot indices) sit in one pinned host block, each at a 256-byte
        offset, so that one copy moves them. Two device input blocks and two
        output buffers alternate between steps, so that the copy of step
        i+1's inputs and the copy of step i-1's output run on their own
        streams while step i computes."""
        parts = [self.q, self.k, self.v, self.a, self.b, self.idx[0]]
        offs, n = [], 0
        for x in parts:
            offs.append(n)
            n += (x.numel() * x.element_size() + 255) // 256 * 256
        self.h_blk = [torch.empty(n, dtype=torch.uint8).pin_memory() for _ in range(self.n_rot)]
        for r, hb in enumerate(self.h_blk):
            for o, x in zip(offs, parts[:-1] + [self.idx[r]]):
                nb = x.numel() * x.element_size()
                hb[o:o + nb].copy_(x.contiguous().view(-1).view(torch.uint8).cpu())
        self.d_blk = [torch.empty(n, dtype=torch.uint8, device="cuda") for _ in range(2)]
        self.d_in = [[blk[o:o + x.numel() * x.element_size()].view(x.dtype).view(x.shape)
                      for o, x in zip(offs, parts)] for blk in self.d_blk]
        self.d_out = [torch.empty_like(self.out) for _ in range(2)]
        self.h_out = [torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory() for _ in range(2)]
        self.s_h2d, self.s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
        self.ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of buffer j on the device
        self.ev_done = [torch.cuda.Event() for _ in range(2)]   # the call that used buffer j finished
        self.ev_out = [torch.cuda.Event() for _ in range(2)]    # output j copied to the host
        self.h2d = sum(x.numel() * x.element_size() for x in parts)
        self.d2h = self.h_out[0].numel() * self.h_out[0].element_size()

    def e2e_step(self, i, comp, first=False):
        """Step i of the end-to-end loop: host-to-device copy of its inputs,
        the decode call through the public binding, device-to-host copy of
        its output; the copies wait only for what they overwrite (``first``:
        the buffer has not been used yet in this sequence of steps)."""
        j = i % 2
        with torch.cuda.stream(self.s_h2d):
            if not first:
                self.s_h2d.wait_event(self.ev_done[j])
            self.d_blk[j].copy_(self.h_blk[i % self.n_rot], non_blocking=True)
            self.ev_in[j].record(self.s_h2d)
        comp.wait_event(self.ev_in[j])
        if not first:
            comp.wait_event(self.ev_out[j])
        q, k, v, a, b, idx = self.d_in[j]
        with torch.cuda.stream(comp):
            self.G.gdn_decode_slots(q, k, v, a, b, self.A_log, self.dt_bias, self.pool, idx,
                                    state_scales=self.scales, state_layout=self.w.layout, block_v=self.w.block_v,
                                    output=self.d_out[j])
            self.ev_done[j].record(comp)
        with torch.cuda.stream(self.s_d2h):
            self.s_d2h.wait_event(self.ev_done[j])
            self.h_out[j].copy_(self.d_out[j], non_blocking=True)
            self.ev_out[j].record(self.s_d2h)

    def e2e_drain(self, comp):
        """Make ``comp`` wait for every copy in flight."""
        comp.wait_stream(self.s_h2d)
        comp.wait_stream(self.s_d2h)

    def e2e_graph(self, n):
        """n end-to-end steps captured into one CUDA graph: the copies from
        and to pinned host memory and the decode calls made through the
        public binding, with the dependencies between the three streams."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            comp = torch.cuda.current_stream()
            self.s_h2d.wait_stream(comp)
            self.s_d2h.wait_stream(comp)
            for i in range(n):
                self.e2e_step(i, comp, first=i < 2)
            self.e2e_drain(comp)
        return g

    def describe(self):
        return describe_slots(self.w)

    def cpu_baseline(self, seconds):
        """The oracle on rank 0's first sequences, as many as fit the time budget."""
        from threadpoolctl import threadpool_limits
        from oracle import gdn as O
        w, t = self.w, self.host_tokens
        nb = min(w.B, 8)
        idx = W.slot_indices(self.seed, w.B, w.num_slots, 0)[:nb]
        states, scales = W.host_pool(self.seed, idx.tolist(), w.HV, w.K, w.V, w.layout, w.state_dtype, w.block_v)
        sl = lambda x: x[:nb]
        done, t0 = 0, time.perf_counter()
        with threadpool_limits(limits=1):
            while True:
                O.gdn_decode_slots(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["a"]), sl(t["b"]), t["A_log"],
                                   t["dt_bias"], states, idx, layout=w.layout, state_dtype=w.state_dtype,
                                   state_scales=scales, block_v=w.block_v)
                done += nb * w.T
                el = time.perf_counter() - t0
                if el >= seconds:
                    break
        return done / el, f"oracle gdn_decode_slots on {nb} of {w.B} sequences x {w.HV} heads, repeated " \
                          f"{done // (nb * w.T)} times in {el:.1f} s"

    def cpu_baseline_all_cores(self, seconds):
        """The oracle on every host core: worker i takes sequences i, i+n, ...
        of the call (n workers, at most one per sequence)."""
        w, t = self.w, self.host_tokens
        n = host_cores(w.B)
        idx = W.slot_indices(self.seed, w.B, w.num_slots, 0)
        jobs = []
        for i in range(n):
            rows = np.arange(i, w.B, n)
            states, scales = W.host_pool(self.seed, idx[rows].tolist(), w.HV, w.K, w.V, w.layout, w.state_dtype,
                                         w.block_v)
            args = tuple(t[name][rows] for name in ("q", "k", "v", "a", "b")) + \
                (t["A_log"], t["dt_bias"], states, idx[rows])
            kw = dict(layout=w.layout, state_dtype=w.state_dtype, state_scales=scales, block_v=w.block_v)
            jobs.append({"fn": "gdn_decode_slots", "args": args, "kw": kw, "tokens_per_call": len(rows) * w.T})
        v = oracle_all_cores(jobs, seconds)
        if v is None:
            return None
        return {"value": v, "unit": "tokens/s", "cores": n, "kind": "oracle",
                "sample": f"oracle gdn_decode_slots, all {w.B} sequences x {w.HV} heads split over {n} "
                          f"single-threaded processes, {seconds:.0f} s window"}


class PagedRun:
    """GDN paged pool, one token (the 'paged' workload). Steps rotate over 4
    page tables that differ in the pages a call reads and writes, so no step
    finds its pages in L2."""

    def __init__(self, w: W.Workload, rank: int):
        import gated_delta_rule_80_b200 as G
        self.G, self.w = G, w
        seed = w.seed + 1000 * rank
        self.seed = seed
        self.n_rot = 4
        base = W.paged_table(seed, w.B, w.page_size, w.max_len, w.n_share, w.share_pages)
        self.pt = base
        # rotation r > 0: the same table with every page a call reads or
        # writes (the last page, and the one before it for a new page)
        # remapped to fresh page ids; untouched pages are shared
        touched = []
        for bb in range(w.B):
            last = int(base.page_indptr[bb + 1]) - 1
            touched.append(last)
            if int(base.last_page_len[bb]) == 1:
                touched.append(last - 1)
        next_id = base.num_pages
        tables = [base.page_indices]
        for r in range(1, self.n_rot):
            ind = base.page_indices.copy()
            for pos in touched:
                ind[pos] = next_id
                next_id += 1
            tables.append(ind)
        self.num_pages = next_id
        t = W.gdn_tokens(seed, w.B, 1, w.H, w.HV, w.K, w.V, w.in_dtype)
        self.host_tokens = t
        self.q, self.k, self.v = in_t(t["q"], w.in_dtype), in_t(t["k"], w.in_dtype), in_t(t["v"], w.in_dtype)
        self.a, self.b = in_t(t["a"], w.in_dtype), in_t(t["b"], w.in_dtype)
        self.A_log, self.dt_bias = in_t(t["A_log"], "f32"), in_t(t["dt_bias"], "f32")
        self.pool, self.scales = W.device_pool(seed, self.num_pages, w.HV, w.K, w.V, w.layout, w.state_dtype)
        pp = torch.from_numpy(base.page_indptr.astype(np.int32)).cuda()
        pl = torch.from_numpy(base.last_page_len.astype(np.int32)).cuda()
        self.tables = [(torch.from_numpy(ind.astype(np.int32)).cuda(), pp, pl) for ind in tables]
        self.out = torch.empty((w.B, 1, w.HV, w.V), dtype=torch.bfloat16, device="cuda")
        ib = 2
        self.bytes_per_token = 2 * w.HV * w.K * w.V * 4 + (2 * w.H * w.K + w.HV * w.V + 2 * w.HV) * ib \
            + w.HV * w.V * 2 + 12
        self.tokens_per_step = w.B
        self.bytes_per_step = self.bytes_per_token * w.B + w.HV * 8
        self.l2_note = (f"rotating {self.n_rot} page tables whose read/write pages are disjoint "
                        f"({self.n_rot * w.B * 2} MiB of state read per cycle, 4x L2)")

    def step(self, i):
        pi, pp, pl = self.tables[i % self.n_rot]
        self.G.gdn_decode_paged(self.q, self.k, self.v, self.A_log, self.a, self.dt_bias, self.b,
                                state_pool=self.pool, page_indices=pi, page_indptr=pp,
                                last_page_len=pl, page_size=self.w.page_size, output=self.out)

    def describe(self):
        w = self.w
        return (f"paged GDN decode T=1: B={w.B}, page_size={w.page_size}, lengths U[2,{w.max_len}], "
                f"{w.n_share} sequences sharing {w.share_pages} full pages, HV={w.HV}, H={w.H}, K=V={w.K}, "
                f"fp32 state_pool [{self.pt.num_pages},{w.HV},{w.V},{w.K}] (+ remapped pages for the rotation), "
                f"int32 CSR, bf16 in/out")


class KdaRun:
    """KDA varlen (the 'kda' workload), 8 pool replicas rotated."""

    def __init__(self, w: W.Workload, rank: int, layout=None):
        import gated_delta_rule_80_b200 as G
        self.G, self.w = G, w
        seed = w.seed + 1000 * rank
        self.layout = layout or w.layout
        self.cu = W.varlen_offsets(seed, w.B, w.max_len, w.min_len)
        total = int(self.cu[-1])
        t = W.kda_tokens(seed, total, w.H, w.HV, w.K, w.V, w.in_dtype)
        self.ins = [in_t(t[n], w.in_dtype) for n in ("q", "k", "v", "raw_gate", "beta_logits")]
        self.a_log, self.dt_bias = in_t(t["a_log"], "f32"), in_t(t["dt_bias"], "f32")
        self.cu_d = torch.from_numpy(self.cu).cuda()
        self.idx = torch.from_numpy(W.slot_indices(seed, w.B, w.num_slots).astype(np.int32)).cuda()
        self.n_rep = 8
        self.pools = [W.device_pool(seed + r, w.num_slots, w.HV, w.K, w.V, self.layout, "f32")[0]
                      for r in range(self.n_rep)]
        self.out = torch.empty((total, w.HV, w.V), dtype=torch.bfloat16, device="cuda")
        self.tokens_per_step = total
        self.bytes_per_step = w.B * 2 * w.HV * w.K * w.V * 4 + total * (
            (2 * w.H * w.K + w.HV * w.V + w.HV * w.K + w.HV) * 2 + w.HV * w.V * 2) + w.HV * (w.K + 1) * 4
        self.bytes_per_token = self.bytes_per_step / total
        self.l2_note = f"rotating {self.n_rep} pool replicas ({self.n_rep * w.num_slots * 2} MiB of state)"

    def step(self, i):
        q, k, v, g, bl = self.ins
        self.G.kda_decode_varlen(q, k, v, g, bl, self.a_log, self.dt_bias, self.cu_d, self.pools[i % self.n_rep],
                                 self.idx, state_layout=self.layout, output=self.out)

    def describe(self):
        w = self.w
        return (f"KDA varlen decode: {w.B} sequences x U[{w.min_len},{w.max_len}] tokens ({self.tokens_per_step} tokens), "
                f"Hk=HV={w.HV}, K=V={w.K}, bf16 inputs, fp32 state_pool [{w.num_slots},{w.HV},{w.K},{w.V}] "
                f"{self.layout}")


class PrefillRun:
    """Paged prefill (the 'prefill' workload): 8 fresh sequences of 1024
    tokens, page_size 64, HV=32, H=16, K=V=128, bf16 in/out, fp32 pages.
    Steps rotate over 4 page sets."""

    def __init__(self, w: W.Workload, rank: int):
        import gated_delta_rule_80_b200 as G
        self.G = G
        seed = 5 + 1000 * rank
        self.B, self.L, self.ps, self.H, self.HV, self.K, self.V = 8, 1024, 64, 16, 32, 128, 128
        npg = self.L // self.ps
        self.n_rot = 4
        total = self.B * self.L
        t = W.varlen_gdn_tokens(seed, total, self.H, self.HV, self.K, self.V, "bf16")
        self.ins = [in_t(t[n], "bf16") for n in ("q", "k", "v", "a", "b")]
        self.A_log, self.dt_bias = in_t(t["A_log"], "f32"), in_t(t["dt_bias"], "f32")
        self.cu = torch.from_numpy(np.arange(self.B + 1, dtype=np.int32) * self.L).cuda()
        self.num_pages = self.n_rot * self.B * npg
        self.pool, _ = W.device_pool(seed, self.num_pages, self.HV, self.K, self.V, "V_FIRST", "f32")
        perm = np.random.default_rng(seed).permutation(self.num_pages).astype(np.int32)
        self.tables = []
        for r in range(self.n_rot):
            ind = perm[r * self.B * npg:(r + 1) * self.B * npg]
            self.tables.append((torch.from_numpy(ind.copy()).cuda(),
                                torch.from_numpy(np.arange(self.B + 1, dtype=np.int32) * npg).cuda(),
                                torch.full((self.B,), self.ps, dtype=torch.int32, device="cuda")))
        self.out = torch.empty((total, self.HV, self.V), dtype=torch.bfloat16, device="cuda")
        self.tokens_per_step = total
        tok_bytes = (2 * self.H * self.K + 2 * self.HV * self.V + 2 * self.HV) * 2
        self.bytes_per_step = total * tok_bytes + self.B * npg * self.HV * self.K * self.V * 4 + self.HV * 8
        self.l2_note = f"rotating {self.n_rot} disjoint page sets ({self.B * npg * 2 * self.n_rot} MiB written per cycle)"

    def step(self, i):
        pi, pp, pl = self.tables[i % self.n_rot]
        q, k, v, a, b = self.ins
        self.G.gdn_prefill_paged(q, k, v, a, b, self.A_log, self.dt_bias, self.cu, state_pool=self.pool,
                                 page_indices=pi, page_indptr=pp, last_page_len=pl, page_size=self.ps,
                                 output=self.out)

    def describe(self):
        return (f"paged GDN prefill: {self.B} fresh sequences x {self.L} tokens, page_size={self.ps}, "
                f"H={self.H}, HV={self.HV}, K=V={self.K}, bf16 in/out, fp32 pages (one snapshot per page)")


def make_run(name, rank, layout=None, batch=0):
    w = W.WORKLOADS.get(name)
    if batch and w is not None:
        w = dataclasses.replace(w, B=batch)
    if name in ("slots", "fp8", "int8", "tiny"):
        return SlotsRun(w, rank)
    if name == "paged":
        return PagedRun(w, rank)
    if name == "prefill":
        return PrefillRun(None, rank)
    return KdaRun(w, rank, layout)


# ----------------------------------------------------------------------------
# the oracle on all host cores
# ----------------------------------------------------------------------------

def host_cores(cap):
    """Cores this process may run on: its CPU affinity, bounded by a cgroup
    CPU quota when one is set, and by ``cap``."""
    n = len(os.sched_getaffinity(0))
    try:
        quota, period = open("/sys/fs/cgroup/cpu.max").read().split()[:2]
        if quota != "max":
            n = min(n, max(1, int(int(quota) // int(period))))
    except (OSError, ValueError):
        pass
    return max(1, min(n, cap))


def oracle_all_cores(jobs, seconds):
    """Runs one oracle worker per job (``oracle.timing``), each its own
    single-threaded interpreter, over one common wall-clock window; returns
    the summed tokens per second, or None when a worker failed."""
    import pickle
    import shutil
    import tempfile
    env = dict(os.environ, OMP_NUM_THREADS="1", OPENBLAS_NUM_THREADS="1", MKL_NUM_THREADS="1")
    tmp = tempfile.mkdtemp(prefix="gdn_oracle_")
    procs = []
    try:
        for i, job in enumerate(jobs):
            path = os.path.join(tmp, f"job{i}.pkl")
            with open(path, "wb") as f:
                pickle.dump(job, f)
            procs.append(subprocess.Popen([sys.executable, "-m", "oracle.timing", path], cwd=ROOT, env=env,
                                          stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True))
        for pr in procs:
            if pr.stdout.readline().strip() != "ready":
                return None
        start = time.time() + 0.5
        window = json.dumps({"start": start, "end": start + seconds}) + "\n"
        for pr in procs:
            pr.stdin.write(window)
            pr.stdin.flush()
        done, finished = 0, start
        for pr in procs:
            out, _ = pr.communicate(timeout=seconds + 120)
            if pr.returncode != 0:
                return None
            r = json.loads(out.strip().splitlines()[-1])
            done += int(r["done"])
            finished = max(finished, float(r["finished"]))
        return done / (finished - start)
    finally:
        for pr in procs:
            if pr.poll() is None:
                pr.kill()
                pr.wait()
        shutil.rmtree(tmp, ignore_errors=True)


# ----------------------------------------------------------------------------
# roofline bookkeeping
# ----------------------------------------------------------------------------

def source_digest(files=None):
    """First 16 hex of the sha256 over the named kernel sources (all of csrc
    when none are named), in sorted order; None when one of them is gone."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_80_b200", "csrc")
    names = sorted(files) if files else sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    for f in names:
        path = os.path.join(csrc, f)
        if not os.path.exists(path):
            return None
        h.update(open(path, "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """(DRAM bytes per launch, source) from the committed ncu summary of this
    workload: a number taken by an earlier ncu capture, not in this run, and
    (None, None) when the kernel sources it names changed since."""
    rel = f"profiles/gdn_decode_{workload}_ncu.md"
    path = os.path.join(ROOT, rel)
    if not os.path.exists(path):
        return None, None
    text = open(path).read()
    dig = re.search(r"source_digest:\s*([0-9a-f]+)", text)
    tb = re.search(r"dram_bytes_per_launch:\s*([0-9.e+]+)", text)
    fl = re.search(r"source_files:\s*([^\n]+)", text)
    files = fl.group(1).split() if fl else None
    if not dig or not tb or dig.group(1) != source_digest(files):
        return None, None
    return float(tb.group(1)), rel + " (committed ncu capture; kernel sources unchanged since, by digest)"


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return float(json.load(open(path))["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------

def capture(run, n):
    """A CUDA graph of n consecutive steps (launches back to back on the device)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run.step(0)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for j in range(n):
            run.step(j)
    return g


def time_steps(run, K, warmup, world, local, min_seconds, warm_seconds=0.3):
    """Times exactly K steps per repetition, repeated until min_seconds of
    device time are covered (at least MIN_REPS repetitions), with NVML
    sampling the clocks over the whole window. Returns the median
    repetition's milliseconds (max over ranks), all repetitions, and the
    clock summary."""
    t_end = time.perf_counter() + warm_seconds  # clocks up, kernels loaded
    i = 0
    while time.perf_counter() < t_end:
        for _ in range(20):
            run.step(i)
            i += 1
        torch.cuda.synchronize()
    g_warm = capture(run, max(1, warmup))
    g_timed = capture(run, K)
    stream = torch.cuda.current_stream()
    g_warm.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g_timed.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    est = max(e0.elapsed_time(e1), 1e-3)
    reps = int(min(MAX_REPS, max(MIN_REPS, math.ceil(min_seconds * 1e3 / est))))
    reps = int(max_over_ranks(reps, world))   # every rank replays the same number of times
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        clk.timing(True)
        for a, b in evs:
            a.record(stream)
            g_timed.replay()
            b.record(stream)
        torch.cuda.synchronize()
        clk.timing(False)
        barrier(world)
    ms = [a.elapsed_time(b) for a, b in evs]
    med = max_over_ranks(statistics.median(ms), world)
    del g_warm, g_timed
    return {"median_ms": med, "reps": reps, "ms": ms, "clocks": clk.summary()}


def roofline_of(run, key, kern_ms, peak):
    achieved = run.bytes_per_step / (kern_ms / 1e3) / 1e9
    traffic, src = profiled_traffic(key)
    return {"achieved": achieved, "frac": achieved / peak, "frac_of_8TBps": achieved / 8000.0,
            "algorithmic_bytes_per_launch": run.bytes_per_step, "traffic": traffic, "traffic_source": src}


# the configurations reported beside the headline, each timed like it
BY_CONFIG = [("tiny", "tiny", {}), ("paged", "paged", {}), ("kda_k_first", "kda", {"layout": "K_FIRST"}),
             ("kda_v_first", "kda", {"layout": "V_FIRST"}), ("kda_long", "kda_long", {}), ("fp8", "fp8", {}),
             ("int8", "int8", {}), ("prefill", "prefill", {})]


def run_b200(args, world, rank, local):
    import gated_delta_rule_80_b200 as G
    G.lib()
    K = args.steps
    peak, peak_kind = measured_peak()
    run = make_run(args.workload, rank, batch=args.batch)
    desc, tps, l2 = run.describe(), run.tokens_per_step, run.l2_note
    tm = time_steps(run, K, args.warmup, world, local, args.seconds, args.warm_seconds)
    total_ms = tm["median_ms"]
    value = world * run.tokens_per_step * K / (total_ms / 1e3)
    ms_per_step = total_ms / K
    kern_avg_ms = ms_per_step     # one launch per step, back to back
    roof = roofline_of(run, args.workload, kern_avg_ms, peak)
    clocks = tm["clocks"]
    if clocks.get("sm_mhz"):
        clocks["kernel_us_x_sm_mhz"] = kern_avg_ms * 1e3 * clocks["sm_mhz"]

    e2e = None
    if not args.no_e2e and hasattr(run, "e2e_setup"):
        run.e2e_setup()
        # E2E_STEPS steps per graph (a multiple of the 2 buffers and the
        # rotation of host blocks); the graph is replayed back to back
        g = run.e2e_graph(E2E_STEPS)
        stream = torch.cuda.current_stream()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        est = max(e0.elapsed_time(e1), 1e-3)
        reps = int(max_over_ranks(max(2, math.ceil(args.seconds * 1e3 / est)), world))
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        Ke = reps * E2E_STEPS
        e2e = {"value": world * run.tokens_per_step * Ke / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": run.h2d, "d2h_bytes_per_step": run.d2h, "steps": Ke,
               "us_per_step": e_ms * 1e3 / Ke,
               "pipeline": f"double-buffered: H2D of step i+1 and D2H of step i-1 on their own streams under "
                           f"step i's kernel, every copy inside the timed window; {E2E_STEPS} steps (copies and "
                           f"calls through the public binding) captured in one CUDA graph, replayed {reps} times"}
        del g
    del run
    torch.cuda.empty_cache()

    by_config = {}
    if not args.headline_only:
        for name, wl, kw in BY_CONFIG:
            r = make_run(wl, rank, **kw)
            t = time_steps(r, K, args.warmup, world, local, args.seconds, args.warm_seconds)
            us = t["median_ms"] * 1e3 / K
            entry = {"workload": r.describe(), "us_per_launch": us,
                     "tokens_per_s": world * r.tokens_per_step * K / (t["median_ms"] / 1e3),
                     "tokens_per_launch": r.tokens_per_step, "repetitions": t["reps"],
                     "launches_per_repetition": K, "l2": r.l2_note,
                     "sm_mhz": t["clocks"].get("sm_mhz"), "clock_reasons": t["clocks"].get("reasons")}
            # the committed kda capture is of the K_FIRST pool
            ro = roofline_of(r, "kda" if name == "kda_k_first" else name, us / 1e3, peak)
            entry.update({"achieved_GBps": ro["achieved"], "frac": ro["frac"],
                          "frac_of_8TBps": ro["frac_of_8TBps"],
                          "algorithmic_bytes_per_launch": ro["algorithmic_bytes_per_launch"],
                          "traffic": ro["traffic"], "traffic_source": ro["traffic_source"]})
            if getattr(r, "latency_bound", False):
                entry["bound_note"] = r.latency_bound
            by_config[name] = entry
            del r
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = make_run(args.workload, rank)
        if hasattr(base, "cpu_baseline"):
            v, sample = base.cpu_baseline(args.cpu_seconds)
            cpu = {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample}
        cpu_all = base.cpu_baseline_all_cores(args.cpu_seconds) if hasattr(base, "cpu_baseline_all_cores") else None
        del base
    else:
        cpu_all = None

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; no dataset on the pages)",
            "config": {"workload": desc, "tokens_per_step_per_gpu": tps,
                       "l2": l2, "parallelism": f"independent sequences per GPU x{world}",
                       "timing": f"median of {tm['reps']} repetitions of {K} graph-replayed steps "
                                 f"(>= {args.seconds:g} s of device time)"},
            "roofline": {"bound": "hbm", "achieved": roof["achieved"], "peak": peak, "unit": "GB/s",
                         "frac": roof["frac"], "traffic": roof["traffic"], "traffic_source": roof["traffic_source"],
                         "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": roof["algorithmic_bytes_per_launch"],
                         "kernel_avg_us": kern_avg_ms * 1e3, "frac_of_8TBps": roof["frac_of_8TBps"]},
            "clocks": clocks,
            "e2e": e2e,
            "gpu_launches": K * tm["reps"],
            "by_config": by_config,
            "cpu_baseline": cpu,
            "cpu_baseline_all_cores": cpu_all,
        }
        print(json.dumps(line), flush=True)


def run_reference(args, world, rank):
    """The oracle as the reference arm (rank 0 only), each step a bounded
    sample of the same workload."""
    if rank != 0:
        return
    from threadpoolctl import threadpool_limits
    from oracle import gdn as O
    w = W.WORKLOADS["slots"]
    nb = 4
    t = W.gdn_tokens(w.seed, w.B, w.T, w.H, w.HV, w.K, w.V, w.in_dtype)
    idx = W.slot_indices(w.seed, w.B, w.num_slots, 0)[:nb]
    states, _ = W.host_pool(w.seed, idx.tolist(), w.HV, w.K, w.V, w.layout, w.state_dtype)
    sl = lambda x: x[:nb]

    def step():
        O.gdn_decode_slots(sl(t["q"]), sl(t["k"]), sl(t["v"]), sl(t["a"]), sl(t["b"]), t["A_log"], t["dt_bias"],
                           states, idx, layout=w.layout, state_dtype=w.state_dtype)

    with threadpool_limits(limits=1):
        for _ in range(args.warmup):
            step()
        K = min(args.steps, 200)
        t0 = time.perf_counter()
        for _ in range(K):
            step()
        el = time.perf_counter() - t0
    value = nb * K / el
    sample = f"oracle gdn_decode_slots on {nb} of {w.B} sequences x {w.HV} heads per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": el / K * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe_slots(w)},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        run_b200(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
