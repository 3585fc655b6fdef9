"""Gated delta-rule recurrent decode for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/gdn.h`` (``libgdn_b200.so``,
built in-tree by ``gated_delta_rule_80_b200.build``). Each function here only
marshals torch CUDA tensors into that ABI: every step of the computation runs
in the library's kernels, on the caller's current CUDA stream. There is no
CPU path: the first call raises if the library has not been built.

Functions (same names as the C entry points):

* ``gdn_decode_slots``      GDN decode of T >= 1 tokens on a slot pool
* ``gdn_decode_paged``      GDN single-token decode on a paged pool
* ``gdn_prefill_paged``     append varlen token runs to paged sequences
* ``gdn_paged_decode_slots`` (read_page, write_page) rows for a page table
* ``kda_decode_varlen``     KDA (per-key-channel gate) varlen decode
* ``gdn_state_quantize_fp8`` / ``gdn_state_dequantize_fp8``  fp8 tile codec
* ``gdn_state_quantize_int8h32`` / ``gdn_state_dequantize_int8h32``
  int8_hadamard32 codec (an int8 pool with fp32 scales [slots, HV, V/32, K])
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn_b200.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA = 0, -1, -2, -3
GDN_F32, GDN_BF16, GDN_FP8_E4M3, GDN_INT8_H32 = 0, 1, 2, 3
GDN_I32, GDN_I64 = 0, 1
GDN_K_FIRST, GDN_V_FIRST = 0, 1
GDN_READOUT_WORKING, GDN_READOUT_STORED = 0, 1
KDA_GATE_ORIGINAL, KDA_GATE_SAFE = 0, 1
KDA_BETA_LOGITS, KDA_BETA_PROBABILITY = 0, 1
GDN_FLAG_SLOT_RANGE, GDN_FLAG_PAGE_RANGE, GDN_FLAG_PAGE_TABLE, GDN_FLAG_SEQLENS, GDN_FLAG_TIMEOUT = 1, 2, 4, 8, 16

_LAYOUTS = {"K_FIRST": GDN_K_FIRST, "V_FIRST": GDN_V_FIRST}
_READOUTS = {"working": GDN_READOUT_WORKING, "stored": GDN_READOUT_STORED}
_GATE_MODES = {"original": KDA_GATE_ORIGINAL, "safe": KDA_GATE_SAFE}
_BETA_MODES = {"logits": KDA_BETA_LOGITS, "probability": KDA_BETA_PROBABILITY}


class GDNError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {gdn_status_string(status)} (status {status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m gated_delta_rule_80_b200.build` "
            "(nvcc, sm_100a). There is no CPU fallback.")
    return ctypes.CDLL(LIB_PATH)


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64


class gdn_state_pool(ctypes.Structure):
    _fields_ = [("data", _vp), ("scales", _vp), ("num_slots", _i64), ("dtype", _i32),
                ("layout", _i32), ("block_v", _i32), ("reserved", _i32)]


class gdn_decode_slots_params(ctypes.Structure):
    _fields_ = [("struct_size", _i32), ("B", _i32), ("T", _i32), ("H", _i32), ("HV", _i32),
                ("K", _i32), ("V", _i32), ("in_dtype", _i32), ("out_dtype", _i32),
                ("index_dtype", _i32), ("readout", _i32), ("use_qk_l2norm", _i32),
                ("scale", ctypes.c_float), ("q", _vp), ("k", _vp), ("v", _vp), ("a", _vp),
                ("b", _vp), ("A_log", _vp), ("dt_bias", _vp), ("state_indices", _vp),
                ("out", _vp), ("err_flags", _vp), ("pool", gdn_state_pool)]


class gdn_decode_paged_params(ctypes.Structure):
    _fields_ = [("struct_size", _i32), ("B", _i32), ("T", _i32), ("H", _i32), ("HV", _i32), ("K", _i32),
                ("V", _i32), ("in_dtype", _i32), ("out_dtype", _i32), ("index_dtype", _i32),
                ("readout", _i32), ("use_qk_l2norm", _i32), ("page_size", _i32),
                ("scale", ctypes.c_float), ("nnz", _i64), ("q", _vp), ("k", _vp), ("v", _vp),
                ("a", _vp), ("b", _vp), ("A_log", _vp), ("dt_bias", _vp), ("page_indices", _vp),
                ("page_indptr", _vp), ("last_page_len", _vp), ("slots", _vp), ("out", _vp),
                ("err_flags", _vp), ("pool", gdn_state_pool)]


class gdn_prefill_paged_params(ctypes.Structure):
    _fields_ = [("struct_size", _i32), ("B", _i32), ("total_tokens", _i32), ("H", _i32), ("HV", _i32),
                ("K", _i32), ("V", _i32), ("in_dtype", _i32), ("out_dtype", _i32), ("index_dtype", _i32),
                ("readout", _i32), ("use_qk_l2norm", _i32), ("page_size", _i32), ("scale", ctypes.c_float),
                ("nnz", _i64), ("q", _vp), ("k", _vp), ("v", _vp), ("a", _vp), ("b", _vp), ("A_log", _vp),
                ("dt_bias", _vp), ("cu_seqlens", _vp), ("page_indices", _vp), ("page_indptr", _vp),
                ("last_page_len", _vp), ("out", _vp), ("err_flags", _vp), ("pool", gdn_state_pool)]


class kda_decode_varlen_params(ctypes.Structure):
    _fields_ = [("struct_size", _i32), ("B", _i32), ("total_tokens", _i32), ("Hk", _i32),
                ("HV", _i32), ("K", _i32), ("V", _i32), ("in_dtype", _i32), ("out_dtype", _i32),
                ("gate_mode", _i32), ("beta_mode", _i32), ("readout", _i32), ("q", _vp),
                ("k", _vp), ("v", _vp), ("raw_gate", _vp), ("beta_logits", _vp), ("a_log", _vp),
                ("dt_bias", _vp), ("cu_seqlens", _vp), ("state_indices", _vp), ("out", _vp),
                ("err_flags", _vp), ("pool", gdn_state_pool)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libgdn_b200.so (loaded on first use; raises if it was never built)."""
    global _lib
    if _lib is None:
        L = _load()
        L.gdn_decode_slots.argtypes = [ctypes.POINTER(gdn_decode_slots_params), _vp]
        L.gdn_decode_paged.argtypes = [ctypes.POINTER(gdn_decode_paged_params), _vp]
        L.kda_decode_varlen.argtypes = [ctypes.POINTER(kda_decode_varlen_params), _vp]
        L.gdn_prefill_paged.argtypes = [ctypes.POINTER(gdn_prefill_paged_params), _vp]
        L.gdn_paged_decode_slots.argtypes = [_vp, _vp, _vp, _i32, _i64, _i32, _i64, _i32, _vp, _vp, _vp]
        L.gdn_state_quantize_fp8.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32, _vp]
        L.gdn_state_dequantize_fp8.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _i32, _vp]
        L.gdn_state_quantize_int8h32.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp]
        L.gdn_state_dequantize_int8h32.argtypes = [_vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp]
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_status_string.restype = ctypes.c_char_p
        for f in ("gdn_decode_slots", "gdn_decode_paged", "kda_decode_varlen", "gdn_paged_decode_slots",
                  "gdn_state_quantize_fp8", "gdn_state_dequantize_fp8", "gdn_prefill_paged",
                  "gdn_state_quantize_int8h32", "gdn_state_dequantize_int8h32"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def gdn_status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("gdn tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("gdn tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _io_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    raise ValueError(f"unsupported input/output dtype {t.dtype}")


def _state_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return GDN_FP8_E4M3
    if t.dtype == torch.int8:
        return GDN_INT8_H32
    raise ValueError(f"unsupported state dtype {t.dtype}")


def _index_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.int32:
        return GDN_I32
    if t.dtype == torch.int64:
        return GDN_I64
    raise ValueError(f"index tensors must be int32 or int64, got {t.dtype}")


def _same_index_dtype(*ts) -> int:
    kinds = {_index_dtype(t) for t in ts if t is not None}
    if len(kinds) != 1:
        raise ValueError("page_indices, page_indptr and last_page_len must share one int dtype")
    return kinds.pop()


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _pool(state_pool, state_scales, layout, block_v, K, V, HV) -> gdn_state_pool:
    lay = _LAYOUTS[layout]
    want = (HV, K, V) if lay == GDN_K_FIRST else (HV, V, K)
    if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != want:
        raise ValueError(f"state_pool must be [slots, {want[0]}, {want[1]}, {want[2]}] for {layout}, "
                         f"got {tuple(state_pool.shape)}")
    sdt = _state_dtype(state_pool)
    if sdt == GDN_FP8_E4M3:
        if state_scales is None or state_scales.dtype != torch.float32:
            raise ValueError("an fp8 state pool needs fp32 state_scales [slots, HV, V/block_v]")
        if tuple(state_scales.shape) != (state_pool.shape[0], HV, V // block_v):
            raise ValueError("state_scales must be [slots, HV, V/block_v]")
    if sdt == GDN_INT8_H32:
        if state_scales is None or state_scales.dtype != torch.float32:
            raise ValueError("an int8_hadamard32 state pool needs fp32 state_scales [slots, HV, V/32, K]")
        if tuple(state_scales.shape) != (state_pool.shape[0], HV, V // 32, K):
            raise ValueError("state_scales must be [slots, HV, V/32, K]")
    coded = sdt in (GDN_FP8_E4M3, GDN_INT8_H32)
    return gdn_state_pool(_ptr(state_pool), _ptr(state_scales) if coded else None,
                          state_pool.shape[0], sdt, lay, block_v, 0)


def _expect(t, shape, name):
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _check(status: int, where: str):
    if status != GDN_OK:
        raise GDNError(status, where)


def _out(output, shape, dtype, like):
    if output is None:
        return torch.empty(shape, dtype=dtype, device=like.device)
    if tuple(output.shape) != tuple(shape):
        raise ValueError(f"output must have shape {tuple(shape)}")
    return output


# ----------------------------------------------------------------------------
# entry points
# ----------------------------------------------------------------------------

def gdn_decode_slots(q, k, v, a, b, A_log, dt_bias, state_pool, state_indices, *,
                     state_scales=None, state_layout="V_FIRST", block_v=64, scale=None,
                     use_qk_l2norm=True, output=None, output_dtype=None, readout="working",
                     err_flags=None):
    """GDN decode of B sequences x T tokens on a slot pool, updated in place.

    q, k [B, T, H, K]; v [B, T, HV, V]; a, b [B, T, HV]; A_log, dt_bias [HV]
    fp32; state_pool [slots, HV, K, V] (K_FIRST) or [slots, HV, V, K]
    (V_FIRST) in fp32, bf16 or fp8 (uint8 codes + state_scales); state_indices
    [B] int32/int64. Returns output [B, T, HV, V].
    """
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    _expect(k, (B, T, H, K), "k")
    _expect(v, (B, T, HV, V), "v")
    _expect(a, (B, T, HV), "a")
    _expect(b, (B, T, HV), "b")
    _expect(A_log, (HV,), "A_log")
    _expect(dt_bias, (HV,), "dt_bias")
    _expect(state_indices, (B,), "state_indices")
    if A_log.dtype != torch.float32 or dt_bias.dtype != torch.float32:
        raise ValueError("A_log and dt_bias must be float32")
    if len({x.dtype for x in (q, k, v, a, b)}) != 1:
        raise ValueError("q, k, v, a, b must share one dtype")
    out_dt = output_dtype or (output.dtype if output is not None else q.dtype)
    out = _out(output, (B, T, HV, V), out_dt, q)
    prm = gdn_decode_slots_params()
    prm.struct_size = ctypes.sizeof(gdn_decode_slots_params)
    prm.B, prm.T, prm.H, prm.HV, prm.K, prm.V = B, T, H, HV, K, V
    prm.in_dtype, prm.out_dtype = _io_dtype(q), _io_dtype(out)
    prm.index_dtype = _index_dtype(state_indices)
    prm.readout = _READOUTS[readout]
    prm.use_qk_l2norm = int(bool(use_qk_l2norm))
    prm.scale = 0.0 if scale is None else float(scale)
    prm.q, prm.k, prm.v, prm.a, prm.b = _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b)
    prm.A_log, prm.dt_bias = _ptr(A_log), _ptr(dt_bias)
    prm.state_indices, prm.out, prm.err_flags = _ptr(state_indices), _ptr(out), _ptr(err_flags)
    prm.pool = _pool(state_pool, state_scales, state_layout, block_v, K, V, HV)
    _check(lib().gdn_decode_slots(ctypes.byref(prm), _stream(q)), "gdn_decode_slots")
    return out


def gdn_decode_paged(q, k, v, A_log, a, dt_bias, b, scale=None, output=None, use_qk_l2norm=True, *,
                     state_pool, page_indices, page_indptr, last_page_len, slots=None,
                     state_scales=None, state_layout="V_FIRST", block_v=64, page_size=0,
                     output_dtype=None, readout="working", err_flags=None):
    """GDN decode of the last T tokens of every sequence on a paged pool
    [num_pages, HV, V, K].

    q, k [B, T, H, K]; v [B, T, HV, V]; a, b [B, T, HV]; the CSR page table
    (page_indices, page_indptr, last_page_len) in one int dtype; slots (T ==
    1 only): an optional int64 [B, 2] tensor of (read_page, write_page) rows
    from ``gdn_paged_decode_slots``. T > 1 needs page_size. Returns output
    [B, T, HV, V].
    """
    B, T, H, K = q.shape
    if T > 1 and page_size <= 0:
        raise ValueError("a multi-token suffix needs page_size")
    if T > 1 and slots is not None:
        raise ValueError("precomputed slots rows describe single-token calls only")
    HV, V = v.shape[2], v.shape[3]
    _expect(k, (B, T, H, K), "k")
    _expect(v, (B, T, HV, V), "v")
    _expect(a, (B, T, HV), "a")
    _expect(b, (B, T, HV), "b")
    _expect(A_log, (HV,), "A_log")
    _expect(dt_bias, (HV,), "dt_bias")
    _expect(page_indptr, (B + 1,), "page_indptr")
    _expect(last_page_len, (B,), "last_page_len")
    if page_indices.dim() != 1:
        raise ValueError("page_indices must be 1-D")
    if A_log.dtype != torch.float32 or dt_bias.dtype != torch.float32:
        raise ValueError("A_log and dt_bias must be float32")
    if len({x.dtype for x in (q, k, v, a, b)}) != 1:
        raise ValueError("q, k, v, a, b must share one dtype")
    out_dt = output_dtype or (output.dtype if output is not None else q.dtype)
    out = _out(output, (B, T, HV, V), out_dt, q)
    prm = gdn_decode_paged_params()
    prm.struct_size = ctypes.sizeof(gdn_decode_paged_params)
    prm.B, prm.T, prm.H, prm.HV, prm.K, prm.V = B, T, H, HV, K, V
    prm.in_dtype, prm.out_dtype = _io_dtype(q), _io_dtype(out)
    prm.index_dtype = _same_index_dtype(page_indices, page_indptr, last_page_len)
    prm.readout = _READOUTS[readout]
    prm.use_qk_l2norm = int(bool(use_qk_l2norm))
    prm.page_size = int(page_size)
    prm.scale = 0.0 if scale is None else float(scale)
    prm.nnz = page_indices.numel()
    prm.q, prm.k, prm.v, prm.a, prm.b = _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b)
    prm.A_log, prm.dt_bias = _ptr(A_log), _ptr(dt_bias)
    prm.page_indices, prm.page_indptr = _ptr(page_indices), _ptr(page_indptr)
    prm.last_page_len = _ptr(last_page_len)
    if slots is not None and (slots.dtype != torch.int64 or tuple(slots.shape) != (B, 2)):
        raise ValueError("slots must be an int64 [B, 2] tensor")
    prm.slots, prm.out, prm.err_flags = _ptr(slots), _ptr(out), _ptr(err_flags)
    prm.pool = _pool(state_pool, state_scales, state_layout, block_v, K, V, HV)
    _check(lib().gdn_decode_paged(ctypes.byref(prm), _stream(q)), "gdn_decode_paged")
    return out


def gdn_prefill_paged(q, k, v, a, b, A_log, dt_bias, cu_seqlens, *, state_pool, page_indices, page_indptr,
                      last_page_len, page_size, state_scales=None, state_layout="V_FIRST", block_v=64,
                      scale=None, use_qk_l2norm=True, output=None, output_dtype=None, readout="working",
                      err_flags=None):
    """Append a varlen run of tokens to every paged sequence (prefill or
    continued prefill); fresh sequences start from a zero state.

    q, k [total, H, K]; v [total, HV, V]; a, b [total, HV]; A_log, dt_bias
    [HV] fp32; cu_seqlens [B+1] int32; the CSR page table, whose
    last_page_len counts the new tokens. Returns output [total, HV, V].
    """
    total, H, K = q.shape
    HV, V = v.shape[1], v.shape[2]
    B = cu_seqlens.numel() - 1
    if page_size <= 0:
        raise ValueError("prefill needs page_size")
    _expect(k, (total, H, K), "k")
    _expect(v, (total, HV, V), "v")
    _expect(a, (total, HV), "a")
    _expect(b, (total, HV), "b")
    _expect(A_log, (HV,), "A_log")
    _expect(dt_bias, (HV,), "dt_bias")
    _expect(page_indptr, (B + 1,), "page_indptr")
    _expect(last_page_len, (B,), "last_page_len")
    if cu_seqlens.dtype != torch.int32 or page_indices.dim() != 1:
        raise ValueError("cu_seqlens must be int32 and page_indices 1-D")
    if A_log.dtype != torch.float32 or dt_bias.dtype != torch.float32:
        raise ValueError("A_log and dt_bias must be float32")
    if len({x.dtype for x in (q, k, v, a, b)}) != 1:
        raise ValueError("q, k, v, a, b must share one dtype")
    out_dt = output_dtype or (output.dtype if output is not None else q.dtype)
    out = _out(output, (total, HV, V), out_dt, q)
    prm = gdn_prefill_paged_params()
    prm.struct_size = ctypes.sizeof(gdn_prefill_paged_params)
    prm.B, prm.total_tokens, prm.H, prm.HV, prm.K, prm.V = B, total, H, HV, K, V
    prm.in_dtype, prm.out_dtype = _io_dtype(q), _io_dtype(out)
    prm.index_dtype = _same_index_dtype(page_indices, page_indptr, last_page_len)
    prm.readout = _READOUTS[readout]
    prm.use_qk_l2norm = int(bool(use_qk_l2norm))
    prm.page_size = int(page_size)
    prm.scale = 0.0 if scale is None else float(scale)
    prm.nnz = page_indices.numel()
    prm.q, prm.k, prm.v, prm.a, prm.b = _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b)
    prm.A_log, prm.dt_bias, prm.cu_seqlens = _ptr(A_log), _ptr(dt_bias), _ptr(cu_seqlens)
    prm.page_indices, prm.page_indptr, prm.last_page_len = _ptr(page_indices), _ptr(page_indptr), _ptr(last_page_len)
    prm.out, prm.err_flags = _ptr(out), _ptr(err_flags)
    prm.pool = _pool(state_pool, state_scales, state_layout, block_v, K, V, HV)
    _check(lib().gdn_prefill_paged(ctypes.byref(prm), _stream(q)), "gdn_prefill_paged")
    return out


def gdn_paged_decode_slots(page_indices, page_indptr, last_page_len, num_pages, page_size=0,
                           slots_out=None, err_flags=None):
    """(read_page, write_page) int64 rows [B, 2] of a paged decode step."""
    B = page_indptr.numel() - 1
    _expect(last_page_len, (B,), "last_page_len")
    slots_out = _out(slots_out, (B, 2), torch.int64, page_indptr)
    idt = _same_index_dtype(page_indices, page_indptr, last_page_len)
    _check(lib().gdn_paged_decode_slots(_ptr(page_indices), _ptr(page_indptr), _ptr(last_page_len), idt,
                                       page_indices.numel(), B, int(num_pages), int(page_size),
                                       _ptr(slots_out), _ptr(err_flags), _stream(page_indptr)),
           "gdn_paged_decode_slots")
    return slots_out


def kda_decode_varlen(q, k, v, raw_gate, beta_logits, a_log, dt_bias, cu_seqlens, state_pool,
                      state_indices, *, output_dtype=None, gate_mode="original", beta_mode="logits",
                      state_layout="K_FIRST", state_scales=None, block_v=64, readout="working",
                      output=None, err_flags=None):
    """KDA recurrence over varlen sequences; mutates state_pool in place.

    q, k [total, Hk, K]; v [total, HV, V]; raw_gate [total, HV, K];
    beta_logits [total, HV]; a_log [HV]; dt_bias [HV, K]; cu_seqlens [B+1]
    int32; state_indices [B] int32. Returns output [total, HV, V].
    """
    total, Hk, K = q.shape
    HV, V = v.shape[1], v.shape[2]
    B = cu_seqlens.numel() - 1
    _expect(k, (total, Hk, K), "k")
    _expect(v, (total, HV, V), "v")
    _expect(raw_gate, (total, HV, K), "raw_gate")
    _expect(beta_logits, (total, HV), "beta_logits")
    _expect(a_log, (HV,), "a_log")
    _expect(dt_bias, (HV, K), "dt_bias")
    _expect(state_indices, (B,), "state_indices")
    if a_log.dtype != torch.float32 or dt_bias.dtype != torch.float32:
        raise ValueError("a_log and dt_bias must be float32")
    if len({x.dtype for x in (q, k, v, raw_gate, beta_logits)}) != 1:
        raise ValueError("q, k, v, raw_gate, beta_logits must share one dtype")
    out_dt = output_dtype or (output.dtype if output is not None else q.dtype)
    out = _out(output, (total, HV, V), out_dt, q)
    if cu_seqlens.dtype != torch.int32 or state_indices.dtype != torch.int32:
        raise ValueError("cu_seqlens and state_indices must be int32")
    prm = kda_decode_varlen_params()
    prm.struct_size = ctypes.sizeof(kda_decode_varlen_params)
    prm.B, prm.total_tokens, prm.Hk, prm.HV, prm.K, prm.V = B, total, Hk, HV, K, V
    prm.in_dtype, prm.out_dtype = _io_dtype(q), _io_dtype(out)
    prm.gate_mode, prm.beta_mode = _GATE_MODES[gate_mode], _BETA_MODES[beta_mode]
    prm.readout = _READOUTS[readout]
    prm.q, prm.k, prm.v = _ptr(q), _ptr(k), _ptr(v)
    prm.raw_gate, prm.beta_logits = _ptr(raw_gate), _ptr(beta_logits)
    prm.a_log, prm.dt_bias = _ptr(a_log), _ptr(dt_bias)
    prm.cu_seqlens, prm.state_indices = _ptr(cu_seqlens), _ptr(state_indices)
    prm.out, prm.err_flags = _ptr(out), _ptr(err_flags)
    prm.pool = _pool(state_pool, state_scales, state_layout, block_v, K, V, HV)
    _check(lib().kda_decode_varlen(ctypes.byref(prm), _stream(q)), "kda_decode_varlen")
    return out


def gdn_state_quantize_fp8(src, *, block_v=64, layout="V_FIRST", codes=None,
                           scales=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """fp32 states [N, K, V] (K_FIRST) or [N, V, K] (V_FIRST) -> (uint8 codes, scales [N, V/block_v])."""
    N = src.shape[0]
    lay = _LAYOUTS[layout]
    K, V = (src.shape[1], src.shape[2]) if lay == GDN_K_FIRST else (src.shape[2], src.shape[1])
    codes = _out(codes, tuple(src.shape), torch.uint8, src)
    scales = _out(scales, (N, V // block_v), torch.float32, src)
    _check(lib().gdn_state_quantize_fp8(_ptr(src), _ptr(codes), _ptr(scales), N, K, V, block_v, lay,
                                       _stream(src)), "gdn_state_quantize_fp8")
    return codes, scales


def gdn_state_dequantize_fp8(codes, scales, *, block_v=64, layout="V_FIRST", out=None) -> torch.Tensor:
    N = codes.shape[0]
    lay = _LAYOUTS[layout]
    K, V = (codes.shape[1], codes.shape[2]) if lay == GDN_K_FIRST else (codes.shape[2], codes.shape[1])
    _expect(scales, (N, V // block_v), "scales")
    out = _out(out, tuple(codes.shape), torch.float32, codes)
    _check(lib().gdn_state_dequantize_fp8(_ptr(codes), _ptr(scales), _ptr(out), N, K, V, block_v, lay,
                                         _stream(codes)), "gdn_state_dequantize_fp8")
    return out


def gdn_state_quantize_int8h32(src, *, layout="V_FIRST", codes=None,
                               scales=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """fp32 states [N, K, V] (K_FIRST) or [N, V, K] (V_FIRST) -> (int8 codes, scales [N, V/32, K])."""
    N = src.shape[0]
    lay = _LAYOUTS[layout]
    K, V = (src.shape[1], src.shape[2]) if lay == GDN_K_FIRST else (src.shape[2], src.shape[1])
    codes = _out(codes, tuple(src.shape), torch.int8, src)
    scales = _out(scales, (N, V // 32, K), torch.float32, src)
    _check(lib().gdn_state_quantize_int8h32(_ptr(src), _ptr(codes), _ptr(scales), N, K, V, lay, _stream(src)),
           "gdn_state_quantize_int8h32")
    return codes, scales


def gdn_state_dequantize_int8h32(codes, scales, *, layout="V_FIRST", out=None) -> torch.Tensor:
    N = codes.shape[0]
    lay = _LAYOUTS[layout]
    K, V = (codes.shape[1], codes.shape[2]) if lay == GDN_K_FIRST else (codes.shape[2], codes.shape[1])
    _expect(scales, (N, V // 32, K), "scales")
    out = _out(out, tuple(codes.shape), torch.float32, codes)
    _check(lib().gdn_state_dequantize_int8h32(_ptr(codes), _ptr(scales), _ptr(out), N, K, V, lay, _stream(codes)),
           "gdn_state_dequantize_int8h32")
    return out


__all__ = ["gdn_decode_slots", "gdn_decode_paged", "gdn_prefill_paged", "gdn_paged_decode_slots", "kda_decode_varlen",
           "gdn_state_quantize_fp8", "gdn_state_dequantize_fp8", "gdn_state_quantize_int8h32",
           "gdn_state_dequantize_int8h32", "gdn_status_string", "GDNError",
           "LIB_PATH", "lib"]
