"""The C ABI on the host: every declared symbol is exported, the ctypes
mirrors match the C struct layouts, and host validation rejects bad calls
before touching CUDA (no GPU needed)."""

import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import gated_delta_rule_80_b200 as G
from gated_delta_rule_80_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return G.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|const char\s*\*)\s*(\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"gdn_decode_slots", "gdn_decode_paged", "gdn_paged_decode_slots", "kda_decode_varlen", "gdn_prefill_paged",
            "gdn_state_quantize_fp8", "gdn_state_dequantize_fp8", "gdn_state_quantize_int8h32",
            "gdn_state_dequantize_int8h32", "gdn_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} is declared in include/gdn.h but not exported"


STRUCTS = {
    "gdn_state_pool": G.gdn_state_pool,
    "gdn_decode_slots_params": G.gdn_decode_slots_params,
    "gdn_decode_paged_params": G.gdn_decode_paged_params,
    "kda_decode_varlen_params": G.kda_decode_varlen_params,
    "gdn_prefill_paged_params": G.gdn_prefill_paged_params,
}


def test_ctypes_layout_matches_c():
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "gdn.h"', "int main(void){"]
    for cname, py in STRUCTS.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines.append("return 0;}")
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "probe.c")
        exe = os.path.join(d, "probe")
        open(src, "w").write("\n".join(lines))
        subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), src, "-o", exe], check=True)
        outp = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {}
    for line in outp:
        if line.strip():
            s, f, v = line.split()
            got[(s, f)] = int(v)
    for cname, py in STRUCTS.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


FAKE = 0x10000   # aligned, never dereferenced: validation rejects before any CUDA call


def _slots_params(**kw):
    p = G.gdn_decode_slots_params()
    p.struct_size = ctypes.sizeof(p)
    p.B, p.T, p.H, p.HV, p.K, p.V = 2, 1, 1, 2, 128, 128
    for f in ("q", "k", "v", "a", "b", "A_log", "dt_bias", "state_indices", "out"):
        setattr(p, f, FAKE)
    p.pool = G.gdn_state_pool(FAKE, None, 4, G.GDN_F32, G.GDN_V_FIRST, 64, 0)
    for k, v in kw.items():
        if k.startswith("pool_"):
            setattr(p.pool, k[5:], v)
        else:
            setattr(p, k, v)
    return p


@pytest.mark.parametrize("kw,expected", [
    (dict(struct_size=8), G.GDN_ERR_INVALID_ARG),
    (dict(K=48), G.GDN_ERR_INVALID_ARG),
    (dict(V=512), G.GDN_ERR_INVALID_ARG),
    (dict(K=96), G.GDN_ERR_INVALID_ARG),
    (dict(H=3), G.GDN_ERR_INVALID_ARG),
    (dict(B=-1), G.GDN_ERR_INVALID_ARG),
    (dict(in_dtype=2), G.GDN_ERR_INVALID_ARG),
    (dict(out_dtype=7), G.GDN_ERR_INVALID_ARG),
    (dict(index_dtype=5), G.GDN_ERR_INVALID_ARG),
    (dict(readout=3), G.GDN_ERR_INVALID_ARG),
    (dict(pool_layout=9), G.GDN_ERR_INVALID_ARG),
    (dict(pool_dtype=G.GDN_FP8_E4M3), G.GDN_ERR_INVALID_ARG),            # fp8 without scales
    (dict(pool_dtype=G.GDN_FP8_E4M3, pool_scales=FAKE, pool_block_v=32), G.GDN_ERR_UNSUPPORTED),
    (dict(pool_dtype=G.GDN_FP8_E4M3, pool_scales=FAKE, pool_block_v=48), G.GDN_ERR_INVALID_ARG),
    (dict(pool_dtype=G.GDN_INT8_H32), G.GDN_ERR_INVALID_ARG),            # int8 without scales
    (dict(pool_dtype=G.GDN_INT8_H32, pool_scales=FAKE + 4), G.GDN_ERR_INVALID_ARG),   # scales not 16-byte aligned
    (dict(pool_dtype=G.GDN_INT8_H32, pool_scales=FAKE, V=32), G.GDN_ERR_UNSUPPORTED),
    (dict(pool_dtype=4, pool_scales=FAKE), G.GDN_ERR_INVALID_ARG),
    (dict(q=FAKE + 4), G.GDN_ERR_INVALID_ARG),                           # misaligned
    (dict(out=None), G.GDN_ERR_INVALID_ARG),
    (dict(B=0), G.GDN_OK),                                               # nothing to do, no launch
    (dict(T=0), G.GDN_OK),
])
def test_slots_validation(lib, kw, expected):
    assert lib.gdn_decode_slots(ctypes.byref(_slots_params(**kw)), None) == expected


def test_null_params_and_status_strings(lib):
    assert lib.gdn_decode_slots(None, None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_decode_paged(None, None) == G.GDN_ERR_INVALID_ARG
    assert lib.kda_decode_varlen(None, None) == G.GDN_ERR_INVALID_ARG
    for s in (0, -1, -2, -3, 5):
        assert G.gdn_status_string(s)


def test_paged_validation(lib):
    p = G.gdn_decode_paged_params()
    p.struct_size = ctypes.sizeof(p)
    p.B, p.T, p.H, p.HV, p.K, p.V, p.nnz = 2, 1, 1, 2, 128, 128, 4
    for f in ("q", "k", "v", "a", "b", "A_log", "dt_bias", "out"):
        setattr(p, f, FAKE)
    p.pool = G.gdn_state_pool(FAKE, None, 4, G.GDN_F32, G.GDN_V_FIRST, 64, 0)
    assert lib.gdn_decode_paged(ctypes.byref(p), None) == G.GDN_ERR_INVALID_ARG   # no table, no slots
    p.nnz = -1
    assert lib.gdn_decode_paged(ctypes.byref(p), None) == G.GDN_ERR_INVALID_ARG
    p.nnz, p.B = 4, 0
    assert lib.gdn_decode_paged(ctypes.byref(p), None) == G.GDN_OK
    p.B, p.T, p.page_size = 2, 3, 0          # a suffix needs page_size
    assert lib.gdn_decode_paged(ctypes.byref(p), None) == G.GDN_ERR_INVALID_ARG
    p.page_size, p.slots = 16, FAKE          # precomputed rows are single-token only
    assert lib.gdn_decode_paged(ctypes.byref(p), None) == G.GDN_ERR_INVALID_ARG


def test_kda_validation(lib):
    p = G.kda_decode_varlen_params()
    p.struct_size = ctypes.sizeof(p)
    p.B, p.total_tokens, p.Hk, p.HV, p.K, p.V = 2, 3, 1, 2, 128, 128
    for f in ("q", "k", "v", "raw_gate", "beta_logits", "a_log", "dt_bias", "cu_seqlens", "state_indices", "out"):
        setattr(p, f, FAKE)
    p.pool = G.gdn_state_pool(FAKE, None, 4, G.GDN_F32, G.GDN_K_FIRST, 64, 0)
    p.gate_mode = G.KDA_GATE_SAFE
    assert lib.kda_decode_varlen(ctypes.byref(p), None) == G.GDN_ERR_UNSUPPORTED
    p.gate_mode, p.beta_mode = G.KDA_GATE_ORIGINAL, 4
    assert lib.kda_decode_varlen(ctypes.byref(p), None) == G.GDN_ERR_INVALID_ARG
    p.beta_mode, p.total_tokens = G.KDA_BETA_LOGITS, 0
    assert lib.kda_decode_varlen(ctypes.byref(p), None) == G.GDN_OK


def test_codec_validation(lib):
    f = lib.gdn_state_quantize_fp8
    assert f(FAKE, FAKE, FAKE, 1, 128, 128, 32, 1, None) == G.GDN_ERR_UNSUPPORTED
    assert f(FAKE, FAKE, FAKE, 1, 128, 100, 64, 1, None) == G.GDN_ERR_INVALID_ARG
    assert f(FAKE, FAKE, FAKE, 0, 128, 128, 64, 1, None) == G.GDN_OK
    assert lib.gdn_state_dequantize_fp8(FAKE, FAKE, FAKE, 1, 128, 128, 64, 7, None) == G.GDN_ERR_INVALID_ARG
    q8, d8 = lib.gdn_state_quantize_int8h32, lib.gdn_state_dequantize_int8h32
    assert q8(FAKE, FAKE, FAKE, 1, 128, 96, 1, None) == G.GDN_ERR_INVALID_ARG        # V not a head dim
    assert q8(FAKE, FAKE, FAKE, 1, 128, 128, 2, None) == G.GDN_ERR_INVALID_ARG       # layout
    assert q8(FAKE, FAKE + 8, FAKE, 1, 128, 128, 1, None) == G.GDN_ERR_INVALID_ARG   # codes misaligned
    assert q8(FAKE, None, FAKE, 1, 128, 128, 0, None) == G.GDN_ERR_INVALID_ARG
    assert q8(FAKE, FAKE, FAKE, 0, 128, 128, 0, None) == G.GDN_OK
    assert d8(FAKE, FAKE, FAKE, -1, 128, 128, 0, None) == G.GDN_ERR_INVALID_ARG
    assert d8(FAKE, FAKE, FAKE, 0, 32, 32, 1, None) == G.GDN_OK
    assert lib.gdn_paged_decode_slots(FAKE, FAKE, FAKE, 3, 4, 2, 8, 0, FAKE, None, None) == G.GDN_ERR_INVALID_ARG
    assert lib.gdn_paged_decode_slots(FAKE, FAKE, FAKE, 0, 4, 0, 8, 0, FAKE, None, None) == G.GDN_OK


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 1, 32)
    with pytest.raises(ValueError):
        G.gdn_decode_slots(x, x, x, torch.zeros(1, 1, 1), torch.zeros(1, 1, 1), torch.zeros(1), torch.zeros(1),
                           torch.zeros(1, 1, 32, 32), torch.zeros(1, dtype=torch.int32))


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library the binding raises; there is no fallback."""
    monkeypatch.setattr(G, "_lib", None)
    monkeypatch.setattr(G, "LIB_PATH", str(tmp_path / "libgdn_b200.so"))
    with pytest.raises(ImportError, match="no CPU fallback"):
        G.lib()
