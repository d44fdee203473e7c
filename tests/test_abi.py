"""The C ABI without a GPU: the library loads, exports every entry point that
include/kvpack.h declares, rejects bad arguments with the documented status
before touching the device, and its footprint accounting reproduces the
pages' LLaVA-1.5-7B figures."""
import ctypes
import json
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kv():
    import __graft_entry__
    __graft_entry__.build_library()
    import rank_compressed_kv_b200 as kv
    return kv


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "kvpack.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvpack_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(kv):
    syms = _declared_symbols()
    assert len(syms) >= 9
    lib = kv.lib()
    for s in syms:
        assert hasattr(lib, s), s


def test_version(kv):
    assert kv.version() == 1


def test_status_strings(kv):
    lib = kv.lib()
    for code, name in kv.STATUS_NAMES.items():
        assert lib.kvpack_status_string(code).decode() == name


def _dims(kv, **over):
    base = dict(batch=2, n_q_heads=16, n_kv_heads=8, T_vis=576, L_text_cap=64)
    base.update(over)
    return kv.Dims(**base)


def _call_decode(kv, dims, ws_bytes=None, ptr=0x10000, L_text=8, scale=1.0, n_layers=1):
    lib = kv.lib()
    ws = kv.decode_workspace(dims, n_layers) if ws_bytes is None else ws_bytes
    p = [ptr] * 9
    return lib.kvpack_decode_attn(ctypes.byref(dims.c()), n_layers, *p, L_text, ptr, scale, ptr, ptr, ptr, ws, None)


def test_decode_rejects_bad_arguments_before_launch(kv):
    assert _call_decode(kv, _dims(kv, head_dim=64)) == 3
    assert _call_decode(kv, _dims(kv, rank=32)) == 3
    assert _call_decode(kv, _dims(kv, n_kv_heads=6)) == 3
    assert _call_decode(kv, _dims(kv, n_q_heads=12)) == 3
    assert _call_decode(kv, _dims(kv, n_q_heads=72, n_kv_heads=8)) == 3      # Hg = 36 > 32
    assert _call_decode(kv, _dims(kv, T_vis=65537)) == 3
    assert _call_decode(kv, _dims(kv, rank_lo=8)) == 3          # reduced rank is 16 or 0 (not decompressed)
    assert _call_decode(kv, _dims(kv, T_vis=0)) == 1
    assert _call_decode(kv, _dims(kv, batch=0)) == 1
    assert _call_decode(kv, _dims(kv), n_layers=0) == 1
    assert _call_decode(kv, _dims(kv), L_text=65) == 1
    assert _call_decode(kv, _dims(kv), scale=0.0) == 1
    assert _call_decode(kv, _dims(kv), ptr=0x10008) == 2
    assert _call_decode(kv, _dims(kv), ws_bytes=16) == 4


def test_text_basis_decode_rejects_bad_arguments_before_launch(kv):
    lib = kv.lib()
    d = _dims(kv)
    ptr = 0x10000

    def call(tb, ws=None, L_c=None):
        n = kv.decode_tb_workspace(d, 1, L_c if L_c is not None else (tb.L_c if tb is not None else 0))
        return lib.kvpack_decode_attn_tb(ctypes.byref(d.c()), 1, *([ptr] * 7), ctypes.byref(tb) if tb else None,
                                         ptr, ptr, 8, ptr, 1.0, ptr, ptr, ptr, n if ws is None else ws, None)

    TB = kv._lib._CTextBasis
    assert call(None) == 1                                             # no text basis
    assert call(TB(ptr, ptr, ptr, ptr, ptr, None, 100)) == 1           # a missing plane
    assert call(TB(ptr, ptr, ptr, ptr, ptr, ptr + 8, 100)) == 2        # a misaligned plane
    assert call(TB(ptr, ptr, ptr, ptr, ptr, ptr, -1), ws=1 << 30) == 1
    assert call(TB(ptr, ptr, ptr, ptr, ptr, ptr, 65537), ws=1 << 30) == 1
    assert call(TB(ptr, ptr, ptr, ptr, ptr, ptr, 100), ws=16) == 4
    # the text tokens' own passes need room of their own; none at L_c = 0
    assert kv.decode_tb_workspace(d, 1, 0) == kv.decode_workspace(d, 1)
    assert kv.decode_tb_workspace(d, 1, 512) > kv.decode_workspace(d, 1)
    assert kv.decode_tb_workspace(d, 1, -1) == 0


def test_select_rejects_bad_arguments_before_launch(kv):
    lib = kv.lib()
    d = _dims(kv).c()
    assert lib.kvpack_select(ctypes.byref(d), 1, 0x1000, 0x1000, 0.0, 577, 0x1000, None) == 1
    assert lib.kvpack_select(ctypes.byref(d), 1, 0x1000, 0x1000, 1.0, 10, 0x1000, None) == 1
    assert lib.kvpack_select(ctypes.byref(d), 1, 0x1000, None, 0.5, 10, 0x1000, None) == 1
    assert lib.kvpack_select(ctypes.byref(d), 1, 0x1004, None, 0.0, 10, 0x1000, None) == 2
    assert lib.kvpack_select(ctypes.byref(d), 1, None, None, 0.0, 10, 0x1000, None) == 1


def test_compress_rejects_bad_arguments_before_launch(kv):
    lib = kv.lib()
    d = _dims(kv)
    ws = kv.compress_workspace(d, 1)
    assert ws > 0
    assert lib.kvpack_compress(ctypes.byref(d.c()), 1, 0x1000, 0x1000, 0x1000, 0x1000, None, 0x1000, ws - 1, None) == 4
    assert lib.kvpack_compress(ctypes.byref(d.c()), 1, 0x1002, 0x1000, 0x1000, 0x1000, None, 0x1000, ws, None) == 2
    assert lib.kvpack_compress(ctypes.byref(d.c()), 1, None, 0x1000, 0x1000, 0x1000, None, 0x1000, ws, None) == 1


def test_rank_zero_variant_is_a_supported_shape(kv):
    assert kv.decode_workspace(_dims(kv, rank_lo=0), 1) == kv.decode_workspace(_dims(kv), 1) > 0
    assert kv.decode_workspace(_dims(kv, rank_lo=8), 1) == 0


def test_workspace_grows_with_splits(kv):
    small = kv.decode_workspace(_dims(kv, T_vis=576), 1)
    big = kv.decode_workspace(_dims(kv, T_vis=65536), 1)
    assert big > small > 0


def test_footprint_reproduces_llava15_7b_figures(kv):
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "llava15_7b_footprint.json")))
    d = kv.Dims(batch=1, n_q_heads=g["n_q_heads"], n_kv_heads=g["n_kv_heads"], T_vis=g["visual_tokens"],
                L_text_cap=g["text_tokens"])
    dense, comp, basis = kv.footprint(d, g["layers"], g["text_tokens"])
    assert abs(dense / 1e6 - g["dense_MB"]) < g["dense_MB_tolerance"]
    assert abs(comp / 1e6 - g["compressed_MB"]) < g["compressed_MB_tolerance"]
    # per visual token: 512 bf16 features of K and V against 64 coefficients each
    d1 = kv.Dims(batch=1, n_q_heads=32, n_kv_heads=32, T_vis=1, L_text_cap=0)
    dn, cm, _ = kv.footprint(d1, 1, 0)
    assert dn // cm == g["per_token_reduction"] and dn % cm == 0
    assert basis == 256 * 64 * 512 * 4
