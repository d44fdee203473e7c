"""kvpack_decode_attn_noalloc: the decode step for callers that cannot give the
library device memory (a framework-owned plugin with no workspace hook, or a
serving loop that bans allocator calls because cudaMalloc / cudaFree can stall
on device-wide synchronisation).  Its scratch is a fixed array inside the
library.  This file sorts last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process.

Checks, through the C ABI:
* a first call on a larger shape (more visual splits per unit, a longer text
  tail) leaves other data in the shared array; two calls in a row on the test
  shape then give exactly the output and mass of the regular entry point
  (caller-allocated workspace, same kernels and same plan), and both agree
  with the fp64 oracle within the decode tolerance of the other GPU tests;
* a call needing more scratch than the array holds is refused before anything
  is launched."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from synth import cases
from gpu_util import DEV, assert_decode_close, bf, oracle_decode, u32

pytestmark = pytest.mark.gpu


def _device_case(kv, w, T, Lcap, n_layers):
    c = cases.decode_case(w, n_layers=n_layers, T=T, Lcap=Lcap)
    dims = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=Lcap)
    g = {k: bf(c[k]) for k in ("q", "CK_lo", "CK_hi", "BK", "CV_lo", "CV_hi", "BV", "K_text", "V_text")}
    return c, dims, g, u32(c["mask"])


def _noalloc_call(kv, dims, n_layers, g, L_text, mask, out, mass):
    return kv.lib().kvpack_decode_attn_noalloc(
        ctypes.byref(dims.c()), n_layers, g["q"].data_ptr(), g["CK_lo"].data_ptr(), g["CK_hi"].data_ptr(),
        g["BK"].data_ptr(), g["CV_lo"].data_ptr(), g["CV_hi"].data_ptr(), g["BV"].data_ptr(),
        g["K_text"].data_ptr(), g["V_text"].data_ptr(), L_text, mask.data_ptr(), 1.0, out.data_ptr(),
        mass.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_entry_point_twice():
    import rank_compressed_kv_b200 as kv
    assert kv.NOALLOC_SCRATCH_BYTES == 64 << 20

    # 1. a larger call first: many visual splits per unit and a long text tail fill more of the array
    wb = synth.Workload("noalloc_big", 78, 1, 1, 32, 8, 20000, 300, 1, "lowrank32")
    cb, dims_b, gb, mask_b = _device_case(kv, wb, wb.T, 300, 1)
    assert kv.decode_workspace(dims_b, 1) <= kv.NOALLOC_SCRATCH_BYTES
    out_b = torch.empty(wb.batch, wb.n_q, 128, dtype=torch.bfloat16, device=DEV)
    mass_b = torch.empty(dims_b.units(1), wb.T, dtype=torch.float32, device=DEV)
    assert _noalloc_call(kv, dims_b, 1, gb, 297, mask_b, out_b, mass_b) == 0
    assert kv.last_device_status() == 0

    # 2. the test shape through the regular entry point
    w = synth.Workload("noalloc", 77, 2, 2, 32, 8, 3000, 48, 1, "lowrank32")
    T, Lcap, L = w.T, 48, 45
    c, dims, g, mask = _device_case(kv, w, T, Lcap, 2)
    assert kv.decode_workspace(dims, 2) < kv.decode_workspace(dims_b, 1)
    ref_out = torch.empty(2 * w.batch, w.n_q, 128, dtype=torch.bfloat16, device=DEV)
    ref_mass = torch.empty(dims.units(2), T, dtype=torch.float32, device=DEV)
    ws = torch.empty(kv.decode_workspace(dims, 2), dtype=torch.uint8, device=DEV)
    kv.decode_attn(dims, 2, g["q"], g["CK_lo"], g["CK_hi"], g["BK"], g["CV_lo"], g["CV_hi"], g["BV"],
                   g["K_text"], g["V_text"], L, mask, 1.0, ref_out, ref_mass, ws)
    assert kv.last_device_status() == 0

    # 3. two no-allocation calls in a row: bit-identical to the regular entry point
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        mass = torch.full_like(ref_mass, float("nan"))
        assert _noalloc_call(kv, dims, 2, g, L, mask, out, mass) == 0
        assert kv.last_device_status() == 0
        assert torch.equal(out, ref_out)
        assert torch.equal(mass, ref_mass)

    # 4. and both match the fp64 oracle
    ref_o, ref_m = oracle_decode(w, c, L)
    assert_decode_close(w, out.float().cpu().numpy(), mass.cpu().numpy(), ref_o, ref_m)


def test_noalloc_refuses_oversized_scratch():
    import rank_compressed_kv_b200 as kv
    dims = kv.Dims(batch=64, n_q_heads=32, n_kv_heads=8, T_vis=65536, L_text_cap=16)
    assert kv.decode_workspace(dims, 32) > kv.NOALLOC_SCRATCH_BYTES
    p = 1 << 20   # never dereferenced: the size check comes before any launch
    st = kv.lib().kvpack_decode_attn_noalloc(ctypes.byref(dims.c()), 32, p, p, p, p, p, p, p, p, p, 8, p, 1.0, p,
                                             p, None)
    assert st == 4   # KVPACK_ERR_WORKSPACE
