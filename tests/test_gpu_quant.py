"""4-bit coefficients through the C ABI.

* kvpack_quantize4: codes and exponents bit-exact against the oracle's quantize4 (exact
  integer decisions: the exponent from an exact comparison, the code from an exact
  power-of-two division rounded half to even), on coefficients of very different scales,
  all-zero planes, values exactly on the grid and ties.
* kvpack_decode_attn_q4: the decode step over the 4-bit planes against the oracle's decode
  of the dequantized coefficients (the values q * 2^e are exact in bf16, so the tolerances
  are those of the 16-bit decode), for query-head groups of 4, 16 and 28, a ragged T, an
  all-full and an all-reduced mask, and the rank-0 variant."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import cases
from gpu_util import DEV, assert_decode_close, bf, u32

pytestmark = pytest.mark.gpu

F64 = oracle.bf16_to_f64


def _quantize_on_gpu(kv, dims, n_layers, T, C):
    U = C.shape[0]
    lo = bf(np.ascontiguousarray(C[:, :, :16]))
    hi = bf(np.ascontiguousarray(C[:, :, 16:]))
    Q_lo = torch.zeros((U, T, 8), dtype=torch.uint8, device=DEV)
    Q_hi = torch.zeros((U, T, 24), dtype=torch.uint8, device=DEV)
    E = torch.zeros((U, T, 2), dtype=torch.int8, device=DEV)
    kv.quantize4(dims, n_layers, T, lo, hi, Q_lo, Q_hi, E)
    assert kv.last_device_status() == 0
    return Q_lo, Q_hi, E


@pytest.mark.parametrize("T", [1, 37, 576])
def test_quantize4_bit_exact(T):
    import rank_compressed_kv_b200 as kv
    g = np.random.default_rng(T)
    U = 3
    C = g.standard_normal((U, T, 64)) * np.exp(g.uniform(-30, 30, size=(U, T, 1)))
    C[0, 0] = 0.0
    if T > 5:
        C[1, 2, :16] = 0.0
        C[1, 3, :] = np.round(C[1, 3, :] * 4) / 4          # values on a coarse grid
        C[2, 4, 0] = 7 * 2.0 ** 5                           # maximum exactly 7 * 2^e
        C[2, 4, 1:16] = 2.5 * 2.0 ** 5 * (np.arange(15) % 2)   # ties
    bits = synth.to_bf16_bits(C)
    dims = kv.Dims(batch=1, n_q_heads=4 * U, n_kv_heads=4 * U, T_vis=T, L_text_cap=1)
    Q_lo, Q_hi, E = _quantize_on_gpu(kv, dims, 1, T, bits)
    codes, exps = oracle.quantize4(F64(bits))
    rlo, rhi = oracle.pack4(codes)
    assert np.array_equal(Q_lo.cpu().numpy(), rlo)
    assert np.array_equal(Q_hi.cpu().numpy(), rhi)
    assert np.array_equal(E.cpu().numpy(), exps)


@pytest.mark.parametrize("name,batch,layers,n_q,n_kv,T,Lcap,L,mask,rank_lo", [
    ("c0", 1, 1, 8, 8, 576, 32, 32, "random", 16),
    ("gqa16", 2, 1, 32, 8, 2304, 64, 50, "random", 16),
    ("gqa28_ragged", 1, 2, 28, 4, 1000, 48, 48, "random", 16),
    ("allfull", 1, 1, 8, 8, 333, 20, 20, "ones", 16),
    ("allred", 1, 1, 16, 8, 700, 20, 20, "zeros", 16),
    ("rank0", 1, 1, 32, 8, 900, 16, 9, "random", 0),
])
def test_decode_q4_matches_oracle(name, batch, layers, n_q, n_kv, T, Lcap, L, mask, rank_lo):
    import rank_compressed_kv_b200 as kv
    w = synth.Workload(name, 90 + T, batch, layers, n_q, n_kv, T, Lcap, 1, "lowrank32")
    c = cases.decode_case(w, n_layers=layers, T=T, Lcap=Lcap, mask=mask)
    dims = kv.Dims(batch=batch, n_q_heads=n_q, n_kv_heads=n_kv, T_vis=T, L_text_cap=Lcap, rank_lo=rank_lo)
    U = dims.units(layers)
    QK = _quantize_on_gpu(kv, dims, layers, T, c["CK"])
    QV = _quantize_on_gpu(kv, dims, layers, T, c["CV"])
    out = torch.full((layers * batch, n_q, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    mass = torch.full((U, T), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(kv.decode_workspace(dims, layers), dtype=torch.uint8, device=DEV)
    kv.decode_attn_q4(dims, layers, bf(c["q"]), QK[0], QK[1], QK[2], bf(c["BK"]), QV[0], QV[1], QV[2], bf(c["BV"]),
                      bf(c["K_text"]), bf(c["V_text"]), L, u32(c["mask"]), 1.0, out, mass, ws)
    st = kv.last_device_status()
    assert st == 0, kv.STATUS_NAMES[st]
    DK = oracle.dequantize4(*oracle.quantize4(F64(c["CK"])))
    DV = oracle.dequantize4(*oracle.quantize4(F64(c["CV"])))
    ref_o, ref_m = oracle.decode(DK, F64(c["BK"]), DV, F64(c["BV"]), F64(c["K_text"][:, :L]), F64(c["V_text"][:, :L]),
                                 c["mask"], F64(cases.per_unit_queries(w, c["q"])), r_lo=rank_lo)
    assert_decode_close(w, out.float().cpu().numpy(), mass.cpu().numpy(), ref_o, ref_m)
