"""The decode step with the text tokens compressed too, by a basis of their own
(kvpack_decode_attn_tb), through the C ABI, against the fp64 oracle's decode_tb
(the compressed text decompressed at the full rank, then dense attention over
visual + compressed text + uncompressed tail).

Cases: query-head groups of 4, 16 and 28; compressed text lengths 1, inside one
128-token tile, across tiles with a ragged last tile, and longer than the
visual cache; an empty tail; two layers; and L_c = 0, which must give exactly
the bits of kvpack_decode_attn."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import cases
from gpu_util import DEV, assert_decode_close, bf, u32

pytestmark = pytest.mark.gpu

F64 = oracle.bf16_to_f64


def _text_planes(w, n_layers, L_c):
    CK, BK, CV, BV = [], [], [], []
    for layer in range(n_layers):
        for b in range(w.batch):
            for g in range(w.groups):
                ck, bk = synth.text_compressed_unit(w, layer, b, g, synth.K_TEXT, L_c)
                cv, bv = synth.text_compressed_unit(w, layer, b, g, synth.V_TEXT, L_c)
                CK.append(ck); BK.append(bk); CV.append(cv); BV.append(bv)
    return np.stack(CK), np.stack(BK), np.stack(CV), np.stack(BV)


def _run(kv, w, c, n_layers, T, Lcap, L, tb_np, L_c):
    dims = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=Lcap)
    g = {k: bf(c[k]) for k in ("q", "CK_lo", "CK_hi", "BK", "CV_lo", "CV_hi", "BV", "K_text", "V_text")}
    CKt, BKt, CVt, BVt = tb_np
    U = dims.units(n_layers)
    if L_c > 0:
        tb = (bf(np.ascontiguousarray(CKt[:, :, :16])), bf(np.ascontiguousarray(CKt[:, :, 16:])), bf(BKt),
              bf(np.ascontiguousarray(CVt[:, :, :16])), bf(np.ascontiguousarray(CVt[:, :, 16:])), bf(BVt), L_c)
    else:
        tb = (None, None, None, None, None, None, 0)
    out = torch.full((n_layers * w.batch, w.n_q, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    mass = torch.full((U, T), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(kv.decode_tb_workspace(dims, n_layers, L_c), dtype=torch.uint8, device=DEV)
    kv.decode_attn_tb(dims, n_layers, g["q"], g["CK_lo"], g["CK_hi"], g["BK"], g["CV_lo"], g["CV_hi"], g["BV"], tb,
                      g["K_text"], g["V_text"], L, u32(c["mask"]), 1.0, out, mass, ws)
    st = kv.last_device_status()
    assert st == 0, kv.STATUS_NAMES[st]
    return out, mass


@pytest.mark.parametrize("name,batch,layers,n_q,n_kv,T,L_c,L", [
    ("c0", 1, 1, 8, 8, 576, 32, 1),
    ("gqa16", 2, 1, 32, 8, 700, 256, 9),
    ("gqa28_notail", 1, 1, 28, 4, 300, 1000, 0),
    ("lc1", 1, 1, 16, 8, 200, 1, 5),
    ("ragged_2layers", 1, 2, 32, 8, 1000, 333, 17),
])
def test_text_basis_decode_matches_oracle(name, batch, layers, n_q, n_kv, T, L_c, L):
    import rank_compressed_kv_b200 as kv
    w = synth.Workload(name, 60 + L_c, batch, layers, n_q, n_kv, T, max(L, 1), 1, "lowrank32")
    Lcap = max(L, 1)
    c = cases.decode_case(w, n_layers=layers, T=T, Lcap=Lcap)
    tb_np = _text_planes(w, layers, L_c)
    out, mass = _run(kv, w, c, layers, T, Lcap, L, tb_np, L_c)
    CKt, BKt, CVt, BVt = (F64(a) for a in tb_np)
    ref_o, ref_m = oracle.decode_tb(F64(c["CK"]), F64(c["BK"]), F64(c["CV"]), F64(c["BV"]), CKt, BKt, CVt, BVt,
                                    F64(c["K_text"][:, :L]), F64(c["V_text"][:, :L]), c["mask"],
                                    F64(cases.per_unit_queries(w, c["q"])))
    assert_decode_close(w, out.float().cpu().numpy(), mass.cpu().numpy(), ref_o, ref_m)


def test_text_basis_of_zero_tokens_is_the_plain_call():
    import rank_compressed_kv_b200 as kv
    from gpu_util import run_decode
    w = synth.Workload("lc0", 61, 2, 1, 32, 8, 900, 24, 1, "lowrank32")
    c = cases.decode_case(w, n_layers=1, T=w.T, Lcap=24)
    out, mass = _run(kv, w, c, 1, w.T, 24, 20, (None, None, None, None), 0)
    o2, m2 = run_decode(kv, w, c, 1, w.T, 24, 20)
    assert np.array_equal(out.float().cpu().numpy(), o2)
    assert np.array_equal(mass.cpu().numpy(), m2)
