"""The baselines behind the fused-kernel comparison, through the C ABI.

* kvpack_dense_decode_attn: standard attention over an uncompressed bf16 cache,
  against the oracle's decode with every token in its uncompressed tail (no
  visual tokens), at lengths inside one chunk, across chunk boundaries and
  with a ragged last chunk; query-head groups of 4, 16 and 28.
* kvpack_decompress: every visual token decompressed at its own rank (64 or
  r_lo = 16 / 0 by its mask bit), against the fp64 product C[:rho] B of the
  same bf16 factors (bf16 rounding of the result), and rows past T untouched.
* decompress-then-attend: kvpack_decompress followed by the dense decode over
  the decompressed visual rows plus the text tail gives the oracle's output
  on the compressed cache (decompress at each token's rank, then attend)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from synth import cases
from gpu_util import DEV, bf, u32

pytestmark = pytest.mark.gpu

F64 = oracle.bf16_to_f64


def _close(w, got, ref):
    got_u = cases.per_unit_outputs(w, got)
    for u in range(ref.shape[0]):
        err = np.abs(got_u[u] - ref[u]).max()
        assert err <= 2e-2 * np.abs(ref[u]).max(), f"unit {u}: {err:.3e}"


@pytest.mark.parametrize("batch,layers,n_q,n_kv,Lcap,L", [(1, 1, 8, 8, 64, 1), (2, 1, 8, 8, 64, 50),
                                                          (1, 2, 32, 8, 2200, 2100), (1, 1, 28, 4, 1100, 1024),
                                                          (2, 1, 32, 8, 3000, 2049)])
def test_dense_decode_matches_oracle(batch, layers, n_q, n_kv, Lcap, L):
    import rank_compressed_kv_b200 as kv
    w = synth.Workload("dense", 31 + L, batch, layers, n_q, n_kv, 1, Lcap, 1, "lowrank32")
    U = w.units_per_layer * layers
    g = np.random.default_rng(L)
    K = synth.to_bf16_bits(g.standard_normal((U, Lcap, 4, 128)))
    V = synth.to_bf16_bits(g.standard_normal((U, Lcap, 4, 128)))
    q = np.stack([synth.query(w, l, b, 0) for l in range(layers) for b in range(batch)])
    dims = kv.Dims(batch=batch, n_q_heads=n_q, n_kv_heads=n_kv, T_vis=1, L_text_cap=0)
    out = torch.full((layers * batch, n_q, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(kv.dense_decode_workspace(dims, layers, Lcap), dtype=torch.uint8, device=DEV)
    kv.dense_decode_attn(dims, layers, bf(q), bf(K), bf(V), Lcap, L, 1.0, out, ws)
    assert kv.last_device_status() == 0
    empty = np.zeros((U, 0, 64))
    ref, _ = oracle.decode(empty, np.zeros((U, 64, 512)), empty, np.zeros((U, 64, 512)), F64(K[:, :L]),
                           F64(V[:, :L]), np.zeros((U, 0), dtype=np.uint32), F64(cases.per_unit_queries(w, q)))
    _close(w, out.float().cpu().numpy(), ref)


@pytest.mark.parametrize("r_lo", [16, 0])
def test_decompress_matches_the_product_at_each_rank(r_lo):
    import rank_compressed_kv_b200 as kv
    w = synth.Workload("decomp", 44, 2, 1, 16, 8, 700, 8, 1, "lowrank32")
    T, Lcap = w.T, w.T + 40
    c = cases.decode_case(w, n_layers=1, T=T, Lcap=8)
    dims = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=8, rank_lo=r_lo)
    U = dims.units(1)
    Ko = torch.full((U, Lcap, 4, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    Vo = torch.full((U, Lcap, 4, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    kv.decompress(dims, 1, bf(c["CK_lo"]), bf(c["CK_hi"]), bf(c["BK"]), bf(c["CV_lo"]), bf(c["CV_hi"]), bf(c["BV"]),
                  u32(c["mask"]), Ko, Vo, Lcap)
    assert kv.last_device_status() == 0
    bits = oracle.mask_bits(c["mask"], T)
    rho = np.where(bits, 64, r_lo)
    keep = np.arange(64)[None, None, :] < rho[:, :, None]
    for side, (C, B, got) in enumerate(((c["CK"], c["BK"], Ko), (c["CV"], c["BV"], Vo))):
        ref = np.einsum("utr,urf->utf", F64(C) * keep, F64(B)).reshape(U, T, 4, 128)
        g = got.double().cpu().numpy()
        assert np.all(g[:, T:] == 7.0)                                   # rows past T untouched
        err = np.abs(g[:, :T] - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-3 * np.abs(ref).max()), f"side {side}: {err.max():.3e}"


@pytest.mark.parametrize("r_lo", [16, 0])
def test_decompress_then_attend_matches_oracle(r_lo):
    import rank_compressed_kv_b200 as kv
    w = synth.Workload("dta", 45, 2, 1, 32, 8, 1500, 64, 1, "lowrank32")
    T, L = w.T, 57
    c = cases.decode_case(w, n_layers=1, T=T, Lcap=64)
    dims = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=64, rank_lo=r_lo)
    U, Lcap = dims.units(1), T + 64
    Kd = torch.empty((U, Lcap, 4, 128), dtype=torch.bfloat16, device=DEV)
    Vd = torch.empty((U, Lcap, 4, 128), dtype=torch.bfloat16, device=DEV)
    Kd[:, T:] = bf(c["K_text"])
    Vd[:, T:] = bf(c["V_text"])
    kv.decompress(dims, 1, bf(c["CK_lo"]), bf(c["CK_hi"]), bf(c["BK"]), bf(c["CV_lo"]), bf(c["CV_hi"]), bf(c["BV"]),
                  u32(c["mask"]), Kd, Vd, Lcap)
    out = torch.empty((w.batch, w.n_q, 128), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(kv.dense_decode_workspace(dims, 1, Lcap), dtype=torch.uint8, device=DEV)
    kv.dense_decode_attn(dims, 1, bf(c["q"]), Kd, Vd, Lcap, T + L, 1.0, out, ws)
    assert kv.last_device_status() == 0
    ref, _ = oracle.decode(F64(c["CK"]), F64(c["BK"]), F64(c["CV"]), F64(c["BV"]), F64(c["K_text"][:, :L]),
                           F64(c["V_text"][:, :L]), c["mask"], F64(cases.per_unit_queries(w, c["q"])), r_lo=r_lo)
    _close(w, out.float().cpu().numpy(), ref)
