"""Parity at the workloads' full sizes, in the launch configuration bench.py times.

* decode + select over every unit of C1..C4 (the bench's device cache: eight
  generated units tiled over all units, a 25 % rank mask -- and 10 % for C4's
  sweep -- chosen by kvpack_select from a random mass): selection bit-exact against the oracle's
  on the same fp32 mass, outputs and attention mass against the fp64 oracle
  on sampled units (first, last, middle and an odd unit), and, on every unit,
  properties that hold at any size (finite outputs; mass >= 0 summing to at
  most the unit's query-head count).
* compression of one unit at C4's T = 65536: the oracle's SVD is out of reach
  at this size, so the checks are size-free facts of a truncated SVD (B has
  orthonormal rows, C's column norms are sigma, C^T C is diagonal, the
  residual is the discarded energy) plus the generator's known leading
  singular values.
* the decode -> select chain over C0's 8 steps, with importance = mass
  (alpha = 0) and with the moving average alpha = 0.5 carried on each side:
  decode parity at every step on the GPU's own mask, and the GPU's next mask
  equal to the oracle's wherever the oracle's importance is decided (relative
  gap to the k-th largest > 1e-3)."""
import numpy as np
import pytest
import torch

import bench
import oracle
import synth
from synth import cases
from gpu_util import DEV, bf, u32

pytestmark = pytest.mark.gpu

F64 = oracle.bf16_to_f64


def _sample_units(U):
    return sorted({0, U - 1, U // 2, (U // 3) | 1} & set(range(U)))


def _oracle_units(w, pool, units, q_np, mask_np, T, L):
    pick = [pool[u % bench.POOL] for u in units]
    CK = np.stack([F64(p["CK"]) for p in pick])
    CV = np.stack([F64(p["CV"]) for p in pick])
    BK = np.stack([F64(p["BK"]) for p in pick])
    BV = np.stack([F64(p["BV"]) for p in pick])
    Kt = np.stack([F64(p["K_text"][:L]) for p in pick])
    Vt = np.stack([F64(p["V_text"][:L]) for p in pick])
    qu = F64(cases.per_unit_queries(w, q_np))[units]
    return oracle.decode(CK, BK, CV, BV, Kt, Vt, mask_np, qu)


@pytest.mark.parametrize("name,hi_frac", [("C1", 0.25), ("C2", 0.25), ("C3", 0.25), ("C4", 0.25), ("C4", 0.10)])
def test_decode_and_select_at_full_size(name, hi_frac):
    import rank_compressed_kv_b200 as kv
    w = synth.WORKLOADS[name].with_hi_frac(hi_frac)
    T, U, Lcap, L = w.T, w.units, w.text0 + 2, w.text0 + 1
    dims = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=Lcap)
    c = bench.build_cache(kv, torch, w, Lcap, DEV)
    q_np = np.stack([synth.query(w, l, b, 1) for l in range(w.layers) for b in range(w.batch)])
    q = bf(q_np)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(1000 + w.seed)
    mass_prev = torch.rand(U, T, generator=gen, device=DEV)
    nwords = (T + 31) // 32
    mask = torch.empty(U, nwords, dtype=torch.int32, device=DEV)
    kv.select(dims, w.layers, mass_prev, None, 0.0, w.k_hi, mask)
    out = torch.full((w.layers * w.batch, w.n_q, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    mass = torch.full((U, T), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(kv.decode_workspace(dims, w.layers), dtype=torch.uint8, device=DEV)
    kv.decode_attn(dims, w.layers, q, c["CK_lo"], c["CK_hi"], c["BK"], c["CV_lo"], c["CV_hi"], c["BV"],
                   c["K_text"], c["V_text"], L, mask, 1.0, out, mass, ws)
    st = kv.last_device_status()
    assert st == 0, kv.STATUS_NAMES[st]

    # every unit: finite outputs, a valid attention mass
    out_f = out.float()
    assert bool(torch.isfinite(out_f).all())
    assert bool(torch.isfinite(mass).all()) and float(mass.min()) >= 0.0
    assert float(mass.sum(dim=1).max()) <= w.Hg * (1 + 1e-4)

    units = _sample_units(U)
    # selection: bit-exact on the same fp32 input
    ref_mask, _ = oracle.select(mass_prev[units].cpu().numpy(), w.k_hi)
    got_mask = mask[units].cpu().numpy().view(np.uint32)
    assert np.array_equal(ref_mask, got_mask)

    # decode: the sampled units against the fp64 oracle on the same bf16 inputs and mask
    pool = [cases.unit_inputs(w, 0, i % w.batch, i % w.groups, T, Lcap, mask="ones") for i in range(bench.POOL)]
    ref_o, ref_m = _oracle_units(w, pool, units, q_np, got_mask, T, L)
    got_o = cases.per_unit_outputs(w, out_f.cpu().numpy())[units]
    got_m = mass[units].cpu().numpy()
    for i, u in enumerate(units):
        err = np.abs(got_o[i] - ref_o[i]).max()
        bound = 2e-2 * np.abs(ref_o[i]).max()
        assert err <= bound, f"{name} unit {u}: output error {err:.3e} > {bound:.3e}"
    np.testing.assert_allclose(got_m, ref_m, rtol=1e-4, atol=1e-10)


def test_compress_one_unit_at_T65536():
    import rank_compressed_kv_b200 as kv
    w = synth.WORKLOADS["C4"]
    T = w.T
    X_bits = synth.visual_kv(w, 0, 0, 0, synth.K_VIS)
    dims = kv.Dims(batch=1, n_q_heads=4, n_kv_heads=4, T_vis=T, L_text_cap=0)
    X = bf(X_bits[None])
    C_lo = torch.empty(1, T, 16, dtype=torch.bfloat16, device=DEV)
    C_hi = torch.empty(1, T, 48, dtype=torch.bfloat16, device=DEV)
    B = torch.empty(1, 64, 512, dtype=torch.bfloat16, device=DEV)
    sig = torch.empty(1, 64, dtype=torch.float32, device=DEV)
    ws = torch.empty(kv.compress_workspace(dims, 1), dtype=torch.uint8, device=DEV)
    kv.compress(dims, 1, X, C_lo, C_hi, B, sig, ws)
    st = kv.last_device_status()
    assert st == 0, kv.STATUS_NAMES[st]
    s = sig[0].double().cpu().numpy()
    Bm = B[0].double().cpu().numpy()
    C = torch.cat([C_lo, C_hi], dim=2)[0].double().cpu().numpy()
    Xf = F64(X_bits)

    assert np.all(np.diff(s) <= 1e-6 * s[0])                       # descending
    assert np.abs(Bm @ Bm.T - np.eye(64)).max() < 1e-2               # orthonormal rows (bf16)
    cn = np.linalg.norm(C, axis=0)
    np.testing.assert_allclose(cn, s, rtol=1e-2)                      # |C[:, i]| = sigma_i
    G = C.T @ C
    off = np.abs(G - np.diag(np.diag(G))).max()
    assert off < 1e-2 * s[0] ** 2                                    # C = U Sigma with orthogonal U
    # the leading singular values follow the generator's signal (noise edge ~ 0.05 (sqrt T + sqrt 512))
    sig_signal = np.concatenate([synth.signal_sigmas(T, 32), np.zeros(32)])
    lead = sig_signal > 10 * 0.05 * (np.sqrt(T) + np.sqrt(512))
    np.testing.assert_allclose(s[:32][lead[:32]], sig_signal[:32][lead[:32]], rtol=1e-2)
    # residual energy = the energy of X outside the kept subspace (a difference of large
    # energies: sigma from the fp32 eigen-solve carries ~1e-5 of the total)
    R = Xf - C @ Bm
    res = float((R * R).sum())
    tot = float((Xf * Xf).sum())
    assert abs(res - (tot - float((s * s).sum()))) <= 5e-2 * res + 1e-5 * tot


@pytest.mark.parametrize("alpha", [0.0, 0.5])
def test_decode_select_chain_c0(alpha):
    import rank_compressed_kv_b200 as kv
    w = synth.WORKLOADS["C0"]
    T, U, steps = w.T, w.units, w.steps
    Lcap = w.text0 + steps
    per = [cases.unit_inputs(w, 0, 0, g, T, Lcap, mask="ones") for g in range(U)]
    dims = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=Lcap)
    dev = {k: bf(np.stack([p[k] for p in per])) for k in ("BK", "BV", "K_text", "V_text")}
    CK = np.stack([p["CK"] for p in per])
    CV = np.stack([p["CV"] for p in per])
    dev["CK_lo"], dev["CK_hi"] = bf(CK[..., :16]), bf(CK[..., 16:])
    dev["CV_lo"], dev["CV_hi"] = bf(CV[..., :16]), bf(CV[..., 16:])
    ws = torch.empty(kv.decode_workspace(dims, 1), dtype=torch.uint8, device=DEV)
    mask = u32(np.stack([synth.all_ones_mask(T)] * U))
    score = torch.zeros(U, T, dtype=torch.float32, device=DEV)    # the GPU's importance state
    ref_score = np.zeros((U, T), dtype=np.float32)                  # the oracle's, from its own masses
    for step in range(steps):
        L = w.text0 + step
        q_np = np.stack([synth.query(w, 0, b, step) for b in range(w.batch)])
        out = torch.empty(w.batch, w.n_q, 128, dtype=torch.bfloat16, device=DEV)
        mass = torch.empty(U, T, dtype=torch.float32, device=DEV)
        kv.decode_attn(dims, 1, bf(q_np), dev["CK_lo"], dev["CK_hi"], dev["BK"], dev["CV_lo"], dev["CV_hi"],
                       dev["BV"], dev["K_text"], dev["V_text"], L, mask, 1.0, out, mass, ws)
        assert kv.last_device_status() == 0
        m_np = mask.cpu().numpy().view(np.uint32)
        ref_o, ref_m = oracle.decode(F64(CK), F64(np.stack([p["BK"] for p in per])), F64(CV),
                                     F64(np.stack([p["BV"] for p in per])),
                                     F64(np.stack([p["K_text"][:L] for p in per])),
                                     F64(np.stack([p["V_text"][:L] for p in per])), m_np,
                                     F64(cases.per_unit_queries(w, q_np)))
        got_o = cases.per_unit_outputs(w, out.float().cpu().numpy())
        for u in range(U):
            assert np.abs(got_o[u] - ref_o[u]).max() <= 2e-2 * np.abs(ref_o[u]).max()
        got_m = mass.cpu().numpy()
        np.testing.assert_allclose(got_m, ref_m, rtol=1e-4, atol=1e-10)
        # next mask: GPU selection from its own mass vs the oracle's from the oracle's mass
        nxt = torch.empty_like(mask)
        kv.select(dims, 1, mass, score if alpha > 0 else None, alpha, w.k_hi, nxt)
        got_next = nxt.cpu().numpy().view(np.uint32)
        ref_next, ref_score = oracle.select(ref_m.astype(np.float32), w.k_hi, alpha=alpha, score=ref_score)
        keys = ref_score if alpha > 0 else ref_m
        bits = lambda m: ((m[:, np.arange(T) >> 5] >> (np.arange(T) & 31).astype(np.uint32)) & 1).astype(bool)
        gb, rb = bits(got_next), bits(ref_next)
        for u in range(U):
            theta = np.sort(keys[u])[::-1][w.k_hi - 1]
            decided = np.abs(keys[u] - theta) > 1e-3 * theta
            assert np.array_equal(gb[u][decided], rb[u][decided]), f"alpha {alpha} step {step} unit {u}"
        mask = nxt
