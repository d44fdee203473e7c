"""Helpers shared by the GPU tests: numpy <-> device tensors and oracle-side references."""
import numpy as np
import torch

import oracle
from synth import cases

DEV = torch.device("cuda:0")


def bf(a):
    """uint16 bf16 bits (numpy) -> torch.bfloat16 on the device."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV).view(torch.bfloat16)


def u32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32).view(np.int32)).to(DEV)


def run_decode(kv, w, c, n_layers, T, Lcap, L_text, scale=1.0, want_mass=True, rank_lo=16):
    dims = kv.Dims(batch=w.batch, n_q_heads=w.n_q, n_kv_heads=w.n_kv, T_vis=T, L_text_cap=Lcap, rank_lo=rank_lo)
    g = {k: bf(c[k]) for k in ("q", "CK_lo", "CK_hi", "BK", "CV_lo", "CV_hi", "BV", "K_text", "V_text")}
    mask = u32(c["mask"])
    out = torch.full((n_layers * w.batch, w.n_q, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    mass = torch.full((dims.units(n_layers), T), float("nan"), dtype=torch.float32, device=DEV) if want_mass else None
    ws = torch.empty(kv.decode_workspace(dims, n_layers), dtype=torch.uint8, device=DEV)
    kv.decode_attn(dims, n_layers, g["q"], g["CK_lo"], g["CK_hi"], g["BK"], g["CV_lo"], g["CV_hi"], g["BV"],
                   g["K_text"], g["V_text"], L_text, mask, scale, out, mass, ws)
    st = kv.last_device_status()
    assert st == 0, kv.STATUS_NAMES[st]
    o = out.float().cpu().numpy()
    return o, (mass.cpu().numpy() if want_mass else None)


def oracle_decode(w, c, L_text, scale=1.0, rank_lo=16):
    f = oracle.bf16_to_f64
    return oracle.decode(f(c["CK"]), f(c["BK"]), f(c["CV"]), f(c["BV"]), f(c["K_text"][:, :L_text]),
                         f(c["V_text"][:, :L_text]), c["mask"], f(cases.per_unit_queries(w, c["q"])), scale=scale,
                         r_lo=rank_lo)


def assert_decode_close(w, got_out, got_mass, ref_out, ref_mass, mass_rtol=1e-4):
    """Output: max-abs error <= 2e-2 * ||o||_inf per unit (fp32 accumulation, bf16 output).
    Mass: relative 1e-4 (q~ carried at ~2^-16, fp32 accumulation, ex2 at ~2^-22)."""
    got = cases.per_unit_outputs(w, got_out)
    for u in range(ref_out.shape[0]):
        err = np.abs(got[u] - ref_out[u]).max()
        bound = 2e-2 * np.abs(ref_out[u]).max()
        assert err <= bound, f"unit {u}: output error {err:.3e} > {bound:.3e}"
    if got_mass is not None:
        np.testing.assert_allclose(got_mass, ref_mass, rtol=mass_rtol, atol=1e-10)
