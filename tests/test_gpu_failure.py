"""Device failure paths, driven without faulting the GPU.

* An expired bounded wait: kvpack_selftest_bounded_wait runs the wait every
  kernel of the library uses on a barrier that nothing completes, with a
  limit of a million SM clocks; the kernel gives up, records
  KVPACK_ERR_TIMEOUT and returns.  The status is read and cleared through the
  C ABI, and a decode step right after still matches the oracle (the context
  is intact).
* The eigen-solver's iteration cap: KVPACK_EIG_MAX_ITER=1 leaves the
  subspace iteration unconverged, so kvpack_compress reports
  KVPACK_ERR_NOCONVERGE; the factors are still written (finite, with B's rows
  of unit norm)."""
import numpy as np
import pytest
import torch

import synth
from synth import cases
from gpu_util import DEV, assert_decode_close, bf, oracle_decode, run_decode

pytestmark = pytest.mark.gpu

TIMEOUT, NOCONVERGE = 7, 6


def test_expired_wait_reports_timeout_and_context_survives():
    import rank_compressed_kv_b200 as kv
    assert kv.last_device_status() == 0
    kv.selftest_bounded_wait(1_000_000)
    assert kv.last_device_status() == TIMEOUT
    assert kv.last_device_status() == 0          # read-and-clear
    w = synth.Workload("after_timeout", 5, 1, 1, 8, 8, 300, 16, 1, "lowrank32")
    c = cases.decode_case(w, n_layers=1, T=300, Lcap=16)
    got_o, got_m = run_decode(kv, w, c, 1, 300, 16, 16)
    ref_o, ref_m = oracle_decode(w, c, 16)
    assert_decode_close(w, got_o, got_m, ref_o, ref_m)


def test_selftest_rejects_bad_limits():
    import rank_compressed_kv_b200 as kv
    with pytest.raises(kv.KvpackError):
        kv.selftest_bounded_wait(0)


def test_iteration_cap_reports_noconverge(monkeypatch):
    import rank_compressed_kv_b200 as kv
    monkeypatch.setenv("KVPACK_EIG_MAX_ITER", "1")
    w = synth.WORKLOADS["C0"]
    T = w.T
    X_bits = synth.visual_kv(w, 0, 0, 0, synth.K_VIS)
    dims = kv.Dims(batch=1, n_q_heads=4, n_kv_heads=4, T_vis=T, L_text_cap=0)
    C_lo = torch.full((1, T, 16), float("nan"), dtype=torch.bfloat16, device=DEV)
    C_hi = torch.full((1, T, 48), float("nan"), dtype=torch.bfloat16, device=DEV)
    B = torch.full((1, 64, 512), float("nan"), dtype=torch.bfloat16, device=DEV)
    sig = torch.full((1, 64), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(kv.compress_workspace(dims, 1), dtype=torch.uint8, device=DEV)
    kv.compress(dims, 1, bf(X_bits[None]), C_lo, C_hi, B, sig, ws)
    assert kv.last_device_status() == NOCONVERGE
    for t in (C_lo, C_hi, B, sig):
        assert bool(torch.isfinite(t.float()).all())
    norms = B[0].double().norm(dim=1).cpu().numpy()
    assert np.all(np.abs(norms - 1.0) < 1e-2)
    monkeypatch.delenv("KVPACK_EIG_MAX_ITER")
    kv.compress(dims, 1, bf(X_bits[None]), C_lo, C_hi, B, sig, ws)
    assert kv.last_device_status() == 0
