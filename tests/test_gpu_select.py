"""GPU top-k rank selection vs the oracle on identical fp32 input: bit-exact,
including ties (to the lower index), -0 / +0, NaN, k in {0, 1, T}, every size
regime of the kernel (warp per unit up to T = 2048, a cluster of 8 CTAs per unit above,
with 1 to 32 keys per thread) and
the moving-average importance update."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import DEV

pytestmark = pytest.mark.gpu


def _mass(T, seed, units=3):
    g = np.random.default_rng(seed)
    m = g.random((units, T)).astype(np.float32) * 1e-2
    if T >= 8:
        idx = g.integers(0, T, size=(units, max(2, T // 8)))
        for u in range(units):
            m[u, idx[u]] = m[u, idx[u][0]]          # a block of exact ties
        m[0, 1] = -0.0
        m[0, 2] = 0.0
        m[1, 3] = np.nan
        m[2, -1] = m[2].max()                       # tie with the maximum at the last index
    return m


def _run(kv, m, k, alpha=0.0, score=None):
    units, T = m.shape
    dims = kv.Dims(batch=units, n_q_heads=4, n_kv_heads=4, T_vis=T, L_text_cap=0)
    md = torch.from_numpy(m).to(DEV)
    sd = torch.from_numpy(score.copy()).to(DEV) if score is not None else None
    out = torch.full((units, (T + 31) // 32), -1, dtype=torch.int32, device=DEV)
    kv.select(dims, 1, md, sd, alpha, k, out)
    assert kv.last_device_status() == 0
    return out.cpu().numpy().view(np.uint32), (sd.cpu().numpy() if sd is not None else None)


@pytest.mark.parametrize("T", [1, 7, 31, 32, 33, 576, 1000, 2047, 2048, 2049, 2304, 4096, 4097, 6272, 8192, 8193, 20000, 32768, 65536])
def test_select_bit_exact(T):
    import rank_compressed_kv_b200 as kv
    m = _mass(T, T)
    for k in sorted({0, 1, T, math.ceil(0.25 * T), math.ceil(0.1 * T)}):
        got, _ = _run(kv, m, k)
        ref, _ = oracle.select(m, k)
        np.testing.assert_array_equal(got, ref, err_msg=f"T={T} k={k}")


@pytest.mark.parametrize("T", [100, 3000, 65536])
def test_moving_average_update_bit_exact(T):
    import rank_compressed_kv_b200 as kv
    g = np.random.default_rng(T + 1)
    m = g.random((3, T)).astype(np.float32)
    s = g.random((3, T)).astype(np.float32)
    k = math.ceil(0.25 * T)
    got, got_s = _run(kv, m, k, alpha=0.3, score=s)
    ref, ref_s = oracle.select(m, k, alpha=0.3, score=s)
    np.testing.assert_array_equal(got_s, ref_s)
    np.testing.assert_array_equal(got, ref)
