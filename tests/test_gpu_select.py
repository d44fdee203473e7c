"""GPU top-k rank selection vs the oracle on identical fp32 input: bit-exact,
including ties (to the lower index), -0 / +0, NaN, k in {0, 1, T}, every size
regime of the kernel (a warp per unit up to T = 2048, a 256-thread block up to 8192, a cluster
of 8 CTAs per unit above), ties that straddle the k-th key, and the moving-average importance
update."""
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


# every size the dispatch reaches: warp rows 1, 2, 4, 8, 12, 16, 18, 24, 32, 48, 64; block rows 9, 12, 16,
# 20, 25, 32; cluster keys per thread 8, 16, 32
@pytest.mark.parametrize("T", [1, 7, 31, 32, 33, 100, 200, 380, 500, 576, 700, 1000, 1500, 2047, 2048, 2049,
                               2304, 2600, 4096, 4097, 5000, 5200, 6272, 8192, 8193, 20000, 32768, 65536])
def test_select_bit_exact(T):
    import rank_compressed_kv_b200 as kv
    m = _mass(T, T)
    for k in sorted({0, 1, T, math.ceil(0.25 * T), math.ceil(0.1 * T)}):
        got, _ = _run(kv, m, k)
        ref, _ = oracle.select(m, k)
        np.testing.assert_array_equal(got, ref, err_msg=f"T={T} k={k}")


@pytest.mark.parametrize("T", [40, 576, 1000, 2304, 4100, 6272, 8192, 20000, 65536])
def test_select_straddling_ties(T):
    """Masses of four distinct values: the k-th key lies inside a large group of equal keys, so
    the first of them in token order must be taken and the rest left out."""
    import rank_compressed_kv_b200 as kv
    g = np.random.default_rng(T + 7)
    m = (g.integers(0, 4, size=(3, T)) / 4).astype(np.float32)
    m[0, 0] = -0.0
    m[1, T // 2] = np.nan
    for k in sorted({1, math.ceil(0.1 * T), math.ceil(0.25 * T), T - 1, T}):
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
