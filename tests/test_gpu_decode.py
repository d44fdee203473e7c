"""GPU decode step vs the fp64 oracle on the same bf16 (C, B, mask, text, q).

Small shapes that still span several 128-token tiles, HI stages and text
stages, with ragged tails, T = 1, empty text, all-full / all-reduced masks,
every head-group size (Hg 4 / 8 / 16 / 28 / 32), a unit split over many CTAs
(long_split: 20000 tokens), multi-layer, multi-batch unit indexing, and the
rank-0 variant (low-importance tokens not decompressed at all: r_lo = 0)."""
import numpy as np
import pytest

import synth
from synth import cases
from gpu_util import assert_decode_close, oracle_decode, run_decode

pytestmark = pytest.mark.gpu

CASES = [
    # name,          batch, layers, n_q, n_kv, T,     Lcap, L_text, mask, r_lo
    ("c0",           1, 1, 8, 8, 576, 32, 32, "random", 16),
    ("ragged_T",     1, 1, 8, 8, 1000, 40, 37, "random", 16),
    ("T1",           2, 1, 8, 8, 1, 4, 3, "ones", 16),
    ("T1_lowrank",   1, 1, 8, 8, 1, 4, 0, "zeros", 16),
    ("no_text",      1, 2, 8, 8, 200, 16, 0, "random", 16),
    ("all_full",     1, 1, 8, 8, 333, 20, 20, "ones", 16),
    ("all_reduced",  1, 1, 8, 8, 333, 20, 20, "zeros", 16),
    ("gqa8",         1, 1, 16, 8, 700, 16, 16, "random", 16),
    ("gqa16_split2", 2, 1, 32, 8, 3000, 64, 50, "random", 16),
    ("gqa28_split3", 1, 2, 28, 4, 2000, 48, 48, "random", 16),
    ("gqa32",        1, 1, 64, 8, 900, 16, 9, "random", 16),
    ("many_units",   3, 2, 16, 16, 100, 8, 5, "random", 16),
    ("long_split",   1, 1, 32, 8, 20000, 300, 271, "random", 16),
    ("rank0_c0",     1, 1, 8, 8, 576, 32, 32, "random", 0),
    ("rank0_gqa28",  1, 1, 28, 4, 2000, 48, 30, "random", 0),
    ("rank0_no_text", 2, 1, 32, 8, 3000, 8, 0, "random", 0),
    ("rank0_all_zero", 1, 1, 8, 8, 300, 8, 5, "zeros", 0),
    # runs of full-rank tokens: blocks without a LO tile, HI tiles that span blocks, units split
    # over many CTAs (segments starting inside a unit, past full-rank tokens)
    ("blocks",       1, 2, 32, 8, 5000, 24, 20, "blocks", 16),
    ("blocks_gqa28", 1, 1, 28, 4, 4100, 16, 7, "blocks", 16),
    ("prefix_long",  2, 1, 16, 8, 9000, 16, 12, "prefix", 16),
    ("rank0_blocks", 1, 1, 32, 8, 3000, 8, 4, "blocks", 0),
]


@pytest.mark.parametrize("name,batch,layers,n_q,n_kv,T,Lcap,L_text,mask,r_lo", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(name, batch, layers, n_q, n_kv, T, Lcap, L_text, mask, r_lo):
    import rank_compressed_kv_b200 as kv
    w = synth.Workload(name, 100 + len(name), batch, layers, n_q, n_kv, T, Lcap, 1, "lowrank32")
    c = cases.decode_case(w, n_layers=layers, T=T, Lcap=Lcap, mask=mask)
    got_o, got_m = run_decode(kv, w, c, layers, T, Lcap, L_text, rank_lo=r_lo)
    ref_o, ref_m = oracle_decode(w, c, L_text, rank_lo=r_lo)
    assert np.all(np.isfinite(got_o))
    assert_decode_close(w, got_o, got_m, ref_o, ref_m)


def test_softmax_scale_and_null_mass():
    import rank_compressed_kv_b200 as kv
    w = synth.Workload("scale", 7, 1, 1, 16, 8, 700, 24, 1, "lowrank32")
    c = cases.decode_case(w, n_layers=1, T=700, Lcap=24)
    got_o, _ = run_decode(kv, w, c, 1, 700, 24, 24, scale=0.37, want_mass=False)
    ref_o, ref_m = oracle_decode(w, c, 24, scale=0.37)
    assert_decode_close(w, got_o, None, ref_o, ref_m)


def test_repeated_calls_agree():
    """The workspace carries nothing between calls that changes the result, and the
    result does not depend on which warp takes which item from the work counters
    (every item and every combine runs the same arithmetic in the same order, with
    no float atomics), so repeated calls agree bit for bit."""
    import rank_compressed_kv_b200 as kv
    w = synth.Workload("rep", 8, 1, 1, 32, 8, 4000, 64, 1, "lowrank32")
    c = cases.decode_case(w, n_layers=1, T=4000, Lcap=64)
    o1, m1 = run_decode(kv, w, c, 1, 4000, 64, 64)
    o2, m2 = run_decode(kv, w, c, 1, 4000, 64, 64)
    assert np.array_equal(o1, o2)
    assert np.array_equal(m1, m2)
