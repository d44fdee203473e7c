"""GPU decode step vs the fp64 oracle on the same bf16 (C, B, mask, text, q).

Small shapes that still span several 128-token tiles, HI stages and text
stages, with ragged tails, T = 1, empty text, all-full / all-reduced masks,
every head-group size (Hg 4 / 16 / 28 / 32), units split into many visual
items (long_split14: 79 items of 256 tokens) and multi-layer, multi-batch unit
indexing."""
import numpy as np
import pytest

import synth
from synth import cases
from gpu_util import assert_decode_close, oracle_decode, run_decode

pytestmark = pytest.mark.gpu

CASES = [
    # name,          batch, layers, n_q, n_kv, T,     Lcap, L_text, mask
    ("c0",           1, 1, 8, 8, 576, 32, 32, "random"),
    ("ragged_T",     1, 1, 8, 8, 1000, 40, 37, "random"),
    ("T1",           2, 1, 8, 8, 1, 4, 3, "ones"),
    ("T1_lowrank",   1, 1, 8, 8, 1, 4, 0, "zeros"),
    ("no_text",      1, 2, 8, 8, 200, 16, 0, "random"),
    ("all_full",     1, 1, 8, 8, 333, 20, 20, "ones"),
    ("all_reduced",  1, 1, 8, 8, 333, 20, 20, "zeros"),
    ("gqa16_split2", 2, 1, 32, 8, 3000, 64, 50, "random"),
    ("gqa28_split3", 1, 2, 28, 4, 2000, 48, 48, "random"),
    ("gqa32",        1, 1, 64, 8, 900, 16, 9, "random"),
    ("many_units",   3, 2, 16, 16, 100, 8, 5, "random"),
    ("long_split14", 1, 1, 32, 8, 20000, 300, 271, "random"),
]


@pytest.mark.parametrize("name,batch,layers,n_q,n_kv,T,Lcap,L_text,mask", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(name, batch, layers, n_q, n_kv, T, Lcap, L_text, mask):
    import rank_compressed_kv_b200 as kv
    w = synth.Workload(name, 100 + len(name), batch, layers, n_q, n_kv, T, Lcap, 1, "lowrank32")
    c = cases.decode_case(w, n_layers=layers, T=T, Lcap=Lcap, mask=mask)
    got_o, got_m = run_decode(kv, w, c, layers, T, Lcap, L_text)
    ref_o, ref_m = oracle_decode(w, c, L_text)
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
