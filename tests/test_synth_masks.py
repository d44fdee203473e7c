"""The synthetic rank masks the decode parity cases use: bit t of word t // 32 (LSB first) marks a
full-rank token; the structured forms exercise whole blocks of full-rank tokens."""
import numpy as np
import pytest

import synth
from synth import cases


def _bits(m, T):
    return np.unpackbits(m.view(np.uint8), bitorder="little")[:T].astype(bool)


@pytest.mark.parametrize("T", [1, 31, 32, 333, 1000, 5000])
def test_mask_forms(T):
    w = synth.Workload("m", 3, 1, 1, 8, 8, T, 8, 1, "lowrank32")
    t = np.arange(T)
    forms = {
        "ones": np.ones(T, bool),
        "zeros": np.zeros(T, bool),
        "blocks": ((t + 256) // 512) % 2 == 1,
        "prefix": t < int(np.ceil(w.hi_frac * T)),
    }
    for name, want in forms.items():
        m = cases.unit_inputs(w, 0, 0, 0, T, 8, name)["mask"]
        assert m.dtype == np.uint32 and m.shape == ((T + 31) // 32,)
        assert np.array_equal(_bits(m, T), want), name
        # no bits past T
        assert np.unpackbits(m.view(np.uint8), bitorder="little")[T:].sum() == 0, name
    r = cases.unit_inputs(w, 0, 0, 0, T, 8, "random")["mask"]
    assert _bits(r, T).sum() == int(np.ceil(w.hi_frac * T))
