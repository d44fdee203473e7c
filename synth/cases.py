"""Decode-step inputs in the layouts of the kvpack C ABI (numpy, bf16 as uint16 bits).

Only draws and arranges inputs (no method arithmetic).  A unit is
(layer, batch row, KV group); u = (layer * batch + b) * groups + g.
"""
import numpy as np

from . import (COEF_K, K_TEXT, K_VIS, V_TEXT, V_VIS, Workload, all_ones_mask, compressed_unit, query,
               random_mask, text_kv)


def unit_inputs(w: Workload, layer: int, b: int, g: int, T: int, Lcap: int, mask: str = "random", k: int = None,
                step: int = 0):
    """One unit's compressed cache, text tail and rank mask.

    mask: "random" (k random bits, default k = ceil(hi_frac T)), "ones", "zeros", "blocks" (runs of
    512 full-rank and 512 reduced tokens, the first run 256 long, so runs straddle 128-token tiles),
    "prefix" (the first k tokens full-rank).
    Returns dict: CK, CV [T, 64]; BK, BV [64, 512]; K_text, V_text [Lcap, 4, 128]; mask [ceil(T/32)] uint32.
    """
    CK, BK = compressed_unit(w, layer, b, g, K_VIS, T)
    CV, BV = compressed_unit(w, layer, b, g, V_VIS, T)
    Kt = text_kv(w, layer, b, g, K_TEXT, Lcap)
    Vt = text_kv(w, layer, b, g, V_TEXT, Lcap)
    if mask == "random":
        m = random_mask(w, layer, b, g, T, k, step)
    elif mask == "ones":
        m = all_ones_mask(T)
    elif mask == "zeros":
        m = np.zeros((T + 31) // 32, dtype=np.uint32)
    elif mask in ("blocks", "prefix"):
        t = np.arange(T)
        if mask == "blocks":
            bits = ((t + 256) // 512) % 2 == 1
        else:
            bits = t < (k if k is not None else int(np.ceil(w.hi_frac * T)))
        padded = np.zeros(((T + 31) // 32) * 32, dtype=bool)
        padded[:T] = bits
        m = (padded.reshape(-1, 32).astype(np.uint64) << np.arange(32, dtype=np.uint64)).sum(axis=1).astype(np.uint32)
    else:
        raise ValueError(mask)
    return dict(CK=CK, CV=CV, BK=BK, BV=BV, K_text=Kt, V_text=Vt, mask=m)


def decode_case(w: Workload, n_layers: int = None, T: int = None, Lcap: int = None, mask: str = "random",
                k: int = None, step: int = 0):
    """Every unit of n_layers layers, stacked in the ABI layout."""
    n_layers = w.layers if n_layers is None else n_layers
    T = w.T if T is None else T
    Lcap = w.text0 if Lcap is None else Lcap
    units = []
    for layer in range(n_layers):
        for b in range(w.batch):
            for g in range(w.groups):
                units.append(unit_inputs(w, layer, b, g, T, Lcap, mask, k, step))
    CK = np.stack([u["CK"] for u in units])
    CV = np.stack([u["CV"] for u in units])
    q = np.stack([query(w, layer, b, step) for layer in range(n_layers) for b in range(w.batch)])
    return dict(
        CK=CK, CV=CV,
        CK_lo=np.ascontiguousarray(CK[:, :, :16]), CK_hi=np.ascontiguousarray(CK[:, :, 16:]),
        CV_lo=np.ascontiguousarray(CV[:, :, :16]), CV_hi=np.ascontiguousarray(CV[:, :, 16:]),
        BK=np.stack([u["BK"] for u in units]), BV=np.stack([u["BV"] for u in units]),
        K_text=np.stack([u["K_text"] for u in units]), V_text=np.stack([u["V_text"] for u in units]),
        mask=np.stack([u["mask"] for u in units]), q=q,
    )


def per_unit_queries(w: Workload, q: np.ndarray) -> np.ndarray:
    """q [n_layers*batch, n_q, 128] -> [units, Hg, 128] (the heads served by each group)."""
    lb, nq, d = q.shape
    return q.reshape(lb, w.groups, w.Hg, d).reshape(lb * w.groups, w.Hg, d)


def per_unit_outputs(w: Workload, out: np.ndarray) -> np.ndarray:
    lb, nq, d = out.shape
    return out.reshape(lb * w.groups, w.Hg, d)
