"""Seeded synthetic inputs for the compressed-KV decode path.

This package is shared by the tests, the oracle checks, bench.py and smoke():
it draws inputs only and holds none of the method's arithmetic.  Every array
is a pure function of (config seed, layer, batch row, group, stream kind[, step]),
drawn from numpy's Philox counter-based generator, so any single unit of any
workload can be regenerated on the host without generating the others.

Workloads (shapes of the pages' VLM evaluations -- LLaVA-1.5, LLaVA-NeXT-style
high resolution, VideoLLaVA-style video; no dataset items are used):

  name  batch x layers  n_q/n_kv  Hg  T_vis  text0  structure
  C0    1 x 1           8/8       4   576    32     rank-32, sigma_i = s0 * 0.9^i, + N(0, 0.05^2)
  C1    64 x 32         32/32     4   576    128    as C0
  C2    32 x 32         32/8      16  2304   256    as C0
  C3    16 x 28         28/4      28  6272   512    rank-24 row basis shared by 32 frames of 196
  C4    4 x 32          32/8      16  65536  1024   as C0

s0 is set so the signal has RMS 1 per element (sum of sigma_i^2 = T * 512).
Text K/V ~ N(0,1); q ~ N(0,1)/sqrt(128); softmax scale 1.  Values are
rounded to bf16 (through binary32, ties to even) and returned as uint16 bits.
"""
from dataclasses import dataclass
import math

import numpy as np
import torch

GROUP = 4
HEAD_DIM = 128
FEAT = GROUP * HEAD_DIM
RANK = 64
RANK_LO = 16
NOISE_STD = 0.05

K_VIS, V_VIS, K_TEXT, V_TEXT, QUERY, COEF_K, COEF_V, MASK, COEF_TK, COEF_TV = range(10)


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    batch: int
    layers: int
    n_q: int
    n_kv: int
    T: int
    text0: int
    steps: int
    structure: str          # "lowrank32" or "video24"
    hi_frac: float = 0.25
    frames: int = 1

    @property
    def groups(self) -> int:
        return self.n_kv // GROUP

    @property
    def Hg(self) -> int:
        return (self.n_q // self.n_kv) * GROUP

    @property
    def units_per_layer(self) -> int:
        return self.batch * self.groups

    @property
    def units(self) -> int:
        return self.layers * self.units_per_layer

    @property
    def k_hi(self) -> int:
        return math.ceil(self.hi_frac * self.T)

    def unit_index(self, layer: int, b: int, g: int) -> int:
        return (layer * self.batch + b) * self.groups + g

    def unit_coords(self, u: int):
        g = u % self.groups
        lb = u // self.groups
        return lb // self.batch, lb % self.batch, g

    def with_hi_frac(self, f: float) -> "Workload":
        return Workload(**{**self.__dict__, "hi_frac": f})


WORKLOADS = {
    "C0": Workload("C0", 0, 1, 1, 8, 8, 576, 32, 8, "lowrank32"),
    "C1": Workload("C1", 1, 64, 32, 32, 32, 576, 128, 128, "lowrank32"),
    "C2": Workload("C2", 2, 32, 32, 32, 8, 2304, 256, 256, "lowrank32"),
    "C3": Workload("C3", 3, 16, 28, 28, 4, 6272, 512, 256, "video24", frames=32),
    "C4": Workload("C4", 4, 4, 32, 32, 8, 65536, 1024, 128, "lowrank32"),
}


def rng(w: Workload, layer: int, b: int, g: int, kind: int, step: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([w.seed, layer, b, g, kind, step])
    return np.random.Generator(np.random.Philox(ss))


def to_bf16_bits(x) -> np.ndarray:
    """Round to bf16 through binary32 (ties to even); uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def _orthonormal_columns(g: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    a = g.standard_normal((rows, cols))
    qm, rm = np.linalg.qr(a)
    return qm * np.sign(np.diag(rm))[None, :]


def signal_sigmas(T: int, rank: int) -> np.ndarray:
    """sigma_i = s0 * 0.9^i, i < rank, with sum sigma_i^2 = T * 512 (signal RMS 1)."""
    decay = 0.9 ** np.arange(rank)
    s0 = math.sqrt(T * FEAT / float(np.sum(decay ** 2)))
    return s0 * decay


def visual_signal(w: Workload, layer: int, b: int, g: int, kind: int, T: int = None):
    """Noise-free fp64 signal of one unit's visual K or V and its exact singular values.

    lowrank32: U (T x 32) and W (512 x 32) with orthonormal columns; S = U diag(sigma) W^T.
    video24:   one W (512 x 24) for the unit, independent U_f (196 x 24) per frame;
               frame f is U_f diag(sigma) W^T with sigma for 196 tokens, so the
               unit's exact singular values are sqrt(frames) * sigma.
    """
    T = w.T if T is None else T
    gen = rng(w, layer, b, g, kind)
    if w.structure == "lowrank32":
        sig = signal_sigmas(T, 32)
        U = _orthonormal_columns(gen, T, 32)
        W = _orthonormal_columns(gen, FEAT, 32)
        return (U * sig[None, :]) @ W.T, sig
    if w.structure == "video24":
        per = T // w.frames
        assert per * w.frames == T
        sig = signal_sigmas(per, 24)
        W = _orthonormal_columns(gen, FEAT, 24)
        S = np.empty((T, FEAT))
        for f in range(w.frames):
            Uf = _orthonormal_columns(gen, per, 24)
            S[f * per:(f + 1) * per] = (Uf * sig[None, :]) @ W.T
        return S, sig * math.sqrt(w.frames)
    raise ValueError(w.structure)


def visual_kv(w: Workload, layer: int, b: int, g: int, kind: int, T: int = None) -> np.ndarray:
    """bf16 bits [T, 512] of one unit's visual K (kind=K_VIS) or V (kind=V_VIS): signal + N(0, 0.05^2)."""
    S, _ = visual_signal(w, layer, b, g, kind, T)
    noise = rng(w, layer, b, g, kind, step=1).standard_normal(S.shape) * NOISE_STD
    return to_bf16_bits(S + noise)


def text_kv(w: Workload, layer: int, b: int, g: int, kind: int, L: int) -> np.ndarray:
    """bf16 bits [L, 4, 128] of one unit's uncompressed text K or V, N(0,1)."""
    return to_bf16_bits(rng(w, layer, b, g, kind).standard_normal((L, GROUP, HEAD_DIM)))


def query(w: Workload, layer: int, b: int, step: int) -> np.ndarray:
    """bf16 bits [n_q, 128] of the decode query of (layer, batch row) at a step: N(0,1)/sqrt(128)."""
    x = rng(w, layer, b, 0, QUERY, step).standard_normal((w.n_q, HEAD_DIM)) / math.sqrt(HEAD_DIM)
    return to_bf16_bits(x)


def coefficient_sigmas(T: int, rank: int = RANK) -> np.ndarray:
    """Column scales of synthetic compressed coefficients: 32 signal values decaying as 0.9^i,
    then values at the top edge of the noise bulk, 0.05 (sqrt(T) + sqrt(512)), tapering by 30 %."""
    sig = np.empty(rank)
    sig[:32] = signal_sigmas(T, 32)
    edge = NOISE_STD * (math.sqrt(T) + math.sqrt(FEAT))
    sig[32:] = edge * (1.0 - 0.3 * np.arange(rank - 32) / (rank - 32))
    return sig


def compressed_unit(w: Workload, layer: int, b: int, g: int, kind: int, T: int = None):
    """Synthetic compressed cache of one unit, shaped like a rank-64 truncated SVD of the
    workload's K or V: coefficients C [T, 64] with N(0, sigma_i^2 / T) columns and a basis
    B [64, 512] with orthonormal rows.  bf16 bits.  Used where a decode-step input is wanted
    without running a compression first."""
    T = w.T if T is None else T
    return _coefficients(rng(w, layer, b, g, COEF_K if kind == K_VIS else COEF_V), T)


def _coefficients(gen: np.random.Generator, T: int):
    sig = coefficient_sigmas(T)
    C = gen.standard_normal((T, RANK)) * (sig / math.sqrt(T))[None, :]
    B = _orthonormal_columns(gen, FEAT, RANK).T
    return to_bf16_bits(C), to_bf16_bits(B)


def text_compressed_unit(w: Workload, layer: int, b: int, g: int, kind: int, L_c: int):
    """Synthetic compressed text of one unit (the text tokens factored with a basis of their own):
    coefficients C [L_c, 64] and basis B [64, 512] drawn like compressed_unit's, from their own
    stream (kind = K_TEXT or V_TEXT).  bf16 bits."""
    return _coefficients(rng(w, layer, b, g, COEF_TK if kind == K_TEXT else COEF_TV), L_c)


def random_mask(w: Workload, layer: int, b: int, g: int, T: int = None, k: int = None, step: int = 0) -> np.ndarray:
    """Packed uint32 rank mask [ceil(T/32)] with exactly k random bits set."""
    T = w.T if T is None else T
    k = w.k_hi if k is None else k
    idx = rng(w, layer, b, g, MASK, step).choice(T, size=min(k, T), replace=False)
    m = np.zeros((T + 31) // 32, dtype=np.uint32)
    np.bitwise_or.at(m, idx >> 5, (np.uint32(1) << (idx & 31).astype(np.uint32)))
    return m


def all_ones_mask(T: int) -> np.ndarray:
    m = np.zeros((T + 31) // 32, dtype=np.uint32)
    full, rem = divmod(T, 32)
    m[:full] = 0xFFFFFFFF
    if rem:
        m[full] = (1 << rem) - 1
    return m
