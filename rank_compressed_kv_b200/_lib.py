"""ctypes front end of libkvpack.so: argument marshalling only."""
import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(HERE, "libkvpack.so")

if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"libkvpack.so not found at {_LIB_PATH}; build it with `python rank_compressed_kv_b200/build.py` "
        "(there is no CPU fallback)")

_L = ctypes.CDLL(_LIB_PATH)

STATUS_NAMES = {
    0: "KVPACK_OK", 1: "KVPACK_ERR_INVALID_ARG", 2: "KVPACK_ERR_ALIGNMENT", 3: "KVPACK_ERR_UNSUPPORTED",
    4: "KVPACK_ERR_WORKSPACE", 5: "KVPACK_ERR_CUDA", 6: "KVPACK_ERR_NOCONVERGE", 7: "KVPACK_ERR_TIMEOUT",
}


class KvpackError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class _CDims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("batch", "n_q_heads", "n_kv_heads", "group", "head_dim", "T_vis", "L_text_cap", "rank", "rank_lo")]


@dataclass(frozen=True)
class Dims:
    batch: int
    n_q_heads: int
    n_kv_heads: int
    T_vis: int
    L_text_cap: int
    group: int = 4
    head_dim: int = 128
    rank: int = 64
    rank_lo: int = 16

    @property
    def groups(self) -> int:
        return self.n_kv_heads // self.group

    @property
    def Hg(self) -> int:
        return (self.n_q_heads // self.n_kv_heads) * self.group

    def units(self, n_layers: int) -> int:
        return n_layers * self.batch * self.groups

    def c(self) -> _CDims:
        return _CDims(self.batch, self.n_q_heads, self.n_kv_heads, self.group, self.head_dim, self.T_vis,
                      self.L_text_cap, self.rank, self.rank_lo)


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_sz = ctypes.c_size_t
_dims_p = ctypes.POINTER(_CDims)

_L.kvpack_version.restype = _i32
_L.kvpack_status_string.argtypes = [ctypes.c_int]
_L.kvpack_status_string.restype = ctypes.c_char_p
_L.kvpack_last_device_status.argtypes = [_vp]
_L.kvpack_last_device_status.restype = ctypes.c_int
_L.kvpack_footprint.argtypes = [_dims_p, _i32, _i32, ctypes.POINTER(ctypes.c_uint64)]
_L.kvpack_footprint.restype = ctypes.c_int
_L.kvpack_compress_workspace.argtypes = [_dims_p, _i32]
_L.kvpack_compress_workspace.restype = _sz
_L.kvpack_compress.argtypes = [_dims_p, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
_L.kvpack_compress.restype = ctypes.c_int
_L.kvpack_decode_workspace.argtypes = [_dims_p, _i32]
_L.kvpack_decode_workspace.restype = _sz
_L.kvpack_decode_attn.argtypes = [_dims_p, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp,
                                  ctypes.c_float, _vp, _vp, _vp, _sz, _vp]
_L.kvpack_decode_attn.restype = ctypes.c_int
_L.kvpack_decode_attn_noalloc.argtypes = [_dims_p, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32,
                                          _vp, ctypes.c_float, _vp, _vp, _vp]
_L.kvpack_decode_attn_noalloc.restype = ctypes.c_int
_L.kvpack_noalloc_scratch_bytes.restype = _sz


class _CTextBasis(ctypes.Structure):
    _fields_ = [("CK_lo", _vp), ("CK_hi", _vp), ("BK", _vp), ("CV_lo", _vp), ("CV_hi", _vp), ("BV", _vp),
                ("L_c", _i32)]


_L.kvpack_quantize4.argtypes = [_dims_p, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp]
_L.kvpack_quantize4.restype = ctypes.c_int
_L.kvpack_decode_attn_q4.argtypes = [_dims_p, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp,
                                     ctypes.c_float, _vp, _vp, _vp, _sz, _vp]
_L.kvpack_decode_attn_q4.restype = ctypes.c_int
_L.kvpack_decode_tb_workspace.argtypes = [_dims_p, _i32, _i32]
_L.kvpack_decode_tb_workspace.restype = _sz
_L.kvpack_decode_attn_tb.argtypes = [_dims_p, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(_CTextBasis),
                                     _vp, _vp, _i32, _vp, ctypes.c_float, _vp, _vp, _vp, _sz, _vp]
_L.kvpack_decode_attn_tb.restype = ctypes.c_int
_L.kvpack_dense_decode_workspace.argtypes = [_dims_p, _i32, _i32]
_L.kvpack_dense_decode_workspace.restype = _sz
_L.kvpack_dense_decode_attn.argtypes = [_dims_p, _i32, _vp, _vp, _vp, _i32, _i32, ctypes.c_float, _vp, _vp, _sz, _vp]
_L.kvpack_dense_decode_attn.restype = ctypes.c_int
_L.kvpack_decompress.argtypes = [_dims_p, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp]
_L.kvpack_decompress.restype = ctypes.c_int
_L.kvpack_selftest_bounded_wait.argtypes = [ctypes.c_int64, _vp]
_L.kvpack_selftest_bounded_wait.restype = ctypes.c_int
_L.kvpack_select.argtypes = [_dims_p, _i32, _vp, _vp, ctypes.c_float, _i32, _vp, _vp]
_L.kvpack_select.restype = ctypes.c_int


def lib():
    return _L


def library_path() -> str:
    return _LIB_PATH


def version() -> int:
    return int(_L.kvpack_version())


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("kvpack takes contiguous tensors")
    return t.data_ptr()


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(status: int, what: str):
    if status != 0:
        raise KvpackError(status, what)


def footprint(dims: Dims, n_layers: int, L_text: int):
    """(dense bytes, compressed coefficients + text bytes, basis bytes) of the cache."""
    out = (ctypes.c_uint64 * 3)()
    _check(_L.kvpack_footprint(ctypes.byref(dims.c()), n_layers, L_text, out), "kvpack_footprint")
    return int(out[0]), int(out[1]), int(out[2])


def compress_workspace(dims: Dims, n_layers: int) -> int:
    return int(_L.kvpack_compress_workspace(ctypes.byref(dims.c()), n_layers))


def decode_workspace(dims: Dims, n_layers: int) -> int:
    return int(_L.kvpack_decode_workspace(ctypes.byref(dims.c()), n_layers))


def compress(dims: Dims, n_layers: int, X, C_lo, C_hi, B, sigma, ws, stream=None):
    _check(_L.kvpack_compress(ctypes.byref(dims.c()), n_layers, _ptr(X), _ptr(C_lo), _ptr(C_hi), _ptr(B),
                              _ptr(sigma), _ptr(ws), _nbytes(ws), _stream(stream)), "kvpack_compress")


def decode_attn(dims: Dims, n_layers: int, q, CK_lo, CK_hi, BK, CV_lo, CV_hi, BV, K_text, V_text, L_text: int,
                mask, scale: float, out, mass, ws, stream=None):
    _check(_L.kvpack_decode_attn(ctypes.byref(dims.c()), n_layers, _ptr(q), _ptr(CK_lo), _ptr(CK_hi), _ptr(BK),
                                 _ptr(CV_lo), _ptr(CV_hi), _ptr(BV), _ptr(K_text), _ptr(V_text), L_text,
                                 _ptr(mask), float(scale), _ptr(out), _ptr(mass), _ptr(ws), _nbytes(ws),
                                 _stream(stream)), "kvpack_decode_attn")


def decode_attn_noalloc(dims: Dims, n_layers: int, q, CK_lo, CK_hi, BK, CV_lo, CV_hi, BV, K_text, V_text,
                        L_text: int, mask, scale: float, out, mass, stream=None):
    """decode_attn with the library's built-in scratch, for callers that cannot allocate device memory."""
    _check(_L.kvpack_decode_attn_noalloc(ctypes.byref(dims.c()), n_layers, _ptr(q), _ptr(CK_lo), _ptr(CK_hi),
                                         _ptr(BK), _ptr(CV_lo), _ptr(CV_hi), _ptr(BV), _ptr(K_text), _ptr(V_text),
                                         L_text, _ptr(mask), float(scale), _ptr(out), _ptr(mass), _stream(stream)),
           "kvpack_decode_attn_noalloc")


NOALLOC_SCRATCH_BYTES = int(_L.kvpack_noalloc_scratch_bytes())


def quantize4(dims: Dims, n_layers: int, T: int, C_lo, C_hi, Q_lo, Q_hi, E, stream=None):
    """4-bit codes (uint8, two per byte) and int8 exponents of the 16-bit coefficient planes."""
    _check(_L.kvpack_quantize4(ctypes.byref(dims.c()), n_layers, int(T), _ptr(C_lo), _ptr(C_hi), _ptr(Q_lo),
                               _ptr(Q_hi), _ptr(E), _stream(stream)), "kvpack_quantize4")


def decode_attn_q4(dims: Dims, n_layers: int, q, QK_lo, QK_hi, EK, BK, QV_lo, QV_hi, EV, BV, K_text, V_text,
                   L_text: int, mask, scale: float, out, mass, ws, stream=None):
    """decode_attn over 4-bit visual coefficients, dequantized inside the decode."""
    _check(_L.kvpack_decode_attn_q4(ctypes.byref(dims.c()), n_layers, _ptr(q), _ptr(QK_lo), _ptr(QK_hi), _ptr(EK),
                                    _ptr(BK), _ptr(QV_lo), _ptr(QV_hi), _ptr(EV), _ptr(BV), _ptr(K_text),
                                    _ptr(V_text), L_text, _ptr(mask), float(scale), _ptr(out), _ptr(mass),
                                    _ptr(ws), _nbytes(ws), _stream(stream)), "kvpack_decode_attn_q4")


def decode_tb_workspace(dims: Dims, n_layers: int, L_c: int) -> int:
    return int(_L.kvpack_decode_tb_workspace(ctypes.byref(dims.c()), n_layers, int(L_c)))


def decode_attn_tb(dims: Dims, n_layers: int, q, CK_lo, CK_hi, BK, CV_lo, CV_hi, BV, text_basis, K_text, V_text,
                   L_text: int, mask, scale: float, out, mass, ws, stream=None):
    """decode_attn with the text tokens compressed by a basis of their own: text_basis =
    (CK_lo, CK_hi, BK, CV_lo, CV_hi, BV, L_c) in the visual planes' layouts with L_c tokens."""
    tk_lo, tk_hi, tbk, tv_lo, tv_hi, tbv, L_c = text_basis
    tb = _CTextBasis(_ptr(tk_lo), _ptr(tk_hi), _ptr(tbk), _ptr(tv_lo), _ptr(tv_hi), _ptr(tbv), int(L_c))
    _check(_L.kvpack_decode_attn_tb(ctypes.byref(dims.c()), n_layers, _ptr(q), _ptr(CK_lo), _ptr(CK_hi), _ptr(BK),
                                    _ptr(CV_lo), _ptr(CV_hi), _ptr(BV), ctypes.byref(tb), _ptr(K_text),
                                    _ptr(V_text), L_text, _ptr(mask), float(scale), _ptr(out), _ptr(mass), _ptr(ws),
                                    _nbytes(ws), _stream(stream)), "kvpack_decode_attn_tb")


def select(dims: Dims, n_layers: int, mass, score, alpha: float, k_hi: int, mask_out, stream=None):
    _check(_L.kvpack_select(ctypes.byref(dims.c()), n_layers, _ptr(mass), _ptr(score), float(alpha), int(k_hi),
                            _ptr(mask_out), _stream(stream)), "kvpack_select")


def dense_decode_workspace(dims: Dims, n_layers: int, L_cap: int) -> int:
    return int(_L.kvpack_dense_decode_workspace(ctypes.byref(dims.c()), n_layers, L_cap))


def dense_decode_attn(dims: Dims, n_layers: int, q, K, V, L_cap: int, L: int, scale: float, out, ws, stream=None):
    """Standard attention over an uncompressed bf16 cache [units][L_cap][4][128] (the baseline)."""
    _check(_L.kvpack_dense_decode_attn(ctypes.byref(dims.c()), n_layers, _ptr(q), _ptr(K), _ptr(V), L_cap, L,
                                       float(scale), _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream)),
           "kvpack_dense_decode_attn")


def decompress(dims: Dims, n_layers: int, CK_lo, CK_hi, BK, CV_lo, CV_hi, BV, mask, K_out, V_out, L_cap: int,
               stream=None):
    """Every visual token decompressed at its rank into rows 0..T-1 of K_out, V_out [units][L_cap][4][128]."""
    _check(_L.kvpack_decompress(ctypes.byref(dims.c()), n_layers, _ptr(CK_lo), _ptr(CK_hi), _ptr(BK), _ptr(CV_lo),
                                _ptr(CV_hi), _ptr(BV), _ptr(mask), _ptr(K_out), _ptr(V_out), L_cap, _stream(stream)),
           "kvpack_decompress")


def selftest_bounded_wait(cycles: int, stream=None):
    """Run the bounded-wait self-test (a wait that nothing completes; expect KVPACK_ERR_TIMEOUT next)."""
    _check(_L.kvpack_selftest_bounded_wait(int(cycles), _stream(stream)), "kvpack_selftest_bounded_wait")


def last_device_status(stream=None) -> int:
    return int(_L.kvpack_last_device_status(_stream(stream)))
