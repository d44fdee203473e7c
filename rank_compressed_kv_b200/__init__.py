"""rank_compressed_kv_b200 -- Python binding of libkvpack (include/kvpack.h).

Decode-time attention over a multi-head, SVD-compressed visual KV cache with
attention-aware partial decompression (AttentionPack), as sm_100a kernels
behind a C ABI.  This module only marshals arguments: torch tensors become
device pointers, the current torch stream becomes the cudaStream_t.  Every
step of the computation runs in the library's CUDA kernels; there is no CPU
path, and importing fails if libkvpack.so has not been built.

Functions mirror the C entry points:

    compress(dims, n_layers, X, C_lo, C_hi, B, sigma, ws)
    decode_attn(dims, n_layers, q, CK_lo, CK_hi, BK, CV_lo, CV_hi, BV,
                K_text, V_text, L_text, mask, scale, out, mass, ws)
    decode_attn_tb(dims, n_layers, q, CK_lo, CK_hi, BK, CV_lo, CV_hi, BV,
                   text_basis, K_text, V_text, L_text, mask, scale, out, mass, ws)
    quantize4(dims, n_layers, T, C_lo, C_hi, Q_lo, Q_hi, E)
    decode_attn_q4(dims, n_layers, q, QK_lo, QK_hi, EK, BK, QV_lo, QV_hi, EV, BV,
                   K_text, V_text, L_text, mask, scale, out, mass, ws)
    select(dims, n_layers, mass, score, alpha, k_hi, mask_out)

bf16 arrays are torch.bfloat16 (or int16 views of bf16 bits); masks are
torch.int32 holding the uint32 words; fp32 arrays are torch.float32.
"""
from ._lib import (  # noqa: F401
    Dims,
    KvpackError,
    STATUS_NAMES,
    compress,
    compress_workspace,
    decode_attn,
    decode_attn_noalloc,
    decode_attn_tb,
    decode_tb_workspace,
    decode_attn_q4,
    quantize4,
    NOALLOC_SCRATCH_BYTES,
    decode_workspace,
    decompress,
    dense_decode_attn,
    dense_decode_workspace,
    footprint,
    last_device_status,
    lib,
    library_path,
    select,
    selftest_bounded_wait,
    version,
)
