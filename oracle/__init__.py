"""Plain CPU oracle for fine-grained online FP8 quantization and the
block-scaled FP8 GEMM -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does: it
shares no code with the oracle, and it fails loudly when its own CUDA
extension is missing instead of falling back to anything here.

This module is argument marshalling around ``fp8_oracle.c`` (numpy arrays
in, numpy arrays out).  What each function computes, and the page passage
it follows, is documented in that file.  bf16 inputs are passed as their
raw 16-bit patterns (``numpy.uint16``); fp32 inputs as ``numpy.float32``.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(library cross-checks, closed forms, invariants and brute force); none is
"parity unpinned".
"""
import ctypes
import os

import numpy as np

from . import build as _build

IN_BF16 = 0
IN_FP32 = 1

_lib = None


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_decode_array.argtypes = [vp, i64, vp]
        L.orc_e4m3_encode_array.argtypes = [vp, i64, vp]
        L.orc_quantize_act_1x128.argtypes = [vp, i32, i64, i64, i64, vp, i64, vp, i64, i64]
        L.orc_quantize_weight_128x128.argtypes = [vp, i32, i64, i64, i64, vp, i32, i64,
                                                  vp, i64, i64]
        L.orc_gemm_ref.argtypes = [vp, i64, vp, i64, i64, vp, i64, i32, vp, i64, i64,
                                   i64, i64, i64, vp, vp]
        L.orc_gemm_ref_entries.argtypes = [vp, i64, vp, i64, i64, vp, i64, i32, vp, i64,
                                           i64, i64, i64, vp, vp, vp, vp]
        L.orc_grouped_gemm_ref.argtypes = [vp, i64, vp, i64, i64, vp, i64, i64, vp, i64,
                                           i64, i64, vp, i32, i64, i64, vp, vp]
        L.orc_gemm_exact.argtypes = [vp, i32, i64, vp, i32, i64, i64, i64, i64, vp]
        L.orc_num_threads.restype = ctypes.c_int
        L.orc_num_threads.argtypes = []
        _lib = L
    return _lib


def _p(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _as_input(x):
    """Return (contiguous array, type code) for a bf16-bits or fp32 array."""
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), IN_BF16
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), IN_FP32
    raise TypeError("oracle inputs are bf16 bit patterns (uint16) or float32, got %s" % x.dtype)


def num_threads() -> int:
    return lib().orc_num_threads()


def e4m3_decode(codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    lib().orc_e4m3_decode_array(_p(c), c.size, _p(out))
    return out


def e4m3_encode(values) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def quantize_act_1x128(x):
    """x [M,K] -> (q uint8 [M,K], sa float32 [M, ceil(K/128)])."""
    x, t = _as_input(x)
    M, K = x.shape
    nkb = (K + 127) // 128
    q = np.empty((M, K), dtype=np.uint8)
    sa = np.empty((M, nkb), dtype=np.float32)
    lib().orc_quantize_act_1x128(_p(x), t, M, K, K, _p(q), K, _p(sa), nkb, 1)
    return q, sa


def quantize_act_128x1(x):
    """x [M,K] -> (qt uint8 [K,M], st float32 [K, ceil(M/128)]): the 1x128
    activation quantization ([KB] "Finkornig kvantisering") of x^T, i.e.
    tiles of 128 consecutive rows of one column of x, as the weight gradient
    X^T dY needs for its contraction over the rows (tokens)."""
    x, _ = _as_input(x)
    return quantize_act_1x128(np.ascontiguousarray(x.T))


def quantize_weight_128x128(w, transpose_out=False):
    """w [K,N] -> (q uint8 [K,N] or [N,K], sb float32 [ceil(K/128), ceil(N/128)])."""
    w, t = _as_input(w)
    K, N = w.shape
    nkb, nnb = (K + 127) // 128, (N + 127) // 128
    if transpose_out:
        q = np.empty((N, K), dtype=np.uint8)
        ldq = K
    else:
        q = np.empty((K, N), dtype=np.uint8)
        ldq = N
    sb = np.empty((nkb, nnb), dtype=np.float32)
    lib().orc_quantize_weight_128x128(_p(w), t, K, N, N, _p(q), int(bool(transpose_out)),
                                      ldq, _p(sb), nnb, 1)
    return q, sb


def _scales(s, name):
    s = np.asarray(s)
    if s.dtype != np.float32:
        raise TypeError("%s must be float32" % name)
    return s


def gemm_ref(qa, sa, qb, sb, b_kmajor=True, sb_transposed=False, want_t=True):
    """fp64 block-scaled GEMM reference.

    qa [M,K] uint8 with sa [M,K/128]; qb [N,K] (b_kmajor) or [K,N] with sb
    [K/128, N/128] (or, when ``sb_transposed``, sb stored [N/128, K/128]).
    Returns (C_ref [M,N] float64, T [M,N] float64 or None).
    """
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(_scales(sa, "sa"))
    sb = np.ascontiguousarray(_scales(sb, "sb"))
    M, K = qa.shape
    N = qb.shape[0] if b_kmajor else qb.shape[1]
    ldb = qb.shape[1]
    if sb_transposed:
        sb_skb, sb_snb = 1, sb.shape[1]
    else:
        sb_skb, sb_snb = sb.shape[1], 1
    C = np.empty((M, N), dtype=np.float64)
    T = np.empty((M, N), dtype=np.float64) if want_t else None
    lib().orc_gemm_ref(_p(qa), K, _p(sa), sa.shape[1], 1, _p(qb), ldb, int(bool(b_kmajor)),
                       _p(sb), sb_skb, sb_snb, M, N, K, _p(C), _p(T))
    return C, T


def gemm_ref_entries(qa, sa, qb, sb, rows, cols, b_kmajor=True, sb_transposed=False):
    """Selected entries C_ref[rows[i], cols[i]] and T of the same, in fp64."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(_scales(sa, "sa"))
    sb = np.ascontiguousarray(_scales(sb, "sb"))
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    K = qa.shape[1]
    ldb = qb.shape[1]
    if sb_transposed:
        sb_skb, sb_snb = 1, sb.shape[1]
    else:
        sb_skb, sb_snb = sb.shape[1], 1
    C = np.empty(rows.shape, dtype=np.float64)
    T = np.empty(rows.shape, dtype=np.float64)
    lib().orc_gemm_ref_entries(_p(qa), K, _p(sa), sa.shape[1], 1, _p(qb), ldb,
                               int(bool(b_kmajor)), _p(sb), sb_skb, sb_snb, K, rows.size,
                               _p(rows), _p(cols), _p(C), _p(T))
    return C, T


def grouped_gemm_ref(qa, sa, qb, sb, offsets):
    """MoE grouped reference: qb [G,N,K] uint8, sb [G,K/128,N/128], offsets [G+1]."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(_scales(sa, "sa"))
    sb = np.ascontiguousarray(_scales(sb, "sb"))
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    G, N, K = qb.shape
    total = qa.shape[0]
    C = np.zeros((total, N), dtype=np.float64)
    T = np.zeros((total, N), dtype=np.float64)
    lib().orc_grouped_gemm_ref(_p(qa), K, _p(sa), sa.shape[1], 1, _p(qb), K, N * K, _p(sb),
                               sb.shape[1] * sb.shape[2], sb.shape[2], 1, _p(off), G, N, K,
                               _p(C), _p(T))
    return C, T


def gemm_exact(x, w):
    """Unquantized fp64 GEMM x[M,K] @ w[K,N] on the original operands."""
    x, xt = _as_input(x)
    w, wt = _as_input(w)
    M, K = x.shape
    N = w.shape[1]
    E = np.empty((M, N), dtype=np.float64)
    lib().orc_gemm_exact(_p(x), xt, K, _p(w), wt, N, M, N, K, _p(E))
    return E


def dequantize(q, s, tile_rows, tile_cols):
    """q * s per tile ([HS] 2.2 FP8BlockQuantizer.dequantize), fp64.

    s[i, j] scales q[i*tile_rows:(i+1)*tile_rows, j*tile_cols:(j+1)*tile_cols].
    """
    v = e4m3_decode(q)
    s64 = np.asarray(s, dtype=np.float64)
    rs = np.repeat(np.repeat(s64, tile_rows, axis=0), tile_cols, axis=1)
    return v * rs[: v.shape[0], : v.shape[1]]


def dequantize_fp32(q, s, tile_rows, tile_cols=128):
    """The dequantized tensor in fp32: E4M3 value of each code times its
    tile's scale, rounded once to fp32 ([HS] 2.2 dequantize: code value x
    scale, computed in fp32).  The product of a 4-bit E4M3 significand and a
    24-bit fp32 scale is exact in fp64, so rounding the fp64 product to fp32
    is the single correctly rounded fp32 multiply.  Tiles are tile_rows x
    tile_cols (1 x 128 activations, 128 x 128 weights); NaN codes give NaN."""
    return dequantize(q, s, tile_rows, tile_cols).astype(np.float32)


def f32_to_bf16_bits(x):
    """bf16 bit patterns of fp32 values, round to nearest, ties to even (the
    16 high bits after adding 0x7FFF plus the lowest kept bit); NaN stays a
    quiet NaN."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r


def gemm_ref_colscale(qa, sa, qb, sb_cols):
    """Block-scaled GEMM whose B scales are per output column and chunk (the
    weight-gradient product dW = X^T dY, both operands quantized in 1x128
    tiles along the contraction): C[i, n] = sum_k (sa[i, k/128] dec(qa[i, k]))
    (sb_cols[n, k/128] dec(qb[n, k])), in fp64, and T = sum_k |.| of the
    same products.  Each dequantized operand (a 4-bit E4M3 significand times
    a 24-bit fp32 scale) is exact in fp64, but the product of two such
    operands can carry up to 56 significant bits, so it and the sum are
    rounded to fp64: a relative error near 2^-53 per term, far inside the
    1e-3 T acceptance bound
    ([KB] "Ökad ackumuleringsprecision"; [HS] 2.2 dequantize).  qa [I, K],
    qb [N, K] (K-major), sa [I, K/128], sb_cols [N, K/128].
    Returns (C, T) as fp64 [I, N]."""
    A = dequantize(qa, sa, 1, 128)
    B = dequantize(qb, sb_cols, 1, 128)
    return A @ B.T, np.abs(A) @ np.abs(B).T
