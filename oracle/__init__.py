"""CPU oracle for AQLM inference (double precision, plain loops in C).

TEST INFRASTRUCTURE ONLY: tests/, the package smoke() check and the
benchmark's CPU-baseline leg may import this module; the CUDA library and its
Python binding never do.  It shares no code with the CUDA path.

Definitions follow "The AQLM Quantization Algorithm, Explained", section
"What is Multi-Codebook Quantization (MCQ)?" (decode a group as the sum of M
codewords, scale per output channel, multiply with the activations), section
"Memory footprint of AQLM-quantized models" (bits per parameter) and, for the
encoding (aqlm_encode_oracle.c), section "AQLM quantization process"
(codebooks initialised by residual k-means, codes learned with the codebooks
fixed; readings E1-E6 in that file).

Parity pins: tests/test_oracle.py checks every function here against closed
forms, brute force and independent library routines.  No function is
parity-unpinned.

All 16-bit floating inputs (codebooks, scales, activations) are numpy arrays
of dtype float16 (or uint16 bit patterns of bfloat16 with ``is_bf16=True``).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _configure(lib):
    """Declare the C signatures on a loaded oracle library."""
    i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
    lib.aqlm_oracle_decode_indices.argtypes = [vp, i64, i64, i32, i32, i32, vp]
    lib.aqlm_oracle_dequant_f64.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, vp]
    lib.aqlm_oracle_gemv_f64.argtypes = [vp, vp, vp, vp, i32, i64, i64, i64, i32, i32, i32, vp]
    lib.aqlm_oracle_matmul_f64.argtypes = [vp, i64, i64, vp, i64, vp]
    lib.aqlm_oracle_dequant_bf16.argtypes = [vp, vp, vp, i64, i64, i32, i32, i32, vp]
    lib.aqlm_oracle_bits_per_param.argtypes = [i64, i64, i32, i32, i32]
    lib.aqlm_oracle_bits_per_param.restype = ctypes.c_double
    lib.aqlm_oracle_half_to_double.argtypes = [ctypes.c_uint16]
    lib.aqlm_oracle_half_to_double.restype = ctypes.c_double
    lib.aqlm_oracle_float_to_bf16.argtypes = [ctypes.c_float]
    lib.aqlm_oracle_float_to_bf16.restype = ctypes.c_uint16
    lib.aqlm_oracle_num_threads.restype = ctypes.c_int
    # encoding (aqlm_encode_oracle.c)
    lib.aqlm_oracle_double_to_half.argtypes = [ctypes.c_double]
    lib.aqlm_oracle_double_to_half.restype = ctypes.c_uint16
    lib.aqlm_oracle_encode_scales.argtypes = [vp, i64, i64, vp, vp]
    lib.aqlm_oracle_nearest.argtypes = [vp, i64, vp, i64, vp, vp, vp]
    lib.aqlm_oracle_kmeans_update.argtypes = [vp, vp, i64, i64, vp, vp, vp]
    lib.aqlm_oracle_residual_kmeans.argtypes = [vp, i64, i32, i64, vp, i32, vp]
    lib.aqlm_oracle_encode_greedy.argtypes = [vp, i64, vp, i32, i64, vp]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(_build.build()))
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check_codes(codes, d_out, d_in, g, M, B):
    want = np.uint8 if B == 8 else (np.int16, np.uint16)
    if B == 8:
        assert codes.dtype == np.uint8, codes.dtype
    else:
        assert codes.dtype in want, codes.dtype
    assert codes.flags.c_contiguous and codes.size == d_out * (d_in // g) * M


def _c16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype in (np.float16, np.uint16), a.dtype
    return a


def decode_indices(codes, d_out, d_in, g, M, B):
    """uint16 [d_out, d_in/g, M]: the codeword index of every (row, group, codebook)."""
    lib = _load()
    codes = np.ascontiguousarray(codes)
    _check_codes(codes, d_out, d_in, g, M, B)
    out = np.empty((d_out, d_in // g, M), dtype=np.uint16)
    assert lib.aqlm_oracle_decode_indices(_ptr(codes), d_out, d_in, g, M, B, _ptr(out)) == 0
    return out


def dequant_f64(codes, codebooks, scales, d_out, d_in, g, M, B):
    """float64 [d_out, d_in]: W[i, g*j+t] = s_i * sum_m C_m[b(i,j,m)][t]."""
    lib = _load()
    codes = np.ascontiguousarray(codes)
    _check_codes(codes, d_out, d_in, g, M, B)
    cb, sc = _c16(codebooks), _c16(scales)
    assert cb.size == M * (1 << B) * g and sc.size == d_out
    W = np.empty((d_out, d_in), dtype=np.float64)
    assert lib.aqlm_oracle_dequant_f64(_ptr(codes), _ptr(cb), _ptr(sc), d_out, d_in, g, M, B, _ptr(W)) == 0
    return W


def gemv_f64(codes, codebooks, scales, x, d_out, d_in, g, M, B, is_bf16=False):
    """float64 [T, d_out]: y[tau, i] = sum_j <s_i * sum_m C_m[b], x[tau, group j]>.

    ``x`` is [T, d_in] float16, or uint16 bfloat16 bit patterns with is_bf16."""
    lib = _load()
    codes = np.ascontiguousarray(codes)
    _check_codes(codes, d_out, d_in, g, M, B)
    cb, sc = _c16(codebooks), _c16(scales)
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    assert x.shape[1] == d_in and x.dtype in (np.float16, np.uint16)
    T = x.shape[0]
    y = np.empty((T, d_out), dtype=np.float64)
    rc = lib.aqlm_oracle_gemv_f64(_ptr(codes), _ptr(cb), _ptr(sc), _ptr(x), int(is_bf16),
                                  T, d_out, d_in, g, M, B, _ptr(y))
    assert rc == 0
    return y


def matmul_f64(W, X):
    """float64 [T, d_out] = X @ W.T with W [d_out, d_in], X [T, d_in] (plain loops)."""
    lib = _load()
    W = np.ascontiguousarray(W, dtype=np.float64)
    X = np.ascontiguousarray(X, dtype=np.float64)
    if X.ndim == 1:
        X = X[None, :]
    d_out, d_in = W.shape
    assert X.shape[1] == d_in
    Y = np.empty((X.shape[0], d_out), dtype=np.float64)
    assert lib.aqlm_oracle_matmul_f64(_ptr(W), d_out, d_in, _ptr(X), X.shape[0], _ptr(Y)) == 0
    return Y


def dequant_bf16(codes, codebooks, scales, d_out, d_in, g, M, B):
    """uint16 bfloat16 bit patterns [d_out, d_in], binary32 steps then RNE rounding."""
    lib = _load()
    codes = np.ascontiguousarray(codes)
    _check_codes(codes, d_out, d_in, g, M, B)
    cb, sc = _c16(codebooks), _c16(scales)
    W = np.empty((d_out, d_in), dtype=np.uint16)
    assert lib.aqlm_oracle_dequant_bf16(_ptr(codes), _ptr(cb), _ptr(sc), d_out, d_in, g, M, B, _ptr(W)) == 0
    return W


def bits_per_param(d_out, d_in, g, M, B):
    return _load().aqlm_oracle_bits_per_param(d_out, d_in, g, M, B)


def half_to_double(bits):
    return _load().aqlm_oracle_half_to_double(int(bits))


def float_to_bf16(f):
    return _load().aqlm_oracle_float_to_bf16(float(f))


def num_threads():
    return _load().aqlm_oracle_num_threads()


def bf16_bits_to_f64(bits):
    """bfloat16 bit patterns -> float64 (the upper half of a binary32)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- encoding
# "The AQLM Quantization Algorithm, Explained", section "AQLM quantization
# process": codes are learned with fixed codebooks and scales, the codebooks
# initialised by residual k-means.  Readings E1-E6 are stated in
# aqlm_encode_oracle.c.

def _f32(a, cols=None):
    a = np.ascontiguousarray(a, dtype=np.float32)
    if cols is not None:
        assert a.size % cols == 0
    return a


def double_to_half(x):
    """binary16 bits of a real number, round to nearest even."""
    return _load().aqlm_oracle_double_to_half(float(x))


def encode_scales(W):
    """E1, E2: (scales float16 [d_out], groups float32 [d_out * d_in / 8, 8])."""
    W = _f32(W)
    d_out, d_in = W.shape
    sc = np.empty(d_out, dtype=np.uint16)
    V = np.empty((d_out * d_in // 8, 8), dtype=np.float32)
    assert _load().aqlm_oracle_encode_scales(_ptr(W), d_out, d_in, _ptr(sc), _ptr(V)) == 0
    return sc.view(np.float16), V


def nearest(V, C):
    """E3: (index int32 [N], distance float64 [N], runner-up distance float64
    [N]) of each group's nearest codeword by the squared Euclidean distance in
    double, ties to the lowest index."""
    V, C = _f32(V, 8), _f32(C, 8)
    N, K = V.size // 8, C.size // 8
    idx = np.empty(N, dtype=np.int32)
    dist = np.empty(N, dtype=np.float64)
    second = np.empty(N, dtype=np.float64)
    assert _load().aqlm_oracle_nearest(_ptr(V), N, _ptr(C), K, _ptr(idx), _ptr(dist), _ptr(second)) == 0
    return idx, dist, second


def kmeans_update(V, idx, C_prev):
    """E4: (centroids float32 [K, 8], counts int64 [K])."""
    V, C_prev = _f32(V, 8), _f32(C_prev, 8)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    N, K = V.size // 8, C_prev.size // 8
    C = np.empty((K, 8), dtype=np.float32)
    counts = np.empty(K, dtype=np.int64)
    assert _load().aqlm_oracle_kmeans_update(_ptr(V), _ptr(idx), N, K, _ptr(C_prev), _ptr(C), _ptr(counts)) == 0
    return C, counts


def residual_kmeans(V, M, K, init_idx, iters):
    """E5: codebooks float32 [M, K, 8]."""
    V = _f32(V, 8)
    init_idx = np.ascontiguousarray(init_idx, dtype=np.int32)
    assert init_idx.size == M * K
    C = np.empty((M, K, 8), dtype=np.float32)
    assert _load().aqlm_oracle_residual_kmeans(_ptr(V), V.size // 8, M, K, _ptr(init_idx), iters, _ptr(C)) == 0
    return C


def encode_greedy(V, codebooks):
    """E6: codes uint16 [N, M] against float16 codebooks [M, K, 8]."""
    V = _f32(V, 8)
    cb = _c16(codebooks)
    M, K = cb.shape[0], cb.shape[1]
    codes = np.empty((V.size // 8, M), dtype=np.uint16)
    assert _load().aqlm_oracle_encode_greedy(_ptr(V), V.size // 8, _ptr(cb), M, K, _ptr(codes)) == 0
    return codes

