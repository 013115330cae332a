"""Validity checks for results of the encoding path that carry rounding error.

Section "AQLM quantization process" of "The AQLM Quantization Algorithm,
Explained" initialises the codebooks by residual k-means and learns the codes
with the codebooks fixed; the readings E1-E6 are stated in
oracle/aqlm_encode_oracle.c.  The oracle evaluates each definition plainly in
double.  A GPU result is compared with it through an error bound derived
below, never through a copy of the GPU's evaluation order, so the kernels may
order their arithmetic as they like.

E1 (row scale, binary16 of the root mean square).  A sum of n non-negative
doubles in any order has relative error at most gamma_n (u = 2^-53), the
division by d_in and the square root add one rounding each and halve nothing
away, so any evaluation lies within eps = (d_in + 4) 2^-53 of the true root
mean square, and so does the oracle's.  The binary16 scale must therefore be
one of the roundings of [rms (1 - 2 eps), rms (1 + 2 eps)] -- the same value
as the oracle's except where that interval holds a rounding boundary.

E3 (nearest codeword, least |v - c|^2, ties to the lowest index).  A binary32
implementation ranks codewords by score(v, c) = |c|^2 - 2 <v, c>, the terms
common to every codeword left out.  Each 8-term sum computed in binary32, in
any order and with or without fused multiply-adds, has error at most
gamma_8 times the sum of its terms' magnitudes, and the final combination adds
one rounding (Higham, "Accuracy and Stability of Numerical Algorithms", 2nd
ed., section 3.1), so
    |score_f32(c) - score(c)| <= beta(c) = gamma_9 (|c|^2 + 2 sum_t |v_t c_t|),
    gamma_n = n u / (1 - n u), u = 2^-24.
A codeword k chosen by least binary32 score therefore satisfies
    d(k) - d_min <= beta(k) + beta(k_min),
d the exact squared distance; and where the two least distances differ by
more than 2 max_k beta(k) (bounded with Cauchy-Schwarz by
2 gamma_9 (max |c|^2 + 2 |v| max |c|)), only the nearest codeword passes.
The distance a binary32 implementation reports for its choice (eight rounded
differences, squared and summed) is within gamma_10 of the exact one.
"""
import numpy as np

import oracle

U32 = 2.0 ** -24
U64 = 2.0 ** -53


def gamma(n, u=U32):
    return n * u / (1 - n * u)


def distances(V, C, idx):
    """Squared distances |v_n - c_idx[n]|^2 in double (float64 [N])."""
    d = np.asarray(V, dtype=np.float64).reshape(-1, 8) - np.asarray(C, dtype=np.float64).reshape(-1, 8)[idx]
    return (d * d).sum(1)


def score_bound(V, C, idx):
    """beta(c_idx[n]) for each group n: the binary32 score's error bound."""
    v = np.asarray(V, dtype=np.float64).reshape(-1, 8)
    c = np.asarray(C, dtype=np.float64).reshape(-1, 8)[idx]
    return gamma(9) * ((c * c).sum(1) + 2 * np.abs(v * c).sum(1))


def check_nearest(V, C, idx, dist=None, what="nearest codeword"):
    """Assert that idx (one codeword index per group of V) is a valid nearest
    codeword choice under reading E3 with the binary32 bound above, exact
    wherever the choice is clear; if dist is given, that it is the chosen
    codeword's distance within gamma_10.  Returns the number of groups whose
    index differs from the oracle's (near ties)."""
    V = np.ascontiguousarray(V, dtype=np.float32).reshape(-1, 8)
    C = np.ascontiguousarray(C, dtype=np.float32).reshape(-1, 8)
    idx = np.asarray(idx).astype(np.int64)
    assert idx.shape == (V.shape[0],), f"{what}: {idx.shape} indices for {V.shape[0]} groups"
    assert ((idx >= 0) & (idx < C.shape[0])).all(), f"{what}: index out of range"
    idx_ref, d_min, second = oracle.nearest(V, C)
    idx_ref = idx_ref.astype(np.int64)
    d_got = distances(V, C, idx)
    v2 = (V.astype(np.float64) ** 2).sum(1)
    c2 = (C.astype(np.float64) ** 2).sum(1)
    slack = 2.0 ** -40 * (v2 + c2.max())          # double rounding of the two distance evaluations
    allowed = score_bound(V, C, idx) + score_bound(V, C, idx_ref) + slack
    bad = np.flatnonzero(d_got - d_min > allowed)
    assert bad.size == 0, (f"{what}: {bad.size} choices farther than the bound allows, e.g. group {bad[0]}: "
                           f"index {idx[bad[0]]} at {d_got[bad[0]]!r}, nearest {idx_ref[bad[0]]} at {d_min[bad[0]]!r}, "
                           f"bound {allowed[bad[0]]!r}")
    uniform = 2 * gamma(9) * (c2.max() + 2 * np.sqrt(v2) * np.sqrt(c2.max())) + slack
    clear = second - d_min > uniform
    wrong = np.flatnonzero(clear & (idx != idx_ref))
    assert wrong.size == 0, f"{what}: {wrong.size} clear choices differ from the nearest, e.g. group {wrong[0]}"
    if dist is not None:
        dist = np.asarray(dist, dtype=np.float64)
        err = np.abs(dist - d_got)
        assert (err <= gamma(10) * d_got + 2.0 ** -126).all(), f"{what}: reported distance off by {err.max()!r}"
    return int((idx != idx_ref).sum())


def half_round(x):
    """binary16 of float64 values, round to nearest even (numpy's conversion)."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float16)


def _scale_of(h):
    out = h.copy()
    out[out.view(np.uint16) & 0x7FFF == 0] = np.float16(1.0)
    return out


def check_scales(W, scales):
    """Assert reading E1 through the bound above: each binary16 scale is a
    rounding of the row's root mean square within the evaluation error (the
    oracle's value wherever no rounding boundary lies inside it), 1.0 where
    that rounds to zero.  Returns the number of rows that differ from the
    oracle's scale."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    d_in = W.shape[1]
    scales = np.asarray(scales).astype(np.float16)
    ref, _ = oracle.encode_scales(W)
    W64 = W.astype(np.float64)
    rms = np.sqrt((W64 * W64).sum(1) / d_in)
    eps = 2 * (d_in + 4) * U64
    lo, hi = _scale_of(half_round(rms * (1 - eps))), _scale_of(half_round(rms * (1 + eps)))
    b, l, h, r = (a.view(np.uint16) for a in (scales, lo, hi, ref))
    assert ((r == l) | (r == h)).all(), "the oracle's scale is outside its own error interval"
    assert ((b == l) | (b == h)).all(), f"scales outside the rounding interval: rows {np.flatnonzero((b != l) & (b != h))[:5]}"
    assert np.array_equal(b[l == h], r[l == h]), "a scale differs from the oracle's where the rounding is clear"
    return int((b != r).sum())


def check_groups(W, scales, V):
    """Reading E2: the groups are the row's values divided by the row's own
    binary16 scale, one correctly rounded binary32 division each (numpy)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    s = np.asarray(scales).astype(np.float16).astype(np.float32)
    want = (W / s[:, None]).reshape(-1, 8)
    assert np.array_equal(np.asarray(V, dtype=np.float32).reshape(-1, 8).view(np.uint32), want.view(np.uint32))


def check_greedy(V, codebooks, codes, what="greedy codes"):
    """Reading E6 carried through on the implementation's own choices: for
    codebook m = 0, 1, ... the code of every group is a valid nearest codeword
    (check_nearest) of the residual its earlier codes left, the residual then
    losing that codeword (binary32 subtraction, numpy).  Returns the number of
    near-tie choices that differ from the oracle's."""
    V = np.ascontiguousarray(V, dtype=np.float32).reshape(-1, 8)
    cb = np.asarray(codebooks).astype(np.float16)
    M = cb.shape[0]
    codes = np.asarray(codes).reshape(V.shape[0], M).astype(np.int64)
    R = V.copy()
    ties = 0
    for m in range(M):
        Cm = cb[m].astype(np.float32)
        ties += check_nearest(R, Cm, codes[:, m], what=f"{what}, codebook {m}")
        R = (R - Cm[codes[:, m]]).astype(np.float32)
    return ties
