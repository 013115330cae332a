"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each pin raises AssertionError when the oracle disagrees with
  - a closed form stated by "The AQLM Quantization Algorithm, Explained"
    (section "What is Multi-Codebook Quantization (MCQ)?": a group is the sum
    of M codewords picked by B-bit indices, scaled per output channel;
    section "Memory footprint of AQLM-quantized models": the three storage
    terms; section "AQLM Performance": 14 GB -> 1.75 GB at 2 bits),
  - an independent routine (numpy float16 conversion, numpy BLAS float64
    matmul, torch's bfloat16 rounding, numpy float32 arithmetic), or
  - brute force written here in pure Python on tiny inputs.

They are plain functions so that tests/test_oracle_mutants.py can run them
against deliberately broken copies of the oracle and show that each planted
mistake is caught.
"""
import itertools
import json
import os

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
FORMATS = [(1, 16), (2, 8), (2, 16)]


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _random_codes(rng, d_out, groups, M, B):
    if B == 8:
        return rng.integers(0, 256, size=(d_out, groups, M), dtype=np.uint8)
    return rng.integers(0, 65536, size=(d_out, groups, M), dtype=np.uint16).view(np.int16)


def _index_encoding_codebooks(M, B):
    """Codebooks whose decoded group spells out the codes in base 16.

    Codebook m writes the B/4 hex digits of its index k into its own disjoint
    block of lanes, lanes m*B/4 .. m*B/4 + B/4 - 1, and zero elsewhere.  All
    values are integers below 16, exact in fp16 and bf16."""
    K, g = 1 << B, 8
    nib = B // 4
    assert M * nib <= g
    C = np.zeros((M, K, g), dtype=np.float16)
    k = np.arange(K)
    for m in range(M):
        for d in range(nib):
            C[m, :, m * nib + d] = (k >> (4 * d)) & 0xF
    return C


def _read_index_encoding(W, M, B):
    """Inverse of the encoding above: W [d_out, d_in] -> codes [d_out, G, M]."""
    d_out, d_in = W.shape
    nib = B // 4
    Wg = np.rint(W).astype(np.int64).reshape(d_out, d_in // 8, 8)
    codes = np.zeros((d_out, d_in // 8, M), dtype=np.int64)
    for m in range(M):
        for d in range(nib):
            codes[..., m] += Wg[..., m * nib + d] << (4 * d)
    return codes


# --------------------------------------------------------------------------

def pin_half_conversion():
    """All 65536 binary16 patterns decode to numpy's float16 -> float64 value."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    # the oracle's own conversion, reached through a one-column dequant
    C = bits.view(np.float16).reshape(1, 65536, 1).repeat(8, axis=2)  # [1][65536][8]
    codes = np.arange(65536, dtype=np.uint16).view(np.int16).reshape(65536, 1, 1)
    scales = np.ones(65536, dtype=np.float16)
    W = oracle.dequant_f64(codes, C, scales, 65536, 8, 8, 1, 16)[:, 0]
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(W), nan)
    assert np.array_equal(W[~nan], ref[~nan])
    for b in (0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0x8001, 0xFC00):
        assert oracle.half_to_double(b) == np.uint16(b).view(np.float16).astype(np.float64)


def pin_bf16_rounding():
    """binary32 -> bf16 RNE equals torch's conversion, ties and specials included."""
    rng = _rng(5)
    f = rng.normal(0, 1, 20000).astype(np.float32)
    u = f.view(np.uint32)
    ties = ((u & 0xFFFF0000) | 0x8000).view(np.float32)           # exact ties
    special = np.array([0.0, -0.0, np.inf, -np.inf, 3.3895314e38, -3.3895314e38,
                        1e-40, -1e-40, 1.0 + 2**-8, 1.0 + 3 * 2**-8], dtype=np.float32)
    for arr in (f[:2000], ties[:2000], special):
        ref = torch.from_numpy(arr).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        got = np.array([oracle.float_to_bf16(v) for v in arr], dtype=np.uint16)
        assert np.array_equal(got, ref), (arr[got != ref][:4], got[got != ref][:4], ref[got != ref][:4])
    assert np.isnan(oracle.bf16_bits_to_f64([oracle.float_to_bf16(float("nan"))])[0])


def pin_decode_indices():
    """Indices are the stored codes, unsigned, in [d_out][G][M] order."""
    for M, B in FORMATS:
        rng = _rng(11 + B + M)
        codes = _random_codes(rng, 7, 5, M, B)
        idx = oracle.decode_indices(codes, 7, 40, 8, M, B)
        want = codes.view(np.uint8 if B == 8 else np.uint16).astype(np.uint16)
        assert idx.dtype == np.uint16 and np.array_equal(idx, want)
    edge = np.array([0, 1, 32767, -32768, -1], dtype=np.int16).reshape(5, 1, 1)
    idx = oracle.decode_indices(edge, 5, 8, 8, 1, 16)
    assert idx.ravel().tolist() == [0, 1, 32767, 32768, 65535]


def pin_index_encoding_recovers_codes():
    """Decoding with index-spelling codebooks and s = 1 returns the codes."""
    for M, B in FORMATS:
        rng = _rng(21 + M * B)
        d_out, d_in = 9, 48
        codes = _random_codes(rng, d_out, d_in // 8, M, B)
        C = _index_encoding_codebooks(M, B)
        s = np.ones(d_out, dtype=np.float16)
        W = oracle.dequant_f64(codes, C, s, d_out, d_in, 8, M, B)
        got = _read_index_encoding(W, M, B)
        want = codes.view(np.uint8 if B == 8 else np.uint16).astype(np.int64)
        assert np.array_equal(got, want)
        Wb = oracle.bf16_bits_to_f64(oracle.dequant_bf16(codes, C, s, d_out, d_in, 8, M, B))
        assert np.array_equal(Wb, W)


def pin_one_hot_activation():
    """A one-hot x picks one column of the scaled decoded weight, exactly."""
    for M, B in FORMATS:
        rng = _rng(31 + M * B)
        d_out, d_in = 6, 32
        codes = _random_codes(rng, d_out, d_in // 8, M, B)
        C = rng.normal(0, 0.02, size=(M, 1 << B, 8)).astype(np.float16)
        s = rng.uniform(0.5, 1.5, d_out).astype(np.float16)
        W = oracle.dequant_f64(codes, C, s, d_out, d_in, 8, M, B)
        for c in (0, 7, 8, 31):
            x = np.zeros((1, d_in), dtype=np.float16)
            x[0, c] = 1.0
            y = oracle.gemv_f64(codes, C, s, x, d_out, d_in, 8, M, B)
            assert np.array_equal(y[0], W[:, c])
        # sign and magnitude of the scale: s = -2 doubles and flips the column
        s2 = np.full(d_out, -2.0, dtype=np.float16)
        W2 = oracle.dequant_f64(codes, C, s2, d_out, d_in, 8, M, B)
        W1 = oracle.dequant_f64(codes, C, np.ones(d_out, np.float16), d_out, d_in, 8, M, B)
        assert np.array_equal(W2, -2.0 * W1)


def pin_linearity():
    """decode(C + C') = decode(C) + decode(C') and decode(alpha*s) = alpha*decode(s),
    with dyadic values that every step represents exactly."""
    for M, B in FORMATS:
        rng = _rng(41 + M * B)
        d_out, d_in = 5, 24
        codes = _random_codes(rng, d_out, d_in // 8, M, B)
        C1 = (rng.integers(-64, 64, size=(M, 1 << B, 8)) / 16).astype(np.float16)
        C2 = (rng.integers(-64, 64, size=(M, 1 << B, 8)) / 16).astype(np.float16)
        s = (rng.integers(1, 32, size=d_out) / 8).astype(np.float16)
        W1 = oracle.dequant_f64(codes, C1, s, d_out, d_in, 8, M, B)
        W2 = oracle.dequant_f64(codes, C2, s, d_out, d_in, 8, M, B)
        W12 = oracle.dequant_f64(codes, (C1 + C2).astype(np.float16), s, d_out, d_in, 8, M, B)
        assert np.array_equal(W12, W1 + W2)
        W4 = oracle.dequant_f64(codes, C1, (s * 4).astype(np.float16), d_out, d_in, 8, M, B)
        assert np.array_equal(W4, 4 * W1)
        x = (rng.integers(-8, 8, size=(2, d_in)) / 4).astype(np.float16)
        y1 = oracle.gemv_f64(codes, C1, s, x, d_out, d_in, 8, M, B)
        y2 = oracle.gemv_f64(codes, C2, s, x, d_out, d_in, 8, M, B)
        y12 = oracle.gemv_f64(codes, (C1 + C2).astype(np.float16), s, x, d_out, d_in, 8, M, B)
        assert np.array_equal(y12, y1 + y2)


def pin_dense_special_case():
    """1x16 with codes i*G + j and codebook rows = the groups of a dense fp16 W:
    the layer is exactly the dense product (s . W) x, checked with numpy BLAS."""
    rng = _rng(51)
    d_out, d_in = 256, 512
    G = d_in // 8
    Wd = rng.normal(0, 0.02, size=(d_out, d_in)).astype(np.float16)
    C = np.zeros((1, 65536, 8), dtype=np.float16)
    C[0, : d_out * G] = Wd.reshape(d_out * G, 8)
    codes = np.arange(d_out * G, dtype=np.uint16).view(np.int16).reshape(d_out, G, 1)
    s = rng.uniform(0.5, 1.5, d_out).astype(np.float16)
    x = rng.normal(0, 1, size=(3, d_in)).astype(np.float16)
    W = oracle.dequant_f64(codes, C, s, d_out, d_in, 8, 1, 16)
    dense = s.astype(np.float64)[:, None] * Wd.astype(np.float64)
    assert np.array_equal(W, dense)
    y = oracle.gemv_f64(codes, C, s, x, d_out, d_in, 8, 1, 16)
    ref = x.astype(np.float64) @ dense.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-13)
    ref32 = (torch.from_numpy(x.astype(np.float32)) @ torch.from_numpy(dense.astype(np.float32)).T).numpy()
    assert np.allclose(y, ref32, rtol=1e-4, atol=1e-4)


def _brute_dense(codes, C, s, d_out, d_in, M, B):
    """Pure-Python decode, one weight at a time."""
    raw = codes.view(np.uint8 if B == 8 else np.uint16)
    W = [[0.0] * d_in for _ in range(d_out)]
    for i in range(d_out):
        for c in range(d_in):
            j, t = divmod(c, 8)
            acc = 0.0
            for m in range(M):
                acc += float(C[m, int(raw[i, j, m]), t])
            W[i][c] = float(s[i]) * acc
    return W


def pin_brute_force_tiny():
    """Grouped oracle == pure-Python decode + triple loop, on tiny layers."""
    for (M, B), (d_out, d_in), T in itertools.product(FORMATS, [(1, 8), (3, 16), (8, 32)], [1, 3]):
        rng = _rng(61 + M * B + d_out + T)
        codes = _random_codes(rng, d_out, d_in // 8, M, B)
        C = rng.normal(0, 0.02, size=(M, 1 << B, 8)).astype(np.float16)
        s = rng.uniform(-1.5, 1.5, d_out).astype(np.float16)
        x = rng.normal(0, 1, size=(T, d_in)).astype(np.float16)
        Wb = _brute_dense(codes, C, s, d_out, d_in, M, B)
        yb = [[sum(Wb[i][k] * float(x[tau, k]) for k in range(d_in)) for i in range(d_out)]
              for tau in range(T)]
        y = oracle.gemv_f64(codes, C, s, x, d_out, d_in, 8, M, B)
        W = oracle.dequant_f64(codes, C, s, d_out, d_in, 8, M, B)
        assert np.allclose(W, np.array(Wb), rtol=1e-12, atol=0)
        assert np.allclose(y, np.array(yb), rtol=1e-12, atol=1e-15)
        # and the two-step path: dense decode, then the plain matmul
        y2 = oracle.matmul_f64(W, x.astype(np.float64))
        assert np.allclose(y2, np.array(yb), rtol=1e-12, atol=1e-15)


def pin_bf16_activations():
    """With is_bf16 the activations are read as bfloat16 bit patterns."""
    rng = _rng(71)
    d_out, d_in = 4, 16
    codes = _random_codes(rng, d_out, 2, 2, 8)
    C = rng.normal(0, 0.02, size=(2, 256, 8)).astype(np.float16)
    s = rng.uniform(0.5, 1.5, d_out).astype(np.float16)
    xf = rng.normal(0, 1, size=(2, d_in)).astype(np.float32)
    xb = torch.from_numpy(xf).to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    y = oracle.gemv_f64(codes, C, s, bits, d_out, d_in, 8, 2, 8, is_bf16=True)
    W = oracle.dequant_f64(codes, C, s, d_out, d_in, 8, 2, 8)
    ref = xb.to(torch.float64).numpy() @ W.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-15)


def pin_matmul():
    rng = _rng(81)
    W = rng.normal(size=(37, 53))
    X = rng.normal(size=(5, 53))
    assert np.allclose(oracle.matmul_f64(W, X), X @ W.T, rtol=1e-12, atol=1e-12)


def pin_dequant_bf16_binary32_steps():
    """The bf16 restatement equals numpy binary32 arithmetic (add, then multiply,
    each rounded) followed by torch's RNE bf16 rounding, bit for bit."""
    for M, B in FORMATS:
        rng = _rng(91 + M * B)
        d_out, d_in = 33, 64
        codes = _random_codes(rng, d_out, d_in // 8, M, B)
        C = rng.normal(0, 0.02, size=(M, 1 << B, 8)).astype(np.float16)
        C[0, :7, 0] = [0.0, -0.0, 6.1e-5, -6.1e-5, 65504, 1e-7, -1e-7]     # specials
        s = rng.uniform(-1.5, 1.5, d_out).astype(np.float16)
        s[:3] = [1.0, -1.0, 0.5]
        raw = codes.view(np.uint8 if B == 8 else np.uint16).astype(np.int64)
        f = C[0].astype(np.float32)[raw[..., 0]]                 # [d_out][G][8]
        for m in range(1, M):
            f = (f + C[m].astype(np.float32)[raw[..., m]]).astype(np.float32)
        w = (f * s.astype(np.float32)[:, None, None]).astype(np.float32).reshape(d_out, d_in)
        ref = torch.from_numpy(w).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        got = oracle.dequant_bf16(codes, C, s, d_out, d_in, 8, M, B)
        assert np.array_equal(got, ref)


def pin_bits_per_parameter():
    """The bit rate equals the stored buffers' size, the values recomputed by hand
    in tests/golden/bits_per_param.json, and the 2-bit footprint example."""
    with open(os.path.join(GOLDEN, "bits_per_param.json")) as fh:
        gold = json.load(fh)
    for row in gold["layers"]:
        d_out, d_in, M, B = row["d_out"], row["d_in"], row["M"], row["B"]
        bpp = oracle.bits_per_param(d_out, d_in, 8, M, B)
        assert abs(bpp - row["bits_per_param"]) < 5e-5, (row, bpp)
        # the same quantity from the size of the buffers the format stores
        code_bytes = d_out * (d_in // 8) * M * B // 8
        codebook_bytes = M * (1 << B) * 8 * 2
        scale_bytes = d_out * 2
        assert abs(bpp - 8 * (code_bytes + codebook_bytes + scale_bytes) / (d_out * d_in)) < 1e-12
        # the code term alone is M*B/g
        assert bpp > M * B / 8
    fp = gold["footprint_example"]
    params = fp["params"]
    code_term = 1 * 16 / 8          # 2-bit formats: M*B/g = 2
    assert params * 16 / 8 / 1e9 == fp["fp16_gb"]
    assert params * code_term / 8 / 1e9 == fp["quantized_gb"]


def pin_worked_example():
    """A tiny hand-computed layer (tests/golden/worked_example_2x8.json)."""
    with open(os.path.join(GOLDEN, "worked_example_2x8.json")) as fh:
        ex = json.load(fh)
    C = np.zeros((2, 256, 8), dtype=np.float16)
    for m, k, vals in ex["codebook_entries"]:
        C[m, k] = vals
    codes = np.array(ex["codes"], dtype=np.uint8)
    s = np.array(ex["scales"], dtype=np.float16)
    x = np.array(ex["x"], dtype=np.float16)
    d_out, d_in = len(s), x.shape[1]
    W = oracle.dequant_f64(codes, C, s, d_out, d_in, 8, 2, 8)
    assert np.array_equal(W, np.array(ex["expected_W"], dtype=np.float64))
    y = oracle.gemv_f64(codes, C, s, x, d_out, d_in, 8, 2, 8)
    assert np.array_equal(y, np.array(ex["expected_y"], dtype=np.float64))


# --------------------------------------------------------------------------- encoding
# Section "AQLM quantization process": codebooks initialised by residual
# k-means, codes learned with the codebooks fixed.  Readings E1-E6 are in
# oracle/aqlm_encode_oracle.c.

def pin_double_to_half():
    """Rounding to binary16 agrees with numpy's float64 -> float16 conversion:
    every binary16 value, the midpoints between neighbours (ties to even),
    values just off the midpoints, the subnormal range and overflow."""
    every = np.arange(65536, dtype=np.uint16).view(np.float16)
    finite = every[np.isfinite(every)].astype(np.float64)
    pos = np.unique(finite[finite >= 0])
    mids = (pos[:-1] + pos[1:]) / 2
    probes = np.concatenate([finite, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                             [65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -26, 0.0, -0.0],
                             _rng(5).standard_normal(4000) * np.exp(_rng(6).uniform(-18, 11, 4000))])
    with np.errstate(over="ignore"):
        want = probes.astype(np.float16).view(np.uint16)
    got = np.array([oracle.double_to_half(v) for v in probes], dtype=np.uint16)
    assert np.array_equal(got, want), np.flatnonzero(got != want)[:5]


def pin_encode_scales():
    """E1/E2: the scale is the row's root mean square rounded to binary16
    (numpy float64 statistics, numpy rounding), 1.0 for an all-zero row, and
    the groups are the row's values divided by it (numpy float32 division)."""
    rng = _rng(21)
    W = (rng.standard_normal((40, 256)) * rng.uniform(0.01, 3.0, (40, 1))).astype(np.float32)
    W[7] = 0.0
    sc, V = oracle.encode_scales(W)
    rms = np.sqrt((W.astype(np.float64) ** 2).mean(axis=1)).astype(np.float16)
    rms[7] = 1.0
    assert np.array_equal(sc.view(np.uint16), rms.view(np.uint16))
    want = (W / sc.astype(np.float32)[:, None]).reshape(-1, 8)
    assert np.array_equal(V, want)


def _brute_nearest(V, C):
    d = ((V.astype(np.float64)[:, None, :] - C.astype(np.float64)[None, :, :]) ** 2).sum(-1)
    return d


def pin_nearest_codeword():
    """E3 against float64 brute force on small inputs: the chosen codeword's
    distance is the least one (to within double rounding), the index is the
    brute-force argmin wherever the two nearest differ by more than double
    rounding, and the reported distance and runner-up distance are the
    brute-force smallest and second smallest; a group equal to a codeword gets
    it at distance 0; a group exactly midway between two codewords (dyadic
    values, so both distances are exact) and duplicated codewords resolve to
    the lowest index."""
    rng = _rng(22)
    C = rng.standard_normal((300, 8)).astype(np.float32)
    V = rng.standard_normal((500, 8)).astype(np.float32)
    V[:50] = C[rng.integers(0, 300, 50)]
    idx, dist, second = oracle.nearest(V, C)
    d = _brute_nearest(V, C)
    srt = np.sort(d, axis=1)
    rows = np.arange(len(V))
    assert np.all(d[rows, idx] <= srt[:, 0] * (1 + 1e-12))
    clear = srt[:, 1] - srt[:, 0] > 1e-9 * srt[:, 1]
    assert clear.mean() > 0.99
    assert np.array_equal(idx[clear], d.argmin(axis=1)[clear])
    assert np.allclose(dist, srt[:, 0], rtol=1e-12, atol=0)
    assert np.allclose(second, srt[:, 1], rtol=1e-12, atol=0)
    assert np.all(dist[:50] == 0)
    # duplicates: codewords 10 and 20 equal, a group equal to them -> 10
    C2 = C.copy()
    C2[20] = C2[10]
    i2, d2, s2 = oracle.nearest(C2[10:11] + np.float32(0), C2)
    assert i2[0] == 10 and d2[0] == 0 and s2[0] == 0
    i3, _, _ = oracle.nearest(C2[20:21], C2[::-1].copy())
    assert i3[0] == 300 - 1 - 20
    # exact midpoint: v = 0.25 * (1, -1, 0, ...), codewords v + e at 7 and v - e at 3 (e dyadic)
    v = np.zeros((1, 8), dtype=np.float32)
    v[0, :2] = [0.25, -0.25]
    e = np.array([0.5, 0.25, -0.125, 0, 0, 0, 0.0625, 0], dtype=np.float32)
    C3 = np.full((9, 8), 4.0, dtype=np.float32)
    C3[7], C3[3] = v[0] + e, v[0] - e
    i4, d4, s4 = oracle.nearest(v, C3)
    assert i4[0] == 3 and d4[0] == s4[0] == float((e.astype(np.float64) ** 2).sum())


def pin_kmeans_update():
    """E4: centroids are the float64 means of their groups rounded to float32
    (numpy, summing in the same order), counts exact, empty clusters keep
    their previous value."""
    rng = _rng(23)
    V = rng.standard_normal((1000, 8)).astype(np.float32)
    K = 40
    idx = rng.integers(0, K - 5, 1000).astype(np.int32)   # the last 5 clusters stay empty
    C_prev = rng.standard_normal((K, 8)).astype(np.float32)
    C, counts = oracle.kmeans_update(V, idx, C_prev)
    assert np.array_equal(counts, np.bincount(idx, minlength=K))
    sums = np.zeros((K, 8), dtype=np.float64)
    np.add.at(sums, idx, V.astype(np.float64))
    want = C_prev.copy()
    nz = counts > 0
    want[nz] = (sums[nz] / counts[nz, None]).astype(np.float32)
    assert np.array_equal(C, want)


def pin_residual_kmeans_recovers_clusters():
    """E5 closed forms: data drawn around K well-separated centres, started
    from one member of each cluster, converge to the cluster means; the second
    codebook (of residuals) is the k-means of the small offsets, and adding
    it never raises the squared error of the codebook-0 approximation."""
    rng = _rng(24)
    K, per = 12, 40
    centres = (rng.standard_normal((K, 8)) * 10).astype(np.float32)
    lab = np.repeat(np.arange(K), per)
    V = (centres[lab] + rng.standard_normal((K * per, 8)).astype(np.float32) * 0.05).astype(np.float32)
    perm = rng.permutation(K * per)
    V, lab = V[perm], lab[perm]
    first = np.array([np.flatnonzero(lab == k)[0] for k in range(K)], dtype=np.int32)
    init = np.stack([first, rng.choice(K * per, K, replace=False).astype(np.int32)])
    C = oracle.residual_kmeans(V, 2, K, init, iters=4)
    means = np.stack([V[lab == k].astype(np.float64).mean(0) for k in range(K)])
    assert np.allclose(C[0], means, atol=1e-5)
    d0 = _brute_nearest(V, C[0])
    i0 = d0.argmin(1)
    R = V - C[0][i0]
    e1 = (R.astype(np.float64) ** 2).sum()
    i1 = _brute_nearest(R, C[1]).argmin(1)
    e2 = ((R - C[1][i1]).astype(np.float64) ** 2).sum()
    assert e2 <= e1 and np.abs(C[1]).max() < 0.5


def pin_greedy_codes_recover_sums():
    """E6 closed form: with codebook 0 on a coarse grid and codebook 1 of
    small offsets (all binary16-exact), a group that is exactly C0[b0] + C1[b1]
    is encoded as (b0, b1); with one codebook a group equal to a codeword gets
    its index (brute force agrees on random groups where the choice is clear)."""
    rng = _rng(25)
    K0, K1 = 64, 16
    C0 = (rng.integers(-8, 8, (K0, 8)) * 4).astype(np.float16)
    C0[1:] += (np.arange(1, K0)[:, None] % 4 == 0) * np.float16(1)    # distinct rows
    C0 = np.unique(C0, axis=0)[:32]
    C1 = (rng.integers(-3, 4, (K1, 8)) / 16).astype(np.float16)
    C1 = np.unique(C1, axis=0)
    k0, k1 = len(C0), len(C1)
    b0 = rng.integers(0, k0, 400)
    b1 = rng.integers(0, k1, 400)
    V = (C0[b0].astype(np.float32) + C1[b1].astype(np.float32))
    cb = np.zeros((2, max(k0, k1), 8), dtype=np.float16)
    cb[0, :k0], cb[1, :k1] = C0, C1
    cb[1, k1:] = np.float16(1000)                     # padding never chosen
    cb[0, k0:] = np.float16(1000)
    codes = oracle.encode_greedy(V, cb)
    assert np.array_equal(codes[:, 0], b0) and np.array_equal(codes[:, 1], b1)
    # one codebook, random groups: brute force where the nearest is clear
    C = rng.standard_normal((1, 200, 8)).astype(np.float16)
    Vr = rng.standard_normal((300, 8)).astype(np.float32)
    c1 = oracle.encode_greedy(Vr, C)[:, 0]
    d = _brute_nearest(Vr, C[0].astype(np.float32))
    srt = np.sort(d, axis=1)
    clear = srt[:, 1] > srt[:, 0] * (1 + 1e-4)
    assert np.array_equal(c1[clear], d.argmin(1)[clear])


def pin_worked_encoding():
    """A two-row layer encoded by hand (tests/golden/worked_example_encode.json):
    binary16 scale bits (including the zero row's 1.0), the groups to within
    one binary32 rounding of their exact quotients, the nearest codeword with
    a tie, and the greedy codes."""
    with open(os.path.join(GOLDEN, "worked_example_encode.json")) as fh:
        ex = json.load(fh)
    W = np.array(ex["W"], dtype=np.float32)
    sc, V = oracle.encode_scales(W)
    assert sc.view(np.uint16).tolist() == ex["expected_scale_bits"]
    want = np.array([[n / d for n, d in row] for row in ex["expected_groups_num_den"]])
    assert np.all(np.abs(V.astype(np.float64) - want) <= np.abs(want) * 2.0 ** -24)
    cb = np.array(ex["codebooks"], dtype=np.float16)
    idx, _, _ = oracle.nearest(V, cb[0].astype(np.float32))
    assert idx.tolist() == ex["expected_nearest_codebook0"]
    assert oracle.encode_greedy(V, cb).tolist() == ex["expected_codes"]


ENCODE_PINS = [pin_double_to_half, pin_encode_scales, pin_nearest_codeword, pin_kmeans_update,
               pin_residual_kmeans_recovers_clusters, pin_greedy_codes_recover_sums, pin_worked_encoding]

ALL_PINS = [pin_half_conversion, pin_bf16_rounding, pin_decode_indices,
            pin_index_encoding_recovers_codes, pin_one_hot_activation, pin_linearity,
            pin_dense_special_case, pin_brute_force_tiny, pin_bf16_activations, pin_matmul,
            pin_dequant_bf16_binary32_steps, pin_bits_per_parameter, pin_worked_example,
            *ENCODE_PINS]
