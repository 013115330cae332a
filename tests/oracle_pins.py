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


ALL_PINS = [pin_half_conversion, pin_bf16_rounding, pin_decode_indices,
            pin_index_encoding_recovers_codes, pin_one_hot_activation, pin_linearity,
            pin_dense_special_case, pin_brute_force_tiny, pin_bf16_activations, pin_matmul,
            pin_dequant_bf16_binary32_steps, pin_bits_per_parameter, pin_worked_example]
