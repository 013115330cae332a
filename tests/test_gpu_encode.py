"""GPU parity of the encoding path (scales, nearest codeword, k-means,
residual k-means, greedy codes, whole-layer encoding) against the CPU oracle.

Section "AQLM quantization process" of "The AQLM Quantization Algorithm,
Explained": codebooks initialised by residual k-means, codes learned with the
codebooks fixed; the readings both sides take are in
oracle/aqlm_encode_oracle.c.  Every integer result (index, code, count) and
every value computed in a fixed order (scales, groups, distances) must agree
bit for bit; centroids are sums in double whose order the GPU does not fix,
so they agree to within one binary32 ulp.
"""
import numpy as np
import pytest
import torch

import additive_codebook_b200 as ac
import oracle
from gpu_util import DEV

pytestmark = pytest.mark.gpu


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _t(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _ulps(a, b):
    a = np.ascontiguousarray(a, dtype=np.float32).view(np.int32).astype(np.int64)
    b = np.ascontiguousarray(b, dtype=np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b).max() if a.size else 0


def test_encode_scales_bit_exact():
    rng = _rng(1)
    W = (rng.standard_normal((300, 1024)) * rng.uniform(1e-3, 5.0, (300, 1))).astype(np.float32)
    W[17] = 0.0
    W[18, :] = 1e-6
    sc, V = ac.encode_scales(_t(W))
    sc_ref, V_ref = oracle.encode_scales(W)
    assert np.array_equal(sc.cpu().numpy().view(np.uint16), sc_ref.view(np.uint16))
    assert np.array_equal(V.cpu().numpy(), V_ref)


@pytest.mark.parametrize("N,K", [(1, 1), (999, 7), (5000, 256), (3000, 1000), (2048, 65536), (100, 65536)])
def test_nearest_codeword_bit_exact(N, K):
    """Indices and distances bit-exact, including groups equal to codewords and
    duplicated codewords (lowest index); (100, 65536) spreads the codewords of
    each group over many CTAs, whose winners meet in the 64-bit atomic minimum."""
    rng = _rng(2 + K)
    C = rng.standard_normal((K, 8)).astype(np.float32)
    V = rng.standard_normal((N, 8)).astype(np.float32)
    if K > 10:
        C[K - 3] = C[5]                       # a duplicate far from its twin
        V[: min(N, 20)] = C[rng.integers(0, K, min(N, 20))]
        V[0] = C[5]
    idx, dist = ac.nearest_codeword(_t(V), _t(C), with_dist=True)
    idx_ref, dist_ref = oracle.nearest(V, C)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    assert np.array_equal(dist.cpu().numpy().view(np.uint32), dist_ref.view(np.uint32))
    if K > 10:
        assert idx_ref[0] == 5


def test_kmeans_update_matches():
    rng = _rng(3)
    N, K = 20000, 300
    V = rng.standard_normal((N, 8)).astype(np.float32)
    idx = rng.integers(0, K - 4, N).astype(np.int32)        # the last 4 centroids have no group
    C_prev = rng.standard_normal((K, 8)).astype(np.float32)
    C, counts = ac.kmeans_update(_t(V), _t(idx), _t(C_prev))
    C_ref, counts_ref = oracle.kmeans_update(V, idx, C_prev)
    assert np.array_equal(counts.cpu().numpy(), counts_ref.astype(np.int32))
    assert _ulps(C.cpu().numpy(), C_ref) <= 1
    assert np.array_equal(C.cpu().numpy()[K - 4:], C_prev[K - 4:])


def test_residual_kmeans_separated_clusters():
    """Codebook 0 of data around separated centres converges to the cluster
    means on both sides; codebook 1 (of the residuals) agrees within rounding."""
    rng = _rng(4)
    K, per = 64, 50
    centres = (rng.standard_normal((K, 8)) * 10).astype(np.float32)
    lab = np.repeat(np.arange(K), per)
    V = (centres[lab] + rng.standard_normal((K * per, 8)).astype(np.float32) * 0.05).astype(np.float32)
    perm = rng.permutation(K * per)
    V, lab = V[perm], lab[perm]
    init = np.stack([np.array([np.flatnonzero(lab == k)[0] for k in range(K)]),
                     rng.choice(K * per, K, replace=False)]).astype(np.int32)
    C = ac.residual_kmeans(_t(V), 2, K, init, iters=5).cpu().numpy()
    C_ref = oracle.residual_kmeans(V, 2, K, init, iters=5)
    assert _ulps(C[0], C_ref[0]) <= 1
    assert np.allclose(C[1], C_ref[1], atol=1e-6)


def test_residual_kmeans_one_codebook_random():
    rng = _rng(5)
    N, K = 8192, 256
    V = rng.standard_normal((N, 8)).astype(np.float32)
    init = rng.choice(N, K, replace=False).astype(np.int32)[None, :]
    C = ac.residual_kmeans(_t(V), 1, K, init, iters=1).cpu().numpy()
    C_ref = oracle.residual_kmeans(V, 1, K, init, iters=1)
    assert _ulps(C, C_ref) <= 1


@pytest.mark.parametrize("M,B", [(1, 16), (2, 8), (2, 16)])
def test_encode_codes_bit_exact(M, B):
    """Greedy codes against fixed fp16 codebooks, written in the inference
    layout: bit-exact with the oracle (2^16 codewords for the 16-bit formats)."""
    rng = _rng(6 + B + M)
    d_out, d_in = 48, 512
    V = rng.standard_normal((d_out * d_in // 8, 8)).astype(np.float32)
    cb = (rng.standard_normal((M, 1 << B, 8)) * (1.0 if M == 1 else 0.7)).astype(np.float16)
    codes = ac.encode_codes(_t(V), _t(cb), d_out, d_in).cpu().numpy()
    ref = oracle.encode_greedy(V, cb).reshape(d_out, d_in // 8, M)
    got = codes.view(np.uint8) if B == 8 else codes.view(np.uint16)
    assert np.array_equal(got.astype(np.uint16), ref)


@pytest.mark.parametrize("M,B", [(2, 8), (1, 16)])
def test_encode_layer_round_trip(M, B):
    """The whole encoding of a layer: scales bit-exact with the oracle's
    pipeline, codebooks within rounding, codes equal (but for near ties that a
    last-bit centroid difference may flip), the encoded layer approximates W as
    well as the oracle's, and it runs through aqlm_gemv like any other layer."""
    rng = _rng(7 + B)
    d_out, d_in = 64, 256 if B == 8 else 512
    W = (rng.standard_normal((d_out, d_in)) * rng.uniform(0.5, 2.0, (d_out, 1))).astype(np.float32)
    n = d_out * d_in // 8
    K = 1 << B
    init = np.stack([rng.choice(n, K, replace=n < K) for _ in range(M)]).astype(np.int32)
    iters = 3 if B == 8 else 1
    enc = ac.encode_layer(_t(W), M, B, init, iters)
    # the oracle's pipeline with the same draw
    sc_ref, V = oracle.encode_scales(W)
    C_ref = oracle.residual_kmeans(V, M, K, init, iters).astype(np.float16)
    codes_ref = oracle.encode_greedy(V, C_ref).reshape(d_out, d_in // 8, M)
    assert np.array_equal(enc["scales"].cpu().numpy().view(np.uint16), sc_ref.view(np.uint16))
    cb = enc["codebooks"].cpu().numpy()
    assert np.abs(cb.astype(np.float32) - C_ref.astype(np.float32)).max() <= \
        2.0 ** -10 * np.abs(C_ref.astype(np.float32)).max()
    codes = enc["codes"].cpu().numpy()
    got = (codes.view(np.uint8) if B == 8 else codes.view(np.uint16)).astype(np.uint16)
    assert (got == codes_ref).mean() >= 0.99
    # decode both exactly (the oracle's double decode) and compare how well they approximate W
    W_gpu = oracle.dequant_f64(codes, cb, enc["scales"].cpu().numpy(), d_out, d_in, 8, M, B)
    W_ref = oracle.dequant_f64(codes_ref.astype(np.uint8) if B == 8 else codes_ref.view(np.int16), C_ref, sc_ref,
                               d_out, d_in, 8, M, B)
    err_gpu = np.linalg.norm(W_gpu - W) / np.linalg.norm(W)
    err_ref = np.linalg.norm(W_ref - W) / np.linalg.norm(W)
    assert err_gpu <= err_ref * 1.02 + 1e-6, (err_gpu, err_ref)
    # the encoded layer runs through the decode path like any other
    x = rng.standard_normal((1, d_in)).astype(np.float16)
    y = ac.aqlm_gemv(enc["codes"], enc["codebooks"], enc["scales"], _t(x)).float().cpu().numpy()
    sc_gpu = enc["scales"].cpu().numpy()
    y_ref = oracle.gemv_f64(codes, cb, sc_gpu, x, d_out, d_in, 8, M, B)
    W64 = oracle.dequant_f64(codes, cb, sc_gpu, d_out, d_in, 8, M, B)
    assert np.abs(y - y_ref).max() <= 2e-3 * np.linalg.norm(x.astype(np.float64)) * np.linalg.norm(W64, axis=1).max()


def test_encoded_groups_recover_their_codes():
    """Closed form: groups that are exactly codewords of codebook 0 (distinct
    rows), with codebook 1 all zeros, encode to (their codeword, 0): the
    residual is 0 after the first codebook and every codeword of the second
    ties at distance 0, so the lowest index wins."""
    rng = _rng(8)
    C = np.zeros((2, 256, 8), dtype=np.float16)
    C[0] = (rng.permutation(256 * 8).reshape(256, 8) % 97 - 48).astype(np.float16)
    assert len(np.unique(C[0], axis=0)) == 256
    b = rng.integers(0, 256, (32, 32))
    V = C[0][b].reshape(-1, 8).astype(np.float32)
    codes = ac.encode_codes(_t(V), _t(C), 32, 256).cpu().numpy()
    assert np.array_equal(codes[:, :, 0], b) and not codes[:, :, 1].any()
