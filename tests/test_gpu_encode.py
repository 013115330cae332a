"""GPU parity of the encoding path (scales, nearest codeword, k-means,
residual k-means, greedy codes, whole-layer encoding) against the CPU oracle.

Section "AQLM quantization process" of "The AQLM Quantization Algorithm,
Explained": codebooks initialised by residual k-means, codes learned with the
codebooks fixed; the readings are stated in oracle/aqlm_encode_oracle.c.  The
oracle evaluates the definitions in double; results that carry rounding error
(the binary16 scale of a row, the choice of a nearest codeword) are held to
the error bounds of tests/encode_checks.py -- the oracle's value wherever the
choice is clear, a choice within the bound elsewhere -- and later steps are
carried through on the GPU's own choices.  Integer results computed from
given choices (counts) and correctly rounded divisions are bit-exact;
centroids are sums in double whose order the GPU does not fix, so they agree
to within one binary32 ulp.
"""
import numpy as np
import pytest
import torch

import additive_codebook_b200 as ac
import oracle
from encode_checks import check_greedy, check_groups, check_nearest, check_scales
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


def test_encode_scales():
    """E1 within its rounding interval (the oracle's value where clear), E2 a
    correctly rounded division by the GPU's own scale, bit for bit."""
    rng = _rng(1)
    W = (rng.standard_normal((300, 1024)) * rng.uniform(1e-3, 5.0, (300, 1))).astype(np.float32)
    W[17] = 0.0
    W[18, :] = 1e-6
    W[19, :] = 2.0 ** -30                      # root mean square below binary16's range: scale 1.0
    sc, V = ac.encode_scales(_t(W))
    sc = sc.cpu().numpy()
    check_scales(W, sc)
    check_groups(W, sc, V.cpu().numpy())
    assert sc[17] == sc[19] == 1.0


@pytest.mark.parametrize("N,K", [(1, 1), (999, 7), (5000, 256), (3000, 1000), (2048, 65536), (100, 65536)])
def test_nearest_codeword(N, K):
    """Each index a valid nearest codeword (exactly the oracle's where the
    choice is clear) and its distance within bound, including groups equal to
    codewords and duplicated codewords (lowest index); (100, 65536) spreads
    the codewords of each group over many CTAs, whose winners meet in the
    64-bit atomic minimum."""
    rng = _rng(2 + K)
    C = rng.standard_normal((K, 8)).astype(np.float32)
    V = rng.standard_normal((N, 8)).astype(np.float32)
    if K > 10:
        C[K - 3] = C[5]                       # a duplicate far from its twin
        V[: min(N, 20)] = C[rng.integers(0, K, min(N, 20))]
        V[0] = C[5]
    idx, dist = ac.nearest_codeword(_t(V), _t(C), with_dist=True)
    idx, dist = idx.cpu().numpy(), dist.cpu().numpy()
    check_nearest(V, C, idx, dist)
    if K > 10:
        assert idx[0] == 5 and dist[0] == 0
        exact = np.flatnonzero((V[: min(N, 20)][:, None, :] == C[None, :, :]).all(-1).any(-1))
        assert (dist[exact] == 0).all()


def test_nearest_codeword_near_ties():
    """Groups at the midpoint of two codewords and groups a few binary32 ulps
    off it: any choice within the bound passes, the far codewords never."""
    rng = _rng(40)
    K = 512
    C = (rng.standard_normal((K, 8)) * 0.5).astype(np.float16).astype(np.float32)
    a, b = rng.integers(0, K, 300), rng.integers(0, K, 300)
    V = ((C[a] + C[b]) / 2).astype(np.float32)
    V[150:] = np.nextafter(V[150:], np.float32(np.inf) * np.sign(rng.standard_normal((150, 8))).astype(np.float32))
    idx = ac.nearest_codeword(_t(V), _t(C)).cpu().numpy()
    check_nearest(V, C, idx)


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
    means, as the oracle's does; codebook 1 (k-means of the residual noise)
    equals the steps taken one call at a time, each valid against the oracle."""
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
    means = np.stack([V[lab == k].astype(np.float64).mean(0) for k in range(K)])
    assert np.allclose(C[0], means, atol=1e-5)
    # codebook 1 clusters noise, where assignments can sit within rounding of a tie
    assert _ulps(C, _residual_kmeans_steps(V, 2, K, init, 5)) <= 1


def _residual_kmeans_steps(V, M, K, init, iters):
    """Reading E5 step by step on the GPU's own choices: every assignment is
    checked as a valid nearest codeword, every update against the oracle's
    update on the same assignment (counts exact, centroids within one ulp),
    and the GPU's centroids are carried on."""
    R = V.copy()
    out = []
    for m in range(M):
        C = R[init[m]].copy()
        for _ in range(iters):
            idx = ac.nearest_codeword(_t(R), _t(C)).cpu().numpy()
            check_nearest(R, C, idx, what=f"k-means assignment, codebook {m}")
            C_gpu, counts = ac.kmeans_update(_t(R), _t(idx), _t(C))
            C_ref, counts_ref = oracle.kmeans_update(R, idx, C)
            assert np.array_equal(counts.cpu().numpy(), counts_ref.astype(np.int32))
            C_gpu = C_gpu.cpu().numpy()
            assert _ulps(C_gpu, C_ref) <= 1
            C = C_gpu
        idx = ac.nearest_codeword(_t(R), _t(C)).cpu().numpy()
        check_nearest(R, C, idx, what=f"final assignment, codebook {m}")
        R = (R - C[idx]).astype(np.float32)
        out.append(C)
    return np.stack(out)


@pytest.mark.parametrize("N,M,K,iters", [(8192, 1, 256, 1), (6000, 2, 256, 3), (20000, 1, 4096, 2)])
def test_residual_kmeans_random(N, M, K, iters):
    """aqlm_residual_kmeans on random groups equals the same steps taken one
    call at a time, each of them valid against the oracle."""
    rng = _rng(5 + M + iters)
    V = rng.standard_normal((N, 8)).astype(np.float32)
    init = np.stack([rng.choice(N, K, replace=False) for _ in range(M)]).astype(np.int32)
    C = ac.residual_kmeans(_t(V), M, K, init, iters=iters).cpu().numpy()
    C_steps = _residual_kmeans_steps(V, M, K, init, iters)
    assert _ulps(C, C_steps) <= 1


@pytest.mark.parametrize("M,B", [(1, 16), (2, 8), (2, 16)])
def test_encode_codes(M, B):
    """Greedy codes against fixed fp16 codebooks, written in the inference
    layout: every code a valid nearest codeword of its residual (2^16
    codewords for the 16-bit formats), carried through on the GPU's choices."""
    rng = _rng(6 + B + M)
    d_out, d_in = 48, 512
    V = rng.standard_normal((d_out * d_in // 8, 8)).astype(np.float32)
    cb = (rng.standard_normal((M, 1 << B, 8)) * (1.0 if M == 1 else 0.7)).astype(np.float16)
    codes = ac.encode_codes(_t(V), _t(cb), d_out, d_in).cpu().numpy()
    got = (codes.view(np.uint8) if B == 8 else codes.view(np.uint16)).astype(np.int64)
    check_greedy(V, cb, got.reshape(-1, M))


@pytest.mark.parametrize("M,B", [(2, 8), (1, 16)])
def test_encode_layer_round_trip(M, B):
    """The whole encoding of a layer: scales valid (E1, E2), codebooks equal to
    residual k-means of the GPU's groups taken step by step and checked
    against the oracle, codes valid greedy codes against the GPU's fp16
    codebooks; the encoded layer approximates W as well as the oracle's own
    pipeline does, and runs through aqlm_gemv like any other layer."""
    rng = _rng(7 + B)
    d_out, d_in = 64, 256 if B == 8 else 512
    W = (rng.standard_normal((d_out, d_in)) * rng.uniform(0.5, 2.0, (d_out, 1))).astype(np.float32)
    n = d_out * d_in // 8
    K = 1 << B
    init = np.stack([rng.choice(n, K, replace=n < K) for _ in range(M)]).astype(np.int32)
    iters = 3 if B == 8 else 1
    enc = ac.encode_layer(_t(W), M, B, init, iters)
    sc = enc["scales"].cpu().numpy()
    check_scales(W, sc)
    V = (W / sc.astype(np.float32)[:, None]).reshape(-1, 8)
    cb = enc["codebooks"].cpu().numpy()
    C_steps = _residual_kmeans_steps(V, M, K, init, iters).astype(np.float16)
    assert np.abs(cb.astype(np.float32) - C_steps.astype(np.float32)).max() <= \
        2.0 ** -10 * np.abs(C_steps.astype(np.float32)).max()
    codes = enc["codes"].cpu().numpy()
    got = (codes.view(np.uint8) if B == 8 else codes.view(np.uint16)).astype(np.int64)
    check_greedy(V, cb, got.reshape(-1, M))
    # the oracle's own pipeline with the same draw, for the approximation quality
    sc_ref, V_ref = oracle.encode_scales(W)
    C_ref = oracle.residual_kmeans(V_ref, M, K, init, iters).astype(np.float16)
    codes_ref = oracle.encode_greedy(V_ref, C_ref).reshape(d_out, d_in // 8, M)
    W_gpu = oracle.dequant_f64(codes, cb, sc, d_out, d_in, 8, M, B)
    W_ref = oracle.dequant_f64(codes_ref.astype(np.uint8) if B == 8 else codes_ref.view(np.int16), C_ref, sc_ref,
                               d_out, d_in, 8, M, B)
    err_gpu = np.linalg.norm(W_gpu - W) / np.linalg.norm(W)
    err_ref = np.linalg.norm(W_ref - W) / np.linalg.norm(W)
    assert err_gpu <= err_ref * 1.02 + 1e-6, (err_gpu, err_ref)
    # the encoded layer runs through the decode path like any other
    x = rng.standard_normal((1, d_in)).astype(np.float16)
    y = ac.aqlm_gemv(enc["codes"], enc["codebooks"], enc["scales"], _t(x)).float().cpu().numpy()
    y_ref = oracle.gemv_f64(codes, cb, sc, x, d_out, d_in, 8, M, B)
    assert np.abs(y - y_ref).max() <= 2e-3 * np.linalg.norm(x.astype(np.float64)) * np.linalg.norm(W_gpu, axis=1).max()


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
