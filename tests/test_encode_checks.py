"""The encoding validity checks (tests/encode_checks.py) on the CPU: they must
accept an independent binary32 evaluation of the definitions, whose rounding
differs from the oracle's, and reject planted mistakes."""
import numpy as np

import oracle
from encode_checks import check_greedy, check_groups, check_nearest, check_scales


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _nearest_f32(V, C):
    """Least binary32 score |c|^2 - 2 <v, c>, ties to the lowest index, with
    numpy's float32 reductions (an evaluation order unlike any kernel's)."""
    V, C = V.astype(np.float32), C.astype(np.float32)
    cc = np.einsum("kt,kt->k", C, C, dtype=np.float32)
    score = cc[None, :] - np.float32(2) * (V @ C.T)
    return score.argmin(1)


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_check_nearest_accepts_binary32_and_rejects_mistakes():
    rng = _rng(31)
    K = 4096
    C = (rng.standard_normal((K, 8)) * 0.3).astype(np.float16).astype(np.float32)
    V = rng.standard_normal((3000, 8)).astype(np.float32)
    V[:40] = C[rng.integers(0, K, 40)]
    V[40:60] = (C[:20] + C[20:40]) / 2           # near-midpoints: ties at binary32 level are possible
    idx32 = _nearest_f32(V, C)
    check_nearest(V, C, idx32)
    idx_ref, d_ref, second = oracle.nearest(V, C)
    check_nearest(V, C, idx_ref, d_ref)
    # planted: the runner-up where the choice is clear
    gap = second - d_ref
    n = int(np.argmax(gap))
    d_all = ((V[n].astype(np.float64) - C.astype(np.float64)) ** 2).sum(1)
    wrong = idx_ref.copy()
    wrong[n] = int(np.argsort(d_all, kind="stable")[1])
    assert _fails(check_nearest, V, C, wrong)
    # planted: an off-by-one index and a distance dropping one lane
    wrong = idx_ref.copy()
    wrong[100] = (wrong[100] + 1) % K
    assert _fails(check_nearest, V, C, wrong)
    d_drop = ((V.astype(np.float64) - C.astype(np.float64)[idx_ref])[:, :7] ** 2).sum(1)
    assert _fails(check_nearest, V, C, idx_ref, d_drop)


def test_check_scales_and_groups():
    rng = _rng(32)
    W = (rng.standard_normal((200, 512)) * rng.uniform(1e-3, 4.0, (200, 1))).astype(np.float32)
    W[5] = 0.0
    sc, V = oracle.encode_scales(W)
    assert check_scales(W, sc) == 0
    check_groups(W, sc, V)
    # a double evaluation in another order (reversed, pairwise) is accepted
    W64 = W.astype(np.float64)[:, ::-1]
    alt = np.sqrt(np.add.reduce(W64 * W64, axis=1) / W.shape[1]).astype(np.float16)
    alt[5] = 1.0
    check_scales(W, alt)
    # planted: one binary16 step up, the mean absolute value, groups divided by the wrong row's scale
    up = sc.copy()
    up[17] = np.nextafter(up[17], np.float16(np.inf))
    assert _fails(check_scales, W, up)
    mean_abs = np.abs(W.astype(np.float64)).mean(1).astype(np.float16)
    mean_abs[5] = 1.0
    assert _fails(check_scales, W, mean_abs)
    assert _fails(check_groups, W, np.roll(sc, 1), V)


def test_check_greedy():
    rng = _rng(33)
    cb = (rng.standard_normal((2, 256, 8)) * 0.6).astype(np.float16)
    V = rng.standard_normal((2000, 8)).astype(np.float32)
    codes = oracle.encode_greedy(V, cb)
    assert check_greedy(V, cb, codes) == 0
    # planted: the second codebook chosen for the group itself, not its residual
    kept = codes.copy()
    kept[:, 1] = oracle.nearest(V, cb[1].astype(np.float32))[0]
    assert _fails(check_greedy, V, cb, kept)
