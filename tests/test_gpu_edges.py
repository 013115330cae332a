"""Edge cases of the decode and dequantisation paths against the oracle:
the smallest and largest supported shapes, a single output row, every token
count on the smallest layer, and degenerate inputs (zero activations, zero
scales) whose outputs are exact.

Definitions: "The AQLM Quantization Algorithm, Explained", section "What is
Multi-Codebook Quantization (MCQ)?" (the oracle follows it).
"""
import numpy as np
import pytest
import torch

import additive_codebook_b200 as ac
import oracle
from gpu_util import DEV, check_fp_output, oracle_W, to_dev
from synth import LayerSpec, make_layer

pytestmark = pytest.mark.gpu

FORMATS = [(1, 16), (2, 8), (2, 16)]
# smallest d_in whose row of codes is a whole number of 16-byte chunks
MIN_D_IN = {(1, 16): 64, (2, 8): 64, (2, 16): 32}
MAX_DIM = 1 << 20


def _gemv_check(L, spec, T):
    d = to_dev(L)
    y = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], d["x"]).cpu().numpy()
    y_ref = oracle.gemv_f64(L["codes"], L["codebooks"], L["scales"], L["x"], spec.d_out, spec.d_in, 8, spec.M, spec.B)
    check_fp_output(y, y_ref, oracle_W(L, spec), L["x"].astype(np.float64), out_rel=2.0 ** -10, acc_rel=2.0 ** -14)
    return y


@pytest.mark.parametrize("M,B", FORMATS)
def test_smallest_layer_every_token_count(M, B):
    """One output row and the smallest input width, 1 to 16 tokens (both
    kernels, every row-kernel template and the tensor-core path's padding)."""
    spec = LayerSpec(1, MIN_D_IN[(M, B)], M, B)
    for T in range(1, ac.GEMV_MAX_TOKENS + 1):
        _gemv_check(make_layer(spec, seed=200 + T, tokens=T), spec, T)


@pytest.mark.parametrize("M,B,T", [(1, 16, 1), (2, 8, 4), (2, 16, 16), (1, 16, 7)])
def test_widest_rows(M, B, T):
    """d_in at the largest supported value (2^20 inputs): the row kernel splits
    the input range into many slices, the tensor-core kernel splits its one
    row tile over every CTA."""
    spec = LayerSpec(3, MAX_DIM, M, B)
    _gemv_check(make_layer(spec, seed=210 + T, tokens=T), spec, T)


@pytest.mark.parametrize("M,B", FORMATS)
def test_most_rows(M, B):
    """d_out at the largest supported value (2^20 rows) with the narrowest
    inputs: sampled rows against the oracle, and the dequantisation of a slice
    bit-exact."""
    d_in = MIN_D_IN[(M, B)]
    spec = LayerSpec(MAX_DIM, d_in, M, B)
    L = make_layer(spec, seed=220 + M + B, tokens=1)
    d = to_dev(L)
    y = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], d["x"]).cpu().numpy()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.choice(MAX_DIM, 2000, replace=False), [0, MAX_DIM - 1]]))
    sub = {"codes": np.ascontiguousarray(L["codes"][rows]), "codebooks": L["codebooks"],
           "scales": np.ascontiguousarray(L["scales"][rows])}
    y_ref = oracle.gemv_f64(sub["codes"], sub["codebooks"], sub["scales"], L["x"], len(rows), d_in, 8, M, B)
    W = oracle.dequant_f64(sub["codes"], sub["codebooks"], sub["scales"], len(rows), d_in, 8, M, B)
    check_fp_output(y[:, rows], y_ref, W, L["x"].astype(np.float64), out_rel=2.0 ** -10, acc_rel=2.0 ** -14)
    Wg = ac.aqlm_dequant(d["codes"], d["codebooks"], d["scales"])
    got = Wg[-4096:].cpu().view(torch.int16).numpy().view(np.uint16)
    want = oracle.dequant_bf16(np.ascontiguousarray(L["codes"][-4096:]), L["codebooks"],
                               np.ascontiguousarray(L["scales"][-4096:]), 4096, d_in, 8, M, B)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("M,B", FORMATS)
@pytest.mark.parametrize("T", [1, 3, 9])
def test_zero_activations_and_zero_scales(M, B, T):
    """x = 0 gives y = +0 exactly; a row whose scale is 0 gives 0 whatever x."""
    spec = LayerSpec(300, 1024, M, B)
    L = make_layer(spec, seed=230 + T, tokens=T)
    d = to_dev(L)
    zero = torch.zeros_like(d["x"])
    y0 = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], zero)
    assert torch.equal(y0, torch.zeros_like(y0))
    sc = d["scales"].clone()
    sc[::7] = 0
    y = ac.aqlm_gemv(d["codes"], d["codebooks"], sc, d["x"])
    assert torch.equal(y[:, ::7], torch.zeros_like(y[:, ::7]))
