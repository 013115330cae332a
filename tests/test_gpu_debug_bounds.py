"""The library built with device bounds checks (-DAQLM_DEBUG_BOUNDS):
every kernel runs a small case through the C ABI with its computed indices
checked before each access, and the recorded violation word must stay 0.
The checks themselves are tested by a kernel that records one on purpose
(touching no memory).  Results are also held to the oracle, so the checking
build computes what the product build does.

No compute-sanitizer here: it is closed on this machine; these checks stand in
for it.
"""
import ctypes

import numpy as np
import pytest
import torch

import additive_codebook_b200 as ac
import oracle
from gpu_util import DEV, check_fp_output, oracle_W, to_dev
from synth import LayerSpec, make_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbg(cuda_device):
    lib = ac.load_debug_bounds_library()
    saved = ac.load_library()
    ac._lib = lib            # the module's wrappers call the checking build
    _read(lib, clear=True)
    yield lib
    ac._lib = saved


def _read(lib, clear=True):
    torch.cuda.synchronize()
    w = ctypes.c_uint64(0)
    assert lib.aqlm_debug_bounds_read(ctypes.byref(w), 1 if clear else 0) == ac.AQLM_OK
    return w.value


def _site(word):
    return word >> 48, word & ((1 << 48) - 1)


def test_trip_records_and_clears(dbg):
    assert dbg.aqlm_test_debug_bounds_trip(12345, None) == ac.AQLM_OK
    assert _site(_read(dbg, clear=False)) == (23, 12345)
    assert dbg.aqlm_test_debug_bounds_trip(7, None) == ac.AQLM_OK      # only the first is kept
    assert _site(_read(dbg)) == (23, 12345)
    assert _read(dbg) == 0


@pytest.mark.parametrize("M,B,T,d_out,d_in", [(1, 16, 1, 200, 576), (2, 8, 4, 200, 576), (2, 16, 3, 100, 28736),
                                               (1, 16, 8, 300, 4160), (2, 16, 16, 96, 4128), (2, 8, 1, 33, 4096)])
def test_gemv_paths_stay_in_bounds(dbg, M, B, T, d_out, d_in):
    """Row kernel (with and without a split input range), tensor-core kernel
    (ragged stage, split tiles), all three formats."""
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=11 + T, tokens=T)
    d = to_dev(L)
    y = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], d["x"]).cpu().numpy()
    assert _read(dbg) == 0
    y_ref = oracle.gemv_f64(L["codes"], L["codebooks"], L["scales"], L["x"], d_out, d_in, 8, M, B)
    check_fp_output(y, y_ref, oracle_W(L, spec), L["x"].astype(np.float64), out_rel=2.0 ** -10, acc_rel=2.0 ** -14)


def test_gemv_multi_and_lut_stay_in_bounds(dbg):
    specs = [LayerSpec(n, 1024, 2, 8) for n in (300, 77)]
    Ls = [make_layer(s, seed=20 + k, tokens=1 if k == 0 else 0) for k, s in enumerate(specs)]
    ds = [to_dev(L) for L in Ls]
    ac.aqlm_gemv_multi(ds, ds[0]["x"])
    assert _read(dbg) == 0
    L = make_layer(LayerSpec(4100, 2560, 2, 8), seed=21, tokens=1)
    d = to_dev(L)
    y = ac.aqlm_gemv_lut(d["codes"], d["codebooks"], d["scales"], d["x"]).cpu().numpy()
    assert _read(dbg) == 0
    y_ref = oracle.gemv_f64(L["codes"], L["codebooks"], L["scales"], L["x"], 4100, 2560, 8, 2, 8)
    check_fp_output(y, y_ref, oracle_W(L, LayerSpec(4100, 2560, 2, 8)), L["x"].astype(np.float64),
                    out_rel=2.0 ** -10, acc_rel=2.0 ** -14)


@pytest.mark.parametrize("M,B", [(1, 16), (2, 8), (2, 16)])
def test_dequant_and_gemms_stay_in_bounds(dbg, M, B):
    spec = LayerSpec(520, 576, M, B)
    L = make_layer(spec, seed=30, tokens=200, x_dtype="bf16")
    d = to_dev(L)
    W = ac.aqlm_dequant(d["codes"], d["codebooks"], d["scales"])
    assert _read(dbg) == 0
    want = oracle.dequant_bf16(L["codes"], L["codebooks"], L["scales"], 520, 576, 8, M, B)
    assert np.array_equal(W.cpu().view(torch.int16).numpy().view(np.uint16), want)
    Y, ws = ac.aqlm_gemm(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ac.aqlm_gemm_check(ws) == ac.AQLM_OK
    Yf, wsf = ac.aqlm_gemm_fused(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ac.aqlm_gemm_check(wsf) == ac.AQLM_OK
    assert _read(dbg) == 0
    assert torch.equal(Y.view(torch.int16), Yf.view(torch.int16))


def test_encoding_stays_in_bounds(dbg):
    rng = np.random.Generator(np.random.PCG64(3))
    W = rng.standard_normal((64, 512)).astype(np.float32)
    init = np.stack([rng.choice(4096, 256, replace=False) for _ in range(2)]).astype(np.int32)
    enc = ac.encode_layer(torch.from_numpy(W).to(DEV), 2, 8, init, 2)
    assert _read(dbg) == 0
    V = torch.from_numpy(rng.standard_normal((3000, 8)).astype(np.float32)).to(DEV)
    C = torch.from_numpy(rng.standard_normal((1000, 8)).astype(np.float32)).to(DEV)
    idx, dist = ac.nearest_codeword(V, C, with_dist=True)
    ac.kmeans_update(V, idx, C)
    assert _read(dbg) == 0
    assert enc["codes"].shape == (64, 64, 2)


def test_probe_stays_in_bounds(dbg):
    table = torch.zeros(1 << 16, dtype=torch.uint8, device=DEV)
    ac.probe_gather(table, 0, ctas_per_sm=1, iters=2)
    ac.probe_gather(table[:8192], 1, ctas_per_sm=1, iters=2)
    assert _read(dbg) == 0
