"""aqlm_gemv_noalloc: the decode product for callers that cannot allocate.

Some callers of this library have no way to allocate device memory when they
call it -- a plugin that its host engine hands only input and output
pointers, or an engine that fixes its device memory at start-up.  For them
aqlm_gemv_noalloc keeps its scratch in an array built into the library
instead of a caller-provided workspace.  These tests call it through the C
ABI, twice in a row on the same shape, and hold its output to the oracle
(the tolerance of the other parity tests) and bit for bit to aqlm_gemv's
output on the same inputs (the same kernels on the same scratch layout); its
status word must survive later calls until aqlm_gemv_noalloc_check reads it.

This file is named so that pytest collects it last: a run that stops at the
first failure has then already run every other test.
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

# shapes whose product needs scratch: a 3-token row-kernel product whose
# activations are split into slices (7 x 64 chunks of 28672 inputs),
# products of several tokens split over the input range to fill the SMs, and
# a 16-token product split because its activations do not fit on chip at once
CASES = [(1024, 28672, 2, 8, 3), (2048, 4096, 2, 8, 6), (1024, 4096, 1, 16, 16), (512, 4160, 2, 16, 8)]


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _call_noalloc(lib, d, x, y):
    shape = ac.shape_of(d["codes"])
    return lib.aqlm_gemv_noalloc(ctypes.c_void_p(d["codes"].data_ptr()), ctypes.c_void_p(d["codebooks"].data_ptr()),
                                 ctypes.c_void_p(d["scales"].data_ptr()), ctypes.c_void_p(x.data_ptr()),
                                 ctypes.c_void_p(y.data_ptr()), x.shape[0], shape, _stream())


@pytest.mark.parametrize("d_out,d_in,M,B,T", CASES)
def test_noalloc_matches_oracle_and_gemv_on_two_calls(cuda_device, d_out, d_in, M, B, T):
    lib = ac.load_library()
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=77 + T, tokens=T)
    d = to_dev(L)
    shape = ac.shape_of(d["codes"])
    assert 0 < lib.aqlm_gemv_workspace_bytes(shape, T) <= lib.aqlm_gemv_noalloc_max_scratch_bytes()
    y_gemv = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], d["x"]).cpu().numpy()
    W = oracle_W(L, spec)
    x64 = L["x"].astype(np.float64)
    y_ref = W @ x64.T
    for _ in range(2):
        y = torch.full((T, d_out), float("nan"), dtype=torch.float16, device=DEV)
        assert _call_noalloc(lib, d, d["x"], y) == ac.AQLM_OK
        assert lib.aqlm_gemv_noalloc_check(_stream()) == ac.AQLM_OK
        y = y.cpu().numpy()
        check_fp_output(y, y_ref.T, W, x64, out_rel=2.0 ** -10, acc_rel=2.0 ** -14)
        assert np.array_equal(y.view(np.uint16), y_gemv.view(np.uint16))


def test_noalloc_status_survives_until_checked(cuda_device):
    """A status word set in the built-in array (as a bounded wait that gave up
    would set it) is reported by aqlm_gemv_noalloc_check even after further
    calls of other shapes and token counts, then cleared; a call rejected for
    its arguments enqueues nothing."""
    lib = ac.load_library()
    assert lib.aqlm_gemv_noalloc_check(_stream()) == ac.AQLM_OK
    assert lib.aqlm_test_gemv_noalloc_set_status(ac.AQLM_ERR_TIMEOUT, _stream()) == ac.AQLM_OK
    for d_out, d_in, M, B, T in CASES:
        L = make_layer(LayerSpec(d_out, d_in, M, B), seed=5, tokens=T)
        d = to_dev(L)
        y = torch.empty((T, d_out), dtype=torch.float16, device=DEV)
        assert _call_noalloc(lib, d, d["x"], y) == ac.AQLM_OK
    assert lib.aqlm_gemv_noalloc_check(_stream()) == ac.AQLM_ERR_TIMEOUT
    assert lib.aqlm_gemv_noalloc_check(_stream()) == ac.AQLM_OK


def test_noalloc_checks_arguments_first(cuda_device):
    """Bad pointers and sizes beyond the array are rejected before anything is
    enqueued (AQLM_ERR_INVALID_ARG, _MISALIGNED, _WORKSPACE)."""
    lib = ac.load_library()
    d_out, d_in, M, B, T = CASES[2]
    shape = ac.Shape(d_out, d_in, 8, M, B)
    x = torch.zeros((T, d_in), dtype=torch.float16, device=DEV)
    y = torch.zeros((T, d_out), dtype=torch.float16, device=DEV)
    codes = torch.zeros(16, dtype=torch.uint8, device=DEV)
    p = ctypes.c_void_p(codes.data_ptr())
    st = lib.aqlm_gemv_noalloc(p, p, p, ctypes.c_void_p(x.data_ptr()), None, T, shape, _stream())
    assert st == ac.AQLM_ERR_INVALID_ARG
    st = lib.aqlm_gemv_noalloc(p, p, p, ctypes.c_void_p(x.data_ptr() + 2), ctypes.c_void_p(y.data_ptr()), T, shape,
                               _stream())
    assert st == ac.AQLM_ERR_MISALIGNED
    # 3 tokens of 28672 inputs on the row kernel (2x8): seven activation
    # slices, 7 x 3 x 131072 fp32 partial sums (11 MB), more than the 8 MiB
    # built in
    big = ac.Shape(131072, 28672, 8, 2, 8)
    assert lib.aqlm_gemv_workspace_bytes(big, 3) > lib.aqlm_gemv_noalloc_max_scratch_bytes()
    st = lib.aqlm_gemv_noalloc(p, p, p, ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()), 3, big,
                               _stream())
    assert st == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemv_noalloc_check(_stream()) == ac.AQLM_OK
