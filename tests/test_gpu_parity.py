"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer work (index unpacking) and the bf16 dequantisation are compared bit
for bit; the fp16/bf16 layer outputs are held to the stated tolerance
max|y - y_ref| <= 2e-3 ||x||_2 max_i ||(s . W^)_i||_2 and to a tighter bound
derived from the arithmetic (one output rounding plus fp32 accumulation).
Sizes span several CTA tiles with ragged tails; the full-size layers of the
benchmark are checked on sampled rows/tokens the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import additive_codebook_b200 as ac
import oracle
from gpu_util import (DEV, bf16_to_np_bits, check_fp_output, layer, oracle_W, to_dev)
from synth import LayerSpec, make_layer, make_x

pytestmark = pytest.mark.gpu

FORMATS = [(1, 16), (2, 8), (2, 16)]


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_device):
    ac.load_library()
    yield


# ---------------------------------------------------------------- indices

@pytest.mark.parametrize("M,B", FORMATS)
def test_decode_indices_bit_exact(M, B):
    spec = LayerSpec(200, 576, M, B)
    L = make_layer(spec, seed=1, tokens=0)
    d = to_dev(L)
    got = ac.aqlm_decode_indices(d["codes"]).cpu().numpy().view(np.uint16)
    want = oracle.decode_indices(L["codes"], spec.d_out, spec.d_in, 8, M, B)
    assert np.array_equal(got, want)


def test_decode_indices_edge_codes():
    codes = np.array([0, 1, 32767, -32768, -1, 12345, -2, 255] * 8, dtype=np.int16).reshape(8, 8, 1)
    got = ac.aqlm_decode_indices(torch.from_numpy(codes).to(DEV)).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, oracle.decode_indices(codes, 8, 64, 8, 1, 16))


# ---------------------------------------------------------------- dequant

@pytest.mark.parametrize("M,B", FORMATS)
@pytest.mark.parametrize("d_out,d_in", [(200, 576), (1000, 1024)])
def test_dequant_bit_exact(M, B, d_out, d_in):
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=2 + d_out, tokens=0)
    L["scales"][:4] = np.array([1.0, -1.0, -0.75, 65504.0], dtype=np.float16)   # signs, overflow to inf
    d = to_dev(L)
    got = bf16_to_np_bits(ac.aqlm_dequant(d["codes"], d["codebooks"], d["scales"]))
    want = oracle.dequant_bf16(L["codes"], L["codebooks"], L["scales"], d_out, d_in, 8, M, B)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("M,B", FORMATS)
def test_dequant_extreme_codes(M, B):
    """All-zero and all-max codes (255 / 65535) and special codebook values."""
    spec = LayerSpec(64, 512, M, B)
    L = make_layer(spec, seed=3, tokens=0)
    L["codes"][: 32] = 0
    L["codes"][32:] = np.array(-1 if B == 16 else 255).astype(L["codes"].dtype)
    L["codebooks"][:, 0, :3] = [0.0, -0.0, 6.0e-8]
    L["codebooks"][:, -1, :3] = [65504.0, -65504.0, np.inf]
    d = to_dev(L)
    got = bf16_to_np_bits(ac.aqlm_dequant(d["codes"], d["codebooks"], d["scales"]))
    want = oracle.dequant_bf16(L["codes"], L["codebooks"], L["scales"], 64, 512, 8, M, B)
    assert np.array_equal(got, want)


def test_dequant_deterministic():
    spec = LayerSpec(512, 1024, 1, 16)
    d = to_dev(make_layer(spec, seed=4, tokens=0))
    a = ac.aqlm_dequant(d["codes"], d["codebooks"], d["scales"])
    b = ac.aqlm_dequant(d["codes"], d["codebooks"], d["scales"])
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


# ---------------------------------------------------------------- gemv

def _gemv_case(M, B, d_out, d_in, T, seed):
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=seed, tokens=T)
    d = to_dev(L)
    y = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], d["x"]).cpu().numpy()
    y_ref = oracle.gemv_f64(L["codes"], L["codebooks"], L["scales"], L["x"], d_out, d_in, 8, M, B)
    W = oracle_W(L, spec)
    return check_fp_output(y, y_ref, W, L["x"].astype(np.float64), out_rel=2.0 ** -10, acc_rel=2.0 ** -14)


@pytest.mark.parametrize("M,B", FORMATS)
@pytest.mark.parametrize("T", [1, 2, 3, 4, 7, 8, 16])
def test_gemv_small(M, B, T):
    # 200 rows: 7 row tiles, the last one ragged; 576 inputs: 72 groups, a
    # chunk count that does not divide evenly over the 8 warps
    _gemv_case(M, B, 200, 576, T, seed=10 + T)


@pytest.mark.parametrize("M,B", FORMATS)
@pytest.mark.parametrize("T", [1, 4, 16])
def test_gemv_split_input_range(M, B, T):
    # d_in = 4160 -> 520 groups; T = 16 needs the split over the input range
    # (slabs of at most 256 groups), T = 4 and T = 1 do not
    _gemv_case(M, B, 96, 4160, T, seed=20 + T)


@pytest.mark.parametrize("M,B,T,d_in", [(1, 16, 1, 82112), (2, 16, 1, 82144), (1, 16, 2, 28736), (2, 16, 3, 28736),
                                         (2, 8, 3, 28736), (2, 8, 4, 28736)]
                         + [(m, b, 2, 20544) for m, b in FORMATS])
def test_gemv_rows_split_input_range(M, B, T, d_in):
    # row-kernel token counts (1x16 up to 2, 2x16 up to 3, 2x8 up to 4) whose
    # activations exceed the row kernel's 32 KiB budget: the input range is
    # split in slices of whole 32-chunk lane slots (3 to 11 of them here, the
    # last one ragged), partial sums meet in the workspace; 100 rows leave some
    # warps without a row
    _gemv_case(M, B, 100, d_in, T, seed=30 + T)


LUT_SHAPES = [(1, 64), (17, 192), (300, 1600), (4100, 2560), (33, 65536), (4096, 4096), (2000, 28672), (28672, 8192)]


@pytest.mark.parametrize("d_out,d_in", LUT_SHAPES)
def test_gemv_lut_shapes(d_out, d_in):
    # aqlm_gemv_lut (2x8, one token; slabs of 32 groups, rows in batches of 16
    # per warp, chunks of 256 rows): last slabs of 8, 24, 8, 0 and 0 groups,
    # row ranges that are not multiples of 16, a single row, 256 slabs (more
    # than SMs), several slabs per CTA (28672 inputs; 28672 rows); each output
    # also bit-identical on a second call through the same workspace
    spec = LayerSpec(d_out, d_in, 2, 8)
    L = make_layer(spec, seed=80 + d_out, tokens=1)
    d = to_dev(L)
    ws = torch.zeros(max(16, ac.gemv_lut_workspace_bytes(ac.shape_of(d["codes"]))), dtype=torch.uint8, device=DEV)
    y = ac.aqlm_gemv_lut(d["codes"], d["codebooks"], d["scales"], d["x"], workspace=ws)
    y2 = ac.aqlm_gemv_lut(d["codes"], d["codebooks"], d["scales"], d["x"], workspace=ws)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    rows = np.arange(d_out)
    if d_out > 4096:      # sampled rows, computed one by one by the oracle
        rng = np.random.Generator(np.random.PCG64(7))
        rows = np.unique(np.concatenate([rng.choice(d_out, 512, replace=False), [0, d_out - 1]]))
    codes = np.ascontiguousarray(L["codes"][rows])
    sc = np.ascontiguousarray(L["scales"][rows])
    y_ref = oracle.gemv_f64(codes, L["codebooks"], sc, L["x"], len(rows), d_in, 8, 2, 8)
    W = oracle.dequant_f64(codes, L["codebooks"], sc, len(rows), d_in, 8, 2, 8)
    check_fp_output(y.cpu().numpy()[:, rows], y_ref, W, L["x"].astype(np.float64), out_rel=2.0 ** -10,
                    acc_rel=2.0 ** -14)


def test_gemv_lut_rejects_other_formats():
    for M, B in ((1, 16), (2, 16)):
        d = to_dev(make_layer(LayerSpec(64, 512, M, B), seed=1, tokens=1))
        with pytest.raises(ac.AqlmError):
            ac.aqlm_gemv_lut(d["codes"], d["codebooks"], d["scales"], d["x"])


@pytest.mark.parametrize("T", [4, 5, 16])
def test_gemv_tensor_core_ragged_stage(T):
    # 2x16 with 516 groups: the last 8-group stage of the tensor-core path holds
    # 4 groups (the rest are zeros in the decoded tile); 300 rows: 3 row tiles,
    # the last ragged
    _gemv_case(2, 16, 300, 4128, T, seed=50 + T)


@pytest.mark.parametrize("M,B", FORMATS)
def test_gemv_check_reports_ok(M, B):
    spec = LayerSpec(256, 1024, M, B)
    for T in (1, 8):
        d = to_dev(make_layer(spec, seed=60 + T, tokens=T))
        need = ac.gemv_workspace_bytes(ac.shape_of(d["codes"]), T)
        ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
        ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], d["x"], workspace=ws)
        assert ac.aqlm_gemv_check(d["codes"], T, ws) == ac.AQLM_OK


def test_gemv_one_hot_returns_columns():
    """x = e_c returns column c of s . W^ (exact up to the fp16 rounding)."""
    spec = LayerSpec(64, 512, 1, 16)
    L = make_layer(spec, seed=5, tokens=0)
    W = oracle_W(L, spec)
    x = np.zeros((4, 512), dtype=np.float16)
    cols = [0, 7, 300, 511]
    for t, c in enumerate(cols):
        x[t, c] = 1.0
    d = to_dev(L)
    y = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], torch.from_numpy(x).to(DEV)).cpu().numpy()
    for t, c in enumerate(cols):
        assert np.array_equal(y[t], W[:, c].astype(np.float16))


def test_gemv_two_calls_identical():
    spec = LayerSpec(4096, 4096, 1, 16)
    d = to_dev(make_layer(spec, seed=6, tokens=1))
    a = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], d["x"])
    b = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert torch.equal(a, b)


@pytest.mark.parametrize("M,B", FORMATS)
@pytest.mark.parametrize("T", [1, 8])
def test_gemv_chain_reads_x_after_the_producer(M, B, T):
    """Back-to-back layers where each x is the previous layer's y (programmatic
    dependent launch must not read x early), with a torch kernel in between."""
    specs = [LayerSpec(1024, 512, M, B), LayerSpec(512, 1024, M, B), LayerSpec(1024, 512, M, B)]
    Ls = [make_layer(s, seed=40 + k, tokens=T if k == 0 else 0) for k, s in enumerate(specs)]
    ds = [to_dev(L) for L in Ls]
    x = ds[0]["x"]
    ys = []
    for k, d in enumerate(ds):
        y = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], x)
        ys.append(y)
        x = y * 0.5 if k == 0 else y      # a torch kernel between the first two layers
    torch.cuda.synchronize()
    xin = [Ls[0]["x"], (ys[0] * 0.5).cpu().numpy(), ys[1].cpu().numpy()]
    for k, (L, s) in enumerate(zip(Ls, specs)):
        y_ref = oracle.gemv_f64(L["codes"], L["codebooks"], L["scales"], xin[k], s.d_out, s.d_in, 8, M, B)
        check_fp_output(ys[k].cpu().numpy(), y_ref, oracle_W(L, s), xin[k].astype(np.float64),
                        out_rel=2.0 ** -10, acc_rel=2.0 ** -14)


FULL_GEMV = [
    ("1x16 4096x4096", 4096, 4096, 1, 16, 1),
    ("2x8 4096x4096", 4096, 4096, 2, 8, 1),
    ("1x16 11008x4096", 11008, 4096, 1, 16, 1),
    ("2x8 4096x11008", 4096, 11008, 2, 8, 1),
    ("1x16 28672x8192 T4", 28672, 8192, 1, 16, 4),
    ("1x16 8192x28672 T4", 8192, 28672, 1, 16, 4),
    ("1x16 8192x28672 T3", 8192, 28672, 1, 16, 3),
    ("2x8 8192x28672 T4", 8192, 28672, 2, 8, 4),
    ("1x16 8192x28672 T16", 8192, 28672, 1, 16, 16),
    ("2x16 8192x8192", 8192, 8192, 2, 16, 1),
    ("2x8 256x512", 256, 512, 2, 8, 1),
]


@pytest.mark.parametrize("name,d_out,d_in,M,B,T", FULL_GEMV, ids=[c[0] for c in FULL_GEMV])
def test_gemv_full_size_sampled_rows(name, d_out, d_in, M, B, T):
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=0, tokens=T)
    d = to_dev(L)
    y = ac.aqlm_gemv(d["codes"], d["codebooks"], d["scales"], d["x"]).cpu().numpy()
    rng = np.random.Generator(np.random.PCG64(123))
    rows = np.unique(np.concatenate([rng.choice(d_out, size=min(d_out, 256), replace=False), [0, d_out - 1]]))
    sub = {"codes": np.ascontiguousarray(L["codes"][rows]), "codebooks": L["codebooks"],
           "scales": np.ascontiguousarray(L["scales"][rows])}
    y_ref = oracle.gemv_f64(sub["codes"], sub["codebooks"], sub["scales"], L["x"], len(rows), d_in, 8, M, B)
    W = oracle.dequant_f64(sub["codes"], sub["codebooks"], sub["scales"], len(rows), d_in, 8, M, B)
    check_fp_output(y[:, rows], y_ref, W, L["x"].astype(np.float64), out_rel=2.0 ** -10, acc_rel=2.0 ** -14)


# ---------------------------------------------------------------- gemm

def _gemm_check(Y, L, spec, X_bits, tokens_idx=None):
    """Y [T, d_out] bf16 against (1) the exact layer and (2) the bf16-rounded W^."""
    X64 = oracle.bf16_bits_to_f64(X_bits)
    W_exact = oracle_W(L, spec)
    Wb = oracle.bf16_bits_to_f64(oracle.dequant_bf16(L["codes"], L["codebooks"], L["scales"],
                                                     spec.d_out, spec.d_in, 8, spec.M, spec.B))
    if tokens_idx is not None:
        X64 = X64[tokens_idx]
        Y = Y[tokens_idx]
    y_exact = oracle.matmul_f64(W_exact, X64)
    y_bw = oracle.matmul_f64(Wb, X64)
    Yf = oracle.bf16_bits_to_f64(Y)
    # stated tolerance against the exact layer
    check_fp_output(Yf, y_exact, W_exact, X64, out_rel=1.0, acc_rel=1.0)
    # the tensor-core product of the bf16 operands: one bf16 rounding + fp32 accumulation
    check_fp_output(Yf, y_bw, Wb, X64, out_rel=2.0 ** -8, acc_rel=2.0 ** -14)


@pytest.mark.parametrize("M,B", FORMATS)
@pytest.mark.parametrize("tokens,d_out,d_in", [(200, 520, 576), (256, 512, 1024), (130, 264, 64)])
def test_gemm_small(M, B, tokens, d_out, d_in):
    if (d_in // 8 * M * B // 8) % 16:
        pytest.skip("row of codes not 16-byte aligned")
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=30 + tokens, tokens=tokens, x_dtype="bf16")
    d = to_dev(L)
    Y, ws = ac.aqlm_gemm(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ac.aqlm_gemm_check(ws) == ac.AQLM_OK
    _gemm_check(bf16_to_np_bits(Y), L, spec, L["x"])


# (tokens, d_out, d_in): bands (256 / 240 / 224 / 192 rows) with a ragged last
# band, k blocks with a ragged last one, one and several pair tiles, widths
# chosen by the rule on 148 SMs (so 4608 outputs take 256-wide tiles)
OVERLAP_CASES = [(200, 520, 576), (256, 512, 1024), (130, 264, 64), (1000, 4608, 1032), (2040, 4096, 520),
                 (1530, 4864, 520), (300, 1000, 4104), (100, 264, 576), (2048, 11008, 4096)]


@pytest.mark.parametrize("M,B", FORMATS)
@pytest.mark.parametrize("tokens,d_out,d_in", OVERLAP_CASES, ids=[f"{t}x{o}x{i}" for t, o, i in OVERLAP_CASES])
def test_gemm_overlapped_decode_equals_two_kernels(M, B, tokens, d_out, d_in):
    """aqlm_gemm_overlap decodes W^ inside the CTA-pair GEMM (decoder warps of
    every CTA, loads gated by per-panel counters).  The W^ it leaves in the
    workspace equals aqlm_dequant's bit for bit, and Y equals the CTA-pair
    GEMM of that W^ at the same width bit for bit, and aqlm_gemm's Y;
    sampled tokens against the oracle."""
    if (d_in // 8 * M * B // 8) % 16:
        pytest.skip("row of codes not 16-byte aligned")
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=60 + tokens + d_in, tokens=tokens, x_dtype="bf16")
    d = to_dev(L)
    Y, ws = ac.aqlm_gemm_overlap(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ac.aqlm_gemm_check(ws) == ac.AQLM_OK
    W_ws = ws[ws.numel() - 2 * d_out * d_in:].view(torch.int16).view(d_out, d_in)
    W_ref = ac.aqlm_dequant(d["codes"], d["codebooks"], d["scales"])
    torch.cuda.synchronize()
    assert torch.equal(W_ws, W_ref.view(torch.int16))
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    width = ac.bf16_gemm_plan(max(tokens, 129), d_out, sms)[1]   # the pair rule's width, at any token count
    Y2, st2 = ac.aqlm_bf16_gemm_config(d["x"], W_ref, 1, width)
    Y3, ws3 = ac.aqlm_gemm(d["codes"], d["codebooks"], d["scales"], d["x"])
    torch.cuda.synchronize()
    assert int(st2.item()) == 0 and ac.aqlm_gemm_check(ws3) == ac.AQLM_OK
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    assert torch.equal(Y.view(torch.int16), Y3.view(torch.int16))
    toks = np.unique(np.array([0, 1, tokens // 2, tokens - 1]))
    _gemm_check(bf16_to_np_bits(Y), L, spec, L["x"], tokens_idx=toks)


@pytest.mark.parametrize("M,B", FORMATS)
def test_gemm_overlap_and_pair_repeatable(M, B):
    """Cross-CTA protocols under repetition: 12 calls of aqlm_gemm_overlap
    (units claimed from global counters, handed to the publisher warp,
    panels counted, TMA loads gated on the counts) and of the CTA-pair GEMM
    leave the same Y bit for bit every time; a load that ran ahead of its
    panel's stores, or a pair whose halves lost step, would not."""
    spec = LayerSpec(4864, 1088, M, B)   # 4864 = 20.3 bands of 240; 17 k blocks
    L = make_layer(spec, seed=77, tokens=1530, x_dtype="bf16")
    d = to_dev(L)
    ws = torch.empty(ac.gemm_workspace_bytes(ac.shape_of(d["codes"]), 1530), dtype=torch.uint8, device=DEV)
    Y0, _ = ac.aqlm_gemm_overlap(d["codes"], d["codebooks"], d["scales"], d["x"], workspace=ws)
    assert ac.aqlm_gemm_check(ws) == ac.AQLM_OK
    W = ac.aqlm_dequant(d["codes"], d["codebooks"], d["scales"])
    P0, st = ac.aqlm_bf16_gemm_config(d["x"], W, 1, 0)
    for _ in range(12):
        Y, _ = ac.aqlm_gemm_overlap(d["codes"], d["codebooks"], d["scales"], d["x"], workspace=ws)
        P, st2 = ac.aqlm_bf16_gemm_config(d["x"], W, 1, 0)
        torch.cuda.synchronize()
        assert ac.aqlm_gemm_check(ws) == ac.AQLM_OK and int(st2.item()) == 0
        assert torch.equal(Y.view(torch.int16), Y0.view(torch.int16))
        assert torch.equal(P.view(torch.int16), P0.view(torch.int16))
    assert torch.equal(Y0.view(torch.int16), P0.view(torch.int16))


@pytest.mark.parametrize("tokens,n,k", [(200, 520, 576), (128, 256, 65536), (130, 264, 64)])
def test_bf16_gemm_ragged_and_deep(tokens, n, k):
    """Ragged tiles in every dimension (200 x 520 x 576), one tile with a long
    k loop (1024 k blocks), and a single k block: against torch (fp32
    accumulation), and bit-identical from call to call."""
    g = torch.Generator(device="cpu").manual_seed(tokens + n)
    X = (torch.randn(tokens, k, generator=g) / 4).to(torch.bfloat16).to(DEV)
    W = (torch.randn(n, k, generator=g) / 4).to(torch.bfloat16).to(DEV)
    Y1, s1 = ac.aqlm_bf16_gemm(X, W)
    Y2, s2 = ac.aqlm_bf16_gemm(X, W)
    torch.cuda.synchronize()
    assert int(s1.item()) == 0 and int(s2.item()) == 0
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    ref = X.float() @ W.float().T
    absdot = X.float().abs() @ W.float().abs().T
    err = (Y1.float() - ref).abs()
    assert bool(torch.all(err <= 2.0 ** -8 * ref.abs() + 2.0 ** -14 * absdot + 1e-6))


# (tokens, n, k) whose tile width on 148 SMs is each of the four (ragged
# tokens, n and k in every case)
TILE_WIDTH_CASES = [(1000, 4608, 1032, 256), (2040, 4096, 520, 240), (1530, 4864, 520, 224), (300, 1000, 4104, 192)]


@pytest.mark.parametrize("tokens,n,k,width", TILE_WIDTH_CASES, ids=[f"BN{c[3]}" for c in TILE_WIDTH_CASES])
def test_bf16_gemm_every_tile_width(tokens, n, k, width):
    """Each instantiation of the tile width of the single-CTA kernel (128x256,
    128x240, 128x224, 128x192 output tiles) against torch (fp32
    accumulation), including the partial last column tile and the 16-column
    remainder of the 240 / 224 epilogue."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if sms == 148:
        assert ac.bf16_gemm_tile_n(tokens, n, sms) == width
    g = torch.Generator(device="cpu").manual_seed(tokens + n + k)
    X = (torch.randn(tokens, k, generator=g) / 4).to(torch.bfloat16).to(DEV)
    W = (torch.randn(n, k, generator=g) / 4).to(torch.bfloat16).to(DEV)
    Y, status = ac.aqlm_bf16_gemm_config(X, W, 0, 0)
    assert int(status.item()) == 0
    ref = X.float() @ W.float().T
    absdot = X.float().abs() @ W.float().abs().T
    err = (Y.float() - ref).abs()
    assert bool(torch.all(err <= 2.0 ** -8 * ref.abs() + 2.0 ** -14 * absdot + 1e-6))


# (tokens, n, k): one pair tile; ragged tokens (the second CTA's rows partly
# and wholly past the end), n and k; a long k loop
PAIR_CASES = [(256, 256, 64), (200, 520, 576), (130, 264, 1032), (1000, 4608, 1032), (300, 1000, 4104),
              (2040, 4096, 520), (384, 512, 16384)]


@pytest.mark.parametrize("width", [256, 240, 224, 192])
@pytest.mark.parametrize("tokens,n,k", PAIR_CASES, ids=[f"{t}x{n}x{k}" for t, n, k in PAIR_CASES])
def test_bf16_gemm_cta_pair_every_width(tokens, n, k, width):
    """The CTA-pair kernel (256 x width tiles, one MMA on the tensor cores of
    two SMs) at each width: against torch (fp32 accumulation), and bit for
    bit against the single-CTA kernel at the same width (the same MMA k
    steps in the same order for every output element)."""
    g = torch.Generator(device="cpu").manual_seed(3 * tokens + n + k)
    X = (torch.randn(tokens, k, generator=g) / 4).to(torch.bfloat16).to(DEV)
    W = (torch.randn(n, k, generator=g) / 4).to(torch.bfloat16).to(DEV)
    Y, status = ac.aqlm_bf16_gemm_config(X, W, 1, width)
    Y1, status1 = ac.aqlm_bf16_gemm_config(X, W, 0, width)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and int(status1.item()) == 0
    ref = X.float() @ W.float().T
    absdot = X.float().abs() @ W.float().abs().T
    err = (Y.float() - ref).abs()
    assert bool(torch.all(err <= 2.0 ** -8 * ref.abs() + 2.0 ** -14 * absdot + 1e-6))
    assert torch.equal(Y.view(torch.int16), Y1.view(torch.int16))


def test_bf16_gemm_matches_torch():
    """The plain tensor-core GEMM against torch.matmul (fp32 accumulation) as a yardstick."""
    g = torch.Generator(device="cpu").manual_seed(7)
    X = torch.randn(384, 1536, generator=g).to(torch.bfloat16).to(DEV)
    W = torch.randn(768, 1536, generator=g).to(torch.bfloat16).to(DEV)
    Y, status = ac.aqlm_bf16_gemm(X, W)
    ref = (X.float() @ W.float().T)
    assert int(status.item()) == 0
    err = (Y.float() - ref).abs()
    # one bf16 rounding of the output (half an ulp, 2^-8 relative) plus fp32
    # accumulation over k = 1536 terms
    absdot = X.float().abs() @ W.float().abs().T
    assert bool(torch.all(err <= 2.0 ** -8 * ref.abs() + 2.0 ** -14 * absdot + 1e-6))


PREFILL = [(11008, 4096, 1, 16), (4096, 11008, 2, 8), (11008, 4096, 2, 8), (4096, 11008, 1, 16)]


@pytest.mark.parametrize("d_out,d_in,M,B", PREFILL, ids=[f"{m}x{b} {o}x{i}" for o, i, m, b in PREFILL])
def test_gemm_full_size_sampled_tokens(d_out, d_in, M, B):
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=0, tokens=2048, x_dtype="bf16")
    d = to_dev(L)
    Y, ws = ac.aqlm_gemm(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ac.aqlm_gemm_check(ws) == ac.AQLM_OK
    rng = np.random.Generator(np.random.PCG64(321))
    toks = np.unique(np.concatenate([rng.choice(2048, size=12, replace=False), [0, 127, 128, 2047]]))
    _gemm_check(bf16_to_np_bits(Y), L, spec, L["x"], tokens_idx=toks)


@pytest.mark.parametrize("M,B", FORMATS)
@pytest.mark.parametrize("tokens,d_out,d_in", [(200, 520, 576), (256, 512, 1024), (130, 264, 64), (128, 256, 160)])
def test_gemm_fused_small(M, B, tokens, d_out, d_in):
    """The fused prefill (W^ decoded inside the GEMM) against the oracle, and
    bit for bit against aqlm_gemm (the same binary32 decoding, the same MMAs);
    160 inputs in 2x16 end on a stage of 4 groups."""
    if (d_in // 8 * M * B // 8) % 16:
        pytest.skip("row of codes not 16-byte aligned")
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=40 + tokens, tokens=tokens, x_dtype="bf16")
    d = to_dev(L)
    Y, ws = ac.aqlm_gemm_fused(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ws.numel() == 256 and ac.aqlm_gemm_check(ws) == ac.AQLM_OK
    Y2, ws2 = ac.aqlm_gemm(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ac.aqlm_gemm_check(ws2) == ac.AQLM_OK
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    _gemm_check(bf16_to_np_bits(Y), L, spec, L["x"])


# (tokens, d_out) whose tile width on 148 SMs is each of the four
FUSED_WIDTH_CASES = [(1000, 4608, 256), (2040, 4096, 240), (1530, 4864, 224), (300, 1000, 192)]


@pytest.mark.parametrize("tokens,d_out,width", FUSED_WIDTH_CASES, ids=[f"BN{c[2]}" for c in FUSED_WIDTH_CASES])
@pytest.mark.parametrize("M,B", [(2, 8), (1, 16)])
def test_gemm_fused_every_tile_width(tokens, d_out, width, M, B):
    """Each tile width of the fused kernel (its decoders fill 256, 240, 224 or
    192 rows of every B tile) equals aqlm_gemm bit for bit; sampled tokens
    against the oracle."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if sms == 148:
        assert ac.bf16_gemm_tile_n(tokens, d_out, sms) == width
    spec = LayerSpec(d_out, 512, M, B)
    L = make_layer(spec, seed=50 + tokens, tokens=tokens, x_dtype="bf16")
    d = to_dev(L)
    Y, ws = ac.aqlm_gemm_fused(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ac.aqlm_gemm_check(ws) == ac.AQLM_OK
    Y2, ws2 = ac.aqlm_gemm(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ac.aqlm_gemm_check(ws2) == ac.AQLM_OK
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    toks = np.array([0, 1, tokens // 2, tokens - 1])
    _gemm_check(bf16_to_np_bits(Y), L, spec, L["x"], tokens_idx=toks)


@pytest.mark.parametrize("d_out,d_in,M,B", [(11008, 4096, 2, 8), (4096, 11008, 1, 16)], ids=["2x8", "1x16"])
def test_gemm_fused_full_size_sampled_tokens(d_out, d_in, M, B):
    spec = LayerSpec(d_out, d_in, M, B)
    L = make_layer(spec, seed=0, tokens=2048, x_dtype="bf16")
    d = to_dev(L)
    Y, ws = ac.aqlm_gemm_fused(d["codes"], d["codebooks"], d["scales"], d["x"])
    assert ac.aqlm_gemm_check(ws) == ac.AQLM_OK
    rng = np.random.Generator(np.random.PCG64(321))
    toks = np.unique(np.concatenate([rng.choice(2048, size=12, replace=False), [0, 127, 128, 2047]]))
    _gemm_check(bf16_to_np_bits(Y), L, spec, L["x"], tokens_idx=toks)


@pytest.mark.parametrize("cta_pair", [0, 1], ids=["single", "pair"])
def test_gemm_bounded_wait_reports_timeout(cta_pair):
    """Loads withheld on purpose: the first wait runs out, the kernel records
    AQLM_ERR_TIMEOUT, frees its tensor memory and returns (with the CTA pair,
    the other CTA's waits end on the abort flag the leader raises in it); the
    context stays usable."""
    X = torch.zeros(256, 64, dtype=torch.bfloat16, device=DEV)
    W = torch.zeros(256, 64, dtype=torch.bfloat16, device=DEV)
    Y = torch.empty(256, 256, dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert ac.aqlm_test_gemm_timeout(X, W, Y, status, 20_000_000, cta_pair) == ac.AQLM_OK
    torch.cuda.synchronize()
    assert int(status.item()) == ac.AQLM_ERR_TIMEOUT
    # the device still works, and a normal GEMM afterwards is correct
    Y2, st2 = ac.aqlm_bf16_gemm_config(torch.ones(256, 64, dtype=torch.bfloat16, device=DEV),
                                       torch.ones(256, 64, dtype=torch.bfloat16, device=DEV), cta_pair, 0)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0 and torch.all(Y2.float() == 64.0)


# ---------------------------------------------------------------- several layers, one launch

@pytest.mark.parametrize("M,B", FORMATS)
@pytest.mark.parametrize("d_in,split", [(4096, False), (28736, True)])
def test_gemv_multi_matches_single_layer_calls(M, B, d_in, split):
    """Layers that read the same x (ragged row counts, q/k/v-like) in one
    launch, within the tolerance of the oracle.  On the row kernel (up to
    aqlm_gemv_row_tokens) each y_l is also bit-for-bit aqlm_gemv's on that
    layer; with 28736 inputs the activations are split over several CTAs per
    row, whose partial sums meet in the shared workspace.  Past that the
    tensor-core kernel runs the layers' row tiles as one work split (its split
    points differ from a single layer's, so only the tolerance applies) and
    aqlm_gemv_multi_check reports no timeout."""
    d_outs = [300, 1000, 77]
    specs = [LayerSpec(n, d_in, M, B) for n in d_outs]
    shape0 = ac.shape_of(torch.empty((1, d_in // 8, M), dtype=torch.uint8 if B == 8 else torch.int16))
    T_max = ac.gemv_row_tokens(shape0)
    for T in sorted({1, T_max, T_max + 1, 16}):
        Ls = [make_layer(s, seed=70 + 3 * k + T, tokens=T if k == 0 else 0) for k, s in enumerate(specs)]
        x = Ls[0]["x"]
        ds = [to_dev(L) for L in Ls]
        xd = torch.from_numpy(x).to(DEV)
        layers = [{"codes": d["codes"], "codebooks": d["codebooks"], "scales": d["scales"]} for d in ds]
        if split:
            assert ac.gemv_multi_workspace_bytes(layers, T) > 0
        need = ac.gemv_multi_workspace_bytes(layers, T)
        ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=DEV)
        ys = ac.aqlm_gemv_multi(layers, xd, workspace=ws if need else None)
        if T > T_max:
            assert ac.aqlm_gemv_multi_check(layers, T, ws) == ac.AQLM_OK
        for k, (L, s) in enumerate(zip(Ls, specs)):
            if T <= T_max:
                single = ac.aqlm_gemv(ds[k]["codes"], ds[k]["codebooks"], ds[k]["scales"], xd)
                assert torch.equal(ys[k].view(torch.int16), single.view(torch.int16)), (k, T)
            y_ref = oracle.gemv_f64(L["codes"], L["codebooks"], L["scales"], x, s.d_out, d_in, 8, M, B)
            check_fp_output(ys[k].cpu().numpy(), y_ref, oracle_W(L, s), x.astype(np.float64),
                            out_rel=2.0 ** -10, acc_rel=2.0 ** -14)


def test_gemv_multi_one_layer_and_four_layers():
    spec = LayerSpec(512, 1024, 1, 16)
    Ls = [make_layer(spec, seed=90 + k, tokens=2 if k == 0 else 0) for k in range(4)]
    ds = [to_dev(L) for L in Ls]
    xd = torch.from_numpy(Ls[0]["x"]).to(DEV)
    for n in (1, 4):
        ys = ac.aqlm_gemv_multi(ds[:n], xd)
        for k in range(n):
            single = ac.aqlm_gemv(ds[k]["codes"], ds[k]["codebooks"], ds[k]["scales"], xd)
            assert torch.equal(ys[k].view(torch.int16), single.view(torch.int16))
