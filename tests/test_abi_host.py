"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/aqlm.h declares, and rejects bad arguments on the
host before any CUDA call (validation never dereferences the pointers, so
fake addresses are safe here)."""
import ctypes
import os
import re

import pytest

import additive_codebook_b200 as ac

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "aqlm.h")).read()
    return re.findall(r"^AQLM_API\s+[\w\s\*]+?\b(aqlm_\w+)\s*\(", text, flags=re.M)


def test_header_and_binding_agree():
    names = header_functions()
    assert len(names) == len(set(names)) and sorted(names) == sorted(ac.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ac.load_library()
    for name in header_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings_and_version():
    assert ac.status_string(ac.AQLM_OK) == "AQLM_OK"
    assert ac.status_string(ac.AQLM_ERR_TIMEOUT) == "AQLM_ERR_TIMEOUT"
    assert ac.status_string(99) == "AQLM_ERR_UNKNOWN"
    assert re.match(r"^\d+\.\d+\.\d+$", ac.version())


A16 = ctypes.c_void_p(0x10000)   # 16-byte aligned fake device addresses
B16 = ctypes.c_void_p(0x20000)
C16 = ctypes.c_void_p(0x30000)
D16 = ctypes.c_void_p(0x40000)
E16 = ctypes.c_void_p(0x50000)
NULL = ctypes.c_void_p(0)
ODD = ctypes.c_void_p(0x10008)


def shape(d_out=256, d_in=512, M=2, B=8, g=8):
    return ac.Shape(d_out, d_in, g, M, B)


@pytest.mark.parametrize("kw,status", [
    (dict(g=4), ac.AQLM_ERR_UNSUPPORTED),
    (dict(M=3, B=8), ac.AQLM_ERR_UNSUPPORTED),
    (dict(M=1, B=8), ac.AQLM_ERR_UNSUPPORTED),
    (dict(M=2, B=12), ac.AQLM_ERR_UNSUPPORTED),
    (dict(d_in=500), ac.AQLM_ERR_UNSUPPORTED),
    (dict(d_in=520), ac.AQLM_ERR_MISALIGNED),          # 65 groups x 2 bytes: row not a 16-byte multiple
    (dict(d_out=0), ac.AQLM_ERR_INVALID_ARG),
    (dict(d_in=0), ac.AQLM_ERR_INVALID_ARG),
    (dict(d_out=1 << 21), ac.AQLM_ERR_INVALID_ARG),
])
def test_shape_validation(kw, status):
    lib = ac.load_library()
    s = shape(**kw)
    # every case fails validation, so nothing is launched with the fake pointers
    assert lib.aqlm_gemv(A16, B16, C16, D16, E16, 1, s, NULL, 0, NULL) == status


def test_gemv_argument_errors():
    lib = ac.load_library()
    s = shape()
    assert lib.aqlm_gemv(NULL, B16, C16, D16, E16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv(A16, NULL, C16, D16, E16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv(A16, B16, NULL, D16, E16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv(A16, B16, C16, NULL, E16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv(A16, B16, C16, D16, NULL, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv(A16, B16, C16, D16, E16, 0, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv(A16, B16, C16, D16, E16, 17, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv(ODD, B16, C16, D16, E16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_MISALIGNED
    assert lib.aqlm_gemv(A16, ODD, C16, D16, E16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_MISALIGNED
    assert lib.aqlm_gemv(A16, B16, C16, ODD, E16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_MISALIGNED


def test_gemv_workspace_rules():
    lib = ac.load_library()
    big = ac.Shape(8192, 8192, 8, 1, 16)
    assert lib.aqlm_gemv_workspace_bytes(big, 1) == 0          # enough row tiles: no split
    assert lib.aqlm_gemv_workspace_bytes(shape(M=1, B=16), 1) == 0   # one token: whole rows per warp
    assert lib.aqlm_gemv_workspace_bytes(shape(), 1) == 0      # 2x8, one token: 2 KiB of activations
    # aqlm_gemv_lut keeps one fp32 sum per row and group of slabs that a CTA
    # covers (plus a counter per row range); a 4096x4096 layer takes one slab
    # of 32 groups per CTA (16 sums per row); rows of one slab need none
    assert lib.aqlm_gemv_lut_workspace_bytes(shape(d_out=4096, d_in=4096)) >= 16 * 4096 * 4
    assert lib.aqlm_gemv_lut_workspace_bytes(shape(d_in=256)) == 0
    assert lib.aqlm_gemv_lut_workspace_bytes(shape(M=1, B=16)) == 0
    assert lib.aqlm_gemv_lut(A16, B16, C16, D16, E16, shape(M=1, B=16), NULL, 0, NULL) == ac.AQLM_ERR_UNSUPPORTED
    assert lib.aqlm_gemv_lut(A16, B16, C16, D16, E16, shape(d_out=4096, d_in=4096), NULL, 0, NULL) == \
        ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemv_lut(NULL, B16, C16, D16, E16, shape(), NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    wide = shape(d_in=4096)                                    # 8 tokens, 2 row tiles: split to fill the SMs
    assert lib.aqlm_gemv_workspace_bytes(shape(d_in=4096, M=1, B=16), 2) == 0   # 16 KiB of activations: one slice
    small = lib.aqlm_gemv_workspace_bytes(wide, 8)
    assert small >= 2 * 8 * 256 * 4
    assert lib.aqlm_gemv(A16, B16, C16, D16, E16, 8, wide, NULL, 0, NULL) == ac.AQLM_ERR_WORKSPACE
    need = lib.aqlm_gemv_workspace_bytes(big, 16)
    assert need >= 2 * 16 * 8192 * 4            # at least two splits of fp32 partial sums
    assert lib.aqlm_gemv(A16, B16, C16, D16, E16, 16, big, NULL, 0, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemv(A16, B16, C16, D16, E16, 16, big, A16, need - 4, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemv(A16, B16, C16, D16, E16, 16, big, ODD, need, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemv_workspace_bytes(big, 0) == 0 and lib.aqlm_gemv_workspace_bytes(big, 17) == 0
    # the row kernel (1x16 up to 2 tokens, 2x16 up to 3, 2x8 up to 4) splits the
    # input range only when T * d_in fp16 activations exceed its shared-memory
    # budget (32 KiB), in slices of whole 32-chunk lane slots (448 chunks of 16
    # bytes per 8192x28672 row in 1x16 and 2x8)
    down = ac.Shape(8192, 28672, 8, 1, 16)
    down8 = ac.Shape(8192, 28672, 8, 2, 8)
    assert lib.aqlm_gemv_workspace_bytes(down, 1) >= 2 * 1 * 8192 * 4   # 56 KiB: two slices of 224 chunks
    assert lib.aqlm_gemv_workspace_bytes(down, 2) >= 4 * 2 * 8192 * 4   # 112 KiB: four slices of 128
    assert lib.aqlm_gemv_workspace_bytes(down8, 3) >= 7 * 3 * 8192 * 4  # 168 KiB: seven slices of 64
    assert lib.aqlm_gemv_workspace_bytes(down8, 4) >= 7 * 4 * 8192 * 4  # 224 KiB: seven slices of 64
    assert lib.aqlm_gemv(A16, B16, C16, D16, E16, 2, down, NULL, 0, NULL) == ac.AQLM_ERR_WORKSPACE
    # past those token counts: the tensor-core kernel, whose workspace always
    # holds a status word
    for s_, T in ((down, 3), (down, 16), (down8, 5), (ac.Shape(8192, 28672, 8, 2, 16), 4)):
        assert lib.aqlm_gemv_workspace_bytes(s_, T) >= 16
        assert lib.aqlm_gemv(A16, B16, C16, D16, E16, T, s_, NULL, 0, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemv_workspace_bytes(ac.Shape(8192, 16384, 8, 1, 16), 1) == 0   # exactly 32 KiB


def test_gemm_argument_errors():
    lib = ac.load_library()
    s = ac.Shape(4096, 4096, 8, 1, 16)
    need = lib.aqlm_gemm_workspace_bytes(s, 2048)
    # status word, the overlapped decoding's counters (8 claim words on their
    # own 128-byte lines + one per 192-row band and k block, k blocks padded
    # to a multiple of 32), the bf16 W^
    counters = 1024 + -(-(-(-4096 // 192) * 64 * 4) // 256) * 256
    assert need == 256 + counters + 4096 * 4096 * 2
    assert lib.aqlm_gemm(A16, B16, C16, D16, E16, 2048, s, NULL, 0, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemm(A16, B16, C16, D16, E16, 2048, s, A16, need - 1, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemm(A16, B16, C16, D16, E16, 0, s, A16, need, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemm(A16, B16, C16, ODD, E16, 16, s, A16, need, NULL) == ac.AQLM_ERR_MISALIGNED
    s_odd = ac.Shape(4100, 4096, 8, 1, 16)
    assert lib.aqlm_gemm(A16, B16, C16, D16, E16, 16, s_odd, A16, 1 << 40, NULL) == ac.AQLM_ERR_UNSUPPORTED
    # the one-kernel prefill validates exactly as aqlm_gemm, with the same workspace
    assert lib.aqlm_gemm_overlap(A16, B16, C16, D16, E16, 2048, s, NULL, 0, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemm_overlap(A16, B16, C16, D16, E16, 2048, s, A16, need - 1, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemm_overlap(A16, B16, C16, D16, E16, 0, s, A16, need, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemm_overlap(A16, B16, C16, ODD, E16, 16, s, A16, need, NULL) == ac.AQLM_ERR_MISALIGNED
    assert lib.aqlm_gemm_overlap(A16, B16, C16, D16, E16, 16, s_odd, A16, 1 << 40, NULL) == ac.AQLM_ERR_UNSUPPORTED
    assert lib.aqlm_bf16_gemm(A16, B16, C16, 16, 100, 64, D16, NULL) == ac.AQLM_ERR_UNSUPPORTED
    assert lib.aqlm_bf16_gemm(A16, B16, C16, 16, 128, 64, NULL, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemm_check(NULL, 0, NULL) == ac.AQLM_ERR_WORKSPACE
    # the variant chooser: unknown kernels and widths are refused before any launch
    for pair, width in ((2, 0), (-2, 0), (1, 128), (0, 250), (0, 512)):
        assert lib.aqlm_bf16_gemm_config(A16, B16, C16, 256, 128, 64, D16, pair, width, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_bf16_gemm_config(A16, B16, C16, 256, 100, 64, D16, 1, 0, NULL) == ac.AQLM_ERR_UNSUPPORTED
    assert lib.aqlm_bf16_gemm_config(ODD, B16, C16, 256, 128, 64, D16, 1, 0, NULL) == ac.AQLM_ERR_MISALIGNED


def test_dequant_and_decode_argument_errors():
    lib = ac.load_library()
    s = shape()
    assert lib.aqlm_dequant(A16, B16, C16, NULL, s, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_dequant(A16, B16, C16, ODD, s, NULL) == ac.AQLM_ERR_MISALIGNED
    assert lib.aqlm_decode_indices(NULL, A16, s, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_decode_indices(A16, ctypes.c_void_p(0x10001), s, NULL) == ac.AQLM_ERR_MISALIGNED
    assert lib.aqlm_test_gemm_timeout(A16, B16, C16, 16, 128, 64, D16, 0, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_test_gemm_timeout(A16, B16, C16, 16, 128, 64, D16, 1000, 2, NULL) == ac.AQLM_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ac, "_lib", None)
    monkeypatch.setattr(ac, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        ac.load_library()


def test_row_tokens_per_format():
    lib = ac.load_library()
    assert lib.aqlm_gemv_row_tokens(shape(M=1, B=16)) == 2
    assert lib.aqlm_gemv_row_tokens(shape(M=2, B=16)) == 3
    assert lib.aqlm_gemv_row_tokens(shape(M=2, B=8)) == 4
    assert lib.aqlm_gemv_row_tokens(shape(M=3, B=8)) == 0
    assert lib.aqlm_gemv_row_tokens(shape(d_in=500)) == 0


def _multi(*d_outs, codes=A16, y=E16):
    arr = (ac.Layer * max(len(d_outs), 1))()
    for k, n in enumerate(d_outs):
        arr[k] = ac.Layer(codes.value, B16.value, C16.value, y.value if y.value else None, n)
    return arr


def test_gemv_multi_argument_errors():
    # every call fails validation on the host, so the fake pointers are never used
    lib = ac.load_library()
    s = shape(d_out=0)   # d_out of the common shape is ignored
    q = _multi(4096, 1024, 1024)
    assert lib.aqlm_gemv_multi(q, 0, D16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv_multi(_multi(8, 8, 8, 8, 8), 5, D16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv_multi(None, 1, D16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv_multi(q, 3, NULL, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv_multi(_multi(64, 0), 2, D16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv_multi(_multi(64, 64, y=NULL), 2, D16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv_multi(_multi(64, 64, codes=ODD), 2, D16, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_MISALIGNED
    assert lib.aqlm_gemv_multi(_multi(64, 64, y=ctypes.c_void_p(0x50001)), 2, D16, 1, s, NULL, 0, NULL) == \
        ac.AQLM_ERR_MISALIGNED
    assert lib.aqlm_gemv_multi(q, 3, ODD, 1, s, NULL, 0, NULL) == ac.AQLM_ERR_MISALIGNED
    assert lib.aqlm_gemv_multi(q, 3, D16, 0, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_gemv_multi(q, 3, D16, 17, s, NULL, 0, NULL) == ac.AQLM_ERR_INVALID_ARG
    # past the row kernel's token count: the tensor-core kernel, whose workspace holds a status word
    s16 = shape(d_out=0, d_in=4096, M=1, B=16)
    assert lib.aqlm_gemv_multi_workspace_bytes(q, 3, s16, 3) >= 16
    assert lib.aqlm_gemv_multi(q, 3, D16, 3, s16, NULL, 0, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemv_multi(q, 3, D16, 1, shape(d_out=0, M=3), NULL, 0, NULL) == ac.AQLM_ERR_UNSUPPORTED


def test_gemv_multi_workspace_rules():
    lib = ac.load_library()
    s = shape(d_out=0, d_in=4096, M=1, B=16)
    q = _multi(4096, 1024, 1024)
    assert lib.aqlm_gemv_multi_workspace_bytes(q, 3, s, 1) == 0       # 8 KiB of activations: no split
    assert lib.aqlm_gemv_multi_workspace_bytes(q, 3, s, 3) >= 16      # tensor cores: status word at least
    assert lib.aqlm_gemv_multi_workspace_bytes(q, 3, s, 17) == 0
    assert lib.aqlm_gemv_multi_workspace_bytes(q, 0, s, 1) == 0
    # 28672 inputs, 1 token: two activation slices; partials for all 6144
    # rows, then one counter per 8 rows of each layer
    wide = shape(d_out=0, d_in=28672, M=1, B=16)
    need = lib.aqlm_gemv_multi_workspace_bytes(q, 3, wide, 1)
    assert need == 2 * 1 * 6144 * 4 + (512 + 128 + 128) * 4
    assert lib.aqlm_gemv_multi(q, 3, D16, 1, wide, NULL, 0, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemv_multi(q, 3, D16, 1, wide, A16, need - 4, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_gemv_multi(q, 3, D16, 1, wide, ODD, need, NULL) == ac.AQLM_ERR_WORKSPACE
    # one layer: the same workspace as aqlm_gemv
    one = _multi(8192)
    assert lib.aqlm_gemv_multi_workspace_bytes(one, 1, wide, 2) == \
        lib.aqlm_gemv_workspace_bytes(ac.Shape(8192, 28672, 8, 1, 16), 2)


def test_encode_argument_errors():
    """The encoding entry points reject bad arguments on the host (nothing is
    launched, so the fake device addresses are never touched)."""
    lib = ac.load_library()
    s = shape(d_out=64, d_in=512, M=2, B=8)
    init_ok = (ctypes.c_int32 * (2 * 256))(*([3] * 512))
    init_bad = (ctypes.c_int32 * (2 * 256))(*([3] * 511 + [64 * 64]))   # one index past the 4096 groups
    ws = lib.aqlm_encode_layer_workspace_bytes(s)
    assert ws > 0 and lib.aqlm_encode_layer_workspace_bytes(shape(M=3)) == 0
    assert lib.aqlm_encode_layer(A16, s, init_bad, 2, B16, C16, D16, E16, ws, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_encode_layer(A16, s, None, 2, B16, C16, D16, E16, ws, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_encode_layer(A16, s, init_ok, -1, B16, C16, D16, E16, ws, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_encode_layer(ODD, s, init_ok, 2, B16, C16, D16, E16, ws, NULL) == ac.AQLM_ERR_MISALIGNED
    assert lib.aqlm_encode_layer(A16, s, init_ok, 2, B16, C16, D16, E16, ws - 1, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_encode_layer(A16, shape(M=3), init_ok, 2, B16, C16, D16, E16, ws, NULL) == \
        ac.AQLM_ERR_UNSUPPORTED
    assert lib.aqlm_encode_scales(A16, 64, 500, B16, C16, NULL) == ac.AQLM_ERR_UNSUPPORTED
    assert lib.aqlm_encode_scales(A16, 0, 512, B16, C16, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_encode_scales(ODD, 64, 512, B16, C16, NULL) == ac.AQLM_ERR_MISALIGNED
    nws = lib.aqlm_nearest_workspace_bytes(1000)
    assert nws >= 1000 * 8
    assert lib.aqlm_nearest_codeword(A16, 1000, B16, 0, C16, NULL, D16, nws, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_nearest_codeword(A16, 1000, B16, 256, C16, NULL, D16, nws - 8, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_nearest_codeword(ODD, 1000, B16, 256, C16, NULL, D16, nws, NULL) == ac.AQLM_ERR_MISALIGNED
    kws = lib.aqlm_kmeans_workspace_bytes(256)
    assert kws >= 256 * 8 * 8 + 256 * 4
    assert lib.aqlm_kmeans_update(A16, B16, 1000, C16, 256, D16, NULL, E16, kws - 1, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_kmeans_update(A16, B16, -1, C16, 256, D16, NULL, E16, kws, NULL) == ac.AQLM_ERR_INVALID_ARG
    rws = lib.aqlm_residual_kmeans_workspace_bytes(4096, 2, 256)
    assert lib.aqlm_residual_kmeans(A16, 4096, 2, 256, init_bad, 3, B16, C16, rws, NULL) == ac.AQLM_ERR_INVALID_ARG
    assert lib.aqlm_residual_kmeans(A16, 4096, 2, 256, init_ok, 3, B16, C16, rws - 1, NULL) == ac.AQLM_ERR_WORKSPACE
    cws = lib.aqlm_encode_codes_workspace_bytes(s)
    assert cws >= 4096 * 8 * 4 + 4096 * 8 + 2 * 256 * 8 * 4
    assert lib.aqlm_encode_codes(A16, B16, C16, s, D16, cws - 1, NULL) == ac.AQLM_ERR_WORKSPACE
    assert lib.aqlm_encode_codes(A16, B16, ODD, s, D16, cws, NULL) == ac.AQLM_ERR_MISALIGNED


def test_gemm_tile_width_rule():
    """The GEMM's tile width: least waves x (128 + width) over {256, 240, 224,
    192}, ties to the wider, checked against the rule restated here over a
    grid of shapes, and the prefill shapes on 148 SMs."""
    def rule(tokens, n, sms):
        best = None
        for bn in (256, 240, 224, 192):
            tiles = -(-tokens // 128) * -(-n // bn)
            cost = -(-tiles // sms) * (128 + bn)
            if best is None or cost < best[0]:
                best = (cost, bn)
        return best[1]
    for tokens in (1, 127, 128, 300, 1000, 2048, 4096):
        for n in (8, 256, 1000, 4096, 4608, 8192, 11008, 28672):
            for sms in (1, 132, 148):
                assert ac.bf16_gemm_tile_n(tokens, n, sms) == rule(tokens, n, sms)
    assert [ac.bf16_gemm_tile_n(2048, n, 148) for n in (11008, 4096, 8192, 28672)] == [240, 240, 224, 240]
    assert ac.bf16_gemm_tile_n(0, 8, 148) == 0 and ac.bf16_gemm_tile_n(8, 8, 0) == 0


def test_gemm_plan_rule():
    """The GEMM kernel choice: the CTA pair past 128 tokens, with the least
    waves x width over sms / 2 pairs of 256-token tiles (ties to the wider),
    the single-CTA kernel and its own rule up to 128 tokens; checked against
    the rule restated here over a grid of shapes."""
    def pair_rule(tokens, n, pairs):
        best = None
        for bn in (256, 240, 224, 192):
            tiles = -(-tokens // 256) * -(-n // bn)
            cost = -(-tiles // pairs) * bn
            if best is None or cost < best[0]:
                best = (cost, bn)
        return best[1]
    for tokens in (1, 128, 129, 300, 1000, 2048, 4096):
        for n in (8, 256, 1000, 4096, 4608, 8192, 11008, 28672):
            for sms in (2, 132, 148):
                pair, width = ac.bf16_gemm_plan(tokens, n, sms)
                if tokens <= 128:
                    assert (pair, width) == (0, ac.bf16_gemm_tile_n(tokens, n, sms))
                else:
                    assert (pair, width) == (1, pair_rule(tokens, n, sms // 2))
    assert [ac.bf16_gemm_plan(2048, n, 148) for n in (11008, 4096, 8192, 28672)] == [(1, 240), (1, 240), (1, 224), (1, 240)]
    lib = ac.load_library()
    p, w = ctypes.c_int32(7), ctypes.c_int32(7)
    assert lib.aqlm_bf16_gemm_plan(2048, 4096, 1, ctypes.byref(p), ctypes.byref(w)) == ac.AQLM_ERR_INVALID_ARG
    assert (p.value, w.value) == (0, 0)
    assert lib.aqlm_bf16_gemm_plan(2048, 4096, 148, None, ctypes.byref(w)) == ac.AQLM_ERR_INVALID_ARG


def test_debug_bounds_entry_points_in_the_product_build():
    """The product library answers the debug-bounds calls with
    AQLM_ERR_UNSUPPORTED (no device checks are compiled in); no CUDA call."""
    lib = ac.load_library()
    w = ctypes.c_uint64(1)
    assert lib.aqlm_debug_bounds_read(ctypes.byref(w), 1) == ac.AQLM_ERR_UNSUPPORTED and w.value == 0
    assert lib.aqlm_test_debug_bounds_trip(1, NULL) == ac.AQLM_ERR_UNSUPPORTED
    assert lib.aqlm_debug_bounds_read(None, 0) == ac.AQLM_ERR_INVALID_ARG


def test_library_builds_with_debug_bounds(tmp_path):
    """-DAQLM_DEBUG_BOUNDS still compiles and links every source, and the
    result exports every declared entry point."""
    from additive_codebook_b200 import build as cuda_build
    lib_path = cuda_build.build(force=True, debug_bounds=True, out_lib=str(tmp_path / "libdbg.so"),
                                objdir=str(tmp_path / "obj"))
    lib = ctypes.CDLL(lib_path)
    for name in ac.EXPORTS:
        assert hasattr(lib, name), name
