"""Python binding of the B200 AQLM library (include/aqlm.h), via ctypes.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libaqlm_b200.so.  torch provides device memory and the current
stream; outputs that the caller does not pass are allocated with torch.
There is no CPU fallback: if the library is missing the calls raise.

Layouts (see include/aqlm.h):
  codes      [d_out, d_in/8, M]  uint8 (B = 8) or int16 (B = 16, read unsigned)
  codebooks  [M, 2^B, 8]          float16
  scales     [d_out]              float16 (a [d_out, 1, 1, 1] tensor is accepted)
  x / y      [T, d_in] / [T, d_out] float16      (aqlm_gemv, T <= 16)
  X / Y      [T, d_in] / [T, d_out] bfloat16     (aqlm_gemm)
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libaqlm_b200.so")
DEBUG_BOUNDS_LIB_PATH = os.path.join(_HERE, "libaqlm_b200_debug_bounds.so")

AQLM_OK = 0
AQLM_ERR_INVALID_ARG = 1
AQLM_ERR_UNSUPPORTED = 2
AQLM_ERR_MISALIGNED = 3
AQLM_ERR_WORKSPACE = 4
AQLM_ERR_CUDA = 5
AQLM_ERR_TIMEOUT = 6
GEMV_MAX_TOKENS = 16

# Every entry point declared in include/aqlm.h.
EXPORTS = ["aqlm_gemv", "aqlm_gemv_workspace_bytes", "aqlm_gemv_row_tokens", "aqlm_gemv_multi",
           "aqlm_gemv_multi_workspace_bytes", "aqlm_gemv_multi_check", "aqlm_gemv_check", "aqlm_dequant", "aqlm_gemm",
           "aqlm_gemm_workspace_bytes", "aqlm_gemm_check", "aqlm_gemm_overlap", "aqlm_bf16_gemm", "aqlm_bf16_gemm_tile_n", "aqlm_bf16_gemm_plan", "aqlm_bf16_gemm_config", "aqlm_decode_indices",
           "aqlm_test_gemm_timeout", "aqlm_gemv_noalloc", "aqlm_gemv_noalloc_max_scratch_bytes",
           "aqlm_gemv_noalloc_check", "aqlm_test_gemv_noalloc_set_status", "aqlm_probe_gather_sink_bytes",
           "aqlm_probe_gather", "aqlm_gemv_lut", "aqlm_gemv_lut_workspace_bytes", "aqlm_gemm_fused",
           "aqlm_gemm_fused_workspace_bytes", "aqlm_debug_bounds_read", "aqlm_test_debug_bounds_trip",
           "aqlm_status_string", "aqlm_version",
           "aqlm_encode_scales", "aqlm_nearest_workspace_bytes", "aqlm_nearest_codeword",
           "aqlm_kmeans_workspace_bytes", "aqlm_kmeans_update", "aqlm_residual_kmeans_workspace_bytes",
           "aqlm_residual_kmeans", "aqlm_encode_codes_workspace_bytes", "aqlm_encode_codes",
           "aqlm_encode_layer_workspace_bytes", "aqlm_encode_layer"]


class AqlmError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


class Shape(ctypes.Structure):
    _fields_ = [("d_out", ctypes.c_int32), ("d_in", ctypes.c_int32), ("group", ctypes.c_int32),
                ("num_codebooks", ctypes.c_int32), ("codebook_bits", ctypes.c_int32)]


MULTI_MAX_LAYERS = 4


class Layer(ctypes.Structure):
    """aqlm_layer: one layer of an aqlm_gemv_multi call (device pointers)."""
    _fields_ = [("codes", ctypes.c_void_p), ("codebooks", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("d_out", ctypes.c_int32)]


_lib = None


def load_library():
    """Load libaqlm_b200.so and declare the C signatures (no CUDA call)."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = _open(LIB_PATH, "python -m additive_codebook_b200.build")
    return _lib


def load_debug_bounds_library():
    """The library built with device bounds checks (libaqlm_b200_debug_bounds.so),
    with the same C signatures; the module's functions keep using the product
    library unless a caller swaps it in."""
    return _open(DEBUG_BOUNDS_LIB_PATH, "python -m additive_codebook_b200.build --debug-bounds")


def _open(path, how):
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `{how}`")
    lib = ctypes.CDLL(path)
    vp, i32, sz, u64, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_int64
    st = ctypes.c_int
    sig = {
        "aqlm_gemv": ([vp, vp, vp, vp, vp, i32, Shape, vp, sz, vp], st),
        "aqlm_gemv_workspace_bytes": ([Shape, i32], sz),
        "aqlm_gemv_row_tokens": ([Shape], i32),
        "aqlm_gemv_multi": ([ctypes.POINTER(Layer), i32, vp, i32, Shape, vp, sz, vp], st),
        "aqlm_gemv_multi_workspace_bytes": ([ctypes.POINTER(Layer), i32, Shape, i32], sz),
        "aqlm_gemv_multi_check": ([ctypes.POINTER(Layer), i32, Shape, i32, vp, sz, vp], st),
        "aqlm_gemv_check": ([Shape, i32, vp, sz, vp], st),
        "aqlm_dequant": ([vp, vp, vp, vp, Shape, vp], st),
        "aqlm_gemm": ([vp, vp, vp, vp, vp, i32, Shape, vp, sz, vp], st),
        "aqlm_gemm_workspace_bytes": ([Shape, i32], sz),
        "aqlm_gemm_check": ([vp, sz, vp], st),
        "aqlm_bf16_gemm": ([vp, vp, vp, i32, i32, i32, vp, vp], st),
        "aqlm_bf16_gemm_tile_n": ([i32, i32, i32], i32),
        "aqlm_decode_indices": ([vp, vp, Shape, vp], st),
        "aqlm_bf16_gemm_plan": ([i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)], st),
        "aqlm_bf16_gemm_config": ([vp, vp, vp, i32, i32, i32, vp, i32, i32, vp], st),
        "aqlm_test_gemm_timeout": ([vp, vp, vp, i32, i32, i32, vp, u64, i32, vp], st),
        "aqlm_gemv_noalloc": ([vp, vp, vp, vp, vp, i32, Shape, vp], st),
        "aqlm_gemv_noalloc_max_scratch_bytes": ([], sz),
        "aqlm_gemv_noalloc_check": ([vp], st),
        "aqlm_test_gemv_noalloc_set_status": ([i32, vp], st),
        "aqlm_probe_gather_sink_bytes": ([i32], sz),
        "aqlm_gemv_lut": ([vp, vp, vp, vp, vp, Shape, vp, sz, vp], st),
        "aqlm_gemv_lut_workspace_bytes": ([Shape], sz),
        "aqlm_gemm_fused": ([vp, vp, vp, vp, vp, i32, Shape, vp, sz, vp], st),
        "aqlm_gemm_overlap": ([vp, vp, vp, vp, vp, i32, Shape, vp, sz, vp], st),
        "aqlm_gemm_fused_workspace_bytes": ([Shape, i32], sz),
        "aqlm_debug_bounds_read": ([ctypes.POINTER(u64), i32], st),
        "aqlm_test_debug_bounds_trip": ([u64, vp], st),
        "aqlm_probe_gather": ([vp, sz, i32, i32, i32, vp, sz, ctypes.POINTER(u64), vp], st),
        "aqlm_encode_scales": ([vp, i32, i32, vp, vp, vp], st),
        "aqlm_nearest_workspace_bytes": ([i64], sz),
        "aqlm_nearest_codeword": ([vp, i64, vp, i32, vp, vp, vp, sz, vp], st),
        "aqlm_kmeans_workspace_bytes": ([i32], sz),
        "aqlm_kmeans_update": ([vp, vp, i64, vp, i32, vp, vp, vp, sz, vp], st),
        "aqlm_residual_kmeans_workspace_bytes": ([i64, i32, i32], sz),
        "aqlm_residual_kmeans": ([vp, i64, i32, i32, vp, i32, vp, vp, sz, vp], st),
        "aqlm_encode_codes_workspace_bytes": ([Shape], sz),
        "aqlm_encode_codes": ([vp, vp, vp, Shape, vp, sz, vp], st),
        "aqlm_encode_layer_workspace_bytes": ([Shape], sz),
        "aqlm_encode_layer": ([vp, Shape, vp, i32, vp, vp, vp, vp, sz, vp], st),
        "aqlm_status_string": ([st], ctypes.c_char_p),
        "aqlm_version": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


def status_string(status):
    return load_library().aqlm_status_string(int(status)).decode()


def version():
    return load_library().aqlm_version().decode()


def _check(status, where):
    if status != AQLM_OK:
        raise AqlmError(status, where)


def _p(t):
    # an int (or None for NULL): ctypes converts it for a c_void_p argument
    return t.data_ptr() if t is not None else None


# the current stream's handle without building a torch.cuda.Stream object
# (which costs microseconds per call); torch builds without it take the slow way
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, device=None):
    """The cudaStream_t handle (an int) of `stream`, else of the current
    stream of `device` (default: the current device)."""
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    return _raw_stream(torch.cuda.current_device() if device is None else device)


_shapes = {}


def shape_of(codes, d_in=None):
    """aqlm_shape from a codes tensor [d_out, G, M] (B from its dtype)."""
    key = (tuple(codes.shape), codes.dtype, d_in)
    sh = _shapes.get(key)
    if sh is None:
        d_out, G, M = codes.shape
        B = 8 if codes.dtype == torch.uint8 else 16
        sh = Shape(d_out, d_in if d_in is not None else G * 8, 8, M, B)
        if len(_shapes) < 4096:
            _shapes[key] = sh
    return sh


def _flat_scales(scales):
    # [d_out] or [d_out, 1, ...]: only the pointer is passed, which a
    # contiguous tensor shares with its flat view
    return scales if scales.is_contiguous() else scales.reshape(-1).contiguous()


_gemv_ws = {}


def _gemv_need(lib, shape, T, device):
    key = (shape.d_out, shape.d_in, shape.num_codebooks, shape.codebook_bits, T, device)
    need = _gemv_ws.get(key)
    if need is None:
        need = int(lib.aqlm_gemv_workspace_bytes(shape, T))
        if len(_gemv_ws) < 4096:
            _gemv_ws[key] = need
    return need


def gemv_workspace_bytes(shape, tokens):
    return int(load_library().aqlm_gemv_workspace_bytes(shape, tokens))


def gemm_workspace_bytes(shape, tokens):
    return int(load_library().aqlm_gemm_workspace_bytes(shape, tokens))


def aqlm_gemv(codes, codebooks, scales, x, y=None, workspace=None, stream=None):
    """y[T, d_out] = fp16(W^ . x) for x [T, d_in] float16, 1 <= T <= 16."""
    lib = _lib if _lib is not None else load_library()
    shape = shape_of(codes)
    if x.dim() == 1:
        x = x.unsqueeze(0)
    T = x.shape[0]
    dev = x.get_device()
    if y is None:
        y = torch.empty((T, shape.d_out), dtype=torch.float16, device=x.device)
    need = _gemv_need(lib, shape, T, dev)
    if need and workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.aqlm_gemv(codes.data_ptr(), codebooks.data_ptr(), _flat_scales(scales).data_ptr(), x.data_ptr(),
                         y.data_ptr(), T, shape, _p(workspace), wbytes, _stream(stream, dev if dev >= 0 else None)),
           "aqlm_gemv")
    return y


def aqlm_gemv_lut(codes, codebooks, scales, x, y=None, workspace=None, stream=None):
    """2x8, one token: y[1, d_out] = fp16(W^ . x) through per-slab lookup tables."""
    lib = load_library()
    shape = shape_of(codes)
    if x.dim() == 1:
        x = x.unsqueeze(0)
    if y is None:
        y = torch.empty((1, shape.d_out), dtype=torch.float16, device=x.device)
    need = lib.aqlm_gemv_lut_workspace_bytes(shape)
    if need and workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.aqlm_gemv_lut(_p(codes), _p(codebooks), _p(_flat_scales(scales)), _p(x), _p(y), shape, _p(workspace),
                             wbytes, _stream(stream)), "aqlm_gemv_lut")
    return y


def gemv_lut_workspace_bytes(shape):
    return int(load_library().aqlm_gemv_lut_workspace_bytes(shape))


def gemv_row_tokens(shape):
    """Most tokens aqlm_gemv runs on the CUDA cores (and aqlm_gemv_multi takes)."""
    return int(load_library().aqlm_gemv_row_tokens(shape))


def _layers(layers, ys):
    arr = (Layer * len(layers))()
    for k, (d, y) in enumerate(zip(layers, ys)):
        arr[k] = Layer(d["codes"].data_ptr(), d["codebooks"].data_ptr(), _flat_scales(d["scales"]).data_ptr(),
                       y.data_ptr() if y is not None else 0, d["codes"].shape[0])
    return arr


def gemv_multi_workspace_bytes(layers, tokens):
    lib = load_library()
    return int(lib.aqlm_gemv_multi_workspace_bytes(_layers(layers, [None] * len(layers)), len(layers),
                                                   shape_of(layers[0]["codes"]), tokens))


def aqlm_gemv_multi(layers, x, ys=None, workspace=None, stream=None):
    """[y_l] = [fp16(W^_l . x)] for layers (dicts with codes, codebooks, scales)
    that read the same x [T, d_in], in one launch."""
    lib = load_library()
    if x.dim() == 1:
        x = x.unsqueeze(0)
    T = x.shape[0]
    if ys is None:
        ys = [torch.empty((T, d["codes"].shape[0]), dtype=torch.float16, device=x.device) for d in layers]
    arr = _layers(layers, ys)
    shape = shape_of(layers[0]["codes"])
    need = int(lib.aqlm_gemv_multi_workspace_bytes(arr, len(layers), shape, T))
    if need and workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.aqlm_gemv_multi(arr, len(layers), _p(x), T, shape, _p(workspace), wbytes, _stream(stream)),
           "aqlm_gemv_multi")
    return ys


def aqlm_gemv_multi_check(layers, tokens, workspace, stream=None):
    """Synchronise and return the status that aqlm_gemv_multi calls with these
    layers, token count and workspace recorded (AQLM_OK or AQLM_ERR_TIMEOUT)."""
    lib = load_library()
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return lib.aqlm_gemv_multi_check(_layers(layers, [None] * len(layers)), len(layers),
                                     shape_of(layers[0]["codes"]), tokens, _p(workspace), wbytes, _stream(stream))


def aqlm_gemv_check(codes, tokens, workspace, stream=None):
    """Synchronise and return the status the aqlm_gemv calls with this layer
    shape, token count and workspace recorded (AQLM_OK or AQLM_ERR_TIMEOUT)."""
    lib = load_library()
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    return lib.aqlm_gemv_check(shape_of(codes), tokens, _p(workspace), wbytes, _stream(stream))


def aqlm_gemv_noalloc(codes, codebooks, scales, x, y=None, stream=None):
    """aqlm_gemv with the library's built-in scratch array (no workspace)."""
    lib = load_library()
    shape = shape_of(codes)
    if x.dim() == 1:
        x = x.unsqueeze(0)
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, shape.d_out), dtype=torch.float16, device=x.device)
    _check(lib.aqlm_gemv_noalloc(_p(codes), _p(codebooks), _p(_flat_scales(scales)), _p(x), _p(y), T, shape,
                                 _stream(stream)), "aqlm_gemv_noalloc")
    return y


def aqlm_gemv_noalloc_check(stream=None):
    """Synchronise and return the status that aqlm_gemv_noalloc calls since the
    last check recorded (AQLM_OK or AQLM_ERR_TIMEOUT); clears it."""
    return load_library().aqlm_gemv_noalloc_check(_stream(stream))


def probe_gather(table, source, ctas_per_sm=8, iters=64, sink=None, stream=None):
    """Launch the random 16-byte gather probe on `table` (a device tensor);
    returns (gathers made, sink).  source 0: through L1/L2 like the 1x16 and
    2x16 codeword loads; 1: from a shared-memory copy (table <= 64 KiB)."""
    lib = load_library()
    nbytes = table.numel() * table.element_size()
    if sink is None:
        sink = torch.empty(lib.aqlm_probe_gather_sink_bytes(ctas_per_sm), dtype=torch.uint8, device=table.device)
    n = ctypes.c_uint64(0)
    _check(lib.aqlm_probe_gather(_p(table), nbytes, source, ctas_per_sm, iters, _p(sink), sink.numel(),
                                 ctypes.byref(n), _stream(stream)), "aqlm_probe_gather")
    return n.value, sink


def aqlm_dequant(codes, codebooks, scales, out=None, stream=None):
    """W^[d_out, d_in] as bfloat16, bit-exact binary32 steps then RNE."""
    lib = load_library()
    shape = shape_of(codes)
    if out is None:
        out = torch.empty((shape.d_out, shape.d_in), dtype=torch.bfloat16, device=codes.device)
    _check(lib.aqlm_dequant(_p(codes), _p(codebooks), _p(_flat_scales(scales)), _p(out), shape, _stream(stream)),
           "aqlm_dequant")
    return out


def aqlm_gemm(codes, codebooks, scales, X, Y=None, workspace=None, stream=None):
    """Y[T, d_out] = bf16(X . W^T): aqlm_dequant into the workspace (W^ in its
    last 2 * d_out * d_in bytes), then the tcgen05 GEMM."""
    lib = load_library()
    shape = shape_of(codes)
    T = X.shape[0]
    if Y is None:
        Y = torch.empty((T, shape.d_out), dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = torch.empty(lib.aqlm_gemm_workspace_bytes(shape, T), dtype=torch.uint8, device=X.device)
    _check(lib.aqlm_gemm(_p(codes), _p(codebooks), _p(_flat_scales(scales)), _p(X), _p(Y), T, shape,
                         _p(workspace), workspace.numel(), _stream(stream)), "aqlm_gemm")
    return Y, workspace


def aqlm_gemm_overlap(codes, codebooks, scales, X, Y=None, workspace=None, stream=None):
    """aqlm_gemm in one kernel: W^ decoded into the workspace by the GEMM's own
    decoder warps, overlapped with the MMAs."""
    lib = load_library()
    shape = shape_of(codes)
    T = X.shape[0]
    if Y is None:
        Y = torch.empty((T, shape.d_out), dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = torch.empty(lib.aqlm_gemm_workspace_bytes(shape, T), dtype=torch.uint8, device=X.device)
    _check(lib.aqlm_gemm_overlap(_p(codes), _p(codebooks), _p(_flat_scales(scales)), _p(X), _p(Y), T, shape,
                                 _p(workspace), workspace.numel(), _stream(stream)), "aqlm_gemm_overlap")
    return Y, workspace


def aqlm_gemm_fused(codes, codebooks, scales, X, Y=None, workspace=None, stream=None):
    """Y[T, d_out] = bf16(X . W^T) with the dequantisation inside the GEMM (no W^ buffer)."""
    lib = load_library()
    shape = shape_of(codes)
    T = X.shape[0]
    if Y is None:
        Y = torch.empty((T, shape.d_out), dtype=torch.bfloat16, device=X.device)
    if workspace is None:
        workspace = torch.empty(lib.aqlm_gemm_fused_workspace_bytes(shape, T), dtype=torch.uint8, device=X.device)
    _check(lib.aqlm_gemm_fused(_p(codes), _p(codebooks), _p(_flat_scales(scales)), _p(X), _p(Y), T, shape,
                               _p(workspace), workspace.numel(), _stream(stream)), "aqlm_gemm_fused")
    return Y, workspace


def aqlm_gemm_check(workspace, stream=None):
    """Synchronise and return the status recorded in the GEMM workspace."""
    lib = load_library()
    return lib.aqlm_gemm_check(_p(workspace), workspace.numel(), _stream(stream))


def bf16_gemm_tile_n(tokens, n, sms):
    """Output tile width the tensor-core GEMM uses for tokens x n on `sms` SMs."""
    return int(load_library().aqlm_bf16_gemm_tile_n(int(tokens), int(n), int(sms)))


def bf16_gemm_plan(tokens, n, sms):
    """(cta_pair, tile_n): the GEMM kernel chosen for tokens x n on `sms` SMs."""
    pair, width = ctypes.c_int32(0), ctypes.c_int32(0)
    _check(load_library().aqlm_bf16_gemm_plan(int(tokens), int(n), int(sms), ctypes.byref(pair),
                                              ctypes.byref(width)), "aqlm_bf16_gemm_plan")
    return int(pair.value), int(width.value)


def aqlm_bf16_gemm_config(X, W, cta_pair, tile_n, Y=None, status=None, stream=None):
    """aqlm_bf16_gemm with the kernel variant chosen by the caller."""
    lib = load_library()
    T, k = X.shape
    n = W.shape[0]
    if Y is None:
        Y = torch.empty((T, n), dtype=torch.bfloat16, device=X.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=X.device)
    _check(lib.aqlm_bf16_gemm_config(_p(X), _p(W), _p(Y), T, n, k, _p(status), int(cta_pair), int(tile_n),
                                     _stream(stream)), "aqlm_bf16_gemm_config")
    return Y, status


def aqlm_bf16_gemm(X, W, Y=None, status=None, stream=None):
    """Y[T, n] = bf16(X[T, k] . W[n, k]^T) on the tensor cores."""
    lib = load_library()
    T, k = X.shape
    n = W.shape[0]
    if Y is None:
        Y = torch.empty((T, n), dtype=torch.bfloat16, device=X.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=X.device)
    _check(lib.aqlm_bf16_gemm(_p(X), _p(W), _p(Y), T, n, k, _p(status), _stream(stream)), "aqlm_bf16_gemm")
    return Y, status


def aqlm_decode_indices(codes, out=None, stream=None):
    """Indices [d_out, G, M]: uint16 bit patterns held in an int16 tensor."""
    lib = load_library()
    shape = shape_of(codes)
    if out is None:
        out = torch.empty(codes.shape, dtype=torch.int16, device=codes.device)
    _check(lib.aqlm_decode_indices(_p(codes), _p(out), shape, _stream(stream)), "aqlm_decode_indices")
    return out


def aqlm_test_gemm_timeout(X, W, Y, status, limit_ns, cta_pair=0, stream=None):
    lib = load_library()
    T, k = X.shape
    n = W.shape[0]
    return lib.aqlm_test_gemm_timeout(_p(X), _p(W), _p(Y), T, n, k, _p(status), limit_ns, int(cta_pair),
                                      _stream(stream))


# --------------------------------------------------------------------------- encoding

def _ws(nbytes, device):
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def encode_scales(W, stream=None):
    """(scales float16 [d_out], groups float32 [d_out*d_in/8, 8]) of W [d_out, d_in] float32."""
    lib = load_library()
    d_out, d_in = W.shape
    scales = torch.empty(d_out, dtype=torch.float16, device=W.device)
    groups = torch.empty((d_out * d_in // 8, 8), dtype=torch.float32, device=W.device)
    _check(lib.aqlm_encode_scales(_p(W), d_out, d_in, _p(scales), _p(groups), _stream(stream)), "aqlm_encode_scales")
    return scales, groups


def nearest_codeword(groups, codebook, with_dist=False, stream=None):
    """int32 index (and float32 distance) of each group's nearest codeword."""
    lib = load_library()
    n, K = groups.shape[0], codebook.shape[0]
    idx = torch.empty(n, dtype=torch.int32, device=groups.device)
    dist = torch.empty(n, dtype=torch.float32, device=groups.device) if with_dist else None
    ws = _ws(lib.aqlm_nearest_workspace_bytes(n), groups.device)
    _check(lib.aqlm_nearest_codeword(_p(groups), n, _p(codebook), K, _p(idx), _p(dist), _p(ws), ws.numel(),
                                     _stream(stream)), "aqlm_nearest_codeword")
    return (idx, dist) if with_dist else idx


def kmeans_update(groups, idx, centroids, stream=None):
    """(centroids float32 [K, 8], counts int32 [K]) after one k-means update."""
    lib = load_library()
    n, K = groups.shape[0], centroids.shape[0]
    out = torch.empty_like(centroids)
    counts = torch.empty(K, dtype=torch.int32, device=groups.device)
    ws = _ws(lib.aqlm_kmeans_workspace_bytes(K), groups.device)
    _check(lib.aqlm_kmeans_update(_p(groups), _p(idx), n, _p(centroids), K, _p(out), _p(counts), _p(ws), ws.numel(),
                                  _stream(stream)), "aqlm_kmeans_update")
    return out, counts


def residual_kmeans(groups, M, K, init_idx, iters, stream=None):
    """float32 codebooks [M, K, 8]; init_idx: host int32 array [M, K] of group indices."""
    import numpy as np
    lib = load_library()
    n = groups.shape[0]
    init = np.ascontiguousarray(init_idx, dtype=np.int32)
    assert init.size == M * K
    out = torch.empty((M, K, 8), dtype=torch.float32, device=groups.device)
    ws = _ws(lib.aqlm_residual_kmeans_workspace_bytes(n, M, K), groups.device)
    _check(lib.aqlm_residual_kmeans(_p(groups), n, M, K, init.ctypes.data_as(ctypes.c_void_p), iters, _p(out), _p(ws),
                                    ws.numel(), _stream(stream)), "aqlm_residual_kmeans")
    return out


def _codes_out(d_out, d_in, M, B, device):
    return torch.empty((d_out, d_in // 8, M), dtype=torch.uint8 if B == 8 else torch.int16, device=device)


def encode_codes(groups, codebooks, d_out, d_in, stream=None):
    """Greedy codes [d_out, d_in/8, M] of the groups against float16 codebooks [M, 2^B, 8]."""
    lib = load_library()
    M, K = codebooks.shape[0], codebooks.shape[1]
    B = 8 if K == 256 else 16
    shape = Shape(d_out, d_in, 8, M, B)
    codes = _codes_out(d_out, d_in, M, B, groups.device)
    ws = _ws(lib.aqlm_encode_codes_workspace_bytes(shape), groups.device)
    _check(lib.aqlm_encode_codes(_p(groups), _p(codebooks), _p(codes), shape, _p(ws), ws.numel(), _stream(stream)),
           "aqlm_encode_codes")
    return codes


def encode_layer(W, M, B, init_idx, iters, stream=None):
    """{codes, codebooks (float16 [M, 2^B, 8]), scales (float16 [d_out])} of W [d_out, d_in] float32."""
    import numpy as np
    lib = load_library()
    d_out, d_in = W.shape
    shape = Shape(d_out, d_in, 8, M, B)
    init = np.ascontiguousarray(init_idx, dtype=np.int32)
    codes = _codes_out(d_out, d_in, M, B, W.device)
    codebooks = torch.empty((M, 1 << B, 8), dtype=torch.float16, device=W.device)
    scales = torch.empty(d_out, dtype=torch.float16, device=W.device)
    ws = _ws(lib.aqlm_encode_layer_workspace_bytes(shape), W.device)
    _check(lib.aqlm_encode_layer(_p(W), shape, init.ctypes.data_as(ctypes.c_void_p), iters, _p(codes), _p(codebooks),
                                 _p(scales), _p(ws), ws.numel(), _stream(stream)), "aqlm_encode_layer")
    return {"codes": codes, "codebooks": codebooks, "scales": scales}

