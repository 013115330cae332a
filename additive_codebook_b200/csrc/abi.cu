// abi.cu -- the extern "C" entry points of include/aqlm.h: host-side
// argument validation, workspace layout and kernel selection.  Nothing here
// allocates memory or keeps state between calls.
#include <cstdint>

#include "common.cuh"

namespace aqlm {
cudaError_t launch_bf16_gemm_ex(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                                int32_t *status, cudaStream_t st, unsigned long long limit_ns, int stall_test);
cudaError_t launch_bf16_gemm_cfg(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                                 int32_t *status, cudaStream_t st, unsigned long long limit_ns, int stall_test,
                                 int cta_pair, int tile_n, bool pdl);
bool overlap_preferred(const Dims &d, int tokens);
cudaError_t launch_bf16_gemm_after_dequant(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n,
                                          int k, int32_t *status, cudaStream_t st);
cudaError_t launch_fused_gemm(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                              const uint16_t *X, uint16_t *Y, int tokens, const Dims &d, int32_t *status,
                              cudaStream_t st);
}

namespace {

using aqlm::Dims;

constexpr size_t kStatusBytes = 256;  // head of the aqlm_gemm workspace
constexpr int32_t kMaxDim = 1 << 20;

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline cudaStream_t to_cuda(aqlm_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

aqlm_status check_shape(const aqlm_shape &s) {
    if (s.d_out < 1 || s.d_in < 1 || s.d_out > kMaxDim || s.d_in > kMaxDim) return AQLM_ERR_INVALID_ARG;
    if (s.group != aqlm::kGroup) return AQLM_ERR_UNSUPPORTED;
    const bool fmt_ok = (s.num_codebooks == 1 && s.codebook_bits == 16) ||
                        (s.num_codebooks == 2 && s.codebook_bits == 8) ||
                        (s.num_codebooks == 2 && s.codebook_bits == 16);
    if (!fmt_ok) return AQLM_ERR_UNSUPPORTED;
    if (s.d_in % aqlm::kGroup) return AQLM_ERR_UNSUPPORTED;
    const int64_t row_bytes = (int64_t)(s.d_in / aqlm::kGroup) * s.num_codebooks * s.codebook_bits / 8;
    if (row_bytes % 16) return AQLM_ERR_MISALIGNED;
    return AQLM_OK;
}

aqlm_status check_layer(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const aqlm_shape &s) {
    if (!codes || !codebooks || !scales) return AQLM_ERR_INVALID_ARG;
    const aqlm_status st = check_shape(s);
    if (st != AQLM_OK) return st;
    if (!aligned(codes, 16) || !aligned(codebooks, 16) || !aligned(scales, 2)) return AQLM_ERR_MISALIGNED;
    return AQLM_OK;
}

inline aqlm_status from_cuda(cudaError_t e) { return e == cudaSuccess ? AQLM_OK : AQLM_ERR_CUDA; }

// Synchronise cs, then read and clear the status word at byte `off` of the
// workspace (off < 0: the path has no status word, AQLM_OK).
aqlm_status read_status_word(long long off, void *workspace, size_t workspace_bytes, cudaStream_t cs) {
    if (off < 0) return cudaStreamSynchronize(cs) == cudaSuccess ? AQLM_OK : AQLM_ERR_CUDA;
    if (!workspace || workspace_bytes < (size_t)off + sizeof(int32_t) || !aligned(workspace, 16))
        return AQLM_ERR_WORKSPACE;
    int32_t *word = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) + off);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, word, sizeof(h), cudaMemcpyDeviceToHost, cs) != cudaSuccess) return AQLM_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return AQLM_ERR_CUDA;
    if (h != 0) {
        if (cudaMemsetAsync(word, 0, sizeof(int32_t), cs) != cudaSuccess) return AQLM_ERR_CUDA;
        if (cudaStreamSynchronize(cs) != cudaSuccess) return AQLM_ERR_CUDA;
    }
    return h == 0 ? AQLM_OK : AQLM_ERR_TIMEOUT;
}

}  // namespace

namespace aqlm {

// The argument checks of aqlm_gemv other than the workspace's.
aqlm_status check_gemv_args(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                            const uint16_t *y, int32_t tokens, const aqlm_shape &shape) {
    const aqlm_status st = check_layer(codes, codebooks, scales, shape);
    if (st != AQLM_OK) return st;
    if (!x || !y || tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return AQLM_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 2)) return AQLM_ERR_MISALIGNED;
    return AQLM_OK;
}

}  // namespace aqlm

extern "C" {

aqlm_status aqlm_decode_indices(const void *codes, uint16_t *idx_out, aqlm_shape shape, aqlm_stream_t stream) {
    if (!codes || !idx_out) return AQLM_ERR_INVALID_ARG;
    const aqlm_status st = check_shape(shape);
    if (st != AQLM_OK) return st;
    if (!aligned(codes, 16) || !aligned(idx_out, 2)) return AQLM_ERR_MISALIGNED;
    return from_cuda(aqlm::launch_decode_indices(codes, idx_out, aqlm::make_dims(shape), to_cuda(stream)));
}

aqlm_status aqlm_dequant(const void *codes, const uint16_t *codebooks, const uint16_t *scales, uint16_t *W_out,
                         aqlm_shape shape, aqlm_stream_t stream) {
    aqlm_status st = check_layer(codes, codebooks, scales, shape);
    if (st != AQLM_OK) return st;
    if (!W_out) return AQLM_ERR_INVALID_ARG;
    if (!aligned(W_out, 16)) return AQLM_ERR_MISALIGNED;
    return from_cuda(aqlm::launch_dequant(codes, codebooks, scales, W_out, aqlm::make_dims(shape), to_cuda(stream)));
}

size_t aqlm_gemv_workspace_bytes(aqlm_shape shape, int32_t tokens) {
    if (check_shape(shape) != AQLM_OK || tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return 0;
    return aqlm::gemv_workspace_bytes(aqlm::make_dims(shape), tokens);
}

aqlm_status aqlm_gemv(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                      uint16_t *y, int32_t tokens, aqlm_shape shape, void *workspace, size_t workspace_bytes,
                      aqlm_stream_t stream) {
    const aqlm_status st = aqlm::check_gemv_args(codes, codebooks, scales, x, y, tokens, shape);
    if (st != AQLM_OK) return st;
    const Dims d = aqlm::make_dims(shape);
    const size_t need = aqlm::gemv_workspace_bytes(d, tokens);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return AQLM_ERR_WORKSPACE;
    return from_cuda(aqlm::launch_gemv(codes, codebooks, scales, x, y, tokens, d, need > 0 ? workspace : nullptr,
                                       to_cuda(stream)));
}

size_t aqlm_gemv_lut_workspace_bytes(aqlm_shape shape) {
    if (check_shape(shape) != AQLM_OK || !aqlm::gemv_lut_supported(aqlm::make_dims(shape), 1)) return 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    return aqlm::gemv_lut_workspace_bytes(aqlm::make_dims(shape), aqlm::num_sms(dev));
}

aqlm_status aqlm_gemv_lut(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                          uint16_t *y, aqlm_shape shape, void *workspace, size_t workspace_bytes, aqlm_stream_t stream) {
    const aqlm_status st = aqlm::check_gemv_args(codes, codebooks, scales, x, y, 1, shape);
    if (st != AQLM_OK) return st;
    const Dims d = aqlm::make_dims(shape);
    if (!aqlm::gemv_lut_supported(d, 1)) return AQLM_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;   // the launch below then reports the error
    const int sms = aqlm::num_sms(dev);
    const size_t need = aqlm::gemv_lut_workspace_bytes(d, sms);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return AQLM_ERR_WORKSPACE;
    return from_cuda(aqlm::launch_gemv_lut(codes, codebooks, scales, x, y, d, need > 0 ? workspace : nullptr, sms,
                                           to_cuda(stream)));
}

int32_t aqlm_gemv_row_tokens(aqlm_shape shape) {
    if (check_shape(shape) != AQLM_OK) return 0;
    return aqlm::gemv_row_tokens(aqlm::make_dims(shape));
}

}  // extern "C"

namespace {

// Validated multi-layer arguments: the layers as the launchers take them.
aqlm_status multi_layers(const aqlm_layer *layers, int32_t n_layers, aqlm_shape shape, aqlm::RowLayerIn *out) {
    if (!layers || n_layers < 1 || n_layers > AQLM_MULTI_MAX_LAYERS) return AQLM_ERR_INVALID_ARG;
    for (int l = 0; l < n_layers; ++l) {
        aqlm_shape s = shape;
        s.d_out = layers[l].d_out;
        const aqlm_status st = check_shape(s);
        if (st != AQLM_OK) return st;
        out[l] = {layers[l].codes, layers[l].codebooks, layers[l].scales, layers[l].y, layers[l].d_out};
    }
    return AQLM_OK;
}

}  // namespace

extern "C" {

size_t aqlm_gemv_multi_workspace_bytes(const aqlm_layer *layers, int32_t n_layers, aqlm_shape shape, int32_t tokens) {
    aqlm::RowLayerIn in[AQLM_MULTI_MAX_LAYERS];
    if (multi_layers(layers, n_layers, shape, in) != AQLM_OK) return 0;
    const Dims d = aqlm::make_dims(shape);
    if (tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return 0;
    return aqlm::gemv_multi_workspace_bytes(in, n_layers, d, tokens);
}

aqlm_status aqlm_gemv_multi(const aqlm_layer *layers, int32_t n_layers, const uint16_t *x, int32_t tokens,
                            aqlm_shape shape, void *workspace, size_t workspace_bytes, aqlm_stream_t stream) {
    aqlm::RowLayerIn in[AQLM_MULTI_MAX_LAYERS];
    aqlm_status st = multi_layers(layers, n_layers, shape, in);
    if (st != AQLM_OK) return st;
    for (int l = 0; l < n_layers; ++l) {
        aqlm_shape s = shape;
        s.d_out = in[l].d_out;
        st = check_layer(in[l].codes, in[l].codebooks, in[l].scales, s);
        if (st != AQLM_OK) return st;
        if (!in[l].y) return AQLM_ERR_INVALID_ARG;
        if (!aligned(in[l].y, 2)) return AQLM_ERR_MISALIGNED;
    }
    if (!x || tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return AQLM_ERR_INVALID_ARG;
    if (!aligned(x, 16)) return AQLM_ERR_MISALIGNED;
    const Dims d = aqlm::make_dims(shape);
    const size_t need = aqlm::gemv_multi_workspace_bytes(in, n_layers, d, tokens);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return AQLM_ERR_WORKSPACE;
    return from_cuda(aqlm::launch_gemv_multi(in, n_layers, x, tokens, d, need > 0 ? workspace : nullptr,
                                             to_cuda(stream)));
}

aqlm_status aqlm_gemv_multi_check(const aqlm_layer *layers, int32_t n_layers, aqlm_shape shape, int32_t tokens,
                                  void *workspace, size_t workspace_bytes, aqlm_stream_t stream) {
    aqlm::RowLayerIn in[AQLM_MULTI_MAX_LAYERS];
    aqlm_status st = multi_layers(layers, n_layers, shape, in);
    if (st != AQLM_OK) return st;
    if (tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return AQLM_ERR_INVALID_ARG;
    const long long off = aqlm::gemv_multi_status_offset(in, n_layers, aqlm::make_dims(shape), tokens);
    return read_status_word(off, workspace, workspace_bytes, to_cuda(stream));
}

aqlm_status aqlm_gemv_check(aqlm_shape shape, int32_t tokens, void *workspace, size_t workspace_bytes,
                            aqlm_stream_t stream) {
    if (check_shape(shape) != AQLM_OK) return AQLM_ERR_UNSUPPORTED;
    if (tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return AQLM_ERR_INVALID_ARG;
    return read_status_word(aqlm::gemv_status_offset(aqlm::make_dims(shape), tokens), workspace, workspace_bytes,
                            to_cuda(stream));
}

size_t aqlm_gemm_workspace_bytes(aqlm_shape shape, int32_t tokens) {
    if (check_shape(shape) != AQLM_OK || tokens < 1) return 0;
    return kStatusBytes + aqlm::overlap_counter_bytes(shape.d_out, shape.d_in) + (size_t)shape.d_out * shape.d_in * 2;
}

aqlm_status aqlm_gemm(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *X,
                      uint16_t *Y, int32_t tokens, aqlm_shape shape, void *workspace, size_t workspace_bytes,
                      aqlm_stream_t stream) {
    aqlm_status st = check_layer(codes, codebooks, scales, shape);
    if (st != AQLM_OK) return st;
    if (!X || !Y || tokens < 1) return AQLM_ERR_INVALID_ARG;
    if (shape.d_out % 8) return AQLM_ERR_UNSUPPORTED;
    if (!aligned(X, 16) || !aligned(Y, 16)) return AQLM_ERR_MISALIGNED;
    const size_t need = aqlm_gemm_workspace_bytes(shape, tokens);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return AQLM_ERR_WORKSPACE;
    const cudaStream_t cs = to_cuda(stream);
    int32_t *status = static_cast<int32_t *>(workspace);
    uint8_t *counters = static_cast<uint8_t *>(workspace) + kStatusBytes;
    uint16_t *W = reinterpret_cast<uint16_t *>(counters + aqlm::overlap_counter_bytes(shape.d_out, shape.d_in));
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), cs);
    if (e != cudaSuccess) return AQLM_ERR_CUDA;
    if (aqlm::overlap_preferred(aqlm::make_dims(shape), tokens)) {
        // the one-kernel prefill of aqlm_gemm_overlap, where it was measured faster
        return from_cuda(aqlm::launch_overlap_gemm(codes, codebooks, scales, X, W, Y, tokens,
                                                   aqlm::make_dims(shape), status, counters, cs));
    }
    e = aqlm::launch_dequant(codes, codebooks, scales, W, aqlm::make_dims(shape), cs);
    if (e != cudaSuccess) return AQLM_ERR_CUDA;
    return from_cuda(aqlm::launch_bf16_gemm_after_dequant(X, W, Y, tokens, shape.d_out, shape.d_in, status, cs));
}

aqlm_status aqlm_gemm_overlap(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                              const uint16_t *X, uint16_t *Y, int32_t tokens, aqlm_shape shape, void *workspace,
                              size_t workspace_bytes, aqlm_stream_t stream) {
    aqlm_status st = check_layer(codes, codebooks, scales, shape);
    if (st != AQLM_OK) return st;
    if (!X || !Y || tokens < 1) return AQLM_ERR_INVALID_ARG;
    if (shape.d_out % 8) return AQLM_ERR_UNSUPPORTED;
    if (!aligned(X, 16) || !aligned(Y, 16)) return AQLM_ERR_MISALIGNED;
    const size_t need = aqlm_gemm_workspace_bytes(shape, tokens);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return AQLM_ERR_WORKSPACE;
    const cudaStream_t cs = to_cuda(stream);
    int32_t *status = static_cast<int32_t *>(workspace);
    uint8_t *counters = static_cast<uint8_t *>(workspace) + kStatusBytes;
    uint16_t *W = reinterpret_cast<uint16_t *>(counters + aqlm::overlap_counter_bytes(shape.d_out, shape.d_in));
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), cs) != cudaSuccess) return AQLM_ERR_CUDA;
    return from_cuda(aqlm::launch_overlap_gemm(codes, codebooks, scales, X, W, Y, tokens, aqlm::make_dims(shape),
                                               status, counters, cs));
}

size_t aqlm_gemm_fused_workspace_bytes(aqlm_shape shape, int32_t tokens) {
    if (check_shape(shape) != AQLM_OK || tokens < 1) return 0;
    return kStatusBytes;
}

aqlm_status aqlm_gemm_fused(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *X,
                            uint16_t *Y, int32_t tokens, aqlm_shape shape, void *workspace, size_t workspace_bytes,
                            aqlm_stream_t stream) {
    aqlm_status st = check_layer(codes, codebooks, scales, shape);
    if (st != AQLM_OK) return st;
    if (!X || !Y || tokens < 1) return AQLM_ERR_INVALID_ARG;
    if (shape.d_out % 8) return AQLM_ERR_UNSUPPORTED;
    if (!aligned(X, 16) || !aligned(Y, 16)) return AQLM_ERR_MISALIGNED;
    if (!workspace || workspace_bytes < kStatusBytes || !aligned(workspace, 16)) return AQLM_ERR_WORKSPACE;
    const cudaStream_t cs = to_cuda(stream);
    int32_t *status = static_cast<int32_t *>(workspace);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), cs) != cudaSuccess) return AQLM_ERR_CUDA;
    return from_cuda(
        aqlm::launch_fused_gemm(codes, codebooks, scales, X, Y, tokens, aqlm::make_dims(shape), status, cs));
}

aqlm_status aqlm_gemm_check(void *workspace, size_t workspace_bytes, aqlm_stream_t stream) {
    if (!workspace || workspace_bytes < kStatusBytes || !aligned(workspace, 16)) return AQLM_ERR_WORKSPACE;
    const cudaStream_t cs = to_cuda(stream);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, cs) != cudaSuccess) return AQLM_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return AQLM_ERR_CUDA;
    if (h != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof(int32_t), cs) != cudaSuccess) return AQLM_ERR_CUDA;
        if (cudaStreamSynchronize(cs) != cudaSuccess) return AQLM_ERR_CUDA;
    }
    return h == 0 ? AQLM_OK : AQLM_ERR_TIMEOUT;
}

aqlm_status aqlm_bf16_gemm(const uint16_t *X, const uint16_t *W, uint16_t *Y, int32_t tokens, int32_t n, int32_t k,
                           int32_t *status, aqlm_stream_t stream) {
    if (!X || !W || !Y || !status || tokens < 1 || n < 1 || k < 1) return AQLM_ERR_INVALID_ARG;
    if (n > kMaxDim || k > kMaxDim || tokens > kMaxDim) return AQLM_ERR_INVALID_ARG;
    if (n % 8 || k % 8) return AQLM_ERR_UNSUPPORTED;
    if (!aligned(X, 16) || !aligned(W, 16) || !aligned(Y, 16) || !aligned(status, 4)) return AQLM_ERR_MISALIGNED;
    return from_cuda(aqlm::launch_bf16_gemm(X, W, Y, tokens, n, k, status, to_cuda(stream)));
}

int32_t aqlm_bf16_gemm_tile_n(int32_t tokens, int32_t n, int32_t sms) {
    if (tokens < 1 || n < 1 || sms < 1) return 0;
    return aqlm::gemm_tile_n(tokens, n, sms);
}

aqlm_status aqlm_bf16_gemm_plan(int32_t tokens, int32_t n, int32_t sms, int32_t *cta_pair, int32_t *tile_n) {
    if (!cta_pair || !tile_n) return AQLM_ERR_INVALID_ARG;
    *cta_pair = 0;
    *tile_n = 0;
    if (tokens < 1 || n < 1 || sms < 2) return AQLM_ERR_INVALID_ARG;
    const bool pair = aqlm::gemm_uses_pair(tokens);
    *cta_pair = pair ? 1 : 0;
    *tile_n = pair ? aqlm::gemm_pair_tile_n(tokens, n, sms / 2) : aqlm::gemm_tile_n(tokens, n, sms);
    return AQLM_OK;
}

static bool known_tile_n(int32_t tile_n) {
    return tile_n == 0 || tile_n == 256 || tile_n == 240 || tile_n == 224 || tile_n == 192;
}

aqlm_status aqlm_bf16_gemm_config(const uint16_t *X, const uint16_t *W, uint16_t *Y, int32_t tokens, int32_t n,
                                  int32_t k, int32_t *status, int32_t cta_pair, int32_t tile_n,
                                  aqlm_stream_t stream) {
    if (!X || !W || !Y || !status || tokens < 1 || n < 1 || k < 1) return AQLM_ERR_INVALID_ARG;
    if (n > kMaxDim || k > kMaxDim || tokens > kMaxDim) return AQLM_ERR_INVALID_ARG;
    if (cta_pair < -1 || cta_pair > 1 || !known_tile_n(tile_n)) return AQLM_ERR_INVALID_ARG;
    if (n % 8 || k % 8) return AQLM_ERR_UNSUPPORTED;
    if (!aligned(X, 16) || !aligned(W, 16) || !aligned(Y, 16) || !aligned(status, 4)) return AQLM_ERR_MISALIGNED;
    return from_cuda(aqlm::launch_bf16_gemm_cfg(X, W, Y, tokens, n, k, status, to_cuda(stream),
                                                aqlm::kGemmWaitLimitNs, 0, cta_pair, tile_n, false));
}

aqlm_status aqlm_test_gemm_timeout(const uint16_t *X, const uint16_t *W, uint16_t *Y, int32_t tokens, int32_t n,
                                   int32_t k, int32_t *status, uint64_t limit_ns, int32_t cta_pair,
                                   aqlm_stream_t stream) {
    if (!X || !W || !Y || !status || tokens < 1 || n < 1 || k < 1 || n % 8 || k % 8) return AQLM_ERR_INVALID_ARG;
    if (limit_ns == 0 || limit_ns > 1000000000ull || cta_pair < -1 || cta_pair > 1) return AQLM_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(W, 16) || !aligned(Y, 16) || !aligned(status, 4)) return AQLM_ERR_MISALIGNED;
    return from_cuda(aqlm::launch_bf16_gemm_cfg(X, W, Y, tokens, n, k, status, to_cuda(stream), limit_ns, 1,
                                                cta_pair, 0, false));
}

// ---- encoding ----

aqlm_status aqlm_encode_scales(const float *W, int32_t d_out, int32_t d_in, uint16_t *scales, float *groups,
                               aqlm_stream_t stream) {
    if (!W || !scales || !groups || d_out < 1 || d_in < 8 || d_out > kMaxDim || d_in > kMaxDim) {
        return AQLM_ERR_INVALID_ARG;
    }
    if (d_in % 8) return AQLM_ERR_UNSUPPORTED;
    if (!aligned(W, 16) || !aligned(groups, 16) || !aligned(scales, 2)) return AQLM_ERR_MISALIGNED;
    return from_cuda(aqlm::launch_encode_scales(W, d_out, d_in, scales, groups, to_cuda(stream)));
}

size_t aqlm_nearest_workspace_bytes(int64_t n) { return n < 0 ? 0 : aqlm::nearest_workspace_bytes(n); }

aqlm_status aqlm_nearest_codeword(const float *groups, int64_t n, const float *codebook, int32_t K, int32_t *idx,
                                  float *dist, void *workspace, size_t workspace_bytes, aqlm_stream_t stream) {
    if (n < 0 || K < 1 || (n > 0 && (!groups || !idx)) || !codebook) return AQLM_ERR_INVALID_ARG;
    if (n > ((int64_t)1 << 40)) return AQLM_ERR_INVALID_ARG;
    if (!aligned(groups, 16) || !aligned(codebook, 16) || !aligned(idx, 4) || !aligned(dist, 4))
        return AQLM_ERR_MISALIGNED;
    const size_t need = aqlm::nearest_workspace_bytes(n);
    if (n > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return AQLM_ERR_WORKSPACE;
    return from_cuda(aqlm::launch_nearest(groups, n, codebook, K, idx, dist, workspace, to_cuda(stream)));
}

size_t aqlm_kmeans_workspace_bytes(int32_t K) { return K < 1 ? 0 : aqlm::kmeans_workspace_bytes(K); }

aqlm_status aqlm_kmeans_update(const float *groups, const int32_t *idx, int64_t n, const float *centroids, int32_t K,
                               float *centroids_out, int32_t *counts, void *workspace, size_t workspace_bytes,
                               aqlm_stream_t stream) {
    if (n < 0 || K < 1 || (n > 0 && (!groups || !idx)) || !centroids || !centroids_out) return AQLM_ERR_INVALID_ARG;
    if (n > ((int64_t)1 << 40)) return AQLM_ERR_INVALID_ARG;
    if (!aligned(groups, 16) || !aligned(idx, 4) || !aligned(centroids, 16) || !aligned(centroids_out, 16) ||
        !aligned(counts, 4))
        return AQLM_ERR_MISALIGNED;
    const size_t need = aqlm::kmeans_workspace_bytes(K);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return AQLM_ERR_WORKSPACE;
    return from_cuda(aqlm::launch_kmeans_update(groups, idx, n, centroids, K, centroids_out, counts, workspace,
                                                to_cuda(stream)));
}

}  // extern "C"

namespace {

// Workspace head of the residual k-means: the copy of init_idx, then the
// launcher's own workspace.
size_t init_copy_bytes(int32_t M, int32_t K) { return ((size_t)M * K * sizeof(int32_t) + 255) / 256 * 256; }

aqlm_status check_init(const int32_t *init_idx, int64_t n, int32_t M, int32_t K) {
    if (!init_idx) return AQLM_ERR_INVALID_ARG;
    for (int64_t i = 0; i < (int64_t)M * K; ++i)
        if (init_idx[i] < 0 || init_idx[i] >= n) return AQLM_ERR_INVALID_ARG;
    return AQLM_OK;
}

// Residual k-means with init_idx already validated; ws has
// aqlm_residual_kmeans_workspace_bytes(n, M, K) bytes.
aqlm_status run_residual_kmeans(const float *groups, int64_t n, int32_t M, int32_t K, const int32_t *init_idx,
                                int32_t iters, float *codebooks, void *ws, cudaStream_t cs) {
    int32_t *init_dev = static_cast<int32_t *>(ws);
    cudaError_t e = cudaMemcpyAsync(init_dev, init_idx, (size_t)M * K * sizeof(int32_t), cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) return AQLM_ERR_CUDA;
    return from_cuda(aqlm::launch_residual_kmeans(groups, n, M, K, init_dev, iters, codebooks,
                                                  static_cast<uint8_t *>(ws) + init_copy_bytes(M, K), cs));
}

size_t layer_groups(const aqlm_shape &s) { return (size_t)s.d_out * (s.d_in / 8); }
inline size_t al256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

extern "C" {

size_t aqlm_residual_kmeans_workspace_bytes(int64_t n, int32_t M, int32_t K) {
    if (n < 1 || M < 1 || K < 1) return 0;
    return init_copy_bytes(M, K) + aqlm::residual_kmeans_workspace_bytes(n, K);
}

aqlm_status aqlm_residual_kmeans(const float *groups, int64_t n, int32_t M, int32_t K, const int32_t *init_idx,
                                 int32_t iters, float *codebooks, void *workspace, size_t workspace_bytes,
                                 aqlm_stream_t stream) {
    if (!groups || !codebooks || n < 1 || M < 1 || M > 8 || K < 1 || iters < 0) return AQLM_ERR_INVALID_ARG;
    if (n > ((int64_t)1 << 40)) return AQLM_ERR_INVALID_ARG;
    aqlm_status st = check_init(init_idx, n, M, K);
    if (st != AQLM_OK) return st;
    if (!aligned(groups, 16) || !aligned(codebooks, 16)) return AQLM_ERR_MISALIGNED;
    const size_t need = aqlm_residual_kmeans_workspace_bytes(n, M, K);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return AQLM_ERR_WORKSPACE;
    return run_residual_kmeans(groups, n, M, K, init_idx, iters, codebooks, workspace, to_cuda(stream));
}

size_t aqlm_encode_codes_workspace_bytes(aqlm_shape shape) {
    if (check_shape(shape) != AQLM_OK) return 0;
    return aqlm::encode_codes_workspace_bytes((long long)layer_groups(shape), shape.num_codebooks,
                                              1 << shape.codebook_bits);
}

aqlm_status aqlm_encode_codes(const float *groups, const uint16_t *codebooks, void *codes, aqlm_shape shape,
                              void *workspace, size_t workspace_bytes, aqlm_stream_t stream) {
    aqlm_status st = check_shape(shape);
    if (st != AQLM_OK) return st;
    if (!groups || !codebooks || !codes) return AQLM_ERR_INVALID_ARG;
    if (!aligned(groups, 16) || !aligned(codebooks, 16) || !aligned(codes, 16)) return AQLM_ERR_MISALIGNED;
    const size_t need = aqlm_encode_codes_workspace_bytes(shape);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return AQLM_ERR_WORKSPACE;
    return from_cuda(aqlm::launch_encode_codes(groups, (long long)layer_groups(shape), codebooks, shape.num_codebooks,
                                               1 << shape.codebook_bits, codes, shape.codebook_bits / 8, workspace,
                                               to_cuda(stream)));
}

// Workspace of the whole encoding: groups, fp32 codebooks, then the larger of
// the residual k-means' and the greedy codes' workspaces.
size_t aqlm_encode_layer_workspace_bytes(aqlm_shape shape) {
    if (check_shape(shape) != AQLM_OK) return 0;
    const int64_t n = (int64_t)layer_groups(shape);
    const int32_t M = shape.num_codebooks, K = 1 << shape.codebook_bits;
    const size_t a = aqlm_residual_kmeans_workspace_bytes(n, M, K), b = aqlm_encode_codes_workspace_bytes(shape);
    return al256((size_t)n * 8 * sizeof(float)) + al256((size_t)M * K * 8 * sizeof(float)) + (a > b ? a : b);
}

aqlm_status aqlm_encode_layer(const float *W, aqlm_shape shape, const int32_t *init_idx, int32_t iters, void *codes,
                              uint16_t *codebooks, uint16_t *scales, void *workspace, size_t workspace_bytes,
                              aqlm_stream_t stream) {
    aqlm_status st = check_shape(shape);
    if (st != AQLM_OK) return st;
    if (!W || !codes || !codebooks || !scales || iters < 0) return AQLM_ERR_INVALID_ARG;
    const int64_t n = (int64_t)layer_groups(shape);
    const int32_t M = shape.num_codebooks, K = 1 << shape.codebook_bits;
    st = check_init(init_idx, n, M, K);
    if (st != AQLM_OK) return st;
    if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(codebooks, 16) || !aligned(scales, 2))
        return AQLM_ERR_MISALIGNED;
    const size_t need = aqlm_encode_layer_workspace_bytes(shape);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 16)) return AQLM_ERR_WORKSPACE;
    const cudaStream_t cs = to_cuda(stream);
    uint8_t *w = static_cast<uint8_t *>(workspace);
    float *groups = reinterpret_cast<float *>(w);
    w += al256((size_t)n * 8 * sizeof(float));
    float *cb32 = reinterpret_cast<float *>(w);
    w += al256((size_t)M * K * 8 * sizeof(float));
    cudaError_t e = aqlm::launch_encode_scales(W, shape.d_out, shape.d_in, scales, groups, cs);
    if (e != cudaSuccess) return AQLM_ERR_CUDA;
    st = run_residual_kmeans(groups, n, M, K, init_idx, iters, cb32, w, cs);
    if (st != AQLM_OK) return st;
    e = aqlm::launch_round_codebooks(cb32, (long long)M * K * 8, codebooks, cs);
    if (e != cudaSuccess) return AQLM_ERR_CUDA;
    return from_cuda(aqlm::launch_encode_codes(groups, n, codebooks, M, K, codes, shape.codebook_bits / 8, w, cs));
}

const char *aqlm_status_string(aqlm_status status) {
    switch (status) {
        case AQLM_OK: return "AQLM_OK";
        case AQLM_ERR_INVALID_ARG: return "AQLM_ERR_INVALID_ARG";
        case AQLM_ERR_UNSUPPORTED: return "AQLM_ERR_UNSUPPORTED";
        case AQLM_ERR_MISALIGNED: return "AQLM_ERR_MISALIGNED";
        case AQLM_ERR_WORKSPACE: return "AQLM_ERR_WORKSPACE";
        case AQLM_ERR_CUDA: return "AQLM_ERR_CUDA";
        case AQLM_ERR_TIMEOUT: return "AQLM_ERR_TIMEOUT";
    }
    return "AQLM_ERR_UNKNOWN";
}

const char *aqlm_version(void) { return "0.1.0"; }

}  // extern "C"
