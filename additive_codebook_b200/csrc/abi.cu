// abi.cu -- the extern "C" entry points of include/aqlm.h: host-side
// argument validation, workspace layout and kernel selection.  Nothing here
// allocates memory or keeps state between calls.
#include <cstdint>

#include "common.cuh"

namespace aqlm {
cudaError_t launch_bf16_gemm_ex(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                                int32_t *status, cudaStream_t st, unsigned long long limit_ns, int stall_test);
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

}  // namespace

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
    aqlm_status st = check_layer(codes, codebooks, scales, shape);
    if (st != AQLM_OK) return st;
    if (!x || !y || tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return AQLM_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 2)) return AQLM_ERR_MISALIGNED;
    const Dims d = aqlm::make_dims(shape);
    const size_t need = aqlm::gemv_workspace_bytes(d, tokens);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return AQLM_ERR_WORKSPACE;
    return from_cuda(aqlm::launch_gemv(codes, codebooks, scales, x, y, tokens, d, need > 0 ? workspace : nullptr,
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
    if (tokens < 1 || tokens > aqlm::gemv_row_tokens(d)) return 0;
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
    if (tokens > aqlm::gemv_row_tokens(d)) return AQLM_ERR_UNSUPPORTED;
    const size_t need = aqlm::gemv_multi_workspace_bytes(in, n_layers, d, tokens);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned(workspace, 16))) return AQLM_ERR_WORKSPACE;
    return from_cuda(aqlm::launch_gemv_multi(in, n_layers, x, tokens, d, need > 0 ? workspace : nullptr,
                                             to_cuda(stream)));
}

aqlm_status aqlm_gemv_check(aqlm_shape shape, int32_t tokens, void *workspace, size_t workspace_bytes,
                            aqlm_stream_t stream) {
    if (check_shape(shape) != AQLM_OK) return AQLM_ERR_UNSUPPORTED;
    if (tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return AQLM_ERR_INVALID_ARG;
    const Dims d = aqlm::make_dims(shape);
    const long long off = aqlm::gemv_status_offset(d, tokens);
    const cudaStream_t cs = to_cuda(stream);
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

size_t aqlm_gemm_workspace_bytes(aqlm_shape shape, int32_t tokens) {
    if (check_shape(shape) != AQLM_OK || tokens < 1) return 0;
    return kStatusBytes + (size_t)shape.d_out * shape.d_in * 2;
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
    uint16_t *W = reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(workspace) + kStatusBytes);
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), cs);
    if (e != cudaSuccess) return AQLM_ERR_CUDA;
    e = aqlm::launch_dequant(codes, codebooks, scales, W, aqlm::make_dims(shape), cs);
    if (e != cudaSuccess) return AQLM_ERR_CUDA;
    return from_cuda(aqlm::launch_bf16_gemm(X, W, Y, tokens, shape.d_out, shape.d_in, status, cs));
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

aqlm_status aqlm_test_gemm_timeout(const uint16_t *X, const uint16_t *W, uint16_t *Y, int32_t tokens, int32_t n,
                                   int32_t k, int32_t *status, uint64_t limit_ns, aqlm_stream_t stream) {
    if (!X || !W || !Y || !status || tokens < 1 || n < 1 || k < 1 || n % 8 || k % 8) return AQLM_ERR_INVALID_ARG;
    if (limit_ns == 0 || limit_ns > 1000000000ull) return AQLM_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(W, 16) || !aligned(Y, 16) || !aligned(status, 4)) return AQLM_ERR_MISALIGNED;
    return from_cuda(aqlm::launch_bf16_gemm_ex(X, W, Y, tokens, n, k, status, to_cuda(stream), limit_ns, 1));
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
