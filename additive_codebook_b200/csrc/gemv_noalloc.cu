// gemv_noalloc.cu -- aqlm_gemv for callers that cannot allocate device memory.
//
// aqlm_gemv needs a caller-allocated scratch buffer (fp32 partial sums,
// arrival counters and, from 4 tokens up, a status word) whenever a row's
// input range is split over several CTAs.  Some callers have no way to
// provide one: a plugin that an inference engine hands only its input and
// output pointers, or an engine that fixes its device memory at start-up and
// forbids any allocation afterwards.  aqlm_gemv_noalloc serves them with a
// scratch array that is part of the library itself: a file-scope __device__
// array of kNoAllocScratchBytes that every GPU which loads the library holds
// until the process exits.  Nothing here calls cudaMalloc, cudaFree or any
// allocating routine.
//
// The array's name is only a host-side stand-in for the device symbol, so the
// host looks up its device address with cudaGetSymbolAddress, once per device
// (with that device current), and passes that address to the kernels.  Only a
// successful lookup is kept: a failed one (say, attempted during a stream
// capture) is retried by the next call.
//
// Every call clears the arrival counters of its layout on the stream, but not
// the status word: a bounded wait that gave up stays recorded there until
// aqlm_gemv_noalloc_check reads and clears it.
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_gemv_scratch[kNoAllocScratchBytes];

std::mutex g_lookup_mu;
std::atomic<void *> g_scratch[kMaxDevices];  // null until a lookup succeeded

// Device address of the scratch array on the current device.
cudaError_t scratch_on_current_device(unsigned char **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    void *p = g_scratch[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_lookup_mu);
        p = g_scratch[dev].load(std::memory_order_relaxed);
        if (!p) {
            e = cudaGetSymbolAddress(&p, g_gemv_scratch);
            if (e != cudaSuccess || !p) return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
            g_scratch[dev].store(p, std::memory_order_release);
        }
    }
    *out = static_cast<unsigned char *>(p);
    return cudaSuccess;
}

// Byte offset of the status word of (shape, tokens)'s layout, or -1 if that
// path has none; the shape and token count must be valid.
long long status_offset(const aqlm_shape &shape, int32_t tokens) {
    return aqlm::gemv_status_offset(aqlm::make_dims(shape), tokens);
}

}  // namespace

extern "C" {

size_t aqlm_gemv_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

aqlm_status aqlm_gemv_noalloc(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                              const uint16_t *x, uint16_t *y, int32_t tokens, aqlm_shape shape,
                              aqlm_stream_t stream) {
    const aqlm_status st = aqlm::check_gemv_args(codes, codebooks, scales, x, y, tokens, shape);
    if (st != AQLM_OK) return st;
    const aqlm::Dims d = aqlm::make_dims(shape);
    const size_t need = aqlm::gemv_workspace_bytes(d, tokens);
    if (need > kNoAllocScratchBytes) return AQLM_ERR_WORKSPACE;
    unsigned char *scratch = nullptr;
    if (need > 0) {
        if (scratch_on_current_device(&scratch) != cudaSuccess) return AQLM_ERR_CUDA;
        // Clear the arrival counters on the stream (an earlier call of another
        // shape may have left partial sums there), up to the status word.
        const size_t off = aqlm::gemv_workspace_counter_offset(d, tokens);
        const long long so = status_offset(shape, tokens);
        const size_t end = so >= 0 ? (size_t)so : need;
        if (end > off &&
            cudaMemsetAsync(scratch + off, 0, end - off, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
            return AQLM_ERR_CUDA;
    }
    return aqlm_gemv(codes, codebooks, scales, x, y, tokens, shape, scratch, need, stream);
}

aqlm_status aqlm_gemv_noalloc_check(aqlm_shape shape, int32_t tokens, aqlm_stream_t stream) {
    if (aqlm_gemv_row_tokens(shape) < 1) return AQLM_ERR_UNSUPPORTED;  // the shape checks of aqlm_gemv_check
    if (tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return AQLM_ERR_INVALID_ARG;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (status_offset(shape, tokens) < 0) return cudaStreamSynchronize(cs) == cudaSuccess ? AQLM_OK : AQLM_ERR_CUDA;
    const size_t need = aqlm_gemv_workspace_bytes(shape, tokens);
    if (need > kNoAllocScratchBytes) return AQLM_ERR_WORKSPACE;
    unsigned char *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return AQLM_ERR_CUDA;
    return aqlm_gemv_check(shape, tokens, scratch, need, stream);
}

aqlm_status aqlm_test_gemv_noalloc_set_status(aqlm_shape shape, int32_t tokens, int32_t value, aqlm_stream_t stream) {
    if (aqlm_gemv_workspace_bytes(shape, tokens) > kNoAllocScratchBytes) return AQLM_ERR_WORKSPACE;
    if (aqlm_gemv_row_tokens(shape) < 1 || tokens < 1 || tokens > AQLM_GEMV_MAX_TOKENS) return AQLM_ERR_INVALID_ARG;
    const long long so = status_offset(shape, tokens);
    if (so < 0) return AQLM_ERR_UNSUPPORTED;
    unsigned char *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return AQLM_ERR_CUDA;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(scratch + so, &value, sizeof(value), cudaMemcpyHostToDevice, cs) != cudaSuccess)
        return AQLM_ERR_CUDA;
    return cudaStreamSynchronize(cs) == cudaSuccess ? AQLM_OK : AQLM_ERR_CUDA;
}

}  // extern "C"
