// gemv_noalloc.cu -- aqlm_gemv for callers that cannot allocate device memory.
//
// aqlm_gemv needs a caller-allocated scratch buffer (fp32 partial sums and
// arrival counters) whenever a row's input range is split over several
// CTAs.  Some callers have no way to provide one: a plugin that an inference
// engine hands only its input and output pointers, or an engine that fixes
// its device memory at start-up and forbids any allocation afterwards.
// aqlm_gemv_noalloc serves them with a scratch array that is part of the
// library itself: a file-scope __device__ array of kNoAllocScratchBytes that
// every GPU which loads the library holds until the process exits.  Nothing
// here calls cudaMalloc, cudaFree or any allocating routine.
//
// The array's name is only a host-side stand-in for the device symbol, so the
// host looks up its device address with cudaGetSymbolAddress, once per device
// (with that device current), and passes that address to the kernels.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_gemv_scratch[kNoAllocScratchBytes];

std::once_flag g_once[kMaxDevices];
void *g_scratch[kMaxDevices];
cudaError_t g_setup_err[kMaxDevices];

// Device address of the scratch array on the current device, looked up on the
// first call on that device.
cudaError_t scratch_on_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(g_once[dev], [dev] {
        void *p = nullptr;
        g_setup_err[dev] = cudaGetSymbolAddress(&p, g_gemv_scratch);
        g_scratch[dev] = (g_setup_err[dev] == cudaSuccess) ? p : nullptr;
    });
    if (g_setup_err[dev] != cudaSuccess) return g_setup_err[dev];
    *out = g_scratch[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

size_t aqlm_gemv_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

aqlm_status aqlm_gemv_noalloc(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                              const uint16_t *x, uint16_t *y, int32_t tokens, aqlm_shape shape,
                              aqlm_stream_t stream) {
    // aqlm_gemv_workspace_bytes validates the shape and token count (0 for both
    // "invalid" and "no scratch needed"; aqlm_gemv below tells them apart).
    const size_t need = aqlm_gemv_workspace_bytes(shape, tokens);
    if (need > kNoAllocScratchBytes) return AQLM_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (need > 0) {
        if (scratch_on_current_device(&scratch) != cudaSuccess) return AQLM_ERR_CUDA;
        // The arrival counters must start at zero; clear them on the stream
        // so the call never depends on what an earlier call left behind.
        const size_t off = aqlm::gemv_workspace_counter_offset(aqlm::make_dims(shape), tokens);
        cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
        if (cudaMemsetAsync(static_cast<unsigned char *>(scratch) + off, 0, need - off, cs) != cudaSuccess)
            return AQLM_ERR_CUDA;
    }
    return aqlm_gemv(codes, codebooks, scales, x, y, tokens, shape, scratch, need, stream);
}

}  // extern "C"
