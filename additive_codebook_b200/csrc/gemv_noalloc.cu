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
// Status word.  From 4 tokens up the product runs on the tensor cores with
// bounded waits, and a wait that gives up records AQLM_ERR_TIMEOUT in the
// workspace's last 16 bytes.  Here every such workspace is placed at the END
// of the array, so that word is always the array's last 16 bytes, whatever
// the shape; the layouts without a status word are placed at the start and
// kept clear of those bytes.  No call's partial sums or counters ever land on
// the word, each call clears only its own counters, and a recorded timeout
// therefore stays until aqlm_gemv_noalloc_check reads and clears it.
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

constexpr size_t kStatusBytes = 16;  // the array's last 16 bytes: the status word

// Where the workspace of (d, tokens) starts inside the array: at the end for
// layouts with a status word (which then falls on the array's last 16 bytes),
// at the start otherwise.
bool has_status_word(const aqlm::Dims &d, int32_t tokens) { return aqlm::gemv_status_offset(d, tokens) >= 0; }

size_t usable_bytes(const aqlm::Dims &d, int32_t tokens) {
    return has_status_word(d, tokens) ? kNoAllocScratchBytes : kNoAllocScratchBytes - kStatusBytes;
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
    if (need > usable_bytes(d, tokens)) return AQLM_ERR_WORKSPACE;
    unsigned char *ws = nullptr;
    if (need > 0) {
        unsigned char *scratch = nullptr;
        if (scratch_on_current_device(&scratch) != cudaSuccess) return AQLM_ERR_CUDA;
        const bool status = has_status_word(d, tokens);
        ws = status ? scratch + (kNoAllocScratchBytes - need) : scratch;  // need is a multiple of 16 there
        // Clear this layout's arrival counters on the stream (an earlier call of
        // another shape may have left partial sums there), not the status word.
        const size_t off = aqlm::gemv_workspace_counter_offset(d, tokens);
        const size_t end = status ? need - kStatusBytes : need;
        if (end > off &&
            cudaMemsetAsync(ws + off, 0, end - off, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
            return AQLM_ERR_CUDA;
    }
    return aqlm_gemv(codes, codebooks, scales, x, y, tokens, shape, ws, need, stream);
}

aqlm_status aqlm_gemv_noalloc_check(aqlm_stream_t stream) {
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    unsigned char *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return AQLM_ERR_CUDA;
    int32_t *word = reinterpret_cast<int32_t *>(scratch + kNoAllocScratchBytes - kStatusBytes);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, word, sizeof(h), cudaMemcpyDeviceToHost, cs) != cudaSuccess) return AQLM_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return AQLM_ERR_CUDA;
    if (h == 0) return AQLM_OK;
    if (cudaMemsetAsync(word, 0, sizeof(int32_t), cs) != cudaSuccess) return AQLM_ERR_CUDA;
    if (cudaStreamSynchronize(cs) != cudaSuccess) return AQLM_ERR_CUDA;
    return AQLM_ERR_TIMEOUT;
}

aqlm_status aqlm_test_gemv_noalloc_set_status(int32_t value, aqlm_stream_t stream) {
    unsigned char *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return AQLM_ERR_CUDA;
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(scratch + kNoAllocScratchBytes - kStatusBytes, &value, sizeof(value), cudaMemcpyHostToDevice,
                        cs) != cudaSuccess)
        return AQLM_ERR_CUDA;
    return cudaStreamSynchronize(cs) == cudaSuccess ? AQLM_OK : AQLM_ERR_CUDA;
}

}  // extern "C"
