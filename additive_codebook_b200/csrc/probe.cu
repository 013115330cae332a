// probe.cu -- the random 16-byte gather rate that bounds the decode kernels.
//
// Section "Key AQLM quantization parameters" of "The AQLM Quantization
// Algorithm, Explained": more codewords make decoding slower.  On this GPU the
// reason is concrete: at one token a decode product needs one random 16-byte
// codeword per group and codebook (d_out * d_in / 8 * M of them), from a 1-2
// MiB codebook that lives in L2 (1x16, 2x16) or from a copy in shared memory
// (2x8).  This kernel measures how many such gathers per second the chip
// delivers through the same load paths the decode kernels use, so that the
// benchmark can state each decode kernel's fraction of that ceiling from a
// number measured in the same run.  It is a measurement, not part of the
// method.
#include "common.cuh"

namespace aqlm {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kProbeUnroll = 8;  // gathers in flight per thread

// Random indices from a 32-bit linear congruential generator (Numerical
// Recipes' constants), mapped to [0, entries) by the high half of a product.
template <int SRC>
__global__ void __launch_bounds__(kProbeThreads) probe_gather_kernel(const uint4 *__restrict__ table,
                                                                      uint32_t entries, int iters,
                                                                      uint32_t *__restrict__ sink) {
    extern __shared__ __align__(16) uint4 stab[];
    if constexpr (SRC == 1) {
        for (uint32_t i = threadIdx.x; i < entries; i += blockDim.x) stab[i] = table[i];
        __syncthreads();
    }
    const uint64_t pol = policy_evict_last();
    uint32_t h = (blockIdx.x * blockDim.x + threadIdx.x) * 2654435761u + 12345u;
    uint32_t acc = 0;
    for (int it = 0; it < iters; ++it) {
        uint4 v[kProbeUnroll];
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u) {
            h = h * 1664525u + 1013904223u;
            const uint32_t i = __umulhi(h, entries);
            v[u] = !AQLM_IN_BOUNDS(i < entries, kSiteProbe, i) ? make_uint4(0, 0, 0, 0)
                   : SRC == 0                                          ? ld_keep_u4(table + i, pol)
                                                                       : stab[i];
        }
#pragma unroll
        for (int u = 0; u < kProbeUnroll; ++u) acc ^= v[u].x + v[u].y + v[u].z + v[u].w;
    }
    sink[blockIdx.x * blockDim.x + threadIdx.x] = acc;
}

#ifdef AQLM_DEBUG_BOUNDS
// Records a bounds violation on purpose (site kSiteTest, index `index`) and
// touches no memory: the test of the debug-bounds mechanism itself.
__global__ void bounds_trip_kernel(uint64_t index) { (void)AQLM_IN_BOUNDS(false, kSiteTest, index); }
#endif

}  // namespace

AQLM_DEFINE_BOUNDS_READER(bounds_word_probe)

}  // namespace aqlm

extern "C" {

aqlm_status aqlm_debug_bounds_read(uint64_t *word, int32_t clear) {
    if (!word) return AQLM_ERR_INVALID_ARG;
    cudaError_t (*readers[])(unsigned long long *, bool) = {
        aqlm::bounds_word_dequant, aqlm::bounds_word_encode, aqlm::bounds_word_gemm, aqlm::bounds_word_lut,
        aqlm::bounds_word_rows,    aqlm::bounds_word_tc,     aqlm::bounds_word_probe};
    *word = 0;
    for (auto rd : readers) {
        unsigned long long w = 0;
        const cudaError_t e = rd(&w, clear != 0);
        if (e == cudaErrorNotSupported) return AQLM_ERR_UNSUPPORTED;
        if (e != cudaSuccess) return AQLM_ERR_CUDA;
        if (w && !*word) *word = w;
    }
    return AQLM_OK;
}

aqlm_status aqlm_test_debug_bounds_trip(uint64_t index, aqlm_stream_t stream) {
#ifdef AQLM_DEBUG_BOUNDS
    return aqlm::launch_kernel(aqlm::bounds_trip_kernel, dim3(1), dim3(1), 0, reinterpret_cast<cudaStream_t>(stream),
                               false, index) == cudaSuccess
               ? AQLM_OK
               : AQLM_ERR_CUDA;
#else
    (void)index;
    (void)stream;
    return AQLM_ERR_UNSUPPORTED;
#endif
}


size_t aqlm_probe_gather_sink_bytes(int32_t ctas_per_sm) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || ctas_per_sm < 1 || ctas_per_sm > 8) return 0;
    return (size_t)aqlm::num_sms(dev) * ctas_per_sm * aqlm::kProbeThreads * sizeof(uint32_t);
}

aqlm_status aqlm_probe_gather(const void *table, size_t table_bytes, int32_t source, int32_t ctas_per_sm,
                              int32_t iters, void *sink, size_t sink_bytes, uint64_t *gathers, aqlm_stream_t stream) {
    if (!table || !sink || !gathers || iters < 1 || ctas_per_sm < 1 || ctas_per_sm > 8) return AQLM_ERR_INVALID_ARG;
    if (source != 0 && source != 1) return AQLM_ERR_INVALID_ARG;
    if (table_bytes < 16 || table_bytes % 16 || table_bytes > (size_t)1 << 30) return AQLM_ERR_INVALID_ARG;
    if (source == 1 && table_bytes > 64 * 1024) return AQLM_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(table) | reinterpret_cast<uintptr_t>(sink)) & 15) return AQLM_ERR_MISALIGNED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return AQLM_ERR_CUDA;
    const int blocks = aqlm::num_sms(dev) * ctas_per_sm;
    if (sink_bytes < (size_t)blocks * aqlm::kProbeThreads * sizeof(uint32_t)) return AQLM_ERR_WORKSPACE;
    const uint32_t entries = (uint32_t)(table_bytes / 16);
    const uint4 *t = static_cast<const uint4 *>(table);
    uint32_t *s = static_cast<uint32_t *>(sink);
    const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (source == 0) {
        e = aqlm::launch_kernel(aqlm::probe_gather_kernel<0>, dim3(blocks), dim3(aqlm::kProbeThreads), 0, cs, false,
                                t, entries, iters, s);
    } else {
        e = aqlm::opt_in_dynamic_smem(aqlm::probe_gather_kernel<1>, table_bytes);
        if (e == cudaSuccess)
            e = aqlm::launch_kernel(aqlm::probe_gather_kernel<1>, dim3(blocks), dim3(aqlm::kProbeThreads),
                                    table_bytes, cs, false, t, entries, iters, s);
    }
    if (e != cudaSuccess) return AQLM_ERR_CUDA;
    *gathers = (uint64_t)blocks * aqlm::kProbeThreads * (uint64_t)iters * aqlm::kProbeUnroll;
    return AQLM_OK;
}

}  // extern "C"
