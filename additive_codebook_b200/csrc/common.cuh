// common.cuh -- small device helpers shared by the library's kernels.
#pragma once

#include <atomic>
#include <cstdint>
#include <mutex>
#include <tuple>
#include <vector>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "aqlm.h"

namespace aqlm {

constexpr int kGroup = 8;  // g: inputs per group, every supported format

// Layer geometry derived from an aqlm_shape.
struct Dims {
    int d_out;
    int d_in;
    int G;          // groups per row, d_in / 8
    int M;          // codebooks
    int B;          // bits per code
    int row_bytes;  // bytes of codes per row, G * M * B / 8
};

inline Dims make_dims(const aqlm_shape &s) {
    Dims d;
    d.d_out = s.d_out;
    d.d_in = s.d_in;
    d.G = s.d_in / kGroup;
    d.M = s.num_codebooks;
    d.B = s.codebook_bits;
    d.row_bytes = d.G * d.M * d.B / 8;
    return d;
}

// One layer of a decode launch that runs several layers reading the same
// activations (device pointers; layout as in aqlm.h).
struct RowLayerIn {
    const void *codes;
    const uint16_t *codebooks;
    const uint16_t *scales;
    uint16_t *y;
    int d_out;
};

// ---- debug bounds checks ------------------------------------------------------
// Built with -DAQLM_DEBUG_BOUNDS (the debug variant of the library), the
// kernels test the index of every computed global or shared-memory access
// before making it: an index out of range is recorded -- the first one, as
// (site << 48 | index) -- in a device word of its source file, and the access
// is skipped.  Nothing traps.  aqlm_debug_bounds_read() collects the words of
// all files.  In the product build AQLM_IN_BOUNDS is `true` and costs nothing.
enum BoundsSite : uint32_t {
    kSiteRowsCodes = 1, kSiteRowsX, kSiteRowsY, kSiteRowsPartial, kSiteRowsSmem,
    kSiteTcCodes, kSiteTcY, kSiteTcPartial, kSiteTcA,
    kSiteLutRing, kSiteLutTable, kSiteLutY, kSiteLutPartial,
    kSiteDequantCodes, kSiteDequantW,
    kSiteGemmY, kSiteGemmB, kSiteGemmCodebook,
    kSiteNearest, kSiteKmeans, kSiteEncode,
    kSiteProbe, kSiteTest
};
#ifdef AQLM_DEBUG_BOUNDS
namespace {
__device__ unsigned long long g_bounds_word;
}  // namespace
__device__ __forceinline__ bool in_bounds(bool ok, uint32_t site, uint64_t index) {
    if (!ok) atomicCAS(&g_bounds_word, 0ull, ((unsigned long long)site << 48) | (index & 0xffffffffffffull));
    return ok;
}
#define AQLM_IN_BOUNDS(cond, site, index) ::aqlm::in_bounds((cond), (site), (uint64_t)(index))
// Host: this file's word (and clear it); cudaErrorNotSupported never.
#define AQLM_DEFINE_BOUNDS_READER(fn)                                                              \
    cudaError_t fn(unsigned long long *word, bool clear) {                                         \
        cudaError_t e = cudaMemcpyFromSymbol(word, g_bounds_word, sizeof(*word));                  \
        if (e == cudaSuccess && clear && *word) {                                                  \
            const unsigned long long z = 0;                                                         \
            e = cudaMemcpyToSymbol(g_bounds_word, &z, sizeof(z));                                   \
        }                                                                                           \
        return e;                                                                                   \
    }
#else
#define AQLM_IN_BOUNDS(cond, site, index) true
#define AQLM_DEFINE_BOUNDS_READER(fn)                                                              \
    cudaError_t fn(unsigned long long *word, bool) {                                               \
        *word = 0;                                                                                  \
        return cudaErrorNotSupported;                                                               \
    }
#endif
// one reader per source file that has device code (defined at its end)
cudaError_t bounds_word_abi(unsigned long long *, bool);
cudaError_t bounds_word_dequant(unsigned long long *, bool);
cudaError_t bounds_word_encode(unsigned long long *, bool);
cudaError_t bounds_word_gemm(unsigned long long *, bool);
cudaError_t bounds_word_lut(unsigned long long *, bool);
cudaError_t bounds_word_rows(unsigned long long *, bool);
cudaError_t bounds_word_tc(unsigned long long *, bool);
cudaError_t bounds_word_probe(unsigned long long *, bool);

// ---- cache-hinted global loads (PTX ISA: ld with L1/L2 eviction priority) ----

// L2 eviction policies (PTX createpolicy), passed to cache-hinted loads.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Streaming read-only 16-byte load: not kept in L1, first out of L2.
__device__ __forceinline__ uint4 ld_stream_u4(const void *p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

// 16-byte load that should stay resident in L1 and L2 (codebooks).  The
// plain (coherent) load path: measured on B200, random codeword gathers
// through the non-coherent read-only path (.nc) were slower (a 4096x4096
// 1x16 product took 13.0 us against 11.1 us).
__device__ __forceinline__ uint4 ld_keep_u4(const void *p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.L1::evict_last.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

// Asynchronous prefetch of [p, p + bytes) into L2 with an evict-last policy
// (cp.async.bulk.prefetch; p and bytes multiples of 16).
__device__ __forceinline__ void prefetch_l2_bulk(const void *p, uint32_t bytes, uint64_t pol) {
    asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;" ::"l"(p), "r"(bytes), "l"(pol)
                 : "memory");
}

// Programmatic dependent launch: wait until the preceding kernel in the
// stream has completed (and its writes are visible); let the next kernel in
// the stream start launching.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

// Eight fp16 values packed in a uint4 -> eight floats (exact conversion).
__device__ __forceinline__ void half8_to_float8(const uint4 &v, float *f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        __half2 h = *reinterpret_cast<const __half2 *>(&w[q]);
        float2 p = __half22float2(h);
        f[2 * q] = p.x;
        f[2 * q + 1] = p.y;
    }
}

// e += lo(c) * lo(x), o += hi(c) * hi(x): the fp16 halves of c and x
// multiplied and accumulated in fp32 by the mixed-precision fma of sm_100
// (PTX `fma.rn.f32.f16`).  The product of two fp16 values is exact in fp32,
// so this rounds exactly like converting both to fp32 first and fusing the
// multiply-add, without the conversions.
__device__ __forceinline__ void fma2_f16_f32(float &e, float &o, uint32_t c, uint32_t x) {
    asm("{.reg .f16 cl, ch, xl, xh;\n\t"
        "mov.b32 {cl, ch}, %2;\n\t"
        "mov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.f16 %0, cl, xl, %0;\n\t"
        "fma.rn.f32.f16 %1, ch, xh, %1;}"
        : "+f"(e), "+f"(o)
        : "r"(c), "r"(x));
}

// The kernels here hold at most a few bytes of static shared memory; opt in
// to the dynamic size whenever static + dynamic could pass the 48 KiB that a
// launch gets without the attribute.
template <typename... KArgs>
cudaError_t opt_in_dynamic_smem(void (*kern)(KArgs...), size_t bytes) {
    if (bytes + 1024 <= 48 * 1024) return cudaSuccess;
    // remember, per (kernel, device), the largest size already set, so that
    // repeated launches skip the driver call
    static std::mutex mu;
    static std::vector<std::tuple<const void *, int, size_t>> done;
    const void *key = reinterpret_cast<const void *>(kern);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const auto &e : done)
            if (std::get<0>(e) == key && std::get<1>(e) == dev && std::get<2>(e) >= bytes) return cudaSuccess;
    }
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && dev >= 0) {
        std::lock_guard<std::mutex> lock(mu);
        bool found = false;
        for (auto &d : done)
            if (std::get<0>(d) == key && std::get<1>(d) == dev) {
                if (std::get<2>(d) < bytes) std::get<2>(d) = bytes;
                found = true;
            }
        if (!found && done.size() < 1024) done.emplace_back(key, dev, bytes);
    }
    return e;
}

// Ask for the largest shared-memory carveout for `kern` (once per kernel and
// device).  An SM runs CTAs of different kernels side by side only under one
// L1 / shared-memory split; a kernel whose launches leave room for the next
// launch's CTA keeps that overlap across layers of different shapes only if
// every launch asks for the same split.
template <typename... KArgs>
cudaError_t prefer_max_shared_carveout(void (*kern)(KArgs...)) {
    static std::mutex mu;
    static std::vector<std::pair<const void *, int>> done;
    const void *key = reinterpret_cast<const void *>(kern);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const auto &e : done)
            if (e.first == key && e.second == dev) return cudaSuccess;
    }
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess && dev >= 0) {
        std::lock_guard<std::mutex> lock(mu);
        if (done.size() < 1024) done.emplace_back(key, dev);
    }
    return e;
}

// Launch through cudaLaunchKernelEx so that the returned error belongs to this
// launch only.  `pdl` allows programmatic dependent launch: the kernel may
// start while the previous kernel in the stream finishes, and must execute
// griddepcontrol.wait before touching memory that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (pdl) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// SM count of a device, queried once per device.
inline int num_sms(int device) {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> cached[kMaxDevices];
    if (device >= 0 && device < kMaxDevices) {
        const int c = cached[device].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device);
    if (n <= 0) return 148;
    if (device >= 0 && device < kMaxDevices) cached[device].store(n, std::memory_order_relaxed);
    return n;
}

// CTAs of `kern` resident per SM at this block size and dynamic shared
// memory (at least 1), cached per (device, kernel, threads, bytes): the
// occupancy query costs microseconds of host time per call.
inline int resident_ctas(const void *kern, int threads, size_t smem) {
    static std::mutex mu;
    static std::vector<std::tuple<int, const void *, int, size_t, int>> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lock(mu);
        for (const auto &e : cache)
            if (std::get<0>(e) == dev && std::get<1>(e) == kern && std::get<2>(e) == threads && std::get<3>(e) == smem)
                return std::get<4>(e);
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem) != cudaSuccess || occ < 1) {
        cudaGetLastError();  // leave no sticky error behind; fall back to one CTA per SM
        return 1;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (cache.size() < 4096) cache.emplace_back(dev, kern, threads, smem, occ);
    return occ;
}

}  // namespace aqlm

// Host-side launchers, one per kernel family (defined in the .cu files).
namespace aqlm {
cudaError_t launch_decode_indices(const void *codes, uint16_t *idx, const Dims &d, cudaStream_t st);
cudaError_t launch_dequant(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                           uint16_t *W, const Dims &d, cudaStream_t st);
aqlm_status check_gemv_args(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                            const uint16_t *y, int32_t tokens, const aqlm_shape &shape);
size_t gemv_workspace_bytes(const Dims &d, int tokens);
size_t gemv_workspace_counter_offset(const Dims &d, int tokens);
long long gemv_status_offset(const Dims &d, int tokens);
cudaError_t launch_gemv(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                        const uint16_t *x, uint16_t *y, int tokens, const Dims &d, void *workspace,
                        cudaStream_t st);
int gemv_row_tokens(const Dims &d);
size_t gemv_multi_workspace_bytes(const RowLayerIn *layers, int n, const Dims &d, int tokens);
size_t gemv_multi_counter_offset(const RowLayerIn *layers, int n, const Dims &d, int tokens);
long long gemv_multi_status_offset(const RowLayerIn *layers, int n, const Dims &d, int tokens);
cudaError_t launch_gemv_multi(const RowLayerIn *layers, int n, const uint16_t *x, int tokens, const Dims &d,
                              void *workspace, cudaStream_t st);
bool gemv_lut_supported(const Dims &d, int T);
size_t gemv_lut_workspace_bytes(const Dims &d, int sms);
cudaError_t launch_gemv_lut(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                            uint16_t *y, const Dims &d, void *workspace, int sms, cudaStream_t st);
cudaError_t launch_bf16_gemm(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                             int32_t *status, cudaStream_t st);
// Bound on any single wait of the GEMM kernels (a whole GEMM takes well under this).
constexpr unsigned long long kGemmWaitLimitNs = 2000000000ull;
int gemm_tile_n(int tokens, int n, int sms);
int gemm_pair_tile_n(int tokens, int n, int pairs);
bool gemm_uses_pair(int tokens);
size_t overlap_counter_bytes(int d_out, int d_in);
cudaError_t launch_overlap_gemm(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                                const uint16_t *X, uint16_t *W, uint16_t *Y, int tokens, const Dims &d,
                                int32_t *status, void *counters, cudaStream_t st);
// encoding (encode.cu)
cudaError_t launch_encode_scales(const float *W, int d_out, int d_in, uint16_t *scales, float *V, cudaStream_t st);
size_t nearest_workspace_bytes(long long N);
cudaError_t launch_nearest(const float *V, long long N, const float *C, int K, int32_t *idx, float *dist,
                           void *workspace, cudaStream_t st);
size_t kmeans_workspace_bytes(int K);
cudaError_t launch_kmeans_update(const float *V, const int32_t *idx, long long N, const float *C_prev, int K,
                                 float *C_out, int32_t *counts_out, void *workspace, cudaStream_t st);
size_t residual_kmeans_workspace_bytes(long long N, int K);
cudaError_t launch_residual_kmeans(const float *V, long long N, int M, int K, const int32_t *init_idx, int iters,
                                   float *C_out, void *workspace, cudaStream_t st);
size_t encode_codes_workspace_bytes(long long N, int M, int K);
cudaError_t launch_encode_codes(const float *V, long long N, const uint16_t *codebooks, int M, int K, void *codes,
                                int code_bytes, void *workspace, cudaStream_t st);
cudaError_t launch_round_codebooks(const float *C, long long n, uint16_t *C16, cudaStream_t st);
}  // namespace aqlm
