// gemv.cu -- host side of the decode-time product: work plan, launch, and
// the fixed-order reduction of split partial sums.  The kernels are in
// gemv_kernels.cuh, instantiated per format in gemv_1x16.cu, gemv_2x8.cu and
// gemv_2x16.cu.
#include "gemv_kernels.cuh"

namespace aqlm {
namespace gemv_detail {
namespace {

// y[t][r] = fp16(s_r * sum over splits of partial[split][t][r]), splits in order.
__global__ void gemv_finalize_kernel(const float *__restrict__ partial, const __half *__restrict__ scales,
                                     __half *__restrict__ y, int d_out, int tokens, int splits) {
    const int n = d_out * tokens;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const int r = i % d_out;
        float sum = 0.f;
        for (int s = 0; s < splits; ++s) sum += partial[(size_t)s * n + i];
        y[i] = __float2half_rn(sum * __half2float(scales[r]));
    }
}

struct Plan {
    int slab_groups;  // groups of the input range one CTA covers
    int splits;       // CTAs along the input dimension
    size_t smem;      // dynamic shared memory per CTA
};

// The whole row's activations (T x d_in fp32) stay on chip when they fit in
// kXsBudget; otherwise the input range is cut into equal slabs (multiples of
// 8 groups, so every slab holds whole 16-byte code chunks).
Plan plan_gemv(const Dims &d, int T) {
    int max_groups = kXsBudget / (kGroup * 4 * T);
    max_groups -= max_groups % 8;
    Plan p;
    if (d.G <= max_groups) {
        p.slab_groups = d.G;
        p.splits = 1;
    } else {
        const int splits = (d.G + max_groups - 1) / max_groups;
        int slab = (d.G + splits - 1) / splits;
        slab = (slab + 7) / 8 * 8;
        p.slab_groups = slab;
        p.splits = (d.G + slab - 1) / slab;
    }
    const size_t cb = (d.B == 8) ? (size_t)d.M * 256 * 16 : 0;
    p.smem = (size_t)T * p.slab_groups * kGroup * 4 + cb + (size_t)kWarps * T * 32 * 4;
    return p;
}

GemvFn pick(int M, int B, int T) {
    if (M == 1) return gemv_pick_1x16(T);
    if (B == 8) return gemv_pick_2x8(T);
    return gemv_pick_2x16(T);
}

}  // namespace
}  // namespace gemv_detail

size_t gemv_workspace_bytes(const Dims &d, int tokens) {
    const gemv_detail::Plan p = gemv_detail::plan_gemv(d, tokens);
    return p.splits > 1 ? (size_t)p.splits * tokens * d.d_out * sizeof(float) : 0;
}

cudaError_t launch_gemv(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                        const uint16_t *x, uint16_t *y, int tokens, const Dims &d, float *workspace,
                        cudaStream_t st) {
    using namespace gemv_detail;
    const Plan p = plan_gemv(d, tokens);
    GemvFn fn = pick(d.M, d.B, tokens);
    if (p.smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid((d.d_out + kRowsPerCta - 1) / kRowsPerCta, p.splits);
    cudaError_t e = launch_kernel(fn, grid, dim3(kThreads), p.smem, st, false,
                                  static_cast<const uint8_t *>(codes), reinterpret_cast<const uint4 *>(codebooks),
                                  reinterpret_cast<const __half *>(scales), reinterpret_cast<const __half *>(x),
                                  reinterpret_cast<__half *>(y), workspace, d.d_out, d.d_in, d.G, d.row_bytes,
                                  p.slab_groups);
    if (e != cudaSuccess || p.splits == 1) return e;
    int dev = 0;
    cudaGetDevice(&dev);
    const int n = d.d_out * tokens;
    int blocks = (n + 255) / 256;
    if (blocks > num_sms(dev) * 8) blocks = num_sms(dev) * 8;
    return launch_kernel(gemv_finalize_kernel, dim3(blocks), dim3(256), 0, st, false,
                         static_cast<const float *>(workspace), reinterpret_cast<const __half *>(scales),
                         reinterpret_cast<__half *>(y), d.d_out, tokens, p.splits);
}

}  // namespace aqlm
