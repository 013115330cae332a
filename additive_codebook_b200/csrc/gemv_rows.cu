// gemv_rows.cu -- layer product for 1..4 tokens with coalesced code streaming.
//
// "The AQLM Quantization Algorithm, Explained", section "What is
// Multi-Codebook Quantization (MCQ)?": y_i = s_i * sum_j < sum_m C_m[b(i,j,m)],
// x_j >.  Section "Why and what do we quantize?": decoding is bound by
// memory traffic, and the codes are the only large stream.
//
// Design for few tokens: a warp owns whole rows; its 32 lanes take the row's
// 16-byte code chunks l, l + 32, l + 64, ... so every code load of the warp
// reads 512 contiguous bytes of one row (full DRAM bursts; measured on B200,
// reading the codes in row-strided 16-byte pieces instead cost about 5 us
// per 4096x4096 layer).  Each lane gathers the codewords of its chunk's
// groups (1x16 / 2x16 through L1/L2 with an evict-last policy; 2x8 from
// shared memory), multiplies them with every token's activations and keeps
// one fp32 partial sum per token; at the end of a row five shuffles per token
// add the 32 partials, lane 0 scales by s_i and rounds once to fp16.  No
// split, no workspace.
//   - Activations are staged once per CTA in shared memory as fp16,
//     transposed by chunk ([group within chunk][chunk]) so that the lanes of
//     a warp, which work on consecutive chunks, read consecutive 16 bytes.
//   - Software pipeline over the warp's (row, chunk) items: the code load of
//     item k+2 and the codeword gathers of item k+1 are in flight while item
//     k is multiplied; it runs across row boundaries.
//   - Programmatic dependent launch: codebooks are prefetched into L2 and
//     the first items' codes and codewords fetched before griddepcontrol.wait
//     (weights are constant); x is read and y written only after it.
#include "common.cuh"

namespace aqlm {
namespace {

constexpr int kRowWarps = 8;
constexpr int kRowThreads = kRowWarps * 32;

struct RowArgs {
    const uint8_t *codes;
    const uint4 *codebooks;
    const __half *scales;
    const __half *x;
    __half *y;
    int d_out, G, row_bytes;
};

template <int M, int B>
struct RowFmt {
    static constexpr int K = 1 << B;
    static constexpr int GPC = 16 / (M * B / 8);  // groups per 16-byte chunk
    static constexpr bool kSmemCodebook = (B == 8);
};

template <int M, int B>
__device__ __forceinline__ uint32_t code_index(const uint4 &ch, int q, int m) {
    const uint32_t w[4] = {ch.x, ch.y, ch.z, ch.w};
    if constexpr (M == 1 && B == 16) {
        return (w[q >> 1] >> (16 * (q & 1))) & 0xffffu;
    } else if constexpr (B == 8) {
        return (w[q >> 1] >> (16 * (q & 1) + 8 * m)) & 0xffu;
    } else {
        return (w[q] >> (16 * m)) & 0xffffu;
    }
}

template <int M, int B, int T>
__global__ void __launch_bounds__(kRowThreads) gemv_rows_kernel(const RowArgs a) {
    using F = RowFmt<M, B>;
    constexpr int GPC = F::GPC;
    extern __shared__ __align__(16) unsigned char smem[];
    const int n_chunks = a.G / GPC;
    uint4 *xs = reinterpret_cast<uint4 *>(smem);  // [T][GPC][n_chunks] groups of 8 fp16
    uint4 *cbs = xs + (size_t)T * a.G;            // 2x8: [M][256] codewords

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total_warps = gridDim.x * kRowWarps;
    const int gwarp = blockIdx.x * kRowWarps + warp;
    const int cpw = (n_chunks + 31) / 32;  // chunk slots per lane per row
    const uint64_t stream_pol = policy_evict_first();
    const uint64_t keep_pol = policy_evict_last();

    if constexpr (!F::kSmemCodebook) {
        if (threadIdx.x == 0) {  // this CTA's share of the (usually cold) codebooks into L2
            const uint32_t cb_bytes = (uint32_t)M * F::K * 16;
            const uint32_t share = ((cb_bytes + gridDim.x - 1) / gridDim.x + 255) & ~255u;
            const uint32_t off = blockIdx.x * share;
            if (off < cb_bytes)
                prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(a.codebooks) + off, min(share, cb_bytes - off),
                                 keep_pol);
        }
    } else {
        for (int c = threadIdx.x; c < M * F::K; c += kRowThreads) cbs[c] = a.codebooks[c];
    }

    // item k of this warp: row gwarp + total_warps * (k / cpw), chunk slot k % cpw
    auto item_row = [&](int k) { return gwarp + total_warps * (k / cpw); };
    auto load_code = [&](int k) -> uint4 {
        const int r = item_row(k);
        const int c = lane + 32 * (k % cpw);
        if (r < a.d_out && c < n_chunks) return ld_stream_u4(a.codes + (size_t)r * a.row_bytes + (size_t)c * 16, stream_pol);
        return make_uint4(0, 0, 0, 0);
    };
    auto gather = [&](const uint4 &ch, int k, uint4 (&cw)[GPC][M]) {
        const bool live = item_row(k) < a.d_out && lane + 32 * (k % cpw) < n_chunks;
#pragma unroll
        for (int q = 0; q < GPC; ++q) {
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const uint32_t idx = code_index<M, B>(ch, q, m);
                if constexpr (F::kSmemCodebook) {
                    cw[q][m] = cbs[m * F::K + idx];
                } else {
                    cw[q][m] = live ? ld_keep_u4(a.codebooks + (size_t)m * F::K + idx, keep_pol) : make_uint4(0, 0, 0, 0);
                }
            }
        }
    };

    uint4 cwA[GPC][M], cwB[GPC][M];
    uint4 ch_next = load_code(1);
    {
        const uint4 ch0 = load_code(0);
        if constexpr (!F::kSmemCodebook) gather(ch0, 0, cwA);
        grid_dep_wait();
        for (int i = threadIdx.x; i < T * a.G; i += kRowThreads) {  // stage x, transposed by chunk
            const int t = i / a.G, g = i - t * a.G;
            const int c = g / GPC, q = g - c * GPC;
            xs[((size_t)t * GPC + q) * n_chunks + c] = *reinterpret_cast<const uint4 *>(a.x + (size_t)i * kGroup);
        }
        __syncthreads();
        if constexpr (F::kSmemCodebook) gather(ch0, 0, cwA);
    }
    grid_dep_launch();

    float acc[T];
#pragma unroll
    for (int t = 0; t < T; ++t) acc[t] = 0.f;
    // y for the item's row once its last chunk slot has been added
    auto finish_item = [&](int k) {
        if (k % cpw != cpw - 1) return;
        const int r = item_row(k);
#pragma unroll
        for (int t = 0; t < T; ++t) {
            float v = acc[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && r < a.d_out) a.y[(size_t)t * a.d_out + r] = __float2half_rn(v * __half2float(a.scales[r]));
            acc[t] = 0.f;
        }
    };
    auto multiply = [&](const uint4 (&cw)[GPC][M], int k) {
        const int c = lane + 32 * (k % cpw);
        if (c >= n_chunks) return;
#pragma unroll
        for (int q = 0; q < GPC; ++q) {
            float w[kGroup], xv[kGroup];
            half8_to_float8(cw[q][0], w);
            if constexpr (M == 2) {
                float f[kGroup];
                half8_to_float8(cw[q][1], f);
#pragma unroll
                for (int e = 0; e < kGroup; ++e) w[e] += f[e];
            }
#pragma unroll
            for (int t = 0; t < T; ++t) {
                half8_to_float8(xs[((size_t)t * GPC + q) * n_chunks + c], xv);
                float s0 = w[0] * xv[0], s1 = w[1] * xv[1];
                s0 = fmaf(w[2], xv[2], s0);
                s1 = fmaf(w[3], xv[3], s1);
                s0 = fmaf(w[4], xv[4], s0);
                s1 = fmaf(w[5], xv[5], s1);
                s0 = fmaf(w[6], xv[6], s0);
                s1 = fmaf(w[7], xv[7], s1);
                acc[t] += s0 + s1;
            }
        }
    };

    // at the top of a trip: cwA holds item k's codewords, ch_next item k+1's codes
    for (int k = 0; item_row(k) < a.d_out; k += 2) {
        gather(ch_next, k + 1, cwB);
        ch_next = load_code(k + 2);
        multiply(cwA, k);
        finish_item(k);
        if (item_row(k + 1) >= a.d_out) break;
        gather(ch_next, k + 2, cwA);
        ch_next = load_code(k + 3);
        multiply(cwB, k + 1);
        finish_item(k + 1);
    }
}

}  // namespace

constexpr int kRowsMaxTokens = 4;

// Whole rows per warp when the tokens are few and T * d_in fp16 activations
// (+ 8 KiB of 2x8 codebooks) fit on chip.
bool gemv_rows_supported(const Dims &d, int T) {
    return T >= 1 && T <= kRowsMaxTokens && (size_t)T * d.d_in * 2 + 8192 <= 160 * 1024;
}

template <int M, int B>
void (*rows_fn(int T))(const RowArgs) {
    switch (T) {
        case 1: return gemv_rows_kernel<M, B, 1>;
        case 2: return gemv_rows_kernel<M, B, 2>;
        case 3: return gemv_rows_kernel<M, B, 3>;
        default: return gemv_rows_kernel<M, B, 4>;
    }
}

cudaError_t launch_gemv_rows(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                             uint16_t *y, int tokens, const Dims &d, int sms, cudaStream_t st) {
    RowArgs a;
    a.codes = static_cast<const uint8_t *>(codes);
    a.codebooks = reinterpret_cast<const uint4 *>(codebooks);
    a.scales = reinterpret_cast<const __half *>(scales);
    a.x = reinterpret_cast<const __half *>(x);
    a.y = reinterpret_cast<__half *>(y);
    a.d_out = d.d_out;
    a.G = d.G;
    a.row_bytes = d.row_bytes;
    const size_t smem = (size_t)tokens * d.G * 16 + ((d.B == 8) ? (size_t)d.M * 256 * 16 : 0);
    int grid = (d.d_out + kRowWarps - 1) / kRowWarps;
    if (grid > 2 * sms) grid = 2 * sms;
    void (*fn)(const RowArgs);
    if (d.M == 1) {
        fn = rows_fn<1, 16>(tokens);
    } else if (d.B == 8) {
        fn = rows_fn<2, 8>(tokens);
    } else {
        fn = rows_fn<2, 16>(tokens);
    }
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_kernel(fn, dim3(grid), dim3(kRowThreads), smem, st, true, a);
}

}  // namespace aqlm
