// gemv_kernels.cuh -- decode-time layer product y = W^ . x for 1..16 tokens.
//
// "The AQLM Quantization Algorithm, Explained", section "What is
// Multi-Codebook Quantization (MCQ)?": every group of 8 inputs of row i is
// sum_m C_m[b(i,j,m)], scaled by s_i; the layer output is the product of the
// decoded rows with the activations.  Section "Why and what do we quantize?":
// decoding is bound by memory bandwidth, so the codes (2 or 4 bytes per
// group) are the only large stream and every other operand stays on chip.
//
// Work decomposition (one CTA = 8 warps = a tile of 32 output rows):
//   - lane l of every warp owns row (tile * 32 + l); the 8 warps split the
//     row's code chunks (16 bytes = 8 groups, or 4 groups for 2x16) into 8
//     contiguous ranges, so every lane streams its own row's codes with
//     128-bit loads that skip L1 and leave L2 first;
//   - the activations of the CTA's input range are staged once in shared
//     memory as fp32; every lane of a warp works on the same group at the
//     same time, so each activation load is a broadcast;
//   - 1x16 and 2x16 codewords are gathered through L1/L2 with an evict-last
//     policy (1-2 MiB of codebooks stay cache resident); the two 2x8
//     codebooks (8 KiB) are staged in shared memory;
//   - each decoded group (M codewords summed in fp32) is reused for all T
//     tokens, so the arithmetic per code byte grows with T;
//   - the 8 warps' partial sums meet in shared memory; the row's sum is
//     scaled by s_i and rounded once to fp16.
// When T activations of the whole row do not fit in shared memory, the input
// range is split over gridDim.y CTAs whose fp32 partial sums go to the
// caller's workspace and a second kernel adds them in a fixed order.
#pragma once

#include <array>
#include <utility>

#include "common.cuh"

namespace aqlm {
namespace gemv_detail {

constexpr int kRowsPerCta = 32;
constexpr int kWarps = 8;
constexpr int kThreads = kRowsPerCta * kWarps;
constexpr int kXsBudget = 128 * 1024;  // bytes of fp32 activations per CTA

template <int M, int B>
struct Fmt {
    static constexpr int K = 1 << B;
    static constexpr int kCodeBytes = M * B / 8;           // per group
    static constexpr int kGroupsPerChunk = 16 / kCodeBytes;  // per 16-byte load
};

// Index of codebook m for group q (0 <= q < groups per chunk) of a 16-byte chunk.
template <int M, int B>
__device__ __forceinline__ uint32_t chunk_index(const uint4 &ch, int q, int m) {
    const uint32_t w[4] = {ch.x, ch.y, ch.z, ch.w};
    if constexpr (M == 1 && B == 16) {
        return (w[q >> 1] >> (16 * (q & 1))) & 0xffffu;
    } else if constexpr (B == 8) {  // 2x8: byte 2q is codebook 0, byte 2q+1 codebook 1
        return (w[q >> 1] >> (16 * (q & 1) + 8 * m)) & 0xffu;
    } else {  // 2x16: word q holds codebook 0 in its low half, codebook 1 in its high half
        return (w[q] >> (16 * m)) & 0xffffu;
    }
}

template <int M, int B, int T>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const uint8_t *__restrict__ codes,
                                                        const uint4 *__restrict__ codebooks,
                                                        const __half *__restrict__ scales,
                                                        const __half *__restrict__ x,
                                                        __half *__restrict__ y,
                                                        float *__restrict__ partial, int d_out,
                                                        int d_in, int G, int row_bytes,
                                                        int slab_groups) {
    using F = Fmt<M, B>;
    constexpr int GPC = F::kGroupsPerChunk;
    extern __shared__ __align__(16) unsigned char smem[];
    const int xs_stride = slab_groups * kGroup;  // floats per token
    float *xs = reinterpret_cast<float *>(smem);
    uint4 *cbs = reinterpret_cast<uint4 *>(smem + (size_t)T * xs_stride * sizeof(float));
    float *red = reinterpret_cast<float *>(cbs + (B == 8 ? M * F::K : 0));

    const int split = blockIdx.y;
    const int g0 = split * slab_groups;
    const int g1 = min(G, g0 + slab_groups);
    const int ng = g1 - g0;

    // Stage this CTA's activations as fp32: T x (ng * 8) values.
    for (int i = threadIdx.x; i < T * ng; i += kThreads) {
        const int t = i / ng, q = i - t * ng;
        const uint4 v = *reinterpret_cast<const uint4 *>(x + (size_t)t * d_in + (size_t)(g0 + q) * kGroup);
        float f[kGroup];
        half8_to_float8(v, f);
        float4 *dst = reinterpret_cast<float4 *>(xs + (size_t)t * xs_stride + q * kGroup);
        dst[0] = make_float4(f[0], f[1], f[2], f[3]);
        dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    if constexpr (B == 8) {
        for (int c = threadIdx.x; c < M * F::K; c += kThreads) cbs[c] = codebooks[c];
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kRowsPerCta + lane;
    const bool valid = row < d_out;
    const int c_lo = g0 / GPC, n_chunks = ng / GPC;  // G and slab_groups are multiples of GPC
    const int wc0 = c_lo + (n_chunks * warp) / kWarps;
    const int wc1 = c_lo + (n_chunks * (warp + 1)) / kWarps;
    const uint8_t *rowp = codes + (size_t)(valid ? row : 0) * row_bytes;

    const uint64_t stream_pol = policy_evict_first();
    const uint64_t keep_pol = policy_evict_last();
    float acc[T];
#pragma unroll
    for (int t = 0; t < T; ++t) acc[t] = 0.f;

    constexpr int kDepth = 4;  // code chunks in flight per lane
    for (int c = wc0; c < wc1; c += kDepth) {
        uint4 ch[kDepth];
#pragma unroll
        for (int u = 0; u < kDepth; ++u) {
            ch[u] = (valid && c + u < wc1) ? ld_stream_u4(rowp + (size_t)(c + u) * 16, stream_pol) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kDepth; ++u) {
            if (c + u >= wc1) break;
#pragma unroll
            for (int q = 0; q < GPC; ++q) {
                float w[kGroup];
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const uint32_t k = chunk_index<M, B>(ch[u], q, m);
                    const uint4 cw = (B == 8) ? cbs[m * F::K + k] : ld_keep_u4(codebooks + (size_t)m * F::K + k, keep_pol);
                    float f[kGroup];
                    half8_to_float8(cw, f);
#pragma unroll
                    for (int e = 0; e < kGroup; ++e) w[e] = (m == 0) ? f[e] : w[e] + f[e];
                }
                const float *xp = xs + ((c + u) * GPC + q - g0) * kGroup;
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const float4 a = *reinterpret_cast<const float4 *>(xp + (size_t)t * xs_stride);
                    const float4 b = *reinterpret_cast<const float4 *>(xp + (size_t)t * xs_stride + 4);
                    float s = acc[t];
                    s = fmaf(w[0], a.x, s);
                    s = fmaf(w[1], a.y, s);
                    s = fmaf(w[2], a.z, s);
                    s = fmaf(w[3], a.w, s);
                    s = fmaf(w[4], b.x, s);
                    s = fmaf(w[5], b.y, s);
                    s = fmaf(w[6], b.z, s);
                    s = fmaf(w[7], b.w, s);
                    acc[t] = s;
                }
            }
        }
    }

#pragma unroll
    for (int t = 0; t < T; ++t) red[(warp * T + t) * 32 + lane] = acc[t];
    __syncthreads();
    for (int i = threadIdx.x; i < T * 32; i += kThreads) {
        const int t = i >> 5, l = i & 31;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) sum += red[(w * T + t) * 32 + l];
        const int r = blockIdx.x * kRowsPerCta + l;
        if (r < d_out) {
            if (gridDim.y == 1) {
                y[(size_t)t * d_out + r] = __float2half_rn(sum * __half2float(scales[r]));
            } else {
                partial[((size_t)split * T + t) * d_out + r] = sum;
            }
        }
    }
}

using GemvFn = void (*)(const uint8_t *, const uint4 *, const __half *, const __half *, __half *, float *,
                        int, int, int, int, int);

template <int M, int B, int... Ts>
constexpr std::array<GemvFn, sizeof...(Ts)> gemv_table(std::integer_sequence<int, Ts...>) {
    return std::array<GemvFn, sizeof...(Ts)>{{&gemv_kernel<M, B, Ts + 1>...}};
}

// Kernel tables, one per format, each defined in its own translation unit.
GemvFn gemv_pick_1x16(int tokens);
GemvFn gemv_pick_2x8(int tokens);
GemvFn gemv_pick_2x16(int tokens);

}  // namespace gemv_detail
}  // namespace aqlm
