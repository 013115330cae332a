// gemv_kernels.cuh -- decode-time layer product y = W^ . x for 1..16 tokens,
// codeword-gather form (every format, every token count).
//
// "The AQLM Quantization Algorithm, Explained", section "What is
// Multi-Codebook Quantization (MCQ)?": every group of 8 inputs of row i is
// sum_m C_m[b(i,j,m)], scaled by s_i; the layer output is the product of the
// decoded rows with the activations.  Section "Why and what do we quantize?":
// decoding is bound by memory traffic, so the codes (2 or 4 bytes per group)
// are the only large stream and everything else stays on chip.
//
// Work decomposition (one CTA = 8 warps = a tile of 32 output rows):
//   - lane l of every warp owns row (tile * 32 + l); the CTA's input range is
//     a run of 16-byte code chunks (8 groups, or 4 for 2x16) that the 8
//     warps split into contiguous pieces, so each lane streams its own row's
//     codes with 128-bit loads that bypass L1 and leave L2 first;
//   - software pipeline per lane: the codeword gathers of chunk c+1 and the
//     code load of chunk c+2 are in flight while chunk c is multiplied;
//   - the activations of the CTA's input range are staged once in shared
//     memory as fp32, token-interleaved ([group][element][token], tokens
//     padded to a multiple of 4); all lanes of a warp work on the same group
//     at the same time, so every activation load is a broadcast, and for
//     several tokens one 16-byte load feeds two packed fp32x2 FMAs;
//   - codewords are gathered through L1/L2 with an evict-last policy (the
//     1-2 MiB of 1x16/2x16 codebooks stay cache resident; measured on B200,
//     random 16-byte gathers from L2 run at about one 32-byte sector per SM
//     clock, which bounds the batch-1 1x16 product);
//   - each decoded group (M codewords summed in fp32) is reused for all T
//     tokens, so the arithmetic per code byte grows with T;
//   - the warps' partial sums meet in shared memory.  When the row's input
//     range is split over gridDim.y CTAs (to fill the SMs, or because T
//     activations of the whole row do not fit on chip), every CTA writes its
//     fp32 partial sums to the caller's workspace and the last CTA of the row
//     tile to arrive (an atomic counter, no waiting) adds them in split order,
//     so the result is deterministic, and resets the counter;
//   - the row's sum is scaled by s_i and rounded once to fp16.
// Programmatic dependent launch: the weights (codes, codebooks, scales) are
// constant, so the first code chunks are loaded and the first chunk's
// codewords gathered before griddepcontrol.wait; x is read and y, the partial
// sums and the counters are written only after it.
#pragma once

#include <array>
#include <utility>

#include "common.cuh"

namespace aqlm {
namespace gemv_detail {

constexpr int kRowsPerCta = 32;
constexpr int kWarps = 8;
constexpr int kThreads = kRowsPerCta * kWarps;
constexpr int kXsBudget = 64 * 1024;  // bytes of fp32 activations per CTA

template <int M, int B>
struct Fmt {
    static constexpr int K = 1 << B;
    static constexpr int kCodeBytes = M * B / 8;             // per group
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

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

struct GemvArgs {
    const uint8_t *codes;
    const uint4 *codebooks;
    const __half *scales;
    const __half *x;
    __half *y;
    float *partial;      // [splits][T][d_out] when splits > 1
    uint32_t *counters;  // [row tiles] when splits > 1, zero between calls
    int d_out, d_in, G, row_bytes;
    int chunks_per_split;
};

// The codeword gathers of one 16-byte code chunk: GPC groups x M codebooks.
template <int M, int B>
__device__ __forceinline__ void gather_chunk(const uint4 &ch, const uint4 *__restrict__ codebooks, uint64_t pol,
                                             uint4 (&cw)[Fmt<M, B>::kGroupsPerChunk][M]) {
    using F = Fmt<M, B>;
#pragma unroll
    for (int q = 0; q < F::kGroupsPerChunk; ++q) {
#pragma unroll
        for (int m = 0; m < M; ++m) cw[q][m] = ld_keep_u4(codebooks + (size_t)m * F::K + chunk_index<M, B>(ch, q, m), pol);
    }
}

// Tokens padded to a multiple of 4 in shared memory (one token stays 1).
template <int T>
struct TokPad {
    static constexpr int value = (T == 1) ? 1 : ((T + 3) & ~3);
};

__device__ __forceinline__ unsigned long long pack2(float lo, float hi) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
// Two fp32 FMAs in one instruction (sm_100 packed fp32): d = a * b + c lane-wise.
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// acc += sum over the chunk's groups of < sum_m C_m[b], x_t[group] > for every
// token t.  Activations in shared memory as xs[(group * 8 + e) * TP + t]
// (fp32), read as warp-wide broadcasts.  One token: two partial sums per
// group shorten the dependent chain.  Several tokens: an LDS.128 brings 4
// tokens of one element and packed FMAs update 2 tokens per instruction.
template <int M, int B, int T>
__device__ __forceinline__ void fma_chunk(const uint4 (&cw)[Fmt<M, B>::kGroupsPerChunk][M], const float *xg,
                                          float (&acc1)[1], unsigned long long (&acc2)[(TokPad<T>::value + 1) / 2]) {
    using F = Fmt<M, B>;
    constexpr int TP = TokPad<T>::value;
#pragma unroll
    for (int q = 0; q < F::kGroupsPerChunk; ++q) {
        float w[kGroup];
        half8_to_float8(cw[q][0], w);
        if constexpr (M == 2) {
            float f[kGroup];
            half8_to_float8(cw[q][1], f);
#pragma unroll
            for (int e = 0; e < kGroup; ++e) w[e] += f[e];
        }
        const float *xq = xg + q * kGroup * TP;
        if constexpr (T == 1) {
            const float4 p = *reinterpret_cast<const float4 *>(xq);
            const float4 r = *reinterpret_cast<const float4 *>(xq + 4);
            float s0 = w[0] * p.x, s1 = w[1] * p.y;
            s0 = fmaf(w[2], p.z, s0);
            s1 = fmaf(w[3], p.w, s1);
            s0 = fmaf(w[4], r.x, s0);
            s1 = fmaf(w[5], r.y, s1);
            s0 = fmaf(w[6], r.z, s0);
            s1 = fmaf(w[7], r.w, s1);
            acc1[0] += s0 + s1;
        } else {
#pragma unroll
            for (int e = 0; e < kGroup; ++e) {
                const unsigned long long ww = pack2(w[e], w[e]);
#pragma unroll
                for (int t4 = 0; t4 < TP / 4; ++t4) {
                    const float4 v = *reinterpret_cast<const float4 *>(xq + e * TP + 4 * t4);
                    acc2[2 * t4] = ffma2(ww, pack2(v.x, v.y), acc2[2 * t4]);
                    acc2[2 * t4 + 1] = ffma2(ww, pack2(v.z, v.w), acc2[2 * t4 + 1]);
                }
            }
        }
    }
}

template <int M, int B, int T>
__global__ void __launch_bounds__(kThreads) gemv_kernel(const GemvArgs a) {
    using F = Fmt<M, B>;
    constexpr int GPC = F::kGroupsPerChunk;
    extern __shared__ __align__(16) unsigned char smem[];

    const int n_chunks_row = a.G / GPC;  // G is a multiple of GPC (rows are 16-byte multiples)
    const int split = blockIdx.y, splits = gridDim.y;
    const int c0 = split * a.chunks_per_split;
    const int c1 = min(n_chunks_row, c0 + a.chunks_per_split);
    const int g0 = c0 * GPC, ng = (c1 - c0) * GPC;
    constexpr int TP = TokPad<T>::value;
    float *xs = reinterpret_cast<float *>(smem);                              // [group][8][TP]
    float *red = xs + (size_t)a.chunks_per_split * GPC * kGroup * TP;         // [kWarps][T][32]
    __shared__ int s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kRowsPerCta + lane;
    const bool valid = row < a.d_out;
    const int nc = c1 - c0;
    const int wc0 = c0 + (nc * warp) / kWarps;
    const int wc1 = c0 + (nc * (warp + 1)) / kWarps;
    const uint8_t *rowp = a.codes + (size_t)(valid ? row : 0) * a.row_bytes;
    const uint64_t stream_pol = policy_evict_first();
    const uint64_t keep_pol = policy_evict_last();

    // The layer's codebooks are usually cold in L2 (every layer has its own):
    // each CTA asks L2 for its share of them before anything else.
    if (threadIdx.x == 0) {
        const uint32_t cb_bytes = (uint32_t)M * F::K * 16;
        const uint32_t n_cta = gridDim.x * gridDim.y;
        const uint32_t share = ((cb_bytes + n_cta - 1) / n_cta + 255) & ~255u;
        const uint32_t off = (blockIdx.y * gridDim.x + blockIdx.x) * share;
        if (off < cb_bytes) {
            prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(a.codebooks) + off, min(share, cb_bytes - off),
                             keep_pol);
        }
    }
    // Weights are constant: before waiting on the kernel that produces x,
    // load the first two code chunks and gather the first chunk's codewords.
    auto load_chunk = [&](int c) -> uint4 {
        return (valid && c < wc1) ? ld_stream_u4(rowp + (size_t)c * 16, stream_pol) : make_uint4(0, 0, 0, 0);
    };
    uint4 ch_cur = load_chunk(wc0);
    uint4 ch_nxt = load_chunk(wc0 + 1);
    uint4 cwA[GPC][M], cwB[GPC][M];
    gather_chunk<M, B>(ch_cur, a.codebooks, keep_pol, cwA);

    grid_dependency_wait();
    for (int i = threadIdx.x; i < TP * ng; i += kThreads) {  // padded tokens are zeros
        const int t = i / ng, q = i - t * ng;
        float f[kGroup];
        if (t < T) {
            half8_to_float8(*reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.d_in + (size_t)(g0 + q) * kGroup), f);
        } else {
#pragma unroll
            for (int e = 0; e < kGroup; ++e) f[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < kGroup; ++e) xs[((size_t)q * kGroup + e) * TP + t] = f[e];
    }
    __syncthreads();
    grid_dependents_launch();

    float acc1[1] = {0.f};
    unsigned long long acc2[(TP + 1) / 2];
#pragma unroll
    for (int i = 0; i < (TP + 1) / 2; ++i) acc2[i] = 0ull;

    // software pipeline, two chunks per trip so both codeword buffers stay in
    // registers: at the top cwA holds chunk c's codewords and ch_nxt chunk
    // c+1's codes; chunk c+1's codewords and chunk c+2's codes are in flight
    // while chunk c is multiplied, and so on
    for (int c = wc0; c < wc1; c += 2) {
        if (c + 1 < wc1) {
            gather_chunk<M, B>(ch_nxt, a.codebooks, keep_pol, cwB);
            ch_nxt = load_chunk(c + 2);
        }
        fma_chunk<M, B, T>(cwA, xs + (size_t)(c * GPC - g0) * kGroup * TP, acc1, acc2);
        if (c + 1 >= wc1) break;
        if (c + 2 < wc1) {
            gather_chunk<M, B>(ch_nxt, a.codebooks, keep_pol, cwA);
            ch_nxt = load_chunk(c + 3);
        }
        fma_chunk<M, B, T>(cwB, xs + (size_t)((c + 1) * GPC - g0) * kGroup * TP, acc1, acc2);
    }

    float acc[T];
    if constexpr (T == 1) {
        acc[0] = acc1[0];
    } else {
#pragma unroll
        for (int i = 0; i < (TP + 1) / 2; ++i) {
            float lo, hi;
            asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc2[i]));
            if (2 * i < T) acc[2 * i] = lo;
            if (2 * i + 1 < T) acc[2 * i + 1] = hi;
        }
    }
#pragma unroll
    for (int t = 0; t < T; ++t) red[(warp * T + t) * 32 + lane] = acc[t];
    __syncthreads();
    const int tile_row0 = blockIdx.x * kRowsPerCta;
    if (splits == 1) {
        for (int i = threadIdx.x; i < T * 32; i += kThreads) {
            const int t = i >> 5, l = i & 31;
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) sum += red[(w * T + t) * 32 + l];
            const int r = tile_row0 + l;
            if (r < a.d_out) a.y[(size_t)t * a.d_out + r] = __float2half_rn(sum * __half2float(a.scales[r]));
        }
        return;
    }
    // Split input range: publish this CTA's partial sums, the last CTA of the
    // row tile to arrive adds all splits in order.
    for (int i = threadIdx.x; i < T * 32; i += kThreads) {
        const int t = i >> 5, l = i & 31;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) sum += red[(w * T + t) * 32 + l];
        const int r = tile_row0 + l;
        if (r < a.d_out) a.partial[((size_t)split * T + t) * a.d_out + r] = sum;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(&a.counters[blockIdx.x], 1u);
        s_last = (prev == (uint32_t)(splits - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int i = threadIdx.x; i < T * 32; i += kThreads) {
        const int t = i >> 5, l = i & 31;
        const int r = tile_row0 + l;
        if (r >= a.d_out) continue;
        // 8 partials in flight per thread, added in split order
        float sum = 0.f;
        for (int s0 = 0; s0 < splits; s0 += 8) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = (s0 + u < splits) ? __ldcg(&a.partial[((size_t)(s0 + u) * T + t) * a.d_out + r]) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) sum += v[u];
        }
        a.y[(size_t)t * a.d_out + r] = __float2half_rn(sum * __half2float(a.scales[r]));
    }
    if (threadIdx.x == 0) a.counters[blockIdx.x] = 0u;
}

using GemvFn = void (*)(const GemvArgs);

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
