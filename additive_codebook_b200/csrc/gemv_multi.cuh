// gemv_multi.cuh -- layer product for 5..16 tokens, several rows per lane.
//
// "The AQLM Quantization Algorithm, Explained", section "What is
// Multi-Codebook Quantization (MCQ)?": y_i = s_i * sum_j < sum_m C_m[b(i,j,m)],
// x_j > for every token.  With T tokens every decoded group is reused T times
// (8*T FMAs per group), so the product is bound by the FMA pipe and by how
// many shared-memory wavefronts feed it: a broadcast LDS.128 costs 4
// wavefronts on B200, so an activation value loaded once per row would cap
// the FMA pipe near a quarter of its rate.  Here each lane owns R rows
// (rows lane, lane+32, ... of the CTA's tile of 32*R rows), so every
// activation value loaded from shared memory feeds R rows' packed fp32x2 FMAs.
//
//   - activations staged once per CTA as fp16, token-interleaved
//     ([group][element][token], tokens padded to 8): one LDS.128 brings 8
//     tokens of one element, converted to 4 fp32 pairs;
//   - per group: the R (x M) codeword gathers of the next group are in
//     flight while the current group is multiplied; code chunks of the next
//     chunk are prefetched a chunk ahead;
//   - 4 warps per CTA split the CTA's input range; partial sums meet in
//     shared memory; an input range split over gridDim.y CTAs (to fill the
//     SMs or to fit T*d_in on chip) publishes fp32 partials to the workspace
//     and the last CTA of the row tile adds them in split order;
//   - programmatic dependent launch: weights only before griddepcontrol.wait.
#pragma once

#include <array>
#include <utility>

#include "common.cuh"

namespace aqlm {
namespace gemv_detail {

// Bytes of staged activations per CTA: small, so that L1 keeps room for the
// codeword gathers in flight (measured on B200, 24 KiB beat 64 KiB by 3-18%
// from 8 to 16 tokens).
constexpr int kXsBudget = 24 * 1024;

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

using GemvFn = void (*)(const GemvArgs);

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

constexpr int kMultiWarps = 4;
constexpr int kMultiThreads = kMultiWarps * 32;

template <int T>
struct MultiCfg {
    static constexpr int R = 4;                   // rows per lane
    static constexpr int TP8 = (T + 7) & ~7;      // tokens padded to 8 in shared memory
    static constexpr int kRows = 32 * R;          // rows per CTA
};

template <int M, int B, int T>
__global__ void __launch_bounds__(kMultiThreads) gemv_multi_kernel(const GemvArgs a) {
    using F = Fmt<M, B>;
    using C = MultiCfg<T>;
    constexpr int GPC = F::kGroupsPerChunk;
    constexpr int R = C::R, TP8 = C::TP8;
    extern __shared__ __align__(16) unsigned char smem[];

    const int n_chunks_row = a.G / GPC;
    const int split = blockIdx.y, splits = gridDim.y;
    const int c0 = split * a.chunks_per_split;
    const int c1 = min(n_chunks_row, c0 + a.chunks_per_split);
    const int g0 = c0 * GPC, ng = (c1 - c0) * GPC;
    __half *xh = reinterpret_cast<__half *>(smem);                                     // [group][8][TP8]
    float *red = reinterpret_cast<float *>(smem + (size_t)a.chunks_per_split * GPC * kGroup * TP8 * 2);
    __shared__ int s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile_row0 = blockIdx.x * C::kRows;
    const int nc = c1 - c0;
    const int wc0 = c0 + (nc * warp) / kMultiWarps;
    const int wc1 = c0 + (nc * (warp + 1)) / kMultiWarps;
    const uint64_t stream_pol = policy_evict_first();
    const uint64_t keep_pol = policy_evict_last();

    if (threadIdx.x == 0) {  // this CTA's share of the (usually cold) codebooks into L2
        const uint32_t cb_bytes = (uint32_t)M * F::K * 16;
        const uint32_t n_cta = gridDim.x * gridDim.y;
        const uint32_t share = ((cb_bytes + n_cta - 1) / n_cta + 255) & ~255u;
        const uint32_t off = (blockIdx.y * gridDim.x + blockIdx.x) * share;
        if (off < cb_bytes)
            prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(a.codebooks) + off, min(share, cb_bytes - off), keep_pol);
    }

    const uint8_t *rowp[R];
    bool valid[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int row = tile_row0 + lane + 32 * r;
        valid[r] = row < a.d_out;
        rowp[r] = a.codes + (size_t)(valid[r] ? row : 0) * a.row_bytes;
    }
    auto load_codes = [&](int c, uint4 (&ch)[R]) {
#pragma unroll
        for (int r = 0; r < R; ++r)
            ch[r] = (valid[r] && c < wc1) ? ld_stream_u4(rowp[r] + (size_t)c * 16, stream_pol) : make_uint4(0, 0, 0, 0);
    };
    auto gather = [&](const uint4 (&ch)[R], int q, uint4 (&cw)[R][M]) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
            for (int m = 0; m < M; ++m)
                cw[r][m] = ld_keep_u4(a.codebooks + (size_t)m * F::K + chunk_index<M, B>(ch[r], q, m), keep_pol);
        }
    };

    uint4 cur[R], nxt[R];
    load_codes(wc0, cur);
    load_codes(wc0 + 1, nxt);
    uint4 cwA[R][M], cwB[R][M];
    gather(cur, 0, cwA);

    grid_dep_wait();
    for (int i = threadIdx.x; i < TP8 * ng; i += kMultiThreads) {  // padded tokens are zeros
        const int t = i / ng, q = i - t * ng;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (t < T) v = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.d_in + (size_t)(g0 + q) * kGroup);
        const __half *h = reinterpret_cast<const __half *>(&v);
#pragma unroll
        for (int e = 0; e < kGroup; ++e) xh[((size_t)q * kGroup + e) * TP8 + t] = h[e];
    }
    __syncthreads();
    grid_dep_launch();

    unsigned long long acc[R][TP8 / 2];
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int i = 0; i < TP8 / 2; ++i) acc[r][i] = 0ull;
    }

    // multiply the group whose codewords are in cw with all tokens
    auto multiply = [&](const uint4 (&cw)[R][M], int g_local) {
        float w[R][kGroup];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            half8_to_float8(cw[r][0], w[r]);
            if constexpr (M == 2) {
                float f[kGroup];
                half8_to_float8(cw[r][1], f);
#pragma unroll
                for (int e = 0; e < kGroup; ++e) w[r][e] += f[e];
            }
        }
        const __half *xg = xh + (size_t)g_local * kGroup * TP8;
#pragma unroll
        for (int e = 0; e < kGroup; ++e) {
#pragma unroll
            for (int t8 = 0; t8 < TP8 / 8; ++t8) {
                const uint4 hv = *reinterpret_cast<const uint4 *>(xg + e * TP8 + 8 * t8);
                const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const float2 xf = __half22float2(*reinterpret_cast<const __half2 *>(&hw[p]));
                    const unsigned long long xx = pack2(xf.x, xf.y);
#pragma unroll
                    for (int r = 0; r < R; ++r) acc[r][4 * t8 + p] = ffma2(pack2(w[r][e], w[r][e]), xx, acc[r][4 * t8 + p]);
                }
            }
        }
    };

    for (int c = wc0; c < wc1; ++c) {
        const int gl = c * GPC - g0;
#pragma unroll
        for (int q = 0; q < GPC; q += 2) {
            // the next group's codewords are in flight while this one is multiplied
            gather(cur, q + 1, cwB);
            multiply(cwA, gl + q);
            if (q + 2 < GPC) {
                gather(cur, q + 2, cwA);
            } else if (c + 1 < wc1) {
                gather(nxt, 0, cwA);
            }
            multiply(cwB, gl + q + 1);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) cur[r] = nxt[r];
        load_codes(c + 2, nxt);
    }

    // partial sums of the 4 warps meet in shared memory: red[warp][t][row of tile]
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int i = 0; i < TP8 / 2; ++i) {
            float lo, hi;
            asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc[r][i]));
            if (2 * i < T) red[((size_t)warp * T + 2 * i) * C::kRows + 32 * r + lane] = lo;
            if (2 * i + 1 < T) red[((size_t)warp * T + 2 * i + 1) * C::kRows + 32 * r + lane] = hi;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < T * C::kRows; i += kMultiThreads) {
        const int t = i / C::kRows, rr = i - t * C::kRows;
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kMultiWarps; ++w) sum += red[((size_t)w * T + t) * C::kRows + rr];
        const int row = tile_row0 + rr;
        if (row >= a.d_out) continue;
        if (splits == 1) {
            a.y[(size_t)t * a.d_out + row] = __float2half_rn(sum * __half2float(a.scales[row]));
        } else {
            a.partial[((size_t)split * T + t) * a.d_out + row] = sum;
        }
    }
    if (splits == 1) return;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(&a.counters[blockIdx.x], 1u);
        s_last = (prev == (uint32_t)(splits - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int i = threadIdx.x; i < T * C::kRows; i += kMultiThreads) {
        const int t = i / C::kRows, rr = i - t * C::kRows;
        const int row = tile_row0 + rr;
        if (row >= a.d_out) continue;
        float sum = 0.f;
        for (int s0 = 0; s0 < splits; s0 += 8) {  // 8 partials in flight, added in split order
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                v[u] = (s0 + u < splits) ? __ldcg(&a.partial[((size_t)(s0 + u) * T + t) * a.d_out + row]) : 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u) sum += v[u];
        }
        a.y[(size_t)t * a.d_out + row] = __float2half_rn(sum * __half2float(a.scales[row]));
    }
    if (threadIdx.x == 0) a.counters[blockIdx.x] = 0u;
}

constexpr int kMultiMinTokens = 5;  // fewer tokens run on the row kernel

template <int M, int B, int... Ts>
constexpr std::array<GemvFn, sizeof...(Ts)> gemv_multi_table(std::integer_sequence<int, Ts...>) {
    return std::array<GemvFn, sizeof...(Ts)>{{&gemv_multi_kernel<M, B, Ts + kMultiMinTokens>...}};
}

// Kernel tables for 5..16 tokens, one per format, each in its own translation unit.
GemvFn gemv_multi_pick_1x16(int tokens);
GemvFn gemv_multi_pick_2x8(int tokens);
GemvFn gemv_multi_pick_2x16(int tokens);

}  // namespace gemv_detail
}  // namespace aqlm
