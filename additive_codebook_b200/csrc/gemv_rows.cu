// gemv_rows.cu -- layer product for 1..3 tokens with coalesced code streaming.
//
// "The AQLM Quantization Algorithm, Explained", section "What is
// Multi-Codebook Quantization (MCQ)?": y_i = s_i * sum_j < sum_m C_m[b(i,j,m)],
// x_j >.  Section "Why and what do we quantize?": decoding is bound by
// memory traffic, and the codes are the only large stream.
//
// Design for few tokens: each CTA owns an equal contiguous range of rows (so
// every SM gets the same share of rows), and its warps own whole rows of
// that range, round robin; a warp's 32 lanes take the row's
// 16-byte code chunks l, l + 32, l + 64, ... so every code load of the warp
// reads 512 contiguous bytes of one row (full DRAM bursts; measured on B200,
// reading the codes in row-strided 16-byte pieces instead cost about 5 us
// per 4096x4096 layer).  Each lane gathers the codewords of its chunk's
// groups (1x16 / 2x16 through L1/L2 with an evict-last policy; 2x8 from
// shared memory), multiplies them with every token's activations and keeps
// one fp32 partial sum per token; at the end of a row five shuffles per token
// add the 32 partials, lane 0 scales by s_i and rounds once to fp16.
//   - Activations are staged once per CTA in shared memory as fp16,
//     transposed by chunk ([group within chunk][chunk]) so that the lanes of
//     a warp, which work on consecutive chunks, read consecutive 16 bytes.
//   - Software pipeline over the warp's (row, chunk) items: the code load of
//     item k+2 and the codeword gathers of item k+1 are in flight while item
//     k is multiplied; it runs across row boundaries.
//   - When T activations of the whole row do not fit the shared-memory
//     budget, the row's chunks are split over gridDim.y CTAs (each stages only
//     its slice of x); each writes fp32 row partials to the caller's workspace
//     and the last CTA of a row range to arrive (an atomic counter, no waiting)
//     adds them in split order, scales, rounds, and resets the counter.
//   - Programmatic dependent launch: codebooks are prefetched into L2 and
//     the first items' codes and codewords fetched before griddepcontrol.wait
//     (weights are constant); x is read and y, the partials and the counters
//     are written only after it.
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
    float *partial;        // [gridDim.y][T][d_out] when the input range is split
    uint32_t *counters;    // [gridDim.x] when split; zero between calls
    int d_out, d_in, G, row_bytes;
    int chunks_per_split;  // 16-byte code chunks of a row per CTA
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
    __shared__ int s_last;
    const int split = blockIdx.y, splits = gridDim.y;
    const int xstride = a.chunks_per_split;
    const int c0 = split * xstride;                       // first chunk of this CTA's slice
    const int n_chunks = min(a.G / GPC - c0, xstride);    // chunks in the slice
    uint4 *xs = reinterpret_cast<uint4 *>(smem);          // [T][GPC][xstride] groups of 8 fp16
    uint4 *cbs = xs + (size_t)T * GPC * xstride;          // 2x8: [M][256] codewords

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's rows: an equal contiguous share [r0, r1) of d_out, so that
    // every SM gets the same number of rows whichever CTAs it holds
    const int r0 = (int)((int64_t)blockIdx.x * a.d_out / gridDim.x);
    const int r1 = (int)((int64_t)(blockIdx.x + 1) * a.d_out / gridDim.x);
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

    // item k of this warp: row r0 + warp + 8 * (k / cpw), chunk slot k % cpw
    auto item_row = [&](int k) { return r0 + warp + kRowWarps * (k / cpw); };
    auto load_code = [&](int k) -> uint4 {
        const int r = item_row(k);
        const int c = lane + 32 * (k % cpw);
        if (r < r1 && c < n_chunks)
            return ld_stream_u4(a.codes + (size_t)r * a.row_bytes + (size_t)(c0 + c) * 16, stream_pol);
        return make_uint4(0, 0, 0, 0);
    };
    auto gather = [&](const uint4 &ch, int k, uint4 (&cw)[GPC][M]) {
        const bool live = item_row(k) < r1 && lane + 32 * (k % cpw) < n_chunks;
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
    const uint4 ch0 = load_code(0);
    {
        if constexpr (!F::kSmemCodebook) gather(ch0, 0, cwA);
        grid_dep_wait();
        const int ng = n_chunks * GPC;  // groups of the slice
        for (int i = threadIdx.x; i < T * ng; i += kRowThreads) {  // stage x, transposed by chunk
            const int t = i / ng, g = i - t * ng;
            const int c = g / GPC, q = g - c * GPC;
            xs[((size_t)t * GPC + q) * xstride + c] =
                *reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.d_in + (size_t)(c0 * GPC + g) * kGroup);
        }
        __syncthreads();
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
            if (lane == 0 && r < r1) {
                if (splits == 1) {
                    a.y[(size_t)t * a.d_out + r] = __float2half_rn(v * __half2float(a.scales[r]));
                } else {
                    a.partial[((size_t)split * T + t) * a.d_out + r] = v;
                }
            }
            acc[t] = 0.f;
        }
    };
    // the decoded group q of item k's chunk times every token's activations
    auto dot_group = [&](const uint4 &cw0, const uint4 &cw1, int q, int c) {
        float w[kGroup], xv[kGroup];
        half8_to_float8(cw0, w);
        if constexpr (M == 2) {
            float f[kGroup];
            half8_to_float8(cw1, f);
#pragma unroll
            for (int e = 0; e < kGroup; ++e) w[e] += f[e];
        }
#pragma unroll
        for (int t = 0; t < T; ++t) {
            half8_to_float8(xs[((size_t)t * GPC + q) * xstride + c], xv);
            float s0 = w[0] * xv[0], s1 = w[1] * xv[1];
            s0 = fmaf(w[2], xv[2], s0);
            s1 = fmaf(w[3], xv[3], s1);
            s0 = fmaf(w[4], xv[4], s0);
            s1 = fmaf(w[5], xv[5], s1);
            s0 = fmaf(w[6], xv[6], s0);
            s1 = fmaf(w[7], xv[7], s1);
            acc[t] += s0 + s1;
        }
    };
    auto multiply = [&](const uint4 (&cw)[GPC][M], int k) {
        const int c = lane + 32 * (k % cpw);
        if (c >= n_chunks) return;
#pragma unroll
        for (int q = 0; q < GPC; ++q) dot_group(cw[q][0], cw[q][M - 1], q, c);
    };

    if constexpr (F::kSmemCodebook) {
        // 2x8: codewords come from shared memory at use (short latency, so no
        // register copies of a whole item ahead); the codes run two items ahead
        uint4 ch = ch0;
        for (int k = 0; item_row(k) < r1; ++k) {
            const uint4 ch_after = load_code(k + 2);
            const int c = lane + 32 * (k % cpw);
            if (c < n_chunks) {
#pragma unroll
                for (int q = 0; q < GPC; ++q)
                    dot_group(cbs[code_index<M, B>(ch, q, 0)], cbs[F::K + code_index<M, B>(ch, q, M - 1)], q, c);
            }
            finish_item(k);
            ch = ch_next;
            ch_next = ch_after;
        }
    } else {
        // at the top of a trip: cwA holds item k's codewords, ch_next item k+1's codes
        for (int k = 0; item_row(k) < r1; k += 2) {
            gather(ch_next, k + 1, cwB);
            ch_next = load_code(k + 2);
            multiply(cwA, k);
            finish_item(k);
            if (item_row(k + 1) >= r1) break;
            gather(ch_next, k + 2, cwA);
            ch_next = load_code(k + 3);
            multiply(cwB, k + 1);
            finish_item(k + 1);
        }
    }
    if (splits == 1) return;

    // split input range: the last CTA of this row range adds the partials in split order
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&a.counters[blockIdx.x], 1u) == (uint32_t)(splits - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int i = threadIdx.x; i < (r1 - r0) * T; i += kRowThreads) {
        const int t = i / (r1 - r0), r = r0 + (i - t * (r1 - r0));
        float sum = 0.f;
        for (int s0 = 0; s0 < splits; s0 += 4) {  // 4 partials in flight, added in split order
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                v[u] = (s0 + u < splits) ? __ldcg(&a.partial[((size_t)(s0 + u) * T + t) * a.d_out + r]) : 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) sum += v[u];
        }
        a.y[(size_t)t * a.d_out + r] = __float2half_rn(sum * __half2float(a.scales[r]));
    }
    if (threadIdx.x == 0) a.counters[blockIdx.x] = 0u;
}

}  // namespace

// From 4 tokens on the tensor-core kernel is faster (measured on B200: 4 tokens
// 28672x8192 174 -> 149 us; at 3 tokens the two are even).
constexpr int kRowsMaxTokens = 3;
// Staged activations (+ 2x8 codebooks) per CTA.  Kept small on purpose: the
// shared-memory carveout comes out of L1, and L1 holds the codeword gathers
// in flight (measured on B200: a 4-token 8192x28672 layer with 114 KiB per
// CTA ran at 299 us, with 32 KiB slices at 176 us).
constexpr size_t kRowsSmemBudget = 32 * 1024;

namespace {

struct RowPlan {
    int splits;            // CTAs along the input range (gridDim.y)
    int chunks_per_split;  // 16-byte code chunks per row per CTA
    size_t smem;
};

// Work plan along the input range: split only as far as the staged
// activations require, in slices of whole 32-chunk lane slots (a slice of 75
// chunks would leave 21 of 32 lanes idle in its last slot).
RowPlan plan_rows(const Dims &d, int T) {
    const int gpc = 16 / (d.M * d.B / 8);
    const int n_chunks = d.G / gpc;
    const size_t cb = (d.B == 8) ? (size_t)d.M * 256 * 16 : 0;
    const size_t per_chunk = (size_t)T * gpc * 16;  // activation bytes per chunk of the slice
    const int max_slots = (int)((kRowsSmemBudget - cb) / (per_chunk * 32));
    const int slots = (n_chunks + 31) / 32;         // lane slots of a whole row
    RowPlan p;
    p.splits = max_slots < 1 ? (n_chunks + 31) / 32 : (slots + max_slots - 1) / max_slots;
    p.chunks_per_split = ((slots + p.splits - 1) / p.splits) * 32;
    if (p.chunks_per_split > n_chunks) p.chunks_per_split = n_chunks;
    p.splits = (n_chunks + p.chunks_per_split - 1) / p.chunks_per_split;
    p.smem = per_chunk * p.chunks_per_split + cb;
    return p;
}

// Row ranges (gridDim.x): as many CTAs as the SMs hold at once over all
// splits (by the kernel's registers and shared memory), at most one per 8 rows.
int rows_grid_x(const Dims &d, const RowPlan &p, int ctas_per_sm, int sms) {
    const int cap = (ctas_per_sm * sms) / p.splits > 0 ? (ctas_per_sm * sms) / p.splits : 1;
    const int sets = (d.d_out + kRowWarps - 1) / kRowWarps;
    return sets < cap ? sets : cap;
}

}  // namespace

size_t gemv_rows_counter_offset(const Dims &d, int T, int sms) {
    (void)sms;
    const RowPlan p = plan_rows(d, T);
    if (p.splits == 1) return 0;
    return ((size_t)p.splits * T * d.d_out * sizeof(float) + 15) / 16 * 16;
}

// Partials, then one arrival counter per possible row range (at most one per 8 rows).
size_t gemv_rows_workspace_bytes(const Dims &d, int T, int sms) {
    const RowPlan p = plan_rows(d, T);
    if (p.splits == 1) return 0;
    return gemv_rows_counter_offset(d, T, sms) + (size_t)((d.d_out + kRowWarps - 1) / kRowWarps) * sizeof(uint32_t);
}

bool gemv_rows_supported(int T) { return T >= 1 && T <= kRowsMaxTokens; }

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
                             uint16_t *y, int tokens, const Dims &d, void *workspace, int sms, cudaStream_t st) {
    const RowPlan p = plan_rows(d, tokens);
    RowArgs a;
    a.codes = static_cast<const uint8_t *>(codes);
    a.codebooks = reinterpret_cast<const uint4 *>(codebooks);
    a.scales = reinterpret_cast<const __half *>(scales);
    a.x = reinterpret_cast<const __half *>(x);
    a.y = reinterpret_cast<__half *>(y);
    a.partial = static_cast<float *>(workspace);
    a.counters = p.splits > 1 ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) +
                                                             gemv_rows_counter_offset(d, tokens, sms))
                              : nullptr;
    a.d_out = d.d_out;
    a.d_in = d.d_in;
    a.G = d.G;
    a.row_bytes = d.row_bytes;
    a.chunks_per_split = p.chunks_per_split;
    void (*fn)(const RowArgs);
    if (d.M == 1) {
        fn = rows_fn<1, 16>(tokens);
    } else if (d.B == 8) {
        fn = rows_fn<2, 8>(tokens);
    } else {
        fn = rows_fn<2, 16>(tokens);
    }
    cudaError_t e = opt_in_dynamic_smem(fn, p.smem);
    if (e != cudaSuccess) return e;
    const int occ = resident_ctas(reinterpret_cast<const void *>(fn), kRowThreads, p.smem);
    return launch_kernel(fn, dim3(rows_grid_x(d, p, occ, sms), p.splits), dim3(kRowThreads), p.smem, st, true, a);
}

}  // namespace aqlm
