// dequant.cu -- code unpacking and bf16 dequantisation.
//
// "The AQLM Quantization Algorithm, Explained", section "What is
// Multi-Codebook Quantization (MCQ)?": a group of g = 8 inputs of a row is
// the sum of M codewords whose indices are the stored B-bit codes; the sum is
// scaled by the row's scale.  Section "Why and what do we quantize?": the
// weights are fetched compressed and dequantised at runtime before the
// matmul.
//
// decode_indices is bound by HBM (2-4 bytes per group in, 2M bytes out).
// dequant reads M*B/8 bytes of codes per group and writes 16 bytes of bf16;
// for 2x8 that write stream is the bound, for 1x16/2x16 the codeword gathers
// from L2 (one 32-byte sector per 16-byte codeword) are.  The grids are a
// multiple of the SM count and stride over the work.
#include "common.cuh"

namespace aqlm {
namespace {

// idx[n] = unsigned value of code n, n over [d_out][G][M].
template <int B>
__global__ void decode_indices_kernel(const void *__restrict__ codes, uint16_t *__restrict__ idx,
                                      int64_t n_codes) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; n < n_codes; n += stride) {
        if constexpr (B == 8) {
            idx[n] = static_cast<const uint8_t *>(codes)[n];
        } else {
            idx[n] = static_cast<const uint16_t *>(codes)[n];
        }
    }
}

// W[i][8j+t] = bf16_rn(fp32(s_i) * (C_0[b0][t] + ... + C_{M-1}[b][t])), the
// additions in codebook order, every operation rounded on its own.
// A warp walks tiles of 32 * kPerLane consecutive groups (lane l handles
// groups l, l + 32, ...: every code load and every 16-byte store of the warp
// covers contiguous memory) in a software pipeline: the codes of tile k+2
// and the codeword gathers of tile k+1 are in flight while tile k is
// converted and stored.  Two groups per lane and at least three CTAs per SM
// (measured on B200: 2x8 11008x4096 took 28.7 us, against 36.9 us with four
// groups per lane at two CTAs per SM).
constexpr int kPerLane = 2;
constexpr int kTile = 32 * kPerLane;

template <int M, int B>
struct DequantStep {
    static constexpr int kCodeBytes = M * B / 8;
};

template <int M, int B>
__device__ __forceinline__ void load_codes(const uint8_t *__restrict__ codes, int64_t g0, int64_t n_groups,
                                           uint32_t (&raw)[kPerLane]) {
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
        const int64_t g = g0 + 32 * i;
        raw[i] = 0;
        if (g < n_groups) {
            if constexpr (DequantStep<M, B>::kCodeBytes == 2) {
                raw[i] = __ldcs(reinterpret_cast<const uint16_t *>(codes) + g);
            } else {
                raw[i] = __ldcs(reinterpret_cast<const uint32_t *>(codes) + g);
            }
        }
    }
}

template <int M, int B>
__device__ __forceinline__ uint32_t raw_index(uint32_t raw, int m) {
    if constexpr (M == 1) return raw & 0xffffu;
    else if constexpr (B == 8) return (raw >> (8 * m)) & 0xffu;
    else return (raw >> (16 * m)) & 0xffffu;
}

// Row of group g without a division per group: division by the invariant
// G as a multiply and a shift (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994): with s = ceil(log2 G)
// and m = floor(2^(31+s) / G) + 1 (< 2^32), floor(g * m / 2^(31+s)) = g / G
// for every 0 <= g < 2^31 (the error term g * (m - 2^(31+s)/G) / 2^(31+s)
// stays below 1/G).  Larger g take the plain 64-bit division.
struct RowDivider {
    int64_t G;
    uint32_t m;
    int shift;  // 31 + s
};

RowDivider make_row_divider(int G) {
    int s = 0;
    while ((1ll << s) < G) ++s;
    RowDivider r;
    r.G = G;
    r.m = (uint32_t)((1ull << (31 + s)) / (uint64_t)G + 1);
    r.shift = 31 + s;
    return r;
}

__device__ __forceinline__ int64_t row_of(int64_t g, const RowDivider &rd) {
    if (g < (1ll << 31)) return (int64_t)(((uint64_t)g * rd.m) >> rd.shift);
    return g / rd.G;
}

template <int M, int B>
__global__ void __launch_bounds__(256, 3) dequant_kernel(const uint8_t *__restrict__ codes,
                                                      const uint4 *__restrict__ codebooks,
                                                      const __half *__restrict__ scales,
                                                      uint4 *__restrict__ W, const RowDivider rd, int64_t n_groups) {
    constexpr int K = 1 << B;
    // the GEMM that reads W^ may launch now: its CTAs fit beside these, set up
    // their barriers and tensor memory, and wait for this grid before loading
    grid_dep_launch();
    // 2x8: both codebooks (2 x 256 codewords x 16 B = 8 KiB) live in shared memory.
    __shared__ uint4 cb_smem[B == 8 ? M * K : 1];
    if constexpr (B == 8) {
        for (int c = threadIdx.x; c < M * K; c += blockDim.x) cb_smem[c] = codebooks[c];
        __syncthreads();
    }
    const uint64_t keep = policy_evict_last();
    if constexpr (B == 16) {
        // every layer has its own 1-2 MiB of codebooks, usually cold in L2:
        // each CTA asks L2 for its share first
        if (threadIdx.x == 0) {
            const uint32_t cb_bytes = (uint32_t)M * K * 16;
            const uint32_t share = ((cb_bytes + gridDim.x - 1) / gridDim.x + 255) & ~255u;
            const uint32_t off = blockIdx.x * share;
            if (off < cb_bytes)
                prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(codebooks) + off, min(share, cb_bytes - off), keep);
        }
    }
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * (blockDim.x >> 5) * kTile;  // groups between a warp's tiles
    int64_t g0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kTile + lane;

    auto gather = [&](const uint32_t (&raw)[kPerLane], uint4 (&cw)[kPerLane][M]) {
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const uint32_t k = raw_index<M, B>(raw[i], m);
                cw[i][m] = (B == 8) ? cb_smem[m * K + k] : ld_keep_u4(codebooks + (size_t)m * K + k, keep);
            }
        }
    };
    auto emit = [&](const uint4 (&cw)[kPerLane][M], int64_t gt) {
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
            const int64_t g = gt + 32 * i;
            if (g >= n_groups) break;
            const int64_t row = row_of(g, rd);   // the division by G through the reciprocal: checked in debug builds
            if (!AQLM_IN_BOUNDS(row * rd.G <= g && g < (row + 1) * rd.G, kSiteDequantW, g)) continue;
            const float s = __half2float(scales[row]);
            float acc[kGroup];
            half8_to_float8(cw[i][0], acc);
#pragma unroll
            for (int m = 1; m < M; ++m) {
                float f[kGroup];
                half8_to_float8(cw[i][m], f);
#pragma unroll
                for (int t = 0; t < kGroup; ++t) acc[t] = __fadd_rn(acc[t], f[t]);
            }
            uint32_t out[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const __nv_bfloat16 lo = __float2bfloat16_rn(__fmul_rn(acc[2 * h], s));
                const __nv_bfloat16 hi = __float2bfloat16_rn(__fmul_rn(acc[2 * h + 1], s));
                out[h] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
            }
            W[g] = make_uint4(out[0], out[1], out[2], out[3]);
        }
    };

    uint32_t rawA[kPerLane], rawB[kPerLane];
    uint4 cwA[kPerLane][M], cwB[kPerLane][M];
    load_codes<M, B>(codes, g0, n_groups, rawA);
    load_codes<M, B>(codes, g0 + stride, n_groups, rawB);
    gather(rawA, cwA);
    // two tiles per trip so both buffers stay in registers
    for (; g0 - lane < n_groups; g0 += 2 * stride) {
        load_codes<M, B>(codes, g0 + 2 * stride, n_groups, rawA);
        gather(rawB, cwB);
        emit(cwA, g0);
        if (g0 + stride - lane >= n_groups) break;
        load_codes<M, B>(codes, g0 + 3 * stride, n_groups, rawB);
        gather(rawA, cwA);
        emit(cwB, g0 + stride);
    }
}

int grid_for(int64_t work, int threads, int per_sm) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int64_t want = (work + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms(dev) * per_sm;
    return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_decode_indices(const void *codes, uint16_t *idx, const Dims &d, cudaStream_t st) {
    const int64_t n = (int64_t)d.d_out * d.G * d.M;
    const int grid = grid_for(n, 256, 8);
    if (d.B == 8) return launch_kernel(decode_indices_kernel<8>, grid, 256, 0, st, false, codes, idx, n);
    return launch_kernel(decode_indices_kernel<16>, grid, 256, 0, st, false, codes, idx, n);
}

// One wave: as many CTAs as the SMs hold at once (by the kernel's register
// use), so every warp's tiles flow through its software pipeline without a
// second wave of CTAs waiting behind the first.
template <typename Kern>
int one_wave_grid(Kern kern, int64_t n_groups) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int occ = resident_ctas(reinterpret_cast<const void *>(kern), 256, 0);
    const int64_t tiles = (n_groups + kTile - 1) / kTile;
    const int64_t want = (tiles + 7) / 8;  // 8 warps per CTA
    const int64_t cap = (int64_t)num_sms(dev) * occ;
    return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

cudaError_t launch_dequant(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                           uint16_t *W, const Dims &d, cudaStream_t st) {
    const int64_t n = (int64_t)d.d_out * d.G;
    auto c = static_cast<const uint8_t *>(codes);
    auto cb = reinterpret_cast<const uint4 *>(codebooks);
    auto s = reinterpret_cast<const __half *>(scales);
    auto w = reinterpret_cast<uint4 *>(W);
    const RowDivider rd = make_row_divider(d.G);
    if (d.M == 1 && d.B == 16) {
        auto k = dequant_kernel<1, 16>;
        return launch_kernel(k, one_wave_grid(k, n), 256, 0, st, false, c, cb, s, w, rd, n);
    }
    if (d.M == 2 && d.B == 8) {
        auto k = dequant_kernel<2, 8>;
        return launch_kernel(k, one_wave_grid(k, n), 256, 0, st, false, c, cb, s, w, rd, n);
    }
    auto k = dequant_kernel<2, 16>;
    return launch_kernel(k, one_wave_grid(k, n), 256, 0, st, false, c, cb, s, w, rd, n);
}

AQLM_DEFINE_BOUNDS_READER(bounds_word_dequant)

}  // namespace aqlm
