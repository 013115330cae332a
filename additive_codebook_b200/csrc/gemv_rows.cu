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
//   - Programmatic dependent launch: codebooks (and, for 2x8, x) are
//     prefetched into L2 and the first items' codes and codewords fetched
//     before griddepcontrol.wait (weights are constant); x is read and y, the
//     partials and the counters are written only after it.
#include "common.cuh"

namespace aqlm {
namespace {

// Fewest warps per CTA (the 1x16 / 2x16 kernels; 2x8 runs 16): the
// workspace keeps one arrival counter per kRowWarps rows.
constexpr int kRowWarps = 8;
constexpr int kRowMaxLayers = AQLM_MULTI_MAX_LAYERS;

// One layer of a launch.  A launch runs the layers that read the same x
// (one layer, or e.g. the q, k and v projections of an attention block):
// CTAs [cta0, next layer's cta0) own this layer's rows.
struct RowLayer {
    const uint8_t *codes;
    const uint4 *codebooks;
    const __half *scales;
    __half *y;
    int d_out;
    int row0;  // first row of the layer in the launch's concatenated rows
    int cta0;  // first CTA (blockIdx.x) of the layer
};

// NL: layers the kernel is built for (1, or kRowMaxLayers for launches of
// several layers; a single layer then skips the layer lookup and passes a
// quarter of the parameters).
template <int NL>
struct RowArgs {
    RowLayer layer[NL];
    int n_layers;
    const __half *x;
    float *partial;        // [gridDim.y][T][total_rows] when the input range is split
    uint32_t *counters;    // [gridDim.x] when split; zero between calls
    int total_rows, d_in, G, row_bytes;
    int chunks_per_split;  // 16-byte code chunks of a row per CTA
};

template <int M, int B>
struct RowFmt {
    static constexpr int K = 1 << B;
    static constexpr int GPC = 16 / (M * B / 8);  // groups per 16-byte chunk
    static constexpr bool kSmemCodebook = (B == 8);
    // 2x8 runs 16 warps (64 registers each) in one CTA per SM, 1x16 / 2x16
    // 8 warps (their codewords of two items ahead take 64 more registers).
    static constexpr int kWarps = kSmemCodebook ? 16 : 8;
    static constexpr int kThreads = kWarps * 32;
};

// 2x8 codebooks are held in shared memory as 8 copies, copy p in bank quad p
// (banks 4p..4p+3): codeword e of copy p is 16-byte word 8e + p.  Lane l
// reads copy l & 7, so the 8 lanes of each quarter warp touch 8 different
// bank quads whatever their codes are -- a warp's 16-byte gathers take 4
// shared-memory wavefronts, the minimum for 512 bytes, where one shared copy
// takes about twice that from bank conflicts.
constexpr int kCbCopies = 8;  // one per bank quad; the indexing below uses << 3 and & 7
static_assert(kCbCopies == 8, "copy index is lane & 7");

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

template <int M, int B, int T, int NL>
__global__ void __launch_bounds__(RowFmt<M, B>::kThreads, 2) gemv_rows_kernel(const RowArgs<NL> a) {
    using F = RowFmt<M, B>;
    constexpr int GPC = F::GPC;
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_last;
    const int split = blockIdx.y, splits = gridDim.y;
    const int xstride = a.chunks_per_split;
    const int c0 = split * xstride;                       // first chunk of this CTA's slice
    const int n_chunks = min(a.G / GPC - c0, xstride);    // chunks in the slice
    uint4 *xs = reinterpret_cast<uint4 *>(smem);          // [T][GPC][xstride] groups of 8 fp16
    uint4 *cbs = xs + (size_t)T * GPC * xstride;          // 2x8: [M][256][8 copies] codewords

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's layer (static indices only: the descriptors stay in the
    // kernel's parameter space) and its CTAs [L.cta0, cta_end)
    RowLayer L = a.layer[0];
    int cta_end = (int)gridDim.x;
#pragma unroll
    for (int i = 1; i < NL; ++i) {
        if (i < a.n_layers) {
            if ((int)blockIdx.x >= a.layer[i].cta0) {
                L = a.layer[i];
            } else if (a.layer[i].cta0 < cta_end) {
                cta_end = a.layer[i].cta0;
            }
        }
    }
    const int bx = NL == 1 ? (int)blockIdx.x : (int)blockIdx.x - L.cta0;
    const int nbx = NL == 1 ? (int)gridDim.x : cta_end - L.cta0;
    const int row0 = NL == 1 ? 0 : L.row0;
    // this CTA's rows: an equal contiguous share [r0, r1) of the layer's
    // d_out, so that every SM gets the same number of rows whichever CTAs it
    // holds; warp w owns rows r0 + w + kWarps j, j < n_rows
    const int r0 = (int)((int64_t)bx * L.d_out / nbx);
    const int r1 = (int)((int64_t)(bx + 1) * L.d_out / nbx);
    const int n_rows = r1 - r0 > warp ? (r1 - r0 - warp + F::kWarps - 1) / F::kWarps : 0;
    const int cpw = (n_chunks + 31) / 32;  // chunk slots per lane per row
    const int n_items = n_rows * cpw;      // item k = (row j = k / cpw, slot k % cpw)
    const uint64_t stream_pol = policy_evict_first();
    const uint64_t keep_pol = policy_evict_last();

    if constexpr (!F::kSmemCodebook) {
        if (threadIdx.x == 0) {  // this CTA's share of the (usually cold) codebooks into L2
            const uint32_t cb_bytes = (uint32_t)M * F::K * 16;
            const uint32_t share = ((cb_bytes + nbx - 1) / nbx + 255) & ~255u;
            const uint32_t off = bx * share;
            if (off < cb_bytes)
                prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(L.codebooks) + off, min(share, cb_bytes - off),
                                 keep_pol);
        }
    } else {
        for (int c = threadIdx.x; c < M * F::K * kCbCopies; c += F::kThreads) cbs[c] = L.codebooks[c >> 3];
        // 2x8 (whose CTA of the next launch is resident early): this CTA's
        // slice of the activations into L2.  A prefetch returns no value, so
        // it may precede the grid-dependency wait: what the previous grid
        // writes to x lands in L2, where the loads after the wait read it.
        // (1x16 / 2x16 CTAs start only as the previous launch's end, with no
        // lead time for it; measured there, it cost 0.1 us per 4096x4096 layer.)
        if (threadIdx.x == 32 && n_chunks > 0) {
            for (int t = 0; t < T; ++t)
                prefetch_l2_bulk(a.x + (size_t)t * a.d_in + (size_t)c0 * GPC * kGroup, (uint32_t)n_chunks * GPC * 16,
                                 keep_pol);
        }
    }
    // the scales of the warp's first 32 rows, lane j holding row j's (weights:
    // read before the grid-dependency wait, off the critical path)
    const float scale_j = (splits == 1 && lane < n_rows) ? __half2float(L.scales[r0 + warp + F::kWarps * lane]) : 0.f;

    // (row, slot) of an item, advanced without divisions
    struct Item {
        int j, s;
    };
    auto next = [&](Item it) -> Item {
        if (++it.s == cpw) {
            it.s = 0;
            ++it.j;
        }
        return it;
    };
    auto lane_live = [&](Item it) { return it.j < n_rows && lane + 32 * it.s < n_chunks; };
    auto load_code = [&](Item it) -> uint4 {
        if (lane_live(it)) {
            const int row = r0 + warp + F::kWarps * it.j, chunk = c0 + lane + 32 * it.s;
            if (AQLM_IN_BOUNDS(row < L.d_out && chunk * 16 < a.row_bytes, kSiteRowsCodes, (size_t)row * a.row_bytes))
                return ld_stream_u4(L.codes + (size_t)row * a.row_bytes + (size_t)chunk * 16, stream_pol);
        }
        return make_uint4(0, 0, 0, 0);
    };
    auto gather = [&](const uint4 &ch, Item it, uint4 (&cw)[GPC][M]) {
        const bool live = lane_live(it);
#pragma unroll
        for (int q = 0; q < GPC; ++q) {
#pragma unroll
            for (int m = 0; m < M; ++m)
                cw[q][m] = live ? ld_keep_u4(L.codebooks + (size_t)m * F::K + code_index<M, B>(ch, q, m), keep_pol)
                                : make_uint4(0, 0, 0, 0);
        }
    };

    // Weights only before the grid-dependency wait: the codes of the first
    // four items and (1x16 / 2x16) the codewords of the first two.
    Item it0 = {0, 0};
    Item it1 = next(it0);
    Item it2 = next(it1);
    Item it3 = next(it2);
    uint4 cwA[F::kSmemCodebook ? 1 : GPC][M], cwB[F::kSmemCodebook ? 1 : GPC][M];
    uint4 ch0 = load_code(it0), ch1 = load_code(it1), ch2 = load_code(it2), ch3 = load_code(it3);
    if constexpr (!F::kSmemCodebook) {
        gather(ch0, it0, cwA);
        gather(ch1, it1, cwB);
    }
    // the next launch may be scheduled from here on (its own wait still
    // holds it until this grid has completed)
    grid_dep_launch();
    grid_dep_wait();
    {
        const int ng = n_chunks * GPC;  // groups of the slice
        for (int i = threadIdx.x; i < T * ng; i += F::kThreads) {  // stage x, transposed by chunk
            const int t = i / ng, g = i - t * ng;
            const int c = g / GPC, q = g - c * GPC;
            if (AQLM_IN_BOUNDS((c0 * GPC + g + 1) * kGroup <= a.d_in && c < xstride, kSiteRowsX, c0 * GPC + g))
                xs[((size_t)t * GPC + q) * xstride + c] =
                    *reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.d_in + (size_t)(c0 * GPC + g) * kGroup);
        }
        __syncthreads();
    }

    // two fp32 chains per token (even and odd lanes of the groups)
    float acc[T], acc2[T];
#pragma unroll
    for (int t = 0; t < T; ++t) acc[t] = acc2[t] = 0.f;
    // y for the item's row once its last chunk slot has been added
    auto finish_item = [&](Item it) {
        if (it.s != cpw - 1) return;
        const int r = r0 + warp + F::kWarps * it.j;
        const float sc = __shfl_sync(0xffffffffu, scale_j, it.j & 31);
#pragma unroll
        for (int t = 0; t < T; ++t) {
            float v = acc[t] + acc2[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) {
                if (splits == 1) {
                    const float s_r = it.j < 32 ? sc : __half2float(L.scales[r]);
                    if (AQLM_IN_BOUNDS(r < L.d_out, kSiteRowsY, r)) L.y[(size_t)t * L.d_out + r] = __float2half_rn(v * s_r);
                } else {
                    if (AQLM_IN_BOUNDS(row0 + r < a.total_rows, kSiteRowsPartial, row0 + r))
                        a.partial[((size_t)split * T + t) * a.total_rows + row0 + r] = v;
                }
            }
            acc[t] = acc2[t] = 0.f;
        }
    };
    // the codewords of group q of the lane's chunk times every token's
    // activations: fp16 x fp16 products accumulated in fp32 (exact products)
    auto dot_group = [&](const uint4 &cw0, const uint4 &cw1, int q, int c) {
#pragma unroll
        for (int t = 0; t < T; ++t) {
            const uint4 xv = AQLM_IN_BOUNDS(c < xstride, kSiteRowsSmem, c) ? xs[((size_t)t * GPC + q) * xstride + c]
                                                                           : make_uint4(0, 0, 0, 0);
            fma2_f16_f32(acc[t], acc2[t], cw0.x, xv.x);
            fma2_f16_f32(acc[t], acc2[t], cw0.y, xv.y);
            fma2_f16_f32(acc[t], acc2[t], cw0.z, xv.z);
            fma2_f16_f32(acc[t], acc2[t], cw0.w, xv.w);
            if constexpr (M == 2) {
                fma2_f16_f32(acc[t], acc2[t], cw1.x, xv.x);
                fma2_f16_f32(acc[t], acc2[t], cw1.y, xv.y);
                fma2_f16_f32(acc[t], acc2[t], cw1.z, xv.z);
                fma2_f16_f32(acc[t], acc2[t], cw1.w, xv.w);
            }
        }
    };

    if constexpr (F::kSmemCodebook) {
        // 2x8: codewords from the shared-memory copies at use (short latency,
        // nothing held ahead in registers); codes four items ahead
        const int copy = lane & 7;
        Item it = it0, ahead = next(it3);
        for (int k = 0; k < n_items; ++k) {
            const uint4 ch_after = load_code(ahead);
            ahead = next(ahead);
            const int c = lane + 32 * it.s;
            if (c < n_chunks) {
#pragma unroll
                for (int q = 0; q < GPC; ++q)
                    dot_group(cbs[(code_index<M, B>(ch0, q, 0) << 3) | copy],
                              cbs[((F::K + code_index<M, B>(ch0, q, M - 1)) << 3) | copy], q, c);
            }
            finish_item(it);
            it = next(it);
            ch0 = ch1;
            ch1 = ch2;
            ch2 = ch3;
            ch3 = ch_after;
        }
    } else {
        // at the top of a trip: cwA / cwB hold items k / k+1's codewords,
        // ch2 / ch3 items k+2 / k+3's codes
        auto multiply = [&](const uint4 (&cw)[GPC][M], Item it) {
            const int c = lane + 32 * it.s;
            if (c >= n_chunks) return;
#pragma unroll
            for (int q = 0; q < GPC; ++q) dot_group(cw[q][0], cw[q][M - 1], q, c);
        };
        Item it = it0, g = it2, l = it3;
        auto refill = [&](uint4 (&cw)[GPC][M]) {  // gather item g, load the codes of item g + 2
            gather(ch2, g, cw);
            g = next(g);
            l = next(l);
            ch2 = ch3;
            ch3 = load_code(l);
        };
        for (int k = 0; k < n_items; k += 2) {
            multiply(cwA, it);
            finish_item(it);
            it = next(it);
            refill(cwA);
            if (k + 1 >= n_items) break;
            multiply(cwB, it);
            finish_item(it);
            it = next(it);
            refill(cwB);
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
    for (int i = threadIdx.x; i < (r1 - r0) * T; i += F::kThreads) {
        const int t = i / (r1 - r0), r = r0 + (i - t * (r1 - r0));
        float sum = 0.f;
        for (int s0 = 0; s0 < splits; s0 += 4) {  // 4 partials in flight, added in split order
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                v[u] = (s0 + u < splits) ? __ldcg(&a.partial[((size_t)(s0 + u) * T + t) * a.total_rows + row0 + r]) : 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) sum += v[u];
        }
        if (AQLM_IN_BOUNDS(r < L.d_out, kSiteRowsY, r))
            L.y[(size_t)t * L.d_out + r] = __float2half_rn(sum * __half2float(L.scales[r]));
    }
    if (threadIdx.x == 0) a.counters[blockIdx.x] = 0u;
}

}  // namespace

// Most tokens per format on this kernel; past them the tensor-core kernel is
// faster.  Measured on B200 (8192x8192, graphs of back-to-back launches, row
// kernel / tensor-core kernel): 1x16 2 tokens 36.7 / 40.5 us, 3 tokens 44.1 /
// 41.0 us; 2x16 3 tokens 69.3 / 72.5 us, 4 tokens 73.2 / 73.0 us; 2x8 (whose
// codebooks this kernel reads from shared memory) 4 tokens 38.1 / 41.3 us.
int rows_max_tokens(const Dims &d) {
    if (d.B == 8) return 4;
    return d.M == 2 ? 3 : 2;
}
// Staged activations per CTA (2x8 adds its 64 KiB of codebook copies).  Kept small on purpose: the
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
    const size_t cb = (d.B == 8) ? (size_t)d.M * 256 * 16 * kCbCopies : 0;
    const size_t per_chunk = (size_t)T * gpc * 16;  // activation bytes per chunk of the slice
    const int max_slots = (int)(kRowsSmemBudget / (per_chunk * 32));
    const int slots = (n_chunks + 31) / 32;         // lane slots of a whole row
    RowPlan p;
    p.splits = max_slots < 1 ? (n_chunks + 31) / 32 : (slots + max_slots - 1) / max_slots;
    p.chunks_per_split = ((slots + p.splits - 1) / p.splits) * 32;
    if (p.chunks_per_split > n_chunks) p.chunks_per_split = n_chunks;
    p.splits = (n_chunks + p.chunks_per_split - 1) / p.chunks_per_split;
    p.smem = per_chunk * p.chunks_per_split + cb;
    return p;
}

int row_warps(const Dims &d) { return d.B == 8 ? RowFmt<2, 8>::kWarps : RowFmt<1, 16>::kWarps; }
// the workspace holds one arrival counter per kRowWarps rows, and a launch
// has at most one CTA per row_warps() rows
static_assert(RowFmt<2, 8>::kWarps >= kRowWarps && RowFmt<1, 16>::kWarps >= kRowWarps &&
                  RowFmt<2, 16>::kWarps >= kRowWarps,
              "fewer warps per CTA than the workspace's counters allow");

// CTAs of one launch per SM.  2x8: one 16-warp CTA, half of what the SM
// holds, so that the next layer's CTA finds a free slot and fills its
// codebook copies and loads its first codes (before the grid-dependency
// wait) while this launch computes; measured on B200 (graph of back-to-back
// launches, 4096x4096): with every slot taken by one launch the next
// launch's CTAs started only as this launch's CTAs ended, and each CTA spent
// 2-3 us on loads before its first multiply.  A 2x8 launch of several layers
// (aqlm_gemv_multi) takes every slot instead: it has three times the rows per
// CTA, so its own warps matter more than the next launch's early start
// (measured: Llama-2-7B q/k/v in one launch 18.3 -> 13.4 us, gate/up 21.4 ->
// 20.8 us).  1x16 / 2x16: every slot, as the random codeword gathers need all
// the warps the SM holds (one 8-warp CTA per SM and launch measured slower:
// 4096x4096 10.6 against 9.8 us).
int ctas_per_sm_per_launch(const Dims &d, int resident, int n_layers) {
    if (d.B == 8 && n_layers == 1) return resident > 1 ? resident / 2 : 1;
    return resident;
}

// CTAs of each layer (gridDim.x is their sum): as many CTAs in all as the
// launch's share of the SMs over all splits, dealt to the layers in
// proportion to their rows, at least one and at most one per warp's worth of
// rows each.
void rows_grid(const int *d_outs, int n, const Dims &d, const RowPlan &p, int ctas_per_sm, int sms, int *ctas) {
    const int cap = (ctas_per_sm * sms) / p.splits > 0 ? (ctas_per_sm * sms) / p.splits : 1;
    const int warps = row_warps(d);
    long long want = 0, rows = 0;
    for (int l = 0; l < n; ++l) {
        want += (d_outs[l] + warps - 1) / warps;
        rows += d_outs[l];
    }
    for (int l = 0; l < n; ++l) {
        const int most = (d_outs[l] + warps - 1) / warps;
        int c = want <= cap ? most : (int)((long long)cap * d_outs[l] / rows);
        ctas[l] = c < 1 ? 1 : (c > most ? most : c);
    }
}

// Workspace: fp32 partials [splits][T][rows of all layers], then one arrival
// counter per CTA (a layer has at most one CTA per kRowWarps rows).
size_t rows_counter_offset(long long rows, const Dims &d, int T) {
    const RowPlan p = plan_rows(d, T);
    if (p.splits == 1) return 0;
    return ((size_t)p.splits * T * rows * sizeof(float) + 15) / 16 * 16;
}
size_t rows_workspace_bytes(const int *d_outs, int n, const Dims &d, int T) {
    const RowPlan p = plan_rows(d, T);
    if (p.splits == 1) return 0;
    long long rows = 0, counters = 0;
    for (int l = 0; l < n; ++l) {
        rows += d_outs[l];
        counters += (d_outs[l] + kRowWarps - 1) / kRowWarps;
    }
    return rows_counter_offset(rows, d, T) + (size_t)counters * sizeof(uint32_t);
}

}  // namespace

size_t gemv_rows_counter_offset(const Dims &d, int T, int sms) {
    (void)sms;
    return rows_counter_offset(d.d_out, d, T);
}

size_t gemv_rows_workspace_bytes(const Dims &d, int T, int sms) {
    (void)sms;
    return rows_workspace_bytes(&d.d_out, 1, d, T);
}

size_t gemv_rows_multi_counter_offset(const RowLayerIn *layers, int n, const Dims &d, int T) {
    long long rows = 0;
    for (int l = 0; l < n; ++l) rows += layers[l].d_out;
    return rows_counter_offset(rows, d, T);
}

size_t gemv_rows_multi_workspace_bytes(const RowLayerIn *layers, int n, const Dims &d, int T) {
    int d_outs[kRowMaxLayers];
    for (int l = 0; l < n; ++l) d_outs[l] = layers[l].d_out;
    return rows_workspace_bytes(d_outs, n, d, T);
}

bool gemv_rows_supported(const Dims &d, int T) { return T >= 1 && T <= rows_max_tokens(d); }

// The kernel for T tokens; token counts past the format's rows_max_tokens()
// are not built (nullptr).
template <int M, int B, int NL>
void (*rows_fn(int T))(const RowArgs<NL>) {
    constexpr int kMax = B == 8 ? 4 : (M == 2 ? 3 : 2);
    switch (T) {
        case 1: return gemv_rows_kernel<M, B, 1, NL>;
        case 2: return gemv_rows_kernel<M, B, 2, NL>;
        case 3: if constexpr (kMax >= 3) return gemv_rows_kernel<M, B, 3, NL>; else return nullptr;
        case 4: if constexpr (kMax >= 4) return gemv_rows_kernel<M, B, 4, NL>; else return nullptr;
        default: return nullptr;
    }
}

namespace {

template <int NL>
cudaError_t launch_rows(const RowLayerIn *layers, int n, const uint16_t *x, int tokens, const Dims &d,
                        void *workspace, int sms, cudaStream_t st) {
    const RowPlan p = plan_rows(d, tokens);
    void (*fn)(const RowArgs<NL>);
    if (d.M == 1) {
        fn = rows_fn<1, 16, NL>(tokens);
    } else if (d.B == 8) {
        fn = rows_fn<2, 8, NL>(tokens);
    } else {
        fn = rows_fn<2, 16, NL>(tokens);
    }
    if (!fn) return cudaErrorInvalidValue;
    if (d.B == 8) {  // one CTA per SM and launch, the next launch's CTA beside it: one carveout for all shapes
        const cudaError_t e = prefer_max_shared_carveout(fn);
        if (e != cudaSuccess) return e;
    }
    const int threads = row_warps(d) * 32;
    const int occ = resident_ctas(reinterpret_cast<const void *>(fn), threads, p.smem);
    int d_outs[kRowMaxLayers], ctas[kRowMaxLayers];
    for (int l = 0; l < n; ++l) d_outs[l] = layers[l].d_out;
    rows_grid(d_outs, n, d, p, ctas_per_sm_per_launch(d, occ, n), sms, ctas);
    RowArgs<NL> a = {};
    int cta0 = 0, row0 = 0;
    for (int l = 0; l < n; ++l) {
        RowLayer &L = a.layer[l];
        L.codes = static_cast<const uint8_t *>(layers[l].codes);
        L.codebooks = reinterpret_cast<const uint4 *>(layers[l].codebooks);
        L.scales = reinterpret_cast<const __half *>(layers[l].scales);
        L.y = reinterpret_cast<__half *>(layers[l].y);
        L.d_out = layers[l].d_out;
        L.row0 = row0;
        L.cta0 = cta0;
        row0 += layers[l].d_out;
        cta0 += ctas[l];
    }
    a.n_layers = n;
    a.x = reinterpret_cast<const __half *>(x);
    a.partial = static_cast<float *>(workspace);
    a.counters = p.splits > 1 ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) +
                                                             rows_counter_offset(row0, d, tokens))
                              : nullptr;
    a.total_rows = row0;
    a.d_in = d.d_in;
    a.G = d.G;
    a.row_bytes = d.row_bytes;
    a.chunks_per_split = p.chunks_per_split;
    cudaError_t e = opt_in_dynamic_smem(fn, p.smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(fn, dim3(cta0, p.splits), dim3(threads), p.smem, st, true, a);
}

}  // namespace

cudaError_t launch_gemv_rows_multi(const RowLayerIn *layers, int n, const uint16_t *x, int tokens, const Dims &d,
                                   void *workspace, int sms, cudaStream_t st) {
    if (n < 1 || n > kRowMaxLayers) return cudaErrorInvalidValue;
    if (n == 1) return launch_rows<1>(layers, n, x, tokens, d, workspace, sms, st);
    return launch_rows<kRowMaxLayers>(layers, n, x, tokens, d, workspace, sms, st);
}

cudaError_t launch_gemv_rows(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                             uint16_t *y, int tokens, const Dims &d, void *workspace, int sms, cudaStream_t st) {
    const RowLayerIn layer = {codes, codebooks, scales, y, d.d_out};
    return launch_gemv_rows_multi(&layer, 1, x, tokens, d, workspace, sms, st);
}

AQLM_DEFINE_BOUNDS_READER(bounds_word_rows)

}  // namespace aqlm
