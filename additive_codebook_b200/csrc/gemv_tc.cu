// gemv_tc.cu -- layer product for 5..16 tokens on the 5th-generation tensor
// cores, decoding the weights into shared memory on the fly.
//
// "The AQLM Quantization Algorithm, Explained", section "What is
// Multi-Codebook Quantization (MCQ)?": y_i = s_i * sum_j < sum_m C_m[b(i,j,m)],
// x_j > for every token.  With T tokens each decoded group is used T times,
// so past a few tokens the product is a skinny matrix product: D[128 rows][16
// tokens] += A[128 rows][64 inputs] . B[16 tokens][64 inputs]^T per stage,
// with A the decoded weights and B the activations, both K-major fp16, fp32
// accumulation in tensor memory.  Nothing is rounded on the way: the
// codewords are fp16 already and are copied into A as they are; with two
// codebooks each gets its own A tile and its own MMA into the same
// accumulator, (C_0[b0] + C_1[b1]) . x = C_0[b0] . x + C_1[b1] . x.
//
// One CTA = 128 output rows x a range of input stages (64 inputs = 8 groups
// each), 6 warps:
//   warps 0-3  decoders, one thread per row: read the row's codes of the
//              stage from the code tile, gather the codewords (1x16 / 2x16
//              through L1/L2 with an evict-last policy, 2x8 from shared
//              memory) one stage ahead, and write them into the stage's A
//              tile in the 128-byte-swizzled K-major layout that the MMA reads;
//              after the last stage they are the epilogue (tcgen05.ld of their
//              TMEM lane quarter, scale, fp16 store or fp32 partials);
//   warp 4     one thread issues the TMA loads: code tiles (64 bytes x 128
//              rows, two slots) and the activation tiles of every stage (64
//              inputs x 16 tokens, tokens past T read as zeros);
//   warp 5     allocates 32 TMEM columns; one thread issues
//              tcgen05.mma.cta_group::1.kind::f16 (M = 128, N = 16, K = 16)
//              and releases each stage with tcgen05.commit.
// An input range split over gridDim.y CTAs publishes fp32 partials to the
// workspace; the last CTA of the row tile to arrive (atomic counter, no
// waiting) adds them in split order.  Every mbarrier wait is bounded in time:
// one that gives up records AQLM_ERR_TIMEOUT in the workspace's status word,
// raises a CTA abort flag that the other roles poll, lets its copies and MMAs
// in flight finish (bounded) and frees its tensor memory; nothing traps.
// Programmatic dependent launch: codes and codebooks (weights) are read
// before griddepcontrol.wait; x, y and the workspace after it.
#include <cuda.h>

#include "common.cuh"

namespace aqlm {
namespace {

constexpr int kTcRows = 128;                 // rows per CTA = MMA M
constexpr int kTcN = 16;                     // tokens padded to the MMA N
constexpr int kStageK = 64;                  // inputs per stage
constexpr int kStageGroups = kStageK / kGroup;
constexpr int kTileBytes = kTcRows * 128;    // one A tile: 128 rows x 64 fp16
constexpr int kXBytes = kTcN * 128;          // one B tile: 16 tokens x 64 fp16
constexpr int kCodeBoxBytes = 64;            // code bytes per row per TMA box
constexpr int kCodeSlots = 2;
constexpr int kTcThreads = 192;
constexpr int kDecoders = 128;
constexpr uint64_t kTcWaitLimitNs = 1000000000ull;  // the whole product takes well under this
// f16 x f16 -> f32, both operands K-major, M = 128, N = 16 (instruction
// descriptor: D format bits 4-5, A/B formats bits 7-12 (0 = f16), N >> 3 at
// bits 17-22, M >> 4 at bits 24-28).
constexpr uint32_t kTcIdesc = (1u << 4) | ((uint32_t)(kTcN >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);

template <int M, int B>
struct TcFmt {
    static constexpr int K = 1 << B;
    static constexpr int kCodeBytesPerGroup = M * B / 8;
    static constexpr int kStageCodeBytes = kStageGroups * kCodeBytesPerGroup;   // 16 or 32
    static constexpr int kStagesPerBox = kCodeBoxBytes / kStageCodeBytes;       // 4 or 2
    static constexpr int kStages = (M == 1) ? 4 : 2;                            // A/B ring depth
    static constexpr int kStageBytes = M * kTileBytes + kXBytes;
    static constexpr int kCbBytes = (B == 8) ? M * K * 16 : 0;
    // ring (1024-aligned), code slots, 2x8 codebooks, barriers, + alignment slack
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + (size_t)kCodeSlots * kTcRows * kCodeBoxBytes +
                                    kCbBytes + 256;
};

struct TcBars {
    uint64_t full[4];
    uint64_t empty[4];
    uint64_t code_full[kCodeSlots];
    uint64_t code_empty[kCodeSlots];
    uint64_t acc_full;
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int last;
};

struct TcArgs {
    const uint4 *codebooks;
    const __half *scales;
    __half *y;
    float *partial;      // [splits][T][d_out] when gridDim.y > 1
    uint32_t *counters;  // [row tiles] when gridDim.y > 1, zero between calls
    int32_t *status;     // AQLM_ERR_TIMEOUT after a wait gave up
    int d_out, G, T;
    int stages_per_split, n_stages;
};

__device__ __forceinline__ uint32_t saddr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Wait for the phase of `parity`, for at most kTcWaitLimitNs; on a timeout
// record the status and raise the abort flag; give up when another role did.
__device__ bool tc_wait(uint32_t bar, uint32_t parity, TcBars *bars, int32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 0) {
            if (*reinterpret_cast<volatile int *>(&bars->abort_flag)) return false;
            if (now_ns() - t0 > kTcWaitLimitNs) {
                *reinterpret_cast<volatile int *>(&bars->abort_flag) = 1;
                atomicExch(status, (int32_t)AQLM_ERR_TIMEOUT);
                return false;
            }
        }
    }
}
// Bounded drain: wait for a phase without looking at the abort flag.
__device__ void tc_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = now_ns();
    while (!mbar_try_wait(bar, parity) && now_ns() - t0 < kTcWaitLimitNs) {
    }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
// Descriptor of a K-major tile in the 128-byte swizzle: rows of 128 bytes,
// 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t a) {
    uint64_t d = 0;
    d |= (uint64_t)((a & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kTcIdesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Index of codebook m of group q (0..7) of a stage from the row's V x 16 code bytes.
template <int M, int B, int V>
__device__ __forceinline__ uint32_t tc_index(const uint4 (&c)[V], int q, int m) {
    if constexpr (M == 1 && B == 16) {
        const uint32_t w[4] = {c[0].x, c[0].y, c[0].z, c[0].w};
        return (w[q >> 1] >> (16 * (q & 1))) & 0xffffu;
    } else if constexpr (B == 8) {  // 2 bytes per group: byte 0 codebook 0, byte 1 codebook 1
        const uint32_t w[4] = {c[0].x, c[0].y, c[0].z, c[0].w};
        return (w[q >> 1] >> (16 * (q & 1) + 8 * m)) & 0xffu;
    } else {  // 2x16: 4 bytes per group, codebook 0 in the low half
        const uint32_t w[8] = {c[0].x, c[0].y, c[0].z, c[0].w, c[1].x, c[1].y, c[1].z, c[1].w};
        return (w[q] >> (16 * m)) & 0xffffu;
    }
}

template <int M, int B>
__global__ void __launch_bounds__(kTcThreads, 2) gemv_tc_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                                                               const __grid_constant__ CUtensorMap tmap_x,
                                                               const TcArgs a) {
    using F = TcFmt<M, B>;
    constexpr int kCodeVecs = F::kStageCodeBytes / 16;  // 16-byte code pieces per row per stage
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = saddr(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw & 1023)) & 1023);
    uint8_t *ring = smem;                                                       // [stage][M A tiles | B tile]
    uint8_t *codes_s = ring + (size_t)F::kStages * F::kStageBytes;              // [slot][128 rows][64 B]
    uint4 *cbs = reinterpret_cast<uint4 *>(codes_s + (size_t)kCodeSlots * kTcRows * kCodeBoxBytes);  // 2x8
    TcBars *bars = reinterpret_cast<TcBars *>(reinterpret_cast<uint8_t *>(cbs) + F::kCbBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile_row0 = blockIdx.x * kTcRows;
    const int split = blockIdx.y, splits = gridDim.y;
    const int st0 = split * a.stages_per_split;
    const int n_st = min(a.n_stages - st0, a.stages_per_split);  // stages of this CTA (> 0)
    const int n_boxes = (n_st + F::kStagesPerBox - 1) / F::kStagesPerBox;

    if (threadIdx.x == 0) {
        for (int s = 0; s < F::kStages; ++s) {
            mbar_init(saddr(&bars->full[s]), kDecoders + 1);
            mbar_init(saddr(&bars->empty[s]), 1);
        }
        for (int s = 0; s < kCodeSlots; ++s) {
            mbar_init(saddr(&bars->code_full[s]), 1);
            mbar_init(saddr(&bars->code_empty[s]), kDecoders);
        }
        mbar_init(saddr(&bars->acc_full), 1);
        mbar_init(saddr(&bars->mma_done), 1);
        bars->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_codes)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    }
    if constexpr (B == 8) {
        for (int c = threadIdx.x; c < M * F::K; c += kTcThreads) cbs[c] = a.codebooks[c];
    } else if (threadIdx.x == 32) {  // this CTA's share of the (usually cold) codebooks into L2
        const uint32_t cb_bytes = (uint32_t)M * F::K * 16;
        const uint32_t n_cta = gridDim.x * gridDim.y;
        const uint32_t share = ((cb_bytes + n_cta - 1) / n_cta + 255) & ~255u;
        const uint32_t off = (blockIdx.y * gridDim.x + blockIdx.x) * share;
        if (off < cb_bytes)
            prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(a.codebooks) + off, min(share, cb_bytes - off),
                             policy_evict_last());
    }
    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&bars->tmem_base)),
                     "r"(32));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    grid_dep_launch();

    if (warp == 4) {
        if (lane == 0) {
            // ---- TMA producer: code boxes (weights) first, activations after the grid dependency ----
            int code_issued[kCodeSlots] = {-1, -1};
            int stage_issued[4] = {-1, -1, -1, -1};
            bool ok = true;
            int next_box = 0;
            auto issue_box = [&](int b) -> bool {
                const int slot = b % kCodeSlots;
                const uint32_t par = (uint32_t)((b / kCodeSlots) & 1);
                if (!tc_wait(saddr(&bars->code_empty[slot]), par ^ 1, bars, a.status)) return false;
                const uint32_t full = saddr(&bars->code_full[slot]);
                mbar_expect_tx(full, kTcRows * kCodeBoxBytes);
                tma_load_2d(saddr(codes_s + (size_t)slot * kTcRows * kCodeBoxBytes), &tmap_codes,
                            (st0 + b * F::kStagesPerBox) * F::kStageCodeBytes, tile_row0, full);
                code_issued[slot] = (int)par;
                return true;
            };
            for (; next_box < n_boxes && next_box < kCodeSlots && ok; ++next_box) ok = issue_box(next_box);
            grid_dep_wait();
            for (int i = 0; i < n_st && ok; ++i) {
                const int s = i % F::kStages;
                const uint32_t par = (uint32_t)((i / F::kStages) & 1);
                if (!tc_wait(saddr(&bars->empty[s]), par ^ 1, bars, a.status)) {
                    ok = false;
                    break;
                }
                const uint32_t full = saddr(&bars->full[s]);
                mbar_expect_tx(full, kXBytes);
                tma_load_2d(saddr(ring + (size_t)s * F::kStageBytes + (size_t)M * kTileBytes), &tmap_x,
                            (st0 + i) * kStageK, 0, full);
                stage_issued[s] = (int)par;
                // code box b reuses the slot of box b - 2, which the decoders release
                // when they store stage (b - 1) * stages-per-box - 1: issue it once
                // the activations up to that stage are on their way (the decoders
                // and the MMAs can always get that far), a box and more ahead of use
                if (next_box < n_boxes && i >= (next_box - 1) * F::kStagesPerBox - 1) {
                    ok = issue_box(next_box);
                    ++next_box;
                }
            }
            for (; next_box < n_boxes && ok; ++next_box) ok = issue_box(next_box);
            // no copy may still be landing in shared memory when the CTA exits
            for (int s = 0; s < kCodeSlots; ++s)
                if (code_issued[s] >= 0) tc_drain(saddr(&bars->code_full[s]), (uint32_t)code_issued[s]);
            for (int s = 0; s < F::kStages; ++s)
                if (stage_issued[s] >= 0) tc_drain(saddr(&bars->full[s]), (uint32_t)stage_issued[s]);
        }
        __syncwarp();
    } else if (warp == 5) {
        if (lane == 0) {
            // ---- MMA issuer ----
            bool ok = true;
            for (int i = 0; i < n_st; ++i) {
                const int s = i % F::kStages;
                const uint32_t par = (uint32_t)((i / F::kStages) & 1);
                if (!tc_wait(saddr(&bars->full[s]), par, bars, a.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = saddr(ring + (size_t)s * F::kStageBytes);
                const uint32_t b0 = a0 + (uint32_t)(M * kTileBytes);
#pragma unroll
                for (int k = 0; k < kStageK / 16; ++k) {
#pragma unroll
                    for (int m = 0; m < M; ++m)
                        mma_f16(tmem, sw128_desc(a0 + (uint32_t)(m * kTileBytes) + 32 * k), sw128_desc(b0 + 32 * k),
                                (i > 0 || k > 0 || m > 0) ? 1u : 0u);
                }
                mma_commit(saddr(&bars->empty[s]));
            }
            if (ok) mma_commit(saddr(&bars->acc_full));
            // tensor memory is freed only after every issued MMA completed
            mma_commit(saddr(&bars->mma_done));
            tc_drain(saddr(&bars->mma_done), 0);
        }
        __syncwarp();
    } else {
        // ---- decoders (thread = row of the tile), then the epilogue ----
        const int r = warp * 32 + lane;
        const int row = tile_row0 + r;
        const uint64_t keep = policy_evict_last();
        bool ok = true;
        uint4 code[kCodeVecs];
        uint4 cwA[kStageGroups][M], cwB[kStageGroups][M];
        // codes of stage i from its box; returns false on an abandoned wait
        auto read_codes = [&](int i) -> bool {
            const int b = i / F::kStagesPerBox, slot = b % kCodeSlots;
            if (i % F::kStagesPerBox == 0) {
                if (!tc_wait(saddr(&bars->code_full[slot]), (uint32_t)((b / kCodeSlots) & 1), bars, a.status))
                    return false;
            }
            const uint4 *src = reinterpret_cast<const uint4 *>(codes_s + (size_t)slot * kTcRows * kCodeBoxBytes +
                                                               (size_t)r * kCodeBoxBytes +
                                                               (size_t)(i % F::kStagesPerBox) * F::kStageCodeBytes);
#pragma unroll
            for (int v = 0; v < kCodeVecs; ++v) code[v] = src[v];
            return true;
        };
        auto gather = [&](uint4 (&cw)[kStageGroups][M]) {
#pragma unroll
            for (int q = 0; q < kStageGroups; ++q) {
#pragma unroll
                for (int m = 0; m < M; ++m) {
                    const uint32_t idx = tc_index<M, B, kCodeVecs>(code, q, m);
                    if constexpr (B == 8) {
                        cw[q][m] = cbs[m * F::K + idx];
                    } else {
                        cw[q][m] = ld_keep_u4(a.codebooks + (size_t)m * F::K + idx, keep);
                    }
                }
            }
        };
        // stage i's codewords into its A tiles (groups past the row end as zeros)
        auto store = [&](const uint4 (&cw)[kStageGroups][M], int i) -> bool {
            const int s = i % F::kStages;
            if (!tc_wait(saddr(&bars->empty[s]), (uint32_t)(((i / F::kStages) & 1) ^ 1), bars, a.status)) return false;
            const int g0 = (st0 + i) * kStageGroups;
            uint8_t *tile = ring + (size_t)s * F::kStageBytes + (size_t)r * 128;
#pragma unroll
            for (int q = 0; q < kStageGroups; ++q) {
                const bool live = g0 + q < a.G;
#pragma unroll
                for (int m = 0; m < M; ++m)
                    *reinterpret_cast<uint4 *>(tile + (size_t)m * kTileBytes + ((q ^ (r & 7)) << 4)) =
                        live ? cw[q][m] : make_uint4(0, 0, 0, 0);
            }
            fence_async_smem();
            mbar_arrive(saddr(&bars->full[s]));
            // the box's codes were consumed by this stage's gathers: its slot may
            // be refilled (released here, after the shared-memory reads of the
            // codes have certainly completed and after the proxy fence, not
            // right after the reads themselves)
            if (i % F::kStagesPerBox == F::kStagesPerBox - 1 || i == n_st - 1)
                mbar_arrive(saddr(&bars->code_empty[(i / F::kStagesPerBox) % kCodeSlots]));
            return true;
        };
        if (n_st > 0) {
            ok = read_codes(0);
            if (ok) gather(cwA);
        }
        // two stages per trip so both codeword buffers stay in registers
        for (int i = 0; i < n_st && ok; i += 2) {
            if (i + 1 < n_st) {
                ok = read_codes(i + 1);
                if (ok) gather(cwB);
            }
            if (ok) ok = store(cwA, i);
            if (!ok || i + 1 >= n_st) break;
            if (i + 2 < n_st) {
                ok = read_codes(i + 2);
                if (ok) gather(cwA);
            }
            if (ok) ok = store(cwB, i + 1);
        }

        // ---- epilogue ----
        grid_dep_wait();
        ok = ok && tc_wait(saddr(&bars->acc_full), 0, bars, a.status);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
            tc_fence_after();
            uint32_t v[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), v);
            if (row < a.d_out) {
                if (splits == 1) {
                    const float sc = __half2float(a.scales[row]);
                    for (int t = 0; t < a.T; ++t) a.y[(size_t)t * a.d_out + row] = __float2half_rn(__uint_as_float(v[t]) * sc);
                } else {
                    for (int t = 0; t < a.T; ++t)
                        a.partial[((size_t)split * a.T + t) * a.d_out + row] = __uint_as_float(v[t]);
                }
            }
        }
        if (splits > 1) {
            // the last CTA of the row tile adds the partials in split order
            __threadfence();
            asm volatile("bar.sync 1, %0;" ::"n"(kDecoders) : "memory");
            if (threadIdx.x == 0) {
                const int all_ok = !*reinterpret_cast<volatile int *>(&bars->abort_flag);
                bars->last = all_ok && (atomicAdd(&a.counters[blockIdx.x], 1u) == (uint32_t)(splits - 1));
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kDecoders) : "memory");
            if (bars->last) {
                __threadfence();
                if (row < a.d_out) {
                    const float sc = __half2float(a.scales[row]);
                    for (int t = 0; t < a.T; ++t) {
                        float sum = 0.f;
                        for (int s0 = 0; s0 < splits; s0 += 4) {  // 4 partials in flight, added in split order
                            float p[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                p[u] = (s0 + u < splits) ? __ldcg(&a.partial[((size_t)(s0 + u) * a.T + t) * a.d_out + row])
                                                         : 0.f;
#pragma unroll
                            for (int u = 0; u < 4; ++u) sum += p[u];
                        }
                        a.y[(size_t)t * a.d_out + row] = __float2half_rn(sum * sc);
                    }
                }
                if (threadIdx.x == 0) a.counters[blockIdx.x] = 0u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(32));
}

// ---- host side ----

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tc_encoder() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 2-D tensor [rows][cols] of `esize`-byte elements, row stride `stride_bytes`.
bool encode_2d(CUtensorMap *map, CUtensorMapDataType type, const void *base, uint64_t cols, uint64_t rows,
               uint64_t stride_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = tc_encoder();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {stride_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, type, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct TcPlan {
    int tiles;             // row tiles of 128 (gridDim.x)
    int splits;            // CTAs along the input range (gridDim.y)
    int stages_per_split;  // stages of 64 inputs per CTA, whole code boxes
    int n_stages;
};

int stages_per_box(const Dims &d) { return kCodeBoxBytes / (kStageGroups * d.M * d.B / 8); }

// About two waves of CTAs (two resident per SM), each a whole number of code
// boxes and at least two of them.
TcPlan plan_tc(const Dims &d, int sms) {
    TcPlan p;
    p.tiles = (d.d_out + kTcRows - 1) / kTcRows;
    p.n_stages = (d.G + kStageGroups - 1) / kStageGroups;
    const int spb = stages_per_box(d);
    int splits = (4 * sms + p.tiles - 1) / p.tiles;
    if (splits < 1) splits = 1;
    int sps = (p.n_stages + splits - 1) / splits;
    sps = (sps + spb - 1) / spb * spb;
    if (sps < 2 * spb) sps = 2 * spb;
    p.stages_per_split = sps;
    p.splits = (p.n_stages + sps - 1) / sps;
    return p;
}

inline size_t al16(size_t v) { return (v + 15) / 16 * 16; }

template <int M, int B>
cudaError_t launch_tc(const CUtensorMap &mc, const CUtensorMap &mx, const TcArgs &a, const TcPlan &p, cudaStream_t st) {
    auto fn = gemv_tc_kernel<M, B>;
    const cudaError_t e = opt_in_dynamic_smem(fn, TcFmt<M, B>::kSmem);
    if (e != cudaSuccess) return e;
    return launch_kernel(fn, dim3(p.tiles, p.splits), dim3(kTcThreads), TcFmt<M, B>::kSmem, st, true, mc, mx, a);
}

}  // namespace

constexpr int kTcMinTokens = 5;

bool gemv_tc_supported(int T) { return T >= kTcMinTokens && T <= AQLM_GEMV_MAX_TOKENS; }

// Workspace: [fp32 partials][arrival counters][status word], the last two
// zero before a call (the counters only when the input range is split).
size_t gemv_tc_counter_offset(const Dims &d, int T, int sms) {
    const TcPlan p = plan_tc(d, sms);
    return p.splits > 1 ? al16((size_t)p.splits * T * d.d_out * sizeof(float)) : 0;
}

size_t gemv_tc_workspace_bytes(const Dims &d, int T, int sms) {
    const TcPlan p = plan_tc(d, sms);
    const size_t counters = p.splits > 1 ? al16((size_t)p.tiles * sizeof(uint32_t)) : 0;
    return gemv_tc_counter_offset(d, T, sms) + counters + 16;
}

size_t gemv_tc_status_offset(const Dims &d, int T, int sms) { return gemv_tc_workspace_bytes(d, T, sms) - 16; }

cudaError_t launch_gemv_tc(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                           uint16_t *y, int tokens, const Dims &d, void *workspace, int sms, cudaStream_t st) {
    const TcPlan p = plan_tc(d, sms);
    CUtensorMap mc, mx;
    if (!encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, (uint64_t)d.row_bytes, (uint64_t)d.d_out,
                   (uint64_t)d.row_bytes, kCodeBoxBytes, kTcRows, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, (uint64_t)d.d_in, (uint64_t)tokens,
                   (uint64_t)d.d_in * 2, kStageK, kTcN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    TcArgs a;
    a.codebooks = reinterpret_cast<const uint4 *>(codebooks);
    a.scales = reinterpret_cast<const __half *>(scales);
    a.y = reinterpret_cast<__half *>(y);
    a.partial = reinterpret_cast<float *>(ws);
    a.counters = p.splits > 1 ? reinterpret_cast<uint32_t *>(ws + gemv_tc_counter_offset(d, tokens, sms)) : nullptr;
    a.status = reinterpret_cast<int32_t *>(ws + gemv_tc_status_offset(d, tokens, sms));
    a.d_out = d.d_out;
    a.G = d.G;
    a.T = tokens;
    a.stages_per_split = p.stages_per_split;
    a.n_stages = p.n_stages;
    if (d.M == 1) return launch_tc<1, 16>(mc, mx, a, p, st);
    if (d.B == 8) return launch_tc<2, 8>(mc, mx, a, p, st);
    return launch_tc<2, 16>(mc, mx, a, p, st);
}

}  // namespace aqlm
