// gemv_tc.cu -- layer product for 4..16 tokens on the 5th-generation tensor
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
// Work decomposition (stream-K): the (row tile of 128, stage of 64 inputs =
// 8 groups) units of the layer, tile-major, are cut into equal contiguous
// ranges, one per CTA, two CTAs per SM, so every SM gets the same work
// whatever the shape.  A CTA's range crosses at most a few tiles: it handles
// them as segments, one accumulator each; a segment that covers its whole
// tile is scaled and stored, the others publish fp32 partial sums to the
// workspace and the last segment of the tile to arrive (an atomic counter,
// no waiting) adds them in input order (deterministic), scales and stores.
// One CTA has 6 warps:
//   warps 0-3  decoders, one thread per row: read the row's codes of the
//              stage from the code tile and copy each codeword straight from
//              the codebook (through L1, L2 evict-last) into the stage's A tile
//              in the 128-byte-swizzled K-major layout that the MMA reads, with
//              16-byte cp.async copies; the stage's full barrier counts a
//              thread's arrival when its copies have landed, so a decoder never
//              waits for its gathers and runs up to the ring depth ahead;
//              after the last stage they are the epilogue (tcgen05.ld of their
//              TMEM lane quarter, scale, fp16 store or fp32 partials);
//   warp 4     one thread issues the TMA loads: code tiles (64 bytes x 128
//              rows in the 64-byte swizzle, two slots) and the activation tiles of every stage (64
//              inputs x 16 tokens, tokens past T read as zeros);
//   warp 5     allocates 32 TMEM columns; one thread issues
//              tcgen05.mma.cta_group::1.kind::f16 (M = 128, N = 16, K = 16)
//              and releases each stage with tcgen05.commit.
// Every mbarrier wait is bounded in time:
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
    // A/B ring depth (4 stages of 18 KiB for one codebook, 2 of 34 KiB for two)
    // and CTAs per SM (measured on B200: a 3-stage ring with three CTAs per SM
    // ran 1.6x slower than this)
    static constexpr int kStages = (M == 1) ? 4 : 2;
    static constexpr int kCtasPerSm = 2;
    static constexpr int kStageBytes = M * kTileBytes + kXBytes;
    // ring (1024-aligned), code slots, barriers, + alignment slack
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + (size_t)kCodeSlots * kTcRows * kCodeBoxBytes + 256;
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

// One layer of a launch.  A launch runs the layers that read the same x (one
// layer, or e.g. the q, k and v projections): their row tiles are numbered one
// after the other, layer l owning tiles [tile0, tile0 + its tiles).
struct TcLayer {
    const uint4 *codebooks;
    const __half *scales;
    __half *y;
    int d_out;
    int tile0;
};

template <int NL>
struct TcArgs {
    TcLayer layer[NL];
    int n_layers;
    float *partial;      // [tiles][max_segs][T][128] partial sums of split tiles
    uint32_t *counters;  // [tiles], zero between calls
    int32_t *status;     // AQLM_ERR_TIMEOUT after a wait gave up
    int G, T;
    int n_stages;        // stages of 64 inputs per row
    int max_segs;        // segments of one tile, at most
    long long units;     // row tiles (all layers) x n_stages
};

// The code tensor maps of a launch's layers (layer l in m[l]).
template <int NL>
struct TcCodeMaps {
    CUtensorMap m[NL];
};

// The layer of global row tile `tile` (static indices only, so the
// descriptors stay in the kernel's parameter space).
template <int NL>
__device__ __forceinline__ int layer_of(int tile, const TcArgs<NL> &a) {
    int l = 0;
#pragma unroll
    for (int i = 1; i < NL; ++i)
        if (i < a.n_layers && tile >= a.layer[i].tile0) l = i;
    return l;
}
template <int NL>
__device__ __forceinline__ TcLayer layer_at(int l, const TcArgs<NL> &a) {
    TcLayer L = a.layer[0];
#pragma unroll
    for (int i = 1; i < NL; ++i)
        if (i == l) L = a.layer[i];
    return L;
}

// CTA c works on units [unit_start(c), unit_start(c + 1)).
template <typename A>
__device__ __forceinline__ long long unit_start(int c, const A &a) {
    return (long long)c * a.units / (long long)gridDim.x;
}
// The CTA whose range holds unit u.
template <typename A>
__device__ int cta_of_unit(long long u, const A &a) {
    int c = (int)(u * (long long)gridDim.x / a.units);
    while (c + 1 < (int)gridDim.x && unit_start(c + 1, a) <= u) ++c;
    while (c > 0 && unit_start(c, a) > u) --c;
    return c;
}
struct Seg {
    int tile, k0, len;  // stages [k0, k0 + len) of row tile `tile`
};
template <typename A>
__device__ __forceinline__ Seg seg_at(long long u, long long u_end, const A &a) {
    Seg g;
    g.tile = (int)(u / a.n_stages);
    g.k0 = (int)(u - (long long)g.tile * a.n_stages);
    const long long left = u_end - u;
    g.len = (int)min((long long)(a.n_stages - g.k0), left);
    return g;
}

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
// 16-byte asynchronous global -> shared copy with an L2 cache policy;
// src_bytes = 0 writes zeros.  kL1: through L1 (.ca) for the 8 KiB of 2x8
// codebooks, which L1 holds; otherwise L2 only (.cg) for the 1-2 MiB
// 1x16 / 2x16 codebooks, whose random codewords L1 cannot hold.  Measured on
// B200: .cg instead of .ca made 1x16 8192x8192 with 4 tokens 46.9 -> 41.6 us
// and 28672x8192 with 16 tokens 149.6 -> 130.8 us, while 2x8 through L2 only
// was 9x slower.
template <bool kL1>
__device__ __forceinline__ void cp_async16_keep(uint32_t dst, const void *src, uint32_t src_bytes, uint64_t pol) {
    if constexpr (kL1) {
        asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst), "l"(src),
                     "r"(src_bytes), "l"(pol)
                     : "memory");
    } else {
        asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst), "l"(src),
                     "r"(src_bytes), "l"(pol)
                     : "memory");
    }
}
// Arrive on an mbarrier once all of this thread's earlier cp.async copies have
// completed (the arrival is part of the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

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

template <int M, int B, int NL>
__global__ void __launch_bounds__(kTcThreads, TcFmt<M, B>::kCtasPerSm)
    gemv_tc_kernel(const __grid_constant__ TcCodeMaps<NL> maps, const __grid_constant__ CUtensorMap tmap_x,
                   const TcArgs<NL> a) {
    using F = TcFmt<M, B>;
    constexpr int kCodeVecs = F::kStageCodeBytes / 16;  // 16-byte code pieces per row per stage
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = saddr(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw & 1023)) & 1023);
    uint8_t *ring = smem;                                                       // [stage][M A tiles | B tile]
    uint8_t *codes_s = ring + (size_t)F::kStages * F::kStageBytes;              // [slot][128 rows][64 B]
    TcBars *bars = reinterpret_cast<TcBars *>(codes_s + (size_t)kCodeSlots * kTcRows * kCodeBoxBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long u_begin = unit_start(blockIdx.x, a), u_end = unit_start(blockIdx.x + 1, a);
    constexpr int SPB = F::kStagesPerBox;

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
#pragma unroll
        for (int l = 0; l < NL; ++l)
            if (l < a.n_layers)
                asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.m[l])) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
    }
    if (threadIdx.x == 32) {  // this CTA's share of each layer's (usually cold) codebooks into L2
        const uint32_t cb_bytes = (uint32_t)M * F::K * 16;
        const uint32_t share = ((cb_bytes + gridDim.x - 1) / gridDim.x + 255) & ~255u;
        const uint32_t off = blockIdx.x * share;
#pragma unroll
        for (int l = 0; l < NL; ++l)
            if (l < a.n_layers && off < cb_bytes)
                prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(layer_at(l, a).codebooks) + off,
                                 min(share, cb_bytes - off), policy_evict_last());
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
            int stage_issued[F::kStages];
            for (int s = 0; s < F::kStages; ++s) stage_issued[s] = -1;
            int slot_last[kCodeSlots] = {0, 0};  // global index of the last stage of the box in each slot
            bool ok = true;
            // box cursor: box bj of the segment starting at unit bu (global stage index bgi)
            long long bu = u_begin;
            int bj = 0, bgi = 0, gb = 0;
            auto issue_box = [&]() -> bool {
                const Seg g = seg_at(bu, u_end, a);
                const int slot = gb % kCodeSlots;
                const uint32_t par = (uint32_t)((gb / kCodeSlots) & 1);
                if (!tc_wait(saddr(&bars->code_empty[slot]), par ^ 1, bars, a.status)) return false;
                const uint32_t full = saddr(&bars->code_full[slot]);
                const int ly = layer_of(g.tile, a);
                const CUtensorMap *map = &maps.m[0];
#pragma unroll
                for (int i = 1; i < NL; ++i)
                    if (i == ly) map = &maps.m[i];
                mbar_expect_tx(full, kTcRows * kCodeBoxBytes);
                tma_load_2d(saddr(codes_s + (size_t)slot * kTcRows * kCodeBoxBytes), map,
                            (g.k0 + bj * SPB) * F::kStageCodeBytes, (g.tile - layer_at(ly, a).tile0) * kTcRows, full);
                code_issued[slot] = (int)par;
                slot_last[slot] = bgi + min(g.len, (bj + 1) * SPB) - 1;
                ++gb;
                if (++bj * SPB >= g.len) {  // next segment
                    bu += g.len;
                    bgi += g.len;
                    bj = 0;
                }
                return true;
            };
            while (bu < u_end && gb < kCodeSlots && ok) ok = issue_box();
            grid_dep_wait();
            int gi = 0;
            for (long long u = u_begin; u < u_end && ok;) {
                const Seg g = seg_at(u, u_end, a);
                for (int l = 0; l < g.len && ok; ++l, ++gi) {
                    const int s = gi % F::kStages;
                    const uint32_t par = (uint32_t)((gi / F::kStages) & 1);
                    if (!tc_wait(saddr(&bars->empty[s]), par ^ 1, bars, a.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = saddr(&bars->full[s]);
                    mbar_expect_tx(full, kXBytes);
                    tma_load_2d(saddr(ring + (size_t)s * F::kStageBytes + (size_t)M * kTileBytes), &tmap_x,
                                (g.k0 + l) * kStageK, 0, full);
                    stage_issued[s] = (int)par;
                    // box gb takes the slot of box gb - 2, which the decoders release when
                    // they store that box's last stage: issue it once the activations of
                    // that stage are on their way (the decoders and the MMAs can always
                    // get that far), well ahead of its use
                    while (ok && bu < u_end && slot_last[gb % kCodeSlots] <= gi) ok = issue_box();
                }
                u += g.len;
            }
            while (ok && bu < u_end) ok = issue_box();
            // no copy may still be landing in shared memory when the CTA exits
            for (int s = 0; s < kCodeSlots; ++s)
                if (code_issued[s] >= 0) tc_drain(saddr(&bars->code_full[s]), (uint32_t)code_issued[s]);
            for (int s = 0; s < F::kStages; ++s)
                if (stage_issued[s] >= 0) tc_drain(saddr(&bars->full[s]), (uint32_t)stage_issued[s]);
        }
        __syncwarp();
    } else if (warp == 5) {
        if (lane == 0) {
            // ---- MMA issuer: one accumulator per segment, released by the epilogue ----
            bool ok = true;
            int gi = 0;
            for (long long u = u_begin; u < u_end && ok;) {
                const Seg g = seg_at(u, u_end, a);
                for (int l = 0; l < g.len; ++l, ++gi) {
                    const int s = gi % F::kStages;
                    const uint32_t par = (uint32_t)((gi / F::kStages) & 1);
                    if (!tc_wait(saddr(&bars->full[s]), par, bars, a.status)) {
                        ok = false;
                        break;
                    }
                    // the A tiles were written by cp.async (generic proxy): order them
                    // before the tensor cores' (async proxy) reads
                    fence_async_smem();
                    tc_fence_after();
                    const uint32_t a0 = saddr(ring + (size_t)s * F::kStageBytes);
                    const uint32_t b0 = a0 + (uint32_t)(M * kTileBytes);
#pragma unroll
                    for (int k = 0; k < kStageK / 16; ++k) {
#pragma unroll
                        for (int m = 0; m < M; ++m)
                            mma_f16(tmem, sw128_desc(a0 + (uint32_t)(m * kTileBytes) + 32 * k),
                                    sw128_desc(b0 + 32 * k), (l > 0 || k > 0 || m > 0) ? 1u : 0u);
                    }
                    mma_commit(saddr(&bars->empty[s]));
                }
                if (ok) mma_commit(saddr(&bars->acc_full));
                u += g.len;
            }
            // tensor memory is freed only after every issued MMA completed
            mma_commit(saddr(&bars->mma_done));
            tc_drain(saddr(&bars->mma_done), 0);
        }
        __syncwarp();
    } else {
        // ---- decoders (thread = row of the tile), then each segment's epilogue ----
        const int r = warp * 32 + lane;
        const uint64_t keep = policy_evict_last();
        bool ok = true;
        int gi0 = 0, gb0 = 0, j = 0;  // global stage and box index of the segment's start, segment count
        bool waited_grid = false;
        for (long long u = u_begin; u < u_end && ok; ++j) {
            const Seg g = seg_at(u, u_end, a);
            const TcLayer L = layer_at(layer_of(g.tile, a), a);
            const int row = (g.tile - L.tile0) * kTcRows + r;
            for (int l = 0; l < g.len; ++l) {
                // the row's codes of local stage l, from its box
                const int gbox = gb0 + l / SPB, slot = gbox % kCodeSlots;
                if (l % SPB == 0 &&
                    !tc_wait(saddr(&bars->code_full[slot]), (uint32_t)((gbox / kCodeSlots) & 1), bars, a.status)) {
                    ok = false;
                    break;
                }
                // the code tile arrives in the 64-byte swizzle: 16-byte piece c of row r
                // sits at piece c ^ ((r >> 1) & 3), so the 8 rows of a quarter warp read
                // 8 different bank quads (unswizzled, rows 64 bytes apart hit only
                // quads 0 and 4: four-way conflicts)
                uint4 code[kCodeVecs];
                const uint8_t *rowp = codes_s + (size_t)slot * kTcRows * kCodeBoxBytes + (size_t)r * kCodeBoxBytes;
#pragma unroll
                for (int v = 0; v < kCodeVecs; ++v) {
                    const int piece = (l % SPB) * kCodeVecs + v;
                    code[v] = AQLM_IN_BOUNDS(piece < kCodeBoxBytes / 16, kSiteTcCodes, piece)
                                  ? *reinterpret_cast<const uint4 *>(rowp + ((piece ^ ((r >> 1) & 3)) << 4))
                                  : make_uint4(0, 0, 0, 0);
                }
                // the stage's A tiles are free once the MMAs of its previous use are done
                const int gi = gi0 + l, s = gi % F::kStages;
                if (!tc_wait(saddr(&bars->empty[s]), (uint32_t)(((gi / F::kStages) & 1) ^ 1), bars, a.status)) {
                    ok = false;
                    break;
                }
                // codewords copied straight from the codebooks into the swizzled A
                // tiles (zeros past the row end); the stage's full barrier counts
                // this thread's arrival when all of its copies have landed
                const int grp0 = (g.k0 + l) * kStageGroups;
                const uint32_t tile = saddr(ring + (size_t)s * F::kStageBytes + (size_t)r * 128);
#pragma unroll
                for (int q = 0; q < kStageGroups; ++q) {
                    const uint32_t bytes = (grp0 + q < a.G) ? 16u : 0u;
#pragma unroll
                    for (int m = 0; m < M; ++m) {
                        const uint32_t k = tc_index<M, B, kCodeVecs>(code, q, m);
                        const bool in = AQLM_IN_BOUNDS(k < (uint32_t)F::K && r * 128 + 128 <= kTileBytes, kSiteTcA, r);
                        cp_async16_keep<B == 8>(tile + (uint32_t)(m * kTileBytes) + (uint32_t)((q ^ (r & 7)) << 4),
                                                L.codebooks + (size_t)m * F::K + (in ? k : 0u), in ? bytes : 0u, keep);
                    }
                }
                cp_async_arrive_noinc(saddr(&bars->full[s]));
                // the box's codes were read into registers and used above: its slot
                // may be refilled once the last stage of the box is issued
                if (l % SPB == SPB - 1 || l == g.len - 1) {
                    fence_async_smem();
                    mbar_arrive(saddr(&bars->code_empty[slot]));
                }
            }

            // ---- the segment's epilogue ----
            if (!waited_grid) {
                grid_dep_wait();
                waited_grid = true;
            }
            ok = ok && tc_wait(saddr(&bars->acc_full), (uint32_t)(j & 1), bars, a.status);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t v[16];
            tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), v);
            tc_fence_before();  // the next segment's MMAs overwrite the accumulator
            if (g.len == a.n_stages) {
                if (row < L.d_out) {
                    const float sc = __half2float(L.scales[row]);
                    for (int t = 0; t < a.T; ++t)
                        if (AQLM_IN_BOUNDS(row < L.d_out, kSiteTcY, row))
                            L.y[(size_t)t * L.d_out + row] = __float2half_rn(__uint_as_float(v[t]) * sc);
                }
            } else {
                const long long t_u0 = (long long)g.tile * a.n_stages;
                const int c_lo = cta_of_unit(t_u0, a);
                const int n_seg = cta_of_unit(t_u0 + a.n_stages - 1, a) - c_lo + 1;
                float *part = a.partial + (size_t)g.tile * a.max_segs * a.T * kTcRows;
                if (AQLM_IN_BOUNDS((int)blockIdx.x - c_lo < a.max_segs && n_seg <= a.max_segs, kSiteTcPartial,
                                   (int)blockIdx.x - c_lo))
                    for (int t = 0; t < a.T; ++t)
                        part[((size_t)(blockIdx.x - c_lo) * a.T + t) * kTcRows + r] = __uint_as_float(v[t]);
                __threadfence();
                asm volatile("bar.sync 1, %0;" ::"n"(kDecoders) : "memory");
                if (threadIdx.x == 0)
                    bars->last = (atomicAdd(&a.counters[g.tile], 1u) == (uint32_t)(n_seg - 1));
                asm volatile("bar.sync 1, %0;" ::"n"(kDecoders) : "memory");
                if (bars->last) {  // the last segment of the tile: add all of them in input order
                    __threadfence();
                    if (row < L.d_out) {
                        const float sc = __half2float(L.scales[row]);
                        // segment by segment, every token's partial at once (up to 16
                        // loads in flight); each token's sum still runs in segment order
                        float sum[kTcN];
#pragma unroll
                        for (int t = 0; t < kTcN; ++t) sum[t] = 0.f;
                        for (int sg = 0; sg < n_seg; ++sg) {
                            float pv[kTcN];
#pragma unroll
                            for (int t = 0; t < kTcN; ++t)
                                pv[t] = t < a.T ? __ldcg(&part[((size_t)sg * a.T + t) * kTcRows + r]) : 0.f;
#pragma unroll
                            for (int t = 0; t < kTcN; ++t) sum[t] += pv[t];
                        }
#pragma unroll
                        for (int t = 0; t < kTcN; ++t)
                            if (t < a.T && AQLM_IN_BOUNDS(row < L.d_out, kSiteTcY, row))
                                L.y[(size_t)t * L.d_out + row] = __float2half_rn(sum[t] * sc);
                    }
                    if (threadIdx.x == 0) a.counters[g.tile] = 0u;
                }
                asm volatile("bar.sync 1, %0;" ::"n"(kDecoders) : "memory");  // bars->last is reused
            }
            u += g.len;
            gi0 += g.len;
            gb0 += (g.len + SPB - 1) / SPB;
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
    int ctas;           // persistent CTAs, two per SM at most
    int tiles;          // row tiles of 128
    int n_stages;       // stages of 64 inputs per row
    long long units;    // tiles x n_stages
    int max_segs;       // segments of one tile, at most
};

// Stream-K plan over `tiles` row tiles (all layers): as many CTAs as are
// resident at once (two per SM), each with an equal contiguous range of at
// least 8 stage units (fewer CTAs for small layers).
TcPlan plan_tc(const Dims &d, long long tiles, int sms) {
    TcPlan p;
    const int per_sm = (d.M == 1) ? TcFmt<1, 16>::kCtasPerSm : TcFmt<2, 16>::kCtasPerSm;
    p.tiles = (int)tiles;
    p.n_stages = (d.G + kStageGroups - 1) / kStageGroups;
    p.units = (long long)p.tiles * p.n_stages;
    constexpr long long kMinUnits = 8;
    long long ctas = (long long)per_sm * sms;
    if (ctas > p.units / kMinUnits) ctas = p.units / kMinUnits;
    if (ctas < 1) ctas = 1;
    p.ctas = (int)ctas;
    // a tile's units meet at most floor(n / units-per-CTA) + 2 CTA ranges
    const long long upc = p.units / ctas;
    long long segs = p.n_stages / upc + 2;
    if (segs > ctas) segs = ctas;
    p.max_segs = (int)segs;
    return p;
}

long long tiles_of(const RowLayerIn *layers, int n) {
    long long t = 0;
    for (int l = 0; l < n; ++l) t += (layers[l].d_out + kTcRows - 1) / kTcRows;
    return t;
}

inline size_t al16(size_t v) { return (v + 15) / 16 * 16; }

// Workspace: [fp32 partials of split tiles][arrival counters][status word],
// the last two zero before a call.
size_t tc_counter_offset(const TcPlan &p, int T) {
    return al16((size_t)p.tiles * p.max_segs * T * kTcRows * sizeof(float));
}
size_t tc_workspace_bytes(const TcPlan &p, int T) {
    return tc_counter_offset(p, T) + al16((size_t)p.tiles * sizeof(uint32_t)) + 16;
}

template <int M, int B, int NL>
cudaError_t launch_tc(const TcCodeMaps<NL> &mc, const CUtensorMap &mx, const TcArgs<NL> &a, const TcPlan &p,
                      cudaStream_t st) {
    auto fn = gemv_tc_kernel<M, B, NL>;
    const cudaError_t e = opt_in_dynamic_smem(fn, TcFmt<M, B>::kSmem);
    if (e != cudaSuccess) return e;
    return launch_kernel(fn, dim3(p.ctas), dim3(kTcThreads), TcFmt<M, B>::kSmem, st, true, mc, mx, a);
}

template <int NL>
cudaError_t launch_tc_layers(const RowLayerIn *layers, int n, const uint16_t *x, int tokens, const Dims &d,
                             void *workspace, int sms, cudaStream_t st) {
    const TcPlan p = plan_tc(d, tiles_of(layers, n), sms);
    TcCodeMaps<NL> mc;
    CUtensorMap mx;
    TcArgs<NL> a = {};
    int tile0 = 0;
    for (int l = 0; l < n; ++l) {
        if (!encode_2d(&mc.m[l], CU_TENSOR_MAP_DATA_TYPE_UINT8, layers[l].codes, (uint64_t)d.row_bytes,
                       (uint64_t)layers[l].d_out, (uint64_t)d.row_bytes, kCodeBoxBytes, kTcRows,
                       CU_TENSOR_MAP_SWIZZLE_64B))
            return cudaErrorInvalidValue;
        TcLayer &L = a.layer[l];
        L.codebooks = reinterpret_cast<const uint4 *>(layers[l].codebooks);
        L.scales = reinterpret_cast<const __half *>(layers[l].scales);
        L.y = reinterpret_cast<__half *>(layers[l].y);
        L.d_out = layers[l].d_out;
        L.tile0 = tile0;
        tile0 += (layers[l].d_out + kTcRows - 1) / kTcRows;
    }
    for (int l = n; l < NL; ++l) mc.m[l] = mc.m[0];
    if (!encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, (uint64_t)d.d_in, (uint64_t)tokens, (uint64_t)d.d_in * 2,
                   kStageK, kTcN, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    a.n_layers = n;
    a.partial = reinterpret_cast<float *>(ws);
    a.counters = reinterpret_cast<uint32_t *>(ws + tc_counter_offset(p, tokens));
    a.status = reinterpret_cast<int32_t *>(ws + tc_workspace_bytes(p, tokens) - 16);
    a.G = d.G;
    a.T = tokens;
    a.n_stages = p.n_stages;
    a.max_segs = p.max_segs;
    a.units = p.units;
    if (d.M == 1) return launch_tc<1, 16, NL>(mc, mx, a, p, st);
    if (d.B == 8) return launch_tc<2, 8, NL>(mc, mx, a, p, st);
    return launch_tc<2, 16, NL>(mc, mx, a, p, st);
}

constexpr int kTcMaxLayers = AQLM_MULTI_MAX_LAYERS;

}  // namespace

// Any token count works (the MMA's N is 16 whatever T is); gemv.cu sends this
// kernel the counts past the row kernel's.
bool gemv_tc_supported(const Dims &d, int T) {
    (void)d;
    return T >= 1 && T <= AQLM_GEMV_MAX_TOKENS;
}

size_t gemv_tc_multi_counter_offset(const RowLayerIn *layers, int n, const Dims &d, int T, int sms) {
    return tc_counter_offset(plan_tc(d, tiles_of(layers, n), sms), T);
}
size_t gemv_tc_multi_workspace_bytes(const RowLayerIn *layers, int n, const Dims &d, int T, int sms) {
    return tc_workspace_bytes(plan_tc(d, tiles_of(layers, n), sms), T);
}
size_t gemv_tc_multi_status_offset(const RowLayerIn *layers, int n, const Dims &d, int T, int sms) {
    return gemv_tc_multi_workspace_bytes(layers, n, d, T, sms) - 16;
}

cudaError_t launch_gemv_tc_multi(const RowLayerIn *layers, int n, const uint16_t *x, int tokens, const Dims &d,
                                 void *workspace, int sms, cudaStream_t st) {
    if (n < 1 || n > kTcMaxLayers) return cudaErrorInvalidValue;
    if (n == 1) return launch_tc_layers<1>(layers, n, x, tokens, d, workspace, sms, st);
    return launch_tc_layers<kTcMaxLayers>(layers, n, x, tokens, d, workspace, sms, st);
}

// single layer: the same layout with one layer
size_t gemv_tc_counter_offset(const Dims &d, int T, int sms) {
    const RowLayerIn one = {nullptr, nullptr, nullptr, nullptr, d.d_out};
    return gemv_tc_multi_counter_offset(&one, 1, d, T, sms);
}
size_t gemv_tc_workspace_bytes(const Dims &d, int T, int sms) {
    const RowLayerIn one = {nullptr, nullptr, nullptr, nullptr, d.d_out};
    return gemv_tc_multi_workspace_bytes(&one, 1, d, T, sms);
}
size_t gemv_tc_status_offset(const Dims &d, int T, int sms) { return gemv_tc_workspace_bytes(d, T, sms) - 16; }

cudaError_t launch_gemv_tc(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                           uint16_t *y, int tokens, const Dims &d, void *workspace, int sms, cudaStream_t st) {
    const RowLayerIn one = {codes, codebooks, scales, y, d.d_out};
    return launch_gemv_tc_multi(&one, 1, x, tokens, d, workspace, sms, st);
}

AQLM_DEFINE_BOUNDS_READER(bounds_word_tc)

}  // namespace aqlm
