// gemm_tcgen05.cu -- dense prefill GEMM on the 5th-generation tensor cores.
//
// Y[m][n] = sum_k X[m][k] * W[n][k]: X = the prefill activations [tokens][d_in]
// and W = the dequantised layer [d_out][d_in], both bf16 and K-major; fp32
// accumulation; bf16 output rounded to nearest even.  This is the product of
// the activations with the dequantised weights in their native precision,
// section "What is Multi-Codebook Quantization (MCQ)?" of "The AQLM
// Quantization Algorithm, Explained".
//
// sm_100a design: a persistent kernel, one CTA per SM, 128 x BN output tiles.
//   warp 0      one thread issues TMA tile loads (128-byte swizzle) into a
//               shared-memory ring (4 stages, 5 for BN = 192),
//               each stage guarded by a pair of mbarriers (full: bytes
//               landed; empty: MMAs done reading);
//   warp 1      allocates the tensor memory of two 128 x BN fp32
//               accumulators and one thread issues tcgen05.mma
//               (cta_group::1, kind::f16, M=128 N=BN K=16), releasing each
//               ring stage with tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld from the accumulator of the previous
//               tile while the MMAs of the next tile run into the other one,
//               bf16 conversion, 16-byte global stores.
// Every mbarrier wait is bounded in time.  A wait that gives up writes
// AQLM_ERR_TIMEOUT to the status word, raises a CTA-wide abort flag that the
// other roles poll, waits (bounded) for its TMA loads and MMAs in flight and
// frees its tensor memory before returning; nothing traps.
//
// The tile width BN is chosen per shape from {256, 240, 224, 192} so that the
// tiles fill the waves of the SMs: with 2048 tokens, 11008 output columns are
// 688 tiles of 128x256 (4.65 waves of 148 SMs, the last one 65% full) but 736
// of 128x240 (4.97 waves).  A tile's time goes with the operand bytes it
// streams, (128 + BN) x K (the ring is fed from L2 at close to its bandwidth),
// so the estimate is waves x (128 + BN); measured on B200 it ranks the widths
// as the clock does (2048 tokens: 11008x4096 141.3 / 135.2 us at BN 256 / 240,
// 4096x11008 141.2 / 137.2, 8192x8192 204.8 / 200.7 / 196.6 at 256 / 240 / 224).
// Narrower tiles lose: 128x112 ran at 60% of the 128x256 rate.
#include <cuda.h>

#include "common.cuh"

namespace aqlm {
namespace {

constexpr int BM = 128, BK = 64;
constexpr int A_BYTES = BM * BK * 2;
constexpr int kMaxStages = 8;
constexpr int kGemmThreads = 192;
constexpr int kEpiWarps = 4;

struct Bars {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

// RESERVE: shared memory the fused decoders keep for their codebook copies.
template <int BN, int RESERVE = 0>
struct GemmCfg {
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M = 128");
    static constexpr int B_BYTES = BN * BK * 2;                // a multiple of 1024: stages stay aligned
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    // the ring gets 200 KiB; a fused kernel with codebook copies 220 KiB less the copies
    static constexpr int BUDGET = RESERVE ? 220 * 1024 - RESERVE : 200 * 1024;
    static constexpr int STAGES = BUDGET / STAGE_BYTES < kMaxStages ? BUDGET / STAGE_BYTES : kMaxStages;
    // each accumulator at a power-of-two column offset; the allocation is a power of two
    static constexpr int ACC_STRIDE = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
    static constexpr uint32_t TMEM_COLS = 2 * ACC_STRIDE;
    // bf16 x bf16 -> fp32, both operands K-major, M = 128, N = BN (tcgen05
    // instruction descriptor: D format bits 4-5, A/B format bits 7-12, N >> 3
    // at bits 17-22, M >> 4 at bits 24-28).
    static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                      ((uint32_t)(BM >> 4) << 24);
    static constexpr size_t SMEM = 1024 /*alignment slack*/ + (size_t)STAGES * STAGE_BYTES + sizeof(Bars) + 16 + RESERVE;
    static_assert(B_BYTES % 1024 == 0 && STAGES >= 2, "ring layout");
};

// ---- fused dequantisation: the B tiles decoded in shared memory -------------
// With FM > 0 (the codebook count of the layer, FB its code bits) the kernel
// reads no W^: eight more warps decode each stage's B tile -- BN rows of W^ x
// 64 inputs -- from the codes, codebooks and scales, with the binary32 steps
// of aqlm_dequant (codewords added in codebook order, times the row's scale,
// rounded to bf16), straight into the 128-byte-swizzled K-major layout the
// MMA reads, then order their stores before the tensor cores' reads (proxy
// fence) and arrive on the stage's full barrier, which the X tile's TMA bytes
// complete.  Every CTA decodes the W^ rows of its own tiles; a row block is
// decoded once per 128-token tile that uses it, and nothing is written to or
// read from a W^ buffer in global memory.
constexpr int kDecWarps = 8;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kCbCopies = 8;   // 2x8: the codebooks in shared memory, copy p in bank quad p

struct DecodeArgs {
    const uint8_t *codes;      // [d_out][G][M]
    const uint4 *codebooks;    // [M][2^B] codewords of 8 fp16
    const __half *scales;      // [d_out]
    int G, row_bytes;
};

template <int FM, int FB>
constexpr int decode_reserve() {
    return (FM > 0 && FB == 8) ? FM * 256 * 16 * kCbCopies : 0;
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
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

// Wait for the phase of `parity` to complete, for at most `limit_ns`.  On a
// timeout record the status and raise the abort flag; give up early when
// another role raised it.
__device__ bool wait_bounded(uint32_t bar, uint32_t parity, Bars *bars, int32_t *status, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 0) {
            if (*reinterpret_cast<volatile int *>(&bars->abort_flag)) return false;
            if (now_ns() - t0 > limit_ns) {
                *reinterpret_cast<volatile int *>(&bars->abort_flag) = 1;
                atomicExch(status, (int32_t)AQLM_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address, 16-byte units
    d |= (uint64_t)1 << 16;                    // leading byte offset (unused for this layout)
    d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                    // descriptor version of sm_100
    d |= (uint64_t)2 << 61;                    // 128-byte swizzle
    return d;
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Columns [n0, n0 + 8 * V) of row m of Y from fp32 accumulator values r,
// rounded to bf16, in 16-byte stores (columns past n_total skipped; n_total
// is a multiple of 8).
template <int V>
__device__ __forceinline__ void store_bf16_row(__nv_bfloat16 *dst, const uint32_t *r, int n0, int n_total) {
#pragma unroll
    for (int v = 0; v < V; ++v) {
        if (n0 + 8 * v < n_total) {
            uint32_t p[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const __nv_bfloat162 b2 =
                    __floats2bfloat162_rn(__uint_as_float(r[8 * v + 2 * h]), __uint_as_float(r[8 * v + 2 * h + 1]));
                p[h] = *reinterpret_cast<const uint32_t *>(&b2);
            }
            *reinterpret_cast<uint4 *>(dst + 8 * v) = make_uint4(p[0], p[1], p[2], p[3]);
        }
    }
}

// Code index of codebook m of group q (0..7) of a stage from a row's code bytes.
template <int FM, int FB, int V>
__device__ __forceinline__ uint32_t stage_code(const uint4 (&c)[V], int q, int m) {
    if constexpr (FM == 1) {
        const uint32_t w[4] = {c[0].x, c[0].y, c[0].z, c[0].w};
        return (w[q >> 1] >> (16 * (q & 1))) & 0xffffu;
    } else if constexpr (FB == 8) {  // byte 0 codebook 0, byte 1 codebook 1
        const uint32_t w[4] = {c[0].x, c[0].y, c[0].z, c[0].w};
        return (w[q >> 1] >> (16 * (q & 1) + 8 * m)) & 0xffu;
    } else {  // 2x16: 4 bytes per group, codebook 0 in the low half
        const uint32_t w[8] = {c[0].x, c[0].y, c[0].z, c[0].w, c[V - 1].x, c[V - 1].y, c[V - 1].z, c[V - 1].w};
        return (w[q] >> (16 * m)) & 0xffffu;
    }
}

template <int BN, int FM, int FB>
__global__ void __launch_bounds__(kGemmThreads + (FM > 0 ? kDecThreads : 0), 1)
gemm_bf16_tcgen05(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  __nv_bfloat16 *__restrict__ Y, int m_total, int n_total, int k_total, int32_t *status,
                  unsigned long long limit_ns, int stall_test, const DecodeArgs da) {
    constexpr int RESERVE = decode_reserve<FM, FB>();
    using C = GemmCfg<BN, RESERVE>;
    constexpr int STAGES = C::STAGES, STAGE_BYTES = C::STAGE_BYTES;
    constexpr bool kFused = FM > 0;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled tiles.
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw & 1023)) & 1023);
    Bars *bars = reinterpret_cast<Bars *>(smem + (size_t)STAGES * STAGE_BYTES);
    uint4 *cbs = reinterpret_cast<uint4 *>(smem + (size_t)STAGES * STAGE_BYTES + ((sizeof(Bars) + 15) & ~size_t(15)));
    if constexpr (kFused && FB == 8) {  // 2x8 codebooks: kCbCopies copies, codeword e of copy p at word 8e + p
        for (int i = threadIdx.x; i < FM * 256 * kCbCopies; i += blockDim.x) cbs[i] = da.codebooks[i >> 3];
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m_tiles = (m_total + BM - 1) / BM;
    const int n_tiles = (n_total + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;
    const int num_kb = (k_total + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // full: the X tile's TMA (one arrival with its bytes) and, fused, each decoder warp
            mbar_init(smem_addr(&bars->full[s]), kFused ? 1 + kDecWarps : 1);
            mbar_init(smem_addr(&bars->empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_addr(&bars->tfull[a]), 1);
            mbar_init(smem_addr(&bars->tempty[a]), kEpiWarps);
        }
        mbar_init(smem_addr(&bars->mma_done), 1);
        bars->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&bars->tmem_base)),
                     "r"(C::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;

    if (warp == 0) {
        if (lane == 0 && !stall_test) {
            // ---- TMA producer ----
            grid_dep_wait();   // launched early after the kernel writing W (a no-op otherwise)
            int stage = 0;
            uint32_t phase = 0;
            int issued_parity[STAGES];
            for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int mb = tile % m_tiles, nb = tile / m_tiles;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!wait_bounded(smem_addr(&bars->empty[stage]), phase ^ 1, bars, status, limit_ns)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full = smem_addr(&bars->full[stage]);
                    const uint32_t dst = smem_addr(smem + (size_t)stage * STAGE_BYTES);
                    mbar_expect_tx(full, (uint32_t)(kFused ? A_BYTES : STAGE_BYTES));
                    tma_load_2d(dst, &tmap_x, kb * BK, mb * BM, full);
                    if constexpr (!kFused) tma_load_2d(dst + A_BYTES, &tmap_w, kb * BK, nb * BN, full);
                    issued_parity[stage] = (int)phase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // No copy may still be landing in shared memory when the CTA exits.
            for (int s = 0; s < STAGES; ++s) {
                if (issued_parity[s] >= 0) {
                    const uint32_t full = smem_addr(&bars->full[s]);
                    const uint64_t t0 = now_ns();
                    while (!mbar_try_wait(full, (uint32_t)issued_parity[s]) && now_ns() - t0 < limit_ns) {
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer ----
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!wait_bounded(smem_addr(&bars->tempty[acc]), acc_phase ^ 1, bars, status, limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * C::ACC_STRIDE);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!wait_bounded(smem_addr(&bars->full[stage]), phase, bars, status, limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_addr(smem + (size_t)stage * STAGE_BYTES);
                    const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        // K step of 16 bf16 = 32 bytes inside the 128-byte swizzled row.
                        mma_bf16(d_tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), C::IDESC,
                                 (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit(smem_addr(&bars->empty[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                mma_commit(smem_addr(&bars->tfull[acc]));
                if (++acc == 2) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            // Tensor memory is freed below only after every issued MMA completed.
            mma_commit(smem_addr(&bars->mma_done));
            const uint64_t t0 = now_ns();
            while (!mbar_try_wait(smem_addr(&bars->mma_done), 0) && now_ns() - t0 < limit_ns) {
            }
        }
        __syncwarp();
    } else if (kFused && warp >= 2 + kEpiWarps) {
        // ---- decoders (fused): thread dt owns row dt of every B tile ----
        // (FM = 0, the plain GEMM, never runs this branch; the constants stay valid for it)
        constexpr int kCodeVecs = FM * FB >= 16 ? (FM * FB) / 16 : 1;        // 16-byte code pieces per row and stage
        constexpr int kGroupsPerVec = FM * FB > 0 ? 16 * 8 / (FM * FB) : 8;  // groups per 16-byte piece
        constexpr int kCodeDepth = 4;                                          // stages of codes held ahead
        const int dt = threadIdx.x - kGemmThreads;
        const int copy = lane & (kCbCopies - 1);
        const uint64_t keep = policy_evict_last();
        const uint64_t stream_pol = policy_evict_first();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            const int nb = tile / m_tiles;
            const int n = nb * BN + dt;
            const bool mine = dt < BN;                   // a row of the tile
            const bool live = mine && n < n_total;       // a row of W^ (past it: zeros)
            const float s = live ? __half2float(da.scales[n]) : 0.f;
            const uint8_t *crow = da.codes + (size_t)(live ? n : 0) * da.row_bytes;
            auto load_codes = [&](int kb, uint4 (&c)[kCodeVecs]) {
#pragma unroll
                for (int v = 0; v < kCodeVecs; ++v) {
                    c[v] = make_uint4(0, 0, 0, 0);
                    if (live && kb < num_kb && kb * 8 + v * kGroupsPerVec < da.G)
                        c[v] = ld_stream_u4(crow + (size_t)kb * 8 * (FM * FB / 8) + 16 * v, stream_pol);
                }
            };
            // the row's codes of the tile: an L2 prefetch of all of them (each 128-byte
            // line once), then register copies kCodeDepth stages ahead of their use
            if (live) {
                const size_t row_code_bytes = (size_t)da.G * (FM * FB / 8);
                for (size_t off = 0; off < row_code_bytes; off += 128)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(crow + off));
            }
            uint4 ring[kCodeDepth][kCodeVecs];
#pragma unroll
            for (int u = 0; u < kCodeDepth; ++u) load_codes(u, ring[u]);
            for (int kb0 = 0; kb0 < num_kb && ok; kb0 += kCodeDepth) {
#pragma unroll
                for (int u = 0; u < kCodeDepth; ++u) {
                    const int kb = kb0 + u;
                    if (kb >= num_kb) break;
                    uint4 code[kCodeVecs];
#pragma unroll
                    for (int v = 0; v < kCodeVecs; ++v) code[v] = ring[u][v];
                    load_codes(kb + kCodeDepth, ring[u]);
                    bool w = true;
                    if (lane == 0)
                        w = wait_bounded(smem_addr(&bars->empty[stage]), phase ^ 1, bars, status, limit_ns);
                    if (!__shfl_sync(0xffffffffu, (int)w, 0)) {
                        ok = false;
                        break;
                    }
                    if (mine) {
                        uint8_t *brow = smem + (size_t)stage * STAGE_BYTES + A_BYTES + (size_t)(dt >> 3) * 1024 +
                                        (size_t)(dt & 7) * 128;
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            uint4 out = make_uint4(0, 0, 0, 0);
                            if (live && kb * 8 + q < da.G) {
                                // W^ = bf16_rn(s * (C_0[b0] + ... )), binary32 steps, as aqlm_dequant
                                // (each lane of the packed pair operations rounds on its own)
                                float2 acc[4];
#pragma unroll
                                for (int m = 0; m < FM; ++m) {
                                    const uint32_t k = stage_code<FM, FB, kCodeVecs>(code, q, m);
                                    const uint4 cw = !AQLM_IN_BOUNDS(k < (1u << FB), kSiteGemmCodebook, k)
                                                         ? make_uint4(0, 0, 0, 0)
                                                         : FB == 8
                                                         ? cbs[((m * 256 + k) << 3) | copy]
                                                         : ld_keep_u4(da.codebooks + (size_t)m * (1u << FB) + k, keep);
                                    const uint32_t wv[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                                    for (int h = 0; h < 4; ++h) {
                                        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&wv[h]));
                                        acc[h] = m == 0 ? f : __fadd2_rn(acc[h], f);
                                    }
                                }
                                const float2 s2 = make_float2(s, s);
                                uint32_t o[4];
#pragma unroll
                                for (int h = 0; h < 4; ++h) {
                                    const __nv_bfloat162 b2 = __float22bfloat162_rn(__fmul2_rn(acc[h], s2));
                                    o[h] = *reinterpret_cast<const uint32_t *>(&b2);
                                }
                                out = make_uint4(o[0], o[1], o[2], o[3]);
                            }
                            if (AQLM_IN_BOUNDS(dt < BN, kSiteGemmB, dt))
                                *reinterpret_cast<uint4 *>(brow + ((q ^ (dt & 7)) << 4)) = out;
                        }
                    }
                    // generic-proxy stores before the tensor cores' (async-proxy) reads
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_addr(&bars->full[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        }
        __syncwarp();
    } else {
        // ---- epilogue: warps 2..5, TMEM lane quarter = warp % 4 ----
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int mb = tile % m_tiles, nb = tile / m_tiles;
            bool ok = wait_bounded(smem_addr(&bars->tfull[acc]), acc_phase, bars, status, limit_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const int m = mb * BM + row_in_tile;
            const uint32_t t_base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * C::ACC_STRIDE);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(t_base + (uint32_t)(c * 32), r);
                const int n0 = nb * BN + c * 32;
                if (m < m_total && AQLM_IN_BOUNDS(nb < n_tiles && mb < m_tiles, kSiteGemmY, (size_t)m * n_total + n0))
                    store_bf16_row<4>(Y + (size_t)m * n_total + n0, r, n0, n_total);
            }
            if constexpr (BN % 32 != 0) {  // the last 16 columns of the tile
                uint32_t r[16];
                tmem_ld16(t_base + (uint32_t)(BN / 32 * 32), r);
                const int n0 = nb * BN + BN / 32 * 32;
                if (m < m_total && AQLM_IN_BOUNDS(nb < n_tiles && mb < m_tiles, kSiteGemmY, (size_t)m * n_total + n0))
                    store_bf16_row<2>(Y + (size_t)m * n_total + n0, r, n0, n_total);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bars->tempty[acc]));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
    }
}

// ---- the CTA-pair GEMM: 256 x BN tiles on two SMs ---------------------------
// tcgen05.mma.cta_group::2 (M = 256) runs one MMA on the tensor cores of a
// pair of SMs, a cluster of two CTAs: CTA r of the pair stages rows
// [128 r, 128 r + 128) of the X tile and rows [r BN/2, (r + 1) BN/2) of the W
// tile in its own shared memory (at the same offsets in both CTAs), the MMA
// reads both CTAs' tiles, and CTA r's tensor memory receives output rows
// [128 r, 128 r + 128) x all BN columns.  Per SM a stage is 128 + BN/2 rows of
// 128 bytes instead of 128 + BN, so each SM streams a third less operand data
// for the same MMA work, and six stages fit where four did.
//   both CTAs   warp 0 lane 0 loads its own halves with TMA; the bytes of both
//               complete the leader's (rank 0) full barrier, which the
//               leader's producer armed with the bytes of the two CTAs;
//   leader      warp 1 lane 0 issues the MMAs and commits to the empty and
//               tfull barriers of both CTAs (tcgen05.commit with a CTA mask);
//   both CTAs   warps 2-5 read their own accumulator rows and arrive on the
//               leader's tempty barrier (4 + 4 arrivals free an accumulator).
// Tensor memory is allocated and freed by warp 1 of both CTAs together
// (.cta_group::2).  Every wait is bounded; a wait that gives up raises the
// abort flag of both CTAs.  Before exiting, each CTA waits (bounded) for the
// arrivals the other CTA or the tensor cores still owe its barriers, and the
// two meet at a cluster barrier that every thread reaches, so that neither
// leaves while the other may still touch its shared or tensor memory.
constexpr int kPairRows = 2 * BM;   // output rows of a pair tile

// RESERVE: shared memory the decoder warps keep for 8-bit codebooks.
template <int BN, int RESERVE = 0>
struct PairCfg {
    static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "MMA N for M = 256");
    static constexpr int B_HALF = BN / 2;                   // rows of W each CTA stages (a multiple of 8)
    static constexpr int B_BYTES = B_HALF * BK * 2;         // a multiple of 1024: stages stay aligned
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int BUDGET = 216 * 1024 - RESERVE;   // of the 227 KiB a CTA may hold
    static constexpr int STAGES = BUDGET / STAGE_BYTES < kMaxStages ? BUDGET / STAGE_BYTES : kMaxStages;
    static constexpr int ACC_STRIDE = BN <= 128 ? 128 : 256;
    static constexpr uint32_t TMEM_COLS = 2 * ACC_STRIDE;
    // as GemmCfg::IDESC with M = 256
    static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                      ((uint32_t)(kPairRows >> 4) << 24);
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(Bars) + 16 + RESERVE;
    static_assert(B_BYTES % 1024 == 0 && STAGES >= 2, "ring layout");
};


__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// The shared::cluster address of the variable at shared address `saddr` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cl_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}
__device__ __forceinline__ void st_remote_u32(uint32_t cl_addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cl_addr), "r"(v) : "memory");
}
// TMA tile load into this CTA's shared memory whose bytes complete the
// barrier at shared::cluster address `bar` in either CTA of the pair.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
// Arrive on the barrier at shared address `bar` of both CTAs (mask 0b11) once
// the MMAs issued before have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    const uint16_t both = 3;
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"(both)
        : "memory");
}

// wait_bounded for a CTA of a pair: a wait that gives up also raises the
// other CTA's abort flag (at shared::cluster address peer_abort).
__device__ bool wait_bounded_pair(uint32_t bar, uint32_t parity, Bars *bars, uint32_t peer_abort, int32_t *status,
                                  uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 0) {
            if (*reinterpret_cast<volatile int *>(&bars->abort_flag)) return false;
            if (now_ns() - t0 > limit_ns) {
                *reinterpret_cast<volatile int *>(&bars->abort_flag) = 1;
                st_remote_u32(peer_abort, 1u);
                atomicExch(status, (int32_t)AQLM_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// ---- overlapped dequantisation: W^ decoded once, in the order the MMAs need it
// With FM > 0 the pair kernel also decodes the layer: eight decoder warps per
// CTA turn codes into W^ rows in global memory (the workspace), with the
// binary32 steps of aqlm_dequant, while the tensor cores run; each CTA's TMA
// producer loads a W tile only once the units that write it are complete.
// The bands [0, band0) that the first wave of tiles needs are decoded before
// the launch (by the dequantisation kernel); the decoder warps take the rest.
// The work is cut into units of 16 rows x 64 inputs (one k block of a 16-row
// slice of a band of BN rows).  Units are numbered in the order the tiles
// need them -- bands in groups of about one wave's worth (GB bands, whose
// first tiles fall in the same wave), k blocks in order within a group -- and
// decoder warps claim the next ones from global counters, so the whole GPU
// decodes what the next waves need first, and no CTA ever waits for a CTA
// that is not running (whoever claims a unit is running and finishes it).
// Claims (U consecutive units) are dealt over kClaimStreams counters: decoder
// warp w of a CTA takes claims w, w + 8, w + 16, ... from counter w, which
// keeps the need order while spreading the atomics over eight L2 lines.  A
// finished unit goes to the CTA's publisher warp, which adds it to its
// panel's counter (see Mailbox); the producer reads the counters of 32 k
// blocks at a time, ahead of need, and loads when a panel holds all BN/16 of
// its units.
// Division of x < 2^31 by an invariant d as a multiply and a shift (the
// scheme of Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994): s = ceil(log2 d), m = floor(2^(31+s) / d) + 1 < 2^32,
// x / d = floor(x m / 2^(31+s)).
struct FastDiv {
    uint32_t d, m;
    int shift;
    __device__ __forceinline__ uint32_t div(uint32_t x) const { return (uint32_t)(((uint64_t)x * m) >> shift); }
};
inline FastDiv make_fast_div(uint32_t d) {
    int s = 0;
    while ((1ull << s) < d) ++s;
    FastDiv f;
    f.d = d;
    f.m = (uint32_t)((1ull << (31 + s)) / d + 1);
    f.shift = 31 + s;
    return f;
}

constexpr int kClaimStreams = 8;   // = the decoder warps of a CTA
constexpr int kClaimBytes = 128 * kClaimStreams;
static_assert(kClaimStreams == kDecWarps, "one claim stream per decoder warp");

struct OverlapArgs {
    const uint8_t *codes;       // [d_out][G] groups of M*B/8 bytes
    const uint4 *codebooks;     // [M][2^B] codewords of 8 fp16
    const __half *scales;       // [d_out]
    uint4 *W;                   // W^ [d_out][d_in] bf16, 8 per uint4 (G per row)
    uint32_t *next_claim;       // kClaimStreams claim counters, 128 bytes apart, zero at launch
    uint32_t *panel_done;       // [n_bands][kb_pad] finished units, zero at launch
    int d_out, G, row_bytes;
    int n_bands, num_kb, kb_pad, GB;
    int band0;                  // bands [0, band0) are decoded before the launch (complete)
    uint32_t total_units;       // (n_bands - band0) * (BN / 16) * num_kb (< 2^31)
    FastDiv per_group;          // units of a group of GB bands
    FastDiv per_kb, per_kb_last;   // units of one k block of a full group, of the last group
};

// Decoder warps hand their finished units to one publisher warp of the CTA
// through shared memory (a ring of kMailSlots per decoder warp, written with
// CTA-scope release), so that no decoder warp ever waits for a GPU-scope
// fence -- which would drain its loads and gathers in flight.  The publisher,
// with no memory traffic of its own, reads the rings (acquire, CTA scope),
// issues one fence.acq_rel.gpu for everything it read and then adds the
// units to their panel counters: the decoders' stores happen before the
// fence (CTA-scope release/acquire), so every SM that sees a count also
// sees the stores.
constexpr int kMailSlots = 32;
struct Mailbox {
    uint32_t head[kDecWarps];                 // entries written by decoder warp w
    uint32_t tail[kDecWarps];                 // entries of warp w the publisher has counted
    uint32_t finished[kDecWarps];             // decoder warp w is done
    uint32_t entry[kDecWarps][kMailSlots];    // packed units
};
constexpr int kMailBytes = (int)((sizeof(Mailbox) + 127) / 128 * 128);
constexpr int kOverlapThreads = kGemmThreads + kDecThreads + 32;   // + the publisher warp

template <int FM, int FB>
constexpr int overlap_reserve() {
    return FM > 0 ? (FB == 8 ? FM * 256 * 16 : 0) + kMailBytes : 0;
}

__device__ __forceinline__ uint32_t ld_acquire_shared(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_shared(uint32_t *p, uint32_t v) {
    asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_addr(p)), "r"(v) : "memory");
}

// Unit u in need order -> band nb, k block kb and 16-row slice r of the band.
template <int CHUNKS>
__device__ __forceinline__ bool unit_coords(uint32_t u, const OverlapArgs &oa, int &nb, int &kb, int &r) {
    if (u >= oa.total_units) return false;
    const uint32_t g = oa.per_group.div(u);
    const uint32_t rem = u - g * oa.per_group.d;
    const int b_lo = oa.band0 + (int)g * oa.GB;
    const FastDiv &fk = oa.n_bands - b_lo < oa.GB ? oa.per_kb_last : oa.per_kb;
    kb = (int)fk.div(rem);
    const uint32_t rem2 = rem - (uint32_t)kb * fk.d;
    nb = b_lo + (int)(rem2 / CHUNKS);
    r = (int)(rem2 % CHUNKS);
    return true;
}

__device__ __forceinline__ void red_relaxed_add(uint32_t *p, uint32_t v) {
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint4 ld_relaxed_u4(const uint32_t *p) {
    uint4 v;
    asm volatile("ld.relaxed.gpu.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

// A claimed unit packed in one word: band << 18 | k block << 4 | slice
// (0xffffffff: no unit, past the last one).
__device__ __forceinline__ uint32_t pack_unit(int nb, int kb, int r) {
    return ((uint32_t)nb << 18) | ((uint32_t)kb << 4) | (uint32_t)r;
}

// The decoder warps' loop.  A claim is U consecutive units; lane l of a
// unit's step s (0..3) handles row 4 s + l / 8 of the 16-row slice and group
// l % 8 of the k block, so each 16-byte store of the warp fills four 128-byte
// lines.  Three claims are in flight at once, one phase apart: the codes of
// the newest are loading, the codewords of the next are being gathered, and
// the oldest is converted, stored and counted -- so a phase waits for one
// memory latency, whose loads, gathers and stores overlap; the ticket of the
// next claim (a global atomic) is taken one phase before it is used.
template <int BN, int FM, int FB>
__device__ void decode_units(const OverlapArgs &oa, const uint4 *cbs, Mailbox *mbx, int stream, int lane,
                             int32_t *status, uint64_t limit_ns) {
    constexpr int CHUNKS = BN / 16;
    constexpr int CB = FM * FB / 8;                       // code bytes per group
    constexpr int U = FM == 2 ? 1 : 2;                    // units per claim (registers: M codewords per group)
    constexpr int S = 4 * U;                              // groups per lane per claim
    const uint64_t keep = policy_evict_last();
    struct Claim {
        uint32_t u0;
        uint32_t pk[U];
    };
    auto claim_of = [&](uint32_t ticket, Claim &c) {
        c.u0 = __shfl_sync(0xffffffffu, ticket, 0);
#pragma unroll
        for (int j = 0; j < U; ++j) {
            int nb, kb, r;
            c.pk[j] = unit_coords<CHUNKS>(c.u0 + j, oa, nb, kb, r) ? pack_unit(nb, kb, r) : 0xffffffffu;
        }
    };
    uint32_t *counter = oa.next_claim + 32 * stream;
    // the first unit of the next claim of this stream (lane 0; shuffled when used)
    auto ticket = [&]() -> uint32_t {
        return lane == 0 ? (atomicAdd(counter, 1u) * kClaimStreams + (uint32_t)stream) * (uint32_t)U : 0u;
    };
    // this lane's first row (step 0) and group in unit j of c; false: no work in the unit
    auto unit_base = [&](const Claim &c, int j, int &row0, int &grp) -> bool {
        const uint32_t pk = c.pk[j];
        row0 = (int)(pk >> 18) * BN + (int)(pk & 15) * 16 + (lane >> 3);
        grp = (int)((pk >> 4) & 0x3fff) * 8 + (lane & 7);
        return pk != 0xffffffffu && grp < oa.G;
    };
    auto load = [&](const Claim &c, uint32_t (&code)[S]) {
#pragma unroll
        for (int j = 0; j < U; ++j) {
            int row0, grp;
            const bool ok = unit_base(c, j, row0, grp);
            const uint8_t *p = oa.codes + (size_t)row0 * oa.row_bytes + (size_t)grp * CB;
            const size_t step = (size_t)4 * oa.row_bytes;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                code[4 * j + t] = 0;
                if (ok && row0 + 4 * t < oa.d_out)
                    code[4 * j + t] = CB == 2 ? (uint32_t)__ldcs(reinterpret_cast<const uint16_t *>(p + t * step))
                                              : __ldcs(reinterpret_cast<const uint32_t *>(p + t * step));
            }
        }
    };
    auto gather = [&](const Claim &c, const uint32_t (&code)[S], uint4 (&cw)[S][FM], float (&sc)[S]) {
#pragma unroll
        for (int s = 0; s < S; ++s) {
            int row0, grp;
            const bool in = unit_base(c, s >> 2, row0, grp) && row0 + 4 * (s & 3) < oa.d_out;
            sc[s] = in ? __half2float(oa.scales[row0 + 4 * (s & 3)]) : 0.f;
#pragma unroll
            for (int m = 0; m < FM; ++m) {
                const uint32_t k = FM == 1 ? (code[s] & 0xffffu)
                                           : FB == 8 ? (code[s] >> (8 * m)) & 0xffu : (code[s] >> (16 * m)) & 0xffffu;
                cw[s][m] = make_uint4(0, 0, 0, 0);
                if (in && AQLM_IN_BOUNDS(k < (1u << FB), kSiteGemmCodebook, k))
                    cw[s][m] = FB == 8 ? cbs[m * 256 + k] : ld_keep_u4(oa.codebooks + ((size_t)m << FB) + k, keep);
            }
        }
    };
    auto emit = [&](const Claim &c, const uint4 (&cw)[S][FM], const float (&sc)[S]) {
#pragma unroll
        for (int s = 0; s < S; ++s) {
            int row0, grp;
            if (!unit_base(c, s >> 2, row0, grp)) continue;
            const int row = row0 + 4 * (s & 3);
            if (row >= oa.d_out) continue;
            // W^ = bf16_rn(s * (C_0[b0] + ...)), binary32 steps in codebook order, as aqlm_dequant
            float acc[kGroup];
            half8_to_float8(cw[s][0], acc);
#pragma unroll
            for (int m = 1; m < FM; ++m) {
                float f[kGroup];
                half8_to_float8(cw[s][m], f);
#pragma unroll
                for (int t = 0; t < kGroup; ++t) acc[t] = __fadd_rn(acc[t], f[t]);
            }
            uint32_t out[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const __nv_bfloat16 lo = __float2bfloat16_rn(__fmul_rn(acc[2 * h], sc[s]));
                const __nv_bfloat16 hi = __float2bfloat16_rn(__fmul_rn(acc[2 * h + 1], sc[s]));
                out[h] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
            }
            const size_t w = (size_t)row * oa.G + grp;
            if (AQLM_IN_BOUNDS(w < (size_t)oa.d_out * oa.G, kSiteGemmB, w)) oa.W[w] = make_uint4(out[0], out[1], out[2], out[3]);
        }
    };
    // Hand the units of claim c to the publisher: the stores ordered before
    // the async-proxy reads of any SM that later sees the counts (proxy
    // fence), then the ring entries, released at CTA scope with the new head.
    uint32_t head = 0;   // lane 0: entries written to this warp's ring
    auto publish = [&](const Claim &c) {
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const uint32_t pk = c.pk[j];
                if (pk == 0xffffffffu) continue;
                // a free slot (the publisher empties the ring within microseconds)
                uint64_t t0 = 0;
                while (head - ld_acquire_shared(&mbx->tail[stream]) >= (uint32_t)kMailSlots) {
                    const uint64_t t = now_ns();
                    if (t0 == 0) t0 = t;
                    else if (t - t0 > limit_ns) {
                        atomicExch(status, (int32_t)AQLM_ERR_TIMEOUT);
                        break;
                    }
                }
                mbx->entry[stream][head % kMailSlots] = pk;
                ++head;
            }
            st_release_shared(&mbx->head[stream], head);
        }
    };

    Claim a, b, c, n;
    uint32_t code[S];
    uint4 cwA[S][FM], cwB[S][FM];
    float scA[S], scB[S];
    // prologue: a's codewords being gathered, b's codes loading, the ticket of the third taken
    claim_of(ticket(), a);
    load(a, code);
    gather(a, code, cwA, scA);
    claim_of(ticket(), b);
    load(b, code);
    uint32_t tk = ticket();
    while (a.u0 < oa.total_units) {
        gather(b, code, cwB, scB);
        claim_of(tk, c);
        tk = ticket();
        load(c, code);
        emit(a, cwA, scA);
        publish(a);
        if (b.u0 >= oa.total_units) break;
        gather(c, code, cwA, scA);
        claim_of(tk, n);
        tk = ticket();
        load(n, code);
        emit(b, cwB, scB);
        publish(b);
        // c's codewords in cwA, n's codes loading: the loop's entry state again
        a = c;
        b = n;
    }
    __syncwarp();
    if (lane == 0) st_release_shared(&mbx->finished[stream], 1u);
}

// The publisher warp's loop (one lane): count the units the decoder warps
// handed over, one GPU-scope fence per batch, until every decoder warp is
// done.  Bounded: gives up (status AQLM_ERR_TIMEOUT) after limit_ns without
// a new entry.
__device__ void publish_units(const OverlapArgs &oa, Mailbox *mbx, int32_t *status, uint64_t limit_ns) {
    uint32_t seen[kDecWarps];
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) seen[w] = 0;
    uint64_t idle_since = now_ns();
    for (;;) {
        uint32_t h[kDecWarps];
        bool all_done = true, any = false;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            all_done &= ld_acquire_shared(&mbx->finished[w]) != 0;   // before the head: a done warp's last head is seen
            h[w] = ld_acquire_shared(&mbx->head[w]);
            any |= h[w] != seen[w];
        }
        if (any) {
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) {
                for (uint32_t i = seen[w]; i != h[w]; ++i) {
                    const uint32_t pk = *reinterpret_cast<volatile uint32_t *>(&mbx->entry[w][i % kMailSlots]);
                    red_relaxed_add(oa.panel_done + (size_t)(pk >> 18) * oa.kb_pad + ((pk >> 4) & 0x3fff), 1u);
                }
                if (h[w] != seen[w]) st_release_shared(&mbx->tail[w], h[w]);
                seen[w] = h[w];
            }
            idle_since = now_ns();
        } else if (all_done) {
            break;
        } else {
            __nanosleep(64);
            if (now_ns() - idle_since > limit_ns) {
                atomicExch(status, (int32_t)AQLM_ERR_TIMEOUT);
                break;
            }
        }
    }
}

// The producer's view of the panel counters: windows of 32 k blocks of one
// band (kb_pad is a multiple of 32), read with 8 relaxed 16-byte loads.  A
// window's loads are issued ahead of need (issue) and evaluated when the
// producer gets there (scan); a panel found incomplete is waited for with
// bounded polling (wait_window).  A successful evaluation is followed by an
// acquire fence (GPU scope) and a proxy fence, so the TMA loads issued after
// it see the decoders' stores.
constexpr int kWindow = 32;

struct PanelWindow {
    uint4 v[kWindow / 4];
    int nb = -1, w = -1;   // band and window index whose counters v holds (or is loading)
    __device__ void issue(const OverlapArgs &oa, int band, int window) {
        const uint32_t *row = oa.panel_done + (size_t)band * oa.kb_pad + window * kWindow;
#pragma unroll
        for (int i = 0; i < kWindow / 4; ++i) v[i] = ld_relaxed_u4(row + 4 * i);
        nb = band;
        w = window;
    }
    // If panel kb of the window is complete: the last k block d >= kb such that
    // kb..d are complete (within the window and the band), else -1.
    template <int CHUNKS>
    __device__ int scan(const OverlapArgs &oa, int kb) const {
        uint32_t done = 0;   // bit i: panel base + i complete
#pragma unroll
        for (int i = 0; i < kWindow / 4; ++i) {
            done |= (uint32_t)(v[i].x >= (uint32_t)CHUNKS) << (4 * i);
            done |= (uint32_t)(v[i].y >= (uint32_t)CHUNKS) << (4 * i + 1);
            done |= (uint32_t)(v[i].z >= (uint32_t)CHUNKS) << (4 * i + 2);
            done |= (uint32_t)(v[i].w >= (uint32_t)CHUNKS) << (4 * i + 3);
        }
        const int base = w * kWindow;
        const uint32_t run = ~(done >> (kb - base));   // first set bit: the first incomplete panel from kb on
        if (run & 1u) return -1;
        const int d = kb + (run ? __ffs((int)run) - 1 : kWindow) - 1;
        const int last = (base + kWindow < oa.num_kb ? base + kWindow : oa.num_kb) - 1;
        return d < last ? d : last;
    }
};

// Bounded wait until panel (nb, kb) is complete; returns the last complete k
// block from kb on (as scan), or -1 after a timeout or an abort.
template <int CHUNKS>
__device__ int wait_window(const OverlapArgs &oa, PanelWindow &pw, int nb, int kb, Bars *bars, uint32_t peer_abort,
                           int32_t *status, uint64_t limit_ns) {
    uint64_t t0 = 0;
    for (;;) {
        pw.issue(oa, nb, kb / kWindow);
        const int d = pw.template scan<CHUNKS>(oa, kb);
        if (d >= 0) return d;
        if (*reinterpret_cast<volatile int *>(&bars->abort_flag)) return -1;
        const uint64_t t = now_ns();
        if (t0 == 0) {
            t0 = t;
        } else if (t - t0 > limit_ns) {
            *reinterpret_cast<volatile int *>(&bars->abort_flag) = 1;
            st_remote_u32(peer_abort, 1u);
            atomicExch(status, (int32_t)AQLM_ERR_TIMEOUT);
            return -1;
        }
    }
}

template <int BN, int FM, int FB>
__global__ void __launch_bounds__(FM > 0 ? kOverlapThreads : kGemmThreads, 1)
gemm_bf16_tcgen05_pair(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                       __nv_bfloat16 *__restrict__ Y, int m_total, int n_total, int k_total, int32_t *status,
                       unsigned long long limit_ns, int stall_test, const OverlapArgs oa) {
    using C = PairCfg<BN, overlap_reserve<FM, FB>()>;
    constexpr int STAGES = C::STAGES, STAGE_BYTES = C::STAGE_BYTES;
    constexpr bool kDecode = FM > 0;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled tiles (the same offsets in both CTAs)
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t *smem = smem_raw + ((1024 - (raw & 1023)) & 1023);
    Bars *bars = reinterpret_cast<Bars *>(smem + (size_t)STAGES * STAGE_BYTES);
    uint4 *cbs = reinterpret_cast<uint4 *>(smem + (size_t)STAGES * STAGE_BYTES + ((sizeof(Bars) + 15) & ~size_t(15)));
    Mailbox *mbx = reinterpret_cast<Mailbox *>(reinterpret_cast<uint8_t *>(cbs) + (FB == 8 ? FM * 256 * 16 : 0));
    if constexpr (kDecode) {
        if constexpr (FB == 8) {  // 8-bit codebooks in shared memory
            for (int i = threadIdx.x; i < FM * 256; i += blockDim.x) cbs[i] = oa.codebooks[i];
        } else if (threadIdx.x == 0) {
            // 16-bit codebooks (1-2 MiB, usually cold): each CTA asks L2 for its share
            const uint32_t cb_bytes = (uint32_t)FM * (1u << FB) * 16;
            const uint32_t share = ((cb_bytes + gridDim.x - 1) / gridDim.x + 255) & ~255u;
            const uint32_t off = blockIdx.x * share;
            if (off < cb_bytes)
                prefetch_l2_bulk(reinterpret_cast<const uint8_t *>(oa.codebooks) + off, min(share, cb_bytes - off),
                                 policy_evict_last());
        }
        for (int i = threadIdx.x; i < (int)(sizeof(Mailbox) / 4); i += blockDim.x)
            reinterpret_cast<uint32_t *>(mbx)[i] = 0;
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();           // 0: the leader, which issues the MMAs
    const int pair_id = (int)cluster_id_x(), pairs = (int)cluster_count_x();
    const int m_tiles = (m_total + kPairRows - 1) / kPairRows;
    const int n_tiles = (n_total + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;
    const int num_kb = (k_total + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_addr(&bars->full[s]), 1);    // leader: its producer's arrival with both CTAs' bytes
            mbar_init(smem_addr(&bars->empty[s]), 1);   // the leader's MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_addr(&bars->tfull[a]), 1);
            mbar_init(smem_addr(&bars->tempty[a]), 2 * kEpiWarps);   // leader: the epilogue warps of both CTAs
        }
        mbar_init(smem_addr(&bars->mma_done), 1);
        bars->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_x)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_w)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(&bars->tmem_base)),
                     "r"(C::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    // the barriers of both CTAs initialised before either CTA uses the other's
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t peer_abort = map_shared(smem_addr(&bars->abort_flag), rank ^ 1u);

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer (both CTAs) ----
            grid_dep_wait();   // launched early after the kernel writing W (a no-op otherwise)
            int stage = 0;
            uint32_t phase = 0;
            int issued_parity[STAGES];
            for (int s = 0; s < STAGES; ++s) issued_parity[s] = -1;
            bool ok = true;
            int poll_nb = -1, done_kb = -1;   // decoded panels known complete: band poll_nb, k blocks <= done_kb
            PanelWindow ahead;                // counters loading ahead of need
            for (int tile = pair_id; tile < num_tiles && ok && !stall_test; tile += pairs) {
                const int mb = tile % m_tiles, nb = tile / m_tiles;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!wait_bounded_pair(smem_addr(&bars->empty[stage]), phase ^ 1, bars, peer_abort, status,
                                           limit_ns)) {
                        ok = false;
                        break;
                    }
                    if constexpr (kDecode) {
                        constexpr int CHUNKS = BN / 16;
                        if (nb < oa.band0) {
                            // decoded before the launch: visible after the grid dependency
                            poll_nb = nb;
                            done_kb = num_kb - 1;
                        } else if (nb != poll_nb || kb > done_kb) {
                            int d = -1;
                            if (ahead.nb == nb && ahead.w == kb / kWindow) d = ahead.template scan<CHUNKS>(oa, kb);
                            if (d < 0) d = wait_window<CHUNKS>(oa, ahead, nb, kb, bars, peer_abort, status, limit_ns);
                            if (d < 0) {
                                ok = false;
                                break;
                            }
                            asm volatile("fence.acq_rel.gpu;" ::: "memory");
                            asm volatile("fence.proxy.async.global;" ::: "memory");
                            poll_nb = nb;
                            done_kb = d;
                            ahead.nb = -1;
                        }
                        // 8 stages before the known-complete panels run out, load the
                        // counters that come next: this band's, or the next tile's band's
                        if (ahead.nb < 0 && kb + 8 >= done_kb) {
                            if (done_kb + 1 < num_kb) {
                                ahead.issue(oa, nb, (done_kb + 1) / kWindow);
                            } else if (tile + pairs < num_tiles) {
                                const int nb_next = (tile + pairs) / m_tiles;
                                if (nb_next != nb && nb_next >= oa.band0) ahead.issue(oa, nb_next, 0);
                            }
                        }
                    }
                    const uint32_t full_local = smem_addr(&bars->full[stage]);
                    const uint32_t full_leader = map_shared(full_local, 0);
                    const uint32_t dst = smem_addr(smem + (size_t)stage * STAGE_BYTES);
                    if (rank == 0) mbar_expect_tx(full_local, (uint32_t)(2 * STAGE_BYTES));
                    tma_load_2d_pair(dst, &tmap_x, kb * BK, mb * kPairRows + (int)rank * BM, full_leader);
                    tma_load_2d_pair(dst + A_BYTES, &tmap_w, kb * BK, nb * BN + (int)rank * C::B_HALF, full_leader);
                    issued_parity[stage] = (int)phase;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            // Every stage released by the MMAs: the commits owed to this CTA's empty barriers have landed.
            for (int s = 0; s < STAGES; ++s) {
                if (!wait_bounded_pair(smem_addr(&bars->empty[stage]), phase ^ 1, bars, peer_abort, status, limit_ns))
                    break;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            // The leader's full barriers count the copies of both CTAs: none may still be landing.
            if (rank == 0) {
                for (int s = 0; s < STAGES; ++s) {
                    if (issued_parity[s] >= 0) {
                        const uint32_t full = smem_addr(&bars->full[s]);
                        const uint64_t t0 = now_ns();
                        while (!mbar_try_wait(full, (uint32_t)issued_parity[s]) && now_ns() - t0 < limit_ns) {
                        }
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            if (rank == 0) {
                // ---- MMA issuer (leader) ----
                int stage = 0;
                uint32_t phase = 0;
                int acc = 0;
                uint32_t acc_phase = 0;
                bool ok = true;
                for (int tile = pair_id; tile < num_tiles && ok; tile += pairs) {
                    if (!wait_bounded_pair(smem_addr(&bars->tempty[acc]), acc_phase ^ 1, bars, peer_abort, status,
                                           limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem + (uint32_t)(acc * C::ACC_STRIDE);
                    for (int kb = 0; kb < num_kb; ++kb) {
                        if (!wait_bounded_pair(smem_addr(&bars->full[stage]), phase, bars, peer_abort, status,
                                               limit_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a0 = smem_addr(smem + (size_t)stage * STAGE_BYTES);
                        const uint32_t b0 = a0 + A_BYTES;
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k) {
                            mma_bf16_pair(d_tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), C::IDESC,
                                          (kb > 0 || k > 0) ? 1u : 0u);
                        }
                        mma_commit_pair(smem_addr(&bars->empty[stage]));
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                    if (!ok) break;
                    mma_commit_pair(smem_addr(&bars->tfull[acc]));
                    if (++acc == 2) {
                        acc = 0;
                        acc_phase ^= 1;
                    }
                }
                mma_commit_pair(smem_addr(&bars->mma_done));
                // Both accumulators released by the epilogues of both CTAs: the
                // peer's arrivals on this CTA's tempty barriers have landed.
                for (int a = 0; a < 2; ++a) {
                    if (!wait_bounded_pair(smem_addr(&bars->tempty[acc]), acc_phase ^ 1, bars, peer_abort, status,
                                           limit_ns))
                        break;
                    if (++acc == 2) {
                        acc = 0;
                        acc_phase ^= 1;
                    }
                }
            }
            // Tensor memory is freed below only after every issued MMA completed
            // (the leader's last commit reaches both CTAs).
            const uint64_t t0 = now_ns();
            while (!mbar_try_wait(smem_addr(&bars->mma_done), 0) && now_ns() - t0 < limit_ns) {
            }
        }
        __syncwarp();
    } else if (kDecode && warp >= 2 + kEpiWarps + kDecWarps) {
        // ---- publisher (both CTAs): the decoders' units to the panel counters ----
        if constexpr (kDecode) {
            if (lane == 0) publish_units(oa, mbx, status, limit_ns);
        }
        __syncwarp();
    } else if (kDecode && warp >= 2 + kEpiWarps) {
        // ---- decoders (both CTAs): W^ for every CTA of the grid ----
        if constexpr (kDecode)
            decode_units<BN, FM, FB>(oa, cbs, mbx, warp - (2 + kEpiWarps), lane, status, limit_ns);
        __syncwarp();
    } else {
        // ---- epilogue (both CTAs): warps 2..5, TMEM lane quarter = warp % 4 ----
        const int quarter = warp & 3;
        const int row_in_tile = (int)rank * BM + quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = pair_id; tile < num_tiles; tile += pairs) {
            const int mb = tile % m_tiles, nb = tile / m_tiles;
            bool ok = wait_bounded_pair(smem_addr(&bars->tfull[acc]), acc_phase, bars, peer_abort, status, limit_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
            const int m = mb * kPairRows + row_in_tile;
            const uint32_t t_base = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * C::ACC_STRIDE);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(t_base + (uint32_t)(c * 32), r);
                const int n0 = nb * BN + c * 32;
                if (m < m_total && AQLM_IN_BOUNDS(nb < n_tiles && mb < m_tiles, kSiteGemmY, (size_t)m * n_total + n0))
                    store_bf16_row<4>(Y + (size_t)m * n_total + n0, r, n0, n_total);
            }
            if constexpr (BN % 32 != 0) {  // the last 16 columns of the tile
                uint32_t r[16];
                tmem_ld16(t_base + (uint32_t)(BN / 32 * 32), r);
                const int n0 = nb * BN + BN / 32 * 32;
                if (m < m_total && AQLM_IN_BOUNDS(nb < n_tiles && mb < m_tiles, kSiteGemmY, (size_t)m * n_total + n0))
                    store_bf16_row<2>(Y + (size_t)m * n_total + n0, r, n0, n_total);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(map_shared(smem_addr(&bars->tempty[acc]), 0));
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
    }

    // Neither CTA leaves (or frees the pair's tensor memory) while the other
    // may still read its shared memory or signal its barriers.
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
    }
}

// ---- host side: tensor maps through the driver entry point ----

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 2-D bf16 tensor [rows][cols] (cols contiguous), box = box_rows x 64 columns.
bool make_map(CUtensorMap *map, const void *base, int rows, int cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace


namespace {
template <int BN, int FM, int FB>
cudaError_t launch_gemm_bn(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                           int32_t *status, cudaStream_t st, unsigned long long limit_ns, int stall_test, int sms,
                           const DecodeArgs &da, bool pdl = false) {
    using C = GemmCfg<BN, decode_reserve<FM, FB>()>;
    CUtensorMap mx, mw;
    if (!make_map(&mx, X, tokens, k, BM)) return cudaErrorInvalidValue;
    if (FM == 0 && !make_map(&mw, W, n, k, BN)) return cudaErrorInvalidValue;
    if (FM > 0) mw = mx;   // unused by the fused kernel
    auto fn = gemm_bf16_tcgen05<BN, FM, FB>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    const int tiles = ((tokens + BM - 1) / BM) * ((n + BN - 1) / BN);
    const int grid = tiles < sms ? tiles : sms;
    return launch_kernel(fn, dim3(grid), dim3(kGemmThreads + (FM > 0 ? kDecThreads : 0)), C::SMEM, st, pdl, mx,
                         mw, reinterpret_cast<__nv_bfloat16 *>(Y), tokens, n, k, status, limit_ns, stall_test, da);
}
}  // namespace

// The tile width for a tokens x n product on `sms` SMs: the one whose tiles,
// dealt round robin, give the least waves x (BM + BN) -- the busiest SM's
// share of operand bytes; ties to the wider tile.
int gemm_tile_n(int tokens, int n, int sms) {
    constexpr int kCands[] = {256, 240, 224, 192};
    const long long m_tiles = (tokens + BM - 1) / BM;
    int best = kCands[0];
    long long best_cost = -1;
    for (int bn : kCands) {
        const long long tiles = m_tiles * ((n + bn - 1) / bn);
        const long long waves = (tiles + sms - 1) / sms;
        const long long cost = waves * (BM + bn);
        if (best_cost < 0 || cost < best_cost) {
            best = bn;
            best_cost = cost;
        }
    }
    return best;
}

namespace {
template <int FM, int FB>
cudaError_t launch_by_width(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                            int32_t *status, cudaStream_t st, unsigned long long limit_ns, int stall_test,
                            const DecodeArgs &da, bool pdl = false) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int sms = num_sms(dev);
    switch (gemm_tile_n(tokens, n, sms)) {
        case 240:
            return launch_gemm_bn<240, FM, FB>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, sms, da, pdl);
        case 224:
            return launch_gemm_bn<224, FM, FB>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, sms, da, pdl);
        case 192:
            return launch_gemm_bn<192, FM, FB>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, sms, da, pdl);
        default:
            return launch_gemm_bn<256, FM, FB>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, sms, da, pdl);
    }
}
}  // namespace

namespace {
// Pairs of SMs that can hold a CTA pair of the kernel at once (0 if the
// device cannot), queried once per device.
template <int BN, int FM, int FB>
int pair_slots(int dev) {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> cached[kMaxDevices];
    if (dev >= 0 && dev < kMaxDevices) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c != 0) return c > 0 ? c : 0;
    }
    using C = PairCfg<BN, overlap_reserve<FM, FB>()>;
    auto fn = gemm_bf16_tcgen05_pair<BN, FM, FB>;
    int count = 0;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * num_sms(dev));
        cfg.blockDim = dim3(FM > 0 ? kOverlapThreads : kGemmThreads);
        cfg.dynamicSmemBytes = C::SMEM;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&count, fn, &cfg) != cudaSuccess) count = 0;
    }
    if (dev >= 0 && dev < kMaxDevices) cached[dev].store(count > 0 ? count : -1, std::memory_order_relaxed);
    return count > 0 ? count : 0;
}

// Tiles of a tokens x n product in 256 x BN pair tiles.
long long pair_tiles(int tokens, int n, int bn) {
    return (long long)((tokens + kPairRows - 1) / kPairRows) * ((n + bn - 1) / bn);
}

// oa: the decoding work (FM > 0); its pair-dependent field GB is set here.
template <int BN, int FM, int FB>
cudaError_t launch_gemm_pair_bn(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                                int32_t *status, cudaStream_t st, unsigned long long limit_ns, int stall_test,
                                int dev, OverlapArgs oa, bool pdl = false) {
    using C = PairCfg<BN, overlap_reserve<FM, FB>()>;
    const int slots = pair_slots<BN, FM, FB>(dev);
    if (slots < 1) return cudaErrorNotSupported;
    CUtensorMap mx, mw;
    if (!make_map(&mx, X, tokens, k, BM)) return cudaErrorInvalidValue;
    if (!make_map(&mw, W, n, k, C::B_HALF)) return cudaErrorInvalidValue;
    auto fn = gemm_bf16_tcgen05_pair<BN, FM, FB>;
    // (pair_slots set it once per device; again here, in case the context was reset since)
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    const long long tiles = pair_tiles(tokens, n, BN);
    const int pairs = tiles < slots ? (int)tiles : slots;
    const int m_tiles = (tokens + kPairRows - 1) / kPairRows;
    oa.GB = (pairs + m_tiles - 1) / m_tiles;   // bands whose first tiles share a wave
    const int rest = oa.n_bands - oa.band0;     // bands the decoder warps decode
    if (rest > 0) {
        constexpr uint32_t CHUNKS = BN / 16;
        const int last = rest - (rest - 1) / oa.GB * oa.GB;   // bands of the last group
        oa.per_group = make_fast_div((uint32_t)oa.GB * CHUNKS * (uint32_t)oa.num_kb);
        oa.per_kb = make_fast_div((uint32_t)oa.GB * CHUNKS);
        oa.per_kb_last = make_fast_div((uint32_t)last * CHUNKS);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs);
    cfg.blockDim = dim3(FM > 0 ? kOverlapThreads : kGemmThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, fn, mx, mw, reinterpret_cast<__nv_bfloat16 *>(Y), tokens, n, k, status, limit_ns,
                              stall_test, oa);
}
}  // namespace

// The tile width of the CTA-pair kernel for a tokens x n product on `pairs`
// SM pairs: a pair tile costs its SMs MMA time in proportion to its width
// (each SM computes 128 x width per k step), so the rule takes the least
// waves x width, ties to the wider tile.
int gemm_pair_tile_n(int tokens, int n, int pairs) {
    constexpr int kCands[] = {256, 240, 224, 192};
    const long long m_tiles = (tokens + kPairRows - 1) / kPairRows;
    int best = kCands[0];
    long long best_cost = -1;
    for (int bn : kCands) {
        const long long tiles = m_tiles * ((n + bn - 1) / bn);
        const long long waves = (tiles + pairs - 1) / pairs;
        const long long cost = waves * bn;
        if (best_cost < 0 || cost < best_cost) {
            best = bn;
            best_cost = cost;
        }
    }
    return best;
}

// The pair kernel serves products of more than one 128-token tile.
bool gemm_uses_pair(int tokens) { return tokens > BM; }

cudaError_t launch_bf16_gemm_cfg(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                                 int32_t *status, cudaStream_t st, unsigned long long limit_ns, int stall_test,
                                 int cta_pair, int tile_n, bool pdl) {
    int dev = 0;
    cudaGetDevice(&dev);
    const bool pair = cta_pair < 0 ? gemm_uses_pair(tokens) : cta_pair != 0;
    if (!pair) {
        const DecodeArgs none = {};
        if (tile_n == 0)
            return launch_by_width<0, 0>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, none, pdl);
        const int sms = num_sms(dev);
        switch (tile_n) {
            case 256:
                return launch_gemm_bn<256, 0, 0>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, sms, none,
                                                 pdl);
            case 240:
                return launch_gemm_bn<240, 0, 0>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, sms, none,
                                                 pdl);
            case 224:
                return launch_gemm_bn<224, 0, 0>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, sms, none,
                                                 pdl);
            case 192:
                return launch_gemm_bn<192, 0, 0>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, sms, none,
                                                 pdl);
            default:
                return cudaErrorInvalidValue;
        }
    }
    if (tile_n == 0) {
        const int slots = pair_slots<256, 0, 0>(dev);
        tile_n = gemm_pair_tile_n(tokens, n, slots > 0 ? slots : 1);
    }
    const OverlapArgs none = {};
    switch (tile_n) {
        case 256:
            return launch_gemm_pair_bn<256, 0, 0>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, dev, none,
                                                  pdl);
        case 240:
            return launch_gemm_pair_bn<240, 0, 0>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, dev, none,
                                                  pdl);
        case 224:
            return launch_gemm_pair_bn<224, 0, 0>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, dev, none,
                                                  pdl);
        case 192:
            return launch_gemm_pair_bn<192, 0, 0>(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, dev, none,
                                                  pdl);
        default:
            return cudaErrorInvalidValue;
    }
}

cudaError_t launch_bf16_gemm_ex(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                                int32_t *status, cudaStream_t st, unsigned long long limit_ns, int stall_test) {
    return launch_bf16_gemm_cfg(X, W, Y, tokens, n, k, status, st, limit_ns, stall_test, -1, 0, false);
}

// The GEMM of aqlm_gemm, launched while the dequantisation before it in the
// stream still runs (programmatic dependent launch): its CTAs set up beside
// the dequantisation's, and its TMA producer waits for that grid before the
// first load.
cudaError_t launch_bf16_gemm_after_dequant(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n,
                                          int k, int32_t *status, cudaStream_t st) {
    return launch_bf16_gemm_cfg(X, W, Y, tokens, n, k, status, st, kGemmWaitLimitNs, 0, -1, 0, true);
}

// ---- prefill with the dequantisation overlapped (CTA pairs) ----
size_t overlap_counter_bytes(int d_out, int d_in) {
    const long long bands = (d_out + 191) / 192;               // the narrowest tile has the most bands
    const long long kb_pad = ((d_in + BK - 1) / BK + 31) / 32 * 32;
    return kClaimBytes + (size_t)((bands * kb_pad * 4 + 255) / 256 * 256);
}

namespace {
template <int BN, int FM, int FB>
cudaError_t launch_overlap_bn(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                              const uint16_t *X, uint16_t *W, uint16_t *Y, int tokens, const Dims &d,
                              int32_t *status, void *counters, cudaStream_t st, int dev) {
    OverlapArgs oa = {};
    oa.codes = static_cast<const uint8_t *>(codes);
    oa.codebooks = reinterpret_cast<const uint4 *>(codebooks);
    oa.scales = reinterpret_cast<const __half *>(scales);
    oa.W = reinterpret_cast<uint4 *>(W);
    oa.next_claim = static_cast<uint32_t *>(counters);
    oa.panel_done = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(counters) + kClaimBytes);
    oa.d_out = d.d_out;
    oa.G = d.G;
    oa.row_bytes = d.row_bytes;
    oa.n_bands = (d.d_out + BN - 1) / BN;
    oa.num_kb = (d.d_in + BK - 1) / BK;
    oa.kb_pad = (oa.num_kb + kWindow - 1) / kWindow * kWindow;
    // The bands the first wave of tiles needs are decoded first, by the
    // dequantisation kernel on the whole GPU (a fraction of its full-layer
    // time); the GEMM, launched early behind it, then starts its MMAs at once
    // instead of waiting for the decoder warps' first panels, which decode
    // the remaining bands in the order the later waves need them.
    const int slots = pair_slots<BN, FM, FB>(dev);
    const long long tiles = pair_tiles(tokens, d.d_out, BN);
    const int pairs = slots < 1 ? 1 : (tiles < slots ? (int)tiles : slots);
    const int m_tiles = (tokens + kPairRows - 1) / kPairRows;
    const int gb = (pairs + m_tiles - 1) / m_tiles;
    oa.band0 = gb < oa.n_bands ? gb : oa.n_bands;
    oa.total_units = (uint32_t)(oa.n_bands - oa.band0) * (BN / 16) * (uint32_t)oa.num_kb;   // < 2^31
    const size_t bytes = kClaimBytes + (size_t)oa.n_bands * oa.kb_pad * 4;
    cudaError_t e = cudaMemsetAsync(counters, 0, bytes, st);
    if (e != cudaSuccess) return e;
    if (oa.band0 > 0) {
        Dims first = d;
        first.d_out = oa.band0 * BN < d.d_out ? oa.band0 * BN : d.d_out;
        e = launch_dequant(codes, codebooks, scales, W, first, st);
        if (e != cudaSuccess) return e;
    }
    return launch_gemm_pair_bn<BN, FM, FB>(X, W, Y, tokens, d.d_out, d.d_in, status, st, kGemmWaitLimitNs, 0, dev,
                                           oa, oa.band0 > 0);
}

template <int FM, int FB>
cudaError_t launch_overlap_fmt(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                               const uint16_t *X, uint16_t *W, uint16_t *Y, int tokens, const Dims &d,
                               int32_t *status, void *counters, cudaStream_t st) {
    int dev = 0;
    cudaGetDevice(&dev);
    const int slots = pair_slots<240, FM, FB>(dev);
    switch (gemm_pair_tile_n(tokens, d.d_out, slots > 0 ? slots : 1)) {
        case 240:
            return launch_overlap_bn<240, FM, FB>(codes, codebooks, scales, X, W, Y, tokens, d, status, counters, st, dev);
        case 224:
            return launch_overlap_bn<224, FM, FB>(codes, codebooks, scales, X, W, Y, tokens, d, status, counters, st, dev);
        case 192:
            return launch_overlap_bn<192, FM, FB>(codes, codebooks, scales, X, W, Y, tokens, d, status, counters, st, dev);
        default:
            return launch_overlap_bn<256, FM, FB>(codes, codebooks, scales, X, W, Y, tokens, d, status, counters, st, dev);
    }
}
}  // namespace

// Whether the one-kernel prefill beats dequantisation + GEMM for a layer
// (measured on B200, 2048 tokens): always for two 16-bit codebooks (their
// dequantisation is the longest: 4096x11008 180.2 vs 190.5 us), otherwise when
// the bands the first wave of tiles needs -- decoded before the kernel -- are
// at most a third of the layer (1x16 11008x4096 161.9 vs 165.9 us; with 10 of
// 18 bands first, 4096x11008 lost: 167.9 vs 163.8 us).
bool overlap_preferred(const Dims &d, int tokens) {
    if (!gemm_uses_pair(tokens)) return false;
    if (d.M == 2 && d.B == 16) return true;
    int dev = 0;
    cudaGetDevice(&dev);
    const int slots = d.M == 1 ? pair_slots<240, 1, 16>(dev) : pair_slots<240, 2, 8>(dev);
    const int bn = gemm_pair_tile_n(tokens, d.d_out, slots > 0 ? slots : 1);
    const long long tiles = pair_tiles(tokens, d.d_out, bn);
    const int pairs = slots < 1 ? 1 : (tiles < slots ? (int)tiles : slots);
    const int m_tiles = (tokens + kPairRows - 1) / kPairRows;
    const long long band0 = (pairs + m_tiles - 1) / m_tiles;
    const long long n_bands = (d.d_out + bn - 1) / bn;
    return 3 * band0 <= n_bands;
}

// Y = X . W^T with W^ decoded into W (d_out x d_in bf16) by the GEMM's own
// decoder warps; counters: overlap_counter_bytes(d_out, d_in) bytes.
cudaError_t launch_overlap_gemm(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                                const uint16_t *X, uint16_t *W, uint16_t *Y, int tokens, const Dims &d,
                                int32_t *status, void *counters, cudaStream_t st) {
    if (d.M == 1) return launch_overlap_fmt<1, 16>(codes, codebooks, scales, X, W, Y, tokens, d, status, counters, st);
    if (d.B == 8) return launch_overlap_fmt<2, 8>(codes, codebooks, scales, X, W, Y, tokens, d, status, counters, st);
    return launch_overlap_fmt<2, 16>(codes, codebooks, scales, X, W, Y, tokens, d, status, counters, st);
}

// Prefill with the dequantisation fused into the GEMM (no W^ in global memory).
cudaError_t launch_fused_gemm(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                              const uint16_t *X, uint16_t *Y, int tokens, const Dims &d, int32_t *status,
                              cudaStream_t st) {
    DecodeArgs da;
    da.codes = static_cast<const uint8_t *>(codes);
    da.codebooks = reinterpret_cast<const uint4 *>(codebooks);
    da.scales = reinterpret_cast<const __half *>(scales);
    da.G = d.G;
    da.row_bytes = d.row_bytes;
    if (d.M == 1) return launch_by_width<1, 16>(X, nullptr, Y, tokens, d.d_out, d.d_in, status, st, kGemmWaitLimitNs, 0, da);
    if (d.B == 8) return launch_by_width<2, 8>(X, nullptr, Y, tokens, d.d_out, d.d_in, status, st, kGemmWaitLimitNs, 0, da);
    return launch_by_width<2, 16>(X, nullptr, Y, tokens, d.d_out, d.d_in, status, st, kGemmWaitLimitNs, 0, da);
}

cudaError_t launch_bf16_gemm(const uint16_t *X, const uint16_t *W, uint16_t *Y, int tokens, int n, int k,
                             int32_t *status, cudaStream_t st) {
    return launch_bf16_gemm_ex(X, W, Y, tokens, n, k, status, st, kGemmWaitLimitNs, 0);
}

AQLM_DEFINE_BOUNDS_READER(bounds_word_gemm)

}  // namespace aqlm
