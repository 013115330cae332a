// gemv_lut.cu -- 2x8 layer product for one token through lookup tables.
//
// "The AQLM Quantization Algorithm, Explained", section "What is
// Multi-Codebook Quantization (MCQ)?": y_i = s_i * sum_j < C_0[b(i,j,0)] +
// C_1[b(i,j,1)], x_j >.  The product is linear in the codewords, so
//   < C_0[b0] + C_1[b1], x_j > = L_0[j][b0] + L_1[j][b1],
//   L_m[j][k] = < C_m[k], x_j >,
// and with 2x8's 2 x 256 codewords a table of all L_m[j][k] for a slab of
// 32 groups is 64 KiB: a decode product becomes two 4-byte table lookups per
// group instead of two 16-byte codeword gathers and eight multiply-adds.
//
// Design (one token, the decode step):
//   - The input groups are cut into slabs of 32 (lane l of every warp owns
//     group l of the slab), the slabs into slab groups of S, the rows into
//     ranges.  CTA (slab group, range) takes its slabs one after the other:
//     it builds the slab's table in shared memory, then looks up every row of
//     its range.  S is chosen per shape (host planner below): one slab per
//     CTA where the rows are few, more where many slabs per row would make
//     the final reduction long.
//   - Table layout [m][k][lane], 4 bytes each: lane l only ever reads bank l,
//     so a warp's 32 lookups take one shared-memory wavefront whatever the
//     codes are.  Building it: warp w computes the entries of codewords w,
//     w + 16, ... for all 32 groups (each lane its own group's dot product:
//     eight exact fp16 x fp16 products summed in fp32), one conflict-free
//     4-byte store per codeword and warp.
//   - The slab's codes (64 bytes per row) stream through a ring of NS chunks
//     of 128 rows in shared memory, copied by cp.async (16 bytes per thread
//     and chunk, L2 only); the first chunks are requested before the
//     grid-dependency wait.  cp.async completion is waited for per thread
//     (cp.async.wait_group), then a CTA barrier: no wait here can hang.
//   - Rows in batches of 8 per warp (a chunk is one batch per warp): each
//     lane adds its group's two table entries per row, and the warp reduces
//     the 8 rows' 32 lane values with 9 shuffles (a butterfly that halves the
//     rows at each step, then the remaining lane pairs), leaving row l & 7's
//     sum in lanes l, l + 8, l + 16, l + 24.
//   - Each CTA adds its slabs' row sums (in shared memory across slabs) and
//     writes them to the workspace; the last CTA of a row range to arrive (an
//     atomic counter, no waiting) adds the slab groups' sums in order, scales,
//     rounds once to fp16 and resets the counter.
//   - Programmatic dependent launch: codebooks and the first code chunks come
//     before griddepcontrol.wait (weights are constant); x is read, and the
//     workspace and y are written, only after it.
// Arithmetic: every table entry is an fp32 sum of eight exact products, every
// row the fp32 sum of its entries in a fixed order (lane pairs, the shuffle
// butterfly, slabs in order, slab groups in order), so results are
// reproducible bit for bit; they differ from the row kernel's by fp32
// rounding only.
#include "common.cuh"

namespace aqlm {
namespace {

constexpr int kLutWarps = 16;
constexpr int kLutThreads = kLutWarps * 32;
constexpr int kSlab = 32;                      // groups per slab (one per lane)
constexpr int kCodewords = 2 * 256;            // both 2x8 codebooks
constexpr int kBatch = 16;                     // rows per warp batch
constexpr int kChunkRows = kBatch * kLutWarps; // 256 rows per code chunk
constexpr int kChunkBytes = kChunkRows * kSlab * 2;   // 16 KiB: 64 bytes of codes per row
constexpr int kCopies = kChunkBytes / 16 / kLutThreads;   // 16-byte copies per thread and chunk
static_assert(kCopies * 16 * kLutThreads == kChunkBytes, "whole 16-byte copies per thread");
constexpr int kRing = 6;                       // chunks in the ring (5 in flight: 80 KiB)
constexpr size_t kTableBytes = (size_t)kCodewords * kSlab * sizeof(float);   // 64 KiB
constexpr size_t kCbBytes = (size_t)kCodewords * 8 * sizeof(float);          // 16 KiB, fp32 copy
constexpr size_t kLutFixedSmem = kTableBytes + kCbBytes + (size_t)kRing * kChunkBytes;
constexpr size_t kMaxRowAcc = 24 * 1024;       // fp32 row sums across slabs (S > 1)

struct LutArgs {
    const uint8_t *codes;      // [d_out][G][2] uint8
    const uint4 *codebooks;    // [2][256] codewords of 8 fp16
    const __half *scales;      // [d_out]
    const __half *x;           // [d_in]
    __half *y;                 // [d_out]
    float *partial;            // [n_groups][d_out]
    uint32_t *counters;        // [n_ranges], zero between calls
    int d_out, G, row_bytes;
    int n_slabs;               // slabs of the row, ceil(G / 32)
    int slabs_per_cta;         // S
    int n_groups;              // slab groups, ceil(n_slabs / S)
    int n_ranges;
};

// 16-byte asynchronous copy global -> shared (L2 only); src_bytes = 0 writes
// 16 zero bytes and reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kLutThreads, 1) gemv_lut_kernel(const LutArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    float *lut = reinterpret_cast<float *>(smem);                                   // [m*256 + k][lane]
    float4 *cbs = reinterpret_cast<float4 *>(smem + kTableBytes);                   // [m*256 + k][2]
    unsigned char *ring = smem + kTableBytes + kCbBytes;                            // [kRing][256 rows][64 B]
    float *rowacc = reinterpret_cast<float *>(smem + kLutFixedSmem);                // [rows of the range], S > 1
    __shared__ int s_last;
    const int grp = blockIdx.x, q = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = (int)((int64_t)q * a.d_out / a.n_ranges);
    const int r1 = (int)((int64_t)(q + 1) * a.d_out / a.n_ranges);
    const int n_chunks = (r1 - r0 + kChunkRows - 1) / kChunkRows;
    const int slab0 = grp * a.slabs_per_cta;
    const int slab1 = min(a.n_slabs, slab0 + a.slabs_per_cta);
    const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);

    // Copies of the next (slab, chunk) step into the ring, in step order; rows
    // past the range and groups past the row read nothing and land as zeros.
    int is = slab0, ic = 0, islot = 0;
    auto issue = [&]() {
        if (is < slab1) {
#pragma unroll
            for (int k = 0; k < kCopies; ++k) {
                const int piece = threadIdx.x + k * kLutThreads;
                const int r = r0 + ic * kChunkRows + (piece >> 2);
                const int g = is * kSlab + (piece & 3) * 8;      // first group of this 16-byte piece
                const bool in = r < r1 && g < a.G;
                const bool ok = AQLM_IN_BOUNDS(islot < kRing && piece * 16 < kChunkBytes && (!in || r < a.d_out),
                                               kSiteLutRing, piece);
                cp_async16(ring_s + (uint32_t)((ok ? islot : 0) * kChunkBytes + (ok ? piece : 0) * 16),
                           in && ok ? a.codes + (size_t)r * a.row_bytes + (size_t)g * 2 : a.codes, in && ok ? 16u : 0u);
            }
            if (++ic == n_chunks) {
                ic = 0;
                ++is;
            }
            if (++islot == kRing) islot = 0;
        }
        cp_async_commit();   // an empty group where nothing was copied keeps the count uniform
    };

    // ---- weights only, before the grid-dependency wait ---------------------
    for (int i = threadIdx.x; i < kCodewords; i += kLutThreads) {
        float f[8];
        half8_to_float8(a.codebooks[i], f);
        cbs[2 * i] = make_float4(f[0], f[1], f[2], f[3]);
        cbs[2 * i + 1] = make_float4(f[4], f[5], f[6], f[7]);
    }
#pragma unroll
    for (int i = 0; i < kRing - 1; ++i) issue();
    grid_dep_launch();
    grid_dep_wait();

    const float *lut0 = lut + lane;
    const float *lut1 = lut + 256 * kSlab + lane;
    const unsigned short *ring_u16 = reinterpret_cast<const unsigned short *>(ring) + lane;
    const bool multi = a.slabs_per_cta > 1;
    int slot = 0;
    for (int s = slab0; s < slab1; ++s) {
        // ---- the slab's tables ---------------------------------------------
        float xf[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (s * kSlab + lane < a.G)                         // the last slab may be narrower
            half8_to_float8(*reinterpret_cast<const uint4 *>(a.x + (size_t)(s * kSlab + lane) * kGroup), xf);
        const float2 x01 = make_float2(xf[0], xf[1]), x23 = make_float2(xf[2], xf[3]);
        const float2 x45 = make_float2(xf[4], xf[5]), x67 = make_float2(xf[6], xf[7]);
        __syncthreads();  // codebook copy complete; the previous slab's lookups done
#pragma unroll 4
        for (int c = warp; c < kCodewords; c += kLutWarps) {
            const float4 lo = cbs[2 * c], hi = cbs[2 * c + 1];
            float2 eo = __fmul2_rn(make_float2(lo.x, lo.y), x01);
            eo = __ffma2_rn(make_float2(lo.z, lo.w), x23, eo);
            eo = __ffma2_rn(make_float2(hi.x, hi.y), x45, eo);
            eo = __ffma2_rn(make_float2(hi.z, hi.w), x67, eo);
            lut[c * kSlab + lane] = eo.x + eo.y;
        }
        // ---- lookups: the slab's chunks, one 16-row batch per warp each -----
        for (int c = 0; c < n_chunks; ++c) {
            cp_async_wait<kRing - 2>();   // this thread's copies of this step landed
            __syncthreads();              // everyone's; the table is complete; the oldest slot is free
            issue();
            const unsigned short *codes_s = ring_u16 + slot * (kChunkBytes / 2) + warp * kBatch * kSlab;
            if (++slot == kRing) slot = 0;
            float v[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                const uint32_t code = codes_s[i * kSlab];
                v[i] = AQLM_IN_BOUNDS(code < 65536u, kSiteLutTable, code)
                           ? lut0[(code & 0xffu) * kSlab] + lut1[(code >> 8) * kSlab]
                           : 0.f;
            }
            // butterfly over the 16 rows: after the step of offset o, v[0..o) hold
            // rows (lane & o ? o..2o : 0..o) of the current half, summed over the lane pair
#pragma unroll
            for (int o = kBatch / 2; o >= 1; o >>= 1) {
                const bool upper = (lane & o) != 0;
#pragma unroll
                for (int i = 0; i < o; ++i) {
                    const float send = upper ? v[i] : v[i + o];
                    const float keep = upper ? v[i + o] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], 16);   // lanes l and l ^ 16 hold row l & 15
            const int rr = c * kChunkRows + warp * kBatch + lane;   // row from r0; lanes 0..15 write
            if (lane < kBatch && r0 + rr < r1 && AQLM_IN_BOUNDS(r1 <= a.d_out && grp < a.n_groups, kSiteLutY, r0 + rr)) {
                if (multi) {
                    rowacc[rr] = (s == slab0 ? 0.f : rowacc[rr]) + v[0];
                } else if (a.n_groups == 1) {
                    a.y[r0 + rr] = __float2half_rn(v[0] * __half2float(a.scales[r0 + rr]));
                } else {
                    a.partial[(size_t)grp * a.d_out + r0 + rr] = v[0];
                }
            }
        }
    }
    cp_async_wait<0>();
    if (multi) {
        __syncthreads();
        for (int r = threadIdx.x; r < r1 - r0; r += kLutThreads) {
            if (a.n_groups == 1) {
                a.y[r0 + r] = __float2half_rn(rowacc[r] * __half2float(a.scales[r0 + r]));
            } else {
                a.partial[(size_t)grp * a.d_out + r0 + r] = rowacc[r];
            }
        }
    }
    if (a.n_groups == 1) return;

    // ---- the last CTA of the row range adds the slab groups in order ---------
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&a.counters[q], 1u) == (uint32_t)(a.n_groups - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int r = r0 + threadIdx.x; r < r1; r += kLutThreads) {
        float sum = 0.f;
        for (int g0 = 0; g0 < a.n_groups; g0 += 16) {  // 16 loads in flight, added in order
            float p[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                p[u] = g0 + u < a.n_groups ? __ldcg(&a.partial[(size_t)(g0 + u) * a.d_out + r]) : 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) sum += p[u];
        }
        a.y[r] = __float2half_rn(sum * __half2float(a.scales[r]));
    }
    if (threadIdx.x == 0) a.counters[q] = 0u;
}

struct LutPlan {
    int n_slabs, slabs_per_cta, n_groups, n_ranges, max_rows;
    size_t smem;
};

// Cost model in SM clocks (rates measured on B200): a slab's table, 512 x 32
// dot products of 8, takes about 1500 clocks; a row of a slab about 3
// (instruction issue of a code read, two lookups and the shuffle reduction);
// the final reduction costs a memory fence, an atomic and one L2 round trip
// per 16 loads in flight per thread (about 2000 clocks and 1400 per round).
// The plan fills the SMs with one wave of CTAs and picks the slab-group size
// S with the least modelled time.
LutPlan plan_lut(const Dims &d, int sms) {
    LutPlan best{};
    double best_t = 1e300;
    const int n_slabs = (d.G + kSlab - 1) / kSlab;
    for (int S = 1; S <= n_slabs; ++S) {
        const int groups = (n_slabs + S - 1) / S;
        if (S > 1 && (n_slabs + S - 2) / (S - 1) == groups) continue;   // same group count as a smaller S
        int R = sms / groups;
        if (R < 1) R = 1;
        const int max_r = (d.d_out + kBatch - 1) / kBatch;
        if (R > max_r) R = max_r;
        const int rows = (d.d_out + R - 1) / R;
        if (S > 1 && (size_t)rows * 4 > kMaxRowAcc) continue;
        const long long ctas = (long long)groups * R;
        const double waves = (double)((ctas + sms - 1) / sms);
        const double per_cta = S * (1500.0 + rows * 3.0);
        const double tail = groups > 1 ? 2000.0 + ((double)rows * groups / (kLutThreads * 16.0) + 1.0) * 1400.0 : 0.0;
        const double t = waves * per_cta + tail;
        if (t < best_t * 0.999) {
            best_t = t;
            best.n_slabs = n_slabs;
            best.slabs_per_cta = S;
            best.n_groups = groups;
            best.n_ranges = R;
            best.max_rows = rows;
        }
    }
    best.smem = kLutFixedSmem + (best.slabs_per_cta > 1 ? ((size_t)best.max_rows * 4 + 15) / 16 * 16 : 0);
    return best;
}

}  // namespace

bool gemv_lut_supported(const Dims &d, int T) { return T == 1 && d.M == 2 && d.B == 8; }

// Workspace: fp32 row sums [slab groups][d_out], then one arrival counter per
// row range (nothing when one slab group covers the row).
size_t gemv_lut_counter_offset(const Dims &d, int sms) {
    const LutPlan p = plan_lut(d, sms);
    if (p.n_groups == 1) return 0;
    return ((size_t)p.n_groups * d.d_out * sizeof(float) + 15) / 16 * 16;
}

size_t gemv_lut_workspace_bytes(const Dims &d, int sms) {
    const LutPlan p = plan_lut(d, sms);
    if (p.n_groups == 1) return 0;
    return gemv_lut_counter_offset(d, sms) + (size_t)p.n_ranges * sizeof(uint32_t);
}

cudaError_t launch_gemv_lut(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                            uint16_t *y, const Dims &d, void *workspace, int sms, cudaStream_t st) {
    const LutPlan p = plan_lut(d, sms);
    LutArgs a;
    a.codes = static_cast<const uint8_t *>(codes);
    a.codebooks = reinterpret_cast<const uint4 *>(codebooks);
    a.scales = reinterpret_cast<const __half *>(scales);
    a.x = reinterpret_cast<const __half *>(x);
    a.y = reinterpret_cast<__half *>(y);
    a.partial = static_cast<float *>(workspace);
    a.counters = p.n_groups > 1 ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) +
                                                               gemv_lut_counter_offset(d, sms))
                                : nullptr;
    a.d_out = d.d_out;
    a.G = d.G;
    a.row_bytes = d.row_bytes;
    a.n_slabs = p.n_slabs;
    a.slabs_per_cta = p.slabs_per_cta;
    a.n_groups = p.n_groups;
    a.n_ranges = p.n_ranges;
    const cudaError_t e = opt_in_dynamic_smem(gemv_lut_kernel, p.smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(gemv_lut_kernel, dim3(p.n_groups, p.n_ranges), dim3(kLutThreads), p.smem, st, true, a);
}

AQLM_DEFINE_BOUNDS_READER(bounds_word_lut)

}  // namespace aqlm
