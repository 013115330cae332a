// gemv_lut.cu -- batch-1 2x8 layer product through per-group lookup tables.
//
// "The AQLM Quantization Algorithm, Explained", section "What is
// Multi-Codebook Quantization (MCQ)?": a group's weights are
// C_0[b0] + C_1[b1] scaled by the row's scale, so by linearity
//   < C_0[b0] + C_1[b1], x_j > = L_0[j][b0] + L_1[j][b1],
//   L_m[j][k] = < C_m[k], x_j >,
// and with two codebooks of 256 codewords the 512 dot products of an input
// group are cheaper to tabulate once per CTA than to recompute for every
// row.  The row sum is then two table lookups per group (section "Key AQLM
// quantization parameters": 2x8 has 512 codewords in total).
//
// Layout: a CTA covers a slab of 32 consecutive groups (lane l <-> group
// j0 + l) and a range of rows.  Its tables L_m[j0 + l][k] live in shared
// memory at word (m * 256 + k) * 32 + l, i.e. in bank l, so the 32 lanes of a
// warp look up 32 different banks whatever their codes are: no bank
// conflicts.  Each warp streams batches of 8 rows (lane l copies 16 bytes =
// 8 groups of row r0 + l/4) through an 8-deep ring of asynchronous copies
// (cp.async) in shared memory, so 64 KiB of codes per CTA are in flight;
// it reads back its own group's two code bytes per row, looks up and adds; a
// 5-step butterfly then reduces the 8 row partials over the 32 lanes.  Slabs of one row
// range publish fp32 partial sums to the caller's workspace; the last CTA of
// the row range to arrive (atomic counter, no waiting) adds them in slab
// order (deterministic), scales by s_i, rounds to fp16 and resets the
// counter.  Programmatic dependent launch: codes and codebooks (constant
// weights) are loaded before griddepcontrol.wait, x after it.
#include "common.cuh"

namespace aqlm {
namespace {

constexpr int kSlab = 32;        // groups per slab, one per lane
constexpr int kLutWarps = 16;
constexpr int kLutThreads = kLutWarps * 32;
constexpr int kRowsPerBatch = 8;  // rows a warp stages at once (32 lanes x 16 bytes)
constexpr int kStages = 8;        // batches in flight per warp (cp.async ring)
constexpr size_t kLutSmem = (size_t)2 * 256 * kSlab * 4    // tables
                            + (size_t)2 * 256 * 8 * 4      // codebooks as fp32
                            + (size_t)kLutWarps * kStages * 32 * 16;  // code ring

struct LutArgs {
    const uint8_t *codes;
    const __half *codebooks;
    const __half *scales;
    const __half *x;
    __half *y;
    float *partial;      // [n_slabs][d_out]
    uint32_t *counters;  // [row chunks], zero between calls
    int d_out, G, row_bytes, rows_per_chunk;
};

__device__ __forceinline__ void gd_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// 16-byte asynchronous global -> shared copy; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void gd_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

__global__ void __launch_bounds__(kLutThreads) gemv_lut_2x8_kernel(const LutArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    float *lut = reinterpret_cast<float *>(smem);               // [2][256][32]
    float *cbf = lut + 2 * 256 * kSlab;                          // [2][256][8]
    uint4 *ring = reinterpret_cast<uint4 *>(cbf + 2 * 256 * 8);  // [warps][stages][32] uint4
    __shared__ int s_last;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slab = blockIdx.x, n_slabs = gridDim.x;
    const int j0 = slab * kSlab;
    const int row_begin = blockIdx.y * a.rows_per_chunk;
    const int row_end = min(a.d_out, row_begin + a.rows_per_chunk);

    // This lane's 16-byte piece of a warp batch: row r0 + lane/4, groups
    // j0 + 8*(lane%4) .. +7.  Pieces past the row's end or past the last row
    // are zero-filled instead of loaded.
    const int piece_row = lane >> 2;
    const int piece_group = j0 + 8 * (lane & 3);
    const bool piece_in_row = piece_group < a.G;
    uint4 *wring = ring + (size_t)warp * kStages * 32;
    auto issue = [&](int batch, int slot) {
        const int r = row_begin + (batch * kLutWarps + warp) * kRowsPerBatch + piece_row;
        const bool ok = r < row_end && piece_in_row;
        const uint8_t *src = ok ? a.codes + (size_t)r * a.row_bytes + (size_t)piece_group * 2 : a.codes;
        cp_async16(wring + slot * 32 + lane, src, ok ? 16u : 0u);
        cp_async_commit();
    };
    const int rows = row_end - row_begin;
    const int n_batches = (rows + kLutWarps * kRowsPerBatch - 1) / (kLutWarps * kRowsPerBatch);
    // codes are constant weights: fill the ring before waiting on x's producer
#pragma unroll
    for (int b = 0; b < kStages; ++b) issue(b, b);

    // codebooks (constant weights) -> fp32 in shared memory
    for (int i = threadIdx.x; i < 2 * 256; i += kLutThreads) {
        float f[8];
        half8_to_float8(reinterpret_cast<const uint4 *>(a.codebooks)[i], f);
        float4 *dst = reinterpret_cast<float4 *>(cbf + i * 8);
        dst[0] = make_float4(f[0], f[1], f[2], f[3]);
        dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    }

    gd_wait();
    // this lane's activation group (zeros past the end of the row)
    float xv[8];
    if (j0 + lane < a.G) {
        half8_to_float8(*reinterpret_cast<const uint4 *>(a.x + (size_t)(j0 + lane) * kGroup), xv);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) xv[e] = 0.f;
    }
    __syncthreads();
    // L_m[j0 + lane][k] for the (m, k) pairs of this warp
    for (int p = warp; p < 2 * 256; p += kLutWarps) {
        const float4 c0 = reinterpret_cast<const float4 *>(cbf + p * 8)[0];
        const float4 c1 = reinterpret_cast<const float4 *>(cbf + p * 8)[1];
        float d = c0.x * xv[0];
        d = fmaf(c0.y, xv[1], d);
        d = fmaf(c0.z, xv[2], d);
        d = fmaf(c0.w, xv[3], d);
        d = fmaf(c1.x, xv[4], d);
        d = fmaf(c1.y, xv[5], d);
        d = fmaf(c1.z, xv[6], d);
        d = fmaf(c1.w, xv[7], d);
        lut[p * kSlab + lane] = d;
    }
    __syncthreads();
    gd_launch();

    const float *lut0 = lut + lane;
    const float *lut1 = lut + 256 * kSlab + lane;
    for (int b = 0; b < n_batches; ++b) {
        const int slot = b % kStages;
        cp_async_wait<kStages - 1>();   // the batch in `slot` has landed
        __syncwarp();
        const uint16_t *codes16 = reinterpret_cast<const uint16_t *>(wring + slot * 32);
        float v[kRowsPerBatch];
#pragma unroll
        for (int q = 0; q < kRowsPerBatch; ++q) {
            const uint32_t code = codes16[q * kSlab + lane];  // byte 2l: codebook 0, byte 2l+1: codebook 1
            v[q] = lut0[(code & 0xffu) * kSlab] + lut1[(code >> 8) * kSlab];
        }
        __syncwarp();
        issue(b + kStages, slot);   // refill the slot (zero-filled past the end)
        // butterfly: lane bits 4,3,2 select the row, the 4 lanes of a quad end
        // up with the full sum of row r0 + lane/4
        float u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool hi = lane & 16;
            const float send = hi ? v[i] : v[i + 4];
            const float keep = hi ? v[i + 4] : v[i];
            u[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
        }
        float w2[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const bool hi = lane & 8;
            const float send = hi ? u[i] : u[i + 2];
            const float keep = hi ? u[i + 2] : u[i];
            w2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
        const bool hi4 = lane & 4;
        float z = (hi4 ? w2[1] : w2[0]) + __shfl_xor_sync(0xffffffffu, hi4 ? w2[0] : w2[1], 4);
        z += __shfl_xor_sync(0xffffffffu, z, 2);
        z += __shfl_xor_sync(0xffffffffu, z, 1);
        const int r = row_begin + (b * kLutWarps + warp) * kRowsPerBatch + (lane >> 2);
        if ((lane & 3) == 0 && r < row_end) {
            if (n_slabs == 1) {
                a.y[r] = __float2half_rn(z * __half2float(a.scales[r]));
            } else {
                a.partial[(size_t)slab * a.d_out + r] = z;
            }
        }
    }
    cp_async_wait<0>();   // nothing may still be landing in shared memory at exit
    if (n_slabs == 1) return;

    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(&a.counters[blockIdx.y], 1u);
        s_last = (prev == (uint32_t)(n_slabs - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // 16 partials in flight per thread, added in slab order
    for (int r = row_begin + threadIdx.x; r < row_end; r += kLutThreads) {
        float sum = 0.f;
        for (int s0 = 0; s0 < n_slabs; s0 += 16) {
            float v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                v[u] = (s0 + u < n_slabs) ? __ldcg(&a.partial[(size_t)(s0 + u) * a.d_out + r]) : 0.f;
#pragma unroll
            for (int u = 0; u < 16; ++u) sum += v[u];
        }
        a.y[r] = __float2half_rn(sum * __half2float(a.scales[r]));
    }
    if (threadIdx.x == 0) a.counters[blockIdx.y] = 0u;
}

struct LutPlan {
    int n_slabs, row_chunks, rows_per_chunk;
};

LutPlan plan_lut(const Dims &d, int sms) {
    LutPlan p;
    p.n_slabs = (d.G + kSlab - 1) / kSlab;
    // about one CTA per SM: every CTA builds its slab's 16384-entry table once
    int chunks = sms / p.n_slabs;
    if (chunks < 1) chunks = 1;
    const int max_chunks = (d.d_out + kRowsPerBatch - 1) / kRowsPerBatch;
    if (chunks > max_chunks) chunks = max_chunks;
    int rpc = (d.d_out + chunks - 1) / chunks;
    rpc = (rpc + kRowsPerBatch - 1) / kRowsPerBatch * kRowsPerBatch;
    p.rows_per_chunk = rpc;
    p.row_chunks = (d.d_out + rpc - 1) / rpc;
    return p;
}

inline size_t align16(size_t v) { return (v + 15) / 16 * 16; }

}  // namespace

size_t gemv_lut_workspace_bytes(const Dims &d, int sms) {
    const LutPlan p = plan_lut(d, sms);
    if (p.n_slabs == 1) return 0;
    return align16((size_t)p.n_slabs * d.d_out * sizeof(float)) + (size_t)p.row_chunks * sizeof(uint32_t);
}

// Offset of the arrival counters (the part that must be zero before a call).
size_t gemv_lut_workspace_counter_offset(const Dims &d, int sms) {
    const LutPlan p = plan_lut(d, sms);
    if (p.n_slabs == 1) return 0;
    return align16((size_t)p.n_slabs * d.d_out * sizeof(float));
}

cudaError_t launch_gemv_lut_2x8(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                                const uint16_t *x, uint16_t *y, const Dims &d, void *workspace, int sms,
                                cudaStream_t st) {
    const LutPlan p = plan_lut(d, sms);
    cudaError_t e = cudaFuncSetAttribute(gemv_lut_2x8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kLutSmem);
    if (e != cudaSuccess) return e;
    LutArgs a;
    a.codes = static_cast<const uint8_t *>(codes);
    a.codebooks = reinterpret_cast<const __half *>(codebooks);
    a.scales = reinterpret_cast<const __half *>(scales);
    a.x = reinterpret_cast<const __half *>(x);
    a.y = reinterpret_cast<__half *>(y);
    a.partial = static_cast<float *>(workspace);
    a.counters = p.n_slabs > 1 ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) +
                                                              align16((size_t)p.n_slabs * d.d_out * sizeof(float)))
                               : nullptr;
    a.d_out = d.d_out;
    a.G = d.G;
    a.row_bytes = d.row_bytes;
    a.rows_per_chunk = p.rows_per_chunk;
    return launch_kernel(gemv_lut_2x8_kernel, dim3(p.n_slabs, p.row_chunks), dim3(kLutThreads), kLutSmem, st,
                         true, a);
}

}  // namespace aqlm
