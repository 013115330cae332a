// encode.cu -- the step before inference: scales, codebooks and codes of a
// layer from its weights.
//
// "The AQLM Quantization Algorithm, Explained", section "AQLM quantization
// process": the codes are learned with the codebooks and scales fixed, the
// codebooks having been initialised "with a residual k-means approach";
// section "What is Multi-Codebook Quantization (MCQ)?": output channels are
// scaled, cut into groups of 8 and each group approximated by the sum of M
// codewords.  The pages give no loss, search or update rule beyond that, so
// every step here is a stated reading of what is computed:
//   scales     the row's root mean square rounded to fp16 (1.0 if that is 0);
//   groups     the row's inputs divided by its scale (binary32 division);
//   nearest    least squared Euclidean distance |v - c|^2, ties to the lowest
//              index;
//   k-means    Lloyd updates: a centroid is the mean of its groups (sums in
//              double), an empty one keeps its value; codebook m is k-means
//              of the residuals left by codebooks 0..m-1, started from the
//              residuals that init_idx names;
//   codes      greedy, codebook by codebook: the nearest codeword of the
//              residual, which then loses that codeword.
// How each is evaluated here (any order meets the same error bounds):
//   scales     the sum of squares in double, lane l of a warp summing inputs
//              l, l+32, ... in order, then a butterfly of shuffles; the
//              binary16 result can differ from a sequential sum's only where
//              the root mean square lies within (d_in + 4) 2^-53 of a
//              binary16 rounding boundary;
//   nearest    ranked by the binary32 score |c|^2 - 2<v, c> (|v|^2 is common
//              to every codeword): each of |c|^2 and <v, c> is the sum of two
//              fused multiply-add chains (lanes 0,2,4,6 and 1,3,5,7, one packed
//              fp32x2 chain), then score = fma(-2, <v, c>, |c|^2).  Its error
//              is at most gamma_9 (|c|^2 + 2 sum_t |v_t c_t|) (u = 2^-24), so
//              the chosen codeword is the exact nearest one unless another lies
//              within twice that of it.  The distance reported for the winner
//              is the same two-chain sum of the squared differences.
//
// The nearest-codeword search is the expensive step (every group against
// every codeword: 2^16 for 1x16) and runs on the CUDA cores in binary32:
// deterministic, with the error bound above.  (On the tensor cores the dot
// products would be tf32 with an accumulation order the hardware does not
// document, and the bound could not be stated.)  Each thread keeps four
// groups in registers and streams the codebook, with each codeword's |c|^2,
// through shared memory; a CTA covers 1024 groups and a range of codewords,
// and the ranges' winners meet through a 64-bit atomic minimum of
// (key(score) << 32 | index), key the order-preserving map of a float onto
// the unsigned integers: equal scores fall to the lower index, exactly the
// tie rule.
#include "common.cuh"

namespace aqlm {
namespace {

constexpr int kNearThreads = 256;
constexpr int kNearPerThread = 4;                           // groups per thread
constexpr int kNearGroups = kNearThreads * kNearPerThread;  // groups per CTA
constexpr int kNearChunk = 512;                             // codewords per shared-memory chunk

// ---- scales and groups ------------------------------------------------------

// One warp per row.
__global__ void __launch_bounds__(256) encode_scales_kernel(const float *__restrict__ W, int d_out, int d_in,
                                                            __half *__restrict__ scales, float *__restrict__ V) {
    const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (row >= d_out) return;
    const float *w = W + (size_t)row * d_in;
    double acc = 0.0;
    for (int k = lane; k < d_in; k += 32) {
        const double v = (double)w[k];
        acc = __dadd_rn(acc, __dmul_rn(v, v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc = __dadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, o));
    const double rms = sqrt(__ddiv_rn(acc, (double)d_in));
    __half h = __double2half(rms);
    if ((__half_as_ushort(h) & 0x7fffu) == 0) h = __float2half(1.0f);
    if (lane == 0) scales[row] = h;
    const float s = __half2float(h);
    float *v = V + (size_t)row * d_in;
    for (int k = lane; k < d_in; k += 32) v[k] = __fdiv_rn(w[k], s);
}

// ---- nearest codeword -------------------------------------------------------

// Order-preserving key of a finite float: sign bit flipped for x >= 0, every
// bit flipped for x < 0 (-0 is taken as +0, so equal values share a key).
__device__ __forceinline__ unsigned long long pack_best(float s, int k) {
    const uint32_t b = __float_as_uint(s == 0.0f ? 0.0f : s);
    const uint32_t key = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
    return ((unsigned long long)key << 32) | (unsigned int)k;
}

// |c|^2 in the pattern of the score: even and odd lanes as fma chains, e + o.
__device__ __forceinline__ float norm2(const float4 a, const float4 b) {
    float e = __fmul_rn(a.x, a.x), o = __fmul_rn(a.y, a.y);
    e = __fmaf_rn(a.z, a.z, e);
    o = __fmaf_rn(a.w, a.w, o);
    e = __fmaf_rn(b.x, b.x, e);
    o = __fmaf_rn(b.y, b.y, o);
    e = __fmaf_rn(b.z, b.z, e);
    o = __fmaf_rn(b.w, b.w, o);
    return __fadd_rn(e, o);
}

// best[n] = min over codewords k in this CTA's range of pack(score, k).
// Codebook C [K][8] fp32; the CTA's range is [k_begin, k_end).
__global__ void __launch_bounds__(kNearThreads) nearest_kernel(const float *__restrict__ V, long long N,
                                                               const float *__restrict__ C, int K, int k_per_cta,
                                                               unsigned long long *__restrict__ best) {
    __shared__ float4 cs[kNearChunk][2];
    __shared__ float cc[kNearChunk];  // |c|^2
    const long long n0 = (long long)blockIdx.x * kNearGroups + threadIdx.x;
    const int k_begin = blockIdx.y * k_per_cta;
    const int k_end = min(K, k_begin + k_per_cta);
    float2 v[kNearPerThread][4];
    float bd[kNearPerThread];
    int bk[kNearPerThread];
#pragma unroll
    for (int p = 0; p < kNearPerThread; ++p) {
        const long long n = n0 + (long long)p * kNearThreads;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
        if (n < N) {
            a = reinterpret_cast<const float4 *>(V)[2 * n];
            b = reinterpret_cast<const float4 *>(V)[2 * n + 1];
        }
        v[p][0] = make_float2(a.x, a.y);
        v[p][1] = make_float2(a.z, a.w);
        v[p][2] = make_float2(b.x, b.y);
        v[p][3] = make_float2(b.z, b.w);
        bd[p] = __int_as_float(0x7f800000);  // +inf
        bk[p] = k_begin;
    }
    for (int c0 = k_begin; c0 < k_end; c0 += kNearChunk) {
        const int cn = min(kNearChunk, k_end - c0);
        __syncthreads();
        for (int i = threadIdx.x; i < cn; i += kNearThreads) {
            const float4 a = reinterpret_cast<const float4 *>(C)[2 * ((long long)c0 + i)];
            const float4 b = reinterpret_cast<const float4 *>(C)[2 * ((long long)c0 + i) + 1];
            cs[i][0] = a;
            cs[i][1] = b;
            cc[i] = norm2(a, b);
        }
        __syncthreads();
        for (int j = 0; j < cn; ++j) {
            const float4 a = cs[j][0], b = cs[j][1];
            const float n2 = cc[j];
            const float2 c01 = make_float2(a.x, a.y), c23 = make_float2(a.z, a.w);
            const float2 c45 = make_float2(b.x, b.y), c67 = make_float2(b.z, b.w);
#pragma unroll
            for (int p = 0; p < kNearPerThread; ++p) {
                // (even, odd) lanes of <v, c>, two fma chains
                float2 eo = __fmul2_rn(v[p][0], c01);
                eo = __ffma2_rn(v[p][1], c23, eo);
                eo = __ffma2_rn(v[p][2], c45, eo);
                eo = __ffma2_rn(v[p][3], c67, eo);
                const float s = __fmaf_rn(-2.0f, __fadd_rn(eo.x, eo.y), n2);
                if (s < bd[p]) {
                    bd[p] = s;
                    bk[p] = c0 + j;
                }
            }
        }
    }
#pragma unroll
    for (int p = 0; p < kNearPerThread; ++p) {
        const long long n = n0 + (long long)p * kNearThreads;
        if (n < N) atomicMin(&best[n], pack_best(bd[p], bk[p]));
    }
}

__global__ void fill_u64_kernel(unsigned long long *p, long long n, unsigned long long v) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        p[i] = v;
}

// idx[n] from the packed winners, and dist[n] = |v - c|^2 of the winner: the
// squared differences' even and odd lanes as fma chains, then e + o.
__global__ void unpack_best_kernel(const unsigned long long *__restrict__ best, long long N,
                                   const float *__restrict__ V, const float *__restrict__ C, int K,
                                   int32_t *__restrict__ idx, float *__restrict__ dist) {
    for (long long n = blockIdx.x * (long long)blockDim.x + threadIdx.x; n < N; n += (long long)gridDim.x * blockDim.x) {
        const uint32_t k = (uint32_t)(best[n] & 0xffffffffull);
        if (!AQLM_IN_BOUNDS(k < (uint32_t)K, kSiteNearest, n)) continue;
        if (idx) idx[n] = (int32_t)k;
        if (dist) {
            float d[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) d[t] = __fsub_rn(V[n * 8 + t], C[(long long)k * 8 + t]);
            float e = __fmul_rn(d[0], d[0]), o = __fmul_rn(d[1], d[1]);
#pragma unroll
            for (int t = 2; t < 8; t += 2) {
                e = __fmaf_rn(d[t], d[t], e);
                o = __fmaf_rn(d[t + 1], d[t + 1], o);
            }
            dist[n] = __fadd_rn(e, o);
        }
    }
}

// ---- k-means update -----------------------------------------------------------

// sums[k][t] += V[n][t] and counts[k] += 1 for idx[n] = k (fp64 atomics).
__global__ void kmeans_accumulate_kernel(const float *__restrict__ V, const int32_t *__restrict__ idx, long long N,
                                         int K, double *__restrict__ sums, unsigned int *__restrict__ counts) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < N * 8;
         i += (long long)gridDim.x * blockDim.x) {
        const long long n = i >> 3;
        const int t = (int)(i & 7);
        const int k = idx[n];
        if (k < 0 || k >= K) continue;  // the host validates nothing on the device: skip bad indices (by design,
                                        // not a bounds error: aqlm_kmeans_update documents that they are ignored)
        atomicAdd(&sums[(long long)k * 8 + t], (double)V[i]);
        if (t == 0) atomicAdd(&counts[k], 1u);
    }
}

__global__ void kmeans_finish_kernel(const double *__restrict__ sums, const unsigned int *__restrict__ counts, int K,
                                     const float *__restrict__ C_prev, float *__restrict__ C_out,
                                     int32_t *__restrict__ counts_out) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (long long)K * 8;
         i += (long long)gridDim.x * blockDim.x) {
        const unsigned int c = counts[i >> 3];
        C_out[i] = c ? __double2float_rn(__ddiv_rn(sums[i], (double)c)) : C_prev[i];
        if (counts_out && (i & 7) == 0) counts_out[i >> 3] = (int32_t)c;
    }
}

// ---- residual k-means and codes -----------------------------------------------

// C[k] = R[init[k]] (the indices were checked against N on the host).
__global__ void gather_rows_kernel(const float *__restrict__ R, const int32_t *__restrict__ init, int K,
                                   float *__restrict__ C) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (long long)K * 8;
         i += (long long)gridDim.x * blockDim.x)
        if (AQLM_IN_BOUNDS(init[i >> 3] >= 0, kSiteKmeans, i)) C[i] = R[(long long)init[i >> 3] * 8 + (i & 7)];
}

// R[n] -= C[best index of n]; optionally the index as the n-th code of codebook m.
__global__ void subtract_nearest_kernel(float *__restrict__ R, const unsigned long long *__restrict__ best,
                                        long long N, const float *__restrict__ C, int K, void *__restrict__ codes,
                                        int M, int m, int code_bytes) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < N * 8;
         i += (long long)gridDim.x * blockDim.x) {
        const long long n = i >> 3;
        const int t = (int)(i & 7);
        const uint32_t k = (uint32_t)(best[n] & 0xffffffffull);
        if (!AQLM_IN_BOUNDS(k < (uint32_t)K, kSiteEncode, n)) continue;
        R[i] = __fsub_rn(R[i], C[(long long)k * 8 + t]);
        if (codes && t == 0) {
            if (code_bytes == 1) {
                static_cast<uint8_t *>(codes)[n * M + m] = (uint8_t)k;
            } else {
                static_cast<uint16_t *>(codes)[n * M + m] = (uint16_t)k;
            }
        }
    }
}

__global__ void half_to_float_kernel(const __half *__restrict__ h, long long n, float *__restrict__ f) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        f[i] = __half2float(h[i]);
}

__global__ void float_to_half_kernel(const float *__restrict__ f, long long n, __half *__restrict__ h) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        h[i] = __float2half_rn(f[i]);
}

int device_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    return num_sms(dev);
}

int elementwise_grid(long long n) {
    const long long want = (n + 255) / 256;
    const long long cap = (long long)device_sms() * 8;
    return (int)(want < 1 ? 1 : (want > cap ? cap : want));
}

inline size_t al256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

// ---- launchers (host) -----------------------------------------------------------

cudaError_t launch_encode_scales(const float *W, int d_out, int d_in, uint16_t *scales, float *V, cudaStream_t st) {
    encode_scales_kernel<<<(d_out + 7) / 8, 256, 0, st>>>(W, d_out, d_in, reinterpret_cast<__half *>(scales), V);
    return cudaGetLastError();
}

size_t nearest_workspace_bytes(long long N) { return al256((size_t)N * sizeof(unsigned long long)); }

// Winners of every group into best[N] (packed), over codewords [0, K).
cudaError_t launch_nearest_packed(const float *V, long long N, const float *C, int K, unsigned long long *best,
                                  cudaStream_t st) {
    if (N == 0) return cudaSuccess;
    fill_u64_kernel<<<elementwise_grid(N), 256, 0, st>>>(best, N, ~0ull);
    const long long ctas_n = (N + kNearGroups - 1) / kNearGroups;
    // split the codewords over grid.y until there are about four CTAs per SM
    const long long want = (long long)device_sms() * 4;
    long long splits = (want + ctas_n - 1) / ctas_n;
    const long long max_splits = (K + kNearChunk - 1) / kNearChunk;
    if (splits > max_splits) splits = max_splits;
    if (splits > 65535) splits = 65535;
    if (splits < 1) splits = 1;
    const int k_per = (int)(((K + splits - 1) / splits + kNearChunk - 1) / kNearChunk * kNearChunk);
    splits = (K + k_per - 1) / k_per;
    if (ctas_n > 0x7fffffffLL) return cudaErrorInvalidValue;
    nearest_kernel<<<dim3((unsigned)ctas_n, (unsigned)splits), kNearThreads, 0, st>>>(V, N, C, K, k_per, best);
    return cudaGetLastError();
}

cudaError_t launch_nearest(const float *V, long long N, const float *C, int K, int32_t *idx, float *dist,
                           void *workspace, cudaStream_t st) {
    auto *best = static_cast<unsigned long long *>(workspace);
    cudaError_t e = launch_nearest_packed(V, N, C, K, best, st);
    if (e != cudaSuccess || N == 0) return e;
    unpack_best_kernel<<<elementwise_grid(N), 256, 0, st>>>(best, N, V, C, K, idx, dist);
    return cudaGetLastError();
}

size_t kmeans_workspace_bytes(int K) {
    return al256((size_t)K * 8 * sizeof(double)) + al256((size_t)K * sizeof(unsigned int));
}

cudaError_t launch_kmeans_update(const float *V, const int32_t *idx, long long N, const float *C_prev, int K,
                                 float *C_out, int32_t *counts_out, void *workspace, cudaStream_t st) {
    auto *sums = static_cast<double *>(workspace);
    auto *counts = reinterpret_cast<unsigned int *>(static_cast<uint8_t *>(workspace) +
                                                    al256((size_t)K * 8 * sizeof(double)));
    cudaError_t e = cudaMemsetAsync(workspace, 0, kmeans_workspace_bytes(K), st);
    if (e != cudaSuccess) return e;
    if (N > 0) kmeans_accumulate_kernel<<<elementwise_grid(N * 8), 256, 0, st>>>(V, idx, N, K, sums, counts);
    kmeans_finish_kernel<<<elementwise_grid((long long)K * 8), 256, 0, st>>>(sums, counts, K, C_prev, C_out,
                                                                             counts_out);
    return cudaGetLastError();
}

// Workspace of the residual k-means: residuals, indices, packed winners,
// k-means sums and counts, one codebook of updated centroids.
size_t residual_kmeans_workspace_bytes(long long N, int K) {
    return al256((size_t)N * 8 * sizeof(float)) + al256((size_t)N * sizeof(int32_t)) + nearest_workspace_bytes(N) +
           kmeans_workspace_bytes(K) + al256((size_t)K * 8 * sizeof(float));
}

cudaError_t launch_residual_kmeans(const float *V, long long N, int M, int K, const int32_t *init_idx, int iters,
                                   float *C_out, void *workspace, cudaStream_t st) {
    uint8_t *w = static_cast<uint8_t *>(workspace);
    float *R = reinterpret_cast<float *>(w);
    w += al256((size_t)N * 8 * sizeof(float));
    int32_t *idx = reinterpret_cast<int32_t *>(w);
    w += al256((size_t)N * sizeof(int32_t));
    auto *best = reinterpret_cast<unsigned long long *>(w);
    w += nearest_workspace_bytes(N);
    void *km = w;
    w += kmeans_workspace_bytes(K);
    float *C_tmp = reinterpret_cast<float *>(w);
    cudaError_t e = cudaMemcpyAsync(R, V, (size_t)N * 8 * sizeof(float), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
    for (int m = 0; m < M; ++m) {
        float *C = C_out + (size_t)m * K * 8;
        gather_rows_kernel<<<elementwise_grid((long long)K * 8), 256, 0, st>>>(R, init_idx + (size_t)m * K, K, C);
        for (int it = 0; it < iters; ++it) {
            if ((e = launch_nearest(R, N, C, K, idx, nullptr, best, st)) != cudaSuccess) return e;
            if ((e = launch_kmeans_update(R, idx, N, C, K, C_tmp, nullptr, km, st)) != cudaSuccess) return e;
            if ((e = cudaMemcpyAsync(C, C_tmp, (size_t)K * 8 * sizeof(float), cudaMemcpyDeviceToDevice, st)) !=
                cudaSuccess)
                return e;
        }
        if ((e = launch_nearest_packed(R, N, C, K, best, st)) != cudaSuccess) return e;
        subtract_nearest_kernel<<<elementwise_grid(N * 8), 256, 0, st>>>(R, best, N, C, K, nullptr, 1, 0, 2);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Workspace of the greedy codes: residuals, packed winners, fp32 codebooks.
size_t encode_codes_workspace_bytes(long long N, int M, int K) {
    return al256((size_t)N * 8 * sizeof(float)) + nearest_workspace_bytes(N) + al256((size_t)M * K * 8 * sizeof(float));
}

cudaError_t launch_encode_codes(const float *V, long long N, const uint16_t *codebooks, int M, int K, void *codes,
                                int code_bytes, void *workspace, cudaStream_t st) {
    uint8_t *w = static_cast<uint8_t *>(workspace);
    float *R = reinterpret_cast<float *>(w);
    w += al256((size_t)N * 8 * sizeof(float));
    auto *best = reinterpret_cast<unsigned long long *>(w);
    w += nearest_workspace_bytes(N);
    float *C = reinterpret_cast<float *>(w);
    cudaError_t e = cudaMemcpyAsync(R, V, (size_t)N * 8 * sizeof(float), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return e;
    half_to_float_kernel<<<elementwise_grid((long long)M * K * 8), 256, 0, st>>>(
        reinterpret_cast<const __half *>(codebooks), (long long)M * K * 8, C);
    for (int m = 0; m < M; ++m) {
        const float *Cm = C + (size_t)m * K * 8;
        if ((e = launch_nearest_packed(R, N, Cm, K, best, st)) != cudaSuccess) return e;
        subtract_nearest_kernel<<<elementwise_grid(N * 8), 256, 0, st>>>(R, best, N, Cm, K, codes, M, m, code_bytes);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_round_codebooks(const float *C, long long n, uint16_t *C16, cudaStream_t st) {
    float_to_half_kernel<<<elementwise_grid(n), 256, 0, st>>>(C, n, reinterpret_cast<__half *>(C16));
    return cudaGetLastError();
}

AQLM_DEFINE_BOUNDS_READER(bounds_word_encode)

}  // namespace aqlm
