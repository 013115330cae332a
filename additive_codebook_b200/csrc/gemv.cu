// gemv.cu -- host side of the decode-time product: kernel choice, work plan,
// workspace layout and the launch (with programmatic dependent launch).
// 1..4 tokens: gemv_rows.cu (coalesced row streaming, the input range split
// when the activations do not fit on chip).  5..16 tokens: the several-rows-per-lane
// kernel of gemv_multi.cuh, instantiated per format in gemv_multi_1x16.cu,
// gemv_multi_2x8.cu and gemv_multi_2x16.cu.
#include "gemv_multi.cuh"

namespace aqlm {

bool gemv_rows_supported(int T);
size_t gemv_rows_workspace_bytes(const Dims &d, int T, int sms);
size_t gemv_rows_counter_offset(const Dims &d, int T, int sms);
cudaError_t launch_gemv_rows(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                             uint16_t *y, int tokens, const Dims &d, void *workspace, int sms, cudaStream_t st);

namespace gemv_detail {
namespace {

struct Plan {
    int tiles;             // row tiles of 32 rows (gridDim.x)
    int splits;            // CTAs along the input range (gridDim.y)
    int chunks_per_split;  // 16-byte code chunks per row per CTA
    size_t smem;
};

inline size_t align16(size_t v) { return (v + 15) / 16 * 16; }

// Several tokens: tiles of 32*R rows.  The input range is split over
// gridDim.y CTAs when (a) T activations of the whole row exceed the on-chip
// budget, or (b) there are too few row tiles to give every SM three CTAs;
// never below one chunk per warp.
Plan plan_multi(const Dims &d, int T, int sms) {
    const int gpc = 16 / (d.M * d.B / 8);
    const int n_chunks = d.G / gpc;
    const int R = 4, tp8 = (T + 7) & ~7;
    Plan p;
    p.tiles = (d.d_out + 32 * R - 1) / (32 * R);
    int max_chunks = kXsBudget / (tp8 * gpc * kGroup * 2);
    if (max_chunks < 1) max_chunks = 1;
    const int ks_min = (n_chunks + max_chunks - 1) / max_chunks;
    int ks_par = (3 * sms) / p.tiles;
    if (ks_par < 1) ks_par = 1;
    int ks_cap = n_chunks / kMultiWarps;
    if (ks_cap < 1) ks_cap = 1;
    int ks = ks_par < ks_cap ? ks_par : ks_cap;
    if (ks < ks_min) ks = ks_min;
    p.chunks_per_split = (n_chunks + ks - 1) / ks;
    p.splits = (n_chunks + p.chunks_per_split - 1) / p.chunks_per_split;
    p.smem = (size_t)tp8 * p.chunks_per_split * gpc * kGroup * 2 + (size_t)kMultiWarps * T * 32 * R * 4;
    return p;
}

size_t multi_workspace_bytes(const Dims &d, int T, int sms) {
    const Plan p = plan_multi(d, T, sms);
    if (p.splits == 1) return 0;
    return align16((size_t)p.splits * T * d.d_out * sizeof(float)) + (size_t)p.tiles * sizeof(uint32_t);
}

GemvFn pick_multi(int M, int B, int T) {
    if (M == 1) return gemv_multi_pick_1x16(T);
    if (B == 8) return gemv_multi_pick_2x8(T);
    return gemv_multi_pick_2x16(T);
}

// Up to four tokens: whole rows per warp with coalesced code streaming.
bool use_rows(int T) { return gemv_rows_supported(T); }

int device_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    return num_sms(dev);
}

}  // namespace
}  // namespace gemv_detail

size_t gemv_workspace_bytes(const Dims &d, int tokens) {
    using namespace gemv_detail;
    const int sms = device_sms();
    if (use_rows(tokens)) return gemv_rows_workspace_bytes(d, tokens, sms);
    return multi_workspace_bytes(d, tokens, sms);
}

// Offset of the arrival counters inside the workspace: the bytes from here to
// the end of the workspace must be zero before a call.
size_t gemv_workspace_counter_offset(const Dims &d, int tokens) {
    using namespace gemv_detail;
    const int sms = device_sms();
    if (use_rows(tokens)) return gemv_rows_counter_offset(d, tokens, sms);
    const Plan p = plan_multi(d, tokens, sms);
    if (p.splits == 1) return 0;
    return align16((size_t)p.splits * tokens * d.d_out * sizeof(float));
}

cudaError_t launch_gemv(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                        const uint16_t *x, uint16_t *y, int tokens, const Dims &d, void *workspace,
                        cudaStream_t st) {
    using namespace gemv_detail;
    const int sms = device_sms();
    if (use_rows(tokens)) return launch_gemv_rows(codes, codebooks, scales, x, y, tokens, d, workspace, sms, st);
    const Plan p = plan_multi(d, tokens, sms);
    GemvFn fn = pick_multi(d.M, d.B, tokens);
    const cudaError_t e = opt_in_dynamic_smem(fn, p.smem);
    if (e != cudaSuccess) return e;
    GemvArgs a;
    a.codes = static_cast<const uint8_t *>(codes);
    a.codebooks = reinterpret_cast<const uint4 *>(codebooks);
    a.scales = reinterpret_cast<const __half *>(scales);
    a.x = reinterpret_cast<const __half *>(x);
    a.y = reinterpret_cast<__half *>(y);
    a.partial = static_cast<float *>(workspace);
    a.counters = p.splits > 1 ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) +
                                                             align16((size_t)p.splits * tokens * d.d_out * 4))
                              : nullptr;
    a.d_out = d.d_out;
    a.d_in = d.d_in;
    a.G = d.G;
    a.row_bytes = d.row_bytes;
    a.chunks_per_split = p.chunks_per_split;
    return launch_kernel(fn, dim3(p.tiles, p.splits), dim3(kMultiThreads), p.smem, st, true, a);
}

}  // namespace aqlm
