// gemv.cu -- host side of the decode-time product: the kernel choice and the
// workspace layout.  Few tokens: gemv_rows.cu (coalesced row streaming on the
// CUDA cores, the input range split when the activations do not fit on chip).
// More tokens: gemv_tc.cu (the weights decoded into shared memory for tcgen05
// tensor-core MMAs).  Both launch with programmatic dependent launch.  The
// lookup-table kernel of gemv_lut.cu (2x8, one token) has its own entry point,
// aqlm_gemv_lut: measured on B200 it does not beat the row kernel, so
// aqlm_gemv does not choose it.
#include "common.cuh"

namespace aqlm {

bool gemv_rows_supported(const Dims &d, int T);
int rows_max_tokens(const Dims &d);
size_t gemv_rows_multi_workspace_bytes(const RowLayerIn *layers, int n, const Dims &d, int T);
size_t gemv_rows_multi_counter_offset(const RowLayerIn *layers, int n, const Dims &d, int T);
cudaError_t launch_gemv_rows_multi(const RowLayerIn *layers, int n, const uint16_t *x, int tokens, const Dims &d,
                                   void *workspace, int sms, cudaStream_t st);
size_t gemv_rows_workspace_bytes(const Dims &d, int T, int sms);
size_t gemv_rows_counter_offset(const Dims &d, int T, int sms);
cudaError_t launch_gemv_rows(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                             uint16_t *y, int tokens, const Dims &d, void *workspace, int sms, cudaStream_t st);
bool gemv_tc_supported(const Dims &d, int T);
size_t gemv_tc_workspace_bytes(const Dims &d, int T, int sms);
size_t gemv_tc_counter_offset(const Dims &d, int T, int sms);
size_t gemv_tc_status_offset(const Dims &d, int T, int sms);
cudaError_t launch_gemv_tc(const void *codes, const uint16_t *codebooks, const uint16_t *scales, const uint16_t *x,
                           uint16_t *y, int tokens, const Dims &d, void *workspace, int sms, cudaStream_t st);
size_t gemv_tc_multi_counter_offset(const RowLayerIn *layers, int n, const Dims &d, int T, int sms);
size_t gemv_tc_multi_workspace_bytes(const RowLayerIn *layers, int n, const Dims &d, int T, int sms);
size_t gemv_tc_multi_status_offset(const RowLayerIn *layers, int n, const Dims &d, int T, int sms);
cudaError_t launch_gemv_tc_multi(const RowLayerIn *layers, int n, const uint16_t *x, int tokens, const Dims &d,
                                 void *workspace, int sms, cudaStream_t st);

namespace {

int device_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    return num_sms(dev);
}

}  // namespace

size_t gemv_workspace_bytes(const Dims &d, int tokens) {
    const int sms = device_sms();
    if (gemv_rows_supported(d, tokens)) return gemv_rows_workspace_bytes(d, tokens, sms);
    if (gemv_tc_supported(d, tokens)) return gemv_tc_workspace_bytes(d, tokens, sms);
    return 0;
}

// Offset of the arrival counters inside the workspace: the bytes from here to
// the end of the workspace must be zero before a call.
size_t gemv_workspace_counter_offset(const Dims &d, int tokens) {
    const int sms = device_sms();
    if (gemv_rows_supported(d, tokens)) return gemv_rows_counter_offset(d, tokens, sms);
    if (gemv_tc_supported(d, tokens)) return gemv_tc_counter_offset(d, tokens, sms);
    return 0;
}

// Offset of the status word inside the workspace, or -1 when the path for
// this shape and token count has no device waits (and no status word).
long long gemv_status_offset(const Dims &d, int tokens) {
    if (gemv_rows_supported(d, tokens) || !gemv_tc_supported(d, tokens)) return -1;
    return (long long)gemv_tc_status_offset(d, tokens, device_sms());
}

cudaError_t launch_gemv(const void *codes, const uint16_t *codebooks, const uint16_t *scales,
                        const uint16_t *x, uint16_t *y, int tokens, const Dims &d, void *workspace,
                        cudaStream_t st) {
    const int sms = device_sms();
    if (gemv_rows_supported(d, tokens))
        return launch_gemv_rows(codes, codebooks, scales, x, y, tokens, d, workspace, sms, st);
    if (gemv_tc_supported(d, tokens))
        return launch_gemv_tc(codes, codebooks, scales, x, y, tokens, d, workspace, sms, st);
    return cudaErrorInvalidValue;
}

// Several layers that read the same activations, in one launch of the
// kernel their token count selects.
int gemv_row_tokens(const Dims &d) { return rows_max_tokens(d); }

size_t gemv_multi_workspace_bytes(const RowLayerIn *layers, int n, const Dims &d, int tokens) {
    if (gemv_rows_supported(d, tokens)) return gemv_rows_multi_workspace_bytes(layers, n, d, tokens);
    return gemv_tc_multi_workspace_bytes(layers, n, d, tokens, device_sms());
}

size_t gemv_multi_counter_offset(const RowLayerIn *layers, int n, const Dims &d, int tokens) {
    if (gemv_rows_supported(d, tokens)) return gemv_rows_multi_counter_offset(layers, n, d, tokens);
    return gemv_tc_multi_counter_offset(layers, n, d, tokens, device_sms());
}

long long gemv_multi_status_offset(const RowLayerIn *layers, int n, const Dims &d, int tokens) {
    if (gemv_rows_supported(d, tokens) || !gemv_tc_supported(d, tokens)) return -1;
    return (long long)gemv_tc_multi_status_offset(layers, n, d, tokens, device_sms());
}

cudaError_t launch_gemv_multi(const RowLayerIn *layers, int n, const uint16_t *x, int tokens, const Dims &d,
                              void *workspace, cudaStream_t st) {
    if (gemv_rows_supported(d, tokens)) return launch_gemv_rows_multi(layers, n, x, tokens, d, workspace, device_sms(), st);
    return launch_gemv_tc_multi(layers, n, x, tokens, d, workspace, device_sms(), st);
}

}  // namespace aqlm
