// gemv_1x16.cu -- the 1x16 instantiations of the decode-time kernel
// (one per token count 1..16), compiled on their own to build in parallel.
#include "gemv_kernels.cuh"

namespace aqlm {
namespace gemv_detail {

GemvFn gemv_pick_1x16(int tokens) {
    static constexpr auto table =
        gemv_table<1, 16>(std::make_integer_sequence<int, AQLM_GEMV_MAX_TOKENS>{});
    return table[tokens - 1];
}

}  // namespace gemv_detail
}  // namespace aqlm
