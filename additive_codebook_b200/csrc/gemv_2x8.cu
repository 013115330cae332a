// gemv_2x8.cu -- the 2x8 instantiations of the decode-time kernel
// (one per token count 1..16), compiled on their own to build in parallel.
#include "gemv_kernels.cuh"

namespace aqlm {
namespace gemv_detail {

GemvFn gemv_pick_2x8(int tokens) {
    static constexpr auto table =
        gemv_table<2, 8>(std::make_integer_sequence<int, AQLM_GEMV_MAX_TOKENS>{});
    return table[tokens - 1];
}

}  // namespace gemv_detail
}  // namespace aqlm
