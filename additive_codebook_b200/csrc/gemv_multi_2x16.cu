// gemv_multi_2x16.cu -- the 2x16 instantiations of the several-token
// kernel (one per token count 5..16), compiled on their own to build in parallel.
#include "gemv_multi.cuh"

namespace aqlm {
namespace gemv_detail {

GemvFn gemv_multi_pick_2x16(int tokens) {
    static constexpr auto table =
        gemv_multi_table<2, 16>(std::make_integer_sequence<int, AQLM_GEMV_MAX_TOKENS - kMultiMinTokens + 1>{});
    return table[tokens - kMultiMinTokens];
}

}  // namespace gemv_detail
}  // namespace aqlm
