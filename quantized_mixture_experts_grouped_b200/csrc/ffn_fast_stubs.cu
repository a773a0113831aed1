// Placeholder entry points of the optimised FFN paths until their kernels land.
#include "common.cuh"

namespace moe {
bool ffn_grouped_supported(const FfnArgs&) { return false; }
int ffn_grouped(const FfnArgs&, cudaStream_t) { return fail(MOE_ERR_SHAPE, "grouped GEMM path not built"); }
int ffn_sequential(const FfnArgs&, cudaStream_t) { return fail(MOE_ERR_SHAPE, "sequential path not built"); }
}  // namespace moe
