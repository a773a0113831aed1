// Sequential W4A16 MoE FFN: the selected experts run one after another instead of in one
// grouped launch - the ablation baseline of "Every Expert Counts: ExactMoE for
// Memory-Efficient W4A16 Inference" (the fused grouped kernels against executing the experts
// sequentially with the same W4A16 kernels).
//
// For every expert e in id order, the path the batch would take anyway (the fused decode kernel
// for small batches, else the grouped GEMM path, else the CUDA-core reference) runs restricted
// to expert e through a one-expert slot table: its pairs are computed, every other expert's are
// skipped. The partial outputs add up in the fp32 accumulator of the workspace and the last
// expert writes the bf16 output, so the result is the same sum as the fused paths' (in a
// different order of the k additions). No host synchronisation: every expert gets its
// launches, including experts no token routes to.
#include "common.cuh"

namespace moe {
namespace {

// tables[e][x] = slot of expert x if x == e, else -1 (skipped)
__global__ void __launch_bounds__(256) one_expert_tables_kernel(const int32_t* __restrict__ slot, int E,
                                                               int32_t* __restrict__ tables) {
  const int e = blockIdx.x;
  for (int x = threadIdx.x; x < E; x += blockDim.x) tables[(size_t)e * E + x] = x == e ? slot_of(slot, x) : -1;
}

}  // namespace

int ffn_sequential(const FfnArgs& a, cudaStream_t s) {
  const WsLayout L = ws_layout(a.T, a.H, a.I, a.E, a.k);
  int32_t* tables = reinterpret_cast<int32_t*>(a.ws + L.seq);
  one_expert_tables_kernel<<<a.E, 256, 0, s>>>(a.slot, a.E, tables);
  if (int rc = check_launch("one_expert_tables_kernel")) return rc;
  for (int e = 0; e < a.E; ++e) {
    FfnArgs b = a;
    b.slot = tables + (size_t)e * a.E;
    b.accumulate = a.accumulate || e > 0;
    b.out = e == a.E - 1 ? a.out : nullptr;
    b.logits = nullptr;                    // routing is given
    int rc;
    if (ffn_decode_supported(b)) rc = ffn_decode(b, s);
    else if (ffn_grouped_supported(b)) rc = ffn_grouped(b, s);
    else rc = ffn_simple(b, s);
    if (rc) return rc;
  }
  return MOE_OK;
}

}  // namespace moe
