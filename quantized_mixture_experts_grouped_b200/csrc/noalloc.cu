// moe_w4a16_layer_noalloc: moe_w4a16_layer with its workspace taken from a fixed array that
// the library itself holds in device memory, for callers that cannot allocate device memory:
// a host program that links this C library directly and runs under a device-memory budget fixed
// up front (no allocator to call into, or none it may call on the request path), or a hot loop
// where a cudaMalloc / cudaFree would synchronise the device or fragment its memory.
//
// The array is a file-scope static __device__ buffer of kNoAllocScratchBytes (16 MiB: enough for
// the fused decode path at up to 16 tokens on a 2048-wide, 64-expert, top-8 layer). Its device
// address is looked up with cudaGetSymbolAddress once per device, the first time this entry
// point runs with that device current; that first call should therefore come before any stream
// capture on the device. Every call on a device shares the one array, so calls that may run at
// the same time (different streams, or different host threads) race and must be serialised by
// the caller. Each call clears, on its stream, the words that must start at zero: the control
// block at the head of the workspace (all but the status word) and the fused-decode counters.
// The status word keeps the first device-side failure until moe_noalloc_status reads it. Nothing
// here allocates: no cudaMalloc / cudaFree, no allocating library.
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array for the current device (looked up once per device).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (int rc = check_cuda(cudaGetDevice(&dev), "moe_w4a16_layer_noalloc: cudaGetDevice")) return rc;
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_ARG, "moe_w4a16_layer_noalloc: device %d not supported", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (int rc = check_cuda(cudaGetSymbolAddress(&p, g_noalloc_scratch),
                            "moe_w4a16_layer_noalloc: cudaGetSymbolAddress of the scratch array"))
      return rc;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace

}  // namespace moe

using namespace moe;

MOE_API int moe_w4a16_layer_noalloc(const uint16_t* x_bf16, const uint16_t* logits_bf16, int T, int H, int I,
                                    int E, int k, const uint8_t* w13, const uint16_t* s13, const uint8_t* w2,
                                    const uint16_t* s2, const int32_t* slot_of_expert, int32_t* idx, float* wts,
                                    uint16_t* out_bf16, int flags, moe_stream_t stream) {
  if (flags & MOE_FLAG_ACCUMULATE)
    return fail(MOE_ERR_ARG, "moe_w4a16_layer_noalloc: MOE_FLAG_ACCUMULATE is not supported (the fp32 "
                             "accumulator would be shared by every call)");
  if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0)
    return fail(MOE_ERR_ARG, "moe_w4a16_layer_noalloc: bad sizes T=%d H=%d I=%d E=%d k=%d", T, H, I, E, k);
  if (T == 0) return MOE_OK;
  const WsLayout L = ws_layout(T, H, I, E, k);
  if (L.total > kNoAllocScratchBytes)
    return fail(MOE_ERR_SHAPE,
                "moe_w4a16_layer_noalloc: these sizes need %zu bytes of workspace, more than the %zu-byte "
                "static scratch; use moe_w4a16_layer with a caller-provided workspace",
                L.total, kNoAllocScratchBytes);
  void* ws = nullptr;
  if (int rc = scratch_for_current_device(&ws)) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // words that must start at zero: the control block after the status word, and the
  // fused-decode counters, which sit together at the head of the workspace
  char* base = static_cast<char*>(ws);
  const size_t keep = sizeof(int32_t) * 2;   // status word and its wait site
  if (int rc = check_cuda(cudaMemsetAsync(base + L.status + keep, 0, L.counts - L.status - keep, s),
                          "moe_w4a16_layer_noalloc: clearing the control block and counters"))
    return rc;
  return moe_w4a16_layer(x_bf16, logits_bf16, T, H, I, E, k, w13, s13, w2, s2, slot_of_expert, idx, wts, ws,
                         kNoAllocScratchBytes, out_bf16, flags, stream);
}

// Status of the calls above on the current device: reads (synchronously, on `stream`) and clears
// the status word of the static array, as moe_workspace_status does for a caller workspace.
MOE_API int moe_noalloc_status(moe_stream_t stream, int* status) {
  if (!status) return fail(MOE_ERR_ARG, "moe_noalloc_status: null pointer");
  void* ws = nullptr;
  if (int rc = scratch_for_current_device(&ws)) return rc;
  return moe_workspace_status(ws, stream, status);
}
