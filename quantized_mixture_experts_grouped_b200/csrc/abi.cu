// C ABI entry points (declared in include/moe_w4a16.h): argument checks, workspace layout,
// dispatch to the kernel paths. Nothing here allocates device memory.
#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <atomic>
#include <string>

#include "common.cuh"

namespace moe {

namespace {
thread_local std::string g_last_error = "no error";
std::atomic<unsigned long long> g_launches{0};
}

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return MOE_OK;
  return fail(MOE_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

WsLayout ws_layout(int T, int H, int I, int E, int k) {
  WsLayout L{};
  const size_t Tk = (size_t)T * k;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  L.status = take(sizeof(int32_t) * kCtlWords);
  L.ctr = take(decode_counter_bytes(H, I, E));
  L.counts = take(sizeof(int32_t) * E);
  L.offsets = take(sizeof(int32_t) * (E + 1));
  L.perm = take(sizeof(int32_t) * Tk);
  L.inv = take(sizeof(int32_t) * Tk);
  L.perm_scratch = take(sizeof(int32_t) * permute_scratch_count(T, k, E));
  L.tiles = take(sizeof(int32_t) * (4 * (E + 1) + 64));
  {
    const size_t chunks = (Tk + 127) / 128 + (size_t)E;
    const size_t blocks = std::max<size_t>(I / 128, H / 128);   // gate/up pairs; down pairs x K halves
    L.tile_list_len = chunks * blocks;
    L.tile_list = take(sizeof(int32_t) * 2 * L.tile_list_len);
  }
  L.xp = take(sizeof(uint16_t) * Tk * H);
  L.hp = take(sizeof(uint16_t) * Tk * I);
  L.yp = take(sizeof(float) * Tk * H);
  L.acc = take(sizeof(float) * (size_t)T * H);
  L.seq = take(sizeof(int32_t) * (size_t)E * E);
  // fused-decode scratch for min(T, 16) tokens: a workspace sized for T also serves every smaller
  // batch (the total never shrinks as T grows)
  L.dec = take(decode_scratch_bytes(std::min(T, 16), H, I, E, k));
  L.total = off;
  return L;
}

}  // namespace moe

using namespace moe;

namespace {

bool dims_ok(int H, int I) { return H > 0 && I > 0 && H % kRowBlock == 0 && I % kRowBlock == 0; }

int check_layer_args(const uint16_t* x, int T, int H, int I, int E, int k, const uint8_t* w13, const uint16_t* s13,
                     const uint8_t* w2, const uint16_t* s2, void* ws, size_t ws_bytes, uint16_t* out, int flags) {
  if (T < 0 || E < 1 || k < 1 || k > E) return fail(MOE_ERR_ARG, "bad sizes T=%d E=%d k=%d", T, E, k);
  if (E > kMaxExperts) return fail(MOE_ERR_SHAPE, "E=%d exceeds %d", E, kMaxExperts);
  if (!dims_ok(H, I)) return fail(MOE_ERR_SHAPE, "H=%d and I=%d must be positive multiples of 128", H, I);
  if (!w13 || !s13 || !w2 || !s2 || !ws) return fail(MOE_ERR_ARG, "null weight or workspace pointer");
  if (T > 0 && !x) return fail(MOE_ERR_ARG, "null x");
  const int path = flags & MOE_PATH_MASK;
  if (path > MOE_PATH_SEQUENTIAL) return fail(MOE_ERR_ARG, "unknown path %d", path);
  const WsLayout L = ws_layout(T, H, I, E, k);
  if (ws_bytes < L.total)
    return fail(MOE_ERR_ARG, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, L.total);
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_ARG, "workspace must be 256-byte aligned");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(out)) & 15)
    return fail(MOE_ERR_ARG, "x and out must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(w13) | reinterpret_cast<uintptr_t>(w2)) & 127)
    return fail(MOE_ERR_ARG, "packed weights must be 128-byte aligned");
  if ((reinterpret_cast<uintptr_t>(s13) | reinterpret_cast<uintptr_t>(s2)) & 15)
    return fail(MOE_ERR_ARG, "scales must be 16-byte aligned");
  return MOE_OK;
}

int run_ffn(const FfnArgs& a, int flags, cudaStream_t s) {
  const int path = flags & MOE_PATH_MASK;
  switch (path) {
    case MOE_PATH_SIMPLE:
      return ffn_simple(a, s);
    case MOE_PATH_SEQUENTIAL:
      return ffn_sequential(a, s);
    case MOE_PATH_DECODE:
      if (!ffn_decode_supported(a)) return fail(MOE_ERR_SHAPE, "fused decode path does not support these sizes");
      return ffn_decode(a, s);
    case MOE_PATH_GROUPED:
      if (!ffn_grouped_supported(a)) return fail(MOE_ERR_SHAPE, "grouped GEMM path does not support these sizes");
      return ffn_grouped(a, s);
    default:
      if (ffn_decode_supported(a)) return ffn_decode(a, s);
      if (ffn_grouped_supported(a)) return ffn_grouped(a, s);
      return ffn_simple(a, s);
  }
}

}  // namespace

MOE_API int moe_abi_version(void) { return 1; }
MOE_API int moe_packed_layout_version(void) { return 2; }
MOE_API const char* moe_last_error_string(void) { return g_last_error.c_str(); }
MOE_API unsigned long long moe_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

MOE_API size_t moe_packed_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || N % kRowBlock || K % kGroup) return 0;
  return (size_t)N * K / 2;
}

MOE_API size_t moe_scales_count(int N, int K) {
  if (N <= 0 || K <= 0 || N % kRowBlock || K % kGroup) return 0;
  return (size_t)N * (K / kGroup);
}

MOE_API int moe_quantize_pack(const uint16_t* w_bf16, int E, int N, int K, uint8_t* packed, uint16_t* scales,
                              moe_stream_t stream) {
  if (!w_bf16 || !packed || !scales || E < 1) return fail(MOE_ERR_ARG, "moe_quantize_pack: null pointer or E < 1");
  if (N <= 0 || K <= 0 || N % kRowBlock || K % kGroup)
    return fail(MOE_ERR_SHAPE, "moe_quantize_pack: N=%d and K=%d must be positive multiples of 128", N, K);
  if ((reinterpret_cast<uintptr_t>(w_bf16) & 3) || (reinterpret_cast<uintptr_t>(packed) & 15))
    return fail(MOE_ERR_ARG, "moe_quantize_pack: misaligned pointer");
  return launch_quantize_pack(w_bf16, E, N, K, packed, scales, reinterpret_cast<cudaStream_t>(stream));
}

MOE_API int moe_route_topk(const uint16_t* logits_bf16, int T, int E, int k, int32_t* idx, float* wts,
                           moe_stream_t stream) {
  if (T < 0 || k < 1 || k > E) return fail(MOE_ERR_ARG, "moe_route_topk: bad sizes T=%d E=%d k=%d", T, E, k);
  if (E > kMaxExperts) return fail(MOE_ERR_SHAPE, "moe_route_topk: E=%d exceeds %d", E, kMaxExperts);
  if (T > 0 && (!logits_bf16 || !idx || !wts)) return fail(MOE_ERR_ARG, "moe_route_topk: null pointer");
  return launch_route(logits_bf16, T, E, k, idx, wts, reinterpret_cast<cudaStream_t>(stream));
}

MOE_API size_t moe_permute_scratch_count(int T, int k, int E) {
  if (T < 0 || k < 1 || E < 1) return 0;
  return permute_scratch_count(T, k, E);
}

MOE_API int moe_permute(const int32_t* idx, int T, int k, int E, int32_t* counts, int32_t* offsets, int32_t* perm,
                        int32_t* inv, int32_t* scratch, moe_stream_t stream) {
  if (T < 0 || k < 1 || E < 1) return fail(MOE_ERR_ARG, "moe_permute: bad sizes");
  if (E > kMaxExperts) return fail(MOE_ERR_SHAPE, "moe_permute: E=%d exceeds %d", E, kMaxExperts);
  if (!counts || !offsets || (T > 0 && (!idx || !perm || !inv || !scratch)))
    return fail(MOE_ERR_ARG, "moe_permute: null pointer");
  return launch_permute(idx, T, k, E, counts, offsets, perm, inv, scratch, reinterpret_cast<cudaStream_t>(stream));
}

MOE_API int moe_workspace_bytes(int T, int H, int I, int E, int k, size_t* bytes) {
  if (!bytes || T < 0 || E < 1 || k < 1 || k > E) return fail(MOE_ERR_ARG, "moe_workspace_bytes: bad arguments");
  if (E > kMaxExperts || !dims_ok(H, I)) return fail(MOE_ERR_SHAPE, "moe_workspace_bytes: unsupported sizes");
  *bytes = ws_layout(T, H, I, E, k).total;
  return MOE_OK;
}

MOE_API int moe_workspace_init(void* workspace, size_t bytes, moe_stream_t stream) {
  if (!workspace) return fail(MOE_ERR_ARG, "moe_workspace_init: null workspace");
  return check_cuda(cudaMemsetAsync(workspace, 0, bytes, reinterpret_cast<cudaStream_t>(stream)),
                    "moe_workspace_init");
}

MOE_API int moe_workspace_status(void* workspace, moe_stream_t stream, int* status) {
  if (!workspace || !status) return fail(MOE_ERR_ARG, "moe_workspace_status: null pointer");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t words[2] = {0, 0};
  if (int rc = check_cuda(cudaMemcpyAsync(words, workspace, sizeof(words), cudaMemcpyDeviceToHost, s),
                          "moe_workspace_status: read"))
    return rc;
  if (int rc = check_cuda(cudaStreamSynchronize(s), "moe_workspace_status: sync")) return rc;
  *status = words[0];
  if (words[0] != 0) {
    fail(words[0], "device status %d (wait site %d)", words[0], words[1]);
    if (int rc = check_cuda(cudaMemsetAsync(workspace, 0, sizeof(words), s), "moe_workspace_status: clear"))
      return rc;
  }
  return MOE_OK;
}

MOE_API int moe_w4a16_ffn(const uint16_t* x_bf16, int T, int H, int I, int E, int k, const int32_t* idx,
                          const float* wts, const uint8_t* w13, const uint16_t* s13, const uint8_t* w2,
                          const uint16_t* s2, const int32_t* slot_of_expert, void* workspace,
                          size_t workspace_bytes, uint16_t* out_bf16, int flags, moe_stream_t stream) {
  if (int rc = check_layer_args(x_bf16, T, H, I, E, k, w13, s13, w2, s2, workspace, workspace_bytes, out_bf16, flags))
    return rc;
  if (T > 0 && (!idx || !wts)) return fail(MOE_ERR_ARG, "moe_w4a16_ffn: null idx/wts");
  if (T == 0) return MOE_OK;
  FfnArgs a{};
  a.x = x_bf16; a.T = T; a.H = H; a.I = I; a.E = E; a.k = k;
  a.idx = idx; a.wts = wts; a.w13 = w13; a.s13 = s13; a.w2 = w2; a.s2 = s2;
  a.slot = slot_of_expert; a.ws = static_cast<char*>(workspace); a.ws_bytes = workspace_bytes;
  a.out = out_bf16; a.accumulate = (flags & MOE_FLAG_ACCUMULATE) != 0;
  return run_ffn(a, flags, reinterpret_cast<cudaStream_t>(stream));
}

MOE_API int moe_w4a16_layer(const uint16_t* x_bf16, const uint16_t* logits_bf16, int T, int H, int I, int E, int k,
                            const uint8_t* w13, const uint16_t* s13, const uint8_t* w2, const uint16_t* s2,
                            const int32_t* slot_of_expert, int32_t* idx, float* wts, void* workspace,
                            size_t workspace_bytes, uint16_t* out_bf16, int flags, moe_stream_t stream) {
  if (int rc = check_layer_args(x_bf16, T, H, I, E, k, w13, s13, w2, s2, workspace, workspace_bytes, out_bf16, flags))
    return rc;
  if (T > 0 && (!logits_bf16 || !idx || !wts)) return fail(MOE_ERR_ARG, "moe_w4a16_layer: null logits/idx/wts");
  if (T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  FfnArgs a{};
  a.x = x_bf16; a.T = T; a.H = H; a.I = I; a.E = E; a.k = k;
  a.idx = idx; a.wts = wts; a.w13 = w13; a.s13 = s13; a.w2 = w2; a.s2 = s2;
  a.slot = slot_of_expert; a.ws = static_cast<char*>(workspace); a.ws_bytes = workspace_bytes;
  a.out = out_bf16; a.accumulate = (flags & MOE_FLAG_ACCUMULATE) != 0;
  const int path = flags & MOE_PATH_MASK;
  const bool fused =
      (path == MOE_PATH_DECODE || path == MOE_PATH_AUTO) && ffn_decode_supported(a);
  if (fused) {
    a.logits = logits_bf16; a.idx_out = idx; a.wts_out = wts;
    return ffn_decode(a, s);
  }
  if (int rc = launch_route(logits_bf16, T, E, k, idx, wts, s)) return rc;
  return run_ffn(a, flags, s);
}

// ---- BF16 comparison layer: the same grouped scheduler and tcgen05 GEMMs on unquantised weights
namespace {

int check_bf16_args(const uint16_t* x, int T, int H, int I, int E, int k, const uint16_t* w13, const uint16_t* w2,
                    void* ws, size_t ws_bytes, int flags) {
  if (T < 0 || E < 1 || k < 1 || k > E) return fail(MOE_ERR_ARG, "bad sizes T=%d E=%d k=%d", T, E, k);
  if (E > kMaxExperts) return fail(MOE_ERR_SHAPE, "E=%d exceeds %d", E, kMaxExperts);
  if (!dims_ok(H, I)) return fail(MOE_ERR_SHAPE, "H=%d and I=%d must be positive multiples of 128", H, I);
  if (!w13 || !w2 || !ws) return fail(MOE_ERR_ARG, "null weight or workspace pointer");
  if (T > 0 && !x) return fail(MOE_ERR_ARG, "null x");
  const int path = flags & MOE_PATH_MASK;
  if (path != MOE_PATH_AUTO && path != MOE_PATH_GROUPED)
    return fail(MOE_ERR_ARG, "the bf16-weight layer runs on the grouped path only (path %d)", path);
  const WsLayout L = ws_layout(T, H, I, E, k);
  if (ws_bytes < L.total)
    return fail(MOE_ERR_ARG, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes, L.total);
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return fail(MOE_ERR_ARG, "workspace must be 256-byte aligned");
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(w13) | reinterpret_cast<uintptr_t>(w2)) & 15)
    return fail(MOE_ERR_ARG, "x and the weights must be 16-byte aligned");
  return MOE_OK;
}

}  // namespace

MOE_API int moe_bf16_ffn(const uint16_t* x_bf16, int T, int H, int I, int E, int k, const int32_t* idx,
                         const float* wts, const uint16_t* w13_bf16, const uint16_t* w2_bf16,
                         const int32_t* slot_of_expert, void* workspace, size_t workspace_bytes, uint16_t* out_bf16,
                         int flags, moe_stream_t stream) {
  if (int rc = check_bf16_args(x_bf16, T, H, I, E, k, w13_bf16, w2_bf16, workspace, workspace_bytes, flags)) return rc;
  if (T > 0 && (!idx || !wts)) return fail(MOE_ERR_ARG, "moe_bf16_ffn: null idx/wts");
  if (T == 0) return MOE_OK;
  FfnArgs a{};
  a.x = x_bf16; a.T = T; a.H = H; a.I = I; a.E = E; a.k = k;
  a.idx = idx; a.wts = wts;
  a.w13 = reinterpret_cast<const uint8_t*>(w13_bf16); a.w2 = reinterpret_cast<const uint8_t*>(w2_bf16);
  a.slot = slot_of_expert; a.ws = static_cast<char*>(workspace); a.ws_bytes = workspace_bytes;
  a.out = out_bf16; a.accumulate = (flags & MOE_FLAG_ACCUMULATE) != 0;
  a.bf16_weights = true;
  if (!ffn_grouped_supported(a)) return fail(MOE_ERR_SHAPE, "grouped GEMM path does not support these sizes");
  return ffn_grouped(a, reinterpret_cast<cudaStream_t>(stream));
}

MOE_API int moe_bf16_layer(const uint16_t* x_bf16, const uint16_t* logits_bf16, int T, int H, int I, int E, int k,
                           const uint16_t* w13_bf16, const uint16_t* w2_bf16, const int32_t* slot_of_expert,
                           int32_t* idx, float* wts, void* workspace, size_t workspace_bytes, uint16_t* out_bf16,
                           int flags, moe_stream_t stream) {
  if (int rc = check_bf16_args(x_bf16, T, H, I, E, k, w13_bf16, w2_bf16, workspace, workspace_bytes, flags)) return rc;
  if (T > 0 && (!logits_bf16 || !idx || !wts)) return fail(MOE_ERR_ARG, "moe_bf16_layer: null logits/idx/wts");
  if (T == 0) return MOE_OK;
  if (int rc = launch_route(logits_bf16, T, E, k, idx, wts, reinterpret_cast<cudaStream_t>(stream))) return rc;
  return moe_bf16_ffn(x_bf16, T, H, I, E, k, idx, wts, w13_bf16, w2_bf16, slot_of_expert, workspace, workspace_bytes,
                      out_bf16, flags, stream);
}
