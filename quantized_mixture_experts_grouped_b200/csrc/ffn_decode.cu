// Fused decode path of the W4A16 MoE layer: routing, gate/up with SiLU*up, down projection and
// the router-weighted combine in ONE launch ("Every Expert Counts: ExactMoE for Memory-Efficient
// W4A16 Inference", Abstract: all selected experts execute through fused grouped MoE kernels;
// the router's top-k is unchanged).
//
// This file holds the path's dispatch: the single-token kernel of ffn_decode_rows.cu at T = 1
// (when its shared-memory plan fits the layer), else the warp-MMA kernel of ffn_decode_mma.cu
// for up to 16 tokens.
#include "decode_common.cuh"

namespace moe {
namespace dec {

unsigned long long* g_trace = nullptr;
int g_num_sms = 0;

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

namespace {

// h bytes per (selected expert, K group of I): the larger of the two kernels' layouts
size_t hbuf_per_tile(int T) { return std::max<size_t>(rows_hbuf_per_tile(), mma_hbuf_per_tile(std::min(T, kMmaMaxT))); }

}  // namespace
}  // namespace dec

// Diagnostics: when set, the fused decode kernels record per-CTA diagnostics (64 x u64 per CTA)
// into this device buffer; NULL turns it off.
MOE_API void moe_debug_set_decode_trace(void* dev_buffer) {
  dec::g_trace = static_cast<unsigned long long*>(dev_buffer);
}

bool ffn_decode_supported(const FfnArgs& a) {
  if (!(a.T >= 1 && a.T <= dec::kMaxT && a.T * a.k <= dec::kMaxTk && a.E <= kMaxExperts && a.H % kRowBlock == 0 &&
        a.I % kRowBlock == 0 && a.H > 0 && a.I > 0))
    return false;
  if (!dec::split_fits(a.T, a.H, a.I, a.E, a.k, dec::kMaxGrid)) return false;
  return dec::mma_stages(a.T, a.H) >= 2;
}

size_t decode_scratch_bytes(int T, int H, int I, int E, int k) {
  if (T < 1 || T > dec::kMaxT || H % kRowBlock || I % kRowBlock || E < 1 || k < 1) return 0;
  return dec::dec_scratch(T, H, I, E, k, dec::hbuf_per_tile(T)).total;
}

// Bytes of the fused-decode counter region (zero between launches; offset independent of T).
size_t decode_counter_bytes(int H, int I, int E) {
  if (H <= 0 || I <= 0 || E <= 0 || H % kRowBlock || I % kRowBlock) return 0;
  return dec::dec_counters(H, I, E).total;
}

// One token runs on the single-token kernel when its plan fits, up to sixteen on the warp-MMA
// kernel.
int ffn_decode(const FfnArgs& a, cudaStream_t s) {
  const WsLayout L = ws_layout(a.T, a.H, a.I, a.E, a.k);
  const dec::DecScratch D = dec::dec_scratch(a.T, a.H, a.I, a.E, a.k, dec::hbuf_per_tile(a.T));
  char* d = a.ws + L.dec;
  dec::DecParams P{};
  P.x = a.x; P.logits = a.logits; P.idx_in = a.idx; P.wts_in = a.wts;
  P.T = a.T; P.H = a.H; P.I = a.I; P.E = a.E; P.k = a.k;
  P.w13 = a.w13; P.s13 = a.s13; P.w2 = a.w2; P.s2 = a.s2; P.slot = a.slot;
  P.idx_out = a.idx_out; P.wts_out = a.wts_out;
  P.out = a.out; P.acc = reinterpret_cast<float*>(a.ws + L.acc); P.accumulate = a.accumulate ? 1 : 0;
  P.ctl = reinterpret_cast<int*>(a.ws + L.status);
  const dec::DecCounters C = dec::dec_counters(a.H, a.I, a.E);
  char* c = a.ws + L.ctr;
  P.hcnt = reinterpret_cast<int*>(c + C.hcnt);
  P.fcnt = reinterpret_cast<int*>(c + C.fcnt);
  P.hdone = reinterpret_cast<int*>(c + C.hdone);
  P.p1 = reinterpret_cast<float*>(d + D.p1);
  P.p2 = reinterpret_cast<float*>(d + D.p2);
  P.hbuf = reinterpret_cast<uint8_t*>(d + D.hbuf);
  P.mul16 = 65536u;
  P.trace = dec::g_trace;
  if (!a.logits && (!a.idx || !a.wts)) return fail(MOE_ERR_ARG, "fused decode: routing missing");

  const int m_max = std::min(a.E, a.T * a.k);
  const long tiles1 = (long)m_max * 2 * (a.I / kRowBlock) * (a.H / kGroup);
  const int grid = (int)std::max<long>(1, std::min<long>(std::min(dec::num_sms(), dec::kMaxGrid), tiles1));
  if (dec::rows_supported(a.T, a.H, a.I, a.E, a.k)) return dec::launch_decode_rows(P, dec::num_sms(), s);
  return dec::launch_decode_mma(P, grid, s);
}

}  // namespace moe
