// Fused decode path of the W4A16 MoE layer: routing, gate/up with SiLU*up, down projection and
// the router-weighted combine in ONE persistent launch ("Every Expert Counts: ExactMoE for
// Memory-Efficient W4A16 Inference", Abstract: all selected experts execute through fused
// grouped MoE kernels; the router's top-k is unchanged).
//
// This file holds the path's dispatch (ffn_decode: the single-token kernel of
// ffn_decode_rows.cu at T = 1, the warp-MMA kernel of ffn_decode_mma.cu up to 16 tokens) and the
// tcgen05 variant of the fused launch described below, which runs on request
// (MOE_PATH_DECODE_TC) as the bf16 tensor-core comparison point.
//
// A decode batch (T <= 16 tokens) reads every selected expert's packed weights exactly once, so
// the layer is bound by HBM bandwidth on those bytes plus the latency of its dependent steps.
// On B200 a CTA only streams near its share of HBM bandwidth when it moves weights in large
// bulk copies (tens of KB each) with several in flight, so the work is cut into byte-balanced
// contiguous runs of packed tiles rather than into whole experts or feature slices:
//  * every CTA routes the batch itself (warp top-k; the renormalised weights are a softmax over
//    the k chosen logits, which equals the full softmax renormalised), lists the selected
//    experts in ascending id, and stages the activations in shared memory as the B operand of
//    every gate/up MMA (all T tokens are MMA columns; columns of unrouted tokens are ignored);
//  * phase 1 (gate/up): the selected experts' W13 tiles, expert by expert in stored order, are
//    split evenly over the CTAs. A CTA accumulates each 128-row block it touches over its part
//    of K and writes the fp32 partial. The CTA that completes the last partial of a feature
//    block (gate rows f..f+127 and up rows I+f..I+f+127) sums the partials in CTA order and
//    writes h = w_router * silu(gate) * up in bf16 (zero for tokens not routed to the expert);
//  * phase 2 (down): W2 tiles ordered (output row block, expert, K group) are split the same
//    way. A CTA accumulates one output row block over all experts and K groups it covers, so
//    the router-weighted sum over experts happens inside the tensor-memory accumulator; the h
//    operand of each tile arrives with it. The CTA completing an output block's last partial
//    sums the partials in CTA order and writes the bf16 outputs. Down weights are prefetched
//    while phase 1 still runs; only their h operands wait until every feature block is done;
//  * warp 0 streams int4 codes + bf16 scales in copies of up to four tiles (32 KB) into a ring
//    of shared-memory stages (TMA bulk copies, evict-first in L2); its lanes issue the copies
//    of a stage side by side, since each issuing thread pays a fixed latency per copy;
//  * warps 6..13 dequantise in two groups that take alternate tiles: a thread owns one weight
//    row and writes bf16 (q * s, one rounding) straight into TENSOR MEMORY (tcgen05.st) as the
//    A operand of tcgen05.mma - the bf16 weights never pass through shared memory;
//  * one thread in each of warps 1 and 14 issues tcgen05.mma (M = 128 weight rows, N = 16
//    tokens, K = 16) for alternate tiles into its own accumulators: with N this small an MMA
//    costs its issuing thread about as much as a full-width one, so two issuers double the
//    rate at which tiles are consumed;
//  * warps 2..5 drain accumulators, add the two issuers' parts, write partials and run the
//    reductions above.
// Every reduction runs in a fixed order, so results are identical run to run. Every wait is
// bounded; on a timeout the kernel records MOE_ERR_TIMEOUT in the workspace, drains its own
// copies and MMAs, frees its tensor memory and exits (the workspace must then be re-initialised).
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

constexpr int kN = 16;                     // MMA N: the batch's tokens (<= 16)
constexpr int kMaxStages = 4;
constexpr int kABufs = 4;                  // dequantised tiles in tensor memory (64 columns each)
constexpr int kIssuers = 2;                // MMA-issuing threads (one per warp)
constexpr int kAcc = 8;                    // accumulators per issuer (16 columns each)
constexpr int kThreads = 480;              // 15 warps
constexpr int kIssuerWarp0 = 1;
constexpr int kEpiWarp0 = 2;               // warps 2..5
constexpr int kDqWarp0 = 6;                // warps 6..13: two groups of four
constexpr int kDqWarpsPerGroup = 4;
constexpr int kIssuerWarp1 = 14;
constexpr int kTmemCols = 512;
constexpr int kAColBase = 0;
constexpr int kAccCol = kABufs * 64;
constexpr int kHTile = 2048;               // one 8-token row group of a 128-wide h tile (bf16)
constexpr int kStageH = 2 * kTilesPerStage * kHTile;
constexpr int kStageBytes = kStageW + kStageS + kStageH;

struct __align__(128) DecSmem {
  uint64_t full[kMaxStages], empty[kMaxStages], hfull[kMaxStages];
  uint64_t afull[kABufs], aempty[kABufs];
  uint64_t accfull[kIssuers][kAcc], accempty[kIssuers][kAcc];
  uint64_t drain[kIssuers];
  RouteSmem rs;
  float wsel[kMaxT];
  uint32_t tmem_base;
  int abort;
  int epi_dec;
  // followed in dynamic shared memory by the activations (kN rows x H, no-swizzle K-major)
  // and by the stage ring
};

__device__ __forceinline__ void report_abort(DecSmem& s, const DecParams& P, int site) {
  s.abort = 1;
  report_status(P.ctl, MOE_ERR_TIMEOUT, site);
}

// 64 int4 codes (two 16-byte chunks of one row) -> 32 bf16x2 columns of tensor memory.
// Codes c of K = 2p and 2p+1 sit at bits 4p and 16+4p of a word, so OR-ing them into the bf16
// pattern 0x4300 (128.0) gives 128 + c exactly; minus 136 gives q = c - 8 exactly; times the
// scale gives bf16(q * s) with a single rounding.
__device__ __forceinline__ void dequant_half(uint4 a, uint4 b, __nv_bfloat162 s2, __nv_bfloat162 off136,
                                             uint32_t taddr) {
  const uint32_t words[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t v[32];
#pragma unroll
  for (int w = 0; w < 8; ++w)
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t t = ((words[w] >> (4 * p)) & 0x000F000Fu) | 0x43004300u;
      const __nv_bfloat162 qv = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&t), off136);
      const __nv_bfloat162 wv = __hmul2(qv, s2);
      v[w * 4 + p] = *reinterpret_cast<const uint32_t*>(&wv);
    }
  tc::tmem_st32(taddr, v);
}

// Element (n, k) of the kN-row, K-major activation operand without swizzle: 8x16-byte core
// matrices, K-direction core stride 256 bytes, row-group stride 128 bytes.
__device__ __forceinline__ uint32_t kmajor_off(int n, int k) {
  return (uint32_t)(((k >> 3) * (kN / 8) + (n >> 3)) * 128 + (n & 7) * 16 + (k & 7) * 2);
}

// The activations as the K-major bf16 B operand of the gate/up MMAs (all kN rows; rows >= T are
// left as they are: those MMA columns are never read).
__device__ void stage_x(const DecParams& P, uint8_t* xs, int tid) {
  const int rowc = P.H / 8;                       // 16-byte chunks per activation row
  const int chunks = P.T * rowc;
  for (int c = tid; c < chunks; c += kThreads)
    *reinterpret_cast<uint4*>(xs + kmajor_off(c / rowc, (c % rowc) * 8)) =
        __ldg(reinterpret_cast<const uint4*>(P.x + (size_t)(c / rowc) * P.H) + c % rowc);
}

__global__ void __launch_bounds__(kThreads, 1) moe_decode_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecSmem& s = *reinterpret_cast<DecSmem*>(smem_raw);
  uint8_t* xs = smem_raw + sizeof(DecSmem);
  uint8_t* ring = xs + (size_t)kN * P.H * 2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NS = P.nstages;

  // ---- set-up that does not read the previous kernel's results: overlaps it under PDL
  if (warp == 2) {
    if (lane < kMaxStages) {
      tc::mbar_init(&s.full[lane], 1);
      tc::mbar_init(&s.empty[lane], 2 * kDqWarpsPerGroup + kIssuers);   // dequant warps + MMA commits
      tc::mbar_init(&s.hfull[lane], 1);
    }
    if (lane < kABufs) { tc::mbar_init(&s.afull[lane], kDqWarpsPerGroup); tc::mbar_init(&s.aempty[lane], 1); }
    if (lane < kIssuers * kAcc) {
      tc::mbar_init(&s.accfull[0][0] + lane, 1);
      tc::mbar_init(&s.accempty[0][0] + lane, 4);
    }
    if (lane == 0) {
      tc::mbar_init(&s.drain[0], 1);
      tc::mbar_init(&s.drain[1], 1);
      s.abort = 0;
    }
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc<kTmemCols>(&s.tmem_base);
    tc::tc_fence_before();
  }
  route_clear(s.rs, tid, kThreads);
  __syncthreads();

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) trace_at(P, 0);
  route_begin(s.rs, P, tid, kThreads);
  stage_x(P, xs, tid);
  __syncthreads();
  route_finish(s.rs, P, tid, kThreads);
  tc::tc_fence_after();
  tc::fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) { trace_at(P, 1); trace_clk(P, 7); }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const uint32_t tmem = s.tmem_base;
  const int G = gridDim.x, cta = blockIdx.x;
  Plan pl;
  pl.init(s.rs.nact, P.H, P.I, G, cta);
  volatile int* abort = &s.abort;
  const int T = P.T;
  const size_t w13_bytes = (size_t)P.I * P.H, s13_count = (size_t)2 * P.I * pl.nH;
  const size_t w2_bytes = (size_t)P.H * P.I / 2, s2_count = (size_t)P.H * pl.nI;
  auto stage_w = [&](int st) { return ring + (size_t)st * kStageBytes; };
  auto stage_s = [&](int st) { return ring + (size_t)st * kStageBytes + kStageW; };
  auto stage_h = [&](int st) { return ring + (size_t)st * kStageBytes + kStageW + kStageS; };
  const int nrg = T > 8 ? 2 : 1;               // 8-token row groups of the h operand
  const int a_base2 = pl.e1 - pl.b1;           // tile counter of this CTA's first phase-2 tile

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    // Lane 0 posts the expected bytes; lanes 0..3 issue the copies of a stage side by side.
    const uint64_t pol = tc::policy_evict_first();
    int it = 0;
    bool ok = true, h_ready = false;
    int first2 = -1;                         // stage index of the first phase-2 stage
    int pend_n = 0, pend_st[kMaxStages], pend_u[kMaxStages], pend_len[kMaxStages];
    int h_issued[kMaxStages];                // h copies issued per slot (for the final drain)
    for (int i = 0; i < kMaxStages; ++i) h_issued[i] = 0;
    const int h_target = pl.m * pl.nI;
    auto issue_h = [&](int st, int u, int n) {
      const int j = (u % pl.tpr2) / pl.nI, g0 = u % pl.nI;
      if (lane == 0) tc::mbar_arrive_expect_tx(&s.hfull[st], (uint32_t)(n * kHTile * nrg));
      __syncwarp();
      if (lane < nrg)
        tc::bulk_g2s(stage_h(st) + lane * (kTilesPerStage * kHTile),
                     P.hbuf + ((size_t)(j * 2 + lane) * pl.nI + g0) * kHTile, (uint32_t)(n * kHTile), &s.hfull[st], pol);
      ++h_issued[st];
    };
    auto poll_h = [&]() -> bool {            // warp-uniform
      int v = 0;
      if (lane == 0) v = tc::ld_acquire(P.hdone) >= h_target;
      return __shfl_sync(kFull, v, 0) != 0;
    };
    auto wait_h = [&]() -> bool {            // every feature block's h is in global memory
      int okw = 1;
      if (lane == 0) {
        const long long t0 = clock64();
        while (tc::ld_acquire(P.hdone) < h_target) {
          if (*abort || clock64() - t0 > tc::kWaitTimeoutCycles) {
            trace_val(P, 8, tc::ld_acquire(P.hdone));
            trace_val(P, 9, h_target);
            okw = 0;
            break;
          }
          __nanosleep(64);
        }
      }
      return __shfl_sync(kFull, okw, 0) != 0;
    };
    auto flush_h = [&]() -> bool {
      if (!h_ready) {
        if (!wait_h()) return false;
        fence_proxy_async_global();
        h_ready = true;
        if (lane == 0) trace_at(P, 4);
      }
      for (int i = 0; i < pend_n; ++i) issue_h(pend_st[i], pend_u[i], pend_len[i]);
      pend_n = 0;
      return true;
    };
    for (int phase = 1; phase <= 2 && ok; ++phase) {
      const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
      if (phase == 2 && ub < ue) first2 = it;
      for (int u = ub; u < ue; ++it) {
        const int n = phase == 1 ? pl.run1(u) : pl.run2(u);
        const int st = it % NS;
        // the slot about to be reused may hold a phase-2 stage still waiting for its h
        if (!h_ready && first2 >= 0 && it >= NS && it - NS >= first2 && !flush_h()) { ok = false; break; }
        if (!warp_wait(&s.empty[st], ((it / NS) & 1) ^ 1, abort)) { ok = false; break; }
        int j, lt;
        pl.locate(phase, u, j, lt);
        const int sl = s.rs.sl[j];
        const uint8_t* wsrc = phase == 1 ? P.w13 + (size_t)sl * w13_bytes : P.w2 + (size_t)sl * w2_bytes;
        const uint16_t* ssrc = phase == 1 ? P.s13 + (size_t)sl * s13_count : P.s2 + (size_t)sl * s2_count;
        if (lane == 0) tc::mbar_arrive_expect_tx(&s.full[st], (uint32_t)(n * (kTileBytes + kRowBlock * 2)));
        __syncwarp();
        if (lane == 0) tc::bulk_g2s(stage_w(st), wsrc + (size_t)lt * kTileBytes, (uint32_t)(n * kTileBytes), &s.full[st], pol);
        if (lane == 1) tc::bulk_g2s(stage_s(st), ssrc + (size_t)lt * kRowBlock, (uint32_t)(n * kRowBlock * 2), &s.full[st], pol);
        if (lane == 0 && it < 4) trace_clk(P, 12 + it);
        if (phase == 2) {
          if (!h_ready && poll_h()) {
            fence_proxy_async_global();
            h_ready = true;
            if (lane == 0) trace_at(P, 4);
          }
          if (h_ready) {
            if (!flush_h()) { ok = false; ++it; break; }
            issue_h(st, u, n);
          } else {
            pend_st[pend_n] = st; pend_u[pend_n] = u; pend_len[pend_n] = n; ++pend_n;
          }
        }
        u += n;
      }
    }
    if (lane == 0) trace_at(P, 3);
    if (ok && pend_n > 0 && !flush_h()) ok = false;
    if (!ok && lane == 0) report_abort(s, P, kSiteHDone);
    // no bulk copy may still be landing in shared memory when the CTA leaves
    if (lane == 0) {
      volatile int never = 0;
      const int nw = it < NS ? it : NS;
      for (int i = 0; i < nw; ++i) {
        const int jst = it - 1 - i;
        tc::mbar_wait(&s.full[jst % NS], (jst / NS) & 1, &never);
      }
      for (int st = 0; st < NS; ++st)
        if (h_issued[st] > 0) tc::mbar_wait(&s.hfull[st], (h_issued[st] - 1) & 1, &never);
    }
    __syncwarp();
  } else if (warp == kIssuerWarp0 || warp == kIssuerWarp1) {
    // ------------------------------------------------------------ MMA issuers
    // issuer `me` takes the tiles whose running index has parity `me` and accumulates them into
    // its own accumulators; the epilogue adds the two partial sums of each block.
    const int me = warp == kIssuerWarp0 ? 0 : 1;
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(128, kN);
      const uint32_t xbase = tc::smem_u32(xs);
      int it = 0, a_it = 0, sg = 0;
      uint32_t hphase = 0;                      // bit st: parity of the next hfull[st] completion
      bool ok = true, started = false;
      for (int phase = 1; phase <= 2 && ok; ++phase) {
        const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
        const int per = phase == 1 ? pl.nH : pl.tpr2;
        for (int u = ub; u < ue && ok; ++it) {
          const int n = phase == 1 ? pl.run1(u) : pl.run2(u);
          const int st = it % NS;
          uint32_t hb = 0;
          if (phase == 2) {
            if (!tc::mbar_wait(&s.hfull[st], (hphase >> st) & 1, abort)) { ok = false; report_abort(s, P, kSiteH); break; }
            hphase ^= 1u << st;
            tc::tc_fence_after();
            hb = tc::smem_u32(stage_h(st));
          }
          for (int i = 0; i < n; ++i, ++a_it) {
            const int uu = u + i;
            const bool seg_first = uu == ub || uu % per == 0;
            const bool seg_last = uu == ue - 1 || (uu + 1) % per == 0;
            const int ac = sg % kAcc;
            if (seg_first) {
              started = false;
              if (!tc::mbar_wait(&s.accempty[me][ac], ((sg / kAcc) & 1) ^ 1, abort)) { ok = false; report_abort(s, P, kSiteAcc); break; }
              tc::tc_fence_after();
            }
            if ((a_it & 1) == me) {
              const int ab = a_it % kABufs;
              if (!tc::mbar_wait(&s.afull[ab], (a_it / kABufs) & 1, abort)) { ok = false; report_abort(s, P, kSiteABuf); break; }
              tc::tc_fence_after();
              if (a_it < 8) trace_clk(P, 40 + a_it);
              const uint32_t a = tmem + kAColBase + ab * 64, d = tmem + kAccCol + (me * kAcc + ac) * kN;
              if (phase == 1) {
                const int g = uu % pl.nH;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  const uint64_t bdesc = tc::smem_desc(xbase + (uint32_t)((g * kGroup + kk * 16) / 8) * 256u, 256, 128, 0);
                  tc::mma_ts(d, a + kk * 8, bdesc, idesc, (started || kk > 0) ? 1u : 0u);
                }
              } else {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                  const uint64_t bdesc = tc::smem_desc(hb + (uint32_t)(i * kHTile + kk * 256), 128,
                                                       kTilesPerStage * kHTile, 0);
                  tc::mma_ts(d, a + kk * 8, bdesc, idesc, (started || kk > 0) ? 1u : 0u);
                }
              }
              started = true;
              tc::mma_commit(&s.aempty[ab]);
              if (a_it < 8) trace_clk(P, 48 + a_it);
            }
            if (seg_last) {
              tc::mma_commit(&s.accfull[me][ac]);
              ++sg;
            }
          }
          if (!ok) break;
          tc::mma_commit(&s.empty[st]);     // the stage's h operand is no longer read by this issuer
          u += n;
        }
      }
      tc::mma_commit(&s.drain[me]);
      volatile int never = 0;
      if (!tc::mbar_wait(&s.drain[me], 0, &never)) report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteDrain);
    }
    __syncwarp();
  } else if (warp >= kDqWarp0 && warp < kDqWarp0 + 2 * kDqWarpsPerGroup) {
    // ------------------------------------------------------------ dequantisers -> TMEM
    // two groups of four warps take alternate tiles (group = parity of the running tile index),
    // a thread owns one row of its group's tiles; every stage barrier is waited for in order
    const int quarter = warp & 3, grp = (warp - kDqWarp0) / kDqWarpsPerGroup;
    const int r = quarter * 32 + lane;
    const uint32_t taddr_row = tmem + ((uint32_t)(quarter * 32) << 16) + kAColBase;
    const __nv_bfloat162 off136 = __floats2bfloat162_rn(136.f, 136.f);
    int it = 0, a_it = 0;
    bool ok = true;
    for (int phase = 1; phase <= 2 && ok; ++phase) {
      const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
      for (int u = ub; u < ue && ok; ++it) {
        const int n = phase == 1 ? pl.run1(u) : pl.run2(u);
        u += n;
        const int st = it % NS;
        if (!warp_wait(&s.full[st], (it / NS) & 1, abort)) { ok = false; break; }
        const uint8_t* sw = stage_w(st) + r * 16;
        const uint16_t* ss = reinterpret_cast<const uint16_t*>(stage_s(st));
        // my tiles in this stage: i = first, first + 2, ...; the stage is released after the
        // loads of the last of them (or at once when there is none)
        const int first = (a_it & 1) == grp ? 0 : 1;
        const int last = (first < n) ? first + ((n - 1 - first) & ~1) : -1;
        if (last < 0) {
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&s.empty[st]);
        }
        for (int i = first; i < n; i += 2) {
          const int ai = a_it + i;
          uint4 c[4];
#pragma unroll
          for (int kq = 0; kq < 4; ++kq) c[kq] = *reinterpret_cast<const uint4*>(sw + i * kTileBytes + kq * 2048);
          const uint32_t sb = ss[i * kRowBlock + r];
          if (i == last) {
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&s.empty[st]);
          }
          const uint32_t s2u = sb | (sb << 16);
          const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&s2u);
          const int ab = ai % kABufs;
          if (!warp_wait(&s.aempty[ab], ((ai / kABufs) & 1) ^ 1, abort)) { ok = false; break; }
          tc::tc_fence_after();
          if (quarter == 0 && lane == 0 && ai < 8) trace_clk(P, 24 + ai);
          dequant_half(c[0], c[1], s2, off136, taddr_row + ab * 64);
          dequant_half(c[2], c[3], s2, off136, taddr_row + ab * 64 + 32);
          tc::tmem_wait_st();
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&s.afull[ab]);
          if (quarter == 0 && lane == 0 && ai < 8) trace_clk(P, 32 + ai);
        }
        a_it += n;
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogues (warps 2..5)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;          // accumulator row (TMEM lane)
    const int etid = tid - kEpiWarp0 * 32;      // 0..127
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    const int nI = pl.nI;
    int sg = 0;
    bool stop = false;
    // Each decision is taken by one thread between two named barriers and read by all, so the
    // four warps always meet at the same barriers.
    for (int phase = 1; phase <= 2 && !stop; ++phase) {
      const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
      if (ub >= ue) continue;
      const int per = phase == 1 ? pl.nH : pl.tpr2;
      const int a0 = phase == 1 ? 0 : a_base2;
      for (int key = ub / per; key <= (ue - 1) / per; ++key, ++sg) {
        const int ac = sg % kAcc;
        // tiles of this block in the CTA's running tile index; which issuers had some
        const int t0 = max(ub, key * per), t1 = min(ue, (key + 1) * per);
        const int af = a0 + (t0 - ub);
        const bool has0 = (t1 - t0) >= 2 || (af & 1) == 0, has1 = (t1 - t0) >= 2 || (af & 1) == 1;
        bool ok = warp_wait(&s.accfull[0][ac], (sg / kAcc) & 1, abort);
        ok = ok && warp_wait(&s.accfull[1][ac], (sg / kAcc) & 1, abort);
        if (etid == 0 && sg < 8) trace_clk(P, 56 + sg);
        float* part = (phase == 1 ? P.p1 : P.p2) + (size_t)(key + cta) * T * kRowBlock;
        if (ok) {
          tc::tc_fence_after();
          uint32_t v0[kN], v1[kN];
          tc::tmem_ld16(trow + kAccCol + ac * kN, v0);
          tc::tmem_ld16(trow + kAccCol + (kAcc + ac) * kN, v1);
          tc::tmem_wait_ld();
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            tc::mbar_arrive(&s.accempty[0][ac]);
            tc::mbar_arrive(&s.accempty[1][ac]);
          }
#pragma unroll
          for (int t = 0; t < kN; ++t)
            if (t < T)
              part[t * kRowBlock + r] = (has0 ? __uint_as_float(v0[t]) : 0.f) + (has1 ? __uint_as_float(v1[t]) : 0.f);
          __threadfence();
        }
        tc::named_bar_sync(1, 128);
        if (etid == 0) s.epi_dec = *abort ? -1 : (block_arrive(pl, P, phase, key) ? 1 : 0);
        tc::named_bar_sync(1, 128);
        const int d = s.epi_dec;
        if (etid == 0) trace_val(P, 10, sg + 1);
        if (d < 0) { stop = true; break; }
        if (d == 1 && phase == 1) {
          // h = w * silu(gate) * up for feature block fb of selected expert j, as bf16 h tiles
          const int j = key / (2 * nI), fb = (key % (2 * nI)) % nI;
          if (etid < T) s.wsel[etid] = route_weight(s.rs, P, etid, s.rs.act[j]);
          tc::named_bar_sync(1, 128);
          float g[kN], up[kN];
          gate_up_sums<kN>(pl, P, j, fb, etid, g, up);
#pragma unroll
          for (int t = 0; t < kN; ++t) {
            if (t < T) {
              const float w = s.wsel[t];
              const float hv = (w != 0.f) ? swiglu(g[t], up[t]) * w : 0.f;
              uint8_t* dst = P.hbuf + ((size_t)(j * 2 + (t >> 3)) * nI + fb) * kHTile;
              *reinterpret_cast<__nv_bfloat16*>(dst + (etid >> 3) * 128 + (t & 7) * 16 + (etid & 7) * 2) =
                  __float2bfloat16_rn(hv);
            }
          }
          fence_proxy_async_global();
          __threadfence();
          tc::named_bar_sync(1, 128);
          if (etid == 0) tc::red_release_add(P.hdone, 1);
        } else if (d == 1) {
          output_block<kN>(pl, P, key, etid);
        }
      }
    }
    if (etid == 0) trace_at(P, 5);
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc<kTmemCols>(tmem);
  }
  finish_launch(pl, P, abort, tid, kThreads);
}

size_t fixed_smem_bytes(int H) { return sizeof(DecSmem) + (size_t)kN * H * 2; }
int decode_stages(int H) {
  const long avail = (long)kSmemLimit - (long)fixed_smem_bytes(H);
  return (int)std::min<long>(kMaxStages, avail > 0 ? avail / kStageBytes : 0);
}
size_t decode_smem_bytes(int H) { return fixed_smem_bytes(H) + (size_t)decode_stages(H) * kStageBytes; }

// h bytes per (selected expert, K group of I): the larger of the two kernels' layouts
size_t hbuf_per_tile(int T) { return std::max<size_t>(2 * kHTile, mma_hbuf_per_tile(std::min(T, kMmaMaxT))); }

int launch_tensor(const DecParams& P0, int grid, cudaStream_t s) {
  DecParams P = P0;
  P.nstages = decode_stages(P.H);
  const size_t smem = decode_smem_bytes(P.H);
  static bool attr_done = false;
  if (!attr_done) {
    if (int rc = check_cuda(cudaFuncSetAttribute(moe_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kSmemLimit), "fused decode: smem attribute"))
      return rc;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, moe_decode_kernel, P);
  note_launch();
  return check_cuda(e, "moe_decode_kernel launch");
}

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
  return (a.T <= dec::kMmaMaxT && !a.tc_decode) ? dec::mma_stages(a.T, a.H) >= 2 : dec::decode_stages(a.H) >= 2;
}

size_t decode_scratch_bytes(int T, int H, int I, int E, int k) {
  if (T < 1 || T > dec::kMaxT || H % kRowBlock || I % kRowBlock || E < 1 || k < 1) return 0;
  return dec::dec_scratch(T, H, I, E, k, dec::hbuf_per_tile(T)).total;
}

// Bytes at the start of the fused-decode scratch that hold counters (zero between launches).
size_t decode_counters_bytes(int T, int H, int I, int E, int k) {
  if (decode_scratch_bytes(T, H, I, E, k) == 0) return 0;
  return dec::dec_scratch(T, H, I, E, k, dec::hbuf_per_tile(T)).p1;
}

// One token runs on the single-token kernel, up to sixteen on the warp-MMA kernel, unless the
// tcgen05 one is asked for.
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
  P.hcnt = reinterpret_cast<int*>(d + D.hcnt);
  P.fcnt = reinterpret_cast<int*>(d + D.fcnt);
  P.hdone = reinterpret_cast<int*>(d + D.hdone);
  P.p1 = reinterpret_cast<float*>(d + D.p1);
  P.p2 = reinterpret_cast<float*>(d + D.p2);
  P.hbuf = reinterpret_cast<uint8_t*>(d + D.hbuf);
  P.mul16 = 65536u;
  P.trace = dec::g_trace;
  if (!a.logits && (!a.idx || !a.wts)) return fail(MOE_ERR_ARG, "fused decode: routing missing");

  const int m_max = std::min(a.E, a.T * a.k);
  const long tiles1 = (long)m_max * 2 * (a.I / kRowBlock) * (a.H / kGroup);
  const int grid = (int)std::max<long>(1, std::min<long>(std::min(dec::num_sms(), dec::kMaxGrid), tiles1));
  if (a.tc_decode || a.T > dec::kMmaMaxT) return dec::launch_tensor(P, grid, s);
  if (dec::rows_supported(a.T, a.H, a.I, a.E, a.k)) return dec::launch_decode_rows(P, dec::num_sms(), s);
  return dec::launch_decode_mma(P, grid, s);
}

}  // namespace moe
