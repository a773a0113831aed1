// CUDA-core fused decode kernel for batches of at most four tokens: routing, gate/up with
// SiLU*up, down projection and the router-weighted combine in ONE launch ("Every Expert Counts:
// ExactMoE for Memory-Efficient W4A16 Inference", Abstract: all selected experts execute through
// fused grouped MoE kernels; the router's top-k is unchanged).
//
// With one to four tokens the layer is a matrix-vector product over every selected expert's
// packed weights, bound by HBM bandwidth. On sm_100a one tcgen05.mma with M = 128, K = 16 costs
// its issuing thread about as much at N = 16 as at N = 256, so a tensor-core path moves at most
// ~2 KB of int4 weights per MMA issue and is issue/latency bound at this batch size; plain FP32
// FMAs on the CUDA cores keep up with the stream instead. The work split, partials and
// reductions are those of decode_common.cuh.
//
// Dequantisation with few integer operations (the integer pipe, at half the FP32 rate, is what
// bounds this kernel). For a packed word w, t = ((w >> 4p) & 0x000F000F) | 0x43004300 holds the
// bf16 values 128 + c of the two codes at bits 4p and 16 + 4p (elements 2p and 2p + 1). Then:
//  * t << 16, read as fp32, is exactly 128 + c_lo;
//  * t itself, read as fp32, is 128 + c_hi + (17152 + c_lo) / 65536: the constant 17152/65536
//    is folded into the correction below, and the residue c_lo / 65536 <= 2.3e-4 perturbs the
//    high element's weight by at most 2.3e-4 * s (bf16 rounding of q * s, which the tensor-core
//    path accepts, is up to 8 * s / 256 = 0.031 * s).
// Eight codes cost three shifts, four LOP3s and four multiplies by 65536 (IMAD instead of a
// fourth kind of shift: on sm_100a shifts are the scarcest integer operation here). The products are accumulated in
// fp32 with packed two-lane FMAs (fma.rn.f32x2), the offsets are removed once per 32 codes with
// a precomputed correction sum_k o_k x_k (o = 136 for even, 136 + 17152/65536 for odd elements),
// and the group's bf16 scale is applied once per 32 codes.
#include "decode_common.cuh"

namespace moe {
namespace dec {
namespace {

constexpr int kGWarps = 19;                // warp 0 producer, warps 1..16 compute, 17..18 epilogue
constexpr int kGThreads = kGWarps * 32;
constexpr int kGComputeWarps = 16;
constexpr int kGEpiWarp = 17;
constexpr int kGMaxStages = 6;
constexpr int kXq = 36;                    // floats per (K quarter, token): 32 operands, correction, pad

template <int TT>
struct Cfg {
  static constexpr int kHTile = 4 * TT * kXq * 4;          // h bytes per (expert, K group)
  static constexpr int kStageH = kTilesPerStage * kHTile;
  static constexpr int kStageBytes = kStageW + kStageS + kStageH;
};

struct __align__(128) GSmem {
  uint64_t full[kGMaxStages], empty[kGMaxStages], hfull[kGMaxStages];
  RouteSmem rs;
  uint64_t redfull[2], redempty[2];
  float red[2][4][kGemvMaxT][kRowBlock];  // per-quarter sums at the end of a block (two buffers)
  int abort;
  // followed in dynamic shared memory by the arranged activations
  // [H/32 quarters][TT][kXq] fp32 and the stage ring
};

// Offset removed from element e's product (see the dequantisation note above).
constexpr float kOffEven = 136.f, kOffOdd = 136.26171875f;

// One warp stores 32 consecutive operands (lane = K offset in the quarter) of one token; lane 0
// also stores the correction sum over the lanes of offset * operand.
__device__ __forceinline__ void arrange32(float* dst, float v, int lane) {
  dst[lane] = v;
  float c = ((lane & 1) ? kOffOdd : kOffEven) * v;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(kFull, c, o);
  if (lane == 0) dst[32] = c;
}

// One 128 x 128 tile, this thread's row and K quarter: seg[t] += s * sum_k q_k x_k[t].
template <int TT>
__device__ __forceinline__ void tile_dot(uint4 wv, float s, const float* xb, uint32_t mul16, float (&seg)[TT]) {
  float ax[TT], ay[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) { ax[t] = 0.f; ay[t] = 0.f; }
  const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t w = words[j];
    float lo[4], hi[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const uint32_t t = ((w >> (4 * p)) & 0x000F000Fu) | 0x43004300u;
      lo[p] = __uint_as_float(t * mul16);    // element 2p, exact (an IMAD: the shift pipe is the busier)
      hi[p] = __uint_as_float(t);            // element 2p + 1, offset folded in the correction
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const float4 xa = *reinterpret_cast<const float4*>(xb + t * kXq + j * 8);
      const float4 xc = *reinterpret_cast<const float4*>(xb + t * kXq + j * 8 + 4);
      ffma2(ax[t], ay[t], lo[0], hi[0], xa.x, xa.y);
      ffma2(ax[t], ay[t], lo[1], hi[1], xa.z, xa.w);
      ffma2(ax[t], ay[t], lo[2], hi[2], xc.x, xc.y);
      ffma2(ax[t], ay[t], lo[3], hi[3], xc.z, xc.w);
    }
  }
#pragma unroll
  for (int t = 0; t < TT; ++t) seg[t] = fmaf(s, (ax[t] + ay[t]) - xb[t * kXq + 32], seg[t]);
}

// sum over c = c0..c1 (in that order) of partial entry (base + c), rows q*32 + lane of each
// quarter q, tokens t < T: the loads of up to KB entries are issued before any is summed.
template <int TT, int KB>
__device__ __forceinline__ void sum_partials(const float* P0, int base, int c0, int c1, int T, int lane,
                                             float (&acc)[4][TT]) {
  for (int cb = c0; cb <= c1; cb += KB) {
    float v[KB][4][TT];
#pragma unroll
    for (int e = 0; e < KB; ++e) {
      const float* pp = P0 + (size_t)(base + cb + e) * T * kRowBlock + lane;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int t = 0; t < TT; ++t)
          v[e][q][t] = (cb + e <= c1 && t < T) ? __ldcg(pp + t * kRowBlock + q * 32) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < KB; ++e)
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int t = 0; t < TT; ++t) acc[q][t] += v[e][q][t];
  }
}

// The same for two ranges at once (gate and up partials of a feature block): each round issues
// the loads of up to KB entries of both before summing, each range in its own order.
template <int TT, int KB>
__device__ __forceinline__ void sum_partials2(const float* P0, int ba, int a0, int a1, float (&acc_a)[4][TT], int bb,
                                              int b0, int b1, float (&acc_b)[4][TT], int T, int lane) {
  for (int r = 0; a0 + r * KB <= a1 || b0 + r * KB <= b1; ++r) {
    float va[KB][4][TT], vb[KB][4][TT];
#pragma unroll
    for (int e = 0; e < KB; ++e) {
      const int ca = a0 + r * KB + e, cb = b0 + r * KB + e;
      const float* pa = P0 + (size_t)(ba + ca) * T * kRowBlock + lane;
      const float* pb = P0 + (size_t)(bb + cb) * T * kRowBlock + lane;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          va[e][q][t] = (ca <= a1 && t < T) ? __ldcg(pa + t * kRowBlock + q * 32) : 0.f;
          vb[e][q][t] = (cb <= b1 && t < T) ? __ldcg(pb + t * kRowBlock + q * 32) : 0.f;
        }
    }
#pragma unroll
    for (int e = 0; e < KB; ++e)
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          acc_a[q][t] += va[e][q][t];
          acc_b[q][t] += vb[e][q][t];
        }
  }
}

template <int TT>
__global__ void __launch_bounds__(kGThreads, 1) moe_decode_gemv_kernel(const __grid_constant__ DecParams P) {
  using C = Cfg<TT>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  GSmem& s = *reinterpret_cast<GSmem*>(smem_raw);
  float* xs = reinterpret_cast<float*>(smem_raw + sizeof(GSmem));
  const int nq = P.H / 32;                               // K quarters of H
  uint8_t* ring = reinterpret_cast<uint8_t*>(xs + (size_t)nq * TT * kXq);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NS = P.nstages;

  if (tid == 0) trace_clk(P, 60);
  // ---- set-up that does not read the previous kernel's results: overlaps it under PDL
  if (warp == 0) {
    if (lane < kGMaxStages) {
      tc::mbar_init(&s.full[lane], 1);
      tc::mbar_init(&s.empty[lane], kGComputeWarps);
      tc::mbar_init(&s.hfull[lane], 1);
    }
    if (lane < 2) {
      tc::mbar_init(&s.redfull[lane], kGComputeWarps);
      tc::mbar_init(&s.redempty[lane], 1);
    }
    if (lane == 0) s.abort = 0;
    tc::fence_barrier_init();
  }
  route_clear(s.rs, tid, kGThreads);
  __syncthreads();

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) trace_at(P, 0);
  if (tid == 0) trace_clk(P, 61);
  // activations, arranged per (K quarter, token); tokens >= T are zero. A warp loads up to eight
  // blocks at a time; the first loads are issued before the routing so the latencies overlap.
  {
    float v[8];
    auto load8 = [&](int b0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int b = b0 + i * kGWarps, q = b / TT, t = b % TT;
        v[i] = (b < nq * TT && t < P.T) ? bf16_bits_to_float(P.x[(size_t)t * P.H + q * 32 + lane]) : 0.f;
      }
    };
    load8(warp);
    route_begin(s.rs, P, tid, kGThreads);
    if (tid == 0) trace_clk(P, 62);
    for (int b0 = warp; b0 < nq * TT; b0 += 8 * kGWarps) {
      if (b0 != warp) load8(b0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int b = b0 + i * kGWarps;
        if (b < nq * TT) arrange32(xs + (size_t)b * kXq, v[i], lane);
      }
    }
  }
  __syncthreads();
  if (tid == 0) trace_clk(P, 63);
  route_finish(s.rs, P, tid, kGThreads);
  if (tid == 0) { trace_at(P, 1); trace_clk(P, 7); }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int G = gridDim.x, cta = blockIdx.x;
  Plan pl;
  pl.init(s.rs.nact, P.H, P.I, G, cta);
  volatile int* abort = &s.abort;
  const int T = P.T;
  const size_t w13_bytes = (size_t)P.I * P.H, s13_count = (size_t)2 * P.I * pl.nH;
  const size_t w2_bytes = (size_t)P.H * P.I / 2, s2_count = (size_t)P.H * pl.nI;
  auto stage_w = [&](int st) { return ring + (size_t)st * C::kStageBytes; };
  auto stage_s = [&](int st) { return ring + (size_t)st * C::kStageBytes + kStageW; };
  auto stage_h = [&](int st) { return ring + (size_t)st * C::kStageBytes + kStageW + kStageS; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    // lane 0 posts the expected bytes; lanes 0..2 issue the copies of a stage side by side
    const uint64_t pol = tc::policy_evict_first();
    int it = 0;
    bool ok = true, h_ready = false;
    int first2 = -1;
    int pend_n = 0, pend_st[kGMaxStages], pend_u[kGMaxStages], pend_len[kGMaxStages];
    int h_issued[kGMaxStages];
    for (int i = 0; i < kGMaxStages; ++i) h_issued[i] = 0;
    const int h_target = pl.m * pl.nI;
    auto issue_h = [&](int st, int u, int n) {
      const int j = (u % pl.tpr2) / pl.nI, g0 = u % pl.nI;
      if (lane == 0) tc::mbar_arrive_expect_tx(&s.hfull[st], (uint32_t)(n * C::kHTile));
      __syncwarp();
      if (lane == 2)
        tc::bulk_g2s(stage_h(st), P.hbuf + ((size_t)j * pl.nI + g0) * C::kHTile, (uint32_t)(n * C::kHTile),
                     &s.hfull[st], pol);
      ++h_issued[st];
    };
    auto poll_h = [&]() -> bool {
      int v = 0;
      if (lane == 0) v = tc::ld_acquire(P.hdone) >= h_target;
      return __shfl_sync(kFull, v, 0) != 0;
    };
    auto wait_h = [&]() -> bool {
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
        if (lane == 0) { trace_at(P, 4); trace_clk(P, 56); }
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
        const int sl = slot_of(P.slot, s.rs.act[j]);
        const uint8_t* wsrc = phase == 1 ? P.w13 + (size_t)sl * w13_bytes : P.w2 + (size_t)sl * w2_bytes;
        const uint16_t* ssrc = phase == 1 ? P.s13 + (size_t)sl * s13_count : P.s2 + (size_t)sl * s2_count;
        if (lane == 0) tc::mbar_arrive_expect_tx(&s.full[st], (uint32_t)(n * (kTileBytes + kRowBlock * 2)));
        __syncwarp();
        if (lane == 0) tc::bulk_g2s(stage_w(st), wsrc + (size_t)lt * kTileBytes, (uint32_t)(n * kTileBytes), &s.full[st], pol);
        if (lane == 1) tc::bulk_g2s(stage_s(st), ssrc + (size_t)lt * kRowBlock, (uint32_t)(n * kRowBlock * 2), &s.full[st], pol);
        if (lane == 0 && it < 8) trace_clk(P, 48 + it);
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
    if (!ok && lane == 0) {
      s.abort = 1;
      report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteHDone);
    }
    if (lane == 0) {   // no bulk copy may still be landing in shared memory when the CTA leaves
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
  } else if (warp <= kGComputeWarps) {
    // ------------------------------------------------------------ compute warps 1..16
    // warp cw = warp - 1 owns K quarter cw / 4 and rows 32 * (cw % 4) .. of every tile. At the end
    // of a block the four quarter sums of each row go to shared memory (two buffers) for the
    // epilogue warp; the compute warps go on with the next tiles.
    const int cw = warp - 1, kq = cw >> 2, r = (cw & 3) * 32 + lane;
    float seg[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) seg[t] = 0.f;
    int it = 0, nblk = 0;
    uint32_t hphase = 0;
    bool ok = true;
    for (int phase = 1; phase <= 2 && ok; ++phase) {
      const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
      const int per = phase == 1 ? pl.nH : pl.tpr2;
      for (int u = ub; u < ue && ok; ++it) {
        const int n = phase == 1 ? pl.run1(u) : pl.run2(u);
        const int st = it % NS;
        if (!warp_wait(&s.full[st], (it / NS) & 1, abort)) { ok = false; break; }
        if (phase == 2) {
          if (!warp_wait(&s.hfull[st], (hphase >> st) & 1, abort)) { ok = false; break; }
          hphase ^= 1u << st;
        }
        if (lane == 0 && cw == 0 && it < 8) trace_clk(P, 16 + it);
        const uint8_t* sw = stage_w(st) + kq * 2048 + r * 16;
        const uint16_t* ss = reinterpret_cast<const uint16_t*>(stage_s(st));
        const float* hsl = reinterpret_cast<const float*>(stage_h(st));
        // block bookkeeping once per stage: where the current block ends
        int blk_end = min(ue, (u / per + 1) * per);
        int g = u % pl.nH;                         // K group of tile u (phase 1)
        for (int i = 0; i < n; ++i, ++g) {
          if (g == pl.nH) g = 0;
          const uint4 wv = *reinterpret_cast<const uint4*>(sw + i * kTileBytes);
          const float sc = __uint_as_float((uint32_t)ss[i * kRowBlock + r] << 16);
          const float* xb = phase == 1 ? xs + ((size_t)(g * 4 + kq) * TT) * kXq
                                       : hsl + ((size_t)(i * 4 + kq) * TT) * kXq;
          tile_dot<TT>(wv, sc, xb, P.mul16, seg);
          if (u + i + 1 == blk_end) {
            const int b = nblk & 1;
            if (nblk >= 2 && !warp_wait(&s.redempty[b], ((nblk >> 1) - 1) & 1, abort)) { ok = false; break; }
#pragma unroll
            for (int t = 0; t < TT; ++t) { s.red[b][kq][t][r] = seg[t]; seg[t] = 0.f; }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&s.redfull[b]);
            ++nblk;
            blk_end = min(ue, blk_end + per);
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.empty[st]);
        if (lane == 0 && cw == 0 && it < 8) trace_clk(P, 24 + it);
        u += n;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    // epilogue warp ew takes the blocks written to quarter-sum buffer ew (every other block), so
    // the reductions of consecutive blocks run side by side: quarter sums -> this CTA's partial;
    // the arrival that completes a block does its reduction (h of a feature block, or an output
    // row block).
    const int ew = warp - kGEpiWarp;
    int nblk = 0, nh = 0;
    for (int phase = 1; phase <= 2; ++phase) {
      const int ub = phase == 1 ? pl.b1 : pl.b2, ue = phase == 1 ? pl.e1 : pl.e2;
      if (ub >= ue) continue;
      const int per = phase == 1 ? pl.nH : pl.tpr2;
      bool stop = false;
      for (int key = ub / per; key <= (ue - 1) / per; ++key, ++nblk) {
        const int b = nblk & 1;
        if (b != ew) continue;
        if (!warp_wait(&s.redfull[b], (nblk >> 1) & 1, abort)) { stop = true; break; }
        float y[4][TT];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int t = 0; t < TT; ++t) {
            const int row = q * 32 + lane;
            y[q][t] = ((s.red[b][0][t][row] + s.red[b][1][t][row]) + s.red[b][2][t][row]) + s.red[b][3][t][row];
          }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.redempty[b]);
        float* part = (phase == 1 ? P.p1 : P.p2) + (size_t)(key + cta) * T * kRowBlock;
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int t = 0; t < TT; ++t)
            if (t < T) part[t * kRowBlock + q * 32 + lane] = y[q][t];
        __syncwarp();   // the lanes' stores are ordered before lane 0's release
        int last = 0;
        if (lane == 0) last = block_arrive(pl, P, phase, key) ? 1 : 0;
        last = __shfl_sync(kFull, last, 0);
        if (nblk < 8 && lane == 0) trace_clk(P, 32 + nblk);
        if (!last) continue;
        if (phase == 1) {
          // h = w * silu(gate) * up for feature block fb of selected expert j, arranged as the
          // operand of the down projection
          const int nI = pl.nI, j = key / (2 * nI), fb = (key % (2 * nI)) % nI;
          if (lane == 0 && nh < 4) trace_clk(P, 40 + 2 * nh);
          float wt = 0.f;
          if (lane < T) wt = route_weight(s.rs, P, lane, s.rs.act[j]);
          float* dst = reinterpret_cast<float*>(P.hbuf + ((size_t)j * nI + fb) * C::kHTile);
          // gate / up sums of features q*32 + lane, partials in CTA order; the loads of one
          // partial for all four quarters are issued together
          const int Rg = j * 2 * nI + fb, Ru = Rg + nI;
          float g[4][TT], up[4][TT];
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int t = 0; t < TT; ++t) { g[q][t] = 0.f; up[q][t] = 0.f; }
          sum_partials2<TT, (TT == 1 ? 4 : 1)>(P.p1, Rg, pl.first1(Rg), pl.last1(Rg), g, Ru, pl.first1(Ru),
                                                pl.last1(Ru), up, T, lane);
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int t = 0; t < TT; ++t) {
              const float w = __shfl_sync(kFull, wt, t);
              arrange32(dst + ((size_t)q * TT + t) * kXq, (t < T && w != 0.f) ? swiglu(g[q][t], up[q][t]) * w : 0.f, lane);
            }
          fence_proxy_async_global();
          __syncwarp();   // the lanes' stores are ordered before lane 0's release
          if (lane == 0) tc::red_release_add(P.hdone, 1);
          if (lane == 0 && nh < 4) trace_clk(P, 41 + 2 * nh);
          ++nh;
        } else {
          // output row block `key`: rows q*32 + lane, partials in CTA order, then the combine
          float yo[4][TT];
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int t = 0; t < TT; ++t) yo[q][t] = 0.f;
          sum_partials<TT, (TT == 1 ? 12 : 8 / TT)>(P.p2, key, pl.first2(key), pl.last2(key), T, lane, yo);
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int t = 0; t < TT; ++t)
              if (t < T) store_output(P, t, key * kRowBlock + q * 32 + lane, yo[q][t]);
        }
      }
      if (stop) break;
    }
    if (lane == 0) trace_at(P, 5);
  }

  __syncthreads();
  finish_launch(pl, P, abort, tid, kGThreads);
}

template <int TT>
int launch_tt(const DecParams& P0, int grid, cudaStream_t s) {
  DecParams P = P0;
  P.nstages = gemv_stages(P.T, P.H);
  const size_t smem = gemv_smem_bytes(P.T, P.H);
  static bool attr_done = false;
  if (!attr_done) {
    if (int rc = check_cuda(cudaFuncSetAttribute(moe_decode_gemv_kernel<TT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kSmemLimit), "fused decode (CUDA cores): smem attribute"))
      return rc;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, moe_decode_gemv_kernel<TT>, P);
  note_launch();
  return check_cuda(e, "moe_decode_gemv_kernel launch");
}

int tt_of(int T) { return T <= 1 ? 1 : (T <= 2 ? 2 : 4); }

}  // namespace

size_t gemv_hbuf_per_tile(int T) { return (size_t)4 * tt_of(T) * kXq * 4; }

size_t gemv_smem_bytes(int T, int H) {
  const int tt = tt_of(T);
  const size_t stage = (size_t)kStageW + kStageS + (size_t)kTilesPerStage * 4 * tt * kXq * 4;
  return sizeof(GSmem) + (size_t)(H / 32) * tt * kXq * 4 + (size_t)gemv_stages(T, H) * stage;
}

int gemv_stages(int T, int H) {
  const int tt = tt_of(T);
  const long stage = (long)kStageW + kStageS + (long)kTilesPerStage * 4 * tt * kXq * 4;
  const long avail = (long)kSmemLimit - (long)sizeof(GSmem) - (long)(H / 32) * tt * kXq * 4;
  return (int)std::min<long>(kGMaxStages, avail > 0 ? avail / stage : 0);
}

int launch_decode_gemv(const DecParams& P, int grid, cudaStream_t s) {
  switch (tt_of(P.T)) {
    case 1: return launch_tt<1>(P, grid, s);
    case 2: return launch_tt<2>(P, grid, s);
    default: return launch_tt<4>(P, grid, s);
  }
}

}  // namespace dec
}  // namespace moe
