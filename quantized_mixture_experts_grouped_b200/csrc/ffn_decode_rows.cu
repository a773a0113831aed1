// Fused single-token decode kernel: routing, gate/up with SiLU*up, down projection and the
// router-weighted combine in ONE launch ("Every Expert Counts: ExactMoE for Memory-Efficient
// W4A16 Inference", Abstract: all selected experts execute through fused grouped MoE kernels;
// the router's top-k is unchanged).
//
// With one token the layer is two chains of matrix-vector products whose cost is the latency of
// their dependent steps as much as the bytes. This kernel cuts the work so that every dot
// product is completed inside one CTA, leaving a single exchange between CTAs:
//  * phase 1 (gate/up): the selected experts' W13 rows are split into slices of 32 features
//    (32 gate rows and the 32 matching up rows, all of K). A CTA takes a contiguous range of
//    slices, computes the complete gate and up sums, and writes h = w * silu(gate) * up of its
//    features, already encoded as the down projection's B operand (16-bit fixed point per
//    32-feature slice, two s8 columns: the MMA k-step of phase 2 is exactly one slice);
//  * one counter: every CTA adds 1 after its slices are written and phase 2 waits until the
//    launch's G arrivals are in. The counter only grows (64-bit): a launch's base is its value
//    at the start rounded down to a multiple of G (arrivals of the same launch are < G), so no
//    CTA resets it and no exit atomic is needed;
//  * phase 2 (down): a CTA takes 16 output rows over every selected expert and all of I, so the
//    router-weighted sum over experts and K ends in its own registers and shared memory, and the
//    bf16 output is written directly. Its W2 rows are in shared memory before h is ready.
// A slice or 16-row block is not contiguous in the packed tile layout (128 x 128 tiles of 16-byte
// row chunks, tile-major scales); a 4-D TMA tensor map (word in a 2048-byte K-quarter chunk,
// K chunk, row block, slot) fetches its codes as one box of contiguous row runs, and another
// (row, K group, row block, slot) its scales. The contraction is the int8 warp-MMA path of the other decode kernel (exact integer
// products of the codes with 16-bit fixed-point activations; decode_common.cuh). Sums run in a
// fixed order, so results are identical run to run. Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "decode_common.cuh"

namespace moe {
namespace dec {
namespace {

constexpr int kRWarps = 18;               // warp 0 producer, warps 1..16 compute, warp 17 h
constexpr int kRThreads = kRWarps * 32;
constexpr int kRCompute = 16;
constexpr int kRStages = 5;
constexpr int kRData = 32768;             // weight bytes per stage
constexpr int kRScales = 1024;            // scale bytes per stage
constexpr int kRStage = kRData + kRScales;
constexpr int kSliceF = 32;               // features per phase-1 slice (= one phase-2 k-step)
constexpr int kSliceB = 72;               // encoded h slice: hi and lo columns (32 B each), {a, a * 8 sum v}
constexpr int kORows = 16;                // output rows per phase-2 block
constexpr int kXPad = 32;                 // bytes after each activation column

struct __align__(128) RSmem {
  uint64_t full[kRStages], empty[kRStages];
  uint64_t hfull;                         // the encoded h of every slice has landed
  uint64_t redfull[2], redempty[2];       // phase-1 slice sums -> h warp
  RouteSmem rs;
  float red1[2][8][2 * kSliceF];          // [buffer][K part][gate rows, up rows]
  float red2[kRCompute][kORows];          // [warp][row] phase-2 sums
  float wsel[kMaxExperts];                // router weight of selected expert j
  int abort;
  // followed in dynamic shared memory by the activation columns [2][H + kXPad] (bytes) and their
  // group records [H/128] x 16 B, the encoded h [m][I/32] x kSliceB, and the stage ring (on a
  // 1024-byte boundary)
};

// D = A * B (zero accumulator), the m16n8k32 u8 x s8 -> s32 warp MMA.
__device__ __forceinline__ void imma0(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// 4-D tensor load: box at coordinates (x, 0, block, slot) of `map` into shared memory.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int block, int slot,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;"
      ::"r"(tc::smem_u32(dst)), "l"(map), "r"(x), "r"(0), "r"(block), "r"(slot), "r"(tc::smem_u32(bar)),
        "l"(policy)
      : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Routing epilogue of the single token, one warp (k <= 32): from the k choices in rs.idx / rs.wts,
// the selected resident experts in ascending id (rs.act, rs.sl, wsel; rank = set bits below the
// expert in the presence mask), rs.nact, and the router outputs. A token routed twice to one
// expert (given routing only) is reported and selects nothing.
__device__ void route_one(RouteSmem& rs, float* wsel, const DecParams& P, int lane) {
  const int k = P.k, E = P.E;
  int e = -1;
  float wv = 0.f;
  if (lane < k) { e = rs.idx[lane]; wv = rs.wts[lane]; }
  int sl = -1;
  if (lane < k && (unsigned)e < (unsigned)E) sl = slot_of(P.slot, e);
  const bool in = sl >= 0;
  const int n_in = __popc(__ballot_sync(kFull, in));
  const int nw = (E + 31) >> 5;
  uint32_t mw = 0;   // lane wd < nw: presence word wd
  for (int wd = 0; wd < nw; ++wd) {
    const uint32_t v = __reduce_or_sync(kFull, (in && (e >> 5) == wd) ? 1u << (e & 31) : 0u);
    if (lane == wd) mw = v;
  }
  int below = 0;
  for (int wd = 0; wd < nw; ++wd) {
    const uint32_t v = __shfl_sync(kFull, mw, wd);
    if (in && wd < (e >> 5)) below += __popc(v);
    if (in && wd == (e >> 5)) below += __popc(v & ((1u << (e & 31)) - 1u));
  }
  const int total = (int)__reduce_add_sync(kFull, (uint32_t)__popc(mw));
  const bool dup = total != n_in;
  if (in && !dup) {
    rs.act[below] = e;
    rs.sl[below] = sl;
    wsel[below] = wv;
  }
  if (lane == 0) {
    rs.nact = dup ? 0 : total;
    rs.over = dup ? 1 : 0;
    if (dup) report_status(P.ctl, MOE_ERR_ARG, kSiteOver);
  }
  if (P.logits && P.idx_out && blockIdx.x == 0 && lane < k) {
    P.idx_out[lane] = e;
    P.wts_out[lane] = wv;
  }
}

// The split of both phases, identical in every CTA.
struct RPlan {
  int m, nH, nI, nS;      // selected experts, K groups of H and I, slices per expert (I / 32)
  int eps;                // experts per phase-2 stage
  int u0, u1;             // this CTA's phase-1 slices
  int n2;                 // phase-2 stages per output block
  __device__ void init(int m_, int H, int I, int G, int c) {
    m = m_; nH = H / kGroup; nI = I / kRowBlock; nS = I / kSliceF;
    eps = nI <= 8 ? 4 : 2;
    const uint32_t U = (uint32_t)(m * nS);
    u0 = (int)((uint32_t)c * U / (uint32_t)G);
    u1 = (int)((uint32_t)(c + 1) * U / (uint32_t)G);
    n2 = (m + eps - 1) / eps;
  }
};

__global__ void __launch_bounds__(kRThreads, 1)
    moe_decode_rows_kernel(const __grid_constant__ DecParams P, const __grid_constant__ CUtensorMap m13,
                           const __grid_constant__ CUtensorMap m2, const __grid_constant__ CUtensorMap ms13,
                           const __grid_constant__ CUtensorMap ms2) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  RSmem& s = *reinterpret_cast<RSmem*>(smem_raw);
  const int H = P.H, I = P.I;
  const int nH = H / kGroup, nI = I / kRowBlock, nS = I / kSliceF;
  const int xcs = H + kXPad;                                    // activation column stride (bytes)
  uint8_t* xq = smem_raw + sizeof(RSmem);
  uint8_t* xrec = xq + 2 * xcs;
  uint8_t* hq = xrec + nH * 16;
  const int m_max = min(P.E, P.k);
  // the stage ring starts on a 1024-byte boundary of the shared address space (tensor copies)
  const uint32_t ring_at = (tc::smem_u32(hq) + (uint32_t)(m_max * nS * kSliceB) + 1023u) & ~1023u;
  uint8_t* ring = hq + (ring_at - tc::smem_u32(hq));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) trace_clk(P, 60);
  if (warp == 0) {
    if (lane < kRStages) {
      tc::mbar_init(&s.full[lane], 1);
      tc::mbar_init(&s.empty[lane], kRCompute);
    }
    if (lane < 2) {
      tc::mbar_init(&s.redfull[lane], kRCompute);
      tc::mbar_init(&s.redempty[lane], 1);
    }
    if (lane == 0) {
      tc::mbar_init(&s.hfull, 1);
      s.abort = 0;
    }
    tc::fence_barrier_init();
  }
  __syncthreads();

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) trace_at(P, 0);
  if (tid == 0) trace_clk(P, 61);
  unsigned long long* hseq = reinterpret_cast<unsigned long long*>(P.hdone + 2);
  unsigned long long seq0 = 0;   // the counter at the start (producer lane 0)
  if (tid == 0) seq0 = ld_relaxed_u64(hseq);
  // the activations of K group warp - 1 (warps 1..17) are loaded before the routing and encoded
  // as B-operand columns after it, while the producer already issues the weight copies
  float xv[4] = {0.f, 0.f, 0.f, 0.f};
  if (warp >= 1 && warp - 1 < nH)
#pragma unroll
    for (int q = 0; q < 4; ++q) xv[q] = bf16_bits_to_float(P.x[(warp - 1) * kGroup + q * 32 + lane]);
  if (warp == 0) {   // routing of the token and its grouping, one warp
    if (P.logits) {
      route_token(s.rs, P, 0, lane);
    } else if (lane < P.k) {
      s.rs.idx[lane] = P.idx_in[lane];
      s.rs.wts[lane] = P.wts_in[lane];
    }
    __syncwarp();
    if (tid == 0) trace_clk(P, 62);
    route_one(s.rs, s.wsel, P, lane);
  }
  __syncthreads();
  if (tid == 0) { trace_at(P, 1); trace_clk(P, 7); }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (warp >= 1) {
    for (int G0 = warp - 1; G0 < nH; G0 += kRWarps - 1) {
      if (G0 != warp - 1)
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = bf16_bits_to_float(P.x[G0 * kGroup + q * 32 + lane]);
      encode_group(xv, xq + G0 * kGroup, xq + xcs + G0 * kGroup, reinterpret_cast<int4*>(xrec) + G0, lane);
    }
    tc::named_bar_sync(2, (kRWarps - 1) * 32);   // the columns are complete for warps 1..17
  }

  const int G = gridDim.x, cta = blockIdx.x;
  RPlan pl;
  pl.init(s.rs.nact, H, I, G, cta);
  volatile int* abort = &s.abort;
  const int nOB = H / kORows;                                   // output blocks
  const uint32_t hq_bytes = (uint32_t)(pl.m * nS * kSliceB);
  const int sstride2 = (32 * nI + 127) & ~127;                  // bytes per expert's W2 scale box (128-aligned)

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = tc::policy_evict_first();
    int st = 0, it = 0, first2 = -1;
    uint32_t ph = 0;
    bool ok = true, h_sent = false;
    auto next = [&]() { ++it; if (++st == kRStages) { st = 0; ph ^= 1; } };
    // the encoded h of every slice: waited for (all CTAs' phase 1) and copied once
    auto send_h = [&]() -> bool {
      int okw = 1;
      if (lane == 0) {
        const long long t0 = clock64();
        const unsigned long long target = seq0 - seq0 % (unsigned long long)G + (unsigned long long)G;
        while (ld_relaxed_u64(hseq) < target) {
          if (*abort || clock64() - t0 > tc::kWaitTimeoutCycles) { okw = 0; break; }
          __nanosleep(32);
        }
        if (okw) {
          // acquire (pairs with the CTAs' release adds), then order the async-proxy copy after it
          asm volatile("fence.acq_rel.gpu;" ::: "memory");
          fence_proxy_async_global();
          trace_at(P, 4);
          trace_clk(P, 37);
          tc::mbar_arrive_expect_tx(&s.hfull, hq_bytes);
          tc::bulk_g2s(hq, P.hbuf, hq_bytes, &s.hfull, pol);
        }
      }
      h_sent = true;
      return __shfl_sync(kFull, okw, 0) != 0;
    };
    // phase-1 stage k: slice u0 + k / 2, gate (k even) or up (k odd) rows
    const int n1 = 2 * (pl.u1 - pl.u0);
    auto issue1 = [&](int k, int sst) {
      const int u = pl.u0 + (k >> 1), j = u / nS, fs = u % nS, slot = s.rs.sl[j];
      uint8_t* dst = ring + (size_t)sst * kRStage;
      const int row0 = fs * kSliceF + (k & 1) * I;               // first W13 row of the slice half
      tc::mbar_arrive_expect_tx(&s.full[sst], (uint32_t)(2048 * nH + 64 * nH));
      tma_load_4d(dst, &m13, (row0 % kRowBlock) * 4, row0 / kRowBlock, slot, &s.full[sst], pol);
      tma_load_4d(dst + kRData, &ms13, row0 % kRowBlock, row0 / kRowBlock, slot, &s.full[sst], pol);
    };
    // the first ring's worth goes out at once, one stage per lane (fresh slots need no wait)
    const int nb = min(n1, kRStages);
    if (lane < nb) issue1(lane, lane);
    __syncwarp();
    if (lane == 0) trace_clk(P, 48);
    for (int k = 0; k < nb; ++k) next();
    for (int k = nb; k < n1 && ok; ++k) {
      if (!warp_wait(&s.empty[st], ph ^ 1, abort)) { ok = false; break; }
      if (lane == 0) issue1(k, st);
      __syncwarp();
      if (lane == 0 && it < 8) trace_clk(P, 48 + it);
      next();
    }
    if (pl.m > 0) {
      for (int ob = cta; ob < nOB && ok; ob += G) {
        for (int e0 = 0; e0 < pl.m && ok; e0 += pl.eps) {
          if (first2 < 0) first2 = it;
          // the slot about to be reused may hold a phase-2 stage that needs h first
          if (!h_sent && it - kRStages >= first2 && !send_h()) { ok = false; break; }
          if (!warp_wait(&s.empty[st], ph ^ 1, abort)) { ok = false; break; }
          const int ne = min(pl.eps, pl.m - e0);
          uint8_t* dst = ring + (size_t)st * kRStage;
          if (lane == 0) tc::mbar_arrive_expect_tx(&s.full[st], (uint32_t)(ne * (1024 * nI + 32 * nI)));
          __syncwarp();
          if (lane < ne) {
            const int slot = s.rs.sl[e0 + lane];
            tma_load_4d(dst + lane * 1024 * nI, &m2, ((ob * kORows) % kRowBlock) * 4, (ob * kORows) / kRowBlock, slot,
                        &s.full[st], pol);
          }
          if (lane < ne) {
            const int slot = s.rs.sl[e0 + lane];
            tma_load_4d(dst + kRData + lane * sstride2, &ms2, (ob * kORows) % kRowBlock, (ob * kORows) / kRowBlock, slot,
                        &s.full[st], pol);
          }
          __syncwarp();
          if (lane == 0 && it < 8) trace_clk(P, 48 + it);
          next();
        }
      }
      if (ok && !h_sent && cta < nOB && !send_h()) ok = false;
    }
    if (lane == 0) trace_at(P, 3);
    if (!ok && lane == 0) {
      s.abort = 1;
      report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteHDone);
    }
    if (lane == 0) {   // no copy may still be landing in shared memory when the CTA leaves
      volatile int never = 0;
      const int nw = it < kRStages ? it : kRStages;
      for (int i = 0; i < nw; ++i) {
        const int jst = it - 1 - i;
        tc::mbar_wait(&s.full[jst % kRStages], (jst / kRStages) & 1, &never);
      }
      if (h_sent && ok) tc::mbar_wait(&s.hfull, 0, &never);
    }
    __syncwarp();
  } else if (warp <= kRCompute) {
    // ------------------------------------------------------------ compute warps 1..16
    const int w = warp - 1, g = lane >> 2, c = lane & 3;
    const uint32_t M = 0x0F0F0F0Fu;
    int st = 0, i = 0;
    uint32_t ph = 0;
    bool ok = true;
    auto next = [&]() { if (++st == kRStages) { st = 0; ph ^= 1; } };
    // phase 1: warp (mt, part) takes rows 16 mt .. + 15 of the slice half and K groups
    // [part nH / 8, (part + 1) nH / 8); lane (g, c) holds rows g, g + 8 of the 16
    const int mt = w & 1, part = w >> 1;
    const int gk0 = part * nH / 8, gk1 = (part + 1) * nH / 8;
    const int ra = 16 * mt + g;
    for (int u = pl.u0; u < pl.u1 && ok; ++u, ++i) {
      const int b = i & 1;
      if (i >= 2 && !warp_wait(&s.redempty[b], ((i >> 1) - 1) & 1, abort)) { ok = false; break; }
      for (int half = 0; half < 2; ++half) {
        if (!warp_wait(&s.full[st], ph, abort)) { ok = false; break; }
        if (w == 0 && lane == 0 && 2 * i + half < 8) trace_clk(P, 16 + 2 * i + half);
        const uint8_t* data = ring + (size_t)st * kRStage;
        const uint16_t* scl = reinterpret_cast<const uint16_t*>(data + kRData);
        float seg0 = 0.f, seg1 = 0.f;
        for (int gk = gk0; gk < gk1; ++gk) {
          int d[4] = {0, 0, 0, 0};
#pragma unroll
          for (int kq = 0; kq < 4; ++kq) {
            const uint8_t* ch = data + (gk * 4 + kq) * 512;
            const uint32_t wa = *reinterpret_cast<const uint32_t*>(ch + ra * 16 + 4 * c);
            const uint32_t wb = *reinterpret_cast<const uint32_t*>(ch + (ra + 8) * 16 + 4 * c);
            uint2 xb = make_uint2(0u, 0u);
            if (g < 2) xb = *reinterpret_cast<const uint2*>(xq + g * xcs + (gk * 16 + kq * 4 + c) * 8);
            imma(d, wa & M, wb & M, (wa >> 4) & M, (wb >> 4) & M, xb.x, xb.y);
          }
          const int4 rec = reinterpret_cast<const int4*>(xrec)[gk];
          const float a = __int_as_float(rec.y);
          const float s0 = __uint_as_float((uint32_t)scl[gk * kSliceF + ra] << 16);
          const float s1 = __uint_as_float((uint32_t)scl[gk * kSliceF + ra + 8] << 16);
          seg0 = fmaf(s0 * a, (float)(d[0] * 256 + d[1] - rec.x - rec.z), seg0);
          seg1 = fmaf(s1 * a, (float)(d[2] * 256 + d[3] - rec.x - rec.z), seg1);
        }
        if (c == 0) {   // column 0 / 1 = token 0 hi / lo
          s.red1[b][part][half * kSliceF + ra] = seg0;
          s.red1[b][part][half * kSliceF + ra + 8] = seg1;
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.empty[st]);
        if (w == 0 && lane == 0 && 2 * i + half < 8) trace_clk(P, 24 + 2 * i + half);
        next();
      }
      if (!ok) break;
      if (lane == 0) tc::mbar_arrive(&s.redfull[b]);
    }
    // phase 2: 16 output rows over every selected expert. A stage holds ne <= eps experts' W2 rows,
    // ne * nI K groups; warp w takes groups [w ne nI / 16, (w + 1) ne nI / 16). A group is four
    // chunks = four h slices, each with its own scale a: the four MMAs run side by side and
    // y += s * (sum_q a_q (256 D_hi + D_lo)_q - sum_q a_q 8 sum(v_q)).
    // (every compute warp runs the same block loop and meets the named barriers even after a
    // timeout; the waits then fail at once and the stores are skipped)
    if (pl.m > 0) {
      bool h_in = false;
      for (int ob = cta; ob < nOB; ob += G) {
        float seg0 = 0.f, seg1 = 0.f;
        for (int e0 = 0; e0 < pl.m && ok; e0 += pl.eps) {
          if (!warp_wait(&s.full[st], ph, abort)) { ok = false; break; }
          if (w == 0 && lane == 0 && e0 == pl.eps) trace_clk(P, 43);
          if (!h_in) {
            if (!warp_wait(&s.hfull, 0, abort)) { ok = false; break; }
            h_in = true;
            if (w == 0 && lane == 0) trace_clk(P, 40);
          }
          const int Gs = min(pl.eps, pl.m - e0) * nI;
          const int gb = (w * Gs) >> 4, ge = ((w + 1) * Gs) >> 4;
          int el = gb / nI, g2 = gb - el * nI;
          for (int gl = gb; gl < ge; ++gl) {
            const uint8_t* data = ring + (size_t)st * kRStage + el * 1024 * nI + g2 * 1024;
            const uint16_t* scl =
                reinterpret_cast<const uint16_t*>(ring + (size_t)st * kRStage + kRData + el * sstride2) + g2 * kORows;
            const uint8_t* hs = hq + ((size_t)(e0 + el) * nS + 4 * g2) * kSliceB;
            int d[4][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint8_t* ch = data + q * 256;
              const uint32_t wa = *reinterpret_cast<const uint32_t*>(ch + g * 16 + 4 * c);
              const uint32_t wb = *reinterpret_cast<const uint32_t*>(ch + (g + 8) * 16 + 4 * c);
              uint2 hb = make_uint2(0u, 0u);
              if (g < 2) hb = *reinterpret_cast<const uint2*>(hs + q * kSliceB + g * 32 + c * 8);
              imma0(d[q], wa & M, wb & M, (wa >> 4) & M, (wb >> 4) & M, hb.x, hb.y);
            }
            const float s0 = __uint_as_float((uint32_t)scl[g] << 16);
            const float s1 = __uint_as_float((uint32_t)scl[g + 8] << 16);
            float t0 = 0.f, t1 = 0.f, cs = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 rec = *reinterpret_cast<const float2*>(hs + q * kSliceB + 64);   // {a, a * 8 sum v}
              t0 = fmaf(rec.x, (float)(d[q][0] * 256 + d[q][1]), t0);
              t1 = fmaf(rec.x, (float)(d[q][2] * 256 + d[q][3]), t1);
              cs += rec.y;
            }
            seg0 = fmaf(s0, t0 - cs, seg0);
            seg1 = fmaf(s1, t1 - cs, seg1);
            if (++g2 == nI) { g2 = 0; ++el; }
          }
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&s.empty[st]);
          if (w == 0 && lane == 0 && e0 == 0) trace_clk(P, 42);
          next();
        }
        if (c == 0) {
          s.red2[w][g] = seg0;
          s.red2[w][g + 8] = seg1;
        }
        if (w == 0 && lane == 0) trace_clk(P, 41);
        tc::named_bar_sync(1, kRCompute * 32);
        if (w == 0 && lane < kORows && !*abort) {
          float y = 0.f;
#pragma unroll
          for (int v = 0; v < kRCompute; ++v) y += s.red2[v][lane];
          store_output(P, 0, ob * kORows + lane, y);
        }
        tc::named_bar_sync(1, kRCompute * 32);
      }
    }
  } else {
    // ------------------------------------------------------------ h warp
    // per slice: gate and up sums (K parts in order), h = w * silu(gate) * up for the 32
    // features (lane = feature), encoded as one phase-2 k-step; then one arrival per CTA
    bool ok = true;
    int i = 0;
    for (int u = pl.u0; u < pl.u1; ++u, ++i) {
      const int b = i & 1;
      if (!warp_wait(&s.redfull[b], (i >> 1) & 1, abort)) { ok = false; break; }
      if (lane == 0 && i < 2) trace_clk(P, 44 + i);
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        gs += s.red1[b][p][lane];
        us += s.red1[b][p][kSliceF + lane];
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.redempty[b]);
      const int j = u / nS, fs = u % nS;
      const float wt = s.wsel[j];
      const float hv = (wt != 0.f) ? __fdividef(gs * us, 1.f + __expf(-gs)) * wt : 0.f;
      float mx = fabsf(hv);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
      const float inv = mx > 0.f ? 32639.f / mx : 0.f;
      const int iv = max(-32639, min(32639, __float2int_rn(hv * inv)));
      const int h8 = (iv + 128) >> 8, l8 = iv - 256 * h8;
      int sum = iv;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
      uint8_t* sl = P.hbuf + ((size_t)j * nS + fs) * kSliceB;
      const int at = (lane >> 3) * 8 + perm_pos(lane & 7);
      sl[at] = (uint8_t)h8;
      sl[32 + at] = (uint8_t)l8;
      if (lane == 0) {
        const float a = mx * (1.f / 32639.f);
        *reinterpret_cast<float2*>(sl + 64) = make_float2(a, a * (float)(8 * sum));
      }
      if (lane == 0 && i < 4) trace_clk(P, 32 + i);
    }
    __syncwarp();   // the lanes' stores are ordered before lane 0's release
    if (lane == 0 && ok && !*abort) red_release_add_u64(hseq, 1ull);
    if (lane == 0) trace_clk(P, 36);
    if (lane == 0) trace_at(P, 5);
  }

  if (pl.m == 0 && !*abort) {   // no expert selected: the outputs come from the accumulator alone
    for (int o = cta * kRThreads + tid; o < H; o += G * kRThreads) {
      const float accv = P.accumulate ? __ldcg(P.acc + o) : 0.f;
      if (P.out) {
        P.out[o] = __bfloat16_as_ushort(__float2bfloat16_rn(accv));
        if (P.accumulate) P.acc[o] = 0.f;
      } else {
        P.acc[o] = accv;
      }
    }
  }
  if (tid == 0) trace_at(P, 6);
}

// ---------------------------------------------------------------- host side
// 4-D view of a packed matrix bank (N rows x K per slot, 128 x 128 tiles; a tile's K quarter is a
// 2048-byte chunk of 128 rows x 16 B): (32-bit word in the chunk, K chunk = 4 * K group + quarter,
// row block, slot). Box: `box_rows` consecutive rows (16 * box_rows bytes of every chunk) of one
// block of one slot, so each of the box's lines is box_rows x 16 contiguous bytes.
int make_bank_map(CUtensorMap* map, const void* base, int N, int K, int slots, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const int nK = K / kGroup, nB = N / kRowBlock;
  const cuuint64_t dims[4] = {512, (cuuint64_t)(4 * nK), (cuuint64_t)nB, (cuuint64_t)slots};
  const cuuint64_t strides[3] = {2048, (cuuint64_t)nK * kTileBytes, (cuuint64_t)N * K / 2};
  const cuuint32_t box[4] = {(cuuint32_t)(box_rows * 4), (cuuint32_t)(4 * nK), 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (weight bank) failed (%d)", (int)r);
  return MOE_OK;
}

// 4-D view of a bank's tile-major scales (bf16; scale(n, g) at ((n/128) K/128 + g) 128 + n%128
// per slot): (row in the block, K group, row block, slot). Box: `box_rows` rows x all K groups.
int make_scales_map(CUtensorMap* map, const void* base, int N, int K, int slots, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
      return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const int nK = K / kGroup, nB = N / kRowBlock;
  const cuuint64_t dims[4] = {(cuuint64_t)kRowBlock, (cuuint64_t)nK, (cuuint64_t)nB, (cuuint64_t)slots};
  const cuuint64_t strides[3] = {(cuuint64_t)kRowBlock * 2, (cuuint64_t)nK * kRowBlock * 2,
                                 (cuuint64_t)N * nK * 2};
  const cuuint32_t box[4] = {(cuuint32_t)box_rows, (cuuint32_t)nK, 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (%d)", (int)r);
  return MOE_OK;
}

size_t rows_smem_bytes(int H, int I, int m_max) {
  const size_t nS = (size_t)I / kSliceF;
  return sizeof(RSmem) + (size_t)2 * (H + kXPad) + (size_t)(H / kGroup) * 16 + (size_t)m_max * nS * kSliceB +
         1024 + (size_t)kRStages * kRStage;
}

}  // namespace

// The single-token kernel takes H <= 2048 (a slice half's 32 rows x all K chunks fit one stage)
// and I <= 2048 (a stage holds 4 or 2 experts' 16-row W2 boxes).
bool rows_supported(int T, int H, int I, int E, int k) {
  if (T != 1 || k > 32) return false;
  const int nH = H / kGroup, nI = I / kRowBlock;
  if (nH < 1 || nH > 16 || nI < 1 || nI > 16) return false;
  return rows_smem_bytes(H, I, std::min(E, k)) <= (size_t)kSmemLimit;
}

size_t rows_hbuf_bytes(int H, int I, int E, int k) {
  return (size_t)std::min(E, k) * (I / kSliceF) * kSliceB;
}

int launch_decode_rows(const DecParams& P, int grid, cudaStream_t s) {
  CUtensorMap m13, m2, ms13, ms2;
  if (int rc = make_bank_map(&m13, P.w13, 2 * P.I, P.H, P.E, kSliceF)) return rc;
  if (int rc = make_bank_map(&m2, P.w2, P.H, P.I, P.E, kORows)) return rc;
  if (int rc = make_scales_map(&ms13, P.s13, 2 * P.I, P.H, P.E, kSliceF)) return rc;
  if (int rc = make_scales_map(&ms2, P.s2, P.H, P.I, P.E, kORows)) return rc;
  const size_t smem = rows_smem_bytes(P.H, P.I, std::min(P.E, P.k));
  static bool attr_done = false;
  if (!attr_done) {
    if (int rc = check_cuda(cudaFuncSetAttribute(moe_decode_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kSmemLimit), "fused decode (one token): smem attribute"))
      return rc;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kRThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, moe_decode_rows_kernel, P, m13, m2, ms13, ms2);
  note_launch();
  return check_cuda(e, "moe_decode_rows_kernel launch");
}

}  // namespace dec
}  // namespace moe
