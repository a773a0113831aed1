// Fused single-token decode kernel: routing, gate/up with SiLU*up, down projection and the
// router-weighted combine in ONE launch ("Every Expert Counts: ExactMoE for Memory-Efficient
// W4A16 Inference", Abstract: all selected experts execute through fused grouped MoE kernels;
// the router's top-k is unchanged).
//
// One token makes the layer two chains of matrix-vector products over the selected experts'
// packed weights (8 x 3.2 MB for an OLMoE-shaped layer): the time is the HBM stream of those
// bytes plus the latency of the dependent steps around it. The kernel is shaped so that every
// SM streams an equal share of the bytes from the first moment and one exchange between CTAs
// remains:
//  * every CTA routes the token itself (warp top-k over order-preserving keys), lists the
//    selected experts in ascending id, computes the same static plan, and issues ALL of its
//    weight copies at once: contiguous 1-D bulk copies of whole 8-row groups (the packed layout
//    keeps one row group's codes over all of K together), about 175 KB per SM, landing in their
//    own places in shared memory (no slot is reused, so nothing waits for a consumer);
//  * phase 1 (gate/up) is cut into units of 8 features of one expert: the 8 gate rows and the
//    8 matching up rows, all of K. The MMA's 16 rows are those 8 + 8 rows, so a unit's gate and
//    up sums finish in the same warps. Every compute warp takes one K group of every unit, with
//    the token's group held in registers as the MMA B operand;
//  * phase 2 (down) is cut into units of 16 output rows over every selected expert and all of I,
//    so an output row's whole sum ends inside one CTA and the bf16 output is stored directly;
//  * the units of both phases are split over the CTAs by bytes (phase-2 units first, one or none
//    per CTA, then phase-1 units filling every CTA up to an equal share);
//  * the exchange: two h warps reduce each phase-1 unit (16 warps' partial sums, fixed order),
//    form h = w_router * silu(gate) * up and write its 8 values to global memory as 16-bit fixed
//    point with their own scale; each CTA then adds 1 to a 64-bit counter (release). CTAs with a
//    phase-2 unit poll until all G arrivals of this launch are in and copy every h block (24 KB)
//    into shared memory; their phase-2 weights have been landing meanwhile.
// The contraction is the int8 warp-MMA path (mma.sync m16n8k32, u8 codes x s8 activations, exact
// in s32): x and h are 16-bit fixed point v = rint(value / a) split into two s8 columns (hi, lo).
// In phase 2 the eight B columns carry four 8-feature h blocks (hi and lo each), every block in
// its own K quarter of the MMA and zero elsewhere, so each lane applies its own block's scale.
// Sums run in a fixed order: results are identical run to run. Every wait is bounded.
//
// The counter only grows: a launch's base is its value at the start rounded down to a multiple
// of the grid size G (= number of SMs, fixed), the arrivals of one launch being fewer than G
// until it completes; no CTA resets it.
#include "decode_common.cuh"

namespace moe {
namespace dec {

// Test hook (moe_debug_set_wait_limit): wait limit in SM cycles (0 = default) and extra arrivals
// the single-token kernel expects.
long long g_wait_cycles = 0;
int g_extra_arrivals = 0;

namespace {

constexpr int kRCompute = 16;                     // compute warps 1..16
constexpr int kRHWarps = 2;                       // h warps 17, 18
constexpr int kRWarps = 1 + kRCompute + kRHWarps;
constexpr int kRThreads = kRWarps * 32;
constexpr int kMaxU1 = 32;                        // phase-1 units per CTA
constexpr int kChunkU = 2;                        // phase-1 units per copy chunk
constexpr int kMaxChunks = kMaxU1 / kChunkU;
constexpr int kMaxU2 = 4;                         // phase-2 units per CTA
constexpr int kMaxSel = 32;                       // selected experts (k <= 32)
constexpr int kRedBufs = 4;                       // phase-1 sum buffers (two per h warp)
constexpr int kHBlock = 32;                       // h block of 8 features: hi[8], lo[8], {a, a*8*sum v}, pad
constexpr int kF = 8;                             // features per phase-1 unit
constexpr int kORows = 16;                        // output rows per phase-2 unit
constexpr long long kDefaultWaitCycles = 4000000000ll;   // ~2 s at the B200's peak clock

struct __align__(128) RSmem {
  uint64_t cfull[kMaxChunks];                     // phase-1 chunk landed
  uint64_t sfull;                                 // phase-1 scales landed
  uint64_t vfull[kMaxU2];                         // phase-2 unit landed
  uint64_t hfull;                                 // every h block landed
  uint64_t wready;                                // router weights in wsel
  uint64_t redfull[kRedBufs], redempty[kRedBufs];
  float red1[kRedBufs][kRCompute][kChunkU * 2 * kF];   // [buffer][warp][unit][gate rows, up rows]
  float red2[kRCompute][kORows];                  // [warp][row] phase-2 sums
  uint32_t key[kMaxSel];                          // winning router key of choice j
  int act[kMaxSel];                               // selected experts, ascending id
  int sl[kMaxSel];                                // their slots
  float wsel[kMaxSel];                            // router weight of selected expert j
  int rank[kMaxSel];                              // choice j -> selected index (-1: not resident)
  int nact;
  int u1b, u1e, u2b, u2e;                         // this CTA's units
  int abort;
  // followed in dynamic shared memory by the h blocks [m][I/8] x 32 B and the weight pieces
};

// The split of both phases over the CTAs, identical in every CTA: the phase-1 units evenly (so that
// phase 1, which the exchange waits for, ends at the same time everywhere), the phase-2 units one
// or none per CTA on top.
struct RPlan {
  uint32_t nU1, nU2;
  __device__ __host__ void init(int m, int H, int I) {
    nU1 = (uint32_t)m * (I / kF);
    nU2 = H / kORows;
  }
  __device__ __host__ uint32_t lo1(int c, int G) const { return (uint32_t)c * nU1 / (uint32_t)G; }
  __device__ __host__ uint32_t lo2(int c, int G) const { return (uint32_t)c * nU2 / (uint32_t)G; }
};

__device__ __forceinline__ void imma0(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Bounded wait on an mbarrier phase (every lane of the calling warp): false when the limit runs
// out (raising *abort) or another warp has raised *abort.
__device__ __forceinline__ bool rwait(uint64_t* bar, uint32_t parity, volatile int* abort, long long limit) {
  bool ok = tc::mbar_try_wait(bar, parity);
  if (!ok) {
    const long long t0 = clock64();
    while (!(ok = tc::mbar_try_wait(bar, parity))) {
      if (*abort) break;
      if (clock64() - t0 > limit) { *abort = 1; break; }
    }
  }
  return __all_sync(kFull, ok);
}

// Top-k of one token with one warp (k <= 32): lane l holds the keys of experts l, l + 32, ...;
// each round takes the warp maximum of the keys (unique: the id is in them) and retires it.
// Lane j < k ends with the key of choice j.
template <int kPer>
__device__ __forceinline__ uint32_t topk_keys(const uint16_t* lt, int E, int k, int lane) {
  uint32_t key[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? route_key(lt[e], e) : 0u;
  }
  uint32_t mine = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t best = key[0];
#pragma unroll
    for (int i = 1; i < kPer; ++i) best = max(best, key[i]);
    const uint32_t win = __reduce_max_sync(kFull, best);
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (key[i] == win) key[i] = 0;
    if (j == lane) mine = win;
  }
  return mine;
}

__device__ __forceinline__ float key_logit(uint32_t w) {
  const uint32_t ord = w >> 16;
  return bf16_bits_to_float((ord & 0x8000u) ? (ord & 0x7fffu) : (~ord & 0xffffu));
}

// Byte position of element e (0..7) of a word in the MMA's permuted order (0, 4, 1, 5, 2, 6, 3, 7).
__device__ __forceinline__ int rperm(int e) { return ((e & 3) << 1) | (e >> 2); }

__global__ void __launch_bounds__(kRThreads, 1) moe_decode_rows_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  RSmem& s = *reinterpret_cast<RSmem*>(smem_raw);
  const int H = P.H, I = P.I;
  const int nH = H / kGroup, nI = I / kGroup, nFB = I / kF;
  const int m_max = min(P.E, P.k);
  uint8_t* hsm = smem_raw + sizeof(RSmem);                                 // h blocks [m][I/8]
  uint8_t* pieces = hsm + (((size_t)m_max * nFB * kHBlock + 127) & ~(size_t)127);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long limit = P.wait_cycles > 0 ? P.wait_cycles : kDefaultWaitCycles;
  volatile int* abort = &s.abort;

  // set-up that reads nothing the previous kernel writes: barriers, and L2 prefetches of the
  // token's logits and activations (a prefetch only warms L2, which stays coherent with the
  // previous kernel's writes; the values are read after the dependency wait)
  unsigned long long t_entry = 0;
  if (tid == 0 && P.trace) t_entry = tc::globaltimer();
  if (tid == 0) {
    for (int i = 0; i < kMaxChunks; ++i) tc::mbar_init(&s.cfull[i], 1);
    tc::mbar_init(&s.sfull, 1);
    for (int i = 0; i < kMaxU2; ++i) tc::mbar_init(&s.vfull[i], 1);
    tc::mbar_init(&s.hfull, 1);
    tc::mbar_init(&s.wready, 1);
    for (int i = 0; i < kRedBufs; ++i) {
      tc::mbar_init(&s.redfull[i], kRCompute);
      tc::mbar_init(&s.redempty[i], 1);
    }
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && P.logits && lane * 64 < P.E) prefetch_l2(P.logits + lane * 64);
  if (warp == 1 && lane * 64 < H) prefetch_l2(P.x + lane * 64);
  __syncthreads();
  const int G = gridDim.x, cta = blockIdx.x;
  // every expert resident and the token's logits given: the routing selects exactly k distinct
  // experts, so the plan (which needs only their number) is made before the dependency wait
  const bool fast = P.logits && !P.slot && P.E <= 64;
  const uint32_t code1 = (uint32_t)nH * kChunkBytes;                        // one row group, all of H
  if (warp == 0 && fast) {
    RPlan pl;
    pl.init(P.k, H, I);
    const uint32_t bnd = lane == 0 ? pl.lo1(cta, G) : lane == 1 ? pl.lo1(cta + 1, G)
                         : lane == 2 ? pl.lo2(cta, G) : pl.lo2(cta + 1, G);
    const int n1 = (int)(__shfl_sync(kFull, bnd, 1) - __shfl_sync(kFull, bnd, 0));
    const int nch = (n1 + kChunkU - 1) / kChunkU;
    if (lane < 4) (&s.u1b)[lane] = (int)bnd;
    if (lane == 0) s.nact = P.k;
    if (lane < nch)
      tc::mbar_arrive_expect_tx(&s.cfull[lane], (uint32_t)(min(kChunkU, n1 - lane * kChunkU) * 2 * code1));
    if (lane == 0 && n1 > 0) tc::mbar_arrive_expect_tx(&s.sfull, (uint32_t)(2 * n1 * nH * 16));
  }

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0 && P.trace) {   // diagnostics: entry, the previous launch's last warp, wait done
    const unsigned long long prev_end = P.trace[blockIdx.x * 64 + 10];
    P.trace[blockIdx.x * 64 + 11] = P.trace[blockIdx.x * 64 + 7];
    P.trace[blockIdx.x * 64 + 10] = 0;
    trace_at(P, 0);
    P.trace[blockIdx.x * 64 + 8] = t_entry;
    P.trace[blockIdx.x * 64 + 9] = prev_end;
  }
  unsigned long long* seq = reinterpret_cast<unsigned long long*>(P.hdone + 2);
  unsigned long long seq0 = 0;
  if (tid == 0) seq0 = ld_relaxed_u64(seq);

  // ---- compute warps: the token's K group as B fragments (16-bit fixed point, registers)
  const int cw = warp - 1, gq = lane >> 2, cq = lane & 3;
  int gk = -1;                                     // this warp's K group of every phase-1 unit
  uint32_t xb0[4] = {0, 0, 0, 0}, xb1[4] = {0, 0, 0, 0};
  float xa = 0.f;
  int xcorr = 0;
  if (warp >= 1 && warp <= kRCompute) {
    const int g0 = cw * nH / kRCompute, g1 = (cw + 1) * nH / kRCompute;
    if (g1 > g0) {   // nH <= 16: at most one group per warp
      gk = g0;
      float xv[4][8];
      if (lane < 8) {
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const uint4 r = *reinterpret_cast<const uint4*>(P.x + gk * kGroup + kq * 32 + 8 * cq);
          const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            xv[kq][2 * e] = bf16_bits_to_float(w4[e] & 0xffffu);
            xv[kq][2 * e + 1] = bf16_bits_to_float(w4[e] >> 16);
          }
        }
      } else {
#pragma unroll
        for (int kq = 0; kq < 4; ++kq)
#pragma unroll
          for (int e = 0; e < 8; ++e) xv[kq][e] = 0.f;
      }
      float mx = 0.f;
#pragma unroll
      for (int kq = 0; kq < 4; ++kq)
#pragma unroll
        for (int e = 0; e < 8; ++e) mx = fmaxf(mx, fabsf(xv[kq][e]));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));   // lanes 0..3 (and 4..7) see the group's max
      const float inv = mx > 0.f ? 32639.f / mx : 0.f;
      int sum = 0;
#pragma unroll
      for (int kq = 0; kq < 4; ++kq) {
        uint32_t b0 = 0, b1 = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int iv = max(-32639, min(32639, __float2int_rn(xv[kq][e] * inv)));
          const int h8 = (iv + 128) >> 8, l8 = iv - 256 * h8;
          const uint32_t byte = (uint32_t)((gq == 0 ? h8 : l8) & 0xff);
          const int pos = rperm(e);                 // 0..3 -> b0, 4..7 -> b1
          if (pos < 4) b0 |= byte << (8 * pos); else b1 |= byte << (8 * (pos - 4));
          sum += iv;
        }
        if (lane < 8) { xb0[kq] = b0; xb1[kq] = b1; }
      }
      sum += __shfl_xor_sync(kFull, sum, 1);
      sum += __shfl_xor_sync(kFull, sum, 2);
      xa = __shfl_sync(kFull, mx, 0) * (1.f / 32639.f);
      xcorr = 8 * __shfl_sync(kFull, sum, 0);
    }
  }

  const size_t w13_slot = (size_t)I * H, s13_slot = (size_t)2 * I * nH;     // bytes / scales per slot
  const size_t w2_slot = (size_t)H * I / 2, s2_slot = (size_t)H * nI;

  // ---- warp 0: routing, plan, the phase-1 copies
  if (warp == 0) {
    const int k = P.k, E = P.E;
    int e = -1;
    uint32_t mykey = 0;
    float wgiven = 0.f;
    int m = 0, below = 0, sl = -1;
    bool in = false;
    if (lane == 0) trace_clk(P, 16);
    if (P.logits && !P.slot && E <= 64) {
      // every expert resident, one token: the k winners are distinct; their presence mask and
      // ranks follow from the winning keys directly
      uint32_t key0 = lane < E ? route_key(P.logits[lane], lane) : 0u;
      uint32_t key1 = lane + 32 < E ? route_key(P.logits[lane + 32], lane + 32) : 0u;
      unsigned long long msk = 0;
      for (int j = 0; j < k; ++j) {
        const uint32_t win = __reduce_max_sync(kFull, max(key0, key1));
        if (key0 == win) key0 = 0;
        if (key1 == win) key1 = 0;
        if (j == lane) mykey = win;
        msk |= 1ull << (0xffff - (win & 0xffffu));
      }
      if (lane == 0) trace_clk(P, 17);
      in = lane < k;
      if (in) {
        e = 0xffff - (int)(mykey & 0xffffu);
        below = __popcll(msk & ((1ull << e) - 1ull));
        sl = e;
      }
      m = k;
    } else {
      if (P.logits) {
        if (E <= 64) mykey = topk_keys<2>(P.logits, E, k, lane);
        else if (E <= 128) mykey = topk_keys<4>(P.logits, E, k, lane);
        else mykey = topk_keys<8>(P.logits, E, k, lane);
        if (lane < k) e = 0xffff - (int)(mykey & 0xffffu);
        if (lane == 0) trace_clk(P, 17);
      } else if (lane < k) {
        e = P.idx_in[lane];
        wgiven = P.wts_in[lane];
      }
      if (lane < k && (unsigned)e < (unsigned)E) sl = slot_of(P.slot, e);
      in = sl >= 0;
      const int n_in = __popc(__ballot_sync(kFull, in));
      const int nw = (E + 31) >> 5;
      uint32_t mw = 0;   // lane wd < nw: presence word wd
      for (int wd = 0; wd < nw; ++wd) {
        const uint32_t v = __reduce_or_sync(kFull, (in && (e >> 5) == wd) ? 1u << (e & 31) : 0u);
        if (lane == wd) mw = v;
      }
      for (int wd = 0; wd < nw; ++wd) {
        const uint32_t v = __shfl_sync(kFull, mw, wd);
        if (in && wd < (e >> 5)) below += __popc(v);
        if (in && wd == (e >> 5)) below += __popc(v & ((1u << (e & 31)) - 1u));
      }
      const int total = (int)__reduce_add_sync(kFull, (uint32_t)__popc(mw));
      const bool dup = total != n_in;
      m = dup ? 0 : total;
      if (dup) in = false;
      if (lane == 0 && dup) report_status(P.ctl, MOE_ERR_ARG, kSiteOver);
    }
    if (in) {
      s.act[below] = e;
      s.sl[below] = sl;
    }
    s.rank[lane] = in ? below : -1;
    s.key[lane] = mykey;
    s.wsel[lane] = wgiven;
    if (lane == 0) trace_clk(P, 18);
    int u1b, u1e, u2b, u2e;
    if (fast) {
      u1b = s.u1b; u1e = s.u1e; u2b = s.u2b; u2e = s.u2e;
    } else {
      RPlan pl;
      pl.init(m, H, I);
      // the four unit boundaries of this CTA, one per lane
      const uint32_t bnd = lane == 0 ? pl.lo1(cta, G) : lane == 1 ? pl.lo1(cta + 1, G)
                           : lane == 2 ? pl.lo2(cta, G) : pl.lo2(cta + 1, G);
      u1b = (int)__shfl_sync(kFull, bnd, 0); u1e = (int)__shfl_sync(kFull, bnd, 1);
      u2b = (int)__shfl_sync(kFull, bnd, 2); u2e = m > 0 ? (int)__shfl_sync(kFull, bnd, 3) : u2b;
      if (lane == 0) {
        s.nact = m;
        s.u1b = u1b; s.u1e = u1e; s.u2b = u2b; s.u2e = u2e;
      }
    }
    if (lane == 0) trace_clk(P, 19);
    __syncwarp();
    // phase-1 copies: chunk c (units 2c, 2c + 1 of this CTA) is one copy of its gate row groups
    // and one of its up row groups (two each when its units belong to two experts); the scales of
    // each expert's run of units are one copy for the gate rows and one for the up rows
    const int n1 = u1e - u1b, nch = (n1 + kChunkU - 1) / kChunkU;
    const int j0 = n1 > 0 ? u1b / nFB : 0, nruns = n1 > 0 ? (u1e - 1) / nFB - j0 + 1 : 0;
    const uint64_t pol = tc::policy_evict_first();
    uint8_t* sc1 = pieces + (size_t)n1 * 2 * code1;                          // phase-1 scales
    if (!fast && lane == 0 && n1 > 0) tc::mbar_arrive_expect_tx(&s.sfull, (uint32_t)(2 * n1 * nH * 16));
    __syncwarp();
    for (int c = lane; c < nch + 2 * nruns; c += 32) {
      if (c < nch) {
        const int i0 = c * kChunkU, nk = min(kChunkU, n1 - i0);
        uint8_t* dst = pieces + (size_t)i0 * 2 * code1;
        if (!fast) tc::mbar_arrive_expect_tx(&s.cfull[c], (uint32_t)(nk * 2 * code1));
        const int ua = u1b + i0, ub = ua + nk - 1, ja = ua / nFB, jb = ub / nFB;
        if (ja == jb) {   // both units of one expert: their row groups follow each other
          const int fb = ua - ja * nFB;
          const uint8_t* src = P.w13 + s.sl[ja] * w13_slot;
          tc::bulk_g2s(dst, src + chunk_offset(fb, 0, nH), nk * code1, &s.cfull[c], pol);
          tc::bulk_g2s(dst + (size_t)nk * code1, src + chunk_offset(I / kRowGroup + fb, 0, nH), nk * code1,
                       &s.cfull[c], pol);
        } else {
          for (int q = 0; q < nk; ++q) {
            const int u = ua + q, j = u / nFB, fb = u - j * nFB;
            const uint8_t* src = P.w13 + s.sl[j] * w13_slot;
            tc::bulk_g2s(dst + (size_t)q * code1, src + chunk_offset(fb, 0, nH), code1, &s.cfull[c], pol);
            tc::bulk_g2s(dst + (size_t)(nk + q) * code1, src + chunk_offset(I / kRowGroup + fb, 0, nH), code1,
                         &s.cfull[c], pol);
          }
        }
      } else {
        const int r = (c - nch) >> 1, up = (c - nch) & 1, j = j0 + r;
        const int ua = max(u1b, j * nFB), ue = min(u1e, (j + 1) * nFB), fb = ua - j * nFB;
        const int R = up ? I / kRowGroup + fb : fb;
        tc::bulk_g2s(sc1 + ((size_t)up * n1 + (ua - u1b)) * nH * 16,
                     P.s13 + s.sl[j] * s13_slot + chunk_scale_index(R, 0, nH), (uint32_t)((ue - ua) * nH * 16),
                     &s.sfull, pol);
      }
    }
    if (lane == 0) trace_clk(P, 21);
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int m = s.nact, u1b = s.u1b, u1e = s.u1e, u2b = s.u2b, u2e = s.u2e;
  const int n1 = u1e - u1b, n2 = u2e - u2b, nch = (n1 + kChunkU - 1) / kChunkU;
  const uint8_t* sc1 = pieces + (size_t)n1 * 2 * code1;
  uint8_t* p2 = pieces + ((((size_t)n1 * 2 * code1 + (size_t)2 * n1 * nH * 16) + 127) & ~(size_t)127);
  const uint32_t code2 = (uint32_t)(2 * nI * kChunkBytes);                 // one expert's two row groups
  uint16_t* sc2 = reinterpret_cast<uint16_t*>(p2 + (size_t)n2 * m * code2);   // phase-2 scales
  const uint32_t hbytes = (uint32_t)(m * nFB * kHBlock);

  if (warp == 0) {
    // ------------------------------------------------------------ router weights, phase-2 copies,
    // exchange
    const int k = P.k;
    if (P.logits) {
      // renormalised weight of choice j = exp(l_j - l_max) / sum over the k chosen
      const uint32_t mykey = s.key[lane];
      const float mx = key_logit(__shfl_sync(kFull, mykey, 0));
      const float el = lane < k ? expf(key_logit(mykey) - mx) : 0.f;
      float sum = el;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
      const float w = el / sum;
      if (lane < k) {
        const int r = s.rank[lane];
        if (r >= 0) s.wsel[r] = w;
        if (P.idx_out && cta == 0) {
          P.idx_out[lane] = 0xffff - (int)(mykey & 0xffffu);
          P.wts_out[lane] = w;
        }
      }
    } else {
      const float w = s.wsel[lane];   // the given weights, choice order
      __syncwarp();
      if (lane < k) {
        const int r = s.rank[lane];
        if (r >= 0) s.wsel[r] = w;
      }
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&s.wready);
    // the phase-2 weights go out once the first phase-1 chunk has landed, so that the HBM queue
    // serves phase 1 first and the exchange overlaps the phase-2 stream
    bool ok = true;
    if (n2 > 0) {
      if (nch > 0) ok = rwait(&s.cfull[0], 0, abort, limit);
      const uint64_t pol = tc::policy_evict_first();
      if (lane == 0)
        for (int v = 0; v < n2; ++v) tc::mbar_arrive_expect_tx(&s.vfull[v], (uint32_t)(m * code2));
      __syncwarp();
      for (int c = lane; c < n2 * m; c += 32) {
        const int v = c / m, j = c - v * m;
        tc::bulk_g2s(p2 + (size_t)c * code2, P.w2 + s.sl[j] * w2_slot + chunk_offset(2 * (u2b + v), 0, nI), code2,
                     &s.vfull[v], pol);
      }
      if (lane == 0) trace_clk(P, 22);
      if (lane == 0 && ok) {
        const unsigned long long target =
            seq0 - seq0 % (unsigned long long)G + (unsigned long long)G + (unsigned long long)P.extra_arrivals;
        const long long t0 = clock64();
        while (ld_relaxed_u64(seq) < target) {
          if (*abort || clock64() - t0 > limit) { ok = false; break; }
          __nanosleep(20);
        }
        if (ok) {
          // acquire (pairs with the CTAs' release adds), then order the async-proxy copy after it
          asm volatile("fence.acq_rel.gpu;" ::: "memory");
          fence_proxy_async_global();
          trace_clk(P, 28);
          tc::mbar_arrive_expect_tx(&s.hfull, hbytes);
          tc::bulk_g2s(hsm, P.hbuf, hbytes, &s.hfull, tc::policy_evict_first());
        } else {
          s.abort = 1;
          report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteHDone);
        }
      }
      ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0) {   // no copy may still be landing in shared memory when the CTA leaves
      volatile int never = 0;
      for (int c = 0; c < nch; ++c) tc::mbar_wait(&s.cfull[c], 0, &never);
      if (n1 > 0) tc::mbar_wait(&s.sfull, 0, &never);
      for (int v = 0; v < n2; ++v) tc::mbar_wait(&s.vfull[v], 0, &never);
      if (n2 > 0 && ok) tc::mbar_wait(&s.hfull, 0, &never);
    }
    __syncwarp();
  } else if (warp <= kRCompute) {
    // ------------------------------------------------------------ compute warps 1..16
    const uint32_t M = 0x0F0F0F0Fu;
    const int ct = tid - 32;                      // 0..511
    // the phase-2 scales of this CTA's units: plain loads into shared memory, long before use
    // ([unit][expert][row group 0 then 1][K group][8 rows], two bf16 per 32-bit word)
    for (int w = ct; w < n2 * m * nI * 8; w += kRCompute * 32) {
      const int per = nI * 8, vj = w / per, rem = w - vj * per, v = vj / m, j = vj - v * m;
      const uint32_t* src = reinterpret_cast<const uint32_t*>(P.s2 + s.sl[j] * s2_slot +
                                                              chunk_scale_index(2 * (u2b + v), 0, nI));
      reinterpret_cast<uint32_t*>(sc2)[w] = src[rem];
    }
    bool ok = true;
    // phase 1, one chunk (up to two units) per step; unit q, K group gk: rows 0..7 of the MMA =
    // gate rows, 8..15 = up rows. The MMAs of a step are independent (one accumulator per K
    // quarter and unit), summed afterwards, so the warp's MMAs overlap instead of forming a chain.
    if (n1 > 0) ok = rwait(&s.sfull, 0, abort, limit);
    for (int c = 0; c < nch && ok; ++c) {
      const int b = c % kRedBufs, nk = min(kChunkU, n1 - c * kChunkU);
      if (c >= kRedBufs && !rwait(&s.redempty[b], ((c / kRedBufs) - 1) & 1, abort, limit)) { ok = false; break; }
      if (!rwait(&s.cfull[c], 0, abort, limit)) { ok = false; break; }
      if (cw == 0 && lane == 0 && c < 16) trace_clk(P, 32 + c);
      if (gk >= 0) {
        const uint8_t* chunk = pieces + (size_t)c * kChunkU * 2 * code1 + (size_t)gk * kChunkBytes + gq * 16 + 4 * cq;
        int d[kChunkU][4][4];
#pragma unroll
        for (int q = 0; q < kChunkU; ++q) {
          if (q < nk) {
            const uint8_t* gch = chunk + (size_t)q * code1;
            const uint8_t* uch = chunk + (size_t)(nk + q) * code1;
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
              const uint32_t wa = *reinterpret_cast<const uint32_t*>(gch + kq * 128);
              const uint32_t wb = *reinterpret_cast<const uint32_t*>(uch + kq * 128);
              imma0(d[q][kq], wa & M, wb & M, (wa >> 4) & M, (wb >> 4) & M, xb0[kq], xb1[kq]);
            }
          }
        }
        if (cq == 0) {   // columns 0 / 1 = hi / lo of the token
#pragma unroll
          for (int q = 0; q < kChunkU; ++q) {
            if (q < nk) {
              const int i = c * kChunkU + q;
              const int dg0 = d[q][0][0] + d[q][1][0] + d[q][2][0] + d[q][3][0];
              const int dg1 = d[q][0][1] + d[q][1][1] + d[q][2][1] + d[q][3][1];
              const int du0 = d[q][0][2] + d[q][1][2] + d[q][2][2] + d[q][3][2];
              const int du1 = d[q][0][3] + d[q][1][3] + d[q][2][3] + d[q][3][3];
              const uint16_t* sg = reinterpret_cast<const uint16_t*>(sc1 + (size_t)i * nH * 16);
              const uint16_t* su = reinterpret_cast<const uint16_t*>(sc1 + (size_t)(n1 + i) * nH * 16);
              s.red1[b][cw][q * 2 * kF + gq] = bf16_bits_to_float(sg[gk * kRowGroup + gq]) * xa * (float)(dg0 * 256 + dg1 - xcorr);
              s.red1[b][cw][q * 2 * kF + kF + gq] = bf16_bits_to_float(su[gk * kRowGroup + gq]) * xa * (float)(du0 * 256 + du1 - xcorr);
            }
          }
        }
      } else if (lane < kChunkU * 2 * kF) {
        s.red1[b][cw][lane] = 0.f;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.redfull[b]);
    }
    if (cw == 0 && lane == 0) trace_clk(P, 27);
    // phase 2: unit v = 16 output rows over every selected expert;
    // warp cw takes the (expert, K group) pairs [cw P / 16, (cw + 1) P / 16), P = m nI. Lane (g, c):
    // A rows g (first row group) and g + 8 (second); B column g holds, in K quarter c, the hi
    // (g even) or lo (g odd) bytes of h block c of the k-step, so D[r][2c], D[r][2c + 1] are block
    // c's hi and lo sums and the lane applies block c's scale. (Every compute warp runs every unit
    // and meets the named barriers, also after a failed wait; its work is then skipped.)
    bool h_in = false;
    for (int v = 0; v < n2; ++v) {
      ok = ok && rwait(&s.vfull[v], 0, abort, limit);
      if (cw == 0 && lane == 0 && v == 0) trace_clk(P, 12);
      if (!h_in) {
        ok = ok && rwait(&s.hfull, 0, abort, limit);
        if (ok && cw == 0 && lane == 0) trace_clk(P, 29);
        h_in = true;
        tc::named_bar_sync(1, kRCompute * 32);   // every warp's phase-2 scales are in shared memory
        if (cw == 0 && lane == 0) trace_clk(P, 13);
      }
      const uint8_t* unit = p2 + (size_t)v * m * code2;
      const uint16_t* scu = sc2 + (size_t)v * m * 2 * nI * kRowGroup;
      const int np = m * nI, q0 = cw * np / kRCompute, q1 = ok ? (cw + 1) * np / kRCompute : q0;
      float y0 = 0.f, y1 = 0.f;
      int j = q0 / nI, g2 = q0 - j * nI;
#pragma unroll 2
      for (int p = q0; p < q1; ++p) {
        const uint8_t* ch0 = unit + (size_t)j * code2 + (size_t)g2 * kChunkBytes + gq * 16 + 4 * cq;
        const uint8_t* ch1 = ch0 + (size_t)nI * kChunkBytes;
        const uint16_t* scl = scu + (size_t)j * 2 * nI * kRowGroup;
        const uint8_t* hb = hsm + ((size_t)j * nFB + g2 * 16) * kHBlock;   // the group's 16 h blocks
        uint32_t wa[4], wb[4];
        uint2 hv[4];
        float2 rec[4];
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          wa[kq] = *reinterpret_cast<const uint32_t*>(ch0 + kq * 128);
          wb[kq] = *reinterpret_cast<const uint32_t*>(ch1 + kq * 128);
          const uint8_t* blk = hb + (kq * 4 + cq) * kHBlock;
          hv[kq] = (gq >> 1) == cq ? *reinterpret_cast<const uint2*>(blk + (gq & 1) * 8) : make_uint2(0u, 0u);
          rec[kq] = *reinterpret_cast<const float2*>(blk + 16);   // {a, a * 8 sum v}
        }
        const float s0 = bf16_bits_to_float(scl[g2 * kRowGroup + gq]);
        const float s1 = bf16_bits_to_float(scl[nI * kRowGroup + g2 * kRowGroup + gq]);
        int d[4][4];
#pragma unroll
        for (int kq = 0; kq < 4; ++kq)
          imma0(d[kq], wa[kq] & M, wb[kq] & M, (wa[kq] >> 4) & M, (wb[kq] >> 4) & M, hv[kq].x, hv[kq].y);
        float t0 = 0.f, t1 = 0.f;
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          t0 += fmaf(rec[kq].x, (float)(d[kq][0] * 256 + d[kq][1]), -rec[kq].y);
          t1 += fmaf(rec[kq].x, (float)(d[kq][2] * 256 + d[kq][3]), -rec[kq].y);
        }
        y0 = fmaf(s0, t0, y0);
        y1 = fmaf(s1, t1, y1);
        if (++g2 == nI) { g2 = 0; ++j; }
      }
      // the four lanes of a row hold four different h blocks: sum them (fixed order)
      y0 += __shfl_xor_sync(kFull, y0, 1);
      y1 += __shfl_xor_sync(kFull, y1, 1);
      y0 += __shfl_xor_sync(kFull, y0, 2);
      y1 += __shfl_xor_sync(kFull, y1, 2);
      if (cq == 0) {
        s.red2[cw][gq] = y0;
        s.red2[cw][gq + 8] = y1;
      }
      if (cw == 0 && lane == 0 && v == 0) trace_clk(P, 14);
      tc::named_bar_sync(1, kRCompute * 32);
      if (cw == 0 && lane < kORows && !*abort) {
        float y = 0.f;
#pragma unroll
        for (int w = 0; w < kRCompute; ++w) y += s.red2[w][lane];
        store_output(P, 0, (u2b + v) * kORows + lane, y);
      }
      if (cw == 0 && lane == 0 && v == 0) trace_clk(P, 15);
      tc::named_bar_sync(1, kRCompute * 32);
    }
    if (!ok && lane == 0) report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteStage);
  } else {
    // ------------------------------------------------------------ h warps 17, 18
    // chunk c goes to h warp c % 2: the 16 warps' sums (fixed order), h = w * silu(gate) * up of
    // its units' 8 features, encoded as the down projection's B operand; then one arrival per CTA
    const int hw = warp - 1 - kRCompute;
    bool ok = rwait(&s.wready, 0, abort, limit);
    for (int c = hw; c < nch && ok; c += kRHWarps) {
      const int b = c % kRedBufs;
      if (!rwait(&s.redfull[b], (c / kRedBufs) & 1, abort, limit)) { ok = false; break; }
      // lane l: entry l of the chunk (unit l / 16, gate (l % 16 < 8) or up row l % 8)
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kRCompute; ++w) sum += s.red1[b][w][lane];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.redempty[b]);
      const float up = __shfl_sync(kFull, sum, (lane & ~15) | ((lane & 7) + kF));
      // lanes 0..7 and 16..23: h of the chunk's units 0 and 1, encoded per 8-feature block as
      // v = rint(h / a), a = max|h| / 32639, hi and lo bytes in the MMA's element order (byte
      // stores into the block), then {a, a * 8 sum v}
      const int q = lane >> 4, i = c * kChunkU + q;
      const bool mine = (lane & 15) < kF && i < n1;
      const int u = u1b + (mine ? i : 0), j = u / nFB, fb = u - j * nFB;
      float hv = 0.f;
      if (mine) {
        const float wt = s.wsel[j];
        hv = (wt != 0.f) ? __fdividef(sum * up, 1.f + __expf(-sum)) * wt : 0.f;
      }
      float mx = fabsf(hv);
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
      const float inv = mx > 0.f ? 32639.f / mx : 0.f;
      const int iv = mine ? max(-32639, min(32639, __float2int_rn(hv * inv))) : 0;
      int sv = iv;
      sv += __shfl_xor_sync(kFull, sv, 1);
      sv += __shfl_xor_sync(kFull, sv, 2);
      sv += __shfl_xor_sync(kFull, sv, 4);
      if (mine) {
        uint8_t* blk = P.hbuf + ((size_t)j * nFB + fb) * kHBlock;
        const int h8 = (iv + 128) >> 8, l8 = iv - 256 * h8, pos = rperm(lane & 7);
        blk[pos] = (uint8_t)h8;
        blk[8 + pos] = (uint8_t)l8;
        if ((lane & 7) == 0) {
          const float a = mx * (1.f / 32639.f);
          *reinterpret_cast<float2*>(blk + 16) = make_float2(a, a * (float)(8 * sv));
        }
      }
      if (lane == 0 && c < 16) trace_clk(P, 48 + c);
    }
    // both h warps meet, then one release: every block of this CTA is ordered before it. Every
    // CTA arrives whenever an expert is selected (also after a failed wait, which the status word
    // records), so the counter stays a multiple of G between launches.
    if (lane == 0 && hw == 0) trace_clk(P, 25);
    tc::named_bar_sync(2, kRHWarps * 32);
    if (hw == 0 && lane == 0 && m > 0) {
      red_release_add_u64(seq, 1ull);
      trace_clk(P, 30);
    }
    if (!ok && lane == 0) report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteH);
  }

  if (m == 0 && !*abort) {   // no expert selected: the outputs come from the accumulator alone
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
  if (tid == 0) { trace_clk(P, 31); trace_at(P, 7); }
  if (lane == 0 && P.trace) atomicMax(P.trace + blockIdx.x * 64 + 10, tc::globaltimer());   // last warp out
}

// ---------------------------------------------------------------- host side
size_t rows_static_smem() { return sizeof(RSmem); }
size_t rows_h_bytes(int I, int m_max) { return ((size_t)m_max * (I / kF) * kHBlock + 127) & ~(size_t)127; }

// Shared memory of a CTA's pieces: phase-1 codes and scales, then (128-aligned) phase-2 codes and
// scales.
size_t rows_pieces_bytes(int H, int I, int m, int n1, int n2) {
  const size_t nH = H / kGroup, nI = I / kGroup;
  const size_t p1 = (size_t)n1 * 2 * nH * kChunkBytes + (size_t)2 * n1 * nH * 16;
  return ((p1 + 127) & ~(size_t)127) + (size_t)n2 * m * 2 * nI * (kChunkBytes + 16);
}

// Whether every CTA's share for m selected experts fits the piece area and the unit limits.
bool rows_plan_fits(int H, int I, int m, int G, size_t cap) {
  RPlan pl;
  pl.init(m, H, I);
  for (int c = 0; c < G; ++c) {
    const int n1 = (int)pl.lo1(c + 1, G) - (int)pl.lo1(c, G);
    const int n2 = (int)pl.lo2(c + 1, G) - (int)pl.lo2(c, G);
    if (n1 < 0 || n1 > kMaxU1 || n2 > kMaxU2) return false;
    if (rows_pieces_bytes(H, I, m, n1, n2) > cap) return false;
  }
  return true;
}

size_t rows_smem_bytes(int, int, int) { return kSmemLimit; }   // the pieces take what is left

}  // namespace

// The single-token kernel takes H <= 2048 (a compute warp holds one K group of the token) and a
// plan whose per-CTA pieces fit shared memory for every possible number of selected experts.
bool rows_supported(int T, int H, int I, int E, int k) {
  if (T != 1 || k > kMaxSel) return false;
  const int nH = H / kGroup, nI = I / kGroup;
  if (nH < 1 || nH > kRCompute || nI < 1) return false;
  const int m_max = std::min(E, k), G = num_sms();
  const long cap = (long)kSmemLimit - (long)rows_static_smem() - (long)rows_h_bytes(I, m_max);
  if (cap <= 0) return false;
  for (int m = 1; m <= m_max; ++m)
    if (!rows_plan_fits(H, I, m, G, (size_t)cap)) return false;
  return true;
}

size_t rows_hbuf_per_tile() { return (size_t)(kGroup / kF) * kHBlock; }   // per (expert, 128 features)

int launch_decode_rows(const DecParams& P0, int grid, cudaStream_t s) {
  DecParams P = P0;
  P.wait_cycles = g_wait_cycles;
  P.extra_arrivals = g_extra_arrivals;
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
  cfg.dynamicSmemBytes = rows_smem_bytes(P.H, P.I, std::min(P.E, P.k));
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, moe_decode_rows_kernel, P);
  note_launch();
  return check_cuda(e, "moe_decode_rows_kernel launch");
}

}  // namespace dec
}  // namespace moe

using namespace moe;

// Testing aid for failure detection (declared in include/moe_w4a16.h).
MOE_API void moe_debug_set_wait_limit(unsigned long long cycles, int extra_arrivals) {
  dec::g_wait_cycles = (long long)cycles;
  dec::g_extra_arrivals = extra_arrivals > 0 ? extra_arrivals : 0;
}
