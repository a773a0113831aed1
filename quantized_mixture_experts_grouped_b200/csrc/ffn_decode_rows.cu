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
constexpr int kMaxU2 = 4;                         // phase-2 units per CTA
constexpr int kMaxSel = 32;                       // selected experts (k <= 32)
constexpr int kRedBufs = 4;                       // phase-1 sum buffers (two per h warp)
constexpr int kHBlock = 24;                       // encoded 8-feature h block: hi[8], lo[8], {a, a*8*sum v}
constexpr int kF = 8;                             // features per phase-1 unit
constexpr int kORows = 16;                        // output rows per phase-2 unit
constexpr long long kDefaultWaitCycles = 4000000000ll;   // ~2 s at the B200's peak clock

struct __align__(128) RSmem {
  uint64_t ufull[kMaxU1];                         // phase-1 unit landed
  uint64_t vfull[kMaxU2];                         // phase-2 unit landed
  uint64_t hfull;                                 // every h block landed
  uint64_t wready;                                // router weights in wsel
  uint64_t redfull[kRedBufs], redempty[kRedBufs];
  float red1[kRedBufs][kRCompute][2 * kF];        // [buffer][warp][gate rows, up rows]
  float red2[kRCompute][kORows];                  // [warp][row] phase-2 sums
  uint32_t key[kMaxSel];                          // winning router key of choice j
  int act[kMaxSel];                               // selected experts, ascending id
  int sl[kMaxSel];                                // their slots
  float wsel[kMaxSel];                            // router weight of selected expert j
  int rank[kMaxSel];                              // choice j -> selected index (-1: not resident)
  int nact;
  int u1b, u1e, u2b, u2e;                         // this CTA's units
  int abort;
  // followed in dynamic shared memory by the h blocks [m][I/8] x 24 B and the weight pieces
};

// The split of both phases over the CTAs, identical in every CTA (bytes per unit: B1, B2).
struct RPlan {
  int nU1, nU2;
  long long B1, B2;
  __device__ __host__ static int lo2(int c, int nU2, int G) { return (int)((long long)c * nU2 / G); }
  // phase-1 unit boundary of CTA c: the byte share c/G of the total minus the phase-2 bytes of
  // CTAs below c, in units of B1 (rounded); non-decreasing whenever one CTA's share is at least
  // its largest phase-2 load, else the phase-1 units are split evenly on their own
  __device__ __host__ int lo1(int c, int G, bool joint) const {
    if (!joint) return (int)((long long)c * nU1 / G);
    const long long total = (long long)nU1 * B1 + (long long)nU2 * B2;
    const long long num = (long long)c * total - (long long)G * B2 * lo2(c, nU2, G);
    long long u = (num + (long long)G * B1 / 2) / ((long long)G * B1);
    if (u < 0) u = 0;
    if (u > nU1) u = nU1;
    return (int)u;
  }
  __device__ __host__ bool joint(int G) const {
    const long long total = (long long)nU1 * B1 + (long long)nU2 * B2;
    const long long max2 = (long long)((nU2 + G - 1) / G) * B2;
    return total >= (long long)G * max2;
  }
  __device__ __host__ void init(int m, int H, int I) {
    const int nH = H / kGroup, nI = I / kGroup;
    nU1 = m * (I / kF);
    nU2 = H / kORows;
    B1 = 2LL * nH * (kChunkBytes + 16);            // gate + up row groups: codes and scales
    B2 = (long long)m * 2 * nI * (kChunkBytes + 16);   // two row groups of every selected expert
  }
};

__device__ __forceinline__ void imma0(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1) {
  asm volatile(
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

  if (tid == 0) {
    for (int i = 0; i < kMaxU1; ++i) tc::mbar_init(&s.ufull[i], 1);
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
  __syncthreads();

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) trace_at(P, 0);
  const int G = gridDim.x, cta = blockIdx.x;
  unsigned long long* seq = reinterpret_cast<unsigned long long*>(P.hdone + 2);
  unsigned long long seq0 = 0;
  if (tid == 0) seq0 = ld_relaxed_u64(seq);

  // ---- compute warps: the token's K group(s) as B fragments (16-bit fixed point, registers)
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

  // ---- warp 0: routing, plan, every weight copy
  if (warp == 0) {
    const int k = P.k, E = P.E;
    int e = -1;
    uint32_t mykey = 0;
    float wgiven = 0.f;
    if (P.logits) {
      if (E <= 64) mykey = topk_keys<2>(P.logits, E, k, lane);
      else if (E <= 128) mykey = topk_keys<4>(P.logits, E, k, lane);
      else mykey = topk_keys<8>(P.logits, E, k, lane);
      if (lane < k) e = 0xffff - (int)(mykey & 0xffffu);
    } else if (lane < k) {
      e = P.idx_in[lane];
      wgiven = P.wts_in[lane];
    }
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
    const int m = dup ? 0 : total;
    if (in && !dup) {
      s.act[below] = e;
      s.sl[below] = sl;
    }
    if (lane < kMaxSel) {
      s.rank[lane] = (in && !dup) ? below : -1;
      s.key[lane] = mykey;
      s.wsel[lane] = wgiven;
    }
    if (lane == 0 && dup) report_status(P.ctl, MOE_ERR_ARG, kSiteOver);
    RPlan pl;
    pl.init(m, H, I);
    const bool joint = pl.joint(G);
    const int u1b = pl.lo1(cta, G, joint), u1e = pl.lo1(cta + 1, G, joint);
    const int u2b = RPlan::lo2(cta, pl.nU2, G), u2e = m > 0 ? RPlan::lo2(cta + 1, pl.nU2, G) : u2b;
    if (lane == 0) {
      s.nact = m;
      s.u1b = u1b; s.u1e = u1e; s.u2b = u2b; s.u2e = u2e;
      trace_at(P, 1);
    }
    __syncwarp();
    // every copy of this CTA, issued by the 32 lanes side by side: phase-1 unit i is copies
    // 4i .. 4i + 3 (gate codes, up codes, gate scales, up scales), then phase-2 unit v and expert j
    // is two copies (codes and scales of the unit's two row groups)
    const int n1 = u1e - u1b, n2 = u2e - u2b;
    const uint64_t pol = tc::policy_evict_first();
    if (lane == 0) {
      for (int i = 0; i < n1; ++i) tc::mbar_arrive_expect_tx(&s.ufull[i], (uint32_t)pl.B1);
      for (int v = 0; v < n2; ++v) tc::mbar_arrive_expect_tx(&s.vfull[v], (uint32_t)pl.B2);
    }
    __syncwarp();
    const size_t w13_slot = (size_t)I * H, s13_slot = (size_t)2 * I * nH;     // bytes / scales per slot
    const size_t w2_slot = (size_t)H * I / 2, s2_slot = (size_t)H * nI;
    const int nc = 4 * n1 + 2 * n2 * m;
    for (int c = lane; c < nc; c += 32) {
      if (c < 4 * n1) {
        const int i = c >> 2, part = c & 3, u = u1b + i, j = u / nFB, fb = u - j * nFB;
        const int R = (part & 1) ? (I / kRowGroup + fb) : fb;       // gate or up row group
        const int slot = s.sl[j];
        uint8_t* dst = pieces + (size_t)i * pl.B1;
        if (part < 2) {
          tc::bulk_g2s(dst + (size_t)part * nH * kChunkBytes, P.w13 + slot * w13_slot + chunk_offset(R, 0, nH),
                       (uint32_t)(nH * kChunkBytes), &s.ufull[i], pol);
        } else {
          tc::bulk_g2s(dst + (size_t)2 * nH * kChunkBytes + (size_t)(part & 1) * nH * 16,
                       P.s13 + slot * s13_slot + chunk_scale_index(R, 0, nH), (uint32_t)(nH * 16), &s.ufull[i], pol);
        }
      } else {
        const int c2 = c - 4 * n1, vj = c2 >> 1, v = vj / m, j = vj - v * m, R = 2 * (u2b + v);
        const int slot = s.sl[j];
        uint8_t* dst = pieces + (size_t)n1 * pl.B1 + (size_t)v * pl.B2 + (size_t)j * 2 * nI * (kChunkBytes + 16);
        if ((c2 & 1) == 0)
          tc::bulk_g2s(dst, P.w2 + slot * w2_slot + chunk_offset(R, 0, nI), (uint32_t)(2 * nI * kChunkBytes),
                       &s.vfull[v], pol);
        else
          tc::bulk_g2s(dst + (size_t)2 * nI * kChunkBytes, P.s2 + slot * s2_slot + chunk_scale_index(R, 0, nI),
                       (uint32_t)(2 * nI * 16), &s.vfull[v], pol);
      }
    }
    if (lane == 0) trace_at(P, 2);
  }
  __syncthreads();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int m = s.nact, u1b = s.u1b, u1e = s.u1e, u2b = s.u2b, u2e = s.u2e;
  const int n1 = u1e - u1b, n2 = u2e - u2b;
  RPlan pl;
  pl.init(m, H, I);
  const uint32_t hbytes = (uint32_t)(m * nFB * kHBlock);

  if (warp == 0) {
    // ------------------------------------------------------------ router weights, exchange
    const int k = P.k;
    if (P.logits) {
      // renormalised weight of choice j = exp(l_j - l_max) / sum over the k chosen
      const uint32_t mykey = lane < kMaxSel ? s.key[lane] : 0u;
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
      const float w = lane < kMaxSel ? s.wsel[lane] : 0.f;   // the given weights, choice order
      __syncwarp();
      if (lane < k) {
        const int r = s.rank[lane];
        if (r >= 0) s.wsel[r] = w;
      }
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&s.wready);
    bool ok = true;
    if (n2 > 0) {
      if (lane == 0) {
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
          trace_at(P, 4);
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
      for (int i = 0; i < n1; ++i) tc::mbar_wait(&s.ufull[i], 0, &never);
      for (int v = 0; v < n2; ++v) tc::mbar_wait(&s.vfull[v], 0, &never);
      if (n2 > 0 && ok) tc::mbar_wait(&s.hfull, 0, &never);
    }
    __syncwarp();
  } else if (warp <= kRCompute) {
    // ------------------------------------------------------------ compute warps 1..16
    const uint32_t M = 0x0F0F0F0Fu;
    bool ok = true;
    // phase 1: unit i, K group gk: rows 0..7 of the MMA = gate rows, 8..15 = up rows
    for (int i = 0; i < n1; ++i) {
      const int b = i % kRedBufs;
      if (i >= kRedBufs && !rwait(&s.redempty[b], ((i / kRedBufs) - 1) & 1, abort, limit)) { ok = false; break; }
      if (!rwait(&s.ufull[i], 0, abort, limit)) { ok = false; break; }
      if (gk >= 0) {
        const uint8_t* unit = pieces + (size_t)i * pl.B1;
        const uint8_t* gch = unit + (size_t)gk * kChunkBytes + gq * 16 + 4 * cq;
        const uint8_t* uch = gch + (size_t)nH * kChunkBytes;
        int d[4] = {0, 0, 0, 0};
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const uint32_t wa = *reinterpret_cast<const uint32_t*>(gch + kq * 128);
          const uint32_t wb = *reinterpret_cast<const uint32_t*>(uch + kq * 128);
          imma(d, wa & M, wb & M, (wa >> 4) & M, (wb >> 4) & M, xb0[kq], xb1[kq]);
        }
        if (cq == 0) {   // columns 0 / 1 = hi / lo of the token
          const uint16_t* scl = reinterpret_cast<const uint16_t*>(unit + (size_t)2 * nH * kChunkBytes);
          const float sg = bf16_bits_to_float(scl[gk * kRowGroup + gq]);
          const float su = bf16_bits_to_float(scl[nH * kRowGroup + gk * kRowGroup + gq]);
          s.red1[b][cw][gq] = sg * xa * (float)(d[0] * 256 + d[1] - xcorr);
          s.red1[b][cw][kF + gq] = su * xa * (float)(d[2] * 256 + d[3] - xcorr);
        }
      } else if (lane < 2 * kF) {
        s.red1[b][cw][lane] = 0.f;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.redfull[b]);
    }
    if (cw == 0 && lane == 0) trace_at(P, 3);
    // phase 2: unit v = 16 output rows over every selected expert. Warp cw takes the (expert,
    // K group) pairs [cw P / 16, (cw + 1) P / 16), P = m nI. Lane (g, c): A rows g (first row
    // group) and g + 8 (second); B column g holds, in K quarter c, the hi (g even) or lo (g odd)
    // bytes of the 8-feature h block c of the k-step, so D[r][2c], D[r][2c + 1] are block c's
    // hi and lo sums and the lane applies block c's scale.
    // (every compute warp runs every phase-2 unit and meets both named barriers, also after a
    // failed wait: its MMAs and stores are then skipped)
    bool h_in = false;
    for (int v = 0; v < n2; ++v) {
      ok = ok && rwait(&s.vfull[v], 0, abort, limit);
      if (ok && !h_in) {
        ok = rwait(&s.hfull, 0, abort, limit);
        h_in = ok;
        if (ok && cw == 0 && lane == 0) trace_at(P, 5);
      }
      const uint8_t* unit = pieces + (size_t)n1 * pl.B1 + (size_t)v * pl.B2;
      const int np = m * nI, p0 = cw * np / kRCompute, p1 = ok ? (cw + 1) * np / kRCompute : p0;
      float y0 = 0.f, y1 = 0.f;
      for (int p = p0; p < p1; ++p) {
        const int j = p / nI, g2 = p - j * nI;
        const uint8_t* ex = unit + (size_t)j * 2 * nI * (kChunkBytes + 16);
        const uint8_t* ch0 = ex + (size_t)g2 * kChunkBytes + gq * 16 + 4 * cq;
        const uint8_t* ch1 = ch0 + (size_t)nI * kChunkBytes;
        const uint16_t* scl = reinterpret_cast<const uint16_t*>(ex + (size_t)2 * nI * kChunkBytes);
        const uint8_t* hb = hsm + ((size_t)j * nFB + g2 * 16) * kHBlock;   // the group's 16 h blocks
        float t0 = 0.f, t1 = 0.f;
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) {
          const uint32_t wa = *reinterpret_cast<const uint32_t*>(ch0 + kq * 128);
          const uint32_t wb = *reinterpret_cast<const uint32_t*>(ch1 + kq * 128);
          const uint8_t* blk = hb + (kq * 4 + cq) * kHBlock;
          uint2 hv = make_uint2(0u, 0u);
          if ((gq >> 1) == cq) hv = *reinterpret_cast<const uint2*>(blk + (gq & 1) * 8);
          int d[4];
          imma0(d, wa & M, wb & M, (wa >> 4) & M, (wb >> 4) & M, hv.x, hv.y);
          const float2 rec = *reinterpret_cast<const float2*>(blk + 16);   // {a, a * 8 sum v}
          t0 += fmaf(rec.x, (float)(d[0] * 256 + d[1]), -rec.y);
          t1 += fmaf(rec.x, (float)(d[2] * 256 + d[3]), -rec.y);
        }
        y0 = fmaf(bf16_bits_to_float(scl[g2 * kRowGroup + gq]), t0, y0);
        y1 = fmaf(bf16_bits_to_float(scl[nI * kRowGroup + g2 * kRowGroup + gq]), t1, y1);
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
      tc::named_bar_sync(1, kRCompute * 32);
      if (cw == 0 && lane < kORows && !*abort) {
        float y = 0.f;
#pragma unroll
        for (int w = 0; w < kRCompute; ++w) y += s.red2[w][lane];
        store_output(P, 0, (u2b + v) * kORows + lane, y);
      }
      tc::named_bar_sync(1, kRCompute * 32);
    }
    if (!ok && lane == 0) report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteStage);
  } else {
    // ------------------------------------------------------------ h warps 17, 18
    // unit i goes to h warp i % 2: the 16 warps' sums (fixed order), h = w * silu(gate) * up of
    // its 8 features, encoded as one 24-byte block; then one arrival per CTA
    const int hw = warp - 1 - kRCompute;
    bool ok = rwait(&s.wready, 0, abort, limit);
    for (int i = hw; i < n1 && ok; i += kRHWarps) {
      const int b = i % kRedBufs;
      if (!rwait(&s.redfull[b], (i / kRedBufs) & 1, abort, limit)) { ok = false; break; }
      float sum = 0.f;
      if (lane < 2 * kF)
#pragma unroll
        for (int w = 0; w < kRCompute; ++w) sum += s.red1[b][w][lane];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.redempty[b]);
      const float up = __shfl_sync(kFull, sum, (lane & 7) + kF);
      const int u = u1b + i, j = u / nFB, fb = u - j * nFB;
      const float wt = s.wsel[j];
      float hv = 0.f;
      if (lane < kF && wt != 0.f) hv = __fdividef(sum * up, 1.f + __expf(-sum)) * wt;
      float mx = fabsf(hv);
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
      const float inv = mx > 0.f ? 32639.f / mx : 0.f;
      const int iv = lane < kF ? max(-32639, min(32639, __float2int_rn(hv * inv))) : 0;
      const int h8 = (iv + 128) >> 8, l8 = iv - 256 * h8;
      int sv = iv;
      sv += __shfl_xor_sync(kFull, sv, 1);
      sv += __shfl_xor_sync(kFull, sv, 2);
      sv += __shfl_xor_sync(kFull, sv, 4);
      // the hi and lo bytes in the permuted element order, gathered into two 64-bit words
      const int pos = rperm(lane & 7);
      unsigned long long hw64 = lane < kF ? (unsigned long long)(h8 & 0xff) << (8 * pos) : 0ull;
      unsigned long long lw64 = lane < kF ? (unsigned long long)(l8 & 0xff) << (8 * pos) : 0ull;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        hw64 |= __shfl_xor_sync(kFull, hw64, o);
        lw64 |= __shfl_xor_sync(kFull, lw64, o);
      }
      if (lane == 0) {
        const float a = mx * (1.f / 32639.f);
        unsigned long long* dst = reinterpret_cast<unsigned long long*>(P.hbuf + ((size_t)j * nFB + fb) * kHBlock);
        const float2 rec = make_float2(a, a * (float)(8 * sv));
        dst[0] = hw64;
        dst[1] = lw64;
        dst[2] = *reinterpret_cast<const unsigned long long*>(&rec);
      }
    }
    // both h warps meet, then one release: every block of this CTA is ordered before it. Every
    // CTA arrives whenever an expert is selected (also after a failed wait, which the status word
    // records), so the counter stays a multiple of G between launches.
    tc::named_bar_sync(2, kRHWarps * 32);
    if (hw == 0 && lane == 0 && m > 0) {
      red_release_add_u64(seq, 1ull);
      trace_at(P, 6);
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
  if (tid == 0) trace_at(P, 7);
}

// ---------------------------------------------------------------- host side
size_t rows_static_smem() { return sizeof(RSmem); }
size_t rows_h_bytes(int I, int m_max) { return ((size_t)m_max * (I / kF) * kHBlock + 127) & ~(size_t)127; }

// Largest piece area and unit counts any CTA needs for m selected experts.
bool rows_plan_fits(int H, int I, int m, int G, size_t cap) {
  RPlan pl;
  pl.init(m, H, I);
  const bool joint = pl.joint(G);
  for (int c = 0; c < G; ++c) {
    const int n1 = pl.lo1(c + 1, G, joint) - pl.lo1(c, G, joint);
    const int n2 = RPlan::lo2(c + 1, pl.nU2, G) - RPlan::lo2(c, pl.nU2, G);
    if (n1 < 0 || n1 > kMaxU1 || n2 > kMaxU2) return false;
    if ((size_t)n1 * pl.B1 + (size_t)n2 * pl.B2 > cap) return false;
  }
  return true;
}

size_t rows_smem_bytes(int H, int I, int m_max) {
  RPlan pl;
  pl.init(m_max, H, I);
  (void)pl;
  return kSmemLimit;   // the piece area takes what the static part and the h blocks leave
}

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
