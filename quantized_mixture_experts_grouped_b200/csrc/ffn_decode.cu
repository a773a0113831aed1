// Fused decode path of the W4A16 MoE layer: routing, grouping, gate/up with SiLU*up, down
// projection and the router-weighted combine in ONE persistent launch ("Every Expert Counts:
// ExactMoE for Memory-Efficient W4A16 Inference", Abstract: all selected experts execute
// through fused grouped MoE kernels; the router's top-k is unchanged).
//
// Small batches (T*k <= 256) read every selected expert's packed weights exactly once, so the
// layer is bound by HBM bandwidth on those bytes. Design for sm_100a:
//  * every CTA routes the batch itself (warp top-k, same rules as moe_route_topk) and builds the
//    expert grouping in shared memory, so no launch precedes the weight stream;
//  * work is cut into ~32 KB units, claimed dynamically through an atomic counter:
//      A units = (expert, 128-row block of I, K split of H)   gate and up tiles
//      B units = (expert, 128-row block of H, K split of I)   down tiles
//    all A units are handed out before any B unit;
//  * warp 0 streams 8 KB int4 tiles + their 256 B of scales into a 12-stage shared-memory ring
//    with bulk async copies (TMA), evict-first in L2, and stages the unit's activations (bf16,
//    K-major, no swizzle) for the MMA;
//  * warps 6..13 dequantise: each thread owns one weight row of the tile, turns 64 int4 codes
//    into bf16 (q * s, rounded once) with nibble-to-bf16 bit tricks, and writes them straight
//    into TENSOR MEMORY with tcgen05.st: the weights are the A operand of tcgen05.mma and never
//    pass through shared memory as bf16;
//  * one thread of warp 1 issues tcgen05.mma (M=128 weight rows, N=16/32 tokens, K=16,
//    A from TMEM, B from shared memory, fp32 accumulators in TMEM);
//  * warps 2..5 drain the accumulators with tcgen05.ld and write split-K partials; the last
//    unit of an (expert, row block) - found with an atomic counter - sums the partials in a
//    fixed order, applies silu(g)*u (bf16) and publishes the rows; B units wait (bounded) until
//    their expert's h is complete; the last B unit of a row block of H does the combine
//    out[t] = sum_j w_j y_j in fixed order. Results are deterministic run to run.
// Every wait is bounded; on a timeout the kernel records MOE_ERR_TIMEOUT in the workspace,
// drains its own copies and MMAs, frees its tensor memory and exits.
#include <algorithm>

#include "common.cuh"
#include "tc.cuh"

namespace moe {

__device__ __forceinline__ uint32_t route_key_d(uint32_t bits, int e) {
  bits &= 0xffffu;
  if (bits == 0x8000u) bits = 0;
  const uint32_t ord = (bits & 0x8000u) ? (~bits & 0xffffu) : (bits | 0x8000u);
  return (ord << 16) | (0xffffu - (uint32_t)e);
}

namespace {

constexpr int kStages = 12;
constexpr int kABufs = 4;
constexpr int kUQ = 4;
constexpr int kMaxTk = 256;
constexpr int kMaxT = 32;
constexpr int kBRowsMax = 32;
constexpr int kBKMax = 512;
constexpr int kThreads = 448;             // 14 warps
constexpr int kEpiWarp0 = 2;              // warps 2..5
constexpr int kDqWarp0 = 6;               // warps 6..13
constexpr int kTmemCols = 512;
constexpr int kAColBase = 0;              // 4 A buffers x 64 columns
constexpr int kDColBase = 256;            // 2 D buffers x (2 x NMMA) columns
constexpr uint32_t kTileTx = 8192 + 256;

// wait sites reported on timeout
enum { kSiteUQ = 1, kSiteStage = 2, kSiteABuf = 3, kSiteB = 4, kSiteD = 5, kSiteReady = 6, kSiteDrain = 7 };

struct DecParams {
  const uint16_t* x; const uint16_t* logits; const int32_t* idx_in; const float* wts_in;
  int T, H, I, E, k;
  const uint8_t* w13; const uint16_t* s13; const uint8_t* w2; const uint16_t* s2;
  const int32_t* slot;
  int32_t* idx_out; float* wts_out;
  uint16_t* out; float* acc; int accumulate;
  int* ctl; int* cntA; int* readyE; int* cntB;
  float* partA; float* partB; uint16_t* hp;
  int gA, gB, KSA, KSB, nmma;
};

struct __align__(128) DecSmem {
  uint8_t stage[kStages][8192];
  uint16_t scale[kStages][128];
  uint8_t bop[2][kBRowsMax * kBKMax * 2];
  int idx[kMaxTk];
  float wts[kMaxTk];
  int inv[kMaxTk];
  int plist[kMaxTk];
  int cnt[kMaxExperts];
  int off[kMaxExperts];
  int act[kMaxExperts];
  int wcount[8][kMaxExperts];
  uint64_t full[kStages], empty[kStages];
  uint64_t afull[kABufs], aempty[kABufs];
  uint64_t bfull[2], bempty[2], dfull[2], dempty[2];
  uint64_t uqf[kUQ], uqe[kUQ];
  uint64_t drain;
  int uq[kUQ];
  uint32_t tmem_base;
  int nact;
  int abort;
  int last_flag;
};

struct Unit {
  int type;    // 0: gate/up (A), 1: down (B)
  int e, slot, blk, ks, ntile, p0, ne;
};

__device__ __forceinline__ Unit decode_unit(const DecSmem& s, const DecParams& P, int u) {
  const int IB = P.I / kRowBlock, HB = P.H / kRowBlock;
  const int nA = s.nact * IB * P.KSA;
  Unit U;
  int a, r;
  if (u < nA) {
    U.type = 0;
    a = u / (IB * P.KSA);
    r = u % (IB * P.KSA);
    U.blk = r / P.KSA;
    U.ks = r % P.KSA;
    U.ntile = 2 * P.gA;
  } else {
    u -= nA;
    U.type = 1;
    a = u / (HB * P.KSB);
    r = u % (HB * P.KSB);
    U.blk = r / P.KSB;
    U.ks = r % P.KSB;
    U.ntile = P.gB;
  }
  U.e = s.act[a];
  U.slot = slot_of(P.slot, U.e);
  U.p0 = s.off[U.e];
  U.ne = s.cnt[U.e];
  return U;
}

// Every lane waits (each gets the barrier's acquire); the outcome is made warp-uniform so that
// a timeout can never leave the lanes of one warp on different paths.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = tc::mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void report_abort(DecSmem& s, const DecParams& P, int site) {
  s.abort = 1;
  report_status(P.ctl, MOE_ERR_TIMEOUT, site);
}

// Routes token t with one warp (same rules as route_kernel): writes s.idx / s.wts.
__device__ void route_token(DecSmem& s, const DecParams& P, int t, int lane) {
  const int E = P.E, k = P.k;
  const uint16_t* lt = P.logits + (size_t)t * E;
  constexpr int kPer = kMaxExperts / 32;
  uint32_t key[kPer];
  float lv[kPer];
  uint32_t taken = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const uint32_t b = lt[e];
      key[i] = route_key_d(b, e);
      lv[i] = bf16_bits_to_float(b);
    } else {
      key[i] = 0;
      lv[i] = -INFINITY;
    }
  }
  float mx = 0.f;
  for (int j = 0; j < k; ++j) {
    uint32_t best = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (!(taken >> i & 1u) && key[i] > best) best = key[i];
    const uint32_t win = __reduce_max_sync(0xffffffffu, best);
    const int e = 0xffff - (int)(win & 0xffffu);
    if ((e & 31) == lane) taken |= 1u << (e >> 5);
    if (lane == 0) s.idx[t * k + j] = e;
    if (j == 0) {
      const uint32_t ord = win >> 16;
      mx = bf16_bits_to_float((ord & 0x8000u) ? (ord & 0x7fffu) : (~ord & 0xffffu));
    }
  }
  __syncwarp();
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if (lane + 32 * i < E) z += expf(lv[i] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  float p[kPer];
  float sel = 0.f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = 32 * i + lane;
    p[i] = 0.f;
    if (j < k) p[i] = expf(bf16_bits_to_float(lt[s.idx[t * k + j]]) - mx) / z;
    sel += p[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sel += __shfl_xor_sync(0xffffffffu, sel, o);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = 32 * i + lane;
    if (j < k) s.wts[t * k + j] = p[i] / sel;
  }
}

// Routing (or loading the given routing) and the expert grouping, by the whole CTA.
__device__ void build_plan(DecSmem& s, const DecParams& P) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Tk = P.T * P.k, E = P.E;
  if (P.logits) {
    for (int t = warp; t < P.T; t += kThreads / 32) route_token(s, P, t, lane);
  } else {
    for (int i = tid; i < Tk; i += kThreads) {
      s.idx[i] = P.idx_in[i];
      s.wts[i] = P.wts_in[i];
    }
  }
  for (int i = tid; i < 8 * kMaxExperts; i += kThreads) (&s.wcount[0][0])[i] = 0;
  __syncthreads();
  if (P.logits && P.idx_out && blockIdx.x == 0)
    for (int i = tid; i < Tk; i += kThreads) {
      P.idx_out[i] = s.idx[i];
      P.wts_out[i] = s.wts[i];
    }
  int e = -1;
  unsigned lower = 0;
  if (warp < 8) {
    if (tid < Tk) {
      e = s.idx[tid];
      if ((unsigned)e >= (unsigned)E || slot_of(P.slot, e) < 0) e = -1;
    }
    const unsigned same = __match_any_sync(0xffffffffu, e);
    lower = same & ((1u << lane) - 1u);
    if (e >= 0 && lower == 0) s.wcount[warp][e] = __popc(same);
  }
  __syncthreads();
  for (int x = tid; x < E; x += kThreads) {
    int c = 0;
    for (int w = 0; w < 8; ++w) c += s.wcount[w][x];
    s.cnt[x] = c;
  }
  __syncthreads();
  if (warp == 0) {   // exclusive prefix over experts + compact list of the active ones
    int carry = 0, nact = 0;
    for (int base = 0; base < E; base += 32) {
      const int x = base + lane;
      const int c = x < E ? s.cnt[x] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (x < E) s.off[x] = carry + incl - c;
      const unsigned act = __ballot_sync(0xffffffffu, c > 0);
      if (c > 0) s.act[nact + __popc(act & ((1u << lane) - 1u))] = x;
      nact += __popc(act);
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    // an expert with more pairs than the MMA has columns (only possible with caller-made
    // routing that repeats an expert within a token) is refused rather than overflowing
    bool over = false;
    for (int x = lane; x < E; x += 32) over |= s.cnt[x] > P.nmma;
    over = __any_sync(0xffffffffu, over);
    if (lane == 0) {
      s.nact = over ? 0 : nact;
      if (over) report_status(P.ctl, MOE_ERR_ARG, 8);
    }
  }
  __syncthreads();
  if (tid < Tk) {
    if (e >= 0) {
      int rank = __popc(lower);
      for (int w = 0; w < warp; ++w) rank += s.wcount[w][e];
      const int pos = s.off[e] + rank;
      s.plist[pos] = tid;
      s.inv[tid] = pos;
    } else {
      s.inv[tid] = -1;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 1) moe_decode_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecSmem& s = *reinterpret_cast<DecSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) { tc::mbar_init(&s.full[i], 1); tc::mbar_init(&s.empty[i], 8); }
    for (int i = 0; i < kABufs; ++i) { tc::mbar_init(&s.afull[i], 8); tc::mbar_init(&s.aempty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&s.bfull[i], 1); tc::mbar_init(&s.bempty[i], 1);
      tc::mbar_init(&s.dfull[i], 1); tc::mbar_init(&s.dempty[i], 4);
    }
    for (int i = 0; i < kUQ; ++i) { tc::mbar_init(&s.uqf[i], 1); tc::mbar_init(&s.uqe[i], 1 + 4 + 8); }
    tc::mbar_init(&s.drain, 1);
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc<kTmemCols>(&s.tmem_base);
    tc::tc_fence_before();
  }
  build_plan(s, P);      // ends with __syncthreads
  tc::tc_fence_after();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (s.nact == 0 && blockIdx.x == 0) {   // no resident expert routed: out = accumulator (or 0)
    for (int i = tid; i < P.T * P.H; i += kThreads) {
      const float v = P.accumulate ? P.acc[i] : 0.f;
      if (P.out) {
        P.out[i] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        if (P.accumulate) P.acc[i] = 0.f;
      } else {
        P.acc[i] = v;
      }
    }
  }
  const uint32_t tmem = s.tmem_base;
  const int IB = P.I / kRowBlock, HB = P.H / kRowBlock;
  const int GH = P.H / kRowBlock, GI = P.I / kRowBlock;
  const int U_total = s.nact * (IB * P.KSA + HB * P.KSB);
  const int nmma = P.nmma;
  volatile int* abort = &s.abort;
  const size_t w13_bytes = (size_t)P.I * P.H, s13_count = (size_t)2 * P.I * GH;
  const size_t w2_bytes = (size_t)P.H * P.I / 2, s2_count = (size_t)P.H * GI;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = tc::policy_evict_first();
    int stage_it = 0;
    for (int unit_it = 0;; ++unit_it) {
      int u = 0;
      if (lane == 0) u = atomicAdd(P.ctl + kCtlClaim, 1);
      u = __shfl_sync(0xffffffffu, u, 0);
      const bool stop = (u >= U_total) || *abort;
      const int q = unit_it % kUQ;
      if (!warp_wait(&s.uqe[q], ((unit_it / kUQ) & 1) ^ 1, abort)) {
        if (lane == 0) report_abort(s, P, kSiteUQ);
        break;
      }
      if (lane == 0) {
        s.uq[q] = stop ? -1 : u;
        tc::mbar_arrive(&s.uqf[q]);
      }
      if (stop) break;
      const Unit U = decode_unit(s, P, u);
      bool ok = true;
      for (int ti = 0; ti < U.ntile && ok; ++ti) {
        const int st = stage_it % kStages;
        ok = warp_wait(&s.empty[st], ((stage_it / kStages) & 1) ^ 1, abort);
        if (!ok) break;
        if (lane == 0) {
          const uint8_t* wsrc;
          const uint16_t* ssrc;
          size_t tile;
          if (U.type == 0) {
            const int rb = (ti & 1) ? IB + U.blk : U.blk;
            const int g = U.ks * P.gA + (ti >> 1);
            tile = (size_t)rb * GH + g;
            wsrc = P.w13 + (size_t)U.slot * w13_bytes + tile * kTileBytes;
            ssrc = P.s13 + (size_t)U.slot * s13_count + tile * kRowBlock;
          } else {
            const int g = U.ks * P.gB + ti;
            tile = (size_t)U.blk * GI + g;
            wsrc = P.w2 + (size_t)U.slot * w2_bytes + tile * kTileBytes;
            ssrc = P.s2 + (size_t)U.slot * s2_count + tile * kRowBlock;
          }
          tc::mbar_arrive_expect_tx(&s.full[st], kTileTx);
          tc::bulk_g2s(s.stage[st], wsrc, 8192, &s.full[st], pol);
          tc::bulk_g2s(s.scale[st], ssrc, 256, &s.full[st], pol);
        }
        ++stage_it;
      }
      if (!ok) {
        if (lane == 0) report_abort(s, P, kSiteStage);
        break;
      }
      // activations of this unit -> B operand buffer (K-major, no swizzle)
      const int bb = unit_it & 1;
      if (!warp_wait(&s.bempty[bb], ((unit_it >> 1) & 1) ^ 1, abort)) {
        if (lane == 0) report_abort(s, P, kSiteB);
        break;
      }
      if (U.type == 1) {   // h of this expert must be complete (every lane acquires the flag)
        bool ready = false;
        const unsigned long long t0 = tc::globaltimer();
        while (true) {
          if (tc::ld_acquire(P.readyE + U.e) >= IB) { ready = true; break; }
          if (*abort) break;
          if (tc::globaltimer() - t0 > tc::kWaitTimeoutNs) break;
          __nanosleep(32);
        }
        ready = __all_sync(0xffffffffu, ready);
        if (!ready) {
          if (lane == 0) report_abort(s, P, kSiteReady);
          break;
        }
      }
      const int kc = (U.type == 0 ? P.gA : P.gB) * kGroup;       // K values of this unit
      const int k0 = U.ks * kc;
      const int chunks_per_row = kc / 8;
      const int nchunks = U.ne * chunks_per_row;
      uint8_t* bdst = s.bop[bb];
      for (int c = lane; c < nchunks; c += 32) {
        const int n = c / chunks_per_row, kq = c % chunks_per_row;
        uint4 v;
        if (U.type == 0) {
          const int t = s.plist[U.p0 + n] / P.k;
          v = __ldg(reinterpret_cast<const uint4*>(P.x + (size_t)t * P.H + k0) + kq);
        } else {
          v = __ldcg(reinterpret_cast<const uint4*>(P.hp + (size_t)(U.p0 + n) * P.I + k0) + kq);
        }
        *reinterpret_cast<uint4*>(bdst + (kq * (nmma / 8) + n / 8) * 128 + (n % 8) * 16) = v;
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.bfull[bb]);
    }
    // make sure no bulk copy is still landing in shared memory before the CTA exits
    if (lane == 0) {
      const int n = stage_it < kStages ? stage_it : kStages;
      for (int i = 0; i < n; ++i) {
        const int it = stage_it - 1 - i;
        volatile int never = 0;
        tc::mbar_wait(&s.full[it % kStages], (it / kStages) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(128, nmma);
      int a_it = 0;
      for (int unit_it = 0;; ++unit_it) {
        const int q = unit_it % kUQ;
        if (!tc::mbar_wait(&s.uqf[q], (unit_it / kUQ) & 1, abort)) { report_abort(s, P, kSiteUQ); break; }
        const int u = s.uq[q];
        tc::mbar_arrive(&s.uqe[q]);
        if (u < 0) break;
        const Unit U = decode_unit(s, P, u);
        const int bb = unit_it & 1, db = unit_it & 1;
        if (!tc::mbar_wait(&s.bfull[bb], (unit_it >> 1) & 1, abort)) { report_abort(s, P, kSiteB); break; }
        if (!tc::mbar_wait(&s.dempty[db], ((unit_it >> 1) & 1) ^ 1, abort)) { report_abort(s, P, kSiteD); break; }
        tc::tc_fence_after();
        const uint32_t dcol = kDColBase + db * 2 * nmma;
        const uint32_t bbase = tc::smem_u32(s.bop[bb]);
        const uint32_t lbo = (nmma / 8) * 128;
        bool ok = true;
        for (int ti = 0; ti < U.ntile; ++ti) {
          const int ab = a_it % kABufs;
          if (!tc::mbar_wait(&s.afull[ab], (a_it / kABufs) & 1, abort)) { ok = false; break; }
          tc::tc_fence_after();
          const int m = (U.type == 0) ? (ti & 1) : 0;
          const int gi = (U.type == 0) ? (ti >> 1) : ti;
          const uint32_t d = tmem + dcol + m * nmma;
          const uint32_t a = tmem + kAColBase + ab * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int kel = gi * kGroup + kk * 16;       // K offset inside the unit
            const uint64_t bdesc = tc::smem_desc(bbase + (kel / 8) * lbo, lbo, 128, 0);
            tc::mma_ts(d, a + kk * 8, bdesc, idesc, (gi > 0 || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(&s.aempty[ab]);
          ++a_it;
        }
        if (!ok) { report_abort(s, P, kSiteABuf); break; }
        tc::mma_commit(&s.dfull[db]);
        tc::mma_commit(&s.bempty[bb]);
      }
      tc::mma_commit(&s.drain);
      volatile int never = 0;
      if (!tc::mbar_wait(&s.drain, 0, &never)) report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteDrain);
    }
    __syncwarp();
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------------------------ dequantisers -> TMEM
    const int quarter = warp & 3, half = (warp - kDqWarp0) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t taddr_row = tmem + ((uint32_t)(quarter * 32) << 16) + kAColBase + half * 32;
    const __nv_bfloat162 off136 = __floats2bfloat162_rn(136.f, 136.f);
    int stage_it = 0, a_it = 0;
    for (int unit_it = 0;; ++unit_it) {
      const int q = unit_it % kUQ;
      if (!warp_wait(&s.uqf[q], (unit_it / kUQ) & 1, abort)) break;
      const int u = s.uq[q];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.uqe[q]);
      if (u < 0) break;
      const Unit U = decode_unit(s, P, u);
      bool ok = true;
      for (int ti = 0; ti < U.ntile; ++ti) {
        const int st = stage_it % kStages;
        if (!warp_wait(&s.full[st], (stage_it / kStages) & 1, abort)) { ok = false; break; }
        const uint4 c0 = *reinterpret_cast<const uint4*>(s.stage[st] + (2 * half) * 2048 + r * 16);
        const uint4 c1 = *reinterpret_cast<const uint4*>(s.stage[st] + (2 * half + 1) * 2048 + r * 16);
        const uint32_t sb = s.scale[st][r];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.empty[st]);
        ++stage_it;
        const uint32_t s2u = sb | (sb << 16);
        const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&s2u);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
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
        const int ab = a_it % kABufs;
        if (!warp_wait(&s.aempty[ab], ((a_it / kABufs) & 1) ^ 1, abort)) { ok = false; break; }
        tc::tc_fence_after();
        tc::tmem_st32(taddr_row + ab * 64, v);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.afull[ab]);
        ++a_it;
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int etid = tid - kEpiWarp0 * 32;      // 0..127
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int unit_it = 0;; ++unit_it) {
      const int q = unit_it % kUQ;
      if (!warp_wait(&s.uqf[q], (unit_it / kUQ) & 1, abort)) break;
      const int u = s.uq[q];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.uqe[q]);
      if (u < 0) break;
      const Unit U = decode_unit(s, P, u);
      const int db = unit_it & 1;
      if (!warp_wait(&s.dfull[db], (unit_it >> 1) & 1, abort)) break;
      tc::tc_fence_after();
      const uint32_t dcol = kDColBase + db * 2 * nmma;
      uint32_t g[kBRowsMax], h[kBRowsMax];
      {
        uint32_t tmp[16];
        tc::tmem_ld16(trow + dcol, tmp);
#pragma unroll
        for (int i = 0; i < 16; ++i) g[i] = tmp[i];
        if (nmma > 16) {
          tc::tmem_ld16(trow + dcol + 16, tmp);
#pragma unroll
          for (int i = 0; i < 16; ++i) g[16 + i] = tmp[i];
        }
        if (U.type == 0) {
          tc::tmem_ld16(trow + dcol + nmma, tmp);
#pragma unroll
          for (int i = 0; i < 16; ++i) h[i] = tmp[i];
          if (nmma > 16) {
            tc::tmem_ld16(trow + dcol + nmma + 16, tmp);
#pragma unroll
            for (int i = 0; i < 16; ++i) h[16 + i] = tmp[i];
          }
        }
      }
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.dempty[db]);

      if (U.type == 0) {
        const size_t rowA = (size_t)2 * P.I;
#pragma unroll
        for (int n = 0; n < kBRowsMax; ++n) {
          if (n >= U.ne) break;
          float* pa = P.partA + ((size_t)(U.p0 + n) * P.KSA + U.ks) * rowA + U.blk * kRowBlock + r;
          pa[0] = __uint_as_float(g[n]);
          pa[P.I] = __uint_as_float(h[n]);
        }
      } else {
#pragma unroll
        for (int n = 0; n < kBRowsMax; ++n) {
          if (n >= U.ne) break;
          P.partB[((size_t)(U.p0 + n) * P.KSB + U.ks) * P.H + U.blk * kRowBlock + r] = __uint_as_float(g[n]);
        }
      }
      __threadfence();
      tc::named_bar_sync(1, 128);
      if (etid == 0) {
        int* cnt = (U.type == 0) ? P.cntA + U.e * IB + U.blk : P.cntB + U.blk;
        const int need = (U.type == 0) ? P.KSA : s.nact * P.KSB;
        s.last_flag = (atomicAdd(cnt, 1) == need - 1);
      }
      tc::named_bar_sync(1, 128);
      if (!s.last_flag) continue;
      __threadfence();
      if (U.type == 0) {
        // all K splits of this (expert, row block) are in: h = silu(g) * u
        const size_t rowA = (size_t)2 * P.I;
        for (int n = 0; n < U.ne; ++n) {
          const float* pa = P.partA + (size_t)(U.p0 + n) * P.KSA * rowA + U.blk * kRowBlock + r;
          float gs = 0.f, us = 0.f;
          for (int ks = 0; ks < P.KSA; ++ks) {
            gs += __ldcg(pa + ks * rowA);
            us += __ldcg(pa + ks * rowA + P.I);
          }
          const float hv = gs / (1.f + expf(-gs)) * us;
          P.hp[(size_t)(U.p0 + n) * P.I + U.blk * kRowBlock + r] = __bfloat16_as_ushort(__float2bfloat16_rn(hv));
        }
        __threadfence();
        tc::named_bar_sync(1, 128);
        if (etid == 0) {
          P.cntA[U.e * IB + U.blk] = 0;
          tc::red_release_add(P.readyE + U.e, 1);
        }
      } else {
        // every expert's contribution to this row block of H is in: combine in fixed order
        const int row = U.blk * kRowBlock + r;
        for (int t = 0; t < P.T; ++t) {
          float v = P.accumulate ? __ldcg(P.acc + (size_t)t * P.H + row) : 0.f;
          for (int j = 0; j < P.k; ++j) {
            const int pos = s.inv[t * P.k + j];
            if (pos < 0) continue;
            float y = 0.f;
            for (int ks = 0; ks < P.KSB; ++ks) y += __ldcg(P.partB + ((size_t)pos * P.KSB + ks) * P.H + row);
            v = fmaf(s.wts[t * P.k + j], y, v);
          }
          if (P.out) {
            P.out[(size_t)t * P.H + row] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            if (P.accumulate) P.acc[(size_t)t * P.H + row] = 0.f;
          } else {
            P.acc[(size_t)t * P.H + row] = v;
          }
        }
        tc::named_bar_sync(1, 128);
        if (etid == 0) P.cntB[U.blk] = 0;
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc<kTmemCols>(tmem);
  }
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(P.ctl + kCtlDone, 1) == (int)gridDim.x - 1) {
      // last CTA out: every unit is finished, reset the cross-CTA state for the next call
      __threadfence();
      for (int e = 0; e < P.E; ++e) P.readyE[e] = 0;
      P.ctl[kCtlClaim] = 0;
      P.ctl[kCtlDone] = 0;
      __threadfence();
    }
  }
}

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

int largest_divisor_le(int n, int cap) {
  for (int d = std::min(n, cap); d >= 1; --d)
    if (n % d == 0) return d;
  return 1;
}

}  // namespace

bool ffn_decode_supported(const FfnArgs& a) {
  return a.T >= 1 && a.T <= kMaxT && a.T * a.k <= kMaxTk && a.E <= kMaxExperts && a.H % kRowBlock == 0 &&
         a.I % kRowBlock == 0;
}

size_t decode_scratch_bytes(int T, int H, int I, int E, int k) {
  if (T < 1 || T > kMaxT || T * k > kMaxTk) return 0;
  const int GH = H / kGroup, GI = I / kGroup;
  const int KSA = GH / largest_divisor_le(GH, 2), KSB = GI / largest_divisor_le(GI, 4);
  const size_t Tk = (size_t)T * k;
  size_t b = 0;
  b += align_up(sizeof(int) * (size_t)E * (I / kRowBlock), 256);     // cntA
  b += align_up(sizeof(int) * (size_t)E, 256);                       // readyE
  b += align_up(sizeof(int) * (size_t)(H / kRowBlock), 256);         // cntB
  b += align_up(sizeof(float) * Tk * KSA * 2 * I, 256);              // partA
  b += align_up(sizeof(float) * Tk * KSB * H, 256);                  // partB
  return b;
}

int ffn_decode(const FfnArgs& a, cudaStream_t s) {
  const WsLayout L = ws_layout(a.T, a.H, a.I, a.E, a.k);
  const int GH = a.H / kGroup, GI = a.I / kGroup;
  DecParams P{};
  P.x = a.x; P.logits = a.logits; P.idx_in = a.idx; P.wts_in = a.wts;
  P.T = a.T; P.H = a.H; P.I = a.I; P.E = a.E; P.k = a.k;
  P.w13 = a.w13; P.s13 = a.s13; P.w2 = a.w2; P.s2 = a.s2; P.slot = a.slot;
  P.idx_out = a.idx_out; P.wts_out = a.wts_out;
  P.out = a.out; P.acc = reinterpret_cast<float*>(a.ws + L.acc); P.accumulate = a.accumulate ? 1 : 0;
  P.gA = largest_divisor_le(GH, 2);
  P.gB = largest_divisor_le(GI, 4);
  P.KSA = GH / P.gA;
  P.KSB = GI / P.gB;
  P.nmma = a.T <= 16 ? 16 : 32;
  char* d = a.ws + L.dec;
  P.ctl = reinterpret_cast<int*>(a.ws + L.status);
  P.cntA = reinterpret_cast<int*>(d);
  d += align_up(sizeof(int) * (size_t)a.E * (a.I / kRowBlock), 256);
  P.readyE = reinterpret_cast<int*>(d);
  d += align_up(sizeof(int) * (size_t)a.E, 256);
  P.cntB = reinterpret_cast<int*>(d);
  d += align_up(sizeof(int) * (size_t)(a.H / kRowBlock), 256);
  P.partA = reinterpret_cast<float*>(d);
  d += align_up(sizeof(float) * (size_t)a.T * a.k * P.KSA * 2 * a.I, 256);
  P.partB = reinterpret_cast<float*>(d);
  P.hp = reinterpret_cast<uint16_t*>(a.ws + L.hp);
  if (!a.logits && (!a.idx || !a.wts)) return fail(MOE_ERR_ARG, "fused decode: routing missing");

  const int max_act = std::min(a.E, a.T * a.k);
  const int max_units = max_act * ((a.I / kRowBlock) * P.KSA + (a.H / kRowBlock) * P.KSB);
  const int grid = std::max(1, std::min(num_sms(), max_units));
  const size_t smem = sizeof(DecSmem);
  static bool attr_done = false;
  if (!attr_done) {
    if (int rc = check_cuda(cudaFuncSetAttribute(moe_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem), "fused decode: smem attribute"))
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

}  // namespace moe
