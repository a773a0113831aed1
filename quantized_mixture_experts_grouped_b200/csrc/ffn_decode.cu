// Fused decode path of the W4A16 MoE layer: routing, grouping, gate/up with SiLU*up, down
// projection and the router-weighted combine in ONE persistent launch ("Every Expert Counts:
// ExactMoE for Memory-Efficient W4A16 Inference", Abstract: all selected experts execute
// through fused grouped MoE kernels; the router's top-k is unchanged).
//
// A decode batch (T <= 16 tokens) reads every selected expert's packed weights exactly once, so
// the layer is bound by HBM bandwidth on those bytes; the design keeps many weight bytes in
// flight per SM and keeps every cross-CTA step off the weight stream's critical path:
//  * every CTA routes the batch itself (warp top-k, same rules as moe_route_topk) and builds
//    the grouping in shared memory; the batch's activations are staged once in shared memory
//    as the B operand of every gate/up MMA (all T tokens are MMA columns; a column whose token
//    is not routed to the expert is computed and ignored);
//  * the work is a static list of units, CTA c taking units c, c+G, c+2G, ...:
//      A units = (expert, 128-row block of I, quarter of H)   gate + up tiles (64 KB)
//      B units = (128-row block of H, 128-wide block of I, chunk of <= 8 experts)  down tiles
//    all A units come first;
//  * warp 0 streams 8 KB int4 tiles + 256 B of scales into a 12-stage ring with bulk async
//    copies (TMA, evict-first in L2);
//  * warps 6..13 dequantise in two groups that take alternate tiles: a thread owns one weight
//    row, turns 128 int4 codes into bf16 (q * s, one rounding) with nibble-to-bf16 bit tricks
//    and writes them straight into TENSOR MEMORY (tcgen05.st) as the A operand of
//    tcgen05.mma - the bf16 weights never pass through shared memory;
//  * one thread of warp 1 issues tcgen05.mma (M = 128 weight rows, N = 16 tokens, K = 16);
//  * A units end with fp32 partial sums of gate and up (split K) written to the workspace and a
//    release increment of a per-(expert, row block) counter - nobody waits for its result;
//  * warps 14..15 build each B unit's operand per expert: they wait for that expert's counter,
//    sum the partials, apply silu(g)*u and the router weight, and write bf16 rows (zero for
//    tokens not routed to the expert). The B unit's MMAs then accumulate EVERY expert of the
//    chunk into one accumulator: the router-weighted combine happens inside the MMA;
//  * the last B unit of a 128-row block of H (atomic counter) adds the split-K / expert-chunk
//    partials in a fixed order and writes the bf16 output. Results are deterministic.
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
constexpr int kBSlots = 8;
constexpr int kMaxTk = 256;
constexpr int kMaxT = 16;
constexpr int kN = 16;                    // MMA N: the batch's tokens (<= 16)
constexpr int kEC = 8;                    // experts per B unit
constexpr int kGAMax = 4;                 // K groups (of 128) per A unit, at most
constexpr int kThreads = 512;             // 16 warps
constexpr int kEpiWarp0 = 2;              // warps 2..5
constexpr int kDqWarp0 = 6;               // warps 6..13
constexpr int kBbWarp0 = 14;              // warps 14..15
constexpr int kTmemCols = 512;
constexpr int kAColBase = 0;              // 4 A buffers x 64 columns
constexpr int kDColBase = 256;            // 2 D buffers x 2 x kN columns
constexpr uint32_t kTileTx = 8192 + 256;
constexpr unsigned kFull = 0xffffffffu;

enum { kSiteStage = 2, kSiteABuf = 3, kSiteB = 4, kSiteD = 5, kSiteReady = 6, kSiteDrain = 7, kSiteOver = 8 };

struct DecParams {
  const uint16_t* x; const uint16_t* logits; const int32_t* idx_in; const float* wts_in;
  int T, H, I, E, k;
  const uint8_t* w13; const uint16_t* s13; const uint8_t* w2; const uint16_t* s2;
  const int32_t* slot;
  int32_t* idx_out; float* wts_out;
  uint16_t* out; float* acc; int accumulate;
  int* ctl; int* cntA; int* cntB;
  float* partA; float* partB;
  int gA, KSA;                  // K groups per A unit, A units per (expert, I-block)
  unsigned long long* trace;    // optional per-CTA timestamps (diagnostics), null in normal use
};

// trace slots per CTA (64 x u64): 0 start, 1 plan done, 2 first tile issued, 3 producer done,
// 4 epilogue done, 5 end, 8..15 epilogue finish time of the i-th unit, 16..47 dequant group 0
// (4 per tile: stage ready, stage read, A buffer free, TMEM written), 48..55 plan phases,
// 56..63 MMA issue of the first 8 tiles
__device__ __forceinline__ void trace_at(const DecParams& P, int slot) {
  if (P.trace) P.trace[blockIdx.x * 64 + slot] = tc::globaltimer();
}

struct __align__(128) DecSmem {
  uint8_t stage[kStages][8192];
  uint16_t scale[kStages][128];
  uint8_t bslot[kBSlots][kN * 128 * 2];     // per-expert down-projection operands (4 KB)
  int idx[kMaxTk];
  float wts[kMaxTk];
  float wgp[kMaxTk];                        // router weight of the pair at grouped position p
  int cnt[kMaxExperts];
  int off[kMaxExperts];
  int act[kMaxExperts];
  uint32_t tokmask[kMaxExperts];            // tokens routed to active expert a
  int16_t posof[kMaxExperts][kMaxT];        // grouped position of (active expert a, token t)
  int wcount[8][kMaxExperts];
  uint64_t full[kStages], empty[kStages];
  uint64_t afull[kABufs], aempty[kABufs];
  uint64_t bfull[kBSlots], bempty[kBSlots];
  uint64_t dfull[2], dempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int nact;
  int abort;
  int last_flag;
  // followed in dynamic shared memory by the activations: kN rows x H, no-swizzle K-major
};

struct Unit {
  int type;       // 0: A (gate/up), 1: B (down)
  int a, e, slot; // A: active expert index, expert, slot
  int blk, ks;    // A: I-block, H-quarter;  B: H-block, I-block
  int ec, na;     // B: expert chunk, experts in it
  int ntile;
};

__device__ __forceinline__ Unit decode_unit(const DecSmem& s, const DecParams& P, int u) {
  const int IB = P.I / kRowBlock, GI = P.I / kGroup;
  const int nA = s.nact * IB * P.KSA;
  const int nEC = (s.nact + kEC - 1) / kEC;
  Unit U;
  if (u < nA) {
    U.type = 0;
    U.a = u / (IB * P.KSA);
    const int r = u % (IB * P.KSA);
    U.blk = r / P.KSA;
    U.ks = r % P.KSA;
    U.e = s.act[U.a];
    U.slot = slot_of(P.slot, U.e);
    U.ec = 0; U.na = 0;
    U.ntile = 2 * P.gA;
  } else {
    u -= nA;
    U.type = 1;
    U.blk = u / (GI * nEC);
    const int r = u % (GI * nEC);
    U.ks = r / nEC;
    U.ec = r % nEC;
    U.na = min(kEC, s.nact - U.ec * kEC);
    U.a = U.e = U.slot = -1;
    U.ntile = U.na;
  }
  return U;
}

__device__ __forceinline__ int total_units(const DecSmem& s, const DecParams& P) {
  const int IB = P.I / kRowBlock, HB = P.H / kRowBlock, GI = P.I / kGroup;
  const int nEC = (s.nact + kEC - 1) / kEC;
  return s.nact * IB * P.KSA + HB * GI * nEC;
}

// Every lane waits (each gets the barrier's acquire); the outcome is made warp-uniform so that
// a timeout can never leave the lanes of one warp on different paths.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = tc::mbar_wait(bar, parity, abort);
  return __all_sync(kFull, ok);
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
    const uint32_t win = __reduce_max_sync(kFull, best);
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
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(kFull, z, o);
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
  for (int o = 16; o > 0; o >>= 1) sel += __shfl_xor_sync(kFull, sel, o);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = 32 * i + lane;
    if (j < k) s.wts[t * k + j] = p[i] / sel;
  }
}

// Element (n, k) of a kN-row, K-major operand without swizzle: 8x16-byte core matrices.
__device__ __forceinline__ uint32_t kmajor_off(int n, int k) {
  return (uint32_t)(((k >> 3) * (kN / 8) + (n >> 3)) * 128 + (n & 7) * 16 + (k & 7) * 2);
}

// Routing (or the given routing), activations into shared memory, expert grouping.
__device__ void build_plan(DecSmem& s, const DecParams& P, uint8_t* xs) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Tk = P.T * P.k, E = P.E;
  // activations: issue the loads first so that their latency overlaps the routing
  const int chunks = kN * (P.H / 8);
  constexpr int kPerThr = 8;
  uint4 xv[kPerThr];
#pragma unroll
  for (int i = 0; i < kPerThr; ++i) {
    const int c = tid + i * kThreads;
    xv[i] = make_uint4(0, 0, 0, 0);
    if (c < chunks) {
      const int n = c / (P.H / 8), kc = c % (P.H / 8);
      if (n < P.T) xv[i] = __ldg(reinterpret_cast<const uint4*>(P.x + (size_t)n * P.H) + kc);
    }
  }
  if (tid == 0) trace_at(P, 48);
  if (P.logits) {
    if (warp < P.T) route_token(s, P, warp, lane);
    if (tid == 0) trace_at(P, 49);
  } else {
    for (int i = tid; i < Tk; i += kThreads) {
      s.idx[i] = P.idx_in[i];
      s.wts[i] = P.wts_in[i];
    }
  }
  for (int i = tid; i < 8 * kMaxExperts; i += kThreads) (&s.wcount[0][0])[i] = 0;
  for (int c = tid + kPerThr * kThreads; c < chunks; c += kThreads) {   // H > 2048 leftovers
    const int n = c / (P.H / 8), kc = c % (P.H / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n < P.T) v = __ldg(reinterpret_cast<const uint4*>(P.x + (size_t)n * P.H) + kc);
    *reinterpret_cast<uint4*>(xs + kmajor_off(n, kc * 8)) = v;
  }
#pragma unroll
  for (int i = 0; i < kPerThr; ++i) {
    const int c = tid + i * kThreads;
    if (c < chunks) {
      const int n = c / (P.H / 8), kc = c % (P.H / 8);
      *reinterpret_cast<uint4*>(xs + kmajor_off(n, kc * 8)) = xv[i];
    }
  }
  __syncthreads();
  if (tid == 0) trace_at(P, 50);
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
    const unsigned same = __match_any_sync(kFull, e);
    lower = same & ((1u << lane) - 1u);
    if (e >= 0 && lower == 0) s.wcount[warp][e] = __popc(same);
  }
  __syncthreads();
  if (tid == 0) trace_at(P, 51);
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
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
      }
      if (x < E) s.off[x] = carry + incl - c;
      const unsigned actm = __ballot_sync(kFull, c > 0);
      if (c > 0) s.act[nact + __popc(actm & ((1u << lane) - 1u))] = x;
      nact += __popc(actm);
      carry += __shfl_sync(kFull, incl, 31);
    }
    bool over = false;          // a token routed twice to one expert (caller-made routing)
    for (int x = lane; x < E; x += 32) over |= s.cnt[x] > P.T;
    over = __any_sync(kFull, over);
    if (lane == 0) {
      s.nact = over ? 0 : nact;
      if (over) report_status(P.ctl, MOE_ERR_ARG, kSiteOver);
    }
  }
  __syncthreads();
  if (tid == 0) trace_at(P, 52);
  for (int i = tid; i < s.nact * kMaxT; i += kThreads) s.posof[i / kMaxT][i % kMaxT] = -1;
  __syncthreads();
  if (tid < Tk && e >= 0) {
    int rank = __popc(lower);
    for (int w = 0; w < warp; ++w) rank += s.wcount[w][e];
    s.wgp[s.off[e] + rank] = s.wts[tid];
  }
  if (tid < s.nact) {    // tokens of active expert a, in token order
    const int a = tid, x = s.act[a];
    uint32_t m = 0;
    int n = 0;
    for (int p = 0; p < Tk; ++p)
      if (s.idx[p] == x) {
        const int t = p / P.k;
        if (!((m >> t) & 1u)) {
          m |= 1u << t;
          s.posof[a][t] = (int16_t)(s.off[x] + n);
        }
        ++n;
      }
    s.tokmask[a] = m;
  }
  __syncthreads();
  if (tid == 0) trace_at(P, 53);
}

__global__ void __launch_bounds__(kThreads, 1) moe_decode_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecSmem& s = *reinterpret_cast<DecSmem*>(smem_raw);
  uint8_t* xs = smem_raw + sizeof(DecSmem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) trace_at(P, 0);
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) { tc::mbar_init(&s.full[i], 1); tc::mbar_init(&s.empty[i], 4); }
    for (int i = 0; i < kABufs; ++i) { tc::mbar_init(&s.afull[i], 4); tc::mbar_init(&s.aempty[i], 1); }
    for (int i = 0; i < kBSlots; ++i) { tc::mbar_init(&s.bfull[i], 1); tc::mbar_init(&s.bempty[i], 1); }
    for (int i = 0; i < 2; ++i) { tc::mbar_init(&s.dfull[i], 1); tc::mbar_init(&s.dempty[i], 4); }
    tc::mbar_init(&s.drain, 1);
    s.abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc<kTmemCols>(&s.tmem_base);
    tc::tc_fence_before();
  }
  build_plan(s, P, xs);      // ends with __syncthreads
  tc::tc_fence_after();
  tc::fence_proxy_async_smem();   // activations written by threads, read by the tensor core
  __syncthreads();
  if (tid == 0) trace_at(P, 1);
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
  const int IB = P.I / kRowBlock, GH = P.H / kGroup, GI = P.I / kGroup;
  const int U_total = total_units(s, P);
  const int nEC = (s.nact + kEC - 1) / kEC;
  const int G = gridDim.x;
  volatile int* abort = &s.abort;
  const size_t w13_bytes = (size_t)P.I * P.H, s13_count = (size_t)2 * P.I * GH;
  const size_t w2_bytes = (size_t)P.H * P.I / 2, s2_count = (size_t)P.H * GI;
  const size_t rowA = (size_t)2 * P.I;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = tc::policy_evict_first();
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < U_total && ok; u += G) {
      const Unit U = decode_unit(s, P, u);
      for (int ti = 0; ti < U.ntile; ++ti, ++it) {
        const int st = it % kStages;
        if (!warp_wait(&s.empty[st], ((it / kStages) & 1) ^ 1, abort)) { ok = false; break; }
        if (lane == 0) {
          const uint8_t* wsrc;
          const uint16_t* ssrc;
          if (U.type == 0) {
            const int rb = (ti & 1) ? IB + U.blk : U.blk;
            const size_t tile = (size_t)rb * GH + U.ks * P.gA + (ti >> 1);
            wsrc = P.w13 + (size_t)U.slot * w13_bytes + tile * kTileBytes;
            ssrc = P.s13 + (size_t)U.slot * s13_count + tile * kRowBlock;
          } else {
            const int e = s.act[U.ec * kEC + ti];
            const int sl = slot_of(P.slot, e);
            const size_t tile = (size_t)U.blk * GI + U.ks;
            wsrc = P.w2 + (size_t)sl * w2_bytes + tile * kTileBytes;
            ssrc = P.s2 + (size_t)sl * s2_count + tile * kRowBlock;
          }
          if (it == 0) trace_at(P, 2);
          tc::mbar_arrive_expect_tx(&s.full[st], kTileTx);
          tc::bulk_g2s(s.stage[st], wsrc, 8192, &s.full[st], pol);
          tc::bulk_g2s(s.scale[st], ssrc, 256, &s.full[st], pol);
        }
      }
    }
    if (!ok && lane == 0) report_abort(s, P, kSiteStage);
    if (lane == 0) trace_at(P, 3);
    if (lane == 0) {   // no bulk copy may still be landing in shared memory when the CTA leaves
      const int n = it < kStages ? it : kStages;
      for (int i = 0; i < n; ++i) {
        const int j = it - 1 - i;
        volatile int never = 0;
        tc::mbar_wait(&s.full[j % kStages], (j / kStages) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16_f32(128, kN);
      const uint32_t xbase = tc::smem_u32(xs);
      constexpr uint32_t lbo = (kN / 8) * 128;
      int a_it = 0, b_it = 0, i = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < U_total && ok; u += G, ++i) {
        const Unit U = decode_unit(s, P, u);
        const int db = i & 1;
        if (!tc::mbar_wait(&s.dempty[db], ((i >> 1) & 1) ^ 1, abort)) { ok = false; report_abort(s, P, kSiteD); break; }
        tc::tc_fence_after();
        const uint32_t dcol = tmem + kDColBase + db * 2 * kN;
        for (int ti = 0; ti < U.ntile; ++ti, ++a_it) {
          const int ab = a_it % kABufs;
          if (!tc::mbar_wait(&s.afull[ab], (a_it / kABufs) & 1, abort)) { ok = false; report_abort(s, P, kSiteABuf); break; }
          if (a_it < 8) trace_at(P, 56 + a_it);
          const uint32_t a = tmem + kAColBase + ab * 64;
          if (U.type == 0) {
            tc::tc_fence_after();
            const int m = ti & 1, gi = ti >> 1;
            const int k0 = (U.ks * P.gA + gi) * kGroup;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bdesc = tc::smem_desc(xbase + ((k0 + kk * 16) / 8) * lbo, lbo, 128, 0);
              tc::mma_ts(dcol + m * kN, a + kk * 8, bdesc, idesc, (gi > 0 || kk > 0) ? 1u : 0u);
            }
          } else {
            const int bs = b_it % kBSlots;
            if (!tc::mbar_wait(&s.bfull[bs], (b_it / kBSlots) & 1, abort)) { ok = false; report_abort(s, P, kSiteB); break; }
            tc::tc_fence_after();
            const uint32_t bbase = tc::smem_u32(s.bslot[bs]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bdesc = tc::smem_desc(bbase + kk * 2 * lbo, lbo, 128, 0);
              tc::mma_ts(dcol, a + kk * 8, bdesc, idesc, (ti > 0 || kk > 0) ? 1u : 0u);
            }
            tc::mma_commit(&s.bempty[bs]);
            ++b_it;
          }
          tc::mma_commit(&s.aempty[ab]);
        }
        if (ok) tc::mma_commit(&s.dfull[db]);
      }
      tc::mma_commit(&s.drain);
      volatile int never = 0;
      if (!tc::mbar_wait(&s.drain, 0, &never)) report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteDrain);
    }
    __syncwarp();
  } else if (warp >= kDqWarp0 && warp < kBbWarp0) {
    // ------------------------------------------------------------ dequantisers -> TMEM
    // two groups of four warps take alternate tiles; a thread owns row r of its group's tile
    const int quarter = warp & 3, grp = (warp - kDqWarp0) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t taddr_row = tmem + ((uint32_t)(quarter * 32) << 16) + kAColBase;
    const __nv_bfloat162 off136 = __floats2bfloat162_rn(136.f, 136.f);
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < U_total && ok; u += G) {
      const Unit U = decode_unit(s, P, u);
      for (int ti = 0; ti < U.ntile; ++ti, ++it) {
        if ((it & 1) != grp) continue;
        const int st = it % kStages;
        if (!warp_wait(&s.full[st], (it / kStages) & 1, abort)) { ok = false; break; }
        const bool tr = (warp == kDqWarp0 && lane == 0 && it < 16);
        if (tr) trace_at(P, 16 + (it >> 1) * 4);
        uint4 c[4];
#pragma unroll
        for (int kq = 0; kq < 4; ++kq) c[kq] = *reinterpret_cast<const uint4*>(s.stage[st] + kq * 2048 + r * 16);
        const uint32_t sb = s.scale[st][r];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.empty[st]);
        if (tr) trace_at(P, 17 + (it >> 1) * 4);
        const uint32_t s2u = sb | (sb << 16);
        const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&s2u);
        const int ab = it % kABufs;
        if (!warp_wait(&s.aempty[ab], ((it / kABufs) & 1) ^ 1, abort)) { ok = false; break; }
        if (tr) trace_at(P, 18 + (it >> 1) * 4);
        tc::tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t words[8] = {c[2 * h].x, c[2 * h].y, c[2 * h].z, c[2 * h].w,
                                     c[2 * h + 1].x, c[2 * h + 1].y, c[2 * h + 1].z, c[2 * h + 1].w};
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
          tc::tmem_st32(taddr_row + ab * 64 + h * 32, v);
        }
        tc::tmem_wait_st();
        if (tr) trace_at(P, 19 + (it >> 1) * 4);
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.afull[ab]);
      }
    }
  } else if (warp >= kBbWarp0) {
    // ------------------------------------------------------------ down-projection operands
    // per (B unit, expert): rows t = bf16(w * silu(g) * u) for tokens routed to the expert,
    // zero rows otherwise; g, u = sums of the gate/up split-K partials
    const int btid = tid - kBbWarp0 * 32;       // 0..63
    int b_it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < U_total && ok; u += G) {
      const Unit U = decode_unit(s, P, u);
      if (U.type == 0) continue;
      for (int ti = 0; ti < U.na && ok; ++ti, ++b_it) {
        const int a = U.ec * kEC + ti, e = s.act[a];
        const int bs = b_it % kBSlots;
        if (!warp_wait(&s.bempty[bs], ((b_it / kBSlots) & 1) ^ 1, abort)) { ok = false; break; }
        // this expert's h for I-block U.ks must be complete
        bool ready = false;
        const unsigned long long t0 = tc::globaltimer();
        while (true) {
          if (tc::ld_acquire(P.cntA + e * IB + U.ks) >= P.KSA) { ready = true; break; }
          if (*abort) break;
          if (tc::globaltimer() - t0 > tc::kWaitTimeoutNs) break;
          __nanosleep(20);
        }
        ready = __all_sync(kFull, ready);
        if (!ready) {
          if (lane == 0) report_abort(s, P, kSiteReady);
          ok = false;
          break;
        }
        uint8_t* dst = s.bslot[bs];
        const uint32_t tm = s.tokmask[a];
        for (int item = btid; item < kN * 16; item += 64) {
          const int t = item >> 4, kc = item & 15;
          uint4 o = make_uint4(0, 0, 0, 0);
          if (t < P.T && ((tm >> t) & 1u)) {
            const int pos = s.posof[a][t];
            const float w = s.wgp[pos];
            const float* pg = P.partA + (size_t)pos * P.KSA * rowA + U.ks * kGroup + kc * 8;
            float g[8], uu[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) { g[j] = 0.f; uu[j] = 0.f; }
            for (int ks = 0; ks < P.KSA; ++ks) {
              const float4 g0 = __ldcg(reinterpret_cast<const float4*>(pg + ks * rowA));
              const float4 g1 = __ldcg(reinterpret_cast<const float4*>(pg + ks * rowA + 4));
              const float4 u0 = __ldcg(reinterpret_cast<const float4*>(pg + ks * rowA + P.I));
              const float4 u1 = __ldcg(reinterpret_cast<const float4*>(pg + ks * rowA + P.I + 4));
              g[0] += g0.x; g[1] += g0.y; g[2] += g0.z; g[3] += g0.w;
              g[4] += g1.x; g[5] += g1.y; g[6] += g1.z; g[7] += g1.w;
              uu[0] += u0.x; uu[1] += u0.y; uu[2] += u0.z; uu[3] += u0.w;
              uu[4] += u1.x; uu[5] += u1.y; uu[6] += u1.z; uu[7] += u1.w;
            }
            uint32_t pk[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float h0 = g[2 * j] / (1.f + expf(-g[2 * j])) * uu[2 * j] * w;
              const float h1 = g[2 * j + 1] / (1.f + expf(-g[2 * j + 1])) * uu[2 * j + 1] * w;
              const __nv_bfloat162 b = __floats2bfloat162_rn(h0, h1);
              pk[j] = *reinterpret_cast<const uint32_t*>(&b);
            }
            o = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          *reinterpret_cast<uint4*>(dst + kmajor_off(t, kc * 8)) = o;
        }
        tc::fence_proxy_async_smem();
        tc::named_bar_sync(2, 64);
        if (btid == 0) tc::mbar_arrive(&s.bfull[bs]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int etid = tid - kEpiWarp0 * 32;      // 0..127
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    int i = 0;
    for (int u = blockIdx.x; u < U_total; u += G, ++i) {
      const Unit U = decode_unit(s, P, u);
      const int db = i & 1;
      if (!warp_wait(&s.dfull[db], (i >> 1) & 1, abort)) break;
      tc::tc_fence_after();
      const uint32_t dcol = kDColBase + db * 2 * kN;
      uint32_t g[kN], h[kN];
      tc::tmem_ld16(trow + dcol, g);
      if (U.type == 0) tc::tmem_ld16(trow + dcol + kN, h);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&s.dempty[db]);

      if (U.type == 0) {
        const uint32_t tm = s.tokmask[U.a];
#pragma unroll
        for (int t = 0; t < kN; ++t) {
          if ((tm >> t) & 1u) {
            const int pos = s.posof[U.a][t];
            float* pa = P.partA + ((size_t)pos * P.KSA + U.ks) * rowA + U.blk * kRowBlock + r;
            pa[0] = __uint_as_float(g[t]);
            pa[P.I] = __uint_as_float(h[t]);
          }
        }
        __threadfence();
        tc::named_bar_sync(1, 128);
        if (etid == 0) tc::red_release_add(P.cntA + U.e * IB + U.blk, 1);
      } else {
        const int np = GI * nEC;                    // partials per H-block
        float* pb = P.partB + ((size_t)U.blk * np + U.ks * nEC + U.ec) * P.T * kRowBlock;
#pragma unroll
        for (int t = 0; t < kN; ++t)
          if (t < P.T) pb[t * kRowBlock + r] = __uint_as_float(g[t]);
        __threadfence();
        tc::named_bar_sync(1, 128);
        if (etid == 0) s.last_flag = (atomicAdd(P.cntB + U.blk, 1) == np - 1);
        tc::named_bar_sync(1, 128);
        if (s.last_flag) {
          __threadfence();
          const int row = U.blk * kRowBlock + r;
          const float* base = P.partB + (size_t)U.blk * np * P.T * kRowBlock + r;
          for (int t = 0; t < P.T; ++t) {
            float v = P.accumulate ? __ldcg(P.acc + (size_t)t * P.H + row) : 0.f;
            for (int q = 0; q < np; ++q) v += __ldcg(base + ((size_t)q * P.T + t) * kRowBlock);
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
      if (etid == 0 && i < 32) trace_at(P, 8 + i);
    }
    if (etid == 0) trace_at(P, 4);
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc<kTmemCols>(tmem);
  }
  if (tid == 0) {
    trace_at(P, 5);
    __threadfence();
    s.last_flag = (atomicAdd(P.ctl + kCtlDone, 1) == (int)gridDim.x - 1);
  }
  __syncthreads();
  if (s.last_flag) {
    // last CTA out: every unit is finished; reset the cross-CTA counters for the next call
    __threadfence();
    for (int i = tid; i < P.E * IB; i += kThreads) P.cntA[i] = 0;
    if (tid == 0) P.ctl[kCtlDone] = 0;
    __threadfence();
  }
}

int g_num_sms = 0;
unsigned long long* g_trace = nullptr;

int num_sms() {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

size_t decode_smem_bytes(int H) { return sizeof(DecSmem) + (size_t)kN * H * 2; }

int groups_per_a_unit(int GH) {
  for (int d = std::min(GH, kGAMax); d >= 1; --d)
    if (GH % d == 0) return d;
  return 1;
}

}  // namespace

// Diagnostics: when set, the fused decode kernel records per-CTA timestamps (64 x u64 per CTA)
// into this device buffer; NULL turns it off.
MOE_API void moe_debug_set_decode_trace(void* dev_buffer) {
  g_trace = static_cast<unsigned long long*>(dev_buffer);
}

bool ffn_decode_supported(const FfnArgs& a) {
  return a.T >= 1 && a.T <= kMaxT && a.T * a.k <= kMaxTk && a.E <= kMaxExperts && a.H % kRowBlock == 0 &&
         a.I % kRowBlock == 0 && decode_smem_bytes(a.H) <= 227 * 1024;
}

size_t decode_scratch_bytes(int T, int H, int I, int E, int k) {
  if (T < 1 || T > kMaxT || T * k > kMaxTk) return 0;
  const int KSA = H / kGroup / groups_per_a_unit(H / kGroup), GI = I / kGroup;
  const size_t Tk = (size_t)T * k;
  const int nEC = (std::min(E, T * k) + kEC - 1) / kEC;
  size_t b = 0;
  b += align_up(sizeof(int) * (size_t)E * (I / kRowBlock), 256);     // cntA
  b += align_up(sizeof(int) * (size_t)(H / kRowBlock), 256);         // cntB
  b += align_up(sizeof(float) * Tk * KSA * 2 * I, 256);              // partA
  b += align_up(sizeof(float) * (size_t)(H / kRowBlock) * GI * nEC * T * kRowBlock, 256);   // partB
  return b;
}

int ffn_decode(const FfnArgs& a, cudaStream_t s) {
  const WsLayout L = ws_layout(a.T, a.H, a.I, a.E, a.k);
  const int GH = a.H / kGroup;
  DecParams P{};
  P.x = a.x; P.logits = a.logits; P.idx_in = a.idx; P.wts_in = a.wts;
  P.T = a.T; P.H = a.H; P.I = a.I; P.E = a.E; P.k = a.k;
  P.w13 = a.w13; P.s13 = a.s13; P.w2 = a.w2; P.s2 = a.s2; P.slot = a.slot;
  P.idx_out = a.idx_out; P.wts_out = a.wts_out;
  P.out = a.out; P.acc = reinterpret_cast<float*>(a.ws + L.acc); P.accumulate = a.accumulate ? 1 : 0;
  P.gA = groups_per_a_unit(GH);
  P.KSA = GH / P.gA;
  char* d = a.ws + L.dec;
  P.ctl = reinterpret_cast<int*>(a.ws + L.status);
  P.cntA = reinterpret_cast<int*>(d);
  d += align_up(sizeof(int) * (size_t)a.E * (a.I / kRowBlock), 256);
  P.cntB = reinterpret_cast<int*>(d);
  d += align_up(sizeof(int) * (size_t)(a.H / kRowBlock), 256);
  P.partA = reinterpret_cast<float*>(d);
  d += align_up(sizeof(float) * (size_t)a.T * a.k * P.KSA * 2 * a.I, 256);
  P.partB = reinterpret_cast<float*>(d);
  P.trace = g_trace;
  if (!a.logits && (!a.idx || !a.wts)) return fail(MOE_ERR_ARG, "fused decode: routing missing");

  const int max_act = std::min(a.E, a.T * a.k);
  const int max_units = max_act * ((a.I / kRowBlock) * P.KSA) +
                        (a.H / kRowBlock) * (a.I / kGroup) * ((max_act + kEC - 1) / kEC);
  const int grid = std::max(1, std::min(num_sms(), max_units));
  const size_t smem = decode_smem_bytes(a.H);
  static bool attr_done = false;
  if (!attr_done) {
    if (int rc = check_cuda(cudaFuncSetAttribute(moe_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 227 * 1024), "fused decode: smem attribute"))
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
