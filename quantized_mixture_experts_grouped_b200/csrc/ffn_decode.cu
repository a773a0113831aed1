// Fused decode path of the W4A16 MoE layer: routing, gate/up with SiLU*up, down projection and
// the router-weighted combine in ONE persistent launch ("Every Expert Counts: ExactMoE for
// Memory-Efficient W4A16 Inference", Abstract: all selected experts execute through fused
// grouped MoE kernels; the router's top-k is unchanged).
//
// A decode batch (T <= 16 tokens) reads every selected expert's packed weights exactly once, so
// the layer is bound by HBM bandwidth on those bytes plus the latency of every dependent step.
// The kernel is shaped to keep that chain short:
//  * every CTA routes the batch itself (warp top-k; the renormalised weights are a softmax over
//    the k chosen logits, which equals the full softmax renormalised) and builds the grouping
//    with a presence bitmap and shared-memory atomics (constant depth); the batch's activations
//    are staged once in shared memory as the B operand of every gate/up MMA (all T tokens are
//    MMA columns; a column whose token is not routed to the expert is computed and ignored);
//  * a unit is (routed expert, 64 intermediate features); CTA c takes units c, c+G, c+2G, ...
//    A unit needs no other CTA: gate and up rows of its 64 features form one 128-row MMA over
//    all of H, the CTA turns the accumulators into h = w * silu(g) * u itself (gate and up
//    rows meet through shared memory), and multiplies h by the matching 64-wide column slice
//    of W2 for every row of H. All units of a CTA accumulate into one tensor-memory
//    accumulator, so the router-weighted sum over experts happens inside the MMA;
//  * warp 0 streams the unit's int4 weights + bf16 scales into an 8-stage shared-memory ring
//    with bulk async copies (TMA, evict-first in L2);
//  * warps 6..13 dequantise in two groups that take alternate stages: a thread owns one weight
//    row and writes bf16 (q * s, one rounding) straight into TENSOR MEMORY (tcgen05.st) as the
//    A operand of tcgen05.mma - the bf16 weights never pass through shared memory;
//  * one thread of warp 1 issues tcgen05.mma (M = 128 weight rows, N = 16 tokens, K = 16);
//  * warps 2..5 run the epilogues: h for each unit, then the CTA's partial output;
//  * a grid-wide barrier (sense-reversing, bounded) separates the units from the final
//    reduction, where every CTA sums one slice of the per-CTA partials in a fixed order and
//    writes bf16 outputs. Results are deterministic run to run.
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

constexpr int kStages = 8;
constexpr int kABufs = 3;
constexpr int kMaxTk = 256;
constexpr int kMaxT = 16;
constexpr int kN = 16;                    // MMA N: the batch's tokens (<= 16)
constexpr int kIF = 64;                   // intermediate features per unit
constexpr int kMaxHB = 16;                // H <= 2048: one accumulator column block per 128 rows
constexpr int kMaxGrid = 160;
constexpr int kThreads = 448;             // 14 warps
constexpr int kWarps = kThreads / 32;
constexpr int kEpiWarp0 = 2;              // warps 2..5
constexpr int kDqWarp0 = 6;               // warps 6..13: two groups of four
constexpr int kTmemCols = 512;
constexpr int kAColBase = 0;              // 3 A buffers x 64 columns
constexpr int kDguCol = 192;              // gate/up accumulators: 2 x kN columns
constexpr int kDhCol = 256;               // partial output: kMaxHB x kN columns
constexpr unsigned kFull = 0xffffffffu;
constexpr int kCtlBarCount = kCtlDecode;      // grid barrier arrivals
constexpr int kCtlBarGen = kCtlDecode + 1;    // grid barrier generation

enum { kSiteStage = 2, kSiteABuf = 3, kSiteB = 4, kSiteD = 5, kSiteGrid = 6, kSiteDrain = 7, kSiteOver = 8 };

struct DecParams {
  const uint16_t* x; const uint16_t* logits; const int32_t* idx_in; const float* wts_in;
  int T, H, I, E, k;
  const uint8_t* w13; const uint16_t* s13; const uint8_t* w2; const uint16_t* s2;
  const int32_t* slot;
  int32_t* idx_out; float* wts_out;
  uint16_t* out; float* acc; int accumulate;
  int* ctl;
  float* ypart;                 // [gridDim][T][H] per-CTA partial outputs
  unsigned long long* trace;    // optional per-CTA timestamps (diagnostics), null in normal use
};

// trace slots per CTA (64 x u64, %globaltimer): 0 start, 1 plan done, 2 first copy issued,
// 3 producer done, 4 epilogue done, 5 grid barrier passed, 6 end
__device__ __forceinline__ void trace_at(const DecParams& P, int slot) {
  if (P.trace) P.trace[blockIdx.x * 64 + slot] = tc::globaltimer();
}

struct __align__(128) DecSmem {
  uint8_t stage[kStages][8192];
  uint16_t scale[kStages][128];
  uint8_t bdown[2][kN * kIF * 2];           // h of a unit: B operand of the down MMA (2 KB each)
  float gx[kIF][kN];                        // gate accumulators handed to the up-row warps
  float red[kThreads];                      // final-reduction scratch
  int idx[kMaxTk];
  float wts[kMaxTk];
  uint32_t present[kMaxExperts / 32];
  int act[kMaxExperts];
  int aidx[kMaxExperts];
  uint32_t tokmask[kMaxExperts];
  float wtok[kMaxExperts][kMaxT];           // router weight of (active expert, token), 0 if not routed
  uint64_t full[kStages], empty[kStages];
  uint64_t afull[kABufs], aempty[kABufs];
  uint64_t gfull[2], gempty[2];             // gate/up accumulators
  uint64_t bfull[2], bempty[2];             // h operand
  uint64_t hfull, drain;
  uint32_t tmem_base;
  int nact;
  int abort;
  int over;
  // followed in dynamic shared memory by the activations: kN rows x H, no-swizzle K-major
};

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

// Element (n, k) of a kN-row, K-major operand without swizzle: 8x16-byte core matrices.
__device__ __forceinline__ uint32_t kmajor_off(int n, int k) {
  return (uint32_t)(((k >> 3) * (kN / 8) + (n >> 3)) * 128 + (n & 7) * 16 + (k & 7) * 2);
}

// Routes token t with one warp (same selection rule as route_kernel): writes s.idx / s.wts and
// marks the chosen experts in the presence bitmap. The chosen logits are decoded back from the
// winning keys; the renormalised weight of choice j is exp(l_j - l_max) / sum over the k chosen.
__device__ void route_token(DecSmem& s, const DecParams& P, int t, int lane) {
  const int E = P.E, k = P.k;
  const uint16_t* lt = P.logits + (size_t)t * E;
  constexpr int kPer = kMaxExperts / 32;
  uint32_t key[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? route_key_d(lt[e], e) : 0u;
  }
  float mx = 0.f, el[kPer];    // lane (j % 32) keeps exp(l_j - l_max) of choice j in el[j / 32]
#pragma unroll
  for (int i = 0; i < kPer; ++i) el[i] = 0.f;
  for (int j = 0; j < k; ++j) {
    uint32_t best = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) best = max(best, key[i]);
    const uint32_t win = __reduce_max_sync(kFull, best);
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (key[i] == win) key[i] = 0;                  // keys are unique (the id is in them)
    const int e = 0xffff - (int)(win & 0xffffu);
    const uint32_t ord = win >> 16;
    const float lw = bf16_bits_to_float((ord & 0x8000u) ? (ord & 0x7fffu) : (~ord & 0xffffu));
    if (j == 0) mx = lw;
    if ((j & 31) == lane) {
      s.idx[t * k + j] = e;
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if ((j >> 5) == i) el[i] = expf(lw - mx);
      if (slot_of(P.slot, e) >= 0) atomicOr(&s.present[e >> 5], 1u << (e & 31));
    }
  }
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) sum += el[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int j = 32 * i + lane;
    if (j < k) s.wts[t * k + j] = el[i] / sum;
  }
}

// Routing (or the given routing), activations into shared memory, active-expert list, and per
// (active expert, token) router weights. Four CTA barriers, each phase of constant depth.
__device__ void build_plan(DecSmem& s, const DecParams& P, uint8_t* xs) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Tk = P.T * P.k, E = P.E;
  const int rowc = P.H / 8;                       // 16-byte chunks per activation row
  const int chunks = P.T * rowc;
  // activations: issue the loads first so that their latency overlaps the routing
  constexpr int kPerThr = (kN * 2048 / 8 + kThreads - 1) / kThreads;
  uint4 xv[kPerThr];
#pragma unroll
  for (int i = 0; i < kPerThr; ++i) {
    const int c = tid + i * kThreads;
    if (c < chunks) xv[i] = __ldg(reinterpret_cast<const uint4*>(P.x + (size_t)(c / rowc) * P.H) + c % rowc);
  }
  if (P.logits) {
    for (int t = warp; t < P.T; t += kWarps) route_token(s, P, t, lane);
  } else {
    for (int p = tid; p < Tk; p += kThreads) {
      const int e = P.idx_in[p];
      s.idx[p] = e;
      s.wts[p] = P.wts_in[p];
      if ((unsigned)e < (unsigned)E && slot_of(P.slot, e) >= 0) atomicOr(&s.present[e >> 5], 1u << (e & 31));
    }
  }
#pragma unroll
  for (int i = 0; i < kPerThr; ++i) {
    const int c = tid + i * kThreads;
    if (c < chunks) *reinterpret_cast<uint4*>(xs + kmajor_off(c / rowc, (c % rowc) * 8)) = xv[i];
  }
  for (int c = tid + kPerThr * kThreads; c < chunks; c += kThreads)
    *reinterpret_cast<uint4*>(xs + kmajor_off(c / rowc, (c % rowc) * 8)) =
        __ldg(reinterpret_cast<const uint4*>(P.x + (size_t)(c / rowc) * P.H) + c % rowc);
  __syncthreads();
  // active experts in ascending id: rank = set bits below in the presence bitmap
  if (tid < E) {
    const int w = tid >> 5;
    if ((s.present[w] >> (tid & 31)) & 1u) {
      int a = __popc(s.present[w] & ((1u << (tid & 31)) - 1u));
      for (int i = 0; i < w; ++i) a += __popc(s.present[i]);
      s.act[a] = tid;
      s.aidx[tid] = a;
    }
  }
  if (P.logits && P.idx_out && blockIdx.x == 0)
    for (int p = tid; p < Tk; p += kThreads) {
      P.idx_out[p] = s.idx[p];
      P.wts_out[p] = s.wts[p];
    }
  __syncthreads();
  for (int p = tid; p < Tk; p += kThreads) {
    const int e = s.idx[p];
    if ((unsigned)e >= (unsigned)E || !((s.present[e >> 5] >> (e & 31)) & 1u)) continue;
    const int a = s.aidx[e], t = p / P.k;
    const uint32_t old = atomicOr(&s.tokmask[a], 1u << t);
    if ((old >> t) & 1u) s.over = 1;             // a token routed twice to one expert
    s.wtok[a][t] = s.wts[p];
  }
  __syncthreads();
  if (tid == 0) {
    int n = 0;
    for (int i = 0; i < (E + 31) / 32; ++i) n += __popc(s.present[i]);
    s.nact = s.over ? 0 : n;
    if (s.over) report_status(P.ctl, MOE_ERR_ARG, kSiteOver);
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 1) moe_decode_kernel(const __grid_constant__ DecParams P) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  DecSmem& s = *reinterpret_cast<DecSmem*>(smem_raw);
  uint8_t* xs = smem_raw + sizeof(DecSmem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- set-up that does not read the previous kernel's results: overlaps it under PDL
  if (warp == 2) {
    if (lane < kStages) { tc::mbar_init(&s.full[lane], 1); tc::mbar_init(&s.empty[lane], 4); }
    if (lane < kABufs) { tc::mbar_init(&s.afull[lane], 4); tc::mbar_init(&s.aempty[lane], 1); }
    if (lane < 2) {
      tc::mbar_init(&s.gfull[lane], 1); tc::mbar_init(&s.gempty[lane], 4);
      tc::mbar_init(&s.bfull[lane], 1); tc::mbar_init(&s.bempty[lane], 1);
    }
    if (lane == 0) {
      tc::mbar_init(&s.hfull, 1);
      tc::mbar_init(&s.drain, 1);
      s.abort = 0;
      s.over = 0;
    }
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc<kTmemCols>(&s.tmem_base);
    tc::tc_fence_before();
  }
  for (int i = tid; i < kMaxExperts / 32; i += kThreads) s.present[i] = 0;
  for (int i = tid; i < kMaxExperts; i += kThreads) s.tokmask[i] = 0;
  for (int i = tid; i < kMaxExperts * kMaxT; i += kThreads) (&s.wtok[0][0])[i] = 0.f;
  for (int i = tid; i < (int)(sizeof(s.bdown) / 16); i += kThreads)
    reinterpret_cast<uint4*>(&s.bdown[0][0])[i] = make_uint4(0, 0, 0, 0);
  for (int i = tid + P.T * (P.H / 8); i < kN * (P.H / 8); i += kThreads)   // token rows >= T stay zero
    *reinterpret_cast<uint4*>(xs + kmajor_off(i / (P.H / 8), (i % (P.H / 8)) * 8)) = make_uint4(0, 0, 0, 0);
  __syncthreads();

  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) trace_at(P, 0);
  build_plan(s, P, xs);
  tc::tc_fence_after();
  tc::fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) trace_at(P, 1);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const uint32_t tmem = s.tmem_base;
  const int IB = P.I / kRowBlock, GH = P.H / kGroup, GI = P.I / kGroup, HB = P.H / kRowBlock;
  const int NF = P.I / kIF;                                   // units per expert
  const int U_total = s.nact * NF;
  const int G = gridDim.x;
  const int my_units = ((int)blockIdx.x < U_total) ? (U_total - 1 - (int)blockIdx.x) / G + 1 : 0;
  volatile int* abort = &s.abort;
  const size_t w13_bytes = (size_t)P.I * P.H, s13_count = (size_t)2 * P.I * GH;
  const size_t w2_bytes = (size_t)P.H * P.I / 2, s2_count = (size_t)P.H * GI;
  const int stages_per_unit = GH + HB;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol = tc::policy_evict_first();
    int it = 0;
    bool ok = true;
    for (int n = 0; n < my_units && ok; ++n) {
      const int u = blockIdx.x + n * G;
      const int e = s.act[u / NF], sl = slot_of(P.slot, e);
      const int i0 = (u % NF) * kIF, rb = i0 / kRowBlock, r0 = i0 % kRowBlock;
      const uint8_t* w13e = P.w13 + (size_t)sl * w13_bytes;
      const uint16_t* s13e = P.s13 + (size_t)sl * s13_count;
      const uint8_t* w2e = P.w2 + (size_t)sl * w2_bytes;
      const uint16_t* s2e = P.s2 + (size_t)sl * s2_count;
      for (int ti = 0; ti < stages_per_unit; ++ti, ++it) {
        const int st = it % kStages;
        if (!warp_wait(&s.empty[st], ((it / kStages) & 1) ^ 1, abort)) { ok = false; break; }
        if (lane == 0) {
          if (it == 0) trace_at(P, 2);
          if (ti < GH) {
            // rows 0..63: gate rows i0.., rows 64..127: the matching up rows, K group ti
            const size_t tg = (size_t)rb * GH + ti, tu = (size_t)(IB + rb) * GH + ti;
            tc::mbar_arrive_expect_tx(&s.full[st], 8192 + 256);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq) {
              tc::bulk_g2s(s.stage[st] + kq * 2048, w13e + tg * kTileBytes + kq * 2048 + r0 * 16, 1024, &s.full[st], pol);
              tc::bulk_g2s(s.stage[st] + kq * 2048 + 1024, w13e + tu * kTileBytes + kq * 2048 + r0 * 16, 1024,
                           &s.full[st], pol);
            }
            tc::bulk_g2s(&s.scale[st][0], s13e + tg * kRowBlock + r0, 128, &s.full[st], pol);
            tc::bulk_g2s(&s.scale[st][64], s13e + tu * kRowBlock + r0, 128, &s.full[st], pol);
          } else {
            // W2 rows of H-block hb, the unit's 64-wide K half of I-group rb
            const size_t t2 = (size_t)(ti - GH) * GI + rb;
            tc::mbar_arrive_expect_tx(&s.full[st], 4096 + 256);
            tc::bulk_g2s(s.stage[st], w2e + t2 * kTileBytes + (r0 / kIF) * 4096, 4096, &s.full[st], pol);
            tc::bulk_g2s(&s.scale[st][0], s2e + t2 * kRowBlock, 256, &s.full[st], pol);
          }
        }
      }
    }
    if (!ok && lane == 0) report_abort(s, P, kSiteStage);
    if (lane == 0) trace_at(P, 3);
    if (lane == 0) {   // no bulk copy may still be landing in shared memory when the CTA leaves
      const int nw = it < kStages ? it : kStages;
      for (int i = 0; i < nw; ++i) {
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
      int a_it = 0;
      bool ok = true;
      for (int n = 0; n < my_units && ok; ++n) {
        const int db = n & 1;
        if (!tc::mbar_wait(&s.gempty[db], ((n >> 1) & 1) ^ 1, abort)) { ok = false; report_abort(s, P, kSiteD); break; }
        tc::tc_fence_after();
        for (int g = 0; g < GH && ok; ++g, ++a_it) {
          const int ab = a_it % kABufs;
          if (!tc::mbar_wait(&s.afull[ab], (a_it / kABufs) & 1, abort)) { ok = false; report_abort(s, P, kSiteABuf); break; }
          tc::tc_fence_after();
          const uint32_t a = tmem + kAColBase + ab * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t bdesc = tc::smem_desc(xbase + ((g * kGroup + kk * 16) / 8) * lbo, lbo, 128, 0);
            tc::mma_ts(tmem + kDguCol + db * kN, a + kk * 8, bdesc, idesc, (g > 0 || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(&s.aempty[ab]);
        }
        if (!ok) break;
        tc::mma_commit(&s.gfull[db]);
        const int bb = n & 1;
        if (!tc::mbar_wait(&s.bfull[bb], (n >> 1) & 1, abort)) { ok = false; report_abort(s, P, kSiteB); break; }
        tc::tc_fence_after();
        const uint32_t hbase = tc::smem_u32(s.bdown[bb]);
        for (int hb = 0; hb < HB && ok; ++hb, ++a_it) {
          const int ab = a_it % kABufs;
          if (!tc::mbar_wait(&s.afull[ab], (a_it / kABufs) & 1, abort)) { ok = false; report_abort(s, P, kSiteABuf); break; }
          tc::tc_fence_after();
          const uint32_t a = tmem + kAColBase + ab * 64;
#pragma unroll
          for (int kk = 0; kk < kIF / 16; ++kk) {
            const uint64_t bdesc = tc::smem_desc(hbase + kk * 2 * lbo, lbo, 128, 0);
            tc::mma_ts(tmem + kDhCol + hb * kN, a + kk * 8, bdesc, idesc, (n > 0 || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(&s.aempty[ab]);
        }
        tc::mma_commit(&s.bempty[bb]);
      }
      if (ok && my_units > 0) tc::mma_commit(&s.hfull);
      tc::mma_commit(&s.drain);
      volatile int never = 0;
      if (!tc::mbar_wait(&s.drain, 0, &never)) report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteDrain);
    }
    __syncwarp();
  } else if (warp >= kDqWarp0) {
    // ------------------------------------------------------------ dequantisers -> TMEM
    // two groups of four warps take alternate stages; a thread owns row r of the stage
    const int quarter = warp & 3, grp = (warp - kDqWarp0) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t taddr_row = tmem + ((uint32_t)(quarter * 32) << 16) + kAColBase;
    const __nv_bfloat162 off136 = __floats2bfloat162_rn(136.f, 136.f);
    int it = 0;
    bool ok = true;
    for (int n = 0; n < my_units && ok; ++n) {
      for (int ti = 0; ti < stages_per_unit; ++ti, ++it) {
        if ((it & 1) != grp) continue;
        const int st = it % kStages;
        const int halves = (ti < GH) ? 2 : 1;       // 128 K (gate/up) or 64 K (down) per row
        if (!warp_wait(&s.full[st], (it / kStages) & 1, abort)) { ok = false; break; }
        uint4 c[4];
#pragma unroll
        for (int kq = 0; kq < 4; ++kq)
          c[kq] = (kq < 2 * halves) ? *reinterpret_cast<const uint4*>(s.stage[st] + kq * 2048 + r * 16)
                                    : make_uint4(0, 0, 0, 0);
        const uint32_t sb = s.scale[st][r];
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.empty[st]);
        const uint32_t s2u = sb | (sb << 16);
        const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&s2u);
        const int ab = it % kABufs;
        if (!warp_wait(&s.aempty[ab], ((it / kABufs) & 1) ^ 1, abort)) { ok = false; break; }
        tc::tc_fence_after();
        dequant_half(c[0], c[1], s2, off136, taddr_row + ab * 64);
        if (halves == 2) dequant_half(c[2], c[3], s2, off136, taddr_row + ab * 64 + 32);
        tc::tmem_wait_st();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.afull[ab]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogues (warps 2..5)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;          // rows 0..63: gate of feature r, 64..127: up of r-64
    const int etid = tid - kEpiWarp0 * 32;      // 0..127 (warp 2 holds rows 64..95)
    const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);
    // Every exit decision is taken after the second named barrier from the CTA's abort flag,
    // so the four warps always meet at the same barriers (a failed wait raises the flag).
    for (int n = 0; n < my_units; ++n) {
      const int u = blockIdx.x + n * G;
      const int a = u / NF;
      const int db = n & 1;
      const bool g_ok = warp_wait(&s.gfull[db], (n >> 1) & 1, abort);
      uint32_t v[kN];
#pragma unroll
      for (int t = 0; t < kN; ++t) v[t] = 0;
      if (g_ok) {
        tc::tc_fence_after();
        tc::tmem_ld16(trow + kDguCol + db * kN, v);
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s.gempty[db]);
        if (r < kIF) {
#pragma unroll
          for (int t = 0; t < kN; ++t) s.gx[r][t] = __uint_as_float(v[t]);
        }
      }
      tc::named_bar_sync(1, 128);
      if (r >= kIF && g_ok && !*abort) {
        const int bb = n & 1;
        if (warp_wait(&s.bempty[bb], ((n >> 1) & 1) ^ 1, abort)) {
          const int f = r - kIF;
          const uint32_t tm = s.tokmask[a];
          uint8_t* dst = s.bdown[bb];
#pragma unroll
          for (int t = 0; t < kN; ++t) {
            float hv = 0.f;
            if ((tm >> t) & 1u) {
              const float g = s.gx[f][t];
              hv = g / (1.f + expf(-g)) * __uint_as_float(v[t]) * s.wtok[a][t];
            }
            *reinterpret_cast<__nv_bfloat16*>(dst + kmajor_off(t, f)) = __float2bfloat16_rn(hv);
          }
          tc::fence_proxy_async_smem();
        }
      }
      tc::named_bar_sync(1, 128);
      if (*abort) break;
      if (etid == 0) tc::mbar_arrive(&s.bfull[n & 1]);
    }
    const bool ok = !*abort;
    // the CTA's partial output: rows hb*128 + r, all tokens
    float* yp = P.ypart + (size_t)blockIdx.x * P.T * P.H;
    if (my_units > 0 && ok && warp_wait(&s.hfull, 0, abort)) {
      tc::tc_fence_after();
      for (int hb = 0; hb < HB; ++hb) {
        uint32_t y[kN];
        tc::tmem_ld16(trow + kDhCol + hb * kN, y);
        tc::tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < kN; ++t)
          if (t < P.T) yp[(size_t)t * P.H + hb * kRowBlock + r] = __uint_as_float(y[t]);
      }
    } else {
      for (int i = etid; i < P.T * P.H; i += 128) yp[i] = 0.f;
    }
    if (etid == 0) trace_at(P, 4);
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc<kTmemCols>(tmem);
  }

  // ---- grid-wide barrier (every CTA is resident: one CTA per SM, grid <= SM count)
  if (tid == 0) {
    const int gen = tc::ld_acquire(P.ctl + kCtlBarGen);
    __threadfence();
    if (atomicAdd(P.ctl + kCtlBarCount, 1) == G - 1) {
      P.ctl[kCtlBarCount] = 0;
      tc::red_release_add(P.ctl + kCtlBarGen, 1);
    } else {
      const long long t0 = clock64();
      while (tc::ld_acquire(P.ctl + kCtlBarGen) == gen) {
        if (clock64() - t0 > tc::kWaitTimeoutCycles) {
          report_status(P.ctl, MOE_ERR_TIMEOUT, kSiteGrid);
          break;
        }
        __nanosleep(64);
      }
    }
    trace_at(P, 5);
  }
  __syncthreads();

  // ---- final reduction: this CTA's slice of the T x H outputs, partials summed in CTA order
  const int total = P.T * P.H;
  const int per = (total + G - 1) / G;
  const int e0 = (int)blockIdx.x * per;
  const int cnt = max(0, min(per, total - e0));
  if (cnt > 0) {
    const int stripes = max(1, min(G, kThreads / cnt));
    const int el = tid % cnt, sp = tid / cnt;
    float v = 0.f;
    if (sp < stripes && tid < stripes * cnt)
      for (int c = sp; c < G; c += stripes) v += __ldcg(P.ypart + (size_t)c * total + e0 + el);
    s.red[tid] = v;
    __syncthreads();
    for (int i = tid; i < cnt; i += kThreads) {
      float accv = P.accumulate ? __ldcg(P.acc + e0 + i) : 0.f;
      for (int q = 0; q < stripes; ++q) accv += s.red[q * cnt + i];
      if (P.out) {
        P.out[e0 + i] = __bfloat16_as_ushort(__float2bfloat16_rn(accv));
        if (P.accumulate) P.acc[e0 + i] = 0.f;
      } else {
        P.acc[e0 + i] = accv;
      }
    }
  }
  if (tid == 0) trace_at(P, 6);
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

}  // namespace

// Diagnostics: when set, the fused decode kernel records per-CTA timestamps (64 x u64 per CTA)
// into this device buffer; NULL turns it off.
MOE_API void moe_debug_set_decode_trace(void* dev_buffer) {
  g_trace = static_cast<unsigned long long*>(dev_buffer);
}

bool ffn_decode_supported(const FfnArgs& a) {
  return a.T >= 1 && a.T <= kMaxT && a.T * a.k <= kMaxTk && a.E <= kMaxExperts && a.H % kRowBlock == 0 &&
         a.I % kRowBlock == 0 && a.H / kRowBlock <= kMaxHB && decode_smem_bytes(a.H) <= 227 * 1024;
}

size_t decode_scratch_bytes(int T, int H, int I, int E, int k) {
  (void)I; (void)E; (void)k;
  if (T < 1 || T > kMaxT) return 0;
  return align_up(sizeof(float) * (size_t)kMaxGrid * T * H, 256);     // per-CTA partial outputs
}

int ffn_decode(const FfnArgs& a, cudaStream_t s) {
  const WsLayout L = ws_layout(a.T, a.H, a.I, a.E, a.k);
  DecParams P{};
  P.x = a.x; P.logits = a.logits; P.idx_in = a.idx; P.wts_in = a.wts;
  P.T = a.T; P.H = a.H; P.I = a.I; P.E = a.E; P.k = a.k;
  P.w13 = a.w13; P.s13 = a.s13; P.w2 = a.w2; P.s2 = a.s2; P.slot = a.slot;
  P.idx_out = a.idx_out; P.wts_out = a.wts_out;
  P.out = a.out; P.acc = reinterpret_cast<float*>(a.ws + L.acc); P.accumulate = a.accumulate ? 1 : 0;
  P.ctl = reinterpret_cast<int*>(a.ws + L.status);
  P.ypart = reinterpret_cast<float*>(a.ws + L.dec);
  P.trace = g_trace;
  if (!a.logits && (!a.idx || !a.wts)) return fail(MOE_ERR_ARG, "fused decode: routing missing");

  const int max_units = std::min(a.E, a.T * a.k) * (a.I / kIF);
  const int grid = std::max(1, std::min(std::min(num_sms(), kMaxGrid), max_units));
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
